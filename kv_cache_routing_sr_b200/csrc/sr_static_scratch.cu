// sr_decode_attention_static_scratch: the decode step for callers that must not
// allocate device memory. The decode kernel's scratch (device error word, per-
// unit arrival counters, split partials) lives in a fixed array compiled into
// this library instead of a caller-provided workspace. Nothing here allocates:
// no cudaMalloc / cudaFree, no library allocator.
#include <cuda_runtime.h>

#include "sinkrouter.h"
#include "sr_internal.h"

namespace {

// One array per GPU that loads the library, kept until the process exits.
// In host code this name is only a stand-in for the symbol: its device address
// comes from cudaGetSymbolAddress (below, with the caller's device current).
static __device__ __align__(256) unsigned char g_static_scratch[SR_STATIC_SCRATCH_BYTES];

// Device address of g_static_scratch on the current device, looked up on
// every call (cheap once the module is loaded on that device), so that no
// address outlives a device reset. The first call on a device may load the
// module there.
cudaError_t scratch_address(void **addr)
{
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess)
        return e;
    if (!p)
        return cudaErrorInvalidSymbol;
    *addr = p;
    return cudaSuccess;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

} // namespace

extern "C" sr_status sr_decode_attention_static_scratch(const sr_dims *dims, const void *q, const void *k_cache,
                                                        const void *v_cache, const void *k0, const void *v0,
                                                        const int32_t *seq_lens, const int32_t *active_list,
                                                        int32_t n_splits, void *out, int32_t *device_error,
                                                        void *stream)
{
    (void)k0;
    if (!dims)
        return SR_ERR_INVALID_ARG;
    if (dims->batch < 1 || dims->n_kv_heads < 1 || dims->n_q_heads < 1 || dims->head_dim < 1 ||
        dims->max_seq_len < 1 || dims->n_q_heads % dims->n_kv_heads != 0)
        return SR_ERR_INVALID_ARG;
    const int M = dims->n_q_heads / dims->n_kv_heads;
    if (dims->head_dim != sr::kHeadDim || (M != 1 && M != 2 && M != 4 && M != 8) ||
        (int64_t)dims->batch * dims->n_kv_heads > SR_MAX_UNITS)
        return SR_ERR_UNSUPPORTED;
    if (!q || !k_cache || !v_cache || !v0 || !seq_lens || !active_list || !out)
        return SR_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(v0, 16) ||
        !aligned(out, 16) || !aligned(seq_lens, 4) || !aligned(active_list, 4) ||
        (device_error && !aligned(device_error, 4)))
        return SR_ERR_INVALID_ARG;
    if (n_splits < 0 || n_splits > SR_MAX_SPLITS)
        return SR_ERR_INVALID_ARG;
    const int U = dims->batch * dims->n_kv_heads;
    const sr::WorkspaceLayout ws = sr::workspace_layout(U, M, sr::slots_needed(U, n_splits));
    if (ws.total > (size_t)SR_STATIC_SCRATCH_BYTES)
        return SR_ERR_WORKSPACE; // these dims need more scratch than the static array holds

    void *scratch = nullptr;
    cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess)
        return sr::record_cuda_failure(e);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // The array keeps the previous call's contents: the error word and the
    // arrival counters must start at zero, the partials need no clearing.
    e = cudaMemsetAsync(scratch, 0, ws.part_o_off, st);
    if (e != cudaSuccess)
        return sr::record_cuda_failure(e);
    sr::DecodeArgs a{q,   k_cache, v_cache,     v0,          seq_lens,         active_list,
                     out, scratch, ws,          dims->batch, dims->n_q_heads, dims->n_kv_heads,
                     dims->max_seq_len, n_splits};
    e = sr::launch_decode(a, st);
    if (e != cudaSuccess)
        return sr::record_cuda_failure(e);
    if (device_error) {
        e = cudaMemcpyAsync(device_error, static_cast<unsigned char *>(scratch) + ws.err_off, sizeof(int32_t),
                            cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess)
            return sr::record_cuda_failure(e);
    }
    return SR_OK;
}
