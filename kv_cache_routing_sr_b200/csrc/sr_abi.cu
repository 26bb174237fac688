// extern "C" entry points of libsinkrouter.so (declared in include/sinkrouter.h):
// host-side validation, workspace layout and kernel dispatch. No function here
// allocates device memory; every buffer is the caller's.
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>
#include <string>

#include "sinkrouter.h"
#include "sr_internal.h"

namespace {

thread_local std::string g_last_cuda_error;

sr_status cuda_fail(cudaError_t e)
{
    g_last_cuda_error = std::string(cudaGetErrorName(e)) + ": " + cudaGetErrorString(e);
    return SR_ERR_CUDA;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Shape checks shared by both calls.
sr_status check_dims(const sr_dims *d)
{
    if (!d)
        return SR_ERR_INVALID_ARG;
    if (d->batch < 1 || d->n_kv_heads < 1 || d->n_q_heads < 1 || d->head_dim < 1 || d->max_seq_len < 1)
        return SR_ERR_INVALID_ARG;
    if (d->n_q_heads % d->n_kv_heads != 0)
        return SR_ERR_INVALID_ARG;
    if (d->head_dim != sr::kHeadDim)
        return SR_ERR_UNSUPPORTED;
    const int M = d->n_q_heads / d->n_kv_heads;
    if (M != 1 && M != 2 && M != 4 && M != 8)
        return SR_ERR_UNSUPPORTED;
    if ((int64_t)d->batch * d->n_kv_heads > SR_MAX_UNITS)
        return SR_ERR_UNSUPPORTED;
    return SR_OK;
}

cudaStream_t as_stream(void *s) { return static_cast<cudaStream_t>(s); }

} // namespace

sr_status sr::record_cuda_failure(cudaError_t e) { return cuda_fail(e); }

extern "C" {

const char *sr_status_string(sr_status s)
{
    switch (s) {
    case SR_OK:
        return "SR_OK";
    case SR_ERR_INVALID_ARG:
        return "SR_ERR_INVALID_ARG: null/misaligned pointer or invalid size";
    case SR_ERR_UNSUPPORTED:
        return "SR_ERR_UNSUPPORTED: head_dim must be 128, group size 1/2/4/8, batch*kv_heads <= SR_MAX_UNITS";
    case SR_ERR_WORKSPACE:
        return "SR_ERR_WORKSPACE: workspace null, misaligned or too small";
    case SR_ERR_CUDA:
        return "SR_ERR_CUDA: a CUDA call failed (see sr_last_cuda_error)";
    }
    return "unknown sr_status";
}

const char *sr_last_cuda_error(void) { return g_last_cuda_error.c_str(); }

sr_status sr_route(const sr_dims *dims, const void *q, const void *k0, float tau, uint8_t *route_mask,
                   int32_t *active_list, void *stream)
{
    const sr_status st = check_dims(dims);
    if (st != SR_OK)
        return st;
    if (!q || !k0 || !route_mask || !active_list || !aligned(q, 16) || !aligned(k0, 16) || !aligned(active_list, 4))
        return SR_ERR_INVALID_ARG;
    if (std::isnan(tau))
        return SR_ERR_INVALID_ARG;
    sr::RouteArgs a{q, k0, tau, route_mask, active_list, dims->batch, dims->n_q_heads, dims->n_kv_heads};
    const cudaError_t e = sr::launch_route(a, as_stream(stream));
    return e == cudaSuccess ? SR_OK : cuda_fail(e);
}

sr_status sr_rope_append_route(const sr_dims *dims, const void *q_in, const void *k_new, const void *v_new,
                               const float *rope_cos, const float *rope_sin, int32_t max_pos, int32_t *seq_lens,
                               void *k_cache, void *v_cache, void *k0, void *v0, float tau, void *q_out,
                               uint8_t *route_mask, int32_t *active_list, int32_t *device_error, void *stream)
{
    const sr_status st = check_dims(dims);
    if (st != SR_OK)
        return st;
    const void *rows[] = {q_in, k_new, v_new, rope_cos, rope_sin, k_cache, v_cache, k0, v0, q_out};
    for (const void *r : rows)
        if (!r || !aligned(r, 16))
            return SR_ERR_INVALID_ARG;
    if (!seq_lens || !aligned(seq_lens, 4) || !route_mask || !active_list || !aligned(active_list, 4))
        return SR_ERR_INVALID_ARG;
    if (device_error && !aligned(device_error, 4))
        return SR_ERR_INVALID_ARG;
    if (max_pos < 1 || std::isnan(tau))
        return SR_ERR_INVALID_ARG;
    sr::PrestepArgs a;
    a.q_in = q_in;
    a.k_new = k_new;
    a.v_new = v_new;
    a.rope_cos = rope_cos;
    a.rope_sin = rope_sin;
    a.seq_lens = seq_lens;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.k0 = k0;
    a.v0 = v0;
    a.q_out = q_out;
    a.mask = route_mask;
    a.active = active_list;
    a.error = device_error;
    a.tau = tau;
    a.batch = dims->batch;
    a.n_q_heads = dims->n_q_heads;
    a.n_kv_heads = dims->n_kv_heads;
    a.max_seq_len = dims->max_seq_len;
    a.max_pos = max_pos;
    const cudaError_t e = sr::launch_rope_append_route(a, as_stream(stream));
    return e == cudaSuccess ? SR_OK : cuda_fail(e);
}

size_t sr_decode_workspace_bytes(const sr_dims *dims, int32_t max_splits)
{
    if (check_dims(dims) != SR_OK || max_splits < 0 || max_splits > SR_MAX_SPLITS)
        return 0;
    const int U = dims->batch * dims->n_kv_heads;
    const int M = dims->n_q_heads / dims->n_kv_heads;
    int64_t slots = sr::slots_needed(U, 0);
    if (max_splits > 0 && sr::slots_needed(U, max_splits) > slots)
        slots = sr::slots_needed(U, max_splits);
    return sr::workspace_layout(U, M, slots).total;
}

sr_status sr_workspace_init(void *workspace, size_t workspace_bytes, void *stream)
{
    if (!workspace || !aligned(workspace, 256) || workspace_bytes == 0)
        return SR_ERR_WORKSPACE;
    const cudaError_t e = cudaMemsetAsync(workspace, 0, workspace_bytes, as_stream(stream));
    return e == cudaSuccess ? SR_OK : cuda_fail(e);
}

sr_status sr_decode_attention(const sr_dims *dims, const void *q, const void *k_cache, const void *v_cache,
                              const void *k0, const void *v0, const int32_t *seq_lens, const int32_t *active_list,
                              int32_t n_splits, void *out, void *workspace, size_t workspace_bytes, void *stream)
{
    (void)k0; // routing already consumed it; the scan reads position 0 from the cache
    const sr_status st = check_dims(dims);
    if (st != SR_OK)
        return st;
    if (!q || !k_cache || !v_cache || !v0 || !seq_lens || !active_list || !out)
        return SR_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(v0, 16) ||
        !aligned(out, 16) || !aligned(seq_lens, 4) || !aligned(active_list, 4))
        return SR_ERR_INVALID_ARG;
    if (n_splits < 0 || n_splits > SR_MAX_SPLITS)
        return SR_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256))
        return SR_ERR_WORKSPACE;
    const int U = dims->batch * dims->n_kv_heads;
    const int M = dims->n_q_heads / dims->n_kv_heads;
    const sr::WorkspaceLayout ws = sr::workspace_layout(U, M, sr::slots_needed(U, n_splits));
    if (workspace_bytes < ws.total)
        return SR_ERR_WORKSPACE;
    sr::DecodeArgs a{q,   k_cache,      v_cache,         v0,         seq_lens,         active_list,
                     out, workspace,    ws,              dims->batch, dims->n_q_heads, dims->n_kv_heads,
                     dims->max_seq_len, n_splits};
    const cudaError_t e = sr::launch_decode(a, as_stream(stream));
    return e == cudaSuccess ? SR_OK : cuda_fail(e);
}

sr_status sr_decode_attention_lse(const sr_dims *dims, const void *q, const void *k_cache, const void *v_cache,
                                  const void *k0, const void *v0, const int32_t *seq_lens, const int32_t *active_list,
                                  int32_t n_splits, void *out, float *lse, void *workspace, size_t workspace_bytes,
                                  void *stream)
{
    (void)k0;
    const sr_status st = check_dims(dims);
    if (st != SR_OK)
        return st;
    if (!q || !k_cache || !v_cache || !v0 || !seq_lens || !active_list || !out || !lse)
        return SR_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(v0, 16) ||
        !aligned(out, 16) || !aligned(seq_lens, 4) || !aligned(active_list, 4) || !aligned(lse, 4))
        return SR_ERR_INVALID_ARG;
    if (n_splits < 0 || n_splits > SR_MAX_SPLITS)
        return SR_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256))
        return SR_ERR_WORKSPACE;
    const int U = dims->batch * dims->n_kv_heads;
    const int M = dims->n_q_heads / dims->n_kv_heads;
    const sr::WorkspaceLayout ws = sr::workspace_layout(U, M, sr::slots_needed(U, n_splits));
    if (workspace_bytes < ws.total)
        return SR_ERR_WORKSPACE;
    sr::DecodeArgs a{q,   k_cache,      v_cache,         v0,         seq_lens,         active_list,
                     out, workspace,    ws,              dims->batch, dims->n_q_heads, dims->n_kv_heads,
                     dims->max_seq_len, n_splits};
    a.lse = lse;
    const cudaError_t e = sr::launch_decode(a, as_stream(stream));
    return e == cudaSuccess ? SR_OK : cuda_fail(e);
}

sr_status sr_decode_attention_partial(const sr_dims *dims, const void *q, const void *k_cache, const void *v_cache,
                                      const void *k0, const void *v0, const int32_t *seq_lens,
                                      const int32_t *active_list, int32_t n_splits, float *o_part, float *lse_part,
                                      void *workspace, size_t workspace_bytes, void *stream)
{
    (void)k0;
    const sr_status st = check_dims(dims);
    if (st != SR_OK)
        return st;
    if (!q || !k_cache || !v_cache || !v0 || !seq_lens || !active_list || !o_part || !lse_part)
        return SR_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(v0, 16) ||
        !aligned(o_part, 16) || !aligned(seq_lens, 4) || !aligned(active_list, 4) || !aligned(lse_part, 4))
        return SR_ERR_INVALID_ARG;
    if (n_splits < 0 || n_splits > SR_MAX_SPLITS)
        return SR_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256))
        return SR_ERR_WORKSPACE;
    const int U = dims->batch * dims->n_kv_heads;
    const int M = dims->n_q_heads / dims->n_kv_heads;
    const sr::WorkspaceLayout ws = sr::workspace_layout(U, M, sr::slots_needed(U, n_splits));
    if (workspace_bytes < ws.total)
        return SR_ERR_WORKSPACE;
    sr::DecodeArgs a{q,       k_cache,      v_cache,         v0,         seq_lens,         active_list,
                     nullptr, workspace,    ws,              dims->batch, dims->n_q_heads, dims->n_kv_heads,
                     dims->max_seq_len, n_splits};
    a.lse = lse_part;
    a.out_f32 = o_part;
    const cudaError_t e = sr::launch_decode(a, as_stream(stream));
    return e == cudaSuccess ? SR_OK : cuda_fail(e);
}

sr_status sr_combine_partials(const sr_dims *dims, int32_t n_parts, const float *o_parts, const float *lse_parts,
                              int64_t part_stride, void *out, void *stream)
{
    // Only the head count and head_dim matter here.
    if (!dims || dims->batch < 1 || dims->n_q_heads < 1 || (int64_t)dims->batch * dims->n_q_heads > INT32_MAX)
        return SR_ERR_INVALID_ARG;
    if (dims->head_dim != sr::kHeadDim)
        return SR_ERR_UNSUPPORTED;
    if (!o_parts || !lse_parts || !out || !aligned(o_parts, 16) || !aligned(lse_parts, 4) || !aligned(out, 16))
        return SR_ERR_INVALID_ARG;
    const int64_t heads = (int64_t)dims->batch * dims->n_q_heads;
    if (n_parts < 1 || n_parts > SR_MAX_PARTS || part_stride % 4 != 0 ||
        (n_parts > 1 && part_stride < heads * sr::kHeadDim))
        return SR_ERR_INVALID_ARG;
    const cudaError_t e = sr::launch_combine((int)heads, n_parts, o_parts, lse_parts, part_stride, out,
                                             as_stream(stream));
    return e == cudaSuccess ? SR_OK : cuda_fail(e);
}

sr_status sr_position0_weight(const sr_dims *dims, const void *q, const void *k_cache, const float *lse, float *p0,
                              void *stream)
{
    const sr_status st = check_dims(dims);
    if (st != SR_OK)
        return st;
    if (!q || !k_cache || !lse || !p0 || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(lse, 4) ||
        !aligned(p0, 4))
        return SR_ERR_INVALID_ARG;
    const cudaError_t e = sr::launch_position0(dims->batch, dims->n_q_heads, dims->n_kv_heads, dims->max_seq_len, q,
                                               k_cache, lse, p0, as_stream(stream));
    return e == cudaSuccess ? SR_OK : cuda_fail(e);
}

sr_status sr_selftest_bounded_wait(int32_t limit_us, int32_t *status, uint64_t *waited_ns, void *stream)
{
    if (limit_us < 1 || limit_us > 2000000 || !status || !aligned(status, 4) || !waited_ns || !aligned(waited_ns, 8))
        return SR_ERR_INVALID_ARG;
    const cudaError_t e = sr::launch_bounded_wait_selftest(
        limit_us, status, reinterpret_cast<unsigned long long *>(waited_ns), as_stream(stream));
    return e == cudaSuccess ? SR_OK : cuda_fail(e);
}

sr_status sr_route_decode_attention(const sr_dims *dims, const void *q, const void *k_cache, const void *v_cache,
                                    const void *k0, const void *v0, const int32_t *seq_lens, float tau,
                                    int32_t n_splits, uint8_t *route_mask, int32_t *active_list, void *out,
                                    void *workspace, size_t workspace_bytes, void *stream)
{
    const sr_status st = check_dims(dims);
    if (st != SR_OK)
        return st;
    if (!q || !k_cache || !v_cache || !k0 || !v0 || !seq_lens || !out)
        return SR_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(k0, 16) ||
        !aligned(v0, 16) || !aligned(out, 16) || !aligned(seq_lens, 4) ||
        (active_list && !aligned(active_list, 4)))
        return SR_ERR_INVALID_ARG;
    if (std::isnan(tau) || n_splits < 0 || n_splits > SR_MAX_SPLITS)
        return SR_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256))
        return SR_ERR_WORKSPACE;
    const int U = dims->batch * dims->n_kv_heads;
    const int M = dims->n_q_heads / dims->n_kv_heads;
    const sr::WorkspaceLayout ws = sr::workspace_layout(U, M, sr::slots_needed(U, n_splits));
    if (workspace_bytes < ws.total)
        return SR_ERR_WORKSPACE;
    sr::DecodeArgs a{q,   k_cache,      v_cache,         v0,         seq_lens,         nullptr,
                     out, workspace,    ws,              dims->batch, dims->n_q_heads, dims->n_kv_heads,
                     dims->max_seq_len, n_splits};
    a.fused = true;
    a.k0 = k0;
    a.tau = tau;
    a.mask_out = route_mask;
    a.active_out = active_list;
    const cudaError_t e = sr::launch_decode(a, as_stream(stream));
    return e == cudaSuccess ? SR_OK : cuda_fail(e);
}

sr_status sr_get_device_error(const void *workspace, int32_t *code, void *stream)
{
    if (!workspace || !aligned(workspace, 256))
        return SR_ERR_WORKSPACE;
    if (!code)
        return SR_ERR_INVALID_ARG;
    cudaError_t e = cudaMemcpyAsync(code, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, as_stream(stream));
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(as_stream(stream));
    return e == cudaSuccess ? SR_OK : cuda_fail(e);
}

sr_status sr_clear_device_error(void *workspace, void *stream)
{
    if (!workspace || !aligned(workspace, 256))
        return SR_ERR_WORKSPACE;
    const cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(int32_t), as_stream(stream));
    return e == cudaSuccess ? SR_OK : cuda_fail(e);
}

int32_t sr_decode_grid_size(void) { return sr::decode_grid_size(); }

} // extern "C"
