// Internal interfaces between the C-ABI layer (sr_abi.cu) and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "sinkrouter.h"

namespace sr {

constexpr int kHeadDim = 128;
constexpr int kMaxGroup = 8;      // query heads per KV head handled by one n8 MMA tile
constexpr int kAutoGridCap = 1024; // persistent CTAs never exceed this (sizes the workspace)

// Workspace layout: [error word | per-unit arrival counters | partial O | partial (m, l)].
struct WorkspaceLayout {
    size_t err_off = 0;
    size_t cnt_off = 256;
    size_t part_o_off = 0;
    size_t part_ml_off = 0;
    size_t total = 0;
    int64_t slots = 0;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Partial slots a launch may touch: automatic splits use slot = cta + active
// index (< grid + units); forced splits use active index * n_splits + split.
inline int64_t slots_needed(int units, int n_splits)
{
    return n_splits > 0 ? (int64_t)units * n_splits : (int64_t)kAutoGridCap + units;
}

inline WorkspaceLayout workspace_layout(int units, int group, int64_t slots)
{
    WorkspaceLayout w;
    w.slots = slots;
    w.part_o_off = align_up(w.cnt_off + sizeof(int32_t) * (size_t)units, 256);
    w.part_ml_off = align_up(w.part_o_off + sizeof(float) * (size_t)slots * group * kHeadDim, 256);
    w.total = align_up(w.part_ml_off + 2 * sizeof(float) * (size_t)slots * group, 256);
    return w;
}

struct RouteArgs {
    const void *q;
    const void *k0;
    float tau;
    uint8_t *mask;
    int32_t *active;
    int batch, n_q_heads, n_kv_heads;
};

struct DecodeArgs {
    const void *q, *k_cache, *v_cache, *v0;
    const int32_t *seq_lens, *active_list;
    void *out;
    void *workspace;
    WorkspaceLayout ws;
    int batch, n_q_heads, n_kv_heads, max_seq_len, n_splits;
    // Fused routing (sr_route_decode_attention): the kernel routes every unit
    // itself from q and k0 instead of reading active_list.
    bool fused = false;
    const void *k0 = nullptr;
    float tau = 0.f;
    uint8_t *mask_out = nullptr;
    int32_t *active_out = nullptr;
    // Optional per-head log-sum-exp output (sr_decode_attention_lse).
    float *lse = nullptr;
    // Partial outputs for context parallelism (sr_decode_attention_partial):
    // fp32 output instead of `out`.
    float *out_f32 = nullptr;
};

// RoPE + append + position-0 capture + routing (sr_rope_append_route).
struct PrestepArgs {
    const void *q_in, *k_new, *v_new;
    const float *rope_cos, *rope_sin;
    int32_t *seq_lens;
    void *k_cache, *v_cache, *k0, *v0, *q_out;
    uint8_t *mask;
    int32_t *active;
    int32_t *error;
    float tau;
    int batch, n_q_heads, n_kv_heads, max_seq_len, max_pos;
};

cudaError_t launch_route(const RouteArgs &a, cudaStream_t stream);
cudaError_t launch_rope_append_route(const PrestepArgs &a, cudaStream_t stream);
// Self-test of the bounded wait (sr_selftest_bounded_wait).
cudaError_t launch_bounded_wait_selftest(int32_t limit_us, int32_t *status, unsigned long long *waited_ns,
                                         cudaStream_t stream);
// Log-sum-exp combination of n_parts partial outputs (sr_combine_partials).
// p0[b, h] = exp(<q[b, h], K[b, g, 0]> / sqrt(d) - lse[b, h]) (sr_position0_weight)
cudaError_t launch_position0(int B, int Hq, int Hkv, int Lmax, const void *q, const void *k_cache, const float *lse,
                             float *p0, cudaStream_t stream);
cudaError_t launch_combine(int n_heads, int n_parts, const float *o_parts, const float *lse_parts, int64_t part_stride,
                           void *out, cudaStream_t stream);
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream);
// Persistent CTAs of the decode kernel on the current device (0 on error).
int decode_grid_size();
// Records a CUDA failure for sr_last_cuda_error and returns SR_ERR_CUDA.
sr_status record_cuda_failure(cudaError_t e);

} // namespace sr
