// Routing kernel: cosine of each query head with its group's position-0 key,
// minimum over the group's heads, threshold, and ordered compaction of the
// active units into a work list.
//
// Method: SinkRouter README (github.com/streamer-AP/SinkRouter), decode-time
// procedure list -- the RoPE query is compared with the cached position-0 key
// and every GQA KV group is routed before the long cache scan; README routing
// controls -- the threshold is a cosine threshold. The min over heads and ">="
// are this library's reading of what the pages leave open.
//
// Layout: one CTA of 32 warps. Each warp owns whole units (b, g): lane l holds
// elements 4l..4l+3 of k0_g and of each query head, so a unit's dot products
// and squared norms are warp shuffle reductions in fp32. The compaction writes
// active units in ascending order with warp ballots and a block prefix, so no
// CTA of the decode kernel is ever bound to a sink unit.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sr_internal.h"

namespace sr {
namespace {

constexpr int kRouteThreads = 1024;
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kUnroll = 4; // units in flight per warp

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ void load4(const __nv_bfloat16 *p, float (&v)[4])
{
    const uint2 raw = *reinterpret_cast<const uint2 *>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
    const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    v[0] = fa.x, v[1] = fa.y, v[2] = fb.x, v[3] = fb.y;
}

__global__ void __launch_bounds__(kRouteThreads, 1)
route_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k0, float tau,
             uint8_t *__restrict__ mask, int32_t *__restrict__ active, int B, int Hq, int Hkv)
{
    extern __shared__ uint8_t sink_flag[]; // [B*Hkv]
    __shared__ int32_t warp_cnt[kRouteWarps];
    __shared__ int32_t warp_off[kRouteWarps + 1];

    const int U = B * Hkv;
    const int M = Hq / Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    for (int base = warp; base < U; base += kRouteWarps * kUnroll) {
        float s[kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k)
            s[k] = INFINITY;
        float kv[kUnroll][4] = {};
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int u = base + k * kRouteWarps;
            if (u < U)
                load4(k0 + (size_t)u * kHeadDim + 4 * lane, kv[k]);
        }
        float kk[kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k)
            kk[k] = warp_sum(kv[k][0] * kv[k][0] + kv[k][1] * kv[k][1] + kv[k][2] * kv[k][2] + kv[k][3] * kv[k][3]);
        for (int m = 0; m < M; ++m) {
            float qv[kUnroll][4] = {};
#pragma unroll
            for (int k = 0; k < kUnroll; ++k) {
                const int u = base + k * kRouteWarps;
                if (u < U) {
                    const int b = u / Hkv, g = u - b * Hkv;
                    load4(q + ((size_t)b * Hq + (size_t)g * M + m) * kHeadDim + 4 * lane, qv[k]);
                }
            }
#pragma unroll
            for (int k = 0; k < kUnroll; ++k) {
                const float dot = warp_sum(qv[k][0] * kv[k][0] + qv[k][1] * kv[k][1] + qv[k][2] * kv[k][2] +
                                           qv[k][3] * kv[k][3]);
                const float qq =
                    warp_sum(qv[k][0] * qv[k][0] + qv[k][1] * qv[k][1] + qv[k][2] * qv[k][2] + qv[k][3] * qv[k][3]);
                const float c = (qq == 0.f || kk[k] == 0.f) ? 0.f : dot / (sqrtf(qq) * sqrtf(kk[k]));
                // A NaN cosine never lowers the minimum (same rule as a "<" scan).
                s[k] = (c < s[k]) ? c : s[k];
            }
        }
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int u = base + k * kRouteWarps;
            if (u < U && lane == 0) {
                const uint8_t sink = (s[k] >= tau) ? 1 : 0;
                mask[u] = sink;
                sink_flag[u] = sink;
            }
        }
    }
    __syncthreads();

    // Ordered compaction of the active units.
    int32_t total = 0;
    for (int c0 = 0; c0 < U; c0 += kRouteThreads) {
        const int u = c0 + (int)threadIdx.x;
        const bool act = (u < U) && !sink_flag[u];
        const unsigned ball = __ballot_sync(0xffffffffu, act);
        const int before = __popc(ball & ((1u << lane) - 1u));
        if (lane == 0)
            warp_cnt[warp] = __popc(ball);
        __syncthreads();
        if (warp == 0) {
            const int v = warp_cnt[lane];
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o)
                    incl += y;
            }
            warp_off[lane] = incl - v;
            if (lane == 31)
                warp_off[kRouteWarps] = incl;
        }
        __syncthreads();
        if (act)
            active[1 + total + warp_off[warp] + before] = u;
        total += warp_off[kRouteWarps];
        __syncthreads();
    }
    if (threadIdx.x == 0)
        active[0] = total;
}

} // namespace

cudaError_t launch_route(const RouteArgs &a, cudaStream_t stream)
{
    const int U = a.batch * a.n_kv_heads;
    route_kernel<<<1, kRouteThreads, (size_t)U, stream>>>(
        static_cast<const __nv_bfloat16 *>(a.q), static_cast<const __nv_bfloat16 *>(a.k0), a.tau, a.mask, a.active,
        a.batch, a.n_q_heads, a.n_kv_heads);
    return cudaGetLastError();
}

} // namespace sr
