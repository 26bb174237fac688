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
// and squared norms are warp shuffle reductions in fp32. All loads of a pass
// are issued before the first reduction (one memory round trip per pass). The compaction writes
// active units in ascending order with warp ballots and a block prefix, so no
// CTA of the decode kernel is ever bound to a sink unit.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sr_internal.h"
#include "sr_ptx.cuh"

namespace sr {
namespace {

constexpr int kRouteThreads = 1024;
constexpr int kRouteWarps = kRouteThreads / 32;

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ void widen4(uint2 raw, float (&v)[4])
{
    const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
    const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
    v[0] = fa.x, v[1] = fa.y, v[2] = fb.x, v[3] = fb.y;
}

__device__ __forceinline__ float dot4(const float (&a)[4], const float (&b)[4])
{
    return a[0] * b[0] + a[1] * b[1] + a[2] * b[2] + a[3] * b[3];
}

// M = query heads per KV head (compile time). Each warp routes UNR units per
// pass, with every load of those units (k0 and the M query heads) issued before
// the first reduction, so a pass costs one memory round trip.
template <int M>
__global__ void __launch_bounds__(kRouteThreads, 1)
route_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k0, float tau,
             uint8_t *__restrict__ mask, int32_t *__restrict__ active, int B, int Hkv)
{
    constexpr int UNR = (8 / M) > 0 ? (8 / M) : 1;
    extern __shared__ uint8_t sink_flag[]; // [B*Hkv]
    __shared__ int32_t warp_cnt[kRouteWarps];
    __shared__ int32_t warp_off[kRouteWarps + 1];

    // Inputs may come from the previous kernel in the stream, and the previous
    // decode step may still read route_mask / active_list: wait for it, then
    // let the decode kernel that follows launch and run its prologue.
    grid_dependency_wait();
    grid_launch_dependents();

    const int U = B * Hkv;
    const int Hq = Hkv * M;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    for (int base = warp; base < U; base += kRouteWarps * UNR) {
        uint2 kraw[UNR], qraw[UNR][M];
#pragma unroll
        for (int k = 0; k < UNR; ++k) {
            const int u = base + k * kRouteWarps;
            kraw[k] = make_uint2(0u, 0u);
#pragma unroll
            for (int m = 0; m < M; ++m)
                qraw[k][m] = make_uint2(0u, 0u);
            if (u < U) {
                const int b = u / Hkv, g = u - b * Hkv;
                kraw[k] = *reinterpret_cast<const uint2 *>(k0 + (size_t)u * kHeadDim + 4 * lane);
#pragma unroll
                for (int m = 0; m < M; ++m)
                    qraw[k][m] = *reinterpret_cast<const uint2 *>(
                        q + ((size_t)b * Hq + (size_t)g * M + m) * kHeadDim + 4 * lane);
            }
        }
#pragma unroll
        for (int k = 0; k < UNR; ++k) {
            const int u = base + k * kRouteWarps;
            float kv[4];
            widen4(kraw[k], kv);
            const float kk = warp_sum(dot4(kv, kv));
            float s = INFINITY;
#pragma unroll
            for (int m = 0; m < M; ++m) {
                float qv[4];
                widen4(qraw[k][m], qv);
                const float dot = warp_sum(dot4(qv, kv));
                const float qq = warp_sum(dot4(qv, qv));
                const float c = (qq == 0.f || kk == 0.f) ? 0.f : dot / (sqrtf(qq) * sqrtf(kk));
                // A NaN cosine never lowers the minimum (same rule as a "<" scan).
                s = (c < s) ? c : s;
            }
            if (u < U && lane == 0) {
                const uint8_t sink = (s >= tau) ? 1 : 0;
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

template <int M>
cudaError_t launch_route_m(const RouteArgs &a, cudaStream_t stream)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(kRouteThreads);
    cfg.dynamicSmemBytes = (size_t)a.batch * a.n_kv_heads;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, route_kernel<M>, static_cast<const __nv_bfloat16 *>(a.q),
                              static_cast<const __nv_bfloat16 *>(a.k0), a.tau, a.mask, a.active, a.batch,
                              a.n_kv_heads);
}

} // namespace

cudaError_t launch_route(const RouteArgs &a, cudaStream_t stream)
{
    cudaError_t e;
    switch (a.n_q_heads / a.n_kv_heads) {
    case 1:
        e = launch_route_m<1>(a, stream);
        break;
    case 2:
        e = launch_route_m<2>(a, stream);
        break;
    case 4:
        e = launch_route_m<4>(a, stream);
        break;
    case 8:
        e = launch_route_m<8>(a, stream);
        break;
    default:
        return cudaErrorInvalidValue;
    }
    return e != cudaSuccess ? e : cudaGetLastError();
}

} // namespace sr
