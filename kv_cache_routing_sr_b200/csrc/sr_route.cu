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
// Layout: one CTA of 256 threads, one thread per (unit, query head) pair per
// pass (a pass covers 256 pairs: every workload here routes in one pass). A
// thread holds both 256-byte rows in registers, so each pass is one memory
// round trip, and the group minimum is a shuffle over adjacent lanes. The compaction writes
// active units in ascending order with warp ballots and a block prefix, so no
// CTA of the decode kernel is ever bound to a sink unit.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sr_internal.h"
#include "sr_ptx.cuh"
#include "sr_route_math.cuh"

namespace sr {
namespace {

constexpr int kRouteThreads = 256;
constexpr int kRouteWarps = kRouteThreads / 32;

// M = query heads per KV head (compile time). One thread per (unit, head)
// pair: it loads the head's query row and the unit's k0 row (2 x 256 bytes,
// all 32 loads in flight at once) and computes the cosine in fp32. The M
// threads of a unit are adjacent lanes, so the minimum over the group's heads
// is a shuffle reduction.
template <int M>
__global__ void __launch_bounds__(kRouteThreads, 1)
route_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k0, float tau,
             uint8_t *__restrict__ mask, int32_t *__restrict__ active, int B, int Hkv)
{
    extern __shared__ uint8_t sink_flag[]; // [B*Hkv]
    __shared__ int32_t warp_cnt[kRouteWarps];
    __shared__ int32_t warp_off[kRouteWarps + 1];

    // Inputs may come from the previous kernel in the stream, and the previous
    // decode step may still read route_mask / active_list: wait for it, then
    // let the decode kernel that follows launch and run its prologue.
    grid_dependency_wait();
    grid_launch_dependents();

    const int U = B * Hkv;
    const int pairs = U * M;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    for (int base = 0; base < pairs; base += kRouteThreads) {
        const int pr = base + (int)threadIdx.x;
        const bool valid = pr < pairs;
        const int u = pr / M, m = pr - (pr / M) * M;
        float c = INFINITY;
        if (valid) {
            const int b = u / Hkv, g = u - b * Hkv;
            c = head_cosine(q + ((size_t)b * Hkv * M + (size_t)g * M + m) * kHeadDim, k0 + (size_t)u * kHeadDim);
        }
        c = group_min<M>(c); // minimum over the M adjacent lanes of the unit
        if (valid && m == 0) {
            const uint8_t sink = (c >= tau) ? 1 : 0;
            mask[u] = sink;
            sink_flag[u] = sink;
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
            const int v = (lane < kRouteWarps) ? warp_cnt[lane] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o)
                    incl += y;
            }
            if (lane < kRouteWarps)
                warp_off[lane] = incl - v;
            if (lane == kRouteWarps - 1)
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
