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
// Layout: one CTA of 256 threads. One warp per GQA group (M >= 4; a warp takes
// 4 / M groups when M < 4): each lane loads its blocks of the query rows and of
// the key row straight from global memory, and shuffle reductions give each
// pair's cosine and the group's minimum (sr_route_math.cuh). A warp with more
// groups to route issues the loads of its next group before reducing the
// current one. The compaction writes active units in ascending order with warp
// ballots and a block prefix, so no CTA of the decode kernel is ever bound to a
// sink unit. No asynchronous copy is used, so nothing is in flight when the
// kernel ends.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sinkrouter.h"
#include "sr_internal.h"
#include "sr_ptx.cuh"
#include "sr_route_math.cuh"
#include "sr_timeline.cuh"

SR_TL_DEFINE(tl_route)
#ifdef SR_TIMELINE
// set by the host to the decode kernel's last-exit word (sr_timeline_last_exit_addr)
static __device__ unsigned long long *tl_exit_ptr;
static __device__ unsigned int tl_route_launch; // ring of per-launch stamps in rows 1 .. 64
extern "C" int sr_timeline_set_exit_ptr(void *p) { return (int)cudaMemcpyToSymbol(tl_exit_ptr, &p, sizeof(p)); }
#endif

namespace sr {
namespace {

constexpr int kRouteThreads = 256;
constexpr int kRouteWarps = kRouteThreads / 32;

// M = query heads per KV head (compile time). The dynamic shared memory holds
// one sink flag per unit.
template <int M>
__global__ void __launch_bounds__(kRouteThreads, 1)
route_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k0, float tau,
             uint8_t *__restrict__ mask, int32_t *__restrict__ active, int B, int Hkv)
{
    extern __shared__ uint8_t sink_flag[]; // [B*Hkv]
    __shared__ int32_t warp_cnt[kRouteWarps];
    __shared__ int32_t warp_off[kRouteWarps + 1];

    const int U = B * Hkv;
    if (threadIdx.x == 0)
        SR_STAMP(tl_route, 0);
    // Inputs may come from the previous kernel in the stream, and the previous
    // decode step may still read route_mask / active_list: wait for it, then
    // let the decode kernel that follows launch and run its prologue.
    grid_dependency_wait();
    grid_launch_dependents();
    if (threadIdx.x == 0)
        SR_STAMP(tl_route, 1);
#ifdef SR_TIMELINE
    if (threadIdx.x == 0) {
        const unsigned long long pe = tl_exit_ptr ? *(volatile unsigned long long *)tl_exit_ptr : 0ull;
        tl_route[0][5] = pe;
        const unsigned int ring = 1 + atomicAdd(&tl_route_launch, 1u) % 64u;
        tl_route[ring][1] = tl_route[0][1];
        tl_route[ring][5] = pe;
        tl_route[ring][0] = tl_route[0][0];
    }
#endif

    route_units_warp<M, true>(reinterpret_cast<const uint4 *>(q), reinterpret_cast<const uint4 *>(k0), U, tau,
                              (int)threadIdx.x >> 5, kRouteWarps, [&](int u, bool sink) {
                                  sink_flag[u] = sink ? 1 : 0;
                                  mask[u] = sink ? 1 : 0;
                              });
    __syncthreads();
    if (threadIdx.x == 0)
        SR_STAMP(tl_route, 3);
    compact_active<kRouteThreads>(sink_flag, U, active, warp_cnt, warp_off);
    if (threadIdx.x == 0)
        SR_STAMP(tl_route, 4);
}

template <int M>
cudaError_t launch_route_m(const RouteArgs &a, cudaStream_t stream)
{
    const int U = a.batch * a.n_kv_heads;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(kRouteThreads);
    cfg.dynamicSmemBytes = (size_t)U; // <= SR_MAX_UNITS = 16 KB: no opt-in needed
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
