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
// Layout: one CTA of 256 threads. The q and k0 rows of a chunk of units (all
// units, for every workload here) are staged in shared memory by two bulk
// copies, then one half-warp per (unit, query head) pair computes the cosine
// (16 lanes of 8 elements each and a shuffle tree) and one thread per unit
// takes the minimum over its heads. The compaction writes
// active units in ascending order with warp ballots and a block prefix, so no
// CTA of the decode kernel is ever bound to a sink unit.
#include <atomic>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sinkrouter.h"
#include "sr_internal.h"
#include "sr_ptx.cuh"
#include "sr_route_math.cuh"

namespace sr {
namespace {

constexpr int kRouteThreads = 256;
constexpr int kRouteWarps = kRouteThreads / 32;

constexpr int kRowBudget = 160 * 1024; // shared bytes for staged q / k0 rows
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Units per staged chunk for group size M.
template <int M> __host__ __device__ constexpr int chunk_units() { return kRowBudget / ((M + 1) * 256); }

// M = query heads per KV head (compile time). The q rows of a chunk of units
// and their k0 rows are contiguous in global memory, so one thread stages them
// with two bulk copies (one memory round trip, whatever the chunk size); then
// each half-warp computes one (unit, head) cosine from shared memory and one
// thread per unit takes the minimum over its heads.
template <int M>
__global__ void __launch_bounds__(kRouteThreads, 1)
route_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k0, float tau,
             uint8_t *__restrict__ mask, int32_t *__restrict__ active, int B, int Hkv, int cu)
{
    extern __shared__ __align__(128) uint8_t dsm[]; // [cu*(M+1)*256 staged rows][B*Hkv sink flags]
    __shared__ __align__(8) uint64_t bar;
    __shared__ int32_t warp_cnt[kRouteWarps];
    __shared__ int32_t warp_off[kRouteWarps + 1];
    __shared__ float cosbuf[chunk_units<M>() * M];

    const int U = B * Hkv;
    uint4 *rows = reinterpret_cast<uint4 *>(dsm);
    uint8_t *sink_flag = dsm + (size_t)cu * (M + 1) * 256;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        fence_mbar_init();
    }
    // Inputs may come from the previous kernel in the stream, and the previous
    // decode step may still read route_mask / active_list: wait for it, then
    // let the decode kernel that follows launch and run its prologue.
    grid_dependency_wait();
    grid_launch_dependents();
    __syncthreads();

    uint32_t ph = 0;
    bool timed_out = false;
    for (int u0 = 0; u0 < U; u0 += cu) {
        const int nu = (U - u0) < cu ? (U - u0) : cu;
        if (threadIdx.x == 0) {
            const uint32_t qbytes = (uint32_t)nu * M * 256, kbytes = (uint32_t)nu * 256;
            mbar_arrive_expect_tx(b, qbytes + kbytes);
            bulk_load(smem_u32(rows), q + (size_t)u0 * M * kHeadDim, qbytes, b);
            bulk_load(smem_u32(rows) + qbytes, k0 + (size_t)u0 * kHeadDim, kbytes, b);
        }
        if (!mbar_try_wait(b, ph)) {
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(b, ph)) {
                if (global_timer_ns() - t0 > kWaitLimitNs) {
                    timed_out = true;
                    break;
                }
            }
        }
        ph ^= 1;
        if (__syncthreads_or(timed_out)) {
            timed_out = true;
            break;
        }
        route_staged<M, kRouteThreads>(rows, u0, nu, tau, sink_flag, mask, cosbuf);
        __syncthreads(); // the rows are overwritten by the next chunk
    }
    if (timed_out) {
        // A copy never completed (never expected): publish an invalid count,
        // which the decode kernel reports as SR_DEVERR_ACTIVE_LIST.
        if (threadIdx.x == 0)
            active[0] = -1;
        return;
    }

    compact_active<kRouteThreads>(sink_flag, U, active, warp_cnt, warp_off);
}

template <int M>
cudaError_t launch_route_m(const RouteArgs &a, cudaStream_t stream)
{
    const int U = a.batch * a.n_kv_heads;
    const int cu = U < chunk_units<M>() ? U : chunk_units<M>();
    const size_t smem = (size_t)cu * (M + 1) * 256 + (size_t)U;
    static std::atomic<bool> configured[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev >= 0 && dev < 64 && !configured[dev].load()) {
        e = cudaFuncSetAttribute(route_kernel<M>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)((size_t)chunk_units<M>() * (M + 1) * 256 + SR_MAX_UNITS));
        if (e != cudaSuccess)
            return e;
        configured[dev].store(true);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(kRouteThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, route_kernel<M>, static_cast<const __nv_bfloat16 *>(a.q),
                              static_cast<const __nv_bfloat16 *>(a.k0), a.tau, a.mask, a.active, a.batch,
                              a.n_kv_heads, cu);
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
