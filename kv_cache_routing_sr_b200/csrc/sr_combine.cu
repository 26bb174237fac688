// Combination of partial attention outputs computed over disjoint position
// ranges of the same heads (context parallelism: each GPU scans its shard of
// the cache, the partials are exchanged, every rank combines them).
//
// Method: the split-K decode with an in-kernel reduction of the SinkRouter
// README (decode-time procedure list) reduces (m, l, O) partials of one GPU's
// splits; across GPUs the same reduction is taken over per-shard results in
// their normalised form. For part r with output o_r = O_r / l_r and log-sum-exp
// lse_r of its logits:
//     lse = log sum_r exp(lse_r),     out = sum_r exp(lse_r - lse) o_r,
// which equals softmax attention over the union of the ranges (the softmax
// denominator of the union is the sum of the parts' denominators). A sink head
// (lse NaN in part 0: no attention was computed, o_0 = v0) is copied.
//
// Layout: one warp per query head, lane c owns output elements 4c .. 4c+3
// (one float4 of every part); the parts' lse values are read by every lane.
#include <cmath>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sinkrouter.h"
#include "sr_internal.h"
#include "sr_ptx.cuh"

namespace sr {
namespace {

constexpr int kWarpsPerBlock = 8;

__device__ __forceinline__ uint32_t pack2(float a, float b)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

__global__ void __launch_bounds__(32 * kWarpsPerBlock)
combine_kernel(const float *__restrict__ o_parts, const float *__restrict__ lse_parts, int64_t stride, int n_parts,
               int n_heads, __nv_bfloat16 *__restrict__ out)
{
    // The partials are the previous kernels' output (the decode kernel, or the
    // exchange): wait for them, then let the next kernel launch.
    grid_dependency_wait();
    grid_launch_dependents();

    const int lane = threadIdx.x & 31;
    const int warp0 = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
    const int nwarps = gridDim.x * kWarpsPerBlock;
    for (int h = warp0; h < n_heads; h += nwarps) {
        const float lse0 = __ldg(lse_parts + h);
        float4 acc;
        if (isnan(lse0)) {
            acc = __ldg(reinterpret_cast<const float4 *>(o_parts + (size_t)h * kHeadDim) + lane);
        } else {
            float mx = -INFINITY;
            for (int r = 0; r < n_parts; ++r)
                mx = fmaxf(mx, __ldg(lse_parts + r * stride + h));
            float den = 0.f;
            acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int r = 0; r < n_parts; ++r) {
                const float wr = expf(__ldg(lse_parts + r * stride + h) - mx); // 0 for an empty part
                const float4 o = __ldg(reinterpret_cast<const float4 *>(o_parts + r * stride +
                                                                        (size_t)h * kHeadDim) + lane);
                den += wr;
                acc.x = fmaf(wr, o.x, acc.x);
                acc.y = fmaf(wr, o.y, acc.y);
                acc.z = fmaf(wr, o.z, acc.z);
                acc.w = fmaf(wr, o.w, acc.w);
            }
            const float inv = 1.f / den;
            acc.x *= inv, acc.y *= inv, acc.z *= inv, acc.w *= inv;
        }
        uint2 packed;
        packed.x = pack2(acc.x, acc.y);
        packed.y = pack2(acc.z, acc.w);
        reinterpret_cast<uint2 *>(out + (size_t)h * kHeadDim)[lane] = packed;
    }
}

} // namespace

cudaError_t launch_combine(int n_heads, int n_parts, const float *o_parts, const float *lse_parts, int64_t part_stride,
                           void *out, cudaStream_t stream)
{
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return e;
    const int want = (n_heads + kWarpsPerBlock - 1) / kWarpsPerBlock;
    const int cap = 8 * sms; // 8 blocks of 8 warps per SM
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(want < cap ? want : cap);
    cfg.blockDim = dim3(32 * kWarpsPerBlock);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, combine_kernel, o_parts, lse_parts, part_stride, n_parts, n_heads,
                           static_cast<__nv_bfloat16 *>(out));
    return e != cudaSuccess ? e : cudaGetLastError();
}

} // namespace sr
