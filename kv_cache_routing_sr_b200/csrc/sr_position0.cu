// The full-attention weight of position 0 for every query head, from the
// log-sum-exp of the scan: p0[b, h] = exp(<q[b, h], K[b, g, 0]> / sqrt(d) -
// lse[b, h]), g = h / M.
//
// Method: the pith.science review of arXiv 2604.16883 (Figure 10 caption)
// builds the routing proxy's reference "oracle sink event" from the
// full-attention weight of the BOS position; sr_decode_attention_lse returns the
// log-sum-exp that makes that weight one dot product away.
//
// Layout: one warp per query head, lane c takes elements 4c .. 4c+3 of the
// query row and of the unit's cached position-0 key (8 bytes each), fp32
// products summed by a fixed xor-shuffle tree.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sinkrouter.h"
#include "sr_internal.h"

namespace sr {
namespace {

constexpr int kWarpsPerBlock = 8;

__device__ __forceinline__ float lo16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi16(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__global__ void __launch_bounds__(32 * kWarpsPerBlock)
position0_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k_cache,
                 const float *__restrict__ lse, float *__restrict__ p0, int n_heads, int Hq, int Hkv, int M,
                 int Lmax)
{
    const int w = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5), lane = (int)(threadIdx.x & 31);
    if (w >= n_heads)
        return;
    const int b = w / Hq, h = w - b * Hq, g = h / M;
    const uint2 qv = reinterpret_cast<const uint2 *>(q + (size_t)w * kHeadDim)[lane];
    const uint2 kv = reinterpret_cast<const uint2 *>(k_cache + ((size_t)(b * Hkv + g) * Lmax) * kHeadDim)[lane];
    float d = lo16(qv.x) * lo16(kv.x);
    d = fmaf(hi16(qv.x), hi16(kv.x), d);
    d = fmaf(lo16(qv.y), lo16(kv.y), d);
    d = fmaf(hi16(qv.y), hi16(kv.y), d);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        d += __shfl_xor_sync(0xffffffffu, d, off);
    if (lane == 0)
        p0[w] = expf(d * 0.08838834764831845f - lse[w]); // 1 / sqrt(128)
}

} // namespace

cudaError_t launch_position0(int B, int Hq, int Hkv, int Lmax, const void *q, const void *k_cache, const float *lse,
                             float *p0, cudaStream_t stream)
{
    const int n_heads = B * Hq;
    const int blocks = (n_heads + kWarpsPerBlock - 1) / kWarpsPerBlock;
    position0_kernel<<<blocks, 32 * kWarpsPerBlock, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k_cache), lse, p0, n_heads, Hq,
        Hkv, Hq / Hkv, Lmax);
    return cudaGetLastError();
}

} // namespace sr
