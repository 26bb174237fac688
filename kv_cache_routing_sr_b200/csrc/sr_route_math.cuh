// Cosine of one query head with its group's position-0 key, shared by the
// routing kernel and the fused route + decode prologue so that both take the
// same decision bit for bit.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace sr {

// <a,b>, <a,a> and <b,b> of two rows of 128 bf16 held as 16 x 16-byte vectors,
// in one pass (each vector is used once, so all 32 loads can be in flight).
__device__ __forceinline__ void dots_row(const uint4 (&a)[16], const uint4 (&b)[16], float &ab, float &aa, float &bb)
{
    ab = aa = bb = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint32_t aw[4] = {a[i].x, a[i].y, a[i].z, a[i].w};
        const uint32_t bw[4] = {b[i].x, b[i].y, b[i].z, b[i].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&aw[j]));
            const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&bw[j]));
            ab = fmaf(fa.x, fb.x, ab);
            ab = fmaf(fa.y, fb.y, ab);
            aa = fmaf(fa.x, fa.x, aa);
            aa = fmaf(fa.y, fa.y, aa);
            bb = fmaf(fb.x, fb.x, bb);
            bb = fmaf(fb.y, fb.y, bb);
        }
    }
}

// cos(q_h, k0_g) in fp32 for query row `qrow` and key row `krow` (128 bf16
// each); 0 when a norm is 0; a NaN result is returned as +inf so that it never
// lowers the group minimum.
__device__ __forceinline__ float head_cosine(const __nv_bfloat16 *__restrict__ qrow,
                                             const __nv_bfloat16 *__restrict__ krow)
{
    uint4 qa[16], ka[16];
    const uint4 *qv = reinterpret_cast<const uint4 *>(qrow);
    const uint4 *kv = reinterpret_cast<const uint4 *>(krow);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        qa[i] = __ldg(qv + i);
        ka[i] = __ldg(kv + i);
    }
    float dot, qq, kk;
    dots_row(qa, ka, dot, qq, kk);
    float c = (qq == 0.f || kk == 0.f) ? 0.f : dot / (sqrtf(qq) * sqrtf(kk));
    if (c != c)
        c = INFINITY;
    return c;
}

// Minimum over groups of M adjacent lanes (M divides 32).
template <int M> __device__ __forceinline__ float group_min(float c)
{
#pragma unroll
    for (int off = 1; off < M; off <<= 1)
        c = fminf(c, __shfl_xor_sync(0xffffffffu, c, off));
    return c;
}

} // namespace sr
