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
// each), read straight from global memory; 0 when a norm is 0; a NaN result is
// returned as +inf so that it never lowers the group minimum. The 16 vectors
// of a row are combined in the same rotated order as head_cosine_smem, so both
// give the same bits for the same `rot`.
__device__ __forceinline__ float head_cosine(const __nv_bfloat16 *__restrict__ qrow,
                                             const __nv_bfloat16 *__restrict__ krow, int rot)
{
    uint4 qa[16], ka[16];
    const uint4 *qv = reinterpret_cast<const uint4 *>(qrow);
    const uint4 *kv = reinterpret_cast<const uint4 *>(krow);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        qa[i] = __ldg(qv + ((i + rot) & 15));
        ka[i] = __ldg(kv + ((i + rot) & 15));
    }
    float dot, qq, kk;
    dots_row(qa, ka, dot, qq, kk);
    float c = (qq == 0.f || kk == 0.f) ? 0.f : dot / (sqrtf(qq) * sqrtf(kk));
    if (c != c)
        c = INFINITY;
    return c;
}

// cos(q_h, k0_g) from rows staged in shared memory (128 bf16 = 16 x 16-byte
// vectors each). The vectors are visited starting at `rot` (mod 16), taken from
// the pair index so that adjacent threads hit different shared-memory banks;
// the visiting order fixes the fp32 rounding, so every caller that uses the
// same pair index gets the same bits. Same conventions as head_cosine.
__device__ __forceinline__ float head_cosine_smem(const uint4 *qrow, const uint4 *krow, int rot)
{
    float ab = 0.f, aa = 0.f, bb = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int k = (i + rot) & 15;
        const uint4 av = qrow[k], bv = krow[k];
        const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
        const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
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
    float c = (aa == 0.f || bb == 0.f) ? 0.f : ab / (sqrtf(aa) * sqrtf(bb));
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

namespace sr {

// Route the nu units u0 .. u0+nu-1 whose rows are staged in shared memory:
// `rows` holds their nu*M query rows (row u*M+m of q) followed by their nu key
// rows, 256 bytes each. NT threads take one (unit, head) pair each per pass
// (NT a multiple of 32, so a unit's M pairs sit in adjacent lanes of one
// warp). Writes sflag[u] = sink, and mask_out[u] when mask_out is not null.
template <int M, int NT>
__device__ __forceinline__ void route_staged(const uint4 *rows, int u0, int nu, float tau, uint8_t *sflag,
                                             uint8_t *mask_out)
{
    const uint4 *kr = rows + nu * M * 16;
    const int pairs = nu * M;
    for (int base = 0; base < pairs; base += NT) {
        const int pr = base + (int)threadIdx.x;
        const bool valid = pr < pairs;
        const int lu = pr / M;
        float c = INFINITY;
        if (valid)
            c = head_cosine_smem(rows + pr * 16, kr + lu * 16, (u0 * M + pr) & 15);
        c = group_min<M>(c);
        if (valid && pr - lu * M == 0) {
            const uint8_t sink = (c >= tau) ? 1 : 0;
            sflag[u0 + lu] = sink;
            if (mask_out)
                mask_out[u0 + lu] = sink;
        }
    }
}

} // namespace sr
