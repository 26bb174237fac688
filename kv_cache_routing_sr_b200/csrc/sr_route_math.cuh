// Cosine of one query head with its group's position-0 key and the ordered
// compaction of the active units, shared by the routing kernel, the fused
// route + decode prologue and the RoPE + append + route step, so that all of
// them take the same decision bit for bit.
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

namespace sr {

// Ordered compaction: active[0] = number of units u < U with sflag[u] == 0,
// active[1..] = those units in ascending order. Warp ballots give each lane's
// rank inside its warp and a one-warp scan of the per-warp counts gives the
// warp offsets, NT threads at a time. Called by all NT threads of the block;
// warp_cnt / warp_off are shared arrays of NT/32 and NT/32 + 1 entries.
template <int NT>
__device__ __forceinline__ void compact_active(const uint8_t *sflag, int U, int32_t *active, int32_t *warp_cnt,
                                               int32_t *warp_off)
{
    constexpr int kWarps = NT / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int32_t total = 0;
    for (int c0 = 0; c0 < U; c0 += NT) {
        const int u = c0 + (int)threadIdx.x;
        const bool act = (u < U) && !sflag[u];
        const unsigned ball = __ballot_sync(0xffffffffu, act);
        const int before = __popc(ball & ((1u << lane) - 1u));
        if (lane == 0)
            warp_cnt[warp] = __popc(ball);
        __syncthreads();
        if (warp == 0) {
            const int v = (lane < kWarps) ? warp_cnt[lane] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o)
                    incl += y;
            }
            if (lane < kWarps)
                warp_off[lane] = incl - v;
            if (lane == kWarps - 1)
                warp_off[kWarps] = incl;
        }
        __syncthreads();
        if (act)
            active[1 + total + warp_off[warp] + before] = u;
        total += warp_off[kWarps];
        __syncthreads();
    }
    if (threadIdx.x == 0)
        active[0] = total;
}

} // namespace sr
