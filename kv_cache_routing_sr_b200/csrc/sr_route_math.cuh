// Cosine of one query head with its group's position-0 key and the ordered
// compaction of the active units, shared by the routing kernel, the fused
// route + decode prologue and the RoPE + append + route step, so that all of
// them take the same decision bit for bit.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace sr {

// The cosine of a (unit, head) pair is computed by the 16 lanes of a
// half-warp: lane l takes the 16-byte block l (elements 8l .. 8l+7) of the
// query row and of the key row, sums its 8 products in element order, and a
// fixed xor-shuffle tree (offsets 8, 4, 2, 1) adds the 16 lane sums. Every
// caller uses this one arithmetic, so they all take the same decision bit for
// bit.

// Lane sums of <a,b>, <a,a> and <b,b> over one 16-byte block (8 bf16) of each row.
__device__ __forceinline__ void dots_vec(const uint4 &a, const uint4 &b, float &ab, float &aa, float &bb)
{
    ab = aa = bb = 0.f;
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
    const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
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

// Sum over the 16 lanes of each half-warp; every lane receives it. All 32
// lanes of the warp must call it.
__device__ __forceinline__ float half_warp_sum(float x)
{
#pragma unroll
    for (int off = 8; off > 0; off >>= 1)
        x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// cos(q_h, k0_g) of one pair from this lane's blocks: 0 when a norm is 0; a
// NaN result is returned as +inf so that it never lowers the group minimum.
// Returned in all 16 lanes of the half-warp. All 32 lanes must call it.
__device__ __forceinline__ float pair_cosine(const uint4 &qv, const uint4 &kv)
{
    float ab, aa, bb;
    dots_vec(qv, kv, ab, aa, bb);
    ab = half_warp_sum(ab);
    aa = half_warp_sum(aa);
    bb = half_warp_sum(bb);
    float c = (aa == 0.f || bb == 0.f) ? 0.f : ab / (sqrtf(aa) * sqrtf(bb));
    if (c != c)
        c = INFINITY;
    return c;
}

// Route the nu units u0 .. u0+nu-1 whose rows are staged in shared memory:
// `rows` holds their nu*M query rows (row u*M+m of q) followed by their nu key
// rows, 256 bytes each. NT threads (a multiple of 32) take NT/8 pairs per
// pass, two per half-warp; the pairs' cosines go to cosbuf (nu*M floats), and
// after a block barrier one thread per unit takes the minimum over its M heads.
// Writes sflag[u] = sink, and mask_out[u] when mask_out is not null. Called by
// all NT threads; ends without a trailing barrier.
template <int M, int NT>
__device__ __forceinline__ void route_staged(const uint4 *rows, int u0, int nu, float tau, uint8_t *sflag,
                                             uint8_t *mask_out, float *cosbuf)
{
    const uint4 *kr = rows + nu * M * 16;
    const int pairs = nu * M;
    const int hw = (int)threadIdx.x >> 4, l16 = (int)threadIdx.x & 15;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    // Two pairs per half-warp and pass: their loads and shuffle chains are
    // independent, so they overlap (each pair's arithmetic is unchanged).
    for (int base = 0; base < pairs; base += NT / 8) {
        const int pa = base + hw, pb = base + NT / 16 + hw;
        const bool va = pa < pairs, vb = pb < pairs;
        const uint4 qa = va ? rows[pa * 16 + l16] : zero;
        const uint4 ka = va ? kr[(pa / M) * 16 + l16] : zero;
        const uint4 qb = vb ? rows[pb * 16 + l16] : zero;
        const uint4 kb = vb ? kr[(pb / M) * 16 + l16] : zero;
        const float ca = pair_cosine(qa, ka);
        const float cb = pair_cosine(qb, kb);
        if (l16 == 0) {
            if (va)
                cosbuf[pa] = ca;
            if (vb)
                cosbuf[pb] = cb;
        }
    }
    __syncthreads();
    for (int lu = (int)threadIdx.x; lu < nu; lu += NT) {
        float s = INFINITY;
#pragma unroll
        for (int m = 0; m < M; ++m)
            s = fminf(s, cosbuf[lu * M + m]);
        const uint8_t sink = (s >= tau) ? 1 : 0;
        sflag[u0 + lu] = sink;
        if (mask_out)
            mask_out[u0 + lu] = sink;
    }
}

} // namespace sr

namespace sr {

// Ordered compaction: active[0] = number of units u < U with sflag[u] == 0,
// active[1..] = those units in ascending order. Warp ballots give each lane's
// rank inside its warp and a one-warp scan of the per-warp counts gives the
// warp offsets, NT threads at a time (one warp alone when U <= 32). Called by
// all NT threads of the block after the flags are visible to them (a block
// barrier); warp_cnt / warp_off are shared arrays of NT/32 and NT/32 + 1 entries.
template <int NT>
__device__ __forceinline__ void compact_active(const uint8_t *sflag, int U, int32_t *active, int32_t *warp_cnt,
                                               int32_t *warp_off)
{
    constexpr int kWarps = NT / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (U <= 32) {
        // One warp's ballot orders everything; no block barrier needed.
        if (warp == 0) {
            const bool act = lane < U && !sflag[lane];
            const unsigned ball = __ballot_sync(0xffffffffu, act);
            if (act)
                active[1 + __popc(ball & ((1u << lane) - 1u))] = lane;
            if (lane == 0)
                active[0] = __popc(ball);
        }
        return;
    }
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
