// Cosine of one query head with its group's position-0 key, the minimum over
// the group's heads, and the ordered compaction of the active units, shared by
// the routing kernel, the fused route + decode prologue and the RoPE + append
// + route step, so that all of them take the same decision bit for bit.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace sr {

// Lane mapping of the routing arithmetic for group size M: W lanes take one
// (unit, query head) pair, each lane V consecutive 16-byte blocks (8V bf16
// elements) of the query row and of the group's key row. A warp holds 32 / W
// pairs: exactly one GQA group when M >= 4 (one warp per group), 4 / M groups
// when M < 4. Every caller (routing kernel, fused route + decode prologue,
// RoPE + append + route step) uses this one arithmetic, so they all take the
// same decision bit for bit.
template <int M> struct RouteLanes {
    static_assert(M == 1 || M == 2 || M == 4 || M == 8, "group size");
    static constexpr int W = (M == 8) ? 4 : 8; // lanes per pair
    static constexpr int V = 16 / W;           // 16-byte blocks of each row per lane
    static constexpr int PAIRS = 32 / W;       // pairs per warp
    static constexpr int UNITS = PAIRS / M;    // units per warp
};

// Adds the products of one 16-byte block (8 bf16) of a and b to ab, aa, bb,
// in element order.
__device__ __forceinline__ void dots_block(const uint4 &a, const uint4 &b, float &ab, float &aa, float &bb)
{
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

// s_g = min over the group's heads of cos(q_h, k0_g), from this lane's blocks
// (qv of its query row, kv of its key row). The W lanes of a pair add their
// sums with a fixed xor tree; the cosine is 0 when a norm is 0, and a NaN
// cosine counts as +inf so that it never lowers the minimum; an xor tree over
// the group's lanes takes the minimum. Every lane of the group receives s_g.
// All 32 lanes must call it.
template <int M>
__device__ __forceinline__ float group_min_cosine(const uint4 (&qv)[RouteLanes<M>::V],
                                                  const uint4 (&kv)[RouteLanes<M>::V])
{
    constexpr int W = RouteLanes<M>::W, V = RouteLanes<M>::V;
    float ab = 0.f, aa = 0.f, bb = 0.f;
#pragma unroll
    for (int v = 0; v < V; ++v)
        dots_block(qv[v], kv[v], ab, aa, bb);
#pragma unroll
    for (int off = W / 2; off > 0; off >>= 1) {
        ab += __shfl_xor_sync(0xffffffffu, ab, off);
        aa += __shfl_xor_sync(0xffffffffu, aa, off);
        bb += __shfl_xor_sync(0xffffffffu, bb, off);
    }
    float c = (aa == 0.f || bb == 0.f) ? 0.f : ab / (sqrtf(aa) * sqrtf(bb));
    if (c != c)
        c = INFINITY;
#pragma unroll
    for (int off = W; off < W * M; off <<= 1)
        c = fminf(c, __shfl_xor_sync(0xffffffffu, c, off));
    return c;
}

// This lane's blocks of warp chunk `chunk` (units chunk*UNITS ..): qrows holds
// nu*M query rows (row u*M+m) and krows nu key rows, 16 blocks each, in global
// memory (kGlobal: read-only loads) or shared memory. Units past nu read as
// zero. Returns this lane's unit.
template <int M, bool kGlobal>
__device__ __forceinline__ int load_route_blocks(const uint4 *qrows, const uint4 *krows, int nu, int chunk,
                                                 uint4 (&qv)[RouteLanes<M>::V], uint4 (&kv)[RouteLanes<M>::V])
{
    using RL = RouteLanes<M>;
    const int lane = (int)threadIdx.x & 31;
    const int pr = lane / RL::W, j = lane % RL::W;
    const int unit = chunk * RL::UNITS + pr / M;
    const size_t qrow = (size_t)chunk * RL::PAIRS + pr;
#pragma unroll
    for (int v = 0; v < RL::V; ++v) {
        if (unit < nu) {
            const uint4 *qp = qrows + qrow * 16 + j * RL::V + v;
            const uint4 *kp = krows + (size_t)unit * 16 + j * RL::V + v;
            qv[v] = kGlobal ? __ldg(qp) : *qp;
            kv[v] = kGlobal ? __ldg(kp) : *kp;
        } else {
            qv[v] = make_uint4(0u, 0u, 0u, 0u);
            kv[v] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    return unit;
}

// Routes units 0 .. nu-1: warp `wid` of `nwarps` takes the warp chunks wid,
// wid + nwarps, ..., and issues the loads of its next chunk before reducing
// the current one. For every unit one lane calls store(u, sink), sink being
// (s_g >= tau). Called by whole warps; no block barrier inside.
template <int M, bool kGlobal, typename Store>
__device__ __forceinline__ void route_units_warp(const uint4 *qrows, const uint4 *krows, int nu, float tau, int wid,
                                                 int nwarps, Store &&store)
{
    using RL = RouteLanes<M>;
    const int lane = (int)threadIdx.x & 31;
    const int nchunks = (nu + RL::UNITS - 1) / RL::UNITS;
    int c = wid;
    if (c >= nchunks)
        return;
    uint4 qa[RL::V], ka[RL::V];
    int ua = load_route_blocks<M, kGlobal>(qrows, krows, nu, c, qa, ka);
    for (; c < nchunks; c += nwarps) {
        uint4 qb[RL::V], kb[RL::V];
        int ub = nu;
        if (c + nwarps < nchunks)
            ub = load_route_blocks<M, kGlobal>(qrows, krows, nu, c + nwarps, qb, kb);
        const float s = group_min_cosine<M>(qa, ka);
        if (lane % (RL::W * M) == 0 && ua < nu)
            store(ua, s >= tau);
#pragma unroll
        for (int v = 0; v < RL::V; ++v) {
            qa[v] = qb[v];
            ka[v] = kb[v];
        }
        ua = ub;
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
