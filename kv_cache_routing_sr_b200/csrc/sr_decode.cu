// Split-K decode attention over the active units, with the sink bypass and the
// cross-split reduction in the same persistent kernel.
//
// Method: SinkRouter README (github.com/streamer-AP/SinkRouter), decode-time
// procedure list -- sink groups return the position-0 value, active groups run
// tiled QK / PV with online softmax, Split-K over the context and an in-kernel
// reduction; sota2 summary, Abstract -- decode attention is memory-bound on the
// KV-cache read. Output definition: pith.science review of arXiv 2604.16883,
// Figure 1 caption, eq. (1) (attention-weighted sum of cached values).
//
// Design (B200, sm_100a):
//  * One persistent CTA per SM: 4 consumer warps + 1 producer warp. The grid
//    never depends on the route result, so the launch needs no host sync; each
//    CTA reads the active list and seq_lens and derives its share of the work.
//  * Automatic splits: the active positions of all units are concatenated and
//    cut into one contiguous chunk per CTA (rounded to whole tiles, >= 256
//    positions), so every SM streams the same number of bytes whatever the mix
//    of unit lengths. A chunk may cover the end of one unit and the start of
//    the next; each (CTA, unit) overlap is one split.
//  * The producer lane walks its splits tile by tile and issues 3-D TMA loads
//    (two 128-byte-wide boxes for K, two for V, 128B swizzle) into a ring of
//    shared-memory stages, each guarded by a full/empty mbarrier pair. A small
//    header in each stage tells the consumers which unit / rows the tile holds.
//  * Each consumer warp owns 16*RB rows of every tile. S^T = K_tile * Q^T on
//    bf16 mma.sync m16n8k16 (positions on M, the group's query heads on N;
//    the tile is read once for all M heads), online softmax in fp32 with exp2,
//    P^T moved into the B-operand layout with movmatrix, O^T += V^T * P^T with
//    ldmatrix.trans. The contraction is tiny (M <= 8 heads), so the tensor
//    cores only serve to keep the issue rate far below the HBM stream rate.
//  * At the end of a split the four warps merge their (m, l, O) in shared
//    memory, write one fp32 partial, and count it on the unit's arrival
//    counter. The CTA that brings the counter to the unit's split count merges
//    all partials of the unit in a fixed order, writes the bf16 output and
//    resets the counter (nobody ever waits for another CTA).
//  * Sink units: while the first tiles are in flight, the consumer warps copy
//    v0 into the output of every unit absent from the active list.
//  * Every wait is bounded in time; a timeout sets a device error bit and the
//    CTA leaves after its in-flight copies have landed.
#include <climits>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <mutex>

#include "sinkrouter.h"
#include "sr_internal.h"
#include "sr_ptx.cuh"
#include "sr_route_math.cuh"
#include "sr_timeline.cuh"

// Two row blocks of 16 per consumer warp (128-row tiles) in two 64 KB stages:
// the same 128 KB in flight per SM as four 64-row stages, with two independent
// MMA chains per warp. Measured back to back at 128K: 49.6-50.0 us per
// layer-step against 50.7 for RB = 1 with four stages (and 52.4 for RB = 2
// with three stages, 192 KB in flight).
#ifndef SR_DECODE_RB
#define SR_DECODE_RB 2 // row blocks of 16 per consumer warp and tile
#endif
#ifndef SR_DECODE_STAGES
#define SR_DECODE_STAGES 2
#endif

SR_TL_DEFINE(tl_decode)
#ifdef SR_TIMELINE
// latest %globaltimer at which a decode CTA left (atomicMax); the next kernel
// reads it after its dependency wait
static __device__ unsigned long long tl_last_exit;
static __device__ unsigned int tl_decode_launch; // ring of CTA 0's stamps in rows 512 .. 575
extern "C" int sr_timeline_last_exit_addr(void **p) { return (int)cudaGetSymbolAddress(p, tl_last_exit); }
#endif

namespace sr {
namespace {

constexpr int kCWarps = 4;
constexpr int kThreads = 32 * (kCWarps + 1);
constexpr long long kMinChunk = 256;
constexpr uint64_t kWaitLimitNs = 2000000000ull; // 2 s: far above any legitimate wait
constexpr int kFirst = 1, kLast = 2, kEnd = 4;
constexpr float kScaleLog2 = 0.12751743082459868f; // log2(e) / sqrt(128)
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kMergeThreads = 32 * kCWarps;
// Partials in flight per thread in the final merge (at most 32: lane k of a
// warp loads the (m, l) of the batch's k-th partial). Each batch costs one
// round trip for lines other SMs have just written (~0.9 us); 25 covers the 74
// partials of a unit at 512K with 2 of 8 units active in 3 batches, and the 37
// at 128K with 4 active in 2.
constexpr int kMergeBatch = 25;
// Row stride (floats) of the split-end scratch that holds each warp's O per
// head: 4 floats of padding put the lanes that store the same row of
// different head pairs in different banks.
constexpr int kCombStride = 128 + 4;
// Bytes per query head in the shared q buffer: the 256-byte row plus 16 bytes,
// so the lanes that read the same word of different heads hit different banks.
constexpr int kQRowBytes = kHeadDim * 2 + 16;
constexpr unsigned kFull = 0xffffffffu;
constexpr int kFastUnits = 32; // launches with at most this many units plan in registers

struct alignas(16) TileHdr {
    int32_t unit;       // flat unit b*Hkv+g
    int32_t pos0;       // unit-local position of tile row 0
    int32_t nvalid;     // rows of the tile inside the split (0: empty split)
    int32_t flags;      // kFirst | kLast | kEnd
    int32_t slot;       // partial slot of this split
    int32_t nseg;       // splits of this unit
    int32_t slot_first; // slot of the unit's first split (its slots are consecutive)
    int32_t pad;
};

#ifndef SR_DECODE_SEQTAB
#define SR_DECODE_SEQTAB 4096
#endif
constexpr int kSeqTab = SR_DECODE_SEQTAB; // seq_lens entries staged in shared memory

// Launches of at most kFastUnits units: the active entry of rank r, prepared by
// lane r of the producer warp so that the producer lane reads its splits from a
// table instead of deriving them one after another.
struct alignas(16) RankInfo {
    long long start; // prefix of the active lengths before this rank
    int32_t unit;    // flat unit b*Hkv+g
    int32_t len;     // length, clamped to [1, Lmax]
    int32_t qrow;    // first query row of the unit, b*Hq + g*M
    int32_t cf;      // automatic splits: first share overlapping the unit
    int32_t cl;      // automatic splits: last share overlapping the unit
    int32_t pad;
};

struct Misc {
    int abort_flag;
    int is_last;
    int i0;
    int pad;
    long long s0;
    long long wsum[kCWarps + 1];
    int first_bad; // first malformed entry of the active list (INT_MAX: none)
    int first_u;   // unit of the producer's first active entry (-1: none)
    uint8_t sflag[32]; // fused routing of at most 32 units: sink flags
};

struct Params {
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *v0;
    const int32_t *seq_lens;
    const int32_t *active;
    __nv_bfloat16 *out;
    int32_t *err;
    int32_t *cnt;
    float *part_o;
    float2 *part_ml;
    int B, Hq, Hkv, M, Lmax, n_splits;
    // fused routing (sr_route_decode_attention) only
    const __nv_bfloat16 *k0;
    float tau;
    uint8_t *mask_out;   // may be null
    int32_t *active_out; // may be null
    float *lse;          // [B, Hq] natural-log log-sum-exp of the logits; may be null
    float *out_f32;      // when set, the output is written here in fp32 instead of `out`
};

template <int RB, int STAGES> struct Cfg {
    static constexpr int BN = 16 * RB * kCWarps; // positions per tile
    static constexpr int HALF = BN * 128;        // one [BN x 64] bf16 box
    static constexpr int STAGE = 4 * HALF;       // K lo, K hi, V lo, V hi
    static constexpr int QBYTES = kMaxGroup * kQRowBytes;
    static constexpr int OFF_Q = STAGES * STAGE;
    static constexpr int OFF_COMB = OFF_Q + STAGES * QBYTES;
    static constexpr int OFF_ML = OFF_COMB + kCWarps * kMaxGroup * kCombStride * 4;
    static constexpr int OFF_HDR = OFF_ML + kCWarps * kMaxGroup * 8;
    static constexpr int OFF_BAR = OFF_HDR + STAGES * (int)sizeof(TileHdr);
    static constexpr int OFF_MISC = OFF_BAR + (2 * STAGES + 2) * 8;
    static constexpr int OFF_BITMAP = OFF_MISC + 256;
    // seq_lens staged outside the stage buffers: the producer reads it while
    // the copies run
    static constexpr int OFF_SEQ = OFF_BITMAP + SR_MAX_UNITS / 8;
    static constexpr int OFF_RANK = OFF_SEQ + kSeqTab * 4; // RankInfo[32] (launches of <= 32 units)
    static constexpr int BYTES = OFF_RANK + 32 * (int)sizeof(RankInfo);
    static constexpr int ALLOC = BYTES + 1024; // room to align the base to 1024 B
    static_assert(sizeof(Misc) <= 256, "misc block");
    // Prologue tables (active lengths, active units, sink flags) live in the
    // stage buffers before the first copy is issued.
    static_assert(SR_MAX_UNITS * 7 <= STAGES * STAGE, "prologue tables");
    static_assert(BN <= 256, "TMA box rows");
    static_assert(ALLOC <= 227 * 1024, "shared memory per CTA");
};

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int *abort_flag)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity))
            return true;
        if (*abort_flag)
            return false;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            return false;
        }
    }
}

// a / b for 0 <= a, 0 < b: 32-bit division when both fit (every workload here),
// else the 64-bit routine.
__device__ __forceinline__ long long div_nonneg(long long a, long long b)
{
    if (((unsigned long long)a | (unsigned long long)b) <= 0xffffffffull)
        return (long long)((unsigned)a / (unsigned)b);
    return a / b;
}

// Sequence length of unit u, clamped to [1, Lmax] (the prologue reports the
// clamp; every later lookup must give the same value), from the shared table
// when the batch fits it.
__device__ __forceinline__ int unit_len(const Params &p, int u, const int32_t *seqtab)
{
    const int L = seqtab ? seqtab[u / p.Hkv] : __ldg(p.seq_lens + u / p.Hkv);
    return L < 1 ? 1 : (L > p.Lmax ? p.Lmax : L);
}

// Smallest set bit >= from in a bitmap of U bits, or U when there is none.
__device__ __forceinline__ int next_set_bit(const uint32_t *bm, int from, int U)
{
    const int nw = (U + 31) >> 5;
    int w = from >> 5;
    if (from >= U || w >= nw)
        return U;
    uint32_t bits = bm[w] & (0xffffffffu << (from & 31));
    while (!bits) {
        if (++w >= nw)
            return U;
        bits = bm[w];
    }
    const int r = (w << 5) + __ffs(bits) - 1;
    return r < U ? r : U;
}

// Inclusive block-wide prefix of a 64-bit value; *total receives the block sum.
__device__ __forceinline__ long long block_scan(long long x, Misc *misc, long long *total)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    long long v = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o)
            v += y;
    }
    if (lane == 31)
        misc->wsum[warp] = v;
    __syncthreads();
    long long before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < kCWarps + 1; ++w) {
        const long long s = misc->wsum[w];
        before += (w < warp) ? s : 0;
        all += s;
    }
    __syncthreads();
    *total = all;
    return before + v;
}

// Fused routing: every CTA routes every unit itself with the routing kernel's
// arithmetic (sr_route_math.cuh, one warp per GQA group, loads straight from
// global memory), so its decisions equal sr_route's bit for bit; CTA 0 also
// writes the route mask. flag[u] = sink. Called by all threads; no barrier.
template <int M>
__device__ __forceinline__ void route_all_units(const Params &p, int U, uint8_t *flag)
{
    route_units_warp<M, true>(reinterpret_cast<const uint4 *>(p.q), reinterpret_cast<const uint4 *>(p.k0), U, p.tau,
                              (int)threadIdx.x >> 5, kThreads / 32, [&](int u, bool sink) {
                                  flag[u] = sink ? 1 : 0;
                                  if (blockIdx.x == 0 && p.mask_out)
                                      p.mask_out[u] = sink ? 1 : 0;
                              });
}

__device__ __forceinline__ void route_all_units(const Params &p, int U, uint8_t *flag, int M)
{
    switch (M) {
    case 1:
        route_all_units<1>(p, U, flag);
        break;
    case 2:
        route_all_units<2>(p, U, flag);
        break;
    case 4:
        route_all_units<4>(p, U, flag);
        break;
    default:
        route_all_units<8>(p, U, flag);
        break;
    }
}

template <int RB, int STAGES, bool FUSED>
__global__ void __launch_bounds__(kThreads, 1)
decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const Params p)
{
    using C = Cfg<RB, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    TileHdr *hdr = reinterpret_cast<TileHdr *>(smem + C::OFF_HDR);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR); // full[S], empty[S], consumer sync
    Misc *misc = reinterpret_cast<Misc *>(smem + C::OFF_MISC);
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(smem + C::OFF_BITMAP);
    float *comb = reinterpret_cast<float *>(smem + C::OFF_COMB);
    float2 *mlsm = reinterpret_cast<float2 *>(smem + C::OFF_ML);
    volatile int *abort_flag = &misc->abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int U = p.B * p.Hkv;
    const int M = p.M;
    const uint32_t full0 = smem_u32(&bars[0]);
    const uint32_t empty0 = smem_u32(&bars[STAGES]);
    const uint32_t cbar = smem_u32(&bars[2 * STAGES]);

    // ---------------------------------------------------------------- prologue
    if (tid == 0)
        SR_STAMP(tl_decode, 0);
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, kCWarps);
        }
        mbar_init(cbar, kCWarps);
        fence_mbar_init();
        misc->abort_flag = 0;
        misc->is_last = 0;
        misc->i0 = INT_MAX;
        misc->s0 = 0;
        misc->first_bad = INT_MAX;
        misc->first_u = -1;
    }
    if (warp == kCWarps && lane == 0) {
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    for (int w = tid; w < (U + 31) / 32; w += kThreads)
        bitmap[w] = 0;
    __syncthreads();
    // Prologue tables in the stage buffers (free until the first copy),
    // sized by the actual batch and unit count (launches with more than
    // kFastUnits units only).
    const bool seq_smem = p.B <= kSeqTab;
    int32_t *seqtab = reinterpret_cast<int32_t *>(smem + C::OFF_SEQ);
    RankInfo *rtab = reinterpret_cast<RankInfo *>(smem + C::OFF_RANK);
    int32_t *ltab = reinterpret_cast<int32_t *>(smem);
    int16_t *utab = reinterpret_cast<int16_t *>(smem + ((4 * U + 127) & ~127));
    uint8_t *sflag = smem + ((4 * U + 127) & ~127) + ((2 * U + 127) & ~127);
    int errbits = 0;
    int n = 0;
    long long P = 0;
    // Launches with at most 32 units: every warp derives the active set in
    // registers from one round of loads (lane r holds the active entry of rank
    // r, its length and the inclusive prefix of the lengths), so no block
    // barrier follows the dependency wait. The producer warp finds its share
    // with a ballot and issues its first copies at once; the consumer warps do
    // the sink bypass from their own copy of the set.
    const bool fast = U <= kFastUnits;
    uint32_t act_bits = 0;
    int lane_unit = 0, lane_len = 0;
    long long lane_incl = 0;
    long long local = 0;
    if (fast) {
        grid_dependency_wait();
        grid_launch_dependents();
        if (tid == 0)
            SR_STAMP(tl_decode, 1);
#ifdef SR_TIMELINE
        if (tid == 0 && blockIdx.x < SR_TL_CTAS)
            tl_decode[blockIdx.x][15] = *(volatile unsigned long long *)&tl_last_exit;
        if (tid == 0 && blockIdx.x == 0) {
            const unsigned int ring = 512 + atomicAdd(&tl_decode_launch, 1u) % 64u;
            tl_decode[ring][1] = tl_decode[0][1];
            tl_decode[ring][15] = tl_decode[0][15];
        }
#endif
        // All inputs are read after the wait: the preceding kernel may write
        // any of them (the routing kernel the list, the append step seq_lens).
        const int sl = (lane < p.B) ? __ldg(p.seq_lens + lane) : 1;
        if constexpr (!FUSED) {
            n = __ldg(p.active);
            const int e = (lane < U) ? __ldg(p.active + 1 + lane) : -1;
            if (n < 0 || n > U) {
                errbits |= SR_DEVERR_ACTIVE_LIST;
                n = n < 0 ? 0 : U;
            }
            // Keep the longest well-formed prefix (entries in range and
            // strictly ascending); a malformed entry ends it and is reported.
            const int prev = __shfl_up_sync(kFull, e, 1);
            const unsigned bad = __ballot_sync(kFull, lane < n && (e < 0 || e >= U || (lane > 0 && e <= prev)));
            if (bad) {
                errbits |= SR_DEVERR_ACTIVE_LIST;
                n = __ffs(bad) - 1;
            }
            lane_unit = (lane < n) ? e : 0;
            act_bits = __reduce_or_sync(kFull, (lane < n) ? (1u << lane_unit) : 0u);
        } else {
            route_all_units(p, U, misc->sflag, M);
            __syncthreads();
            act_bits = __ballot_sync(kFull, lane < U && !misc->sflag[lane]);
            n = __popc(act_bits);
            const int r = (int)__fns(act_bits, 0, lane + 1); // unit of rank `lane`
            lane_unit = (lane < n && r >= 0 && r < U) ? r : 0;
            if (blockIdx.x == 0 && warp == kCWarps && p.active_out) {
                if (lane < n)
                    p.active_out[1 + lane] = lane_unit;
                if (lane == 0)
                    p.active_out[0] = n;
            }
        }
        int L = __shfl_sync(kFull, sl, lane_unit / p.Hkv);
        if (__ballot_sync(kFull, lane < n && (L < 1 || L > p.Lmax)))
            errbits |= SR_DEVERR_SEQ_LEN;
        L = L < 1 ? 1 : (L > p.Lmax ? p.Lmax : L);
        lane_len = (lane < n) ? L : 0;
        lane_incl = lane_len;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_up_sync(kFull, lane_incl, o);
            if (lane >= o)
                lane_incl += y;
        }
        P = __shfl_sync(kFull, lane_incl, 31);
        if (warp == kCWarps) { // the tables the producer lane walks
            if (lane < p.B)
                seqtab[lane] = sl;
            if (lane == 0)
                bitmap[0] = act_bits;
        }
        if (tid == 0)
            SR_STAMP(tl_decode, 2);
        if (errbits && blockIdx.x == 0 && warp == kCWarps && lane == 0)
            atomicOr(p.err, errbits);
    } else if constexpr (!FUSED) {
        // The preceding kernel may have written every input (the routing
        // kernel writes the active list; the append step also advances
        // seq_lens), so all of them are read after the dependency wait, the
        // length table and the list count in the same round trip.
        grid_dependency_wait();
        grid_launch_dependents();
        if (tid == 0)
            SR_STAMP(tl_decode, 1);
        __syncthreads();

        n = __ldg(p.active);
        if (seq_smem)
            for (int b = tid; b < p.B; b += kThreads)
                seqtab[b] = __ldg(p.seq_lens + b);
        if (n < 0 || n > U) {
            errbits |= SR_DEVERR_ACTIVE_LIST;
            n = n < 0 ? 0 : U;
        }
        // Keep the longest well-formed prefix of the list (indices in range and
        // strictly ascending); a malformed entry ends it and is reported.
        for (int i = tid; i < U; i += kThreads) {
            const int u = __ldg(p.active + 1 + i);
            const int prev = (i > 0) ? __ldg(p.active + i) : -1;
            if (i >= n)
                continue;
            if (u < 0 || u >= U || u <= prev)
                atomicMin(&misc->first_bad, i);
            else
                utab[i] = (int16_t)u;
        }
        __syncthreads();
        if (tid == 0)
            SR_STAMP(tl_decode, 2);
        if (misc->first_bad < n) {
            errbits |= SR_DEVERR_ACTIVE_LIST;
            n = misc->first_bad;
        }
        for (int i = tid; i < n; i += kThreads) {
            const int u = utab[i];
            int L = seq_smem ? seqtab[u / p.Hkv] : __ldg(p.seq_lens + u / p.Hkv);
            if (L < 1 || L > p.Lmax) {
                errbits |= SR_DEVERR_SEQ_LEN;
                L = L < 1 ? 1 : p.Lmax;
            }
            atomicOr(&bitmap[u >> 5], 1u << (u & 31));
            ltab[i] = L;
            local += L;
        }
    } else {
        // Routing inside the kernel: every input may come from the preceding
        // kernel, so everything is read after the dependency wait.
        grid_dependency_wait();
        grid_launch_dependents();
        if (seq_smem)
            for (int b = tid; b < p.B; b += kThreads)
                seqtab[b] = __ldg(p.seq_lens + b);
        route_all_units(p, U, sflag, M);
        __syncthreads();
        // Ordered compaction of the active units into the same tables the
        // work-list path builds.
        for (int c0 = 0; c0 < U; c0 += kThreads) {
            const int u = c0 + tid;
            const bool act = (u < U) && !sflag[u];
            long long tot;
            const long long incl = block_scan(act ? 1 : 0, misc, &tot);
            if (act) {
                const int i = n + (int)incl - 1;
                int L = seq_smem ? seqtab[u / p.Hkv] : __ldg(p.seq_lens + u / p.Hkv);
                if (L < 1 || L > p.Lmax) {
                    errbits |= SR_DEVERR_SEQ_LEN;
                    L = L < 1 ? 1 : p.Lmax;
                }
                atomicOr(&bitmap[u >> 5], 1u << (u & 31));
                ltab[i] = L;
                utab[i] = (int16_t)u;
                local += L;
                if (blockIdx.x == 0 && p.active_out)
                    p.active_out[1 + i] = u;
            }
            n += (int)tot;
        }
        if (blockIdx.x == 0 && tid == 0 && p.active_out)
            p.active_out[0] = n;
    }
    if (!fast) {
        (void)block_scan(local, misc, &P);
        if (errbits && blockIdx.x == 0)
            atomicOr(p.err, errbits);
    }

    const int G = gridDim.x;
    long long chunk = 1, r0 = 0, r1 = 0;
    // The producer lane issued the copies of its first tile before finishing
    // the plan; its first emit only writes the header and arrives.
    bool early = false;
    if (p.n_splits == 0 && P > 0) {
        chunk = div_nonneg(P + G - 1, G);
        chunk = (chunk + C::BN - 1) / C::BN * C::BN;
        chunk = chunk < kMinChunk ? kMinChunk : chunk;
        r0 = (long long)blockIdx.x * chunk;
        r1 = r0 + chunk < P ? r0 + chunk : P;
    }
    if (fast) {
        if (warp == kCWarps) {
            // This CTA's first active entry: the rank whose positions contain
            // r0 (automatic splits), or rank 0 (forced splits).
            int i0 = INT_MAX;
            long long s0 = 0;
            if (p.n_splits != 0) {
                i0 = 0;
            } else if (P > 0 && r0 < P) {
                // never empty: the last valid lane holds the total P > r0
                const unsigned gt = __ballot_sync(kFull, lane < n && lane_incl > r0);
                const int i = gt ? __ffs(gt) - 1 : 0;
                s0 = __shfl_sync(kFull, lane_incl - lane_len, i);
                i0 = gt ? i : INT_MAX;
            }
            const int fu = (i0 < n) ? __shfl_sync(kFull, lane_unit, i0 < 32 ? i0 : 0) : -1;
            const int lb = lane_unit / p.Hkv;
            const int lane_qrow = lb * p.Hq + (lane_unit - lb * p.Hkv) * M;
            const int fq = __shfl_sync(kFull, lane_qrow, i0 < 32 ? i0 : 0);
            if (lane == 0 && p.n_splits == 0 && i0 < n) {
                // The first tile of this CTA's first split (unit fu from
                // position r0 - s0, with the group's q rows) into stage 0 now:
                // its full barrier expects the bytes but cannot complete
                // before the header is written and the producer arrives.
                const uint32_t sb = smem_u32(smem);
                const uint64_t pol0 = l2_policy_evict_first();
                mbar_expect_tx(full0, (uint32_t)C::STAGE + (uint32_t)(M * kHeadDim * 2));
                const int pos0 = (int)(r0 - s0);
                tma_load_3d(sb, &tmK, full0, 0, pos0, fu, pol0);
                tma_load_3d(sb + C::HALF, &tmK, full0, 64, pos0, fu, pol0);
                tma_load_3d(sb + 2 * C::HALF, &tmV, full0, 0, pos0, fu, pol0);
                tma_load_3d(sb + 3 * C::HALF, &tmV, full0, 64, pos0, fu, pol0);
                const uint8_t *qsrc = reinterpret_cast<const uint8_t *>(p.q + (size_t)fq * kHeadDim);
                for (int hq = 0; hq < M; ++hq)
                    bulk_load(smem_u32(smem + C::OFF_Q + hq * kQRowBytes), qsrc + hq * kHeadDim * 2, kHeadDim * 2,
                              full0);
                SR_STAMP(tl_decode, 4);
                early = true;
            }
            if (lane == 0) {
                misc->i0 = i0;
                misc->s0 = s0;
                misc->first_u = fu;
            }
            if (lane < n) {
                RankInfo ri;
                ri.start = lane_incl - lane_len;
                ri.unit = lane_unit;
                ri.len = lane_len;
                ri.qrow = lane_qrow;
                ri.cf = (p.n_splits == 0) ? (int)div_nonneg(ri.start, chunk) : 0;
                ri.cl = (p.n_splits == 0) ? (int)div_nonneg(ri.start + lane_len - 1, chunk) : 0;
                ri.pad = 0;
                rtab[lane] = ri;
            }
            __syncwarp();
        }
    } else {
        if (p.n_splits == 0 && P > 0 && r0 < P) { // find the active entry whose positions contain r0
            long long carry = 0;
            for (int base = 0; base < n; base += kThreads) {
                const int i = base + tid;
                const int L = (i < n) ? ltab[i] : 0;
                long long tot;
                const long long incl = block_scan(L, misc, &tot);
                const long long S = carry + incl - L;
                if (i < n && L > 0 && S <= r0 && r0 < S + L) {
                    misc->i0 = i;
                    misc->s0 = S;
                }
                carry += tot;
            }
        }
        // Generic stores into the stage buffers (tables) must be ordered
        // before the TMA writes that will reuse those bytes.
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            // The producer walks the active units in the bitmap from its first
            // entry on (rank i0 for automatic splits, rank 0 for forced ones).
            const int i0 = (p.n_splits == 0) ? misc->i0 : 0;
            misc->i0 = i0;
            misc->first_u = (i0 < n) ? (int)utab[i0] : -1;
        }
        __syncthreads(); // the stage buffers are free for the copies from here on
    }
    if (fast ? tid == 32 * kCWarps : tid == 0)
        SR_STAMP(tl_decode, 3);

    // ---------------------------------------------------------------- producer
    if (warp == kCWarps) {
        if (lane != 0)
            return;
        const uint64_t pol = l2_policy_evict_first();
        SR_STAMP(tl_decode, 16);
        int stage = 0;
        uint32_t ph = 0;
        int issued_parity[STAGES];
#pragma unroll
        for (int s = 0; s < STAGES; ++s)
            issued_parity[s] = -1;
        if (early)
            issued_parity[0] = 0; // the first tile's copies are in flight
        bool ok = true;

        auto emit = [&](const TileHdr &h, const void *qsrc, uint32_t qbytes) -> bool {
#ifdef SR_TIMELINE
            const bool tl_first = issued_parity[stage] < 0 && stage == 0 && ph == 0;
            if (tl_first)
                SR_STAMP(tl_decode, 17);
#endif
            if (!wait_bar(empty0 + 8 * stage, ph ^ 1, abort_flag))
                return false;
#ifdef SR_TIMELINE
            if (tl_first)
                SR_STAMP(tl_decode, 18);
#endif
            hdr[stage] = h;
            const uint32_t fb = full0 + 8 * stage;
            if (early) {
                // this tile's copies were issued in the prologue (same unit,
                // position and q rows): publish the header and arrive
                early = false;
                mbar_arrive(fb);
                if (++stage == STAGES) {
                    stage = 0;
                    ph ^= 1;
                }
                return true;
            }
            const uint32_t bytes = (h.nvalid > 0 ? (uint32_t)C::STAGE : 0u) + qbytes;
            if (bytes) {
                mbar_arrive_expect_tx(fb, bytes);
                if (h.nvalid > 0) {
                    const uint32_t sb = smem_u32(smem + stage * C::STAGE);
#ifdef SR_TIMELINE
                    if (tl_first)
                        SR_STAMP(tl_decode, 19);
#endif
                    tma_load_3d(sb, &tmK, fb, 0, h.pos0, h.unit, pol);
                    tma_load_3d(sb + C::HALF, &tmK, fb, 64, h.pos0, h.unit, pol);
                    tma_load_3d(sb + 2 * C::HALF, &tmV, fb, 0, h.pos0, h.unit, pol);
                    tma_load_3d(sb + 3 * C::HALF, &tmV, fb, 64, h.pos0, h.unit, pol);
                }
                // the group's q rows, one copy per head into the padded rows
                if (qbytes)
                    for (int hq = 0; hq < M; ++hq)
                        bulk_load(smem_u32(smem + C::OFF_Q + stage * C::QBYTES + hq * kQRowBytes),
                                  static_cast<const uint8_t *>(qsrc) + hq * kHeadDim * 2, kHeadDim * 2, fb);
                if (issued_parity[stage] < 0 && stage == 0 && ph == 0)
                    SR_STAMP(tl_decode, 4);
                issued_parity[stage] = (int)ph;
            } else {
                mbar_arrive(fb);
            }
            if (++stage == STAGES) {
                stage = 0;
                ph ^= 1;
            }
            return true;
        };

        auto emit_split = [&](int u, int qrow, long long b0, long long e0, int slot, int nseg,
                              int slot_first) -> bool {
            const long long len = e0 - b0;
            const long long ntiles = len > 0 ? (len + C::BN - 1) / C::BN : 1;
            const __nv_bfloat16 *qsrc = p.q + (size_t)qrow * kHeadDim;
#ifdef SR_TIMELINE
            if (issued_parity[0] < 0)
                SR_STAMP(tl_decode, 21);
#endif
            for (long long t = 0; t < ntiles; ++t) {
                TileHdr h;
                h.unit = u;
                h.pos0 = (int)(b0 + t * C::BN);
                const long long rem = e0 - h.pos0;
                h.nvalid = len > 0 ? (int)(rem < C::BN ? rem : C::BN) : 0;
                h.flags = (t == 0 ? kFirst : 0) | (t == ntiles - 1 ? kLast : 0);
                h.slot = slot;
                h.nseg = nseg;
                h.slot_first = slot_first;
                h.pad = 0;
                const uint32_t qb = (t == 0 && len > 0) ? (uint32_t)(M * kHeadDim * 2) : 0u;
                if (!emit(h, qsrc, qb))
                    return false;
            }
            return true;
        };

        // Active entry of rank i, for non-decreasing i: ranks follow the set
        // bits of the bitmap in ascending unit order, starting at first_u.
        int wi = misc->i0, wu = misc->first_u;
        SR_STAMP(tl_decode, 22);
        auto unit_at = [&](int i) -> int {
            while (wi < i && wu < U) {
                wu = next_set_bit(bitmap, wu + 1, U);
                ++wi;
            }
            return wu;
        };
        // Active entry of rank i (non-decreasing i) whose positions start at S:
        // from the rank table when the launch has at most kFastUnits units,
        // else from the bitmap walk and the length table. u < 0 ends the walk.
        struct Rank {
            int u, L, qrow;
            long long cf, cl;
        };
        auto rank_at = [&](int i, long long S) -> Rank {
            Rank r;
            if (fast) {
                const RankInfo ri = rtab[i];
                r.u = ri.unit;
                r.L = ri.len;
                r.qrow = ri.qrow;
                r.cf = ri.cf;
                r.cl = ri.cl;
                return r;
            }
            r.u = unit_at(i);
            if (r.u < 0 || r.u >= U) {
                r.u = -1;
                return r;
            }
            r.L = unit_len(p, r.u, seq_smem ? seqtab : nullptr);
            const int b = r.u / p.Hkv;
            r.qrow = b * p.Hq + (r.u - b * p.Hkv) * M;
            if (p.n_splits == 0) {
                r.cf = div_nonneg(S, chunk);
                r.cl = div_nonneg(S + r.L - 1, chunk);
            }
            return r;
        };
        if (p.n_splits == 0) {
            if (P > 0 && r0 < P) {
                int i = misc->i0;
                long long S = misc->s0;
                while (ok && i < n && S < r1) {
                    const Rank r = rank_at(i, S);
                    if (r.u < 0)
                        break;
                    const long long b0 = (r0 > S ? r0 : S) - S;
                    const long long e0 = (r1 < S + r.L ? r1 : S + r.L) - S;
#ifdef SR_TIMELINE
                    if (i == misc->i0)
                        SR_STAMP(tl_decode, 20);
#endif
                    ok = emit_split(r.u, r.qrow, b0, e0, (int)blockIdx.x + i, (int)(r.cl - r.cf + 1), (int)r.cf + i);
                    S += r.L;
                    ++i;
                }
            }
        } else {
            const int ns = p.n_splits;
            for (long long j = blockIdx.x; ok && j < (long long)n * ns; j += G) {
                const int i = (int)div_nonneg(j, ns), s = (int)(j - (long long)i * ns);
                const Rank r = rank_at(i, 0);
                if (r.u < 0)
                    break;
                const long long b0 = (long long)s * r.L / ns, e0 = (long long)(s + 1) * r.L / ns;
                ok = emit_split(r.u, r.qrow, b0, e0, (int)j, ns, i * ns);
            }
        }
        if (ok) {
            TileHdr h{};
            h.unit = -1;
            h.flags = kEnd;
            ok = emit(h, nullptr, 0);
            SR_STAMP(tl_decode, 14);
        }
        if (!ok) {
            atomicOr(p.err, SR_DEVERR_TIMEOUT);
            if (early) // its phase completes only once the producer has arrived
                mbar_arrive(full0);
            // Let every copy still in flight land before this CTA can exit.
            volatile int never = 0;
            for (int s = 0; s < STAGES; ++s)
                if (issued_parity[s] >= 0)
                    (void)wait_bar(full0 + 8 * s, (uint32_t)issued_parity[s], &never);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int w = warp;
    const int g = lane >> 2, t = lane & 3;
    const int mi = lane >> 3, ri = lane & 7;
    const int ctid = tid; // 0 .. 32*kCWarps-1

    // Sink bypass: out[b, h] = v0[b, g] for every unit not in the active list.
    {
        const int gw = blockIdx.x * kCWarps + w, nw = gridDim.x * kCWarps;
        for (int u = gw; u < U; u += nw) {
            if (fast ? ((act_bits >> u) & 1u) : (bitmap[u >> 5] & (1u << (u & 31))))
                continue;
            const int b = u / p.Hkv, gg = u - b * p.Hkv;
            const size_t row0 = (size_t)b * p.Hq + (size_t)gg * M;
            if (p.out_f32) {
                // fp32 copy of v0 (exact): lane c4 widens elements 4 c4 .. 4 c4 + 3
                const uint2 v = __ldg(reinterpret_cast<const uint2 *>(p.v0 + (size_t)u * kHeadDim) + lane);
                const float4 f = make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                                             __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
                for (int hh = 0; hh < M; ++hh)
                    reinterpret_cast<float4 *>(p.out_f32 + (row0 + hh) * kHeadDim)[lane] = f;
            } else {
                const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p.v0 + (size_t)u * kHeadDim) + (lane & 15));
                for (int e = lane; e < M * 16; e += 32) {
                    uint4 *dst = reinterpret_cast<uint4 *>(p.out + (row0 + (e >> 4)) * kHeadDim);
                    dst[e & 15] = v;
                }
            }
            if (p.lse && lane < M) // no attention was computed for a sink head
                p.lse[(size_t)b * p.Hq + (size_t)gg * M + lane] = __int_as_float(0x7fc00000);
        }
    }

    if (ctid == 0)
        SR_STAMP(tl_decode, 5);
    const uint32_t sbase = smem_u32(smem);
    uint32_t rowK[RB], rowV[RB];
#pragma unroll
    for (int rb = 0; rb < RB; ++rb) {
        const int r = (w * RB + rb) * 16;
        rowK[rb] = (uint32_t)(r + ri + 8 * (mi & 1)) * 128u;
        rowV[rb] = (uint32_t)(r + ri + 8 * (mi >> 1)) * 128u;
    }
    const int my_row0 = w * RB * 16;

    float o[8][4];
    float mrun[2], lrun[2];
    uint32_t qf[8][2];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
        qf[j][0] = qf[j][1] = 0u;
    }
    mrun[0] = mrun[1] = -INFINITY;
    lrun[0] = lrun[1] = 0.f;

    int stage = 0;
    uint32_t ph = 0, cph = 0;
    bool ok = true;

    // Final output of one float4 column: acc * inv, in bf16 (round to nearest
    // even of the same fp32 products) or, for partial outputs, in fp32.
    auto store_out = [&](int b, int gg, int head, int d4, const float4 &acc, float inv) {
        const size_t off = ((size_t)b * p.Hq + (size_t)gg * M + head) * kHeadDim + d4;
        const float4 r = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        if (p.out_f32) {
            *reinterpret_cast<float4 *>(p.out_f32 + off) = r;
        } else {
            uint2 packed;
            packed.x = pack_bf16x2(r.x, r.y);
            packed.y = pack_bf16x2(r.z, r.w);
            *reinterpret_cast<uint2 *>(p.out + off) = packed;
        }
    };

    auto cbar_sync = [&]() -> bool {
        __syncwarp();
        if (lane == 0)
            mbar_arrive(cbar);
        bool r = wait_bar(cbar, cph, abort_flag);
        cph ^= 1;
        return __all_sync(0xffffffffu, r);
    };

#ifdef SR_TIMELINE
    bool tl_first = true;
    int tl_splits = 0, tl_last = 0;
#endif
    for (;;) {
        if (!__all_sync(0xffffffffu, wait_bar(full0 + 8 * stage, ph, abort_flag))) {
            ok = false;
            break;
        }
#ifdef SR_TIMELINE
        if (tl_first && ctid == 0)
            SR_STAMP(tl_decode, 6);
        tl_first = false;
#endif
        const TileHdr h = hdr[stage];
        if (h.flags & kEnd)
            break;
        const uint32_t st = sbase + stage * C::STAGE;
        if (h.flags & kFirst) {
            // (m, l, O) are at their initial values here: the kernel starts
            // with them and every split's last tile resets them.
            if (h.nvalid > 0) {
                const uint32_t *qs = reinterpret_cast<const uint32_t *>(smem + C::OFF_Q + stage * C::QBYTES);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    qf[ks][0] = (g < M) ? qs[g * (kQRowBytes / 4) + ks * 8 + t] : 0u;
                    qf[ks][1] = (g < M) ? qs[g * (kQRowBytes / 4) + ks * 8 + 4 + t] : 0u;
                }
            }
        }

        if (h.nvalid > my_row0) {
            if (h.nvalid < my_row0 + RB * 16) {
                // Rows past the split may be padding (even NaN): zero this
                // warp's V rows there so that P = 0 contributes exactly 0.
                const int z0 = h.nvalid, nz = my_row0 + RB * 16 - z0;
                for (int e = lane; e < nz * 16; e += 32) {
                    const int row = z0 + (e >> 4), c = e & 15;
                    uint4 *dst = reinterpret_cast<uint4 *>(smem + stage * C::STAGE + (2 + (c >> 3)) * C::HALF +
                                                           row * 128 + (c & 7) * 16);
                    *dst = make_uint4(0u, 0u, 0u, 0u);
                }
                fence_proxy_async_smem();
                __syncwarp();
            }

            // S^T[16 rows x 8 heads] per row block, two accumulators per block.
            float sacc[RB][4];
            {
                float sa[RB][4], sb[RB][4];
#pragma unroll
                for (int rb = 0; rb < RB; ++rb)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        sa[rb][e] = sb[rb][e] = 0.f;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t kb = st + (uint32_t)(ks >> 2) * C::HALF;
                    const uint32_t cx = (uint32_t)(((ks & 3) * 2 + (mi >> 1)) ^ ri) << 4;
#pragma unroll
                    for (int rb = 0; rb < RB; ++rb) {
                        uint32_t a[4];
                        ldmatrix_x4(a, kb + rowK[rb] + cx);
                        if (ks & 1)
                            mma_bf16_16816(sb[rb], a, qf[ks][0], qf[ks][1]);
                        else
                            mma_bf16_16816(sa[rb], a, qf[ks][0], qf[ks][1]);
                    }
                }
#pragma unroll
                for (int rb = 0; rb < RB; ++rb)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int row = my_row0 + rb * 16 + g + (e >> 1) * 8;
                        sacc[rb][e] = (row < h.nvalid) ? (sa[rb][e] + sb[rb][e]) * kScaleLog2 : -INFINITY;
                    }
            }

            // Online softmax (log2 domain); lane holds heads 2t and 2t+1.
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int rb = 0; rb < RB; ++rb) {
                mx0 = fmaxf(mx0, fmaxf(sacc[rb][0], sacc[rb][2]));
                mx1 = fmaxf(mx1, fmaxf(sacc[rb][1], sacc[rb][3]));
            }
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
            }
            const float mn0 = fmaxf(mrun[0], mx0), mn1 = fmaxf(mrun[1], mx1);
            const float mu0 = (mn0 == -INFINITY) ? 0.f : mn0;
            const float mu1 = (mn1 == -INFINITY) ? 0.f : mn1;
            const float al0 = exp2f(mrun[0] - mu0), al1 = exp2f(mrun[1] - mu1);
            mrun[0] = mn0;
            mrun[1] = mn1;
            float ps0 = 0.f, ps1 = 0.f;
            uint32_t pf[RB][2];
#pragma unroll
            for (int rb = 0; rb < RB; ++rb) {
                const float p0 = exp2f(sacc[rb][0] - mu0), p1 = exp2f(sacc[rb][1] - mu1);
                const float p2 = exp2f(sacc[rb][2] - mu0), p3 = exp2f(sacc[rb][3] - mu1);
                ps0 += p0 + p2;
                ps1 += p1 + p3;
                pf[rb][0] = movmatrix_trans(pack_bf16x2(p0, p1));
                pf[rb][1] = movmatrix_trans(pack_bf16x2(p2, p3));
            }
            lrun[0] = lrun[0] * al0 + ps0;
            lrun[1] = lrun[1] * al1 + ps1;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                o[j][0] *= al0;
                o[j][1] *= al1;
                o[j][2] *= al0;
                o[j][3] *= al1;
            }

            // O^T[128 x 8 heads] += V^T * P^T, 16 head-dim rows per MMA.
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t vb = st + (uint32_t)(2 + (j >> 2)) * C::HALF;
                const uint32_t cx = (uint32_t)(((j & 3) * 2 + (mi & 1)) ^ ri) << 4;
#pragma unroll
                for (int rb = 0; rb < RB; ++rb) {
                    uint32_t a[4];
                    ldmatrix_x4_trans(a, vb + rowV[rb] + cx);
                    mma_bf16_16816(o[j], a, pf[rb][0], pf[rb][1]);
                }
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(empty0 + 8 * stage);

        if (h.flags & kLast) {
#ifdef SR_TIMELINE
            if (ctid == 0)
                SR_STAMP(tl_decode, 7);
            ++tl_splits;
#endif
            // ---- merge the four warps' states into one partial of this split
            float l0 = lrun[0], l1 = lrun[1];
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                l0 += __shfl_xor_sync(0xffffffffu, l0, off);
                l1 += __shfl_xor_sync(0xffffffffu, l1, off);
            }
            if (g == 0) {
                mlsm[w * kMaxGroup + 2 * t] = make_float2(mrun[0], l0);
                mlsm[w * kMaxGroup + 2 * t + 1] = make_float2(mrun[1], l1);
            }
            // Unscaled O of this warp; the readers below weight the four warps.
            float *cw = comb + w * (kMaxGroup * kCombStride);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int d0 = 16 * j + g;
                if (2 * t < M) {
                    cw[(2 * t) * kCombStride + d0] = o[j][0];
                    cw[(2 * t) * kCombStride + d0 + 8] = o[j][2];
                }
                if (2 * t + 1 < M) {
                    cw[(2 * t + 1) * kCombStride + d0] = o[j][1];
                    cw[(2 * t + 1) * kCombStride + d0 + 8] = o[j][3];
                }
            }
            if (!(ok = cbar_sync()))
                break;
            // Partial of the split, one float4 column per thread: the warps'
            // states weighted by 2^(m_w - max_w m_w) (0 for a warp that saw no
            // row of this split).
            float *po = p.part_o + (size_t)h.slot * M * kHeadDim;
            for (int idx = ctid; idx < M * 32; idx += 32 * kCWarps) {
                const int head = idx >> 5, d4 = (idx & 31) * 4;
                float2 ml[kCWarps];
                float Mh = -INFINITY;
#pragma unroll
                for (int ww = 0; ww < kCWarps; ++ww) {
                    ml[ww] = mlsm[ww * kMaxGroup + head];
                    Mh = fmaxf(Mh, ml[ww].x);
                }
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                float Lh = 0.f;
#pragma unroll
                for (int ww = 0; ww < kCWarps; ++ww) {
                    const float f = (ml[ww].x == -INFINITY) ? 0.f : exp2f(ml[ww].x - Mh);
                    const float4 x =
                        *reinterpret_cast<const float4 *>(comb + ww * (kMaxGroup * kCombStride) + head * kCombStride + d4);
                    acc.x = fmaf(x.x, f, acc.x);
                    acc.y = fmaf(x.y, f, acc.y);
                    acc.z = fmaf(x.z, f, acc.z);
                    acc.w = fmaf(x.w, f, acc.w);
                    Lh = fmaf(ml[ww].y, f, Lh);
                }
                __stcg(reinterpret_cast<float4 *>(po + head * kHeadDim + d4), acc);
                if (d4 == 0)
                    __stcg(p.part_ml + (size_t)h.slot * M + head, make_float2(Mh, Lh));
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
                o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
            mrun[0] = mrun[1] = -INFINITY;
            lrun[0] = lrun[1] = 0.f;
            // Publish the partial: the consumer barrier orders every thread's
            // stores before thread 0's gpu-scope release, which the last
            // arriving CTA's acquire (the same atomic) pairs with; its own
            // barrier then orders the acquire before every thread's merge
            // loads. No separate fences.
            if (!(ok = cbar_sync()))
                break;
            if (ctid == 0)
                SR_STAMP(tl_decode, 8);
            if (ctid == 0)
                misc->is_last = (atom_add_acq_rel_gpu(p.cnt + h.unit, 1) == h.nseg - 1) ? 1 : 0;
            if (!(ok = cbar_sync()))
                break;
            if (ctid == 0)
                SR_STAMP(tl_decode, 9);
            if (misc->is_last) {
                // ---- last split of the unit to finish: merge all its partials.
                // Threads own float4 columns of the unit's [M x 128] output;
                // when M < 4 the threads also split the partials into groups.
                // Each thread keeps kMergeBatch partials in flight; the merge
                // order is fixed, so the result does not depend on which CTA
                // finished last.
                const int b = h.unit / p.Hkv, gg = h.unit - b * p.Hkv;
                const int ncol = M * 32;
                const int cpg = ncol < kMergeThreads ? ncol : kMergeThreads;
                const int sgrp = kMergeThreads / cpg;
                const int grp = ctid / cpg;
                for (int col = ctid % cpg; col < ncol; col += cpg) {
                    const int head = col >> 5, d4 = (col & 31) * 4;
                    float m = -INFINITY, l = 0.f;
                    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                    // All lanes of a warp share the head and the partial group:
                    // lane k loads the (m, l) of the batch's k-th partial and
                    // the weights reach the other lanes by shuffles, so only
                    // the O values take registers in every lane.
                    for (int j0 = grp; j0 < h.nseg; j0 += sgrp * kMergeBatch) {
                        const int jl = j0 + lane * sgrp;
                        float2 xl = make_float2(-INFINITY, 0.f);
                        if (lane < kMergeBatch && jl < h.nseg)
                            xl = __ldcg(p.part_ml + (size_t)(h.slot_first + jl) * M + head);
                        float4 y[kMergeBatch];
#pragma unroll
                        for (int k = 0; k < kMergeBatch; ++k) {
                            const int j = j0 + k * sgrp;
                            y[k] = (j < h.nseg) ? __ldcg(reinterpret_cast<const float4 *>(
                                                      p.part_o + ((size_t)(h.slot_first + j) * M + head) * kHeadDim + d4))
                                                : make_float4(0.f, 0.f, 0.f, 0.f);
                        }
                        float mb = xl.x;
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1)
                            mb = fmaxf(mb, __shfl_xor_sync(kFull, mb, off));
                        const float mn = fmaxf(m, mb);
                        if (mn != -INFINITY) {
                            const float a = exp2f(m - mn);
                            const float cw = (xl.x == -INFINITY) ? 0.f : exp2f(xl.x - mn);
                            float ls = xl.y * cw;
#pragma unroll
                            for (int off = 16; off > 0; off >>= 1)
                                ls += __shfl_xor_sync(kFull, ls, off);
                            l = l * a + ls;
                            acc.x *= a, acc.y *= a, acc.z *= a, acc.w *= a;
#pragma unroll
                            for (int k = 0; k < kMergeBatch; ++k) {
                                const float c = __shfl_sync(kFull, cw, k);
                                acc.x += y[k].x * c;
                                acc.y += y[k].y * c;
                                acc.z += y[k].z * c;
                                acc.w += y[k].w * c;
                            }
                            m = mn;
                        }
                    }
                    if (sgrp == 1) {
                        if (p.lse && d4 == 0)
                            p.lse[(size_t)b * p.Hq + (size_t)gg * M + head] = (m + log2f(l)) * kLn2;
                        store_out(b, gg, head, d4, acc, 1.f / l);
                    } else {
                        *reinterpret_cast<float4 *>(comb + 4 * ctid) = acc;
                        *reinterpret_cast<float2 *>(comb + 4 * kMergeThreads + 2 * ctid) = make_float2(m, l);
                    }
                }
                if (sgrp > 1) {
                    if (!(ok = cbar_sync()))
                        break;
                    if (ctid < cpg) {
                        const int head = ctid >> 5, d4 = (ctid & 31) * 4;
                        float m = -INFINITY;
                        for (int q = 0; q < sgrp; ++q)
                            m = fmaxf(m, comb[4 * kMergeThreads + 2 * (q * cpg + ctid)]);
                        float l = 0.f;
                        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                        for (int q = 0; q < sgrp; ++q) {
                            const int e = q * cpg + ctid;
                            const float2 ml = *reinterpret_cast<const float2 *>(comb + 4 * kMergeThreads + 2 * e);
                            if (ml.x == -INFINITY)
                                continue;
                            const float c = exp2f(ml.x - m);
                            const float4 y = *reinterpret_cast<const float4 *>(comb + 4 * e);
                            l += ml.y * c;
                            acc.x += y.x * c, acc.y += y.y * c, acc.z += y.z * c, acc.w += y.w * c;
                        }
                        if (p.lse && d4 == 0)
                            p.lse[(size_t)b * p.Hq + (size_t)gg * M + head] = (m + log2f(l)) * kLn2;
                        store_out(b, gg, head, d4, acc, 1.f / l);
                    }
                }
                if (ctid == 0)
                    p.cnt[h.unit] = 0;
                // Shared scratch (comb, mlsm) is reused by the next split's end.
                if (!(ok = cbar_sync()))
                    break;
#ifdef SR_TIMELINE
                if (ctid == 0)
                    SR_STAMP(tl_decode, 10);
                ++tl_last;
#endif
            }
        }
        if (++stage == STAGES) {
            stage = 0;
            ph ^= 1;
        }
    }
    if (!ok && lane == 0)
        atomicOr(p.err, SR_DEVERR_TIMEOUT);
#ifdef SR_TIMELINE
    if (ctid == 0) {
        unsigned long long t_;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));
        atomicMax(&tl_last_exit, t_);
        SR_STAMP(tl_decode, 11);
        tl_decode[blockIdx.x][12] = (unsigned long long)tl_splits;
        tl_decode[blockIdx.x][13] = (unsigned long long)tl_last;
    }
#endif
}

// ---- host side ------------------------------------------------------------------------

using KernelFn = void (*)(const CUtensorMap, const CUtensorMap, const Params);

struct DeviceInfo {
    int sms = 0;
    int grid = 0;
    bool configured = false;
};

constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 3-D view [units][Lmax][128] of a bf16 cache; a box is 64 columns (128 bytes,
// swizzled 128B) by `rows` positions of one unit. Rows past Lmax read as zero.
bool make_cache_map(CUtensorMap *map, const void *base, int units, int lmax, int rows)
{
    auto fn = encode_fn();
    if (!fn)
        return false;
    cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)lmax, (cuuint64_t)units};
    cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)lmax * kHeadDim * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

using DecodeCfg = Cfg<SR_DECODE_RB, SR_DECODE_STAGES>;

cudaError_t configure(int dev, DeviceInfo &info)
{
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (info.configured)
        return cudaSuccess;
    cudaError_t e = cudaDeviceGetAttribute(&info.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return e;
    KernelFn k = decode_kernel<SR_DECODE_RB, SR_DECODE_STAGES, false>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, DecodeCfg::ALLOC);
    if (e != cudaSuccess)
        return e;
    e = cudaFuncSetAttribute(decode_kernel<SR_DECODE_RB, SR_DECODE_STAGES, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, DecodeCfg::ALLOC);
    if (e != cudaSuccess)
        return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kThreads, DecodeCfg::ALLOC);
    if (e != cudaSuccess)
        return e;
    if (per_sm < 1)
        return cudaErrorInvalidConfiguration;
    info.grid = info.sms * per_sm;
    if (info.grid > kAutoGridCap)
        info.grid = kAutoGridCap;
    info.configured = true;
    return cudaSuccess;
}

cudaError_t device_info(DeviceInfo **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    e = configure(dev, g_dev[dev]);
    *out = &g_dev[dev];
    return e;
}

} // namespace

int decode_grid_size()
{
    DeviceInfo *info = nullptr;
    if (device_info(&info) != cudaSuccess)
        return 0;
    return info->grid;
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream)
{
    DeviceInfo *info = nullptr;
    cudaError_t e = device_info(&info);
    if (e != cudaSuccess)
        return e;
    const int U = a.batch * a.n_kv_heads;
    CUtensorMap tmK, tmV;
    if (!make_cache_map(&tmK, a.k_cache, U, a.max_seq_len, DecodeCfg::BN) ||
        !make_cache_map(&tmV, a.v_cache, U, a.max_seq_len, DecodeCfg::BN))
        return cudaErrorInvalidValue;
    uint8_t *ws = static_cast<uint8_t *>(a.workspace);
    Params p;
    p.q = static_cast<const __nv_bfloat16 *>(a.q);
    p.v0 = static_cast<const __nv_bfloat16 *>(a.v0);
    p.seq_lens = a.seq_lens;
    p.active = a.active_list;
    p.out = static_cast<__nv_bfloat16 *>(a.out);
    p.err = reinterpret_cast<int32_t *>(ws + a.ws.err_off);
    p.cnt = reinterpret_cast<int32_t *>(ws + a.ws.cnt_off);
    p.part_o = reinterpret_cast<float *>(ws + a.ws.part_o_off);
    p.part_ml = reinterpret_cast<float2 *>(ws + a.ws.part_ml_off);
    p.B = a.batch;
    p.Hq = a.n_q_heads;
    p.Hkv = a.n_kv_heads;
    p.M = a.n_q_heads / a.n_kv_heads;
    p.Lmax = a.max_seq_len;
    p.n_splits = a.n_splits;
    p.k0 = static_cast<const __nv_bfloat16 *>(a.k0);
    p.tau = a.tau;
    p.mask_out = a.mask_out;
    p.active_out = a.active_out;
    p.lse = a.lse;
    p.out_f32 = a.out_f32;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(info->grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = DecodeCfg::ALLOC;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (a.fused)
        e = cudaLaunchKernelEx(&cfg, decode_kernel<SR_DECODE_RB, SR_DECODE_STAGES, true>, tmK, tmV, p);
    else
        e = cudaLaunchKernelEx(&cfg, decode_kernel<SR_DECODE_RB, SR_DECODE_STAGES, false>, tmK, tmV, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}

} // namespace sr
