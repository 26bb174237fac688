// The step just before the cache scan, in one launch: rotary position
// embedding of the query heads and of the new key, the append of the new key /
// value at each sequence's next slot, the position-0 capture that prefill
// leaves for routing, the routing decision and the ordered active list, and the
// length update.
//
// Method: SinkRouter README (github.com/streamer-AP/SinkRouter), decode-time
// procedure list -- routing compares the RoPE'd query with the cached
// position-0 key (recorded when the first token is written) and the new
// token's key and value join the cache before the scan. The rotation is the
// rotate-half form (element i pairs with element i + 64 of a 128-wide head)
// driven by caller-supplied cos / sin tables, so no frequency schedule is
// built in.
//
// Exactness: each rotated element is a*c - b*s (or b*c + a*s) with a, b bf16
// and c, s fp32, so both products are exact in fp64 and one fp64 rounding of
// their sum is the only error before the narrowing. The narrowing to bf16
// rounds to odd into fp32 and then to nearest-even into bf16, which equals a
// single round-to-nearest-even of the fp64 value (Boldo and Melquiond, rounding
// to odd: an intermediate with at least two more bits than the target, at every
// exponent, makes the double rounding innocuous; fp32 has sixteen more than
// bf16). The result is the correctly rounded bf16 of the fp64 rotation.
//
// Layout: one CTA of 512 threads walking the units in chunks whose rows fit in
// shared memory. Per chunk, in one pass where each thread takes its own item:
// eight threads per new key rotate it (each takes 8 elements and their 8
// partners), write the cache slot, and stage the group's position-0 key (the
// captured one at slot 0, else the stored k0); eight threads per query row
// rotate it into q_out and the staged rows; the staged rows are routed with the routing kernel's own
// routine (one warp per GQA group), so the decision equals sr_route on
// (q_out, k0) bit for bit. Lengths advance after every read of
// them; the compaction is the routing kernel's.
#include <atomic>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sinkrouter.h"
#include "sr_internal.h"
#include "sr_ptx.cuh"
#include "sr_route_math.cuh"

namespace sr {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kRowBudget = 160 * 1024; // shared bytes for staged q / k0 rows

template <int M> __host__ __device__ constexpr int chunk_units() { return kRowBudget / ((M + 1) * 256); }

struct PrestepParams {
    const __nv_bfloat16 *q_in, *k_new, *v_new;
    const float *rope_cos, *rope_sin;
    int32_t *seq_lens;
    __nv_bfloat16 *k_cache, *v_cache, *k0, *v0, *q_out;
    uint8_t *mask;
    int32_t *active;
    int32_t *error;
    float tau;
    int B, Hkv, Lmax, max_pos;
};

// Correctly rounded fp64 -> bf16 (nearest, ties to even) through round-to-odd
// into fp32: truncate, and if the truncation was inexact force the last fp32
// bit to 1; the fp32 -> bf16 step then rounds to nearest even.
__device__ __forceinline__ uint32_t bf16_bits_rn(double x)
{
    float f = __double2float_rz(x);
    if ((double)f != x)
        f = __uint_as_float(__float_as_uint(f) | 1u);
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ double bf16_lo(uint32_t w) { return (double)__uint_as_float(w << 16); }
__device__ __forceinline__ double bf16_hi(uint32_t w) { return (double)__uint_as_float(w & 0xffff0000u); }

// Rotate 8 elements x_lo (positions 8j .. 8j+7) against their partners x_hi
// (positions 64+8j ..) with c, s the table entries for those 8 pairs:
//   lo' = lo c - hi s,  hi' = hi c + lo s.
__device__ __forceinline__ void rope8(uint4 x_lo, uint4 x_hi, const float4 (&c)[2], const float4 (&s)[2], uint4 &o_lo,
                                      uint4 &o_hi)
{
    const uint32_t lw[4] = {x_lo.x, x_lo.y, x_lo.z, x_lo.w};
    const uint32_t hw[4] = {x_hi.x, x_hi.y, x_hi.z, x_hi.w};
    const float cf[8] = {c[0].x, c[0].y, c[0].z, c[0].w, c[1].x, c[1].y, c[1].z, c[1].w};
    const float sf[8] = {s[0].x, s[0].y, s[0].z, s[0].w, s[1].x, s[1].y, s[1].z, s[1].w};
    uint32_t ol[4], oh[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint32_t rl[2], rh[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const double a = e ? bf16_hi(lw[k]) : bf16_lo(lw[k]);
            const double b = e ? bf16_hi(hw[k]) : bf16_lo(hw[k]);
            const double cc = (double)cf[2 * k + e], ss = (double)sf[2 * k + e];
            rl[e] = bf16_bits_rn(fma(a, cc, -(b * ss)));
            rh[e] = bf16_bits_rn(fma(b, cc, a * ss));
        }
        ol[k] = rl[0] | (rl[1] << 16);
        oh[k] = rh[0] | (rh[1] << 16);
    }
    o_lo = make_uint4(ol[0], ol[1], ol[2], ol[3]);
    o_hi = make_uint4(oh[0], oh[1], oh[2], oh[3]);
}

// Slot of sequence b, or -1 when it is outside [0, min(Lmax, max_pos)). Plain
// loads: this kernel writes seq_lens at the end.
__device__ __forceinline__ int slot_of(const PrestepParams &p, int b)
{
    const int pos = p.seq_lens[b];
    return (pos >= 0 && pos < p.Lmax && pos < p.max_pos) ? pos : -1;
}

__device__ __forceinline__ void load_table8(const float *tab, int pos, int j, float4 (&v)[2])
{
    const float4 *t = reinterpret_cast<const float4 *>(tab + (size_t)pos * (kHeadDim / 2) + 8 * j);
    v[0] = __ldg(t);
    v[1] = __ldg(t + 1);
}

template <int M>
__global__ void __launch_bounds__(kThreads, 1) rope_append_route_kernel(PrestepParams p, int cu)
{
    extern __shared__ __align__(128) uint8_t dsm[]; // [cu*(M+1)*256 staged rows][B*Hkv sink flags]
    __shared__ int32_t warp_cnt[kWarps];
    __shared__ int32_t warp_off[kWarps + 1];

    const int U = p.B * p.Hkv;
    uint4 *rows = reinterpret_cast<uint4 *>(dsm);
    uint8_t *sink_flag = dsm + (size_t)cu * (M + 1) * 256;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);

    // Every input may come from the preceding kernel, and the previous decode
    // step may still read the cache, seq_lens and the routing outputs: wait for
    // it. The decode kernel that follows reads all of its inputs after its own
    // dependency wait, so it may launch now and run its prologue.
    grid_dependency_wait();
    grid_launch_dependents();

    // Query row item `it` of the chunk starting at unit u0: rotate into q_out and
    // the staged rows; a sequence with no valid slot gets a zero query.
    auto query_item = [&](int it, int u0) {
        const int r = it >> 3, j = it & 7;
        const int u = u0 + r / M;
        const size_t row = ((size_t)u0 * M + r) * kHeadDim;
        // plain loads: q_out may be q_in (rotated in place)
        const uint4 *qi = reinterpret_cast<const uint4 *>(p.q_in + row);
        const uint4 qlo = qi[j], qhi = qi[j + 8];
        const int pos = slot_of(p, u / p.Hkv);
        uint4 *qs = rows + r * 16;
        uint4 *qd = reinterpret_cast<uint4 *>(p.q_out + row);
        uint4 lo = zero, hi = zero;
        if (pos >= 0) {
            float4 c[2], s[2];
            load_table8(p.rope_cos, pos, j, c);
            load_table8(p.rope_sin, pos, j, s);
            rope8(qlo, qhi, c, s, lo, hi);
        }
        qs[j] = lo;
        qs[j + 8] = hi;
        qd[j] = lo;
        qd[j + 8] = hi;
    };

    bool bad_slot = false;
    for (int u0 = 0; u0 < U; u0 += cu) {
        const int nu = (U - u0) < cu ? (U - u0) : cu;
        uint4 *krows = rows + (size_t)nu * M * 16;
        // One pass over the chunk's items, each thread on its own item (at the
        // 8B shape every item has a thread), so that no thread takes a key and
        // a query row one after the other: items [0, nu*8) are the new keys,
        // the rest the query rows.
        for (int it = threadIdx.x; it < nu * 8 + nu * M * 8; it += kThreads) {
            if (it >= nu * 8) {
                query_item(it - nu * 8, u0);
                continue;
            }
            // New key: rotate, append, capture or stage k0. New value: append.
            const int lu = it >> 3, j = it & 7;
            const int u = u0 + lu;
            // The new key and value do not depend on the slot: load them in the
            // same round trip as the slot itself.
            const uint4 *kn = reinterpret_cast<const uint4 *>(p.k_new + (size_t)u * kHeadDim);
            const uint4 *vn = reinterpret_cast<const uint4 *>(p.v_new + (size_t)u * kHeadDim);
            const uint4 klo = __ldg(kn + j), khi = __ldg(kn + j + 8);
            const uint4 vlo = __ldg(vn + j), vhi = __ldg(vn + j + 8);
            const int pos = slot_of(p, u / p.Hkv);
            uint4 *ks = krows + lu * 16;
            uint4 *k0g = reinterpret_cast<uint4 *>(p.k0 + (size_t)u * kHeadDim);
            if (pos < 0) {
                bad_slot = true;
                ks[j] = k0g[j];
                ks[j + 8] = k0g[j + 8];
                continue;
            }
            float4 c[2], s[2];
            load_table8(p.rope_cos, pos, j, c);
            load_table8(p.rope_sin, pos, j, s);
            uint4 lo, hi;
            rope8(klo, khi, c, s, lo, hi);
            const size_t slot = ((size_t)u * p.Lmax + pos) * kHeadDim;
            uint4 *kd = reinterpret_cast<uint4 *>(p.k_cache + slot);
            uint4 *vd = reinterpret_cast<uint4 *>(p.v_cache + slot);
            kd[j] = lo;
            kd[j + 8] = hi;
            vd[j] = vlo;
            vd[j + 8] = vhi;
            if (pos == 0) {
                uint4 *v0g = reinterpret_cast<uint4 *>(p.v0 + (size_t)u * kHeadDim);
                k0g[j] = lo;
                k0g[j + 8] = hi;
                v0g[j] = vlo;
                v0g[j + 8] = vhi;
                ks[j] = lo;
                ks[j + 8] = hi;
            } else {
                ks[j] = k0g[j];
                ks[j + 8] = k0g[j + 8];
            }
        }
        __syncthreads();
        route_units_warp<M, false>(rows, krows, nu, p.tau, (int)threadIdx.x >> 5, kWarps, [&](int lu, bool sink) {
            sink_flag[u0 + lu] = sink ? 1 : 0;
            p.mask[u0 + lu] = sink ? 1 : 0;
        });
        __syncthreads(); // the rows are overwritten by the next chunk
    }

    // Every read of seq_lens is behind the barriers above.
    for (int b = threadIdx.x; b < p.B; b += kThreads) {
        const int pos = slot_of(p, b);
        if (pos >= 0)
            p.seq_lens[b] = pos + 1;
    }
    if (p.error && __syncthreads_or(bad_slot) && threadIdx.x == 0)
        atomicOr(p.error, SR_DEVERR_APPEND_SLOT);
    compact_active<kThreads>(sink_flag, U, p.active, warp_cnt, warp_off);
}

template <int M>
cudaError_t launch_m(const PrestepArgs &a, cudaStream_t stream)
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
        e = cudaFuncSetAttribute(rope_append_route_kernel<M>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)((size_t)chunk_units<M>() * (M + 1) * 256 + SR_MAX_UNITS));
        if (e != cudaSuccess)
            return e;
        configured[dev].store(true);
    }
    PrestepParams p;
    p.q_in = static_cast<const __nv_bfloat16 *>(a.q_in);
    p.k_new = static_cast<const __nv_bfloat16 *>(a.k_new);
    p.v_new = static_cast<const __nv_bfloat16 *>(a.v_new);
    p.rope_cos = a.rope_cos;
    p.rope_sin = a.rope_sin;
    p.seq_lens = a.seq_lens;
    p.k_cache = static_cast<__nv_bfloat16 *>(a.k_cache);
    p.v_cache = static_cast<__nv_bfloat16 *>(a.v_cache);
    p.k0 = static_cast<__nv_bfloat16 *>(a.k0);
    p.v0 = static_cast<__nv_bfloat16 *>(a.v0);
    p.q_out = static_cast<__nv_bfloat16 *>(a.q_out);
    p.mask = a.mask;
    p.active = a.active;
    p.error = a.error;
    p.tau = a.tau;
    p.B = a.batch;
    p.Hkv = a.n_kv_heads;
    p.Lmax = a.max_seq_len;
    p.max_pos = a.max_pos;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, rope_append_route_kernel<M>, p, cu);
}

} // namespace

cudaError_t launch_rope_append_route(const PrestepArgs &a, cudaStream_t stream)
{
    cudaError_t e;
    switch (a.n_q_heads / a.n_kv_heads) {
    case 1:
        e = launch_m<1>(a, stream);
        break;
    case 2:
        e = launch_m<2>(a, stream);
        break;
    case 4:
        e = launch_m<4>(a, stream);
        break;
    case 8:
        e = launch_m<8>(a, stream);
        break;
    default:
        return cudaErrorInvalidValue;
    }
    return e != cudaSuccess ? e : cudaGetLastError();
}

} // namespace sr
