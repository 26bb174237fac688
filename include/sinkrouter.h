/*
 * sinkrouter.h -- C ABI of libsinkrouter.so: SinkRouter single-token decode
 * attention on NVIDIA B200 (sm_100a).
 *
 * The method (SinkRouter README, github.com/streamer-AP/SinkRouter, the
 * decode-time procedure list; sota2 summary of "SinkRouter: Sink-Aware Routing
 * for Efficient Long-Context Decoding ...", Abstract): at each decode step, every
 * GQA KV-head group is routed before the long KV-cache scan by comparing its
 * RoPE'd query heads with the cached position-0 key. Sink groups skip the scan
 * and return the position-0 value; active groups run split-K softmax attention
 * over the whole cache with an in-kernel reduction across splits.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor pointer is a DEVICE pointer owned by the caller, contiguous,
 *    row-major, 16-byte aligned. The library never allocates or frees memory.
 *  - bf16 tensors are IEEE bfloat16 bit patterns (2 bytes per element).
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream). Calls are asynchronous on that stream and never synchronise the
 *    host, except sr_get_device_error, which synchronises `stream`.
 *  - Host-visible argument errors return a status and launch nothing. Errors
 *    that depend on device data (seq_lens, active_list contents) cannot be seen
 *    on the host: the kernels clamp or skip and set bits in a device error word
 *    kept in the workspace (sr_get_device_error). No kernel traps.
 *  - A "unit" is one (sequence b, KV head g) pair, flat index u = b*Hkv + g.
 *    Query head h belongs to KV head g = h / M, M = Hq / Hkv (contiguous blocks).
 */
#ifndef SINKROUTER_H
#define SINKROUTER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Shapes of one attention layer's decode step. */
typedef struct sr_dims {
    int32_t batch;       /* B >= 1 */
    int32_t n_q_heads;   /* Hq, a multiple of n_kv_heads */
    int32_t n_kv_heads;  /* Hkv >= 1; group size M = Hq / Hkv must be 1, 2, 4 or 8 */
    int32_t head_dim;    /* d; must be 128 */
    int32_t max_seq_len; /* Lmax >= 1: positions allocated per unit in the caches */
} sr_dims;

typedef enum sr_status {
    SR_OK = 0,
    SR_ERR_INVALID_ARG = 1, /* null or misaligned pointer, non-positive size, bad n_splits */
    SR_ERR_UNSUPPORTED = 2, /* shape the kernels do not implement (d != 128, M not in {1,2,4,8},
                               B*Hkv > SR_MAX_UNITS) */
    SR_ERR_WORKSPACE = 3,   /* workspace pointer null/misaligned or smaller than needed */
    SR_ERR_CUDA = 4         /* a CUDA runtime call or kernel launch failed */
} sr_status;

/* Largest B*Hkv the kernels accept. */
#define SR_MAX_UNITS 16384
/* Largest forced split count per unit. */
#define SR_MAX_SPLITS 4096

/* Bits of the device error word (sr_get_device_error). */
#define SR_DEVERR_SEQ_LEN 1     /* a seq_lens entry was outside [1, Lmax]; it was clamped */
#define SR_DEVERR_ACTIVE_LIST 2 /* active_list count or an entry was out of range or out of
                                   order; the bad entries were skipped */
#define SR_DEVERR_TIMEOUT 4     /* a pipeline wait exceeded its time bound (a bug, never
                                   expected); outputs of that launch are invalid and the
                                   workspace must be re-initialised with sr_workspace_init */
#define SR_DEVERR_APPEND_SLOT 8 /* sr_rope_append_route: a sequence's slot seq_lens[b] was
                                   outside [0, min(Lmax, max_pos)); nothing was appended for it */

/*
 * sr_route -- cosine routing of every unit (README decode list: compare the RoPE
 * query with the cached position-0 key and route each KV group before the scan;
 * README routing controls: cosine threshold). For unit (b, g):
 *     c_h = <q_h, k0_g> / (|q_h| |k0_g|)   for the M query heads h of group g
 *           (c_h = 0 when either norm is 0)
 *     s_g = min_h c_h;   sink  <=>  s_g >= tau
 * The min over heads and the ">=" are this library's reading; the pages leave
 * the combination open. Computed in fp32 from the bf16 inputs.
 *
 *   q           bf16 [B, Hq, d]   decode query after RoPE
 *   k0          bf16 [B, Hkv, d]  cached position-0 key (RoPE at position 0 is
 *                                 the identity)
 *   tau         threshold; +INFINITY routes nothing, -INFINITY routes every unit
 *   route_mask  out uint8 [B*Hkv]: 1 = sink, 0 = active
 *   active_list out int32 [1 + B*Hkv]: [0] = number of active units n, then
 *               their flat indices in ascending order; entries past 1+n are
 *               left untouched
 * One launch; no workspace. Errors: SR_ERR_INVALID_ARG, SR_ERR_UNSUPPORTED,
 * SR_ERR_CUDA.
 */
sr_status sr_route(const sr_dims *dims, const void *q, const void *k0, float tau,
                   uint8_t *route_mask, int32_t *active_list, void *stream);

/*
 * sr_rope_append_route -- the step just before the scan, in one launch, for one
 * new token per sequence (README decode list: routing compares the RoPE'd query
 * with the cached position-0 key, which is recorded when the first token is
 * written; the new token's key and value join the cache before the scan). For
 * sequence b the token takes slot p = seq_lens[b]:
 *     q_out[b, h]   = rope(q_in[b, h], p)                  every query head h
 *     K[b, g, p]    = rope(k_new[b, g], p);   V[b, g, p] = v_new[b, g]
 *     k0[b, g] = K[b, g, 0], v0[b, g] = V[b, g, 0]          when p == 0
 *     route_mask / active_list = sr_route(q_out, k0, tau)  (bit for bit)
 *     seq_lens[b]   = p + 1
 * rope is the rotate-half rotary embedding: for i < d/2, with c = cos[p, i],
 * s = sin[p, i],
 *     y[i] = x[i] c - x[i + d/2] s,    y[i + d/2] = x[i + d/2] c + x[i] s,
 * each element the correctly rounded bf16 (nearest, ties to even) of that
 * value computed from the bf16 x and the fp32 table entries. The tables are
 * the caller's, so any frequency schedule (base, scaling) can be used.
 *
 *   q_in        bf16 [B, Hq, d]   query before RoPE (may be the same buffer as
 *                                 q_out: rotated in place)
 *   k_new       bf16 [B, Hkv, d]  new key before RoPE; must not overlap the caches
 *   v_new       bf16 [B, Hkv, d]  new value; must not overlap the caches
 *   rope_cos    fp32 [max_pos, d/2] cos table, row p for position p
 *   rope_sin    fp32 [max_pos, d/2] sin table
 *   max_pos     rows of the tables (>= 1)
 *   seq_lens    in/out int32 [B]: the slot to write, advanced by one
 *   k_cache, v_cache  in/out bf16 [B, Hkv, Lmax, d]: slot p is written
 *   k0, v0      in/out bf16 [B, Hkv, d]: written when p == 0, else read (k0)
 *   tau         routing threshold, as for sr_route
 *   q_out       out bf16 [B, Hq, d]: the RoPE'd query sr_decode_attention takes
 *   route_mask, active_list  out, as for sr_route
 *   device_error optional device int32 (NULL = not wanted): SR_DEVERR_APPEND_SLOT
 *               is ORed in when a sequence's slot is outside [0, min(Lmax,
 *               max_pos)) -- its cache, k0/v0 and length are left untouched,
 *               its q_out rows are zero and its groups are routed from those
 *               rows (so the mask still equals sr_route(q_out, k0, tau))
 * One launch of one CTA; no workspace. It waits for the preceding kernel in the
 * stream before reading anything and lets the next one (sr_decode_attention,
 * which reads all of its inputs after its own wait) launch early. Errors:
 * SR_ERR_INVALID_ARG, SR_ERR_UNSUPPORTED, SR_ERR_CUDA.
 */
sr_status sr_rope_append_route(const sr_dims *dims, const void *q_in, const void *k_new,
                               const void *v_new, const float *rope_cos, const float *rope_sin,
                               int32_t max_pos, int32_t *seq_lens, void *k_cache, void *v_cache,
                               void *k0, void *v0, float tau, void *q_out, uint8_t *route_mask,
                               int32_t *active_list, int32_t *device_error, void *stream);

/*
 * sr_decode_workspace_bytes -- size of the workspace sr_decode_attention needs
 * for any call with these dims and n_splits <= max_splits (0 = automatic
 * splits only). Holds the device error word, one self-resetting arrival
 * counter per unit and the fp32 split partials (m, l, O) of every split.
 * Returns 0 for invalid or unsupported dims.
 */
size_t sr_decode_workspace_bytes(const sr_dims *dims, int32_t max_splits);

/*
 * sr_workspace_init -- zero the workspace (cudaMemsetAsync on `stream`). Call
 * once after allocating it; afterwards every launch leaves the counters at zero.
 */
sr_status sr_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/*
 * sr_decode_attention -- routed split-K decode attention for one layer step.
 * Sink units (not listed in active_list): out[b, h] = v0[b, g] for every query
 * head h of the group, bit for bit, with no cache read (README decode list,
 * sink bypass). Active units: standard softmax attention over cache positions
 * 0 .. L_b-1 (position 0 read from the cache), scale 1/sqrt(d):
 *     out[b, h] = sum_j softmax_j(<q_h, K[b, g, j]> / sqrt(d)) V[b, g, j]
 * (README decode list: tiled QK/PV, online softmax, Split-K with in-kernel
 * reduction; pith.science review of arXiv 2604.16883, Figure 1 caption,
 * eq. (1)). fp32 arithmetic on bf16 inputs; out is rounded to bf16 (RNE).
 *
 *   q           bf16 [B, Hq, d]
 *   k_cache     bf16 [B, Hkv, Lmax, d]
 *   v_cache     bf16 [B, Hkv, Lmax, d]
 *   k0          bf16 [B, Hkv, d]; not read by this call (routing already used
 *               it); may be NULL
 *   v0          bf16 [B, Hkv, d]  cached position-0 value
 *   seq_lens    int32 [B] device: valid positions per sequence, 1 <= L_b <= Lmax
 *               (out of range: clamped, SR_DEVERR_SEQ_LEN). Positions >= L_b
 *               are never used and may hold anything, NaN included.
 *   active_list int32 [1 + B*Hkv] as written by sr_route (count, then strictly
 *               ascending unit indices)
 *   n_splits    0 = automatic: the active positions of all units are cut into
 *               one contiguous share per persistent CTA (balanced across the
 *               SMs, at least 256 positions each), decided on the device from
 *               active_list and seq_lens. > 0: every active unit is cut into
 *               exactly n_splits equal splits (<= SR_MAX_SPLITS).
 *   out         bf16 [B, Hq, d]
 *   workspace   device buffer of >= sr_decode_workspace_bytes(dims, n_splits)
 *               bytes, 256-byte aligned, zeroed once by sr_workspace_init.
 *               Two calls that overlap on the GPU must not share a workspace.
 * Must run after sr_route on the same stream (or be ordered after it). One
 * kernel launch. Errors: SR_ERR_INVALID_ARG, SR_ERR_UNSUPPORTED,
 * SR_ERR_WORKSPACE, SR_ERR_CUDA.
 */
sr_status sr_decode_attention(const sr_dims *dims, const void *q, const void *k_cache,
                              const void *v_cache, const void *k0, const void *v0,
                              const int32_t *seq_lens, const int32_t *active_list,
                              int32_t n_splits, void *out, void *workspace,
                              size_t workspace_bytes, void *stream);

/*
 * sr_decode_attention_lse -- sr_decode_attention that also returns, for every
 * query head of an active unit, the natural-log log-sum-exp of its scaled
 * logits over positions 0 .. L_b-1:
 *     lse[b, h] = log sum_j exp(<q_h, K[b, g, j]> / sqrt(d))
 * so that any attention weight can be recovered, e.g. the weight of position 0
 * p0 = exp(<q_h, K[b, g, 0]> / sqrt(d) - lse[b, h]). The pith.science review of
 * arXiv 2604.16883 (Figure 10 caption) defines the routing proxy's reference
 * event from these full-attention position-0 weights. Sink heads get NaN (no
 * attention is computed for them).
 *
 *   lse   out fp32 [B, Hq], device, 4-byte aligned
 * Other arguments, results and errors: as sr_decode_attention.
 */
sr_status sr_decode_attention_lse(const sr_dims *dims, const void *q, const void *k_cache,
                                  const void *v_cache, const void *k0, const void *v0,
                                  const int32_t *seq_lens, const int32_t *active_list,
                                  int32_t n_splits, void *out, float *lse, void *workspace,
                                  size_t workspace_bytes, void *stream);

/*
 * sr_position0_weight -- the full-attention weight of position 0 for every query
 * head, from the log-sum-exp that sr_decode_attention_lse returns:
 *     p0[b, h] = exp(<q[b, h], k_cache[b, g, 0]> / sqrt(d) - lse[b, h]),  g = h / M
 * (fp32 dot product of the bf16 rows). The pith.science review of arXiv
 * 2604.16883 (Figure 10 caption) defines the routing proxy's reference "oracle
 * sink event" from these weights. Heads whose lse is NaN (sinks) get NaN.
 *
 *   q        bf16 [B, Hq, d], 16-byte aligned: the query the lse was computed for
 *   k_cache  bf16 [B, Hkv, Lmax, d], 16-byte aligned: position 0 of every unit is read
 *   lse      fp32 [B, Hq], device, 4-byte aligned
 *   p0       out fp32 [B, Hq], device, 4-byte aligned
 * One launch (one warp per head), asynchronous on `stream`, no workspace.
 * Errors: SR_ERR_INVALID_ARG, SR_ERR_UNSUPPORTED, SR_ERR_CUDA.
 */
sr_status sr_position0_weight(const sr_dims *dims, const void *q, const void *k_cache, const float *lse,
                              float *p0, void *stream);

/*
 * sr_route_decode_attention -- sr_route followed by sr_decode_attention in ONE
 * kernel launch: every CTA of the decode kernel routes all units itself (the
 * same fp32 arithmetic as sr_route, so the decisions are identical) and builds
 * the work list in shared memory, which removes the routing launch and the
 * hand-off between the two kernels from the step. Same method and passages as
 * the two calls above; the result (route decisions and out) equals theirs bit
 * for bit.
 *
 *   q, k_cache, v_cache, v0, seq_lens, n_splits, out, workspace, workspace_bytes:
 *               as for sr_decode_attention
 *   k0, tau     as for sr_route (k0 is required here)
 *   route_mask  optional out uint8 [B*Hkv] (NULL = not written)
 *   active_list optional out int32 [1 + B*Hkv] in sr_route's format (NULL = not
 *               written); this call never reads it
 * Errors: SR_ERR_INVALID_ARG, SR_ERR_UNSUPPORTED, SR_ERR_WORKSPACE, SR_ERR_CUDA.
 */
sr_status sr_route_decode_attention(const sr_dims *dims, const void *q, const void *k_cache,
                                    const void *v_cache, const void *k0, const void *v0,
                                    const int32_t *seq_lens, float tau, int32_t n_splits,
                                    uint8_t *route_mask, int32_t *active_list, void *out,
                                    void *workspace, size_t workspace_bytes, void *stream);

/* Largest number of parts sr_combine_partials accepts. */
#define SR_MAX_PARTS 1024

/*
 * sr_decode_attention_partial -- sr_decode_attention over the positions this
 * call's cache holds, with each head's result left in the form that combines
 * across calls over disjoint position ranges (context parallelism: each GPU
 * holds one contiguous shard of every sequence's cache and scans it; the
 * shards' results are exchanged and combined with sr_combine_partials). The
 * README's split-K decode reduces such partials inside one kernel; this is the
 * same reduction carried across GPUs.
 *
 * Arguments are those of sr_decode_attention, with the output replaced by:
 *   o_part   out fp32 [B, Hq, d]: for an active head, softmax attention over
 *            the L_b positions of this call's cache, normalised and NOT rounded
 *            to bf16 (bf16 of it equals sr_decode_attention's out bit for bit);
 *            for a sink head, v0 widened to fp32 (exact)
 *   lse_part out fp32 [B, Hq]: natural-log log-sum-exp of the scaled logits
 *            (q . k_j / sqrt(d)) over those positions; NaN for sink heads
 * Every rank must route identically (same q, k0, tau) and pass the same active
 * list; seq_lens holds the lengths of this call's shard (>= 1 each).
 * Errors: as sr_decode_attention.
 */
sr_status sr_decode_attention_partial(const sr_dims *dims, const void *q, const void *k_cache,
                                      const void *v_cache, const void *k0, const void *v0,
                                      const int32_t *seq_lens, const int32_t *active_list,
                                      int32_t n_splits, float *o_part, float *lse_part,
                                      void *workspace, size_t workspace_bytes, void *stream);

/*
 * sr_combine_partials -- combine R partial results over disjoint position
 * ranges into the attention output over their union: per head
 *     lse = log sum_r exp(lse_r),    out = bf16( sum_r exp(lse_r - lse) o_r )
 * (the union's softmax denominator is the sum of the parts' denominators). A
 * head whose part-0 lse is NaN is a sink head and gets bf16(o_0) = v0. A part
 * with lse = -inf (no positions) weighs 0; if every part does, the output is
 * undefined.
 *   dims        batch and n_q_heads give the B*Hq heads (n_kv_heads and
 *               max_seq_len are not read); head_dim must be 128
 *   n_parts     R, 1 .. SR_MAX_PARTS
 *   o_parts     fp32: part r's o_part [B, Hq, d] at o_parts + r * part_stride
 *   lse_parts   fp32: part r's lse_part [B, Hq] at lse_parts + r * part_stride
 *   part_stride floats from one part to the next (the same for both arrays): a
 *               multiple of 4, and >= B*Hq*d when R > 1. A gathered buffer of
 *               [R][o_part | lse_part] rows uses o_parts = base,
 *               lse_parts = base + B*Hq*d and its row length as the stride.
 *   out         bf16 [B, Hq, d]
 * One launch (one warp per head), asynchronous on `stream`, no workspace.
 * Errors: SR_ERR_INVALID_ARG, SR_ERR_UNSUPPORTED, SR_ERR_CUDA.
 */
sr_status sr_combine_partials(const sr_dims *dims, int32_t n_parts, const float *o_parts,
                              const float *lse_parts, int64_t part_stride, void *out, void *stream);

/*
 * sr_selftest_bounded_wait -- exercise the time-bounded wait that every kernel
 * of this library uses instead of an unbounded spin: one warp waits on an
 * mbarrier that nothing ever arrives on, gives up after limit_us microseconds
 * (read from %globaltimer) and reports it. (An engineering self-test; the
 * pages have no counterpart.)
 *   limit_us   1 .. 2000000 (the kernels' own bound is 2 s)
 *   status     out device int32: SR_DEVERR_TIMEOUT when the wait ran out (the
 *              expected result), 0 if it completed
 *   waited_ns  out device uint64: how long the warp waited
 * One launch of one warp on `stream`; the context stays usable afterwards.
 * Errors: SR_ERR_INVALID_ARG, SR_ERR_CUDA.
 */
sr_status sr_selftest_bounded_wait(int32_t limit_us, int32_t *status, uint64_t *waited_ns, void *stream);

/* Static description of a status code. */
const char *sr_status_string(sr_status s);

/*
 * sr_get_device_error -- read the device error word of a workspace into *code
 * (an OR of SR_DEVERR_* bits; 0 = none). Synchronises `stream`. Debug use.
 */
sr_status sr_get_device_error(const void *workspace, int32_t *code, void *stream);

/* sr_clear_device_error -- reset the device error word to 0 (async on `stream`). */
sr_status sr_clear_device_error(void *workspace, void *stream);

/*
 * sr_decode_grid_size -- number of persistent CTAs sr_decode_attention launches
 * on the current device (its SM count times resident CTAs per SM). Returns 0
 * when no device is usable.
 */
int32_t sr_decode_grid_size(void);

/* Message of the last CUDA error seen by this library on this thread ("" if none). */
const char *sr_last_cuda_error(void);

/* Size of the fixed scratch array behind sr_decode_attention_static_scratch. */
#define SR_STATIC_SCRATCH_BYTES (8u << 20)

/*
 * sr_decode_attention_static_scratch -- sr_decode_attention without a
 * workspace argument, for callers that cannot allocate device memory. (An
 * engineering addition: the paper and its code have no counterpart.)
 *
 * Who needs it: code that only ever receives its input and output buffers and
 * may not call cudaMalloc -- a plugin whose host framework owns every device
 * allocation and passes no scratch buffer through its fixed interface, a
 * serving runtime that plans all memory at start-up and forbids allocation on
 * the decode path (cudaMalloc can synchronise the device and fragment a
 * pre-planned pool), or a certified deployment that bans dynamic allocation
 * after initialisation.
 *
 * The decode kernel's scratch (error word, per-unit counters, split partials)
 * is a fixed array of SR_STATIC_SCRATCH_BYTES compiled into this library; every
 * GPU that loads the library holds it until the process exits. Arguments,
 * results and errors are those of sr_decode_attention, with these differences:
 *   - no workspace: dims and n_splits whose scratch would exceed
 *     SR_STATIC_SCRATCH_BYTES are rejected with SR_ERR_WORKSPACE (at n_splits =
 *     0 this admits B*Hkv up to about 990 with M = 8, 3000 with M = 4, 15000
 *     with M = 1);
 *   - device_error: optional device pointer (NULL = not wanted) that receives
 *     the launch's device error word (SR_DEVERR_* bits), stream-ordered;
 *   - every call looks up the array's device address on the current device
 *     (cudaGetSymbolAddress, cheap once the module is loaded there), so no
 *     address survives a device reset; the first call on a device may load
 *     the module there, so make that first call before any stream capture;
 *   - every call on a device shares the one array: each call clears the error
 *     word and the counters it needs, so calls in sequence on one stream are
 *     fine, but calls that overlap on the GPU (different streams, or host
 *     threads without ordering) race on the array and must be serialised.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 */
sr_status sr_decode_attention_static_scratch(const sr_dims *dims, const void *q, const void *k_cache,
                                             const void *v_cache, const void *k0, const void *v0,
                                             const int32_t *seq_lens, const int32_t *active_list,
                                             int32_t n_splits, void *out, int32_t *device_error,
                                             void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SINKROUTER_H */
