/*
 * SinkRouter decode-attention oracle: plain fp64 CPU reference.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark load this library. The product path (the CUDA library) never
 * links, calls or imports it, and this file shares no code with it.
 *
 * What it computes, for one single-token decode step of one attention layer
 * (SinkRouter README, github.com/streamer-AP/SinkRouter, the decode-time
 * procedure list; sota2 summary of "SinkRouter: Sink-Aware Routing for
 * Efficient Long-Context Decoding", Abstract):
 *
 *   1. Routing, per GQA KV-head group (b, g): every query head h of the group is
 *      compared with the cached position-0 key by cosine similarity; the group
 *      score is the minimum over its heads, and the group is a sink when that
 *      score is at least tau. (README decode list: compare the RoPE query with
 *      the position-0 key, route each KV group before the scan; README routing
 *      controls: a cosine routing threshold. The min-over-heads combination and
 *      the ">=" are the specification's reading; the pages do not fix them.)
 *   2. A sink group returns the position-0 value for each of its heads, with no
 *      scan of the cache (README decode list, sink bypass).
 *   3. An active group runs standard softmax attention over every cached
 *      position 0 .. L_b-1, scale 1/sqrt(d) (README decode list, active path;
 *      pith.science review of arXiv 2604.16883, Figure 1 caption, eq. (1): the
 *      head update is the attention-weighted sum of the cached values).
 *
 * The split-K scan, online softmax and in-kernel reduction of the GPU path reach
 * exactly this result up to rounding, so the oracle is the definition written
 * out: no tiling, no online rescaling, no splitting.
 *
 * Inputs are bf16 bit patterns (uint16). Each is widened to fp64 exactly.
 * All arithmetic is fp64.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SR_ORACLE_OK 0
#define SR_ORACLE_BAD_ARG 1
#define SR_ORACLE_NO_MEM 2

/* Exact widening of a bf16 bit pattern: bf16 is the top half of an IEEE fp32. */
static double widen_bf16(uint16_t bits)
{
    uint32_t w = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/*
 * Cosine of the angle between a query head and the position-0 key.
 * A zero-norm vector has no direction; the pages are silent, and the reading
 * taken here is cosine := 0.
 */
static double cosine_q_k0(const uint16_t *qh, const uint16_t *k0g, int d)
{
    double dot = 0.0, qq = 0.0, kk = 0.0;
    for (int i = 0; i < d; ++i) {
        double a = widen_bf16(qh[i]);
        double b = widen_bf16(k0g[i]);
        dot += a * b;
        qq += a * a;
        kk += b * b;
    }
    if (qq == 0.0 || kk == 0.0)
        return 0.0;
    return dot / (sqrt(qq) * sqrt(kk));
}

/*
 * Routing (step 1 above).
 *   q      [B, Hq, d]  bf16 bits (post-RoPE decode query)
 *   k0     [B, Hkv, d] bf16 bits (cached position-0 key)
 *   tau    threshold; +inf routes nothing, -inf routes every group
 *   mask   out [B*Hkv]: 1 = sink, 0 = active
 *   active out [1 + B*Hkv]: [0] = number of active groups, then their flat
 *          indices b*Hkv + g in ascending order
 *   score  out [B*Hkv] (may be NULL): s_g = min over the group's heads of cos
 * Query head h belongs to group h / (Hq/Hkv) (contiguous blocks of heads).
 */
int sr_oracle_route(int B, int Hq, int Hkv, int d,
                    const uint16_t *q, const uint16_t *k0, double tau,
                    uint8_t *mask, int32_t *active, double *score)
{
    if (B < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv != 0 || d < 1 || !q || !k0 || !mask || !active)
        return SR_ORACLE_BAD_ARG;
    int M = Hq / Hkv;
    int32_t count = 0;
    for (int b = 0; b < B; ++b) {
        for (int g = 0; g < Hkv; ++g) {
            const uint16_t *k0g = k0 + ((size_t)b * Hkv + g) * d;
            double s = INFINITY;
            for (int m = 0; m < M; ++m) {
                int h = g * M + m;
                double c = cosine_q_k0(q + ((size_t)b * Hq + h) * d, k0g, d);
                if (c < s)
                    s = c;
            }
            int unit = b * Hkv + g;
            int sink = (s >= tau);
            mask[unit] = (uint8_t)sink;
            if (score)
                score[unit] = s;
            if (!sink)
                active[1 + count++] = unit;
        }
    }
    active[0] = count;
    return SR_ORACLE_OK;
}

/*
 * Round-to-nearest-even of an fp64 value to bf16 (the top half of an IEEE
 * fp32), in one rounding step: the value is scaled so that the bf16 spacing
 * at its magnitude becomes 1, rounded with rint (ties to even in the default
 * rounding mode) and scaled back; the result has at most 8 significant bits,
 * so its conversion to fp32 is exact (or overflows to infinity).
 */
static uint16_t narrow_to_bf16(double x)
{
    if (isnan(x))
        return 0x7fc0;
    if (x == 0.0)
        return signbit(x) ? 0x8000 : 0x0000;
    int e;
    (void)frexp(x, &e); /* |x| = m 2^e with m in [0.5, 1) */
    int spacing = e - 8;
    if (spacing < -133) /* bf16 subnormals share fp32's exponent range */
        spacing = -133;
    double y = ldexp(rint(ldexp(x, -spacing)), spacing);
    float f = (float)y;
    uint32_t w;
    memcpy(&w, &f, sizeof w);
    return (uint16_t)(w >> 16);
}

/*
 * Rotary position embedding of one row of d values at one position
 * (rotate-half form: element i pairs with element i + d/2):
 *   out[i]       = x[i] c_i - x[i + d/2] s_i
 *   out[i + d/2] = x[i + d/2] c_i + x[i] s_i,      i < d/2
 * with c, s the rows of the cos / sin tables for that position.
 */
static void rope_row(const uint16_t *x, const float *c, const float *s, int d, uint16_t *out)
{
    int h = d / 2;
    for (int i = 0; i < h; ++i) {
        double a = widen_bf16(x[i]), b = widen_bf16(x[i + h]);
        out[i] = narrow_to_bf16(a * (double)c[i] - b * (double)s[i]);
        out[i + h] = narrow_to_bf16(b * (double)c[i] + a * (double)s[i]);
    }
}

/*
 * The step just before the scan, for one new token per sequence (SinkRouter
 * README, decode-time procedure list: routing compares the RoPE query with the
 * cached position-0 key, which prefill records; the new token's key and value
 * join the cache). For sequence b the token takes slot p = seq_lens[b]:
 *   q_out[b, h]  = bf16(rope(q_in[b, h], p))                for every query head
 *   K[b, g, p]   = bf16(rope(k_new[b, g], p)),  V[b, g, p] = v_new[b, g]
 *   k0[b, g] = K[b, g, 0], v0[b, g] = V[b, g, 0]            when p == 0
 *   seq_lens[b] = p + 1
 * rope_cos / rope_sin: fp32 [max_pos, d/2]. A slot outside [0, min(Lmax,
 * max_pos)) is an error (status SR_ORACLE_BAD_ARG): that sequence's cache,
 * k0/v0 and length are left alone and its q_out rows are zero (there is no
 * table row to rotate by; the pages do not cover a full cache).
 */
int sr_oracle_rope_append(int B, int Hq, int Hkv, int d, int Lmax, int max_pos,
                          const uint16_t *q_in, const uint16_t *k_new, const uint16_t *v_new,
                          const float *rope_cos, const float *rope_sin, int32_t *seq_lens,
                          uint16_t *k_cache, uint16_t *v_cache, uint16_t *k0, uint16_t *v0, uint16_t *q_out)
{
    if (B < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv != 0 || d < 2 || d % 2 != 0 || Lmax < 1 || max_pos < 1 ||
        !q_in || !k_new || !v_new || !rope_cos || !rope_sin || !seq_lens || !k_cache || !v_cache || !k0 || !v0 ||
        !q_out)
        return SR_ORACLE_BAD_ARG;
    int status = SR_ORACLE_OK;
    for (int b = 0; b < B; ++b) {
        int p = seq_lens[b];
        if (p < 0 || p >= Lmax || p >= max_pos) {
            status = SR_ORACLE_BAD_ARG;
            memset(q_out + (size_t)b * Hq * d, 0, sizeof(uint16_t) * (size_t)Hq * d);
            continue;
        }
        const float *c = rope_cos + (size_t)p * (d / 2);
        const float *s = rope_sin + (size_t)p * (d / 2);
        for (int h = 0; h < Hq; ++h)
            rope_row(q_in + ((size_t)b * Hq + h) * d, c, s, d, q_out + ((size_t)b * Hq + h) * d);
        for (int g = 0; g < Hkv; ++g) {
            size_t unit = (size_t)b * Hkv + g;
            uint16_t *kslot = k_cache + (unit * Lmax + p) * d;
            uint16_t *vslot = v_cache + (unit * Lmax + p) * d;
            rope_row(k_new + unit * d, c, s, d, kslot);
            memcpy(vslot, v_new + unit * d, sizeof(uint16_t) * (size_t)d);
            if (p == 0) {
                memcpy(k0 + unit * d, kslot, sizeof(uint16_t) * (size_t)d);
                memcpy(v0 + unit * d, vslot, sizeof(uint16_t) * (size_t)d);
            }
        }
        seq_lens[b] = p + 1;
    }
    return status;
}

typedef struct {
    int B, Hq, Hkv, d, Lmax;
    const uint16_t *q, *kc, *vc, *v0;
    const int32_t *seq_lens;
    const uint8_t *mask;
    const int32_t *units; /* units to compute (flat b*Hkv+g) */
    int n_units;
    double *out; /* [B, Hq, d] */
    double *p0;  /* [B, Hq] */
    int tid, n_threads;
    int status;
} oracle_job;

/*
 * One head m of one group (steps 2 and 3 above).
 * Active path: logits l_j = <q_h, K_j> / sqrt(d) for j = 0 .. L-1 (position 0
 * read from the cache), p = exp(l - max l) / sum, out = sum_j p_j V_j, and the
 * weight p_0 of position 0 is also returned. Sink path: out = v0 exactly and
 * p_0 is reported as NaN (no attention was computed). Each head of a group is
 * computed on its own, so splitting the work by head changes no arithmetic.
 */
static int oracle_head(const oracle_job *J, int unit, int m, double *logit)
{
    int M = J->Hq / J->Hkv;
    int b = unit / J->Hkv, g = unit % J->Hkv;
    int d = J->d;
    int L = J->seq_lens[b];
    if (L < 1 || L > J->Lmax)
        return SR_ORACLE_BAD_ARG;
    const uint16_t *K = J->kc + ((size_t)b * J->Hkv + g) * (size_t)J->Lmax * d;
    const uint16_t *V = J->vc + ((size_t)b * J->Hkv + g) * (size_t)J->Lmax * d;
    double scale = 1.0 / sqrt((double)d);
    int h = g * M + m;
    double *o = J->out + ((size_t)b * J->Hq + h) * d;
    if (J->mask[unit]) {
        const uint16_t *v0g = J->v0 + ((size_t)b * J->Hkv + g) * d;
        for (int i = 0; i < d; ++i)
            o[i] = widen_bf16(v0g[i]);
        if (J->p0)
            J->p0[(size_t)b * J->Hq + h] = NAN;
        return SR_ORACLE_OK;
    }
    const uint16_t *qh = J->q + ((size_t)b * J->Hq + h) * d;
    double mx = -INFINITY;
    for (int j = 0; j < L; ++j) {
        double acc = 0.0;
        const uint16_t *kj = K + (size_t)j * d;
        for (int i = 0; i < d; ++i)
            acc += widen_bf16(qh[i]) * widen_bf16(kj[i]);
        logit[j] = acc * scale;
        if (logit[j] > mx)
            mx = logit[j];
    }
    double z = 0.0;
    for (int j = 0; j < L; ++j) {
        logit[j] = exp(logit[j] - mx);
        z += logit[j];
    }
    for (int i = 0; i < d; ++i)
        o[i] = 0.0;
    for (int j = 0; j < L; ++j) {
        double p = logit[j] / z;
        const uint16_t *vj = V + (size_t)j * d;
        for (int i = 0; i < d; ++i)
            o[i] += p * widen_bf16(vj[i]);
    }
    if (J->p0)
        J->p0[(size_t)b * J->Hq + h] = logit[0] / z;
    return SR_ORACLE_OK;
}

static void *oracle_worker(void *arg)
{
    oracle_job *J = (oracle_job *)arg;
    double *logit = (double *)malloc(sizeof(double) * (size_t)J->Lmax);
    if (!logit) {
        J->status = SR_ORACLE_NO_MEM;
        return NULL;
    }
    int M = J->Hq / J->Hkv;
    for (long k = J->tid; k < (long)J->n_units * M; k += J->n_threads) {
        int st = oracle_head(J, J->units[k / M], (int)(k % M), logit);
        if (st != SR_ORACLE_OK) {
            J->status = st;
            break;
        }
    }
    free(logit);
    return NULL;
}

/*
 * Routed decode attention (steps 2 and 3) for the listed groups.
 *   q [B,Hq,d], k_cache/v_cache [B,Hkv,Lmax,d], v0 [B,Hkv,d]: bf16 bits
 *   seq_lens [B]: valid positions per sequence, 1 <= L_b <= Lmax
 *   mask [B*Hkv]: the route decision (1 = sink), e.g. from sr_oracle_route
 *   units [n_units]: flat group indices to compute; NULL = every group
 *   out [B,Hq,d] fp64 and p0 [B,Hq] fp64 (p0 may be NULL): only the heads of
 *   the listed groups are written
 *   n_threads: worker threads; the (group, head) pairs are dealt round-robin,
 *   each head is computed whole by one thread, so the result does not depend
 *   on it
 */
int sr_oracle_decode(int B, int Hq, int Hkv, int d, int Lmax,
                     const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                     const uint16_t *v0, const int32_t *seq_lens, const uint8_t *mask,
                     const int32_t *units, int n_units,
                     double *out, double *p0, int n_threads)
{
    if (B < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv != 0 || d < 1 || Lmax < 1 || !q || !k_cache ||
        !v_cache || !v0 || !seq_lens || !mask || !out)
        return SR_ORACLE_BAD_ARG;
    int32_t *all = NULL;
    if (!units) {
        n_units = B * Hkv;
        all = (int32_t *)malloc(sizeof(int32_t) * (size_t)n_units);
        if (!all)
            return SR_ORACLE_NO_MEM;
        for (int u = 0; u < n_units; ++u)
            all[u] = u;
        units = all;
    }
    for (int k = 0; k < n_units; ++k)
        if (units[k] < 0 || units[k] >= B * Hkv) {
            free(all);
            return SR_ORACLE_BAD_ARG;
        }
    if (n_threads < 1)
        n_threads = 1;
    if ((long)n_threads > (long)n_units * (Hq / Hkv))
        n_threads = n_units > 0 ? n_units * (Hq / Hkv) : 1;
    oracle_job *jobs = (oracle_job *)calloc((size_t)n_threads, sizeof(oracle_job));
    pthread_t *th = (pthread_t *)calloc((size_t)n_threads, sizeof(pthread_t));
    if (!jobs || !th) {
        free(jobs);
        free(th);
        free(all);
        return SR_ORACLE_NO_MEM;
    }
    for (int t = 0; t < n_threads; ++t) {
        oracle_job J = {B, Hq, Hkv, d, Lmax, q, k_cache, v_cache, v0, seq_lens, mask,
                        units, n_units, out, p0, t, n_threads, SR_ORACLE_OK};
        jobs[t] = J;
    }
    int status = SR_ORACLE_OK;
    if (n_threads == 1) {
        oracle_worker(&jobs[0]);
    } else {
        int started = 0;
        for (int t = 0; t < n_threads; ++t) {
            if (pthread_create(&th[t], NULL, oracle_worker, &jobs[t]) != 0)
                break;
            ++started;
        }
        for (int t = 0; t < started; ++t)
            pthread_join(th[t], NULL);
        for (int t = started; t < n_threads; ++t)
            oracle_worker(&jobs[t]);
    }
    for (int t = 0; t < n_threads; ++t)
        if (jobs[t].status != SR_ORACLE_OK)
            status = jobs[t].status;
    free(jobs);
    free(th);
    free(all);
    return status;
}
