/*
 * moe_oracle.c -- plain, slow CPU restatement of the routed Mixture-of-Experts
 * layer with a per-layer LFU expert slot cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  The CUDA
 * product path never links, calls or reads anything here, and nothing here is
 * shared with it (no headers, helpers, tables or constants).
 *
 * Sources (the pages are news/blog summaries of the TurboFieldfare runtime):
 *   [yodev]  "Gemma 4 26B en ~2 GB de RAM: el runtime en Swift que streamea los
 *            experts desde el SSD", sections "Por que funciona: el A4B del
 *            nombre" (per-token loop) and "Por que pread y no mmap".
 *   [hada]   "TurboFieldfare: motor open source para ejecutar Gemma 4 26B con
 *            2 GB de RAM", sections "Estructura de ejecucion para reducir
 *            memoria" (4-bit MLX affine, group 64, 8-bit router) and "Proceso
 *            de generacion de tokens" (top-8 ids vs a 16-slot LFU per layer,
 *            shared branch during the reads, combine).
 *   [stork]  "El milagro de la IA de 2GB en Apple Silicon", section "Mas
 *            inteligente que tu RAM" (30 layers, LFU keeps 16 of 128 experts,
 *            a miss replaces the least frequently used expert in memory) and
 *            "Por que la mayor parte de tu modelo de IA es peso muerto"
 *            (router picks the 8 most relevant of 128).
 *   [imasters] "Engine open source roda Gemma 4 26B ...", section "O truque"
 *            (top-8 ids planned against a 16-slot LFU, 4-bit group-64 affine).
 * Where the pages are silent the reading taken is stated next to the code.
 *
 * Precision: fp64 everywhere except the router logits, whose fp32 values decide
 * an integer result (the top-8 ids).  Those are computed in the kernel's
 * precision with the fixed FMA order documented at orc_router_logits.
 *
 * Parity status: every function here is pinned by tests in tests/ (golden
 * layout points, closed forms, brute force, library routines, a naive LFU
 * simulator).  No function is "parity unpinned".
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "moe_oracle.h"

/* ---------------------------------------------------------------- numbers */

/* IEEE 754 binary16 -> double, from the format's definition
 * (1 sign bit, 5 exponent bits with bias 15, 10 fraction bits). */
double orc_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int m = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24); /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE binary32. */
float orc_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* GELU, tanh form: 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))). */
double orc_gelu_tanh(double v)
{
    const double c = sqrt(2.0 / 3.14159265358979323846);
    return 0.5 * v * (1.0 + tanh(c * (v + 0.044715 * v * v * v)));
}

/* ------------------------------------------------------- expert blob layout
 *
 * An expert is one contiguous kernel-ready blob ([stork] "El arma secreta de
 * Apple": the stored weights already are the 4-bit layout the GPU kernel
 * consumes, so reading the file needs no conversion).
 * The pages fix only that the blob is the kernel's own layout; the byte layout
 * below is this library's definition of it.  For an expert with model width D
 * and FFN width F, group G = 64:
 *
 *   matrices   gate W_g [F x D], up W_u [F x D], down W_d [D x F];
 *              w[n][k] = s[n][k/64] * q[n][k] + b[n][k/64], q in 0..15,
 *              s, b IEEE binary16 ([hada] 4-bit MLX affine, group 64).
 *   chunk      32 rows x KS inputs, 18*KS bytes:
 *                q part  (KS/32 word-quads) x (32 rows) x 16 bytes; byte
 *                        ((wq*32 + r)*16 + 4*word + j/2) holds input
 *                        k = 32*wq + 8*word + j of row r in its low nibble
 *                        (j even) or high nibble (j odd);
 *                sb part (KS/64 groups) x (32 rows) x 4 bytes: s then b.
 *   gate/up    section 0: F/16 tiles x D/256 slices (KS = 256), tile-major;
 *              tile t rows 0..15 are gate rows 16t..16t+15, rows 16..31 are
 *              up rows 16t..16t+15.
 *   down       section 1 (right after section 0): D/32 tiles x F/KS slices,
 *              KS = F if F <= 704 else 704, tile-major; tile t rows 0..31 are
 *              down rows 32t..32t+31.
 */
static int down_ks(int F) { return F <= 704 ? F : 704; }

size_t orc_blob_bytes(int D, int F)
{
    size_t gu = (size_t)(F / 16) * (size_t)(D / 256) * 18u * 256u;
    size_t dn = (size_t)(D / 32) * (size_t)(F / down_ks(F)) * 18u * (size_t)down_ks(F);
    return gu + dn;
}

/* Byte offset of the q nibble of (matrix m, row n, input k), whether it is the
 * high nibble, and the byte offset of that row's (s, b) pair for k's group.
 * m: 0 = gate, 1 = up, 2 = down. */
static void orc_locate(int D, int F, int m, int n, int k,
                       size_t *qbyte, int *hi, size_t *sbbyte)
{
    size_t base, chunk;
    int r, kk, ks;
    if (m == 0 || m == 1) {
        int t = n / 16;
        int s = k / 256;
        ks = 256;
        kk = k % 256;
        r = (n % 16) + 16 * m;
        base = 0;
        chunk = base + ((size_t)t * (size_t)(D / 256) + (size_t)s) * 18u * 256u;
    } else {
        int t = n / 32;
        int s;
        ks = down_ks(F);
        s = k / ks;
        kk = k % ks;
        r = n % 32;
        base = (size_t)(F / 16) * (size_t)(D / 256) * 18u * 256u;
        chunk = base + ((size_t)t * (size_t)(F / ks) + (size_t)s) * 18u * (size_t)ks;
    }
    {
        int wq = kk / 32, word = (kk % 32) / 8, j = kk % 8;
        *qbyte = chunk + ((size_t)wq * 32u + (size_t)r) * 16u + 4u * (size_t)word + (size_t)(j / 2);
        *hi = j & 1;
        *sbbyte = chunk + 16u * (size_t)ks + ((size_t)(kk / 64) * 32u + (size_t)r) * 4u;
    }
}

static uint16_t rd16(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }

/* One dequantised weight: w = s*q + b (exact in double: an 11-bit scale times
 * a 4-bit integer plus an 11-bit bias fits in 53 bits). */
double orc_weight(const uint8_t *blob, int D, int F, int m, int n, int k)
{
    size_t qb, sb;
    int hi, q;
    double s, b;
    orc_locate(D, F, m, n, k, &qb, &hi, &sb);
    q = hi ? (blob[qb] >> 4) & 15 : blob[qb] & 15;
    s = orc_f16_to_f64(rd16(blob + sb));
    b = orc_f16_to_f64(rd16(blob + sb + 2));
    return s * (double)q + b;
}

/* Whole matrix, row-major [N][Kin]. */
void orc_dequant(const uint8_t *blob, int D, int F, int m, double *W)
{
    int N = (m == 2) ? D : F, Kin = (m == 2) ? F : D;
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < Kin; ++k)
            W[(size_t)n * Kin + k] = orc_weight(blob, D, F, m, n, k);
}

/* ----------------------------------------------------------- expert FFN
 * One expert FFN ([hada] routed and shared experts are 4-bit FFNs):
 *   g = W_g x, u = W_u x, h = gelu_tanh(g) * u, y = W_d h,
 * all in double.  Reading: the pages name no activation; GELU in its tanh
 * form is the gated-FFN activation of the Gemma model family. */
void orc_expert_ffn(const uint8_t *blob, int D, int F, const double *x, double *y)
{
    double *W = (double *)malloc(sizeof(double) * (size_t)F * (size_t)D);
    double *g = (double *)malloc(sizeof(double) * (size_t)F);
    double *u = (double *)malloc(sizeof(double) * (size_t)F);
    double *h = (double *)malloc(sizeof(double) * (size_t)F);
    orc_dequant(blob, D, F, 0, W);
    for (int n = 0; n < F; ++n) {
        double a = 0.0;
        for (int k = 0; k < D; ++k) a += W[(size_t)n * D + k] * x[k];
        g[n] = a;
    }
    orc_dequant(blob, D, F, 1, W);
    for (int n = 0; n < F; ++n) {
        double a = 0.0;
        for (int k = 0; k < D; ++k) a += W[(size_t)n * D + k] * x[k];
        u[n] = a;
    }
    for (int n = 0; n < F; ++n) h[n] = orc_gelu_tanh(g[n]) * u[n];
    orc_dequant(blob, D, F, 2, W); /* [D][F] */
    for (int r = 0; r < D; ++r) {
        double a = 0.0;
        for (int n = 0; n < F; ++n) a += W[(size_t)r * F + n] * h[n];
        y[r] = a;
    }
    free(W); free(g); free(u); free(h);
}

/* --------------------------------------------------------------- router
 * 8-bit router over E experts ([hada] "Estructura de ejecucion": the router
 * weights are 8-bit; [stork] each MoE layer has its own small router).  Reading taken: symmetric int8 weights with an
 * fp16 scale per group of 64 inputs and no offset; an optional fp32 per-expert
 * logit bias is added last (the synthetic popularity bias).
 *
 * The fp32 result decides the top-8 ids, so it is computed in the kernel's
 * precision with this fixed order (every step one correctly rounded fp32 FMA):
 *   S_g    = fma chain over k ascending inside group g, starting from 0:
 *            S <- fma(float(q[e][k]), float(x[k]), S)
 *   acc    = fma chain over groups g ascending, starting from 0:
 *            acc <- fma(float(s[e][g]), S_g, acc)
 *   logit  = acc + bias[e]   (one fp32 add; skipped when bias is NULL)
 */
void orc_router_logits(const uint16_t *x_bf16, const int8_t *wq, const uint16_t *ws_f16,
                       const float *bias, int E, int D, int G, float *logits)
{
    int ng = D / G;
    for (int e = 0; e < E; ++e) {
        float acc = 0.0f;
        for (int g = 0; g < ng; ++g) {
            float S = 0.0f;
            for (int k = g * G; k < (g + 1) * G; ++k)
                S = fmaf((float)wq[(size_t)e * D + k], orc_bf16_to_f32(x_bf16[k]), S);
            acc = fmaf((float)orc_f16_to_f64(ws_f16[(size_t)e * ng + g]), S, acc);
        }
        if (bias) acc = acc + bias[e];
        logits[e] = acc;
    }
}

/* Top-K ([stork] "Por que la mayor parte...": per token the router keeps the
 * 8 most relevant of the 128 experts; [hada] the CPU receives those 8 ids).  Order: logit descending, ties
 * broken by the lower expert id (reading: the pages give no tie rule).
 * Returns 0, or -1 when any logit is NaN (no order exists then). */
int orc_topk(const float *logits, int E, int K, int32_t *ids)
{
    unsigned char *taken;
    if (E <= 0 || K <= 0 || K > E) return -1;
    for (int e = 0; e < E; ++e)
        if (isnan(logits[e])) return -1;
    taken = (unsigned char *)calloc((size_t)E, 1);
    for (int i = 0; i < K; ++i) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e]) continue;
            if (best < 0 || logits[e] > logits[best]) best = e;
        }
        taken[best] = 1;
        ids[i] = best;
    }
    free(taken);
    return 0;
}

/* Gate weights (reading: the pages only say "top-8"; the weights are taken as
 * a softmax restricted to the selected experts): over the K selected logits,
 * in double,
 *   w_i = exp(l_i - m) / sum_j exp(l_j - m),  m = max_j l_j,
 * which equals the softmax over all E experts renormalised to the K chosen. */
void orc_gate_weights(const float *logits, const int32_t *ids, int K, double *w)
{
    double m = -INFINITY, z = 0.0;
    for (int i = 0; i < K; ++i) m = fmax(m, (double)logits[ids[i]]);
    for (int i = 0; i < K; ++i) { w[i] = exp((double)logits[ids[i]] - m); z += w[i]; }
    for (int i = 0; i < K; ++i) w[i] /= z;
}

/* ----------------------------------------------------------- whole layer
 * One token through the layer ([yodev] "Por que funciona": the per-token loop;
 * [hada] "Proceso de generacion de tokens"): router -> top-K -> gate weights
 * -> shared-expert branch and routed experts -> combine
 *   y = y_shared + sum_{i=0..K-1} w_i * y_{ids[i]}    (i ascending).
 * Reading: the shared branch is added with weight 1 (the pages only say that
 * the shared and routed outputs are combined).
 * expert_blobs[e] points at expert e's blob (which memory tier holds it does
 * not change the arithmetic).  Returns 0, or -1 on NaN logits. */
int orc_moe_token(int D, int E, int K, int F, int FS, int G,
                  const uint16_t *x_bf16,
                  const int8_t *wq, const uint16_t *ws_f16, const float *bias,
                  const uint8_t *shared_blob, const uint8_t *const *expert_blobs,
                  int32_t *ids, double *gate_w, float *logits, double *y)
{
    double *x = (double *)malloc(sizeof(double) * (size_t)D);
    double *ye = (double *)malloc(sizeof(double) * (size_t)D);
    int rc;
    orc_router_logits(x_bf16, wq, ws_f16, bias, E, D, G, logits);
    rc = orc_topk(logits, E, K, ids);
    if (rc != 0) { free(x); free(ye); return rc; }
    orc_gate_weights(logits, ids, K, gate_w);
    for (int k = 0; k < D; ++k) x[k] = (double)orc_bf16_to_f32(x_bf16[k]);
    if (shared_blob)
        orc_expert_ffn(shared_blob, D, FS, x, y);
    else
        for (int r = 0; r < D; ++r) y[r] = 0.0;
    for (int i = 0; i < K; ++i) {
        orc_expert_ffn(expert_blobs[ids[i]], D, F, x, ye);
        for (int r = 0; r < D; ++r) y[r] += gate_w[i] * ye[r];
    }
    free(x); free(ye);
    return 0;
}

/* -------------------------------------------------------------- LFU plan
 * Per-layer expert slot cache ([stork] "Mas inteligente que tu RAM": each of
 * the 30 layers keeps 16 of its 128 experts in an LFU cache, and a miss loads
 * the expert and replaces the least frequently used one currently resident;
 * [hada] "Proceso de generacion de tokens": the top-8 ids are checked against
 * the layer's 16-slot LFU and misses are filled by bounded parallel reads).
 *
 * State (caller-owned): count[E], last_use[E], slot_of[E] (-1: not resident),
 * expert_in[S] (-1: empty); all zero / -1 at cold start.
 * Readings where the pages are silent:
 *   - count[e] is the number of (token, k) selections of e so far; it persists
 *     across evictions (frequency over the whole history);
 *   - the victim is the resident expert with the smallest (count, last_use,
 *     expert id), never one selected by the current wave;
 *   - an empty slot, lowest index first, is used before any eviction;
 *   - distinct selected experts are handled in ascending id order, in waves of
 *     at most S experts (a decode token, K = 8 <= S, is one wave);
 *   - all counts of the call are added before the first wave;
 *   - after a wave, last_use[e] = step + 1 for each of its experts.
 * Outputs: pair_slot[T*K] (slot holding the pair's expert during its wave),
 * and per distinct expert u (ascending id): u_expert, u_slot, u_hit (1 hit,
 * 0 miss), u_victim (evicted expert or -1), u_wave.  *n_u = number of distinct
 * experts.  Returns the number of waves, or -1 on an out-of-range id.
 *
 * Replacement-policy variants ([yodev] "La parte que se gana la confianza":
 * the project logged which cache policies lost to LFU, without defining
 * them; these readings are the plain ones), all with the same waves,
 * pinning, empty-slot and last_use rules:
 *   ORC_POLICY_LFU        the rule above;
 *   ORC_POLICY_LRU        victim = smallest (last_use, expert id);
 *   ORC_POLICY_LFU_DECAY  LFU whose counts are halved (integer shift) at the
 *                         start of every call whose step is a positive
 *                         multiple of decay_period, before the call's
 *                         selections are added;
 *   ORC_POLICY_LFU_IN_CACHE  LFU whose count of an expert restarts at 0 when
 *                         it is evicted (frequency while resident). */
int orc_cache_plan(int E, int S, int policy, uint32_t decay_period,
                   uint32_t *count, uint32_t *last_use,
                   int32_t *slot_of, int32_t *expert_in,
                   const int32_t *ids, int T, int K, uint32_t step,
                   int32_t *pair_slot, int32_t *u_expert, int32_t *u_slot,
                   int32_t *u_hit, int32_t *u_victim, int32_t *u_wave, int *n_u)
{
    int n = 0, waves;
    unsigned char *sel;
    if (policy < ORC_POLICY_LFU || policy > ORC_POLICY_LFU_IN_CACHE) return -1;
    sel = (unsigned char *)calloc((size_t)E, 1);
    for (int p = 0; p < T * K; ++p) {
        if (ids[p] < 0 || ids[p] >= E) { free(sel); return -1; }
        sel[ids[p]] = 1;
    }
    if (policy == ORC_POLICY_LFU_DECAY && decay_period > 0u && step > 0u && step % decay_period == 0u)
        for (int e = 0; e < E; ++e) count[e] >>= 1;
    for (int p = 0; p < T * K; ++p) count[ids[p]] += 1u;
    for (int e = 0; e < E; ++e)
        if (sel[e]) u_expert[n++] = e;
    *n_u = n;
    waves = (n + S - 1) / S;
    for (int w = 0; w < waves; ++w) {
        int lo = w * S, hi = (w + 1) * S < n ? (w + 1) * S : n;
        for (int i = lo; i < hi; ++i) {
            int e = u_expert[i], slot = -1;
            u_wave[i] = w;
            u_victim[i] = -1;
            if (slot_of[e] >= 0) {
                u_hit[i] = 1;
                u_slot[i] = slot_of[e];
                continue;
            }
            u_hit[i] = 0;
            for (int s = 0; s < S; ++s)
                if (expert_in[s] < 0) { slot = s; break; }
            if (slot < 0) {
                int victim = -1;
                for (int s = 0; s < S; ++s) {
                    int r = expert_in[s], pinned = 0;
                    for (int j = lo; j < hi; ++j)
                        if (u_expert[j] == r) { pinned = 1; break; }
                    if (pinned) continue;
                    if (policy == ORC_POLICY_LRU) {
                        if (victim < 0 || last_use[victim] > last_use[r] ||
                            (last_use[victim] == last_use[r] && victim > r))
                            victim = r;
                    } else if (victim < 0 ||
                        count[r] < count[victim] ||
                        (count[r] == count[victim] &&
                         (last_use[r] < last_use[victim] ||
                          (last_use[r] == last_use[victim] && r < victim))))
                        victim = r;
                }
                slot = slot_of[victim];
                slot_of[victim] = -1;
                if (policy == ORC_POLICY_LFU_IN_CACHE) count[victim] = 0u;
                u_victim[i] = victim;
            }
            slot_of[e] = slot;
            expert_in[slot] = e;
            u_slot[i] = slot;
        }
        for (int i = lo; i < hi; ++i) {
            int e = u_expert[i];
            for (int p = 0; p < T * K; ++p)
                if (ids[p] == e) pair_slot[p] = u_slot[i];
            last_use[e] = step + 1u;
        }
    }
    free(sel);
    return waves;
}

int orc_lfu_plan(int E, int S, uint32_t *count, uint32_t *last_use,
                 int32_t *slot_of, int32_t *expert_in,
                 const int32_t *ids, int T, int K, uint32_t step,
                 int32_t *pair_slot, int32_t *u_expert, int32_t *u_slot,
                 int32_t *u_hit, int32_t *u_victim, int32_t *u_wave, int *n_u)
{
    return orc_cache_plan(E, S, ORC_POLICY_LFU, 0u, count, last_use, slot_of, expert_in, ids, T, K, step,
                          pair_slot, u_expert, u_slot, u_hit, u_victim, u_wave, n_u);
}

/* --------------------------------------------------- layer chaining step
 * Not a step of the MoE layer itself: what the tests and the benchmark put
 * between two MoE layers so that layer l+1 is routed on layer l's output.
 * The pages run the routed layers in order, token by token ([hada] "Proceso
 * de generacion de tokens": the routed-layer loop repeats for every token;
 * [yodev] "Por que funciona": per layer the router, the fetch plan, the reads
 * and the combine), so a layer's experts are only known once the layers below
 * it have run; the rest of the model between two MoE layers is out of scope
 * and stood in for by a residual stream and an RMS normalisation without a
 * weight (a stated choice, not the model's own block):
 *   r_out = r_in + y,   x_next = bf16( r_out / sqrt(mean(r_out^2) + 1e-6) ).
 * fp64 arithmetic; bf16 rounding is round to nearest, ties to even, straight
 * from the double value (orc_f64_to_bf16). */

/* bfloat16 (1 sign, 8 exponent bits with bias 127, 7 fraction bits) nearest
 * to v, ties to the even pattern; beyond the largest finite value (half an
 * ulp past it) the result is infinity.  NaN gives the quiet NaN 0x7FC0. */
uint16_t orc_f64_to_bf16(double v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v), q;
    int e;
    if (isnan(v)) return 0x7FC0u;
    if (a == 0.0) return sign;
    frexp(a, &e);                       /* a = m * 2^e, 0.5 <= m < 1 */
    if (e < -125) e = -125;             /* subnormal range: spacing 2^-133 */
    q = rint(ldexp(a, 8 - e));          /* significand in units of the spacing 2^(e-8), ties to even */
    a = ldexp(q, e - 8);
    if (a >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80u);
    {
        float f = (float)a;             /* exact: at most 8 significant bits */
        uint32_t u;
        memcpy(&u, &f, sizeof u);
        return (uint16_t)(sign | (u >> 16));
    }
}

void orc_residual_rmsnorm(const double *r_in, const double *y, int D, double *r_out, uint16_t *x_next)
{
    double ss = 0.0, rms;
    for (int i = 0; i < D; ++i) {
        r_out[i] = r_in[i] + y[i];
        ss += r_out[i] * r_out[i];
    }
    rms = sqrt(ss / (double)D + 1e-6);
    for (int i = 0; i < D; ++i) x_next[i] = orc_f64_to_bf16(r_out[i] / rms);
}

/* ------------------------------------------------ prefill token grouping
 * Prefill chunk ([hada] "Proceso de generacion de tokens": the prompt is
 * prefilled in chunks of up to 128 tokens so that an expert fetched once
 * serves several rows): the T*K (token, k) pairs are grouped by expert.
 * Definition: pairs in ascending (expert id, pair index p = t*K + k) order;
 * offsets[e] .. offsets[e+1] delimit expert e's pairs.
 * Returns 0, or -1 on an out-of-range id. */
int orc_group_by_expert(const int32_t *ids, int T, int K, int E,
                        int32_t *offsets, int32_t *pairs)
{
    int pos = 0;
    for (int p = 0; p < T * K; ++p)
        if (ids[p] < 0 || ids[p] >= E) return -1;
    for (int e = 0; e < E; ++e) {
        offsets[e] = pos;
        for (int p = 0; p < T * K; ++p)
            if (ids[p] == e) pairs[pos++] = p;
    }
    offsets[E] = pos;
    return 0;
}

/* ------------------------------------------------ decode attention
 * The other per-token kernel of the layer loop ([hada] "Proceso de generacion
 * de tokens": decode attention is an exact split-K/V method; the fp16 KV cache
 * is a bounded ring for the 25 sliding-window layers and linear storage for the
 * 5 full-attention layers, as also in [yodev] "Por que funciona: el A4B del
 * nombre").  "Exact" means that splitting the keys and values into parts and
 * merging them changes nothing but rounding, so the oracle is softmax attention
 * itself, written out:
 *   o[h] = sum_p w[h][p] * v[g][slot(p)],
 *   w[h] = softmax over p of (scale * q[h] . k[g][slot(p)]),  g = h / (Hq / Hkv).
 * Readings where the pages are silent: a cache of capacity cap holds position p
 * in slot p mod cap (a ring; a linear cache has cap >= n, so its slot is p);
 * the token at position n-1 attends to positions max(0, n - cap) .. n-1, its
 * own key included (the window is the ring's capacity); query heads that share
 * a KV head are consecutive.  Layouts: q bf16 [Hq][hd]; k, v binary16
 * [Hkv][cap][hd]; o fp64 [Hq][hd].  Arithmetic in fp64; the largest score is
 * subtracted before exponentiating, which leaves the softmax unchanged.
 * Returns 0, or -1 on bad sizes (n < 1, cap < 1, Hq not a multiple of Hkv). */
int orc_attn_decode(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                    int Hq, int Hkv, int hd, int cap, int n, double scale, double *o)
{
    if (n < 1 || cap < 1 || Hkv < 1 || hd < 1 || Hq < Hkv || Hq % Hkv != 0) return -1;
    const int grp = Hq / Hkv;
    const int first = n > cap ? n - cap : 0;
    const int np = n - first;
    double *w = (double *)malloc(sizeof(double) * (size_t)np);
    if (!w) return -1;
    for (int h = 0; h < Hq; ++h) {
        const int g = h / grp;
        const uint16_t *kg = k + (size_t)g * (size_t)cap * (size_t)hd;
        const uint16_t *vg = v + (size_t)g * (size_t)cap * (size_t)hd;
        double mx = -INFINITY, z = 0.0;
        for (int i = 0; i < np; ++i) {
            const size_t slot = (size_t)((first + i) % cap);
            double a = 0.0;
            for (int d = 0; d < hd; ++d)
                a += (double)orc_bf16_to_f32(q[(size_t)h * hd + d]) * orc_f16_to_f64(kg[slot * hd + d]);
            w[i] = scale * a;
            if (w[i] > mx) mx = w[i];
        }
        for (int i = 0; i < np; ++i) {
            w[i] = exp(w[i] - mx);
            z += w[i];
        }
        for (int d = 0; d < hd; ++d) {
            double acc = 0.0;
            for (int i = 0; i < np; ++i) {
                const size_t slot = (size_t)((first + i) % cap);
                acc += w[i] * orc_f16_to_f64(vg[slot * hd + d]);
            }
            o[(size_t)h * hd + d] = acc / z;
        }
    }
    free(w);
    return 0;
}
