/*
 * CSA2 oracle -- a plain, slow, obviously-correct CPU restatement of the CSA2
 * sparse-attention step over an FP4 KV cache described in
 * "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression".
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path (the
 * CUDA library and its Python binding) never calls, links or imports it, and
 * the two share no code, headers, tables or constants.
 *
 * Citations name the web page and the section on it:
 *   [jaehun "2) CSA2"]       jaehun.me review, section "2) CSA2" (paper sec. 2.3)
 *   [jaehun "3) FP4 ..."]     jaehun.me review, section "3) FP4 main KV + SWA
 *                            Bounded Replay" (paper sec. 2.4.4, 3.2.2)
 *   [jaehun toy example]     jaehun.me review, section "작동 원리" (paper 2.3.1, 4.2.1)
 *   [ainewsway "encoder"]    ainewsway.com article, paragraph on the cache axes
 * Where the pages are silent the reading used is stated at the function.
 *
 * Precision: scalar codecs work in IEEE binary32 exactly as the readings
 * define them (so that every quantised byte is decided in the same precision
 * as the kernels); dot products that feed selection and attention are exact
 * integers or binary64.  Build with -ffp-contract=off so no multiply-add is
 * fused behind our back; fmaf() is called explicitly where a fused operation
 * is part of a definition.
 *
 * Parity status: every function below is pinned by tests/test_oracle_*.py
 * except the absolute semantics of the m=2 gate (the pages lost the formula)
 * and the block score of the hierarchical pool (not given); those two are
 * pinned only by invariants of our reading.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* bit helpers                                                              */
/* ------------------------------------------------------------------------ */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bf16 is the upper 16 bits of a binary32. */
float orc_bf16_to_f32(uint16_t h) { return f32_from_bits((uint32_t)h << 16); }

/* Round a binary64 value to the nearest bf16 (ties to even) in one step. */
uint16_t orc_f64_to_bf16(double x)
{
    if (isnan(x)) return 0x7FC0;
    if (x == 0.0) return signbit(x) ? 0x8000 : 0x0000;
    double a = fabs(x);
    int e = ilogb(a);                 /* a in [2^e, 2^(e+1)) */
    if (e < -126) e = -126;           /* subnormal spacing is 2^-133 */
    double q = nearbyint(ldexp(a, 7 - e));   /* 8 significant bits, RNE */
    double r = ldexp(q, e - 7);
    uint16_t h;
    if (r > 3.3895313892515355e38) h = 0x7F80;            /* overflow to inf */
    else h = (uint16_t)(bits_from_f32((float)r) >> 16);    /* r is exact in bf16 */
    return signbit(x) ? (uint16_t)(h | 0x8000) : h;
}

/* ------------------------------------------------------------------------ */
/* E2M1 and E4M3 decode, straight from the bit definitions                  */
/* [jaehun "3) FP4 ..."]: main KV entries are E2M1 values with one E4M3     */
/* scale per 16 channels; the window KV stays FP8 (E4M3 reading).           */
/* ------------------------------------------------------------------------ */

/* E2M1: sign | 2 exponent bits (bias 1) | 1 mantissa bit, no inf/NaN. */
double orc_e2m1_value(int code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* E4M3 ("FN"): sign | 4 exponent bits (bias 7) | 3 mantissa bits.
 * S.1111.111 is NaN; there is no infinity; the largest finite value is 448. */
double orc_e4m3_value(int byte)
{
    int s = (byte >> 7) & 1, e = (byte >> 3) & 15, m = byte & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    mag = (e == 0) ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* ------------------------------------------------------------------------ */
/* Encoders: nearest representable magnitude, ties to the even code,        */
/* saturating at the largest finite value (the magnitudes are increasing in */
/* the code, so "even code" is "even mantissa").                            */
/* ------------------------------------------------------------------------ */

static double e4m3_mag[127];   /* codes 0x00..0x7E */
static double e2m1_mag[8];     /* codes 0..7       */

__attribute__((constructor)) static void build_tables(void)
{
    for (int c = 0; c < 127; ++c) e4m3_mag[c] = orc_e4m3_value(c);
    for (int c = 0; c < 8; ++c) e2m1_mag[c] = orc_e2m1_value(c);
}

/* Index of the nearest entry of an increasing table to a >= 0; ties go to
 * the even index; anything above the last entry maps to the last entry. */
static int nearest_even(const double *tab, int n, double a)
{
    int lo = 0, hi = n - 1;
    if (a >= tab[n - 1]) return n - 1;
    while (lo < hi) {                  /* first index with tab[i] >= a */
        int mid = (lo + hi) / 2;
        if (tab[mid] >= a) hi = mid; else lo = mid + 1;
    }
    if (lo == 0) return 0;
    double dl = a - tab[lo - 1], dh = tab[lo] - a;
    if (dl < dh) return lo - 1;
    if (dh < dl) return lo;
    return ((lo - 1) % 2 == 0) ? lo - 1 : lo;
}

/* binary32 -> E4M3, round to nearest even, saturate to +-448; the sign of
 * the input is kept (so -0 and negative values that round to zero give 0x80). */
uint8_t orc_e4m3_encode(float x)
{
    if (isnan(x)) return 0x7F;
    int c = nearest_even(e4m3_mag, 127, fabs((double)x));
    return (uint8_t)(c | (signbit(x) ? 0x80 : 0));
}

/* binary32 -> E2M1 code, same rule, saturating at +-6, sign kept. */
uint8_t orc_e2m1_encode(float y)
{
    int c = nearest_even(e2m1_mag, 8, fabs((double)y));
    return (uint8_t)(c | (signbit(y) ? 0x8 : 0));
}

/* ------------------------------------------------------------------------ */
/* FP4 entry quantisation  [jaehun "3) FP4 ..."]                            */
/* Reading (the pages give only the format): per group of 16 channels       */
/*   amax = max |x|;  scale byte = E4M3(amax / 6.0f) (binary32 division);   */
/*   s = decoded scale;  code_c = E2M1(x_c / s) (binary32 division);        */
/*   amax == 0 or s == 0 -> scale byte 0x00 and all codes 0.                */
/* Packing: byte i of the row = code(ch 2i) | code(ch 2i+1) << 4.           */
/* ------------------------------------------------------------------------ */

void orc_quant_fp4_row(const float *x, int D, uint8_t *codes, uint8_t *scales)
{
    for (int g = 0; g < D / 16; ++g) {
        const float *xg = x + 16 * g;
        float amax = 0.0f;
        uint8_t cg[16];
        for (int c = 0; c < 16; ++c) { float a = fabsf(xg[c]); if (a > amax) amax = a; }
        uint8_t sb = (amax == 0.0f) ? 0 : orc_e4m3_encode(amax / 6.0f);
        float s = (float)orc_e4m3_value(sb);
        for (int c = 0; c < 16; ++c) cg[c] = (s == 0.0f) ? 0 : orc_e2m1_encode(xg[c] / s);
        scales[g] = (s == 0.0f) ? 0 : sb;
        for (int i = 0; i < 8; ++i) codes[8 * g + i] = (uint8_t)(cg[2 * i] | (cg[2 * i + 1] << 4));
    }
}

/* Dequantised value of channel c of an FP4 row: E2M1 x E4M3 (exact). */
double orc_fp4_value(const uint8_t *codes, const uint8_t *scales, int c)
{
    int code = (codes[c / 2] >> ((c & 1) * 4)) & 0xF;
    return orc_e2m1_value(code) * orc_e4m3_value(scales[c / 16]);
}

/* ------------------------------------------------------------------------ */
/* e^x for x in [-80, 0] in binary32, for the m=2 gate.                      */
/* Textbook method (Cody & Waite range reduction, Taylor polynomial):       */
/*   n = rint(x * log2 e),  r = x - n*ln2 with ln2 split into a 17-bit head */
/*   (n*head is exact for |n| < 128) and a rounded tail, both subtracted by  */
/*   fused multiply-add;  e^r ~ sum_{k<=7} r^k/k!  by Horner's rule with     */
/*   fmaf (|r| <= ln2/2, truncation < r^8/8! < 6e-9);  result = p * 2^n      */
/*   (2^n built from its exponent field; exact, n >= -116 stays normal).     */
/* Arguments below -80 return +0.  The constants are the binary32 roundings */
/* of log2(e), 1/k! and of ln2 - head.                                       */
/* ------------------------------------------------------------------------ */

float orc_exp_neg(float x)
{
    const float log2e = 0x1.715476p+0f;
    const float ln2_head = 0x1.62e4p-1f;
    const float ln2_tail = 0x1.7f7d1cp-20f;
    if (!(x >= -80.0f)) return 0.0f;
    if (x > 0.0f) x = 0.0f;
    float n = rintf(x * log2e);
    float r = fmaf(-n, ln2_head, x);
    r = fmaf(-n, ln2_tail, r);
    float p = 0x1.a01a02p-13f;          /* 1/7! */
    p = fmaf(p, r, 0x1.6c16c2p-10f);    /* 1/6! */
    p = fmaf(p, r, 0x1.111112p-7f);     /* 1/5! */
    p = fmaf(p, r, 0x1.555556p-5f);     /* 1/4! */
    p = fmaf(p, r, 0x1.555556p-3f);     /* 1/3! */
    p = fmaf(p, r, 0.5f);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    float two_n = f32_from_bits((uint32_t)((int)n + 127) << 23);
    return p * two_n;
}

/* ------------------------------------------------------------------------ */
/* m = 2 sequence compression  [jaehun "2) CSA2"; ainewsway "encoder"]       */
/* Pages: m consecutive tokens become one entry, no overlap between entries, */
/* no absolute-position term; the projection formula (eq. 1, W_KV, W_Z) was  */
/* lost.  Reading: a per-channel softmax over the pair's gate logits,        */
/*   d = |z_a - z_b|, e = exp(-d), s = 1 + e, w_big = 1/s, w_small = e/s,    */
/*   the larger logit takes w_big;  pooled = fl(w_a*kv_a) + fl(w_b*kv_b).   */
/* All in binary32 so the kernels can reproduce the pooled value exactly.   */
/* ------------------------------------------------------------------------ */

void orc_pool_pair(const uint16_t *kv_a, const uint16_t *kv_b,
                   const uint16_t *z_a, const uint16_t *z_b, int D, float *out)
{
    for (int c = 0; c < D; ++c) {
        float za = orc_bf16_to_f32(z_a[c]), zb = orc_bf16_to_f32(z_b[c]);
        float d = fabsf(za - zb);
        float e = orc_exp_neg(-d);
        float s = 1.0f + e;
        float w_big = 1.0f / s, w_small = e / s;
        float wa = (za >= zb) ? w_big : w_small;
        float wb = (za >= zb) ? w_small : w_big;
        float ta = wa * orc_bf16_to_f32(kv_a[c]);
        float tb = wb * orc_bf16_to_f32(kv_b[c]);
        out[c] = ta + tb;
    }
}

/* ------------------------------------------------------------------------ */
/* FP8 scaling rule used for the indexer key and the indexer query:         */
/*   s = amax / 448 (binary32), codes = E4M3(v / s); amax == 0 -> s = 0 and  */
/*   all codes 0.                                                            */
/* ------------------------------------------------------------------------ */

void orc_quant_fp8_row(const float *v, int n, uint8_t *codes, float *scale)
{
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) { float a = fabsf(v[i]); if (a > amax) amax = a; }
    float s = amax / 448.0f;
    for (int i = 0; i < n; ++i) codes[i] = (s == 0.0f) ? 0 : orc_e4m3_encode(v[i] / s);
    *scale = s;
}

/* Indexer query of one head  (FP8 contraction named with the score formula):
 * bf16 q -> binary32 -> the FP8 rule above. */
void orc_quant_query(const uint16_t *q, int dI, uint8_t *codes, float *scale)
{
    float v[1024];
    for (int i = 0; i < dI; ++i) v[i] = orc_bf16_to_f32(q[i]);
    orc_quant_fp8_row(v, dI, codes, scale);
}

/* ------------------------------------------------------------------------ */
/* Indexer key projected from the main KV  [jaehun "2) CSA2": the indexer K  */
/* is obtained by projecting the main KV instead of a separate compression   */
/* path].  Reading: project the dequantised stored FP4 entry x^ with a bf16  */
/* matrix W[D][dI]:  k_i = sum_c x^_c * W[c][i], in binary32 as ONE fused    */
/* multiply-add chain per output, channels in ascending order, starting from */
/* +0:  acc = fmaf(x^_c, W[c][i], acc) for c = 0 .. D-1.  That is the plain  */
/* left-to-right sum of the definition with each product fused into its      */
/* addition; the pages give no other order.                                  */
/* ------------------------------------------------------------------------ */

void orc_project_key(const uint8_t *codes, const uint8_t *scales, const uint16_t *W,
                     int D, int dI, float *k)
{
    float xh[4096];
    for (int c = 0; c < D; ++c) xh[c] = (float)orc_fp4_value(codes, scales, c);
    for (int i = 0; i < dI; ++i) {
        float acc = 0.0f;
        for (int c = 0; c < D; ++c) acc = fmaf(xh[c], orc_bf16_to_f32(W[(size_t)c * dI + i]), acc);
        k[i] = acc;
    }
}

/* The key's FP8 form: the rule above (s_k = amax/448, E4M3 codes of k/s_k). */
void orc_index_key(const uint8_t *codes, const uint8_t *scales, const uint16_t *W,
                   int D, int dI, uint8_t *ik, float *ik_scale)
{
    float k[1024];
    orc_project_key(codes, scales, W, D, dI, k);
    orc_quant_fp8_row(k, dI, ik, ik_scale);
}

/* ------------------------------------------------------------------------ */
/* Append  [jaehun "2) CSA2", "3) FP4 ..."]                                  */
/* New tokens p = pos0[b] + tau (tau < T) of sequence b.  Entry e covers     */
/* tokens m*e .. m*e+m-1 (no overlap, no position term) and is written when  */
/* its last token arrives; a token that opens an incomplete pair waits in    */
/* the pending buffer.  Each written entry is quantised to FP4 and its       */
/* indexer key is projected.  n_entries[b] = floor((pos0[b]+T)/m).           */
/* The window cache gets E4M3(x / s_swa) of each of the last min(T, W_cap)   */
/* tokens in ring slot p mod W_cap.                                          */
/* Layouts: codes[B][cap][D/2], scales[B][cap][D/16], ik[B][cap][dI],        */
/* ik_scale[B][cap], kv/gate/kv_swa[B][T][D], pending_*[B][D],               */
/* swa_rows[B][W_cap][D].  Pointers for an absent part may be NULL.          */
/* ------------------------------------------------------------------------ */

void orc_append(int B, int cap, int D, int dI, int m,
                uint8_t *codes, uint8_t *scales, uint8_t *ik, float *ik_scale,
                int32_t *n_entries, uint16_t *pending_kv, uint16_t *pending_gate,
                const uint16_t *kv, const uint16_t *gate, const uint16_t *W,
                uint8_t *swa_rows, int W_cap, float s_swa, const uint16_t *kv_swa,
                const int32_t *pos0, int T)
{
    float *x = (float *)malloc(sizeof(float) * D);
    for (int b = 0; b < B; ++b) {
        int p0 = pos0[b];
        if (codes) {
            for (int tau = 0; tau < T; ++tau) {
                int p = p0 + tau;
                const uint16_t *kv_t = kv + ((size_t)b * T + tau) * D;
                if (m == 1) {
                    for (int c = 0; c < D; ++c) x[c] = orc_bf16_to_f32(kv_t[c]);
                } else {
                    const uint16_t *g_t = gate + ((size_t)b * T + tau) * D;
                    if (p % 2 == 0) {                     /* opens a pair */
                        if (tau == T - 1) {
                            memcpy(pending_kv + (size_t)b * D, kv_t, 2 * (size_t)D);
                            memcpy(pending_gate + (size_t)b * D, g_t, 2 * (size_t)D);
                        }
                        continue;
                    }
                    const uint16_t *kv_a, *g_a;           /* token p-1 */
                    if (tau == 0) { kv_a = pending_kv + (size_t)b * D; g_a = pending_gate + (size_t)b * D; }
                    else { kv_a = kv_t - D; g_a = g_t - D; }
                    orc_pool_pair(kv_a, kv_t, g_a, g_t, D, x);
                }
                int e = (m == 1) ? p : (p - 1) / 2;
                if (e < 0 || e >= cap) continue;
                size_t r = (size_t)b * cap + e;
                orc_quant_fp4_row(x, D, codes + r * (D / 2), scales + r * (D / 16));
                if (ik) orc_index_key(codes + r * (D / 2), scales + r * (D / 16), W, D, dI,
                                      ik + r * dI, ik_scale + r);
            }
            if (n_entries) n_entries[b] = (p0 + T) / m;
        }
        if (swa_rows) {
            int first = T - (T < W_cap ? T : W_cap);
            for (int tau = first; tau < T; ++tau) {
                int p = p0 + tau;
                const uint16_t *xs = kv_swa + ((size_t)b * T + tau) * D;
                uint8_t *row = swa_rows + ((size_t)b * W_cap + (p % W_cap)) * D;
                for (int c = 0; c < D; ++c) row[c] = orc_e4m3_encode(orc_bf16_to_f32(xs[c]) / s_swa);
            }
        }
    }
    free(x);
}

/* ------------------------------------------------------------------------ */
/* CED decoder-KV projection  [jaehun "1) CED": the decoder's global KV is   */
/* obtained by projecting the final encoder hidden state H_{L/2} with each   */
/* decoder layer's W_KV^l (the flowchart edge names W_KV^l and W_Z^l; the     */
/* equation itself was lost)].  Reading: the plainest linear projection,     */
/* kv_t = H_t W_KV, with no bias and no normalisation.  W_Z can only enter   */
/* as the gate of an m >= 2 pooling; the decoder's caches are m = 1, where a */
/* softmax over one token is 1, so the decoder entry is kv_t itself.         */
/* Value: the exact sum of the bf16 products rounded once to binary32.  The  */
/* products are exact in binary64; the sum is carried in binary64 with       */
/* Neumaier's compensated summation (error ~2^-106 relative to the sum of    */
/* magnitudes, far below binary32's rounding) and then rounded to binary32.  */
/* H: [d] bf16 (one token), W: [d][D] bf16, kv: [D].                         */
/* ------------------------------------------------------------------------ */

void orc_project_kv(const uint16_t *H, int d, const uint16_t *W, int D, float *kv)
{
    for (int c = 0; c < D; ++c) {
        double s = 0.0, comp = 0.0;
        for (int i = 0; i < d; ++i) {
            double x = (double)orc_bf16_to_f32(H[i]) * (double)orc_bf16_to_f32(W[(size_t)i * D + c]);
            double t = s + x;
            if (fabs(s) >= fabs(x)) comp += (s - t) + x;
            else comp += (x - t) + s;
            s = t;
        }
        kv[c] = (float)(s + comp);
    }
}

/* Append T projected tokens per sequence to an m = 1 main cache: token p =  */
/* pos0[b] + tau is entry p; kv = H W_KV (above), then the FP4 entry and its */
/* indexer key exactly as orc_append does; n_entries[b] = pos0[b] + T.       */
/* H: [B][T][d] bf16.                                                        */
void orc_append_project(int B, int cap, int D, int dI,
                        uint8_t *codes, uint8_t *scales, uint8_t *ik, float *ik_scale, int32_t *n_entries,
                        const uint16_t *H, int d, const uint16_t *W_kv, const uint16_t *W_ik,
                        const int32_t *pos0, int T)
{
    float *x = (float *)malloc(sizeof(float) * D);
    for (int b = 0; b < B; ++b) {
        for (int tau = 0; tau < T; ++tau) {
            int e = pos0[b] + tau;
            if (e < 0 || e >= cap) continue;
            orc_project_kv(H + ((size_t)b * T + tau) * d, d, W_kv, D, x);
            size_t r = (size_t)b * cap + e;
            orc_quant_fp4_row(x, D, codes + r * (D / 2), scales + r * (D / 16));
            orc_index_key(codes + r * (D / 2), scales + r * (D / 16), W_ik, D, dI, ik + r * dI, ik_scale + r);
        }
        n_entries[b] = pos0[b] + T;
    }
    free(x);
}

/* ------------------------------------------------------------------------ */
/* Visibility: entry e is complete for a query at token t iff m*e+m-1 <= t.  */
/* n_vis = min(n_entries, floor((t+1)/m)).                                   */
/* ------------------------------------------------------------------------ */

int orc_n_visible(int n_entries, int t, int m)
{
    int v = (t + 1) / m;
    return v < n_entries ? v : n_entries;
}

/* ------------------------------------------------------------------------ */
/* Indexer score  (score_j = sum_h w_h ReLU(q_h . k_j) as an FP8 contraction) */
/* logit_hj = s_q,h * s_k,j * <q8_h, k8_j>; the FP8 dot is exact: every E4M3 */
/* value times 2^9 is an integer, so the dot is an int64 sum times 2^-18.    */
/* score_j = sum_h w_h * max(0, logit_hj) in binary64, ascending h.  No      */
/* further scale (w absorbs it).                                             */
/* ik: [n][dI] E4M3 of this sequence; q: [H_I][dI] bf16; w: [H_I].           */
/* ------------------------------------------------------------------------ */

void orc_index_scores_at(const uint8_t *ik, const float *ik_scale, const int32_t *ent,
                         int n, int dI, const uint16_t *q, const float *w, int H_I,
                         double *out);

static int64_t e4m3_int(int byte)   /* E4M3 value * 2^9, exact */
{
    double v = orc_e4m3_value(byte);
    return (int64_t)llround(ldexp(v, 9));
}

void orc_index_scores(const uint8_t *ik, const float *ik_scale, int n, int dI,
                      const uint16_t *q, const float *w, int H_I, double *out)
{
    orc_index_scores_at(ik, ik_scale, NULL, n, dI, q, w, H_I, out);
}

/* Same, for a list of entries: out[j] scores entry ent[j]; ent[j] < 0 gives
 * -inf (absent).  ent == NULL means entries 0..n-1. */
void orc_index_scores_at(const uint8_t *ik, const float *ik_scale, const int32_t *ent,
                         int n, int dI, const uint16_t *q, const float *w, int H_I,
                         double *out)
{
    uint8_t *q8 = (uint8_t *)malloc((size_t)H_I * dI);
    float *sq = (float *)malloc(sizeof(float) * H_I);
    int64_t *qi = (int64_t *)malloc(sizeof(int64_t) * (size_t)H_I * dI);
    int64_t lut[256];
    for (int v = 0; v < 256; ++v) lut[v] = ((v & 0x7F) == 0x7F) ? 0 : e4m3_int(v);
    for (int h = 0; h < H_I; ++h) {
        orc_quant_query(q + (size_t)h * dI, dI, q8 + (size_t)h * dI, &sq[h]);
        for (int i = 0; i < dI; ++i) qi[(size_t)h * dI + i] = lut[q8[(size_t)h * dI + i]];
    }
    for (int j = 0; j < n; ++j) {
        int e = ent ? ent[j] : j;
        if (e < 0) { out[j] = -INFINITY; continue; }
        const uint8_t *kj = ik + (size_t)e * dI;
        double score = 0.0;
        for (int h = 0; h < H_I; ++h) {
            int64_t dot = 0;
            for (int i = 0; i < dI; ++i) dot += qi[(size_t)h * dI + i] * lut[kj[i]];
            double logit = (double)sq[h] * (double)ik_scale[e] * ldexp((double)dot, -18);
            score += (double)w[h] * (logit > 0.0 ? logit : 0.0);
        }
        out[j] = score;
    }
    free(q8); free(sq); free(qi);
}

/* ------------------------------------------------------------------------ */
/* Top-K  [jaehun "2) CSA2": each Full layer picks Top-512; toy example]     */
/* Reading: the K largest finite scores; ties -> smaller index; fewer than K */
/* finite scores -> all of them, the rest of the output is -1.  The output  */
/* lists the chosen indices in ascending order.  Non-finite = absent.        */
/* ------------------------------------------------------------------------ */

typedef struct { double s; int32_t i; } cand_t;

static int by_score_desc_index_asc(const void *pa, const void *pb)
{
    const cand_t *a = (const cand_t *)pa, *b = (const cand_t *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->i > b->i) - (a->i < b->i);
}

static int by_index(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

void orc_topk(const double *s, int n, int K, int32_t *out)
{
    cand_t *c = (cand_t *)malloc(sizeof(cand_t) * (size_t)(n > 0 ? n : 1));
    int cnt = 0;
    for (int j = 0; j < n; ++j) if (isfinite(s[j])) { c[cnt].s = s[j]; c[cnt].i = j; ++cnt; }
    qsort(c, (size_t)cnt, sizeof(cand_t), by_score_desc_index_asc);
    int take = cnt < K ? cnt : K;
    for (int k = 0; k < take; ++k) out[k] = c[k].i;
    qsort(out, (size_t)take, sizeof(int32_t), by_index);
    for (int k = take; k < K; ++k) out[k] = -1;
    free(c);
}

/* ------------------------------------------------------------------------ */
/* Hierarchical candidate pool  [jaehun "2) CSA2": the first Full layer     */
/* scans all entries and builds a pool of at most 2,048 blocks x 8 positions */
/* that the later Reindex layers rescore].  Reading: block b = entries       */
/* [8b, 8b+8) of the n scored ones; block score = max of its finite scores; */
/* blocks without one are absent; the P best blocks (ties -> smaller block)  */
/* in ascending order, -1 padded.  Max guarantees Full's Top-K is inside.    */
/* ------------------------------------------------------------------------ */

void orc_block_pool(const double *s, int n, int P, int32_t *out)
{
    int nb = (n + 7) / 8;
    double *bs = (double *)malloc(sizeof(double) * (size_t)(nb > 0 ? nb : 1));
    for (int b = 0; b < nb; ++b) {
        double mx = -INFINITY;
        for (int j = 8 * b; j < 8 * b + 8 && j < n; ++j) if (isfinite(s[j]) && s[j] > mx) mx = s[j];
        bs[b] = mx;
    }
    orc_topk(bs, nb, P, out);
    free(bs);
}

/* ------------------------------------------------------------------------ */
/* Reindex scoring  [jaehun "2) CSA2", toy example: a Reindex layer keeps    */
/* the inherited KV (and, our reading, the inherited indexer K) and rescores */
/* only the pool with its own indexer query].  Column c = 8*g + r is entry   */
/* pool[g]*8 + r; columns whose block is -1 or whose entry is not visible    */
/* score -inf (absent).                                                      */
/* ------------------------------------------------------------------------ */

void orc_reindex_scores(const uint8_t *ik, const float *ik_scale, int n_vis, int dI,
                        const uint16_t *q, const float *w, int H_I,
                        const int32_t *pool, int P, double *out)
{
    int32_t *ent = (int32_t *)malloc(sizeof(int32_t) * (size_t)(P > 0 ? P : 1) * 8);
    for (int g = 0; g < P; ++g)
        for (int r = 0; r < 8; ++r) {
            int e = pool[g] >= 0 ? pool[g] * 8 + r : -1;
            ent[8 * g + r] = (e >= 0 && e < n_vis) ? e : -1;
        }
    orc_index_scores_at(ik, ik_scale, ent, 8 * P, dI, q, w, H_I, out);
    free(ent);
}

/* Map selected pool columns back to entry ids (-1 stays -1). */
void orc_columns_to_entries(const int32_t *cols, int K, const int32_t *pool, int32_t *out)
{
    for (int k = 0; k < K; ++k)
        out[k] = cols[k] < 0 ? -1 : pool[cols[k] / 8] * 8 + cols[k] % 8;
}

/* ------------------------------------------------------------------------ */
/* Sparse MQA attention  [jaehun "2) CSA2": global sparse retrieval plus a   */
/* 128-token local window; ainewsway: 128-token sliding window combined with */
/* global sparse retrieval].  One query token at position t, H heads that    */
/* share one KV (K = V).  The attended set is the selected FP4 entries       */
/* (idx != -1, each listed index once per listing) plus the window rows of   */
/* tokens max(0, t-window+1) .. t.  logit = scale * q_h . x^ (binary64),     */
/* one softmax over the whole set, out_h = sum p x^, rounded to bf16 (RNE).  */
/* x^ of an FP4 entry = E2M1 * E4M3; of a window row = E4M3 * s_swa.  No     */
/* position term anywhere.  An empty set gives zeros.                        */
/* q: [H][D] bf16; codes/scales of this sequence: [cap][D/2], [cap][D/16];   */
/* swa_rows of this sequence: [W_cap][D]; out: [H][D] bf16.                  */
/* ------------------------------------------------------------------------ */

void orc_attention(const uint16_t *q, int H, int D,
                   const uint8_t *codes, const uint8_t *scales, int cap,
                   const int32_t *idx, int K,
                   const uint8_t *swa_rows, int W_cap, float s_swa, int window, int t,
                   float scale, uint16_t *out)
{
    int lo = t - window + 1; if (lo < 0) lo = 0;
    int nsel = 0;
    for (int k = 0; k < K; ++k) if (idx[k] >= 0 && idx[k] < cap) ++nsel;
    int nwin = (window > 0 && t >= 0) ? t - lo + 1 : 0;
    int n = nsel + nwin;
    double *x = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * D);
    double *lg = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    int r = 0;
    for (int k = 0; k < K; ++k) {
        if (idx[k] < 0 || idx[k] >= cap) continue;
        const uint8_t *cr = codes + (size_t)idx[k] * (D / 2);
        const uint8_t *sr = scales + (size_t)idx[k] * (D / 16);
        for (int c = 0; c < D; ++c) x[(size_t)r * D + c] = orc_fp4_value(cr, sr, c);
        ++r;
    }
    for (int p = lo; p <= t && nwin > 0; ++p) {
        const uint8_t *row = swa_rows + (size_t)(p % W_cap) * D;
        for (int c = 0; c < D; ++c) x[(size_t)r * D + c] = orc_e4m3_value(row[c]) * (double)s_swa;
        ++r;
    }
    for (int h = 0; h < H; ++h) {
        const uint16_t *qh = q + (size_t)h * D;
        uint16_t *oh = out + (size_t)h * D;
        if (n == 0) { for (int c = 0; c < D; ++c) oh[c] = 0; continue; }
        double mx = -INFINITY;
        for (int j = 0; j < n; ++j) {
            double acc = 0.0;
            for (int c = 0; c < D; ++c) acc += (double)orc_bf16_to_f32(qh[c]) * x[(size_t)j * D + c];
            lg[j] = (double)scale * acc;
            if (lg[j] > mx) mx = lg[j];
        }
        double l = 0.0;
        for (int j = 0; j < n; ++j) { lg[j] = exp(lg[j] - mx); l += lg[j]; }
        for (int c = 0; c < D; ++c) {
            double o = 0.0;
            for (int j = 0; j < n; ++j) o += lg[j] * x[(size_t)j * D + c];
            oh[c] = orc_f64_to_bf16(o / l);
        }
    }
    free(x); free(lg);
}
