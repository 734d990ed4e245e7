/*
 * la_oracle.c -- plain, slow, obviously correct CPU oracle for the recurrent-state
 * step of linear attention.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and
 * the benchmark's CPU-baseline leg call it; the product library never does, and this
 * file shares no code, header or constant generator with the CUDA path.
 *
 * What it computes (written from the pages, not from any listing):
 *
 *   "Gated DeltaNet" (inferencex glossary), Technical definition: at each step the
 *   running state is decayed by a gate, corrected by a rank-one delta-rule term and
 *   projected by the query.
 *   "Seven Architectures Replacing KV Cache With Bounded Mutable State", section
 *   "ONNX LinearAttention / FlashInfer": update_rule in {linear (plain additive update),
 *   gated (update decayed by a gate), delta (delta correction, no gate), gated_delta}; state
 *   tensors past_state / present_state of shape (B, H_kv, d_k, d_v).
 *   Same page, section "Kimi Linear": the channel-wise gate of Kimi Delta Attention,
 *   S_t = Diag(alpha_t) S_{t-1} + beta_t k_t (v_t - (Diag(alpha_t) S_{t-1})^T k_t)^T with
 *   alpha_t in R^{d_k} (rule kda); with a scalar gate it is the Gated DeltaNet rule.
 *
 * Per state head, with S (d_k x d_v), per token t:
 *
 *   u_t = b_t * (v_t - c_t * S_{t-1}^T k_t)
 *   S_t = a_t * S_{t-1} + k_t u_t^T
 *   o_t = scale * S_t^T q_t                 (readout from the UPDATED state)
 *
 *   rule         a_t   b_t    c_t
 *   linear       1     1      0
 *   gated        g_t   1      0
 *   delta        1     beta_t 1
 *   gated_delta  g_t   beta_t g_t
 *   kda          Diag(alpha_t) beta_t, prediction from the decayed state Diag(alpha_t) S_{t-1}
 *
 * For kda the gate array holds d_k values per (token, head): row i of the state decays by
 * alpha_t[i].  The formula's "Diag(alpha_t) S_{t-1}^T k_t" is read as the transpose of the
 * decayed state times k (the only reading whose shapes agree when d_k != d_v).
 *
 * Arithmetic is IEEE double throughout.  Rounding happens only where the method
 * stores a value ("Recurrent state" glossary, Why it matters: state stored in BF16
 * while computed in a wider type): the state after each decode step, the state at the
 * end of a scan, and each output o_t (to the io type).  Storage types: 0 = f64 (no
 * rounding), 1 = f32, 2 = bf16 (round-to-nearest-even from the IEEE definition), 3 = q8
 * (the mixed INT8 / BF16 format below; state only).
 *
 * Layouts (row-major, last index contiguous):
 *   pool   [n_slots, H_v, d_k, d_v]
 *   q, k   [B or T, H_qk, d_k]        state head h reads q/k head h / (H_v / H_qk)
 *   v, o   [B or T, H_v, d_v]
 *   g, beta[B or T, H_v]               (kda: g is [B or T, H_v, d_k])
 *
 * Slots ("Recurrent state" glossary, Engineering details / Why it matters; "Gated
 * DeltaNet" glossary, Why it matters): a request reads its state from read_slot[b]
 * (NULL: slot b) and writes it to write_slot[b] (NULL: slot b), so a checkpoint slot
 * survives a step that continues from it.  A request whose slot index is outside the
 * pool is skipped (its outputs and destination are left untouched) and an error bit
 * is returned: 1 = read slot, 2 = write slot, 4 = bad cu_seqlens.
 */
#include "la_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define LAO_ERR_READ_SLOT 1
#define LAO_ERR_WRITE_SLOT 2
#define LAO_ERR_CU_SEQLENS 4

/* ---- rounding to a storage type ------------------------------------------------ */

/* Largest finite bfloat16: (2 - 2^-7) * 2^127. */
static const double BF16_MAX = 3.38953138925153547590470800371487866880e38;

/* Round x to the nearest bfloat16 value, ties to even.  bfloat16 has 8 significant
 * bits, the binary32 exponent range, and subnormals down to 2^-133.  The quantum of
 * the binade holding |x| is 2^(e-8) where |x| = m 2^e, m in [0.5, 1); below the
 * normal range the quantum stays 2^-133.  x / quantum is exact in double, rint()
 * rounds it half-to-even, and the product is exact again.  A result beyond the
 * largest finite value overflows to infinity.  NaN stays NaN. */
double lao_round_bf16(double x)
{
    if (isnan(x) || isinf(x) || x == 0.0) return x;
    int e;
    frexp(fabs(x), &e);
    int qe = e - 8;
    if (qe < -133) qe = -133;
    double y = ldexp(rint(ldexp(x, -qe)), qe);
    if (fabs(y) > BF16_MAX) return copysign(INFINITY, x);
    return y;
}

double lao_round_to(double x, int dtype)
{
    if (dtype == LAO_F32) return (double)(float)x;
    if (dtype == LAO_BF16) return lao_round_bf16(x);
    return x;
}

/* ---- mixed INT8 / BF16 state storage ------------------------------------------------
 *
 * "Seven Architectures ...", sections "ONNX LinearAttention / FlashInfer" and the
 * Practical Implications: DAMP stores the recurrent state at about 9.9 bits per value,
 * the high-risk key channels in a higher precision and the rest in INT8, a 69.1 %
 * reduction of state storage.  The pages fix no layout; the reading taken here (format
 * code 3, "q8"), per (slot, head) tile of d_k x d_v:
 *   - a per-head mask of d_k bits marks the n_hp high-precision key channels (rows);
 *   - every other row is stored as INT8 codes in groups of 32 consecutive columns, each
 *     group with an FP32 scale s = absmax * fl(1/127) (absmax of the group's FP32 values)
 *     and inverse scale inv = fl(1/absmax) * 127 (every operation a correctly rounded FP32
 *     one); code = rint(x * inv) clamped to [-127, 127] (NaN to 0), decoded as code * s;
 *     a group of zeros has s = inv = 0 and codes 0;
 *   - high-precision rows are stored in BF16 (round to nearest even).
 * Byte layout of a tile: codes [d_k - n_hp][d_v] int8, then scales [d_k - n_hp][d_v / 32]
 * float32, then BF16 rows [n_hp][d_v]; rows of each block in increasing row index.  The
 * codes are decided in FP32 from the FP32 value (the value the kernels hold).  With
 * n_hp = d_k / 8 the tile holds 9.875 bits per value. */

size_t lao_q8_tile_bytes(int dk, int dv, int n_hp)
{
    const size_t n8 = (size_t)(dk - n_hp);
    return n8 * (size_t)dv + n8 * (size_t)(dv / 32) * 4 + (size_t)n_hp * (size_t)dv * 2;
}

static int hp_row(const unsigned *mask, int i)
{
    return (int)((mask[i / 32] >> (i % 32)) & 1u);
}

static unsigned short bf16_bits(float x)
{
    float y = (float)lao_round_bf16((double)x);
    unsigned u;
    memcpy(&u, &y, 4);
    return (unsigned short)(u >> 16);
}

static void q8_encode_tile(const float *x, int dk, int dv, int n_hp, const unsigned *mask, unsigned char *out)
{
    const int n8 = dk - n_hp, ng = dv / 32;
    unsigned char *sc = out + (size_t)n8 * dv;
    unsigned char *hp = sc + (size_t)n8 * ng * 4;
    int r8 = 0, rh = 0;
    for (int i = 0; i < dk; ++i) {
        const float *row = x + (size_t)i * dv;
        if (hp_row(mask, i)) {
            for (int j = 0; j < dv; ++j) {
                unsigned short b = bf16_bits(row[j]);
                memcpy(hp + ((size_t)rh * dv + j) * 2, &b, 2);
            }
            ++rh;
            continue;
        }
        for (int gi = 0; gi < ng; ++gi) {
            float amax = 0.0f;
            for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(row[gi * 32 + j]));
            const float k127 = 1.0f / 127.0f;
            const float s = amax > 0.0f ? amax * k127 : 0.0f;
            const float inv = amax > 0.0f ? (1.0f / amax) * 127.0f : 0.0f;
            memcpy(sc + ((size_t)r8 * ng + gi) * 4, &s, 4);
            for (int j = 0; j < 32; ++j) {
                const float y = rintf(row[gi * 32 + j] * inv);
                const float c = isnan(y) ? 0.0f : fminf(fmaxf(y, -127.0f), 127.0f);
                out[(size_t)r8 * dv + gi * 32 + j] = (unsigned char)(signed char)c;
            }
        }
        ++r8;
    }
}

static void q8_decode_tile(const unsigned char *in, int dk, int dv, int n_hp, const unsigned *mask, float *x)
{
    const int n8 = dk - n_hp, ng = dv / 32;
    const unsigned char *sc = in + (size_t)n8 * dv;
    const unsigned char *hp = sc + (size_t)n8 * ng * 4;
    int r8 = 0, rh = 0;
    for (int i = 0; i < dk; ++i) {
        float *row = x + (size_t)i * dv;
        if (hp_row(mask, i)) {
            for (int j = 0; j < dv; ++j) {
                unsigned short b;
                memcpy(&b, hp + ((size_t)rh * dv + j) * 2, 2);
                unsigned u = (unsigned)b << 16;
                memcpy(&row[j], &u, 4);
            }
            ++rh;
            continue;
        }
        for (int gi = 0; gi < ng; ++gi) {
            float s;
            memcpy(&s, sc + ((size_t)r8 * ng + gi) * 4, 4);
            for (int j = 0; j < 32; ++j)
                row[gi * 32 + j] = (float)(signed char)in[(size_t)r8 * dv + gi * 32 + j] * s;
        }
        ++r8;
    }
}

/* x [n][H][dk][dv] float <-> q8 slots [n][H][tile bytes]; masks [H][dk / 32].  Returns -1
 * when a head's mask does not hold exactly n_hp rows, else 0. */
static int q8_masks_ok(const unsigned *masks, int H, int dk, int n_hp)
{
    for (int h = 0; h < H; ++h) {
        int c = 0;
        for (int i = 0; i < dk; ++i) c += hp_row(masks + (size_t)h * (dk / 32), i);
        if (c != n_hp) return 0;
    }
    return 1;
}

int lao_q8_encode(const float *x, int n, int H, int dk, int dv, int n_hp, const unsigned *masks,
                  unsigned char *out)
{
    if (!q8_masks_ok(masks, H, dk, n_hp)) return -1;
    const size_t tb = lao_q8_tile_bytes(dk, dv, n_hp);
    for (int t = 0; t < n * H; ++t)
        q8_encode_tile(x + (size_t)t * dk * dv, dk, dv, n_hp, masks + (size_t)(t % H) * (dk / 32), out + (size_t)t * tb);
    return 0;
}

int lao_q8_decode(const unsigned char *in, int n, int H, int dk, int dv, int n_hp, const unsigned *masks, float *x)
{
    if (!q8_masks_ok(masks, H, dk, n_hp)) return -1;
    const size_t tb = lao_q8_tile_bytes(dk, dv, n_hp);
    for (int t = 0; t < n * H; ++t)
        q8_decode_tile(in + (size_t)t * tb, dk, dv, n_hp, masks + (size_t)(t % H) * (dk / 32), x + (size_t)t * dk * dv);
    return 0;
}

/* Rounds one tile to its storage type: elementwise for f64 / f32 / bf16; for q8 the
 * FP32 value encoded and decoded again (mask: the head's d_k / 32 mask words). */
static void round_tile(double *S, int dk, int dv, int dtype, const unsigned *mask)
{
    const size_t tile = (size_t)dk * dv;
    if (dtype != LAO_Q8) {
        for (size_t e = 0; e < tile; ++e) S[e] = lao_round_to(S[e], dtype);
        return;
    }
    int n_hp = 0;
    for (int i = 0; i < dk; ++i) n_hp += hp_row(mask, i);
    float *x = (float *)malloc(sizeof(float) * (tile ? tile : 1));
    unsigned char *b = (unsigned char *)malloc(lao_q8_tile_bytes(dk, dv, n_hp) + 1);
    if (!x || !b || !tile) { free(x); free(b); return; }
    for (size_t e = 0; e < tile; ++e) x[e] = (float)S[e];
    q8_encode_tile(x, dk, dv, n_hp, mask, b);
    q8_decode_tile(b, dk, dv, n_hp, mask, x);
    for (size_t e = 0; e < tile; ++e) S[e] = (double)x[e];
    free(x);
    free(b);
}

/* ---- one state head, one token ------------------------------------------------- */

static void rule_coefficients(int rule, double g, double beta, double *a, double *b, double *c)
{
    switch (rule) {
    case LAO_RULE_LINEAR:      *a = 1.0; *b = 1.0;  *c = 0.0; break;
    case LAO_RULE_GATED:       *a = g;   *b = 1.0;  *c = 0.0; break;
    case LAO_RULE_DELTA:       *a = 1.0; *b = beta; *c = 1.0; break;
    default: /* gated_delta */ *a = g;   *b = beta; *c = g;   break;
    }
}

/* S (dk x dv, in/out) <- a S + k u^T with u = b (v - c S^T k); then, for each of the nq
 * queries q_r = q + r * q_stride, o_r = scale * S_new^T q_r stored at o + r * o_stride.
 * For kda (alpha != NULL, dk values): S <- Diag(alpha) S + k u^T with
 * u = beta (v - (Diag(alpha) S)^T k).  u is scratch of length dv. */
static void token_update(int rule, int dk, int dv, double *S, int nq, const double *q, size_t q_stride,
                         const double *k, const double *v, double g, const double *alpha, double beta,
                         double scale, double *o, size_t o_stride, double *u)
{
    double a, b, c;
    rule_coefficients(rule, g, beta, &a, &b, &c);
    if (rule == LAO_RULE_KDA) { b = beta; c = 1.0; }
    for (int j = 0; j < dv; ++j) {
        double pj = 0.0; /* (S^T k)_j, or ((Diag(alpha) S)^T k)_j */
        for (int i = 0; i < dk; ++i)
            pj += (rule == LAO_RULE_KDA ? alpha[i] * S[(size_t)i * dv + j] : S[(size_t)i * dv + j]) * k[i];
        u[j] = b * (v[j] - c * pj);
    }
    for (int i = 0; i < dk; ++i) {
        const double ai = rule == LAO_RULE_KDA ? alpha[i] : a;
        for (int j = 0; j < dv; ++j)
            S[(size_t)i * dv + j] = ai * S[(size_t)i * dv + j] + k[i] * u[j];
    }
    for (int r = 0; r < nq; ++r, q += q_stride, o += o_stride)
        for (int j = 0; j < dv; ++j) {
            double oj = 0.0; /* (S_new^T q)_j */
            for (int i = 0; i < dk; ++i) oj += S[(size_t)i * dv + j] * q[i];
            o[j] = scale * oj;
        }
}

static int head_group(int n_qk_heads, int n_v_heads, int h)
{
    return h / (n_v_heads / n_qk_heads);
}

/* Head bookkeeping of one call.  Default direction (n_q_heads == 0): q and k have
 * n_qk_heads heads and state head h reads q/k head h / (H_v / H_qk), one output per state
 * head.  Query-group direction of the ONNX operator (n_q_heads > 0; "Seven Architectures
 * ...", ONNX section: each KV head and its state shared by a group of query heads): k has
 * one head per state head, q and o have n_q_heads heads, and query head i reads state head
 * i / (n_q_heads / H_v); the state is updated once per state head. */
typedef struct {
    int nk;      /* k heads */
    int nqh;     /* q heads */
    int grp;     /* queries per state head (1 in the default direction) */
    int no;      /* o heads */
} heads_t;

static heads_t heads_of(int n_qk_heads, int n_v_heads, int n_q_heads)
{
    heads_t hd;
    if (n_q_heads > 0) {
        hd.nk = n_v_heads; hd.nqh = n_q_heads; hd.grp = n_q_heads / n_v_heads; hd.no = n_q_heads;
    } else {
        hd.nk = n_qk_heads; hd.nqh = n_qk_heads; hd.grp = 1; hd.no = n_v_heads;
    }
    return hd;
}

/* q row of the first query of state head h, k row of state head h (token or request row t) */
static size_t q_row(heads_t hd, int n_qk_heads, int n_v_heads, int n_q_heads, size_t t, int h)
{
    return t * hd.nqh + (n_q_heads > 0 ? (size_t)h * hd.grp : (size_t)head_group(n_qk_heads, n_v_heads, h));
}
static size_t k_row(heads_t hd, int n_qk_heads, int n_v_heads, int n_q_heads, size_t t, int h)
{
    return t * hd.nk + (n_q_heads > 0 ? (size_t)h : (size_t)head_group(n_qk_heads, n_v_heads, h));
}

/* ---- batched decode step -------------------------------------------------------- */

static int step_impl(int rule, int n_qk_heads, int n_v_heads, int n_q_heads, int dk, int dv,
                     const double *src_pool, int src_slots,
                     double *dst_pool, int dst_slots, int dst_dtype,
                     const int *read_slot, const int *write_slot, int B,
                     const double *q, const double *k, const double *v, int io_dtype,
                     const double *g, const double *beta, double scale, double *o, const unsigned *q8_masks)
{
    const heads_t hd = heads_of(n_qk_heads, n_v_heads, n_q_heads);
    const size_t tile = (size_t)dk * dv;
    const size_t slot = (size_t)n_v_heads * tile;
    int err = 0;
    /* New states are computed for every request before any is written, so a request
     * that reads and writes the same slot sees its old state. */
    double *next = (double *)malloc(sizeof(double) * (B > 0 ? (size_t)B : 1) * slot);
    unsigned char *ok = (unsigned char *)calloc(B > 0 ? (size_t)B : 1, 1);
    if (!next || !ok) { free(next); free(ok); return -1; }

    for (int b = 0; b < B; ++b) {
        int rs = read_slot ? read_slot[b] : b;
        int ws = write_slot ? write_slot[b] : b;
        if (rs < 0 || rs >= src_slots) { err |= LAO_ERR_READ_SLOT; continue; }
        if (ws < 0 || ws >= dst_slots) { err |= LAO_ERR_WRITE_SLOT; continue; }
        ok[b] = 1;
    }

#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < n_v_heads; ++h) {
            if (!ok[b]) continue;
            int rs = read_slot ? read_slot[b] : b;
            double *S = next + (size_t)b * slot + (size_t)h * tile;
            double *u = (double *)malloc(sizeof(double) * (size_t)dv);
            memcpy(S, src_pool + (size_t)rs * slot + (size_t)h * tile, sizeof(double) * tile);
            double *ob = o + ((size_t)b * hd.no + (size_t)h * hd.grp) * dv;
            token_update(rule, dk, dv, S, hd.grp,
                         q + q_row(hd, n_qk_heads, n_v_heads, n_q_heads, (size_t)b, h) * dk, (size_t)dk,
                         k + k_row(hd, n_qk_heads, n_v_heads, n_q_heads, (size_t)b, h) * dk,
                         v + ((size_t)b * n_v_heads + h) * dv,
                         g && rule != LAO_RULE_KDA ? g[(size_t)b * n_v_heads + h] : 1.0,
                         rule == LAO_RULE_KDA ? g + ((size_t)b * n_v_heads + h) * dk : NULL,
                         beta ? beta[(size_t)b * n_v_heads + h] : 1.0,
                         scale, ob, (size_t)dv, u);
            for (int j = 0; j < dv * hd.grp; ++j) ob[j] = lao_round_to(ob[j], io_dtype);
            round_tile(S, dk, dv, dst_dtype, q8_masks ? q8_masks + (size_t)h * (dk / 32) : NULL);
            free(u);
        }
    }

    for (int b = 0; b < B; ++b) {
        if (!ok[b]) continue;
        int ws = write_slot ? write_slot[b] : b;
        memcpy(dst_pool + (size_t)ws * slot, next + (size_t)b * slot, sizeof(double) * slot);
    }
    free(next);
    free(ok);
    return err;
}

int lao_step(int rule, int n_qk_heads, int n_v_heads, int dk, int dv,
             const double *src_pool, int src_slots,
             double *dst_pool, int dst_slots, int dst_dtype,
             const int *read_slot, const int *write_slot, int B,
             const double *q, const double *k, const double *v, int io_dtype,
             const double *g, const double *beta, double scale, double *o)
{
    return step_impl(rule, n_qk_heads, n_v_heads, 0, dk, dv, src_pool, src_slots, dst_pool, dst_slots, dst_dtype,
                     read_slot, write_slot, B, q, k, v, io_dtype, g, beta, scale, o, NULL);
}

/* Decode step whose destination is stored in the q8 format (masks [H_v][d_k / 32]); the
 * source pool holds decoded values. */
int lao_step_q8(int rule, int n_qk_heads, int n_v_heads, int dk, int dv,
                const double *src_pool, int src_slots, double *dst_pool, int dst_slots,
                const int *read_slot, const int *write_slot, int B,
                const double *q, const double *k, const double *v, int io_dtype,
                const double *g, const double *beta, double scale, double *o, const unsigned *q8_masks)
{
    return step_impl(rule, n_qk_heads, n_v_heads, 0, dk, dv, src_pool, src_slots, dst_pool, dst_slots, LAO_Q8,
                     read_slot, write_slot, B, q, k, v, io_dtype, g, beta, scale, o, q8_masks);
}

/* ---- short causal convolution fused ahead of the decode step ---------------------------
 *
 * "Gated DeltaNet" glossary, Engineering details: Conv1D is fused with the recurrence into
 * one kernel.  The pages give nothing else; the reading taken: before the recurrence, the
 * q, k and v projections of each token pass through a causal depthwise convolution of
 * width W along time (per channel c: y_t = sum_{j<W} w[c][j] x_{t-W+1+j}, the W - 1 earlier
 * inputs kept per request as the convolution state), optionally followed by SiLU
 * (y / (1 + e^-y)), and q and k are optionally scaled to unit length per head
 * (x / sqrt(|x|^2 + 1e-6)).  The convolution state is kept per state head: head h holds
 * the histories of its q/k head's 2 d_k channels and of its own d_v v channels, so every
 * state head owns its history (heads that share a q/k head hold equal copies).
 *
 * Layouts: xq, xk [B, H_qk, d_k], xv [B, H_v, d_v] (pre-convolution inputs, already in
 * the io type); weights wq, wk [H_qk, d_k, W], wv [H_v, d_v, W]; convolution pools
 * [n_slots, H_v, 2 d_k + d_v, W - 1] (q channels, then k, then v; oldest input first),
 * read from read_slot[b] of conv_src and written to write_slot[b] of conv_dst like the
 * recurrent state.  Post-convolution values are not rounded (the fused kernel keeps them
 * in FP32 registers). */

/* One (request, state head): post-convolution q, k (d_k each) and v (d_v) from the inputs
 * and the history `hist` ([2 d_k + d_v][W - 1]); the new history goes to `hist_out`. */
static void conv_head(int dk, int dv, int W, int act, int l2norm, const double *xq, const double *xk,
                      const double *xv, const double *wq, const double *wk, const double *wv, const double *hist,
                      double *hist_out, double *q, double *k, double *v)
{
    const int C = 2 * dk + dv;
    for (int c = 0; c < C; ++c) {
        const double *w = c < dk ? wq + (size_t)c * W : c < 2 * dk ? wk + (size_t)(c - dk) * W
                                                                  : wv + (size_t)(c - 2 * dk) * W;
        const double x = c < dk ? xq[c] : c < 2 * dk ? xk[c - dk] : xv[c - 2 * dk];
        const double *h = hist + (size_t)c * (W - 1);
        double y = w[W - 1] * x;
        for (int j = 0; j < W - 1; ++j) y += w[j] * h[j];
        if (act) y = y / (1.0 + exp(-y));
        double *dstv = c < dk ? q + c : c < 2 * dk ? k + (c - dk) : v + (c - 2 * dk);
        *dstv = y;
        double *ho = hist_out + (size_t)c * (W - 1);
        for (int j = 0; j < W - 2; ++j) ho[j] = h[j + 1];
        if (W > 1) ho[W - 2] = x;
    }
    if (l2norm) {
        double sq = 0.0, sk = 0.0;
        for (int i = 0; i < dk; ++i) { sq += q[i] * q[i]; sk += k[i] * k[i]; }
        const double rq = 1.0 / sqrt(sq + 1e-6), rk = 1.0 / sqrt(sk + 1e-6);
        for (int i = 0; i < dk; ++i) { q[i] *= rq; k[i] *= rk; }
    }
}

/* The convolution alone for B requests (dense: request b uses history b): post-convolution
 * q, k [B, H_v, d_k] (per state head) and v [B, H_v, d_v]; the new histories to hist_out. */
void lao_conv(int n_qk_heads, int n_v_heads, int dk, int dv, int W, int act, int l2norm, int B,
              const double *xq, const double *xk, const double *xv, const double *wq, const double *wk,
              const double *wv, const double *hist, double *hist_out, double *q, double *k, double *v)
{
    const size_t C = (size_t)(2 * dk + dv) * (W - 1);
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < n_v_heads; ++h) {
            const int hq = head_group(n_qk_heads, n_v_heads, h);
            const size_t t = (size_t)b * n_v_heads + h;
            conv_head(dk, dv, W, act, l2norm, xq + ((size_t)b * n_qk_heads + hq) * dk,
                      xk + ((size_t)b * n_qk_heads + hq) * dk, xv + t * dv, wq + (size_t)hq * dk * W,
                      wk + (size_t)hq * dk * W, wv + (size_t)h * dv * W, hist + t * C, hist_out + t * C,
                      q + t * dk, k + t * dk, v + t * dv);
        }
}

/* Decode step with the convolution fused ahead of it: lao_conv on the histories of the
 * read slots, then the step of lao_step with one q/k row per state head (H_qk = H_v for
 * the recurrence); the new histories go to the write slots of conv_dst. */
int lao_step_conv(int rule, int n_qk_heads, int n_v_heads, int dk, int dv,
                  const double *src_pool, int src_slots, double *dst_pool, int dst_slots, int dst_dtype,
                  const int *read_slot, const int *write_slot, int B,
                  const double *xq, const double *xk, const double *xv, int io_dtype,
                  const double *g, const double *beta, double scale, double *o,
                  int W, int act, int l2norm, const double *wq, const double *wk, const double *wv,
                  const double *conv_src, double *conv_dst)
{
    const size_t C = (size_t)(2 * dk + dv) * (W - 1);
    const size_t cslot = (size_t)n_v_heads * C;
    int err = 0;
    for (int b = 0; b < B; ++b) {
        int rs = read_slot ? read_slot[b] : b, ws = write_slot ? write_slot[b] : b;
        if (rs < 0 || rs >= src_slots) err |= LAO_ERR_READ_SLOT;
        if (ws < 0 || ws >= dst_slots) err |= LAO_ERR_WRITE_SLOT;
    }
    if (err) return err;
    double *hist = (double *)calloc((size_t)B * cslot + 1, sizeof(double));
    double *hout = (double *)malloc(sizeof(double) * ((size_t)B * cslot + 1));
    double *q = (double *)malloc(sizeof(double) * ((size_t)B * n_v_heads * dk + 1));
    double *k = (double *)malloc(sizeof(double) * ((size_t)B * n_v_heads * dk + 1));
    double *v = (double *)malloc(sizeof(double) * ((size_t)B * n_v_heads * dv + 1));
    if (!hist || !hout || !q || !k || !v) { free(hist); free(hout); free(q); free(k); free(v); return -1; }
    for (int b = 0; b < B; ++b)
        memcpy(hist + (size_t)b * cslot, conv_src + (size_t)(read_slot ? read_slot[b] : b) * cslot,
               sizeof(double) * cslot);
    lao_conv(n_qk_heads, n_v_heads, dk, dv, W, act, l2norm, B, xq, xk, xv, wq, wk, wv, hist, hout, q, k, v);
    err = step_impl(rule, n_v_heads, n_v_heads, 0, dk, dv, src_pool, src_slots, dst_pool, dst_slots, dst_dtype,
                    read_slot, write_slot, B, q, k, v, io_dtype, g, beta, scale, o, NULL);
    for (int b = 0; b < B; ++b)
        memcpy(conv_dst + (size_t)(write_slot ? write_slot[b] : b) * cslot, hout + (size_t)b * cslot,
               sizeof(double) * cslot);
    free(hist); free(hout); free(q); free(k); free(v);
    return err;
}

/* Decode step in the query-group direction: k [B, H_v, d_k], q [B, n_q_heads, d_k],
 * o [B, n_q_heads, d_v]; query head i reads the updated state of head i / (n_q_heads / H_v). */
int lao_step_qgroups(int rule, int n_q_heads, int n_v_heads, int dk, int dv,
                     const double *src_pool, int src_slots,
                     double *dst_pool, int dst_slots, int dst_dtype,
                     const int *read_slot, const int *write_slot, int B,
                     const double *q, const double *k, const double *v, int io_dtype,
                     const double *g, const double *beta, double scale, double *o)
{
    return step_impl(rule, n_v_heads, n_v_heads, n_q_heads, dk, dv, src_pool, src_slots, dst_pool, dst_slots,
                     dst_dtype, read_slot, write_slot, B, q, k, v, io_dtype, g, beta, scale, o, NULL);
}

/* The readout of one decode step written in the rearranged form of the "Gated DeltaNet"
 * glossary (Engineering details): the decayed state times the query plus the current
 * token's contribution, a scalar (k . q) times the write vector u.
 *   o = scale * ( a * (S_{t-1}^T q) + (k . q) * u ).
 * Used only to check the identity against the direct readout of lao_step.  Dense mode
 * (request b reads slot b of src_pool); state is not written. */
void lao_readout_rearranged(int rule, int n_qk_heads, int n_v_heads, int dk, int dv,
                            const double *src_pool, int B,
                            const double *q, const double *k, const double *v,
                            const double *g, const double *beta, double scale, double *o)
{
    const size_t tile = (size_t)dk * dv;
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < n_v_heads; ++h) {
            int hq = head_group(n_qk_heads, n_v_heads, h);
            const double *S = src_pool + ((size_t)b * n_v_heads + h) * tile;
            const double *qb = q + ((size_t)b * n_qk_heads + hq) * dk;
            const double *kb = k + ((size_t)b * n_qk_heads + hq) * dk;
            const double *vb = v + ((size_t)b * n_v_heads + h) * dv;
            const int kda = rule == LAO_RULE_KDA;
            const double *al = kda ? g + ((size_t)b * n_v_heads + h) * dk : NULL;
            double a, bc, c;
            rule_coefficients(rule, g && !kda ? g[(size_t)b * n_v_heads + h] : 1.0,
                              beta ? beta[(size_t)b * n_v_heads + h] : 1.0, &a, &bc, &c);
            if (kda) { a = 1.0; c = 1.0; }
            double kq = 0.0;
            for (int i = 0; i < dk; ++i) kq += kb[i] * qb[i];
            for (int j = 0; j < dv; ++j) {
                /* kda: the decay sits on each row, so (Diag(alpha) S)^T k and (Diag(alpha) S)^T q */
                double pj = 0.0, rj = 0.0;
                for (int i = 0; i < dk; ++i) {
                    const double sij = kda ? al[i] * S[(size_t)i * dv + j] : S[(size_t)i * dv + j];
                    pj += sij * kb[i];
                    rj += sij * qb[i];
                }
                double uj = bc * (vb[j] - c * pj);
                o[((size_t)b * n_v_heads + h) * dv + j] = scale * (a * rj + kq * uj);
            }
        }
    }
}

/* ---- token-serial scan over packed variable-length sequences -------------------- */

/* Scan with intermediate checkpoints ("Gated DeltaNet" glossary, Why it matters:
 * hybrid prefix caching keeps checkpoint slots at KV-cache block boundaries; "Seven
 * Architectures ...", Limitations: state snapshots for speculative-decoding rollback).
 * With ckpt_every > 0, checkpoint j of sequence s (j < ckpt_cu[s+1] - ckpt_cu[s]) is the
 * state after the sequence's first (j + 1) * ckpt_every tokens, rounded to dst_dtype and
 * stored to dst_pool slot ckpt_slots[ckpt_cu[s] + j].  A checkpoint position beyond the
 * sequence is reported (bit 4) and skipped; an out-of-range checkpoint slot is reported
 * (bit 2) and skipped.  ckpt_every <= 0: no checkpoints (lao_scan). */
static int scan_impl(int rule, int n_qk_heads, int n_v_heads, int n_q_heads, int dk, int dv,
                     const double *src_pool, int src_slots, const int *read_slot,
                     double *dst_pool, int dst_slots, int dst_dtype, const int *write_slot,
                     int n_seqs, const int *cu_seqlens, int total_tokens,
                     const double *q, const double *k, const double *v, int io_dtype,
                     const double *g, const double *beta, double scale, double *o,
                     int ckpt_every, const int *ckpt_cu, const int *ckpt_slots, const unsigned *q8_masks)
{
    const heads_t hd = heads_of(n_qk_heads, n_v_heads, n_q_heads);
    const size_t tile = (size_t)dk * dv;
    const size_t slot = (size_t)n_v_heads * tile;
    int err = 0;
    double *next = (double *)malloc(sizeof(double) * (n_seqs > 0 ? (size_t)n_seqs : 1) * slot);
    unsigned char *ok = (unsigned char *)calloc(n_seqs > 0 ? (size_t)n_seqs : 1, 1);
    if (!next || !ok) { free(next); free(ok); return -1; }

    if (n_seqs > 0 && cu_seqlens[0] != 0) err |= LAO_ERR_CU_SEQLENS;
    for (int s = 0; s < n_seqs; ++s) {
        int t0 = cu_seqlens[s], t1 = cu_seqlens[s + 1];
        if (t0 < 0 || t1 < t0 || t1 > total_tokens) { err |= LAO_ERR_CU_SEQLENS; continue; }
        if (read_slot && (read_slot[s] < 0 || read_slot[s] >= src_slots)) { err |= LAO_ERR_READ_SLOT; continue; }
        int ws = write_slot ? write_slot[s] : s;
        if (ws < 0 || ws >= dst_slots) { err |= LAO_ERR_WRITE_SLOT; continue; }
        ok[s] = 1;
        if (ckpt_every > 0) {
            const int n_ck = ckpt_cu[s + 1] - ckpt_cu[s];
            for (int j = 0; j < n_ck; ++j) {
                if ((long long)(j + 1) * ckpt_every > (long long)(t1 - t0)) { err |= LAO_ERR_CU_SEQLENS; break; }
                const int cs = ckpt_slots[ckpt_cu[s] + j];
                if (cs < 0 || cs >= dst_slots) err |= LAO_ERR_WRITE_SLOT;
            }
        }
    }

#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int s = 0; s < n_seqs; ++s) {
        for (int h = 0; h < n_v_heads; ++h) {
            if (!ok[s]) continue;
            double *S = next + (size_t)s * slot + (size_t)h * tile;
            double *u = (double *)malloc(sizeof(double) * (size_t)dv);
            if (read_slot)
                memcpy(S, src_pool + (size_t)read_slot[s] * slot + (size_t)h * tile, sizeof(double) * tile);
            else
                memset(S, 0, sizeof(double) * tile);
            for (int t = cu_seqlens[s]; t < cu_seqlens[s + 1]; ++t) {
                double *ot = o + ((size_t)t * hd.no + (size_t)h * hd.grp) * dv;
                token_update(rule, dk, dv, S, hd.grp,
                             q + q_row(hd, n_qk_heads, n_v_heads, n_q_heads, (size_t)t, h) * dk, (size_t)dk,
                             k + k_row(hd, n_qk_heads, n_v_heads, n_q_heads, (size_t)t, h) * dk,
                             v + ((size_t)t * n_v_heads + h) * dv,
                             g && rule != LAO_RULE_KDA ? g[(size_t)t * n_v_heads + h] : 1.0,
                             rule == LAO_RULE_KDA ? g + ((size_t)t * n_v_heads + h) * dk : NULL,
                             beta ? beta[(size_t)t * n_v_heads + h] : 1.0,
                             scale, ot, (size_t)dv, u);
                for (int j = 0; j < dv * hd.grp; ++j) ot[j] = lao_round_to(ot[j], io_dtype);
                const int pos = t - cu_seqlens[s] + 1; /* tokens of this sequence consumed */
                if (ckpt_every > 0 && pos % ckpt_every == 0) {
                    const int j = pos / ckpt_every - 1;
                    if (j < ckpt_cu[s + 1] - ckpt_cu[s]) {
                        const int cs = ckpt_slots[ckpt_cu[s] + j];
                        if (cs >= 0 && cs < dst_slots) {
                            double *D = dst_pool + (size_t)cs * slot + (size_t)h * tile;
                            memcpy(D, S, sizeof(double) * tile);
                            round_tile(D, dk, dv, dst_dtype, q8_masks ? q8_masks + (size_t)h * (dk / 32) : NULL);
                        }
                    }
                }
            }
            round_tile(S, dk, dv, dst_dtype, q8_masks ? q8_masks + (size_t)h * (dk / 32) : NULL);
            free(u);
        }
    }

    for (int s = 0; s < n_seqs; ++s) {
        if (!ok[s]) continue;
        int ws = write_slot ? write_slot[s] : s;
        memcpy(dst_pool + (size_t)ws * slot, next + (size_t)s * slot, sizeof(double) * slot);
    }
    free(next);
    free(ok);
    return err;
}

int lao_scan_ckpt(int rule, int n_qk_heads, int n_v_heads, int dk, int dv,
                  const double *src_pool, int src_slots, const int *read_slot,
                  double *dst_pool, int dst_slots, int dst_dtype, const int *write_slot,
                  int n_seqs, const int *cu_seqlens, int total_tokens,
                  const double *q, const double *k, const double *v, int io_dtype,
                  const double *g, const double *beta, double scale, double *o,
                  int ckpt_every, const int *ckpt_cu, const int *ckpt_slots)
{
    return scan_impl(rule, n_qk_heads, n_v_heads, 0, dk, dv, src_pool, src_slots, read_slot, dst_pool,
                     dst_slots, dst_dtype, write_slot, n_seqs, cu_seqlens, total_tokens, q, k, v, io_dtype,
                     g, beta, scale, o, ckpt_every, ckpt_cu, ckpt_slots, NULL);
}

/* Scan whose final states (and checkpoints) are stored in the q8 format. */
int lao_scan_q8(int rule, int n_qk_heads, int n_v_heads, int dk, int dv,
                const double *src_pool, int src_slots, const int *read_slot,
                double *dst_pool, int dst_slots, const int *write_slot,
                int n_seqs, const int *cu_seqlens, int total_tokens,
                const double *q, const double *k, const double *v, int io_dtype,
                const double *g, const double *beta, double scale, double *o,
                int ckpt_every, const int *ckpt_cu, const int *ckpt_slots, const unsigned *q8_masks)
{
    return scan_impl(rule, n_qk_heads, n_v_heads, 0, dk, dv, src_pool, src_slots, read_slot, dst_pool,
                     dst_slots, LAO_Q8, write_slot, n_seqs, cu_seqlens, total_tokens, q, k, v, io_dtype,
                     g, beta, scale, o, ckpt_every, ckpt_cu, ckpt_slots, q8_masks);
}

int lao_scan(int rule, int n_qk_heads, int n_v_heads, int dk, int dv,
             const double *src_pool, int src_slots, const int *read_slot,
             double *dst_pool, int dst_slots, int dst_dtype, const int *write_slot,
             int n_seqs, const int *cu_seqlens, int total_tokens,
             const double *q, const double *k, const double *v, int io_dtype,
             const double *g, const double *beta, double scale, double *o)
{
    return lao_scan_ckpt(rule, n_qk_heads, n_v_heads, dk, dv, src_pool, src_slots, read_slot, dst_pool,
                         dst_slots, dst_dtype, write_slot, n_seqs, cu_seqlens, total_tokens, q, k, v, io_dtype,
                         g, beta, scale, o, 0, NULL, NULL);
}

/* Scan in the query-group direction (layouts as lao_step_qgroups, T rows). */
int lao_scan_qgroups(int rule, int n_q_heads, int n_v_heads, int dk, int dv,
                     const double *src_pool, int src_slots, const int *read_slot,
                     double *dst_pool, int dst_slots, int dst_dtype, const int *write_slot,
                     int n_seqs, const int *cu_seqlens, int total_tokens,
                     const double *q, const double *k, const double *v, int io_dtype,
                     const double *g, const double *beta, double scale, double *o)
{
    return scan_impl(rule, n_v_heads, n_v_heads, n_q_heads, dk, dv, src_pool, src_slots, read_slot, dst_pool,
                     dst_slots, dst_dtype, write_slot, n_seqs, cu_seqlens, total_tokens, q, k, v, io_dtype,
                     g, beta, scale, o, 0, NULL, NULL, NULL);
}

/* Scan with the convolution ahead of every token: each (sequence, head) history starts
 * from conv_src at read_slot[s] (zero when read_slot is NULL), runs through the sequence's
 * tokens, and the history after its last token goes to conv_dst at write_slot[s] (slot s
 * when NULL); an empty sequence passes its history through unchanged.  Histories have
 * src_slots / dst_slots slots like the pools.  Then the scan of lao_scan with one q/k row
 * per state head. */
int lao_scan_conv(int rule, int n_qk_heads, int n_v_heads, int dk, int dv,
                  const double *src_pool, int src_slots, const int *read_slot,
                  double *dst_pool, int dst_slots, int dst_dtype, const int *write_slot,
                  int n_seqs, const int *cu_seqlens, int total_tokens,
                  const double *xq, const double *xk, const double *xv, int io_dtype,
                  const double *g, const double *beta, double scale, double *o,
                  int W, int act, int l2norm, const double *wq, const double *wk, const double *wv,
                  const double *conv_src, double *conv_dst)
{
    const size_t C = (size_t)(2 * dk + dv) * (W - 1);
    const size_t cslot = (size_t)n_v_heads * C;
    const size_t T = total_tokens > 0 ? (size_t)total_tokens : 1;
    double *q = (double *)calloc(T * n_v_heads * dk, sizeof(double));
    double *k = (double *)calloc(T * n_v_heads * dk, sizeof(double));
    double *v = (double *)calloc(T * n_v_heads * dv, sizeof(double));
    double *hist = (double *)calloc(cslot + 1, sizeof(double));
    double *hout = (double *)calloc(cslot + 1, sizeof(double));
    if (!q || !k || !v || !hist || !hout) { free(q); free(k); free(v); free(hist); free(hout); return -1; }
    for (int s = 0; s < n_seqs; ++s) {
        const int t0 = cu_seqlens[s], t1 = cu_seqlens[s + 1];
        const int rs = read_slot ? read_slot[s] : 0, ws = write_slot ? write_slot[s] : s;
        if (t0 < 0 || t1 < t0 || t1 > total_tokens) continue;             /* reported by the scan */
        if ((read_slot && (rs < 0 || rs >= src_slots)) || ws < 0 || ws >= dst_slots) continue;
        if (read_slot) memcpy(hist, conv_src + (size_t)rs * cslot, sizeof(double) * cslot);
        else memset(hist, 0, sizeof(double) * cslot);
        for (int t = t0; t < t1; ++t) {
            lao_conv(n_qk_heads, n_v_heads, dk, dv, W, act, l2norm, 1, xq + (size_t)t * n_qk_heads * dk,
                     xk + (size_t)t * n_qk_heads * dk, xv + (size_t)t * n_v_heads * dv, wq, wk, wv, hist, hout,
                     q + (size_t)t * n_v_heads * dk, k + (size_t)t * n_v_heads * dk, v + (size_t)t * n_v_heads * dv);
            memcpy(hist, hout, sizeof(double) * cslot);
        }
        memcpy(conv_dst + (size_t)ws * cslot, hist, sizeof(double) * cslot);
    }
    const int err = scan_impl(rule, n_v_heads, n_v_heads, 0, dk, dv, src_pool, src_slots, read_slot, dst_pool,
                              dst_slots, dst_dtype, write_slot, n_seqs, cu_seqlens, total_tokens, q, k, v, io_dtype,
                              g, beta, scale, o, 0, NULL, NULL, NULL);
    free(q); free(k); free(v); free(hist); free(hout);
    return err;
}

/* ---- slot pool: whole-slot byte copies ------------------------------------------ */
/* Checkpoints and snapshots ("Recurrent state" glossary, Why it matters; "Seven
 * Architectures", ONNX section on saving and restoring state snapshots) are plain byte
 * copies of whole slots.  All sources are read before any destination is written. */

int lao_pool_copy(unsigned char *pool, size_t slot_bytes, int n_slots, int n,
                  const int *src_slots, const int *dst_slots)
{
    int err = 0;
    unsigned char *tmp = (unsigned char *)malloc(slot_bytes * (n > 0 ? (size_t)n : 1));
    if (!tmp) return -1;
    for (int i = 0; i < n; ++i) {
        if (src_slots[i] < 0 || src_slots[i] >= n_slots) { err |= LAO_ERR_READ_SLOT; continue; }
        memcpy(tmp + (size_t)i * slot_bytes, pool + (size_t)src_slots[i] * slot_bytes, slot_bytes);
    }
    for (int i = 0; i < n; ++i) {
        if (src_slots[i] < 0 || src_slots[i] >= n_slots) continue;
        if (dst_slots[i] < 0 || dst_slots[i] >= n_slots) { err |= LAO_ERR_WRITE_SLOT; continue; }
        memcpy(pool + (size_t)dst_slots[i] * slot_bytes, tmp + (size_t)i * slot_bytes, slot_bytes);
    }
    free(tmp);
    return err;
}

int lao_pool_gather(const unsigned char *pool, size_t slot_bytes, int n_slots, int n,
                    const int *slots, unsigned char *dense)
{
    int err = 0;
    for (int i = 0; i < n; ++i) {
        if (slots[i] < 0 || slots[i] >= n_slots) { err |= LAO_ERR_READ_SLOT; continue; }
        memcpy(dense + (size_t)i * slot_bytes, pool + (size_t)slots[i] * slot_bytes, slot_bytes);
    }
    return err;
}

int lao_pool_scatter(unsigned char *pool, size_t slot_bytes, int n_slots, int n,
                     const int *slots, const unsigned char *dense)
{
    int err = 0;
    for (int i = 0; i < n; ++i) {
        if (slots[i] < 0 || slots[i] >= n_slots) { err |= LAO_ERR_WRITE_SLOT; continue; }
        memcpy(pool + (size_t)slots[i] * slot_bytes, dense + (size_t)i * slot_bytes, slot_bytes);
    }
    return err;
}

int lao_pool_zero(unsigned char *pool, size_t slot_bytes, int n_slots, int n, const int *slots)
{
    int err = 0;
    for (int i = 0; i < n; ++i) {
        if (slots[i] < 0 || slots[i] >= n_slots) { err |= LAO_ERR_WRITE_SLOT; continue; }
        memset(pool + (size_t)slots[i] * slot_bytes, 0, slot_bytes);
    }
    return err;
}

/* ---- threads -------------------------------------------------------------------- */

int lao_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void lao_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
