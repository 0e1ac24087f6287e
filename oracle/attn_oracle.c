/*
 * Exact-attention oracle: plain, slow, fp64 CPU reference.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header or constant with the CUDA path, and the CUDA path never calls it.
 *
 * What it computes (the plain definition, written out):
 *   "Hardware-Aware FP4 FlashAttention-4", section "Planteamiento del
 *   Problema": attention is the product QK^T, a row softmax of the scores,
 *   then the product PV.  Section "Causal Backward Cuantizado": the forward
 *   keeps the per-row log-sum-exp normaliser (LSE) and the backward rebuilds
 *   the probabilities from it.  "FlashAttention-4发布", section "从V1到V4",
 *   first bullet: the tiled method is exact -- it reaches this same result
 *   without writing the N x N matrix -- so the oracle is the untiled
 *   definition, computed row by row with a two-pass softmax (deliberately not
 *   the online form).  Masks follow the patterns named in "El FlexAttention
 *   de PyTorch con FlashAttention-4", intro (sliding window, document
 *   masking) plus causal; grouped heads follow the FlashAttention-2 bullet of
 *   "从V1到V4" (GQA/MQA).
 *
 * Readings where the pages say nothing (each also listed in the design notes):
 *   - causal alignment when Sq != Sk is bottom-right: key j allowed for query
 *     i iff j <= i + (Sk - Sq);
 *   - window: allowed iff i+(Sk-Sq)-window_left <= j <= i+(Sk-Sq)+window_right,
 *     a negative bound meaning unbounded on that side;
 *   - document mask: token t belongs to document d iff
 *     offsets[d] <= t < offsets[d+1]; query i may see key j only if both lie
 *     in the same document.  It combines (AND) with causal and window;
 *   - grouped heads: query head hq reads key/value head hq / (Hq / Hkv);
 *   - a row with no allowed key has O = 0 and LSE = -inf;
 *   - score modifiers ("El FlexAttention de PyTorch con FlashAttention-4",
 *     intro: soft-capping and ALiBi), applied in this order to the scaled
 *     score s = scale * <q_i, k_j>: soft-capping s <- c * tanh(s / c) for a
 *     cap c > 0; ALiBi s <- s - slope_hq * |i + (Sk - Sq) - j| (a linear
 *     distance penalty per query head, measured from the bottom-right
 *     aligned diagonal); then the mask.
 *
 * Parity pins (tests, CPU only): closed forms (equal logits -> mean of V,
 * one dominant logit -> that V row, constant V -> rows of P sum to one,
 * causal row 0), library softmax / logsumexp on dense masked scores, mask
 * and GQA invariants, finite differences for the backward; the e4m3 decoder
 * against torch's float8_e4m3fn conversion for all 256 codes; for the FP4
 * Direct-P forward, the E2M1 table, brute-force nearest rounding, hand-worked
 * constant-score rows, exact agreement with the softmax for scores on the
 * E2M1 grid, integer-shift invariance, masking and the NVFP4 / MXFP4
 * decoding.  Nothing here is "parity unpinned".
 *
 * Layouts (row-major, contiguous):
 *   q, o, dq, do : [B, Sq, Hq,  D]
 *   k, v, dk, dv : [B, Sk, Hkv, D]
 *   lse          : [B, Hq, Sq]
 * Inputs are either bf16 bit patterns (uint16) converted exactly to double,
 * or doubles (used by the finite-difference tests).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int B, Hq, Hkv, Sq, Sk, D;
    double scale;
    int causal, window_left, window_right;
    const int *doc_offsets; /* host int32[num_docs + 1] or NULL */
    int num_docs;
    double softcap;             /* > 0: scores pass through softcap * tanh(s / softcap) */
    const double *alibi_slopes; /* host double[Hq] or NULL */
    /* 0: the exact softmax.  1, 2: Direct-P probabilities (affine or
     * exponential classifier, see direct_p_row); `scale` then maps the dot
     * product to log2 units. */
    int direct_p;
} oracle_shape_t;

/* ------------------------------------------------------------------ input */

static double bf16_bits_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16; /* bf16 is the top half of an fp32 */
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Copy D elements starting at element index `idx` into `out` as doubles. */
static void load_vec(const void *base, int is_bf16, size_t idx, int D, double *out) {
    if (is_bf16) {
        const uint16_t *p = (const uint16_t *)base + idx;
        for (int d = 0; d < D; ++d) out[d] = bf16_bits_to_double(p[d]);
    } else {
        const double *p = (const double *)base + idx;
        for (int d = 0; d < D; ++d) out[d] = p[d];
    }
}

static size_t q_index(const oracle_shape_t *s, int b, int i, int h) {
    return (((size_t)b * s->Sq + i) * s->Hq + h) * s->D;
}
static size_t kv_index(const oracle_shape_t *s, int b, int j, int h) {
    return (((size_t)b * s->Sk + j) * s->Hkv + h) * s->D;
}

/* ------------------------------------------------------------------- mask */

/* Document of token t, or -1 when t lies outside every document. */
static int document_of(const oracle_shape_t *s, long t) {
    for (int d = 0; d < s->num_docs; ++d)
        if (s->doc_offsets[d] <= t && t < s->doc_offsets[d + 1]) return d;
    return -1;
}

/* The mask predicate, written directly from its definition. */
static int key_allowed(const oracle_shape_t *s, long i, long j) {
    long diag = i + (long)(s->Sk - s->Sq);
    if (s->causal && j > diag) return 0;
    if (s->window_left >= 0 && j < diag - s->window_left) return 0;
    if (s->window_right >= 0 && j > diag + s->window_right) return 0;
    if (s->doc_offsets) {
        int di = document_of(s, i);
        if (di < 0 || di != document_of(s, j)) return 0;
    }
    return 1;
}

static int kv_head_of(const oracle_shape_t *s, int hq) {
    return hq / (s->Hq / s->Hkv);
}

/* --------------------------------------------------------------- forward */

/*
 * One query row.  Scores s_j = scale * <q_i, k_j> for allowed j; two passes:
 * M = max_j s_j, Z = sum_j exp(s_j - M); LSE = M + log Z;
 * P_j = exp(s_j - LSE); O = sum_j P_j v_j.
 * Work buffers: s (Sk), qi/kj (D).  kd/vd hold this head's K and V rows
 * already converted to double ([Sk][D]).
 */
/* The score of (i, j) from the raw dot product: scale, soft-cap, ALiBi. */
static double modified_score(const oracle_shape_t *s, int hq, long i, long j, double dot) {
    double x = s->scale * dot;
    if (s->softcap > 0.0) x = s->softcap * tanh(x / s->softcap);
    if (s->alibi_slopes) {
        const double dist = fabs((double)(i + (long)(s->Sk - s->Sq) - j));
        x -= s->alibi_slopes[hq] * dist;
    }
    return x;
}

/* d(score)/d(dot): the chain rule through the soft-cap (ALiBi is constant). */
static double score_grad(const oracle_shape_t *s, double dot) {
    if (s->softcap > 0.0) {
        const double t = tanh(s->scale * dot / s->softcap);
        return s->scale * (1.0 - t * t);
    }
    return s->scale;
}

static void direct_p_row(const double *y, const unsigned char *allow, long n,
                         const double *vd, int D, int classifier, double *o_out,
                         double *lse_out);

static void forward_row(const oracle_shape_t *s, int hq, const double *qi,
                        const double *kd, const double *vd, long i,
                        double *srow, unsigned char *allow,
                        double *o_out, double *lse_out) {
    const int D = s->D, Sk = s->Sk;
    double M = -INFINITY;
    long n_allowed = 0;
    for (long j = 0; j < Sk; ++j) {
        allow[j] = (unsigned char)key_allowed(s, i, j);
        if (!allow[j]) continue;
        const double *kj = kd + (size_t)j * D;
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += qi[d] * kj[d];
        srow[j] = modified_score(s, hq, i, j, dot);
        if (srow[j] > M) M = srow[j];
        ++n_allowed;
    }
    if (s->direct_p) {
        direct_p_row(srow, allow, Sk, vd, D, s->direct_p, o_out, lse_out);
        return;
    }
    for (int d = 0; d < D; ++d) o_out[d] = 0.0;
    if (n_allowed == 0) {
        *lse_out = -INFINITY;
        return;
    }
    double Z = 0.0;
    for (long j = 0; j < Sk; ++j)
        if (allow[j]) Z += exp(srow[j] - M);
    const double lse = M + log(Z);
    for (long j = 0; j < Sk; ++j) {
        if (!allow[j]) continue;
        const double p = exp(srow[j] - lse);
        const double *vj = vd + (size_t)j * D;
        for (int d = 0; d < D; ++d) o_out[d] += p * vj[d];
    }
    *lse_out = lse;
}

/* Convert the K and V rows of one (b, hkv) head to double, [Sk][D]. */
static void load_head(const oracle_shape_t *s, const void *k, const void *v,
                      int in_bf16, int b, int hkv, double *kd, double *vd) {
    for (int j = 0; j < s->Sk; ++j) {
        load_vec(k, in_bf16, kv_index(s, b, j, hkv), s->D, kd + (size_t)j * s->D);
        load_vec(v, in_bf16, kv_index(s, b, j, hkv), s->D, vd + (size_t)j * s->D);
    }
}

static int shape_ok(const oracle_shape_t *s) {
    if (s->B < 1 || s->Hq < 1 || s->Hkv < 1 || s->Sq < 1 || s->Sk < 1 || s->D < 1)
        return 0;
    if (s->Hq % s->Hkv != 0) return 0;
    if (s->doc_offsets && s->num_docs < 1) return 0;
    return 1;
}

/*
 * Forward.  rows == NULL: every row; o is [B,Sq,Hq,D], lse is [B,Hq,Sq].
 * rows != NULL: n_rows triples (b, hq, i); o is [n_rows, D], lse [n_rows].
 * Returns 0 on success, -1 on a bad shape, -2 on allocation failure.
 */
static int attn_fwd_core(const oracle_shape_t *s, const void *q, const void *k,
                         const void *v, int in_bf16, double *o, double *lse,
                         const int64_t *rows, int64_t n_rows) {
    if (!shape_ok(s)) return -1;
    const int D = s->D;
    const size_t head_elems = (size_t)s->Sk * D;
    double *kd = (double *)malloc(head_elems * sizeof(double));
    double *vd = (double *)malloc(head_elems * sizeof(double));
    if (!kd || !vd) { free(kd); free(vd); return -2; }
    int status = 0;

    for (int b = 0; b < s->B && status == 0; ++b) {
        for (int hkv = 0; hkv < s->Hkv && status == 0; ++hkv) {
            /* Skip heads no requested row touches. */
            if (rows) {
                int used = 0;
                for (int64_t r = 0; r < n_rows && !used; ++r)
                    used = rows[3 * r] == b && kv_head_of(s, (int)rows[3 * r + 1]) == hkv;
                if (!used) continue;
            }
            load_head(s, k, v, in_bf16, b, hkv, kd, vd);
            const int group = s->Hq / s->Hkv;
            const int64_t n_items = rows ? n_rows : (int64_t)group * s->Sq;
#pragma omp parallel
            {
                double *srow = (double *)malloc((size_t)s->Sk * sizeof(double));
                unsigned char *allow = (unsigned char *)malloc((size_t)s->Sk);
                double *qi = (double *)malloc((size_t)D * sizeof(double));
                if (!srow || !allow || !qi) {
#pragma omp atomic write
                    status = -2;
                } else {
#pragma omp for schedule(dynamic, 16)
                    for (int64_t it = 0; it < n_items; ++it) {
                        int hq, i;
                        double *o_dst, *lse_dst;
                        if (rows) {
                            if (rows[3 * it] != b || kv_head_of(s, (int)rows[3 * it + 1]) != hkv)
                                continue;
                            hq = (int)rows[3 * it + 1];
                            i = (int)rows[3 * it + 2];
                            o_dst = o + (size_t)it * D;
                            lse_dst = lse + it;
                        } else {
                            hq = hkv * group + (int)(it / s->Sq);
                            i = (int)(it % s->Sq);
                            o_dst = o + q_index(s, b, i, hq);
                            lse_dst = lse + ((size_t)b * s->Hq + hq) * s->Sq + i;
                        }
                        load_vec(q, in_bf16, q_index(s, b, i, hq), D, qi);
                        forward_row(s, hq, qi, kd, vd, i, srow, allow, o_dst, lse_dst);
                    }
                }
                free(srow);
                free(allow);
                free(qi);
            }
        }
    }
    free(kd);
    free(vd);
    return status;
}

/* -------------------------------------------------------------- backward */

/*
 * Backward of L = sum(O * dO) for one (b, hkv) group, from the definition:
 *   P_ij  = exp(s_ij - LSE_i)                (rebuilt from the forward's LSE)
 *   D_i   = sum_d dO_id * O_id               (O from this oracle's forward)
 *   dV_j += sum_i P_ij dO_i
 *   dP_ij = <dO_i, v_j>
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = sum_j dS_ij s'_ij k_j
 *   dK_j += sum_i dS_ij s'_ij q_i
 * where s'_ij is the derivative of the score w.r.t. <q_i, k_j> (scale, times
 * 1 - tanh^2 under a soft-cap; ALiBi adds a constant).
 * dK and dV sum over the Hq/Hkv query heads of the group.  ("Hardware-Aware
 * FP4 FlashAttention-4", section "Causal Backward Cuantizado": the backward
 * reconstructs the probabilities from the saved LSE.)
 */
static int attn_bwd_core(const oracle_shape_t *s, const void *q, const void *k,
                         const void *v, const void *dout, int in_bf16,
                         double *dq, double *dk, double *dv,
                         double *o_opt, double *lse_opt) {
    if (!shape_ok(s)) return -1;
    const int D = s->D, Sq = s->Sq, Sk = s->Sk;
    const int group = s->Hq / s->Hkv;
    int status = 0;

    memset(dq, 0, (size_t)s->B * Sq * s->Hq * D * sizeof(double));
    memset(dk, 0, (size_t)s->B * Sk * s->Hkv * D * sizeof(double));
    memset(dv, 0, (size_t)s->B * Sk * s->Hkv * D * sizeof(double));

#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < s->B; ++b) {
        for (int hkv = 0; hkv < s->Hkv; ++hkv) {
            const size_t head_elems = (size_t)Sk * D;
            double *kd = (double *)malloc(head_elems * sizeof(double));
            double *vd = (double *)malloc(head_elems * sizeof(double));
            double *srow = (double *)malloc((size_t)Sk * sizeof(double));
            unsigned char *allow = (unsigned char *)malloc((size_t)Sk);
            double *qi = (double *)malloc((size_t)D * sizeof(double));
            double *doi = (double *)malloc((size_t)D * sizeof(double));
            double *oi = (double *)malloc((size_t)D * sizeof(double));
            if (!kd || !vd || !srow || !allow || !qi || !doi || !oi) {
#pragma omp atomic write
                status = -2;
            } else {
                load_head(s, k, v, in_bf16, b, hkv, kd, vd);
                for (int g = 0; g < group; ++g) {
                    const int hq = hkv * group + g;
                    for (int i = 0; i < Sq; ++i) {
                        double lse;
                        load_vec(q, in_bf16, q_index(s, b, i, hq), D, qi);
                        load_vec(dout, in_bf16, q_index(s, b, i, hq), D, doi);
                        forward_row(s, hq, qi, kd, vd, i, srow, allow, oi, &lse);
                        if (o_opt)
                            memcpy(o_opt + q_index(s, b, i, hq), oi, (size_t)D * sizeof(double));
                        if (lse_opt) lse_opt[((size_t)b * s->Hq + hq) * Sq + i] = lse;
                        if (isinf(lse)) continue; /* no allowed key: zero gradient */
                        double Di = 0.0;
                        for (int d = 0; d < D; ++d) Di += doi[d] * oi[d];
                        double *dqi = dq + q_index(s, b, i, hq);
                        for (int j = 0; j < Sk; ++j) {
                            if (!allow[j]) continue;
                            const double *kj = kd + (size_t)j * D;
                            const double *vj = vd + (size_t)j * D;
                            const double p = exp(srow[j] - lse);
                            double dp = 0.0;
                            for (int d = 0; d < D; ++d) dp += doi[d] * vj[d];
                            const double ds = p * (dp - Di);
                            double dot = 0.0;
                            for (int d = 0; d < D; ++d) dot += qi[d] * kj[d];
                            const double g = ds * score_grad(s, dot);  /* dL/d(q_i . k_j) */
                            double *dkj = dk + kv_index(s, b, j, hkv);
                            double *dvj = dv + kv_index(s, b, j, hkv);
                            for (int d = 0; d < D; ++d) {
                                dvj[d] += p * doi[d];
                                dqi[d] += g * kj[d];
                                dkj[d] += g * qi[d];
                            }
                        }
                    }
                }
            }
            free(kd); free(vd); free(srow); free(allow); free(qi); free(doi); free(oi);
        }
    }
    return status;
}

/* ------------------------------------------------------------ public API */

#define ORACLE_SHAPE                                                        \
    oracle_shape_t s = {B, Hq, Hkv, Sq, Sk, D, scale, causal, window_left,  \
                        window_right, doc_offsets, num_docs, softcap, alibi_slopes}

int oracle_attn_fwd_bf16(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         double *o, double *lse, int B, int Hq, int Hkv, int Sq,
                         int Sk, int D, double scale, int causal, int window_left,
                         int window_right, const int *doc_offsets, int num_docs,
                         double softcap, const double *alibi_slopes,
                         const int64_t *rows, int64_t n_rows) {
    ORACLE_SHAPE;
    return attn_fwd_core(&s, q, k, v, 1, o, lse, rows, n_rows);
}

int oracle_attn_fwd_f64(const double *q, const double *k, const double *v,
                        double *o, double *lse, int B, int Hq, int Hkv, int Sq,
                        int Sk, int D, double scale, int causal, int window_left,
                        int window_right, const int *doc_offsets, int num_docs,
                        double softcap, const double *alibi_slopes,
                        const int64_t *rows, int64_t n_rows) {
    ORACLE_SHAPE;
    return attn_fwd_core(&s, q, k, v, 0, o, lse, rows, n_rows);
}

/* ------------------------------------------------------- fp8 (e4m3) inputs
 * The low-precision forward ("Hardware-Aware FP4 FlashAttention-4", the
 * "HAO" FP8 path that "Precisión" compares against): Q, K, V arrive as fp8
 * e4m3 codes with one fp32 dequantisation factor per tensor.  The oracle
 * decodes every code exactly, multiplies by its factor in fp64 and computes
 * exact attention of those values -- the result the fp8 path approximates.
 *
 * e4m3 (the variant without infinities): bit 7 sign, bits 6-3 exponent with
 * bias 7, bits 2-0 mantissa.  Exponent field 0 encodes the subnormals
 * m/8 * 2^-6; the code with all exponent and mantissa bits set is NaN; the
 * largest finite magnitude is 1.75 * 2^8 = 448. */
static double e4m3_to_double(uint8_t c) {
    const int e = (c >> 3) & 15, m = c & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp((double)m / 8.0, -6);
    else mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return (c & 0x80) ? -mag : mag;
}

double oracle_e4m3_to_double(int code) { return e4m3_to_double((uint8_t)code); }

static double *decode_e4m3(const uint8_t *x, size_t n, double mul) {
    double *d = (double *)malloc((n ? n : 1) * sizeof(double));
    if (!d) return NULL;
    for (size_t t = 0; t < n; ++t) d[t] = e4m3_to_double(x[t]) * mul;
    return d;
}

int oracle_attn_fwd_e4m3(const uint8_t *q, const uint8_t *k, const uint8_t *v,
                         double q_descale, double k_descale, double v_descale,
                         double *o, double *lse, int B, int Hq, int Hkv, int Sq,
                         int Sk, int D, double scale, int causal, int window_left,
                         int window_right, const int *doc_offsets, int num_docs,
                         const int64_t *rows, int64_t n_rows) {
    const double softcap = 0.0;
    const double *alibi_slopes = NULL;
    ORACLE_SHAPE;
    if (!shape_ok(&s)) return -1;
    const size_t nq = (size_t)B * Sq * Hq * D, nkv = (size_t)B * Sk * Hkv * D;
    double *qd = decode_e4m3(q, nq, q_descale);
    double *kd = decode_e4m3(k, nkv, k_descale);
    double *vd = decode_e4m3(v, nkv, v_descale);
    int status = -2;
    if (qd && kd && vd) status = attn_fwd_core(&s, qd, kd, vd, 0, o, lse, rows, n_rows);
    free(qd);
    free(kd);
    free(vd);
    return status;
}

/* ------------------------------------------- FP4 inputs, Direct-P forward
 * "Hardware-Aware FP4 FlashAttention-4", "Metodología", item 1 (Direct-P):
 * Q and K arrive in NVFP4, V in MXFP4, and the probabilities P are built as
 * MXFP4 values -- E2M1 codes with one power-of-two scale per 32 keys --
 * straight from the normalised log2 scores; the softmax normaliser is the
 * sum of exactly those represented values ("consistent normalisation"), so
 * numerator and denominator describe the same approximate operator.
 *
 * Formats (from their definitions):
 *   E2M1 (4 bits): bit 3 sign, bits 2-1 exponent with bias 1, bit 0
 *     mantissa; exponent field 0 holds the subnormal m * 0.5.  The eight
 *     magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6.
 *   NVFP4: one e4m3 scale per 16 consecutive elements of a row (along D)
 *     times a per-tensor fp32 factor: x = g * e4m3(scale) * e2m1(code); the
 *     scale is an unsigned magnitude (nvfp4_scale_to_double).
 *   MXFP4: one UE8M0 scale (2^(u - 127), u = 255 is NaN) per 32 elements:
 *     here 32 consecutive keys of one (batch, head, d) column of V, the
 *     contraction direction of PV, times a per-tensor factor.
 *   Two codes per byte, element 2j in the low nibble.
 *
 * The Direct-P probabilities of one row (readings where the page is silent,
 * listed in the design notes):
 *   y_j        = log2-unit score of key j (the page's normalised log score;
 *                the anchor it is measured from cancels out, see below);
 *   block      = keys [32 g, 32 g + 32), aligned to the key index, the
 *                32-key producer fragments the page pairs with MXFP4;
 *   E_g        = floor(max_{j in block, allowed} y_j) - 2: the OCP MX rule
 *                (shared exponent = floor(log2 amax) - 2 for E2M1), which
 *                puts the block maximum at 2^(y - E) in [4, 8);
 *   code_j     = the E2M1 magnitude chosen for r_j = y_j - E_g:
 *                affine classifier (the page's fast path): index
 *                clamp(rint(2 r + 2), 0, 7) -- the line through the
 *                half-octave grid on which the magnitudes 1, 2, 4 sit at
 *                indices 2, 4, 6 -- decoded as an E2M1 magnitude;
 *                exponential classifier (the page's "native exponentials"):
 *                2^r rounded to the nearest E2M1 magnitude, ties to the even
 *                code, saturating at 6;
 *   w_j        = code_j * 2^E_g (0 for masked keys);
 *   l          = sum_j w_j;  O = sum_j w_j v_j / l;  LSE = ln(l) (natural
 *                units: w_j approximates 2^y_j = e^s_j).
 * Shifting every y of a row by an integer changes every E_g by the same
 * integer and no code, so the result does not depend on which integer
 * anchor the scores are measured from; the range guard of the page (an
 * anchor that keeps the block scales in range) is therefore exact here and
 * this function works with the row maximum's floor only to keep doubles in
 * range. */
static const double kE2m1Mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

static double e2m1_to_double(unsigned c) {
    const unsigned e = (c >> 1) & 3u, m = c & 1u;
    const double mag = e == 0 ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
    return (c & 8u) ? -mag : mag;
}

static double ue8m0_to_double(uint8_t u) { return u == 255 ? NAN : ldexp(1.0, (int)u - 127); }

/* Round x >= 0 to the nearest E2M1 magnitude (ties to the even code index),
 * saturating at 6; returns the magnitude. */
static double e2m1_round(double x) {
    if (!(x < 6.0)) return 6.0;
    int k = 0;
    while (k < 7 && kE2m1Mag[k + 1] <= x) ++k; /* kE2m1Mag[k] <= x < kE2m1Mag[k+1] */
    const double lo = kE2m1Mag[k], hi = kE2m1Mag[k + 1], mid = 0.5 * (lo + hi);
    if (x < mid) return lo;
    if (x > mid) return hi;
    return (k & 1) ? hi : lo;
}

static double direct_p_code(double r, int classifier) {
    if (classifier == 2) return e2m1_round(exp2(r));
    double t = nearbyint(2.0 * r + 2.0);
    if (!(t > 0.0)) t = 0.0; /* also r = -inf */
    if (t > 7.0) t = 7.0;
    return kE2m1Mag[(int)t];
}

static void direct_p_row(const double *y, const unsigned char *allow, long n,
                         const double *vd, int D, int classifier, double *o_out,
                         double *lse_out) {
    double M = -INFINITY;
    for (long j = 0; j < n; ++j)
        if (allow[j] && y[j] > M) M = y[j];
    for (int d = 0; d < D; ++d) o_out[d] = 0.0;
    if (M == -INFINITY) {
        *lse_out = -INFINITY;
        return;
    }
    const double Mi = floor(M);
    double l = 0.0;
    for (long g0 = 0; g0 < n; g0 += 32) {
        const long g1 = g0 + 32 < n ? g0 + 32 : n;
        double bmax = -INFINITY;
        for (long j = g0; j < g1; ++j)
            if (allow[j] && y[j] > bmax) bmax = y[j];
        if (bmax == -INFINITY) continue;
        const double E = floor(bmax) - 2.0;
        for (long j = g0; j < g1; ++j) {
            if (!allow[j]) continue;
            const double w = ldexp(direct_p_code(y[j] - E, classifier), (int)(E - Mi));
            if (w == 0.0) continue;
            l += w;
            const double *vj = vd + (size_t)j * D;
            for (int d = 0; d < D; ++d) o_out[d] += w * vj[d];
        }
    }
    for (int d = 0; d < D; ++d) o_out[d] /= l;
    *lse_out = log(2.0) * (Mi + log2(l));
}

double oracle_e2m1_to_double(int code) { return e2m1_to_double((unsigned)code & 15u); }
double oracle_ue8m0_to_double(int u) { return ue8m0_to_double((uint8_t)u); }
double oracle_e2m1_round(double x) { return e2m1_round(x); }

/* One Direct-P row on given log2 scores y[n] (allow[n] != 0 marks the
 * allowed keys) and value rows v[n][D]. */
int oracle_direct_p_row(const double *y, const unsigned char *allow, int64_t n,
                        const double *v, int D, int classifier, double *o, double *lse) {
    if (n < 1 || D < 1 || (classifier != 1 && classifier != 2)) return -1;
    direct_p_row(y, allow, (long)n, v, D, classifier, o, lse);
    return 0;
}

/* An NVFP4 block scale: an unsigned e4m3 magnitude (the pages name NVFP4
 * for Q and K without a sign rule; the format's scale, as the FP4 tensor
 * cores read it, has none).  A byte outside the format -- NaN, or the sign
 * bit set with a nonzero magnitude -- makes its block read as 0 (the library
 * reports ATTN_ERR_RANGE for it); -0 is a zero scale. */
static double nvfp4_scale_to_double(uint8_t s) {
    if ((s & 0x7F) == 0x7F || s > 0x80) return 0.0;
    return e4m3_to_double((uint8_t)(s & 0x7F));
}

/* NVFP4 tensor of n elements (rows of D, D a multiple of 16) to doubles,
 * times `mul`. */
static double *decode_nvfp4(const uint8_t *codes, const uint8_t *scales, size_t n,
                            double mul) {
    double *d = (double *)malloc((n ? n : 1) * sizeof(double));
    if (!d) return NULL;
    for (size_t t = 0; t < n; ++t) {
        const unsigned c = (codes[t / 2] >> (4 * (t & 1))) & 15u;
        d[t] = mul * nvfp4_scale_to_double(scales[t / 16]) * e2m1_to_double(c);
    }
    return d;
}

/* MXFP4 V [B][Sk][H][D] with scales [B][ceil(Sk/32)][H][D] to doubles. */
static double *decode_mxfp4_v(const uint8_t *codes, const uint8_t *scales, int B, int Sk,
                              int H, int D, double mul) {
    const size_t n = (size_t)B * Sk * H * D;
    const int nblk = (Sk + 31) / 32;
    double *d = (double *)malloc((n ? n : 1) * sizeof(double));
    if (!d) return NULL;
    for (size_t t = 0; t < n; ++t) {
        const size_t row = t / (size_t)D;
        const int dd = (int)(t % (size_t)D);
        const int h = (int)(row % (size_t)H);
        const int j = (int)((row / (size_t)H) % (size_t)Sk);
        const int b = (int)(row / ((size_t)H * Sk));
        const uint8_t u = scales[(((size_t)b * nblk + j / 32) * H + h) * D + dd];
        const unsigned c = (codes[t / 2] >> (4 * (t & 1))) & 15u;
        d[t] = mul * ue8m0_to_double(u) * e2m1_to_double(c);
    }
    return d;
}

/*
 * Direct-P forward of NVFP4 Q/K and MXFP4 V.  classifier 1 = affine,
 * 2 = exponential.  The log2 score is <q', k'> * c with q', k' decoded
 * without their per-tensor factors and c = scale * q_global * k_global *
 * log2 e in fp64: the code decisions are taken on the exact score (where c
 * and the block scales are powers of two, fp32 holds the same value, so a
 * kernel computing in fp32 takes the same decisions).  O includes v_global; LSE is in
 * natural units of the scores scale * <q, k>.  Layouts as the kernel's:
 * codes [B][S][H][D/2], Q/K scales [B][S][H][D/16], V scales
 * [B][ceil(Sk/32)][Hkv][D].
 */
int oracle_attn_fwd_fp4(const uint8_t *q_codes, const uint8_t *q_scales, double q_global,
                        const uint8_t *k_codes, const uint8_t *k_scales, double k_global,
                        const uint8_t *v_codes, const uint8_t *v_scales, double v_global,
                        double *o, double *lse, int B, int Hq, int Hkv, int Sq, int Sk,
                        int D, double scale, int causal, int window_left, int window_right,
                        const int *doc_offsets, int num_docs, int classifier,
                        const int64_t *rows, int64_t n_rows) {
    if (classifier != 1 && classifier != 2) return -1;
    if (D % 32 != 0) return -1;
    const double softcap = 0.0;
    const double *alibi_slopes = NULL;
    const double c = scale * q_global * k_global * 1.4426950408889634;
    ORACLE_SHAPE;
    s.scale = c;
    s.direct_p = classifier;
    if (!shape_ok(&s)) return -1;
    const size_t nq = (size_t)B * Sq * Hq * D, nkv = (size_t)B * Sk * Hkv * D;
    double *qd = decode_nvfp4(q_codes, q_scales, nq, 1.0);
    double *kd = decode_nvfp4(k_codes, k_scales, nkv, 1.0);
    double *vd = decode_mxfp4_v(v_codes, v_scales, B, Sk, Hkv, D, v_global);
    int status = -2;
    if (qd && kd && vd) status = attn_fwd_core(&s, qd, kd, vd, 0, o, lse, rows, n_rows);
    free(qd);
    free(kd);
    free(vd);
    return status;
}

int oracle_attn_bwd_bf16(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         const uint16_t *dout, double *dq, double *dk, double *dv,
                         double *o, double *lse, int B, int Hq, int Hkv, int Sq,
                         int Sk, int D, double scale, int causal, int window_left,
                         int window_right, const int *doc_offsets, int num_docs,
                         double softcap, const double *alibi_slopes) {
    ORACLE_SHAPE;
    return attn_bwd_core(&s, q, k, v, dout, 1, dq, dk, dv, o, lse);
}

int oracle_attn_bwd_f64(const double *q, const double *k, const double *v,
                        const double *dout, double *dq, double *dk, double *dv,
                        double *o, double *lse, int B, int Hq, int Hkv, int Sq,
                        int Sk, int D, double scale, int causal, int window_left,
                        int window_right, const int *doc_offsets, int num_docs,
                        double softcap, const double *alibi_slopes) {
    ORACLE_SHAPE;
    return attn_bwd_core(&s, q, k, v, dout, 0, dq, dk, dv, o, lse);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
