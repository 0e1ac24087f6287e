/*
 * tiled_attention_blackwell_b200 -- C ABI of a fused, IO-aware exact
 * attention library for NVIDIA B200 (sm_100a).
 *
 * The operation ("Hardware-Aware FP4 FlashAttention-4", section
 * "Planteamiento del Problema": the product QK^T, a row softmax, the product
 * PV; section "Causal Backward Cuantizado": the forward keeps the per-row
 * log-sum-exp; "FlashAttention-4发布", section "从V1到V4", first bullet: the
 * result is computed tile by tile so the N x N score matrix never reaches
 * HBM):
 *
 *   for every batch b, query head hq, query row i:
 *     hkv      = hq / (Hq / Hkv)                       (grouped heads, GQA/MQA)
 *     s_ij     = scale * <q[b,i,hq,:], k[b,j,hkv,:]>   for allowed keys j
 *     LSE[b,hq,i] = log sum_j exp(s_ij)                (natural log, fp32)
 *     O[b,i,hq,:] = sum_j exp(s_ij - LSE) * v[b,j,hkv,:]   (bf16, RN)
 *
 *   Key j is allowed for query i (shift = Sk - Sq, bottom-right alignment):
 *     causal != 0        :  j <= i + shift
 *     window_left  >= 0  :  j >= i + shift - window_left
 *     window_right >= 0  :  j <= i + shift + window_right
 *     doc_offsets != NULL:  i and j lie in the same document, where token t
 *                           belongs to document d iff
 *                           doc_offsets[d] <= t < doc_offsets[d+1]
 *   (the sliding-window and document masks are two of the patterns named in
 *   "El FlexAttention de PyTorch con FlashAttention-4", intro).  A row with
 *   no allowed key gets O = 0 and LSE = -inf.
 *
 * Memory layout (all contiguous, row-major, device memory owned by the
 * caller; the library allocates nothing per call):
 *   q, o : bf16 [B, Sq, Hq,  D]
 *   k, v : bf16 [B, Sk, Hkv, D]
 *   lse  : fp32 [B, Hq, Sq]
 *   doc_offsets : int32 [num_docs + 1] in device memory, shared by all
 *                 batches; must be non-decreasing with doc_offsets[0] = 0 and
 *                 doc_offsets[num_docs] = Sq.  Malformed offsets give
 *                 unspecified output values but never out-of-bounds access.
 *
 * Calls are asynchronous on `stream` (a cudaStream_t, NULL = the legacy
 * default stream).  Argument errors are reported before anything is
 * launched.  A kernel that gives up waiting (every device-side wait is
 * bounded) records ATTN_ERR_DEVICE_TIMEOUT in a per-device status word,
 * read back with attn_get_device_status().
 */
#ifndef TILED_ATTENTION_B200_ATTN_H
#define TILED_ATTENTION_B200_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ATTN_ABI_VERSION 2

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = 1,    /* bad shape, null pointer, bad mask argument */
    ATTN_ERR_UNSUPPORTED = 2,    /* valid request outside what is built (e.g. D) */
    ATTN_ERR_MISALIGNED = 3,     /* a tensor pointer is not 16-byte aligned */
    ATTN_ERR_LAUNCH = 4,         /* the CUDA launch itself failed */
    ATTN_ERR_DEVICE_TIMEOUT = 5, /* a bounded device-side wait expired */
    ATTN_ERR_CUDA = 6,           /* another CUDA runtime error (see detail) */
    ATTN_ERR_RANGE = 7           /* an input value outside the range the path
                                    represents (FP4 scales; see attn_fwd_fp4) */
} attn_status_t;

/* Tuning knobs of the forward.  Pass NULL for the defaults.  None of them
 * changes the mathematical result, only rounding. */
typedef struct {
    /* Online-softmax rescale threshold in log2 units ("La ventaja técnica" of
     * "FlashAttention-4 de NVIDIA": rescale only when the running
     * maximum moves significantly).  The running max of a row, and with it
     * the output accumulator, is updated only when a new block raises the
     * row maximum by more than this amount; in between, unnormalised
     * probabilities may reach 2^threshold.  0 = classic online softmax.
     * Valid range [0, 16].  Default 8. */
    float rescale_threshold;
    /* exp2 evaluation ("La ventaja técnica": part of the exponentials run as
     * a cubic polynomial on the FMA units instead of the special-function
     * units).  0 = all on the MUFU ex2 unit; 1 = the tuned split
     * (default); 2 = every column of unmasked tiles by polynomial. */
    int exp2_mode;
    /* Bound of every device-side wait of the forward, in microseconds
     * (0 = the default, 1 s).  A wait that runs out makes the kernel record
     * ATTN_ERR_DEVICE_TIMEOUT, finish its in-flight copies and MMAs, free its
     * tensor memory and return.  Valid range [0, 60000000]. */
    int wait_timeout_us;
    /* Testing only (keep 0): 1 makes the first CTA withhold the copy of its
     * first key block, so its MMA warp's wait runs out and the call reports
     * ATTN_ERR_DEVICE_TIMEOUT through attn_get_device_status().  Nothing
     * faults; the outputs of that CTA are left unwritten. */
    int debug_withhold_kv;
    /* Score modifiers ("El FlexAttention de PyTorch con FlashAttention-4",
     * intro: soft-capping, ALiBi), applied in this order to the scaled score
     * s = scale * <q_i, k_j> before the mask:
     *   softcap > 0        : s <- softcap * tanh(s / softcap)
     *   alibi_slopes != 0  : s <- s - alibi_slopes[hq] * |i + (Sk - Sq) - j|
     * softcap = 0 and alibi_slopes = NULL (the defaults) leave s unchanged.
     * alibi_slopes is device memory, fp32 [Hq], 4-byte aligned.  With a
     * modifier the exponentials all run on MUFU (exp2_mode is ignored). */
    float softcap;
    int reserved0; /* must be zero */
    const float *alibi_slopes;
    int reserved[4]; /* must be zero */
} attn_fwd_options_t;

/* Score modifiers of the backward: the same meaning as in
 * attn_fwd_options_t, and they must match the forward that produced O and
 * LSE.  Pass NULL to attn_bwd_ex for none. */
typedef struct {
    float softcap;
    int reserved0; /* must be zero */
    const float *alibi_slopes;
    int reserved[4]; /* must be zero */
} attn_bwd_options_t;

/* Fills *opts with the defaults. */
ATTN_API void attn_fwd_default_options(attn_fwd_options_t *opts);

/*
 * Forward: O and LSE.  D must be 64 or 128; Hq % Hkv == 0; Sq, Sk >= 1;
 * scale > 0 and finite; window bounds -1 (unbounded) or >= 0; a document
 * mask requires Sq == Sk and num_docs >= 1.  q, k, v, o must be 16-byte
 * aligned.  Returns ATTN_OK once the kernel is enqueued.
 */
ATTN_API attn_status_t attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                       int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale,
                       int causal, int window_left, int window_right,
                       const int *doc_offsets, int num_docs, void *stream);

/* attn_fwd with explicit tuning options (NULL = defaults). */
ATTN_API attn_status_t attn_fwd_ex(const void *q, const void *k, const void *v, void *o, float *lse,
                          int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale,
                          int causal, int window_left, int window_right,
                          const int *doc_offsets, int num_docs,
                          const attn_fwd_options_t *opts, void *stream);

/*
 * Low-precision forward ("Hardware-Aware FP4 FlashAttention-4", "Precisión":
 * the FP8 path that Direct-P is measured against).  q, k, v hold fp8 e4m3
 * codes (1 byte each, same [B,S,H,D] layouts, 16-byte aligned); the values
 * they stand for are q_descale * q, k_descale * k, v_descale * v (each factor
 * > 0 and finite).  Both products QK^T and PV run on the tensor cores in
 * e4m3 with fp32 accumulation; the probabilities P are rounded to e4m3
 * after scaling by 2^(8 - rescale_threshold), which keeps them inside e4m3's
 * range (the row sum l is taken from the unrounded values, as in attn_fwd).
 * O is bf16 and LSE fp32 as in attn_fwd, for the dequantized inputs.
 * D must be 128; rescale_threshold must be <= 8 (smaller values keep more
 * precision for small probabilities at the cost of more rescales); score
 * modifiers are not supported (ATTN_ERR_UNSUPPORTED).  opts may be NULL.
 */
ATTN_API attn_status_t attn_fwd_fp8(const void *q, const void *k, const void *v,
                                    float q_descale, float k_descale, float v_descale,
                                    void *o, float *lse, int B, int Hq, int Hkv, int Sq,
                                    int Sk, int D, float scale, int causal, int window_left,
                                    int window_right, const int *doc_offsets, int num_docs,
                                    const attn_fwd_options_t *opts, void *stream);

/*
 * FP4 Direct-P forward ("Hardware-Aware FP4 FlashAttention-4",
 * "Metodología", item 1).  Q and K arrive in NVFP4, V in MXFP4; the
 * probabilities are built directly as MXFP4 values and the softmax
 * normaliser is the sum of exactly those values, so the output is the
 * weighted mean of V under the quantised weights:
 *
 *   per row i and 32-key block g (keys [32g, 32g+32), allowed keys only):
 *     y_j   = log2-unit score  scale * q_global * k_global * <q'_i, k'_j> / ln 2
 *             (q', k': the NVFP4 values without their per-tensor factors)
 *     E_g   = floor(max_j y_j) - 2                 (the OCP MX exponent rule)
 *     r_j   = y_j - E_g                            (< 3)
 *     c_j   = E2M1 magnitude (0, 0.5, 1, 1.5, 2, 3, 4, 6) chosen by
 *             ATTN_DIRECT_P_AFFINE: index clamp(rint(2 r_j + 2), 0, 7)
 *             ATTN_DIRECT_P_EXP2:   2^r_j rounded to nearest (ties even), max 6
 *     w_j   = c_j * 2^E_g
 *   O_i   = v_global * sum_j w_j v'_j / sum_j w_j       (bf16)
 *   LSE_i = ln(sum_j w_j)                              (fp32, natural log)
 *
 * The scores are measured from an integer anchor that follows the running
 * row maximum (rescaled only when the maximum rises by more than
 * rescale_threshold, always by an exact power of two); shifting a row's
 * log2 scores by an integer changes no code, so the result does not depend
 * on the anchor.  A block whose maximum lies more than
 * 26 - ceil(rescale_threshold) octaves below the anchor contributes nothing
 * (its values would leave the normal range of the f16 container; both
 * product paths below apply the same rule, so they compute the same codes
 * and weights).  Scores
 * are handled in fp32 as in attn_fwd; log2 scores must stay below 2^21 in
 * magnitude (beyond that fp32 cannot resolve their fractional part, on which
 * the codes depend).
 *
 * Inputs (device memory, 16-byte aligned, caller-owned):
 *   q_codes  uint8 [B, Sq, Hq,  D/2]  two E2M1 codes per byte, element 2j
 *   k_codes  uint8 [B, Sk, Hkv, D/2]  in the low nibble (bit 3 = sign)
 *   q_scales uint8 [B, Sq, Hq,  D/16] e4m3 scale per 16 elements of a row
 *   k_scales uint8 [B, Sk, Hkv, D/16]
 *   v_codes  uint8 [B, Sk, Hkv, D/2]
 *   v_scales uint8 [B, ceil(Sk/32), Hkv, D]  UE8M0 scale (2^(u - 127)) per
 *            32 keys of each (batch, head, d) column of V
 *   q_global, k_global, v_global: per-tensor fp32 factors, > 0 and finite.
 * An NVFP4 block scale is an unsigned e4m3 magnitude (the scale format of
 * the FP4 tensor cores; -0 is a zero scale).  A nonzero code whose scale is
 * NaN or negative (sign bit set, nonzero magnitude), or (V) whose u - 127
 * lies outside [-13, 13], reads as 0 and makes attn_get_device_status()
 * report ATTN_ERR_RANGE.
 * Outputs: o bf16 [B, Sq, Hq, D], lse fp32 [B, Hq, Sq].
 * workspace: at least attn_fwd_fp4_workspace_size() bytes, 16-byte aligned
 * (contents on entry ignored).
 * D must be 64 or 128; masks, GQA and shape rules as attn_fwd; no score
 * modifiers.  opts may be NULL.
 *
 * Products (opts->mma).  ATTN_FP4_MMA_BLOCK_SCALED (D = 128): both run on
 * the block-scaled FP4 tensor cores, Q K^T as NVFP4 x NVFP4 (kind::mxf4nvf4,
 * UE4M3 scale per 16) and P V as MXFP4 x MXFP4 (kind::mxf4, UE8M0 scale per
 * 32 keys: P's codes with their 2^E_g, V's with its scales); a preparation
 * pass lays the scales out for tensor memory and transposes V's codes into
 * the workspace.  ATTN_FP4_MMA_F16: a pass widens Q, K, V to f16 (exactly)
 * in the workspace and both products run as f16 MMAs.  Every product of two
 * FP4 values is exact in fp32, so the paths differ only in the order of the
 * fp32 accumulation.  ATTN_FP4_MMA_AUTO (default): block-scaled for D = 128,
 * f16 for D = 64.
 */
#define ATTN_DIRECT_P_AFFINE 0
#define ATTN_DIRECT_P_EXP2 1
#define ATTN_FP4_MMA_AUTO 0
#define ATTN_FP4_MMA_F16 1
#define ATTN_FP4_MMA_BLOCK_SCALED 2

typedef struct {
    /* Online rescale threshold of the integer anchor, in log2 units,
     * [0, 8].  Default 8. */
    float rescale_threshold;
    /* ATTN_DIRECT_P_AFFINE (default) or ATTN_DIRECT_P_EXP2. */
    int classifier;
    /* Bound of every device-side wait, microseconds (0 = 1 s); as in
     * attn_fwd_options_t.  Valid range [0, 60000000]. */
    int wait_timeout_us;
    /* ATTN_FP4_MMA_AUTO (default), ATTN_FP4_MMA_F16 or
     * ATTN_FP4_MMA_BLOCK_SCALED (D = 128 only, else ATTN_ERR_UNSUPPORTED). */
    int mma;
    int reserved[4]; /* must be zero */
} attn_fp4_options_t;

/* Fills *opts with the defaults. */
ATTN_API void attn_fp4_default_options(attn_fp4_options_t *opts);

/* Workspace bytes attn_fwd_fp4 needs for these sizes (0 for invalid ones). */
ATTN_API size_t attn_fwd_fp4_workspace_size(int B, int Hq, int Hkv, int Sq, int Sk, int D);

ATTN_API attn_status_t attn_fwd_fp4(const void *q_codes, const void *q_scales, float q_global,
                                    const void *k_codes, const void *k_scales, float k_global,
                                    const void *v_codes, const void *v_scales, float v_global,
                                    void *o, float *lse, int B, int Hq, int Hkv, int Sq, int Sk,
                                    int D, float scale, int causal, int window_left,
                                    int window_right, const int *doc_offsets, int num_docs,
                                    void *workspace, size_t workspace_bytes,
                                    const attn_fp4_options_t *opts, void *stream);

/*
 * Backward ("Hardware-Aware FP4 FlashAttention-4", "Causal Backward
 * Cuantizado": gradients from the saved LSE, probabilities rebuilt rather
 * than stored).  For L with dO = dL/dO:
 *   D_i   = sum_d dO[b,i,hq,d] * O[b,i,hq,d]
 *   P_ij  = exp(s_ij - LSE[b,hq,i])           (allowed keys, else 0)
 *   dS_ij = P_ij * (<dO_i, v_j> - D_i)
 *   dQ_i  = scale * sum_j dS_ij k_j
 *   dK_j  = scale * sum_i dS_ij q_i            (summed over the query heads
 *   dV_j  =         sum_i P_ij dO_i             of a GQA group)
 * Inputs: q, k, v as for attn_fwd; o (bf16 [B,Sq,Hq,D]) and lse (fp32
 * [B,Hq,Sq]) from attn_fwd on the same inputs and mask; dout bf16
 * [B,Sq,Hq,D].  Outputs: dq fp32 [B,Sq,Hq,D]; dk, dv bf16 [B,Sk,Hkv,D].
 * Every output element is written.  workspace: device memory of at least
 * attn_bwd_workspace_size() bytes, 16-byte aligned, owned by the caller
 * (holds D_i between the kernels of one call; contents on entry ignored).
 * Same shape, mask and alignment rules as attn_fwd (dq, dk, dv, o, dout
 * 16-byte aligned).  The result is deterministic (no atomics).  Calls are
 * asynchronous on `stream`.
 */
ATTN_API size_t attn_bwd_workspace_size(int B, int Hq, int Hkv, int Sq, int Sk, int D);

ATTN_API attn_status_t attn_bwd(const void *q, const void *k, const void *v, const void *o,
                                const float *lse, const void *dout, float *dq, void *dk,
                                void *dv, int B, int Hq, int Hkv, int Sq, int Sk, int D,
                                float scale, int causal, int window_left, int window_right,
                                const int *doc_offsets, int num_docs, void *workspace,
                                size_t workspace_bytes, void *stream);

/* attn_bwd with score modifiers (NULL = none).  Under a soft-cap the
 * gradients carry the cap's derivative: dL/d<q_i,k_j> = dS_ij * scale *
 * (1 - tanh^2(s_ij / softcap)). */
ATTN_API attn_status_t attn_bwd_ex(const void *q, const void *k, const void *v, const void *o,
                                   const float *lse, const void *dout, float *dq, void *dk,
                                   void *dv, int B, int Hq, int Hkv, int Sq, int Sk, int D,
                                   float scale, int causal, int window_left, int window_right,
                                   const int *doc_offsets, int num_docs, void *workspace,
                                   size_t workspace_bytes, const attn_bwd_options_t *opts,
                                   void *stream);

/*
 * attn_bwd without a workspace argument, for callers that cannot allocate
 * device memory at the point where they run the backward: a framework
 * plugin or kernel hook that is handed only its input and output pointers
 * and has no allocator of its own, or a serving/training loop that must not
 * call cudaMalloc on its hot path (an allocation can synchronise the device
 * and stall every stream, and can fail with out-of-memory mid-step).  (The
 * attention pages have no counterpart of this entry point; it exists for
 * such callers.)
 *
 * Same arguments, contract and results as attn_bwd, minus the workspace.
 * The D_i scratch lives in one fixed device array inside the library (4 MiB,
 * held on every GPU that loads the library until the process exits), so:
 *   - B * Hq * Sq must not exceed 1048576 rows; larger calls return
 *     ATTN_ERR_UNSUPPORTED before anything is launched;
 *   - the first call on a device looks up that array's device address (and
 *     prepares the kernels); make that first call before any stream
 *     capture on that device;
 *   - every call on a device shares the array: calls that can run on the GPU
 *     at the same time (different streams, different host threads) race on
 *     it and must be ordered by the caller (same stream, or events).  Nothing
 *     in it needs to start at zero: each call writes every entry it reads.
 * Nothing is allocated: no cudaMalloc / cudaFree, no library allocator.
 */
ATTN_API attn_status_t attn_bwd_noalloc(const void *q, const void *k, const void *v,
                                        const void *o, const float *lse, const void *dout,
                                        float *dq, void *dk, void *dv, int B, int Hq, int Hkv,
                                        int Sq, int Sk, int D, float scale, int causal,
                                        int window_left, int window_right,
                                        const int *doc_offsets, int num_docs, void *stream);

/* Synchronises `stream`, then reads and clears the device status word of
 * the current device.  Returns ATTN_OK, ATTN_ERR_DEVICE_TIMEOUT or
 * ATTN_ERR_RANGE (or ATTN_ERR_CUDA if the synchronisation itself failed). */
ATTN_API attn_status_t attn_get_device_status(void *stream);

/* Static description of a status code. */
ATTN_API const char *attn_status_string(attn_status_t status);

/* Detail of the last error returned on the calling host thread ("" if none). */
ATTN_API const char *attn_last_error_detail(void);

/* ATTN_ABI_VERSION of the built library. */
ATTN_API int attn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TILED_ATTENTION_B200_ATTN_H */
