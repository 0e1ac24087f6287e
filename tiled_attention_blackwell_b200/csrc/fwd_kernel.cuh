// Fused exact-attention forward for B200 (sm_100a).
//
// One CTA owns two 128-row query tiles of one (batch, query head) -- the
// 256 x 128 tile shape the FlexAttention page gives for Blackwell ("El
// FlexAttention de PyTorch con FlashAttention-4", "Limitaciones actuales")
// -- and streams the key/value blocks its mask allows through shared memory.
// The two query tiles ping-pong between the tensor cores and the softmax
// warps ("Hardware-Aware FP4 FlashAttention-4", "Metodología": the two-query
// pipeline and its tensor-memory ownership protocol).
//
// Warp roles (384 threads):
//   warps 0-3   softmax + correction + epilogue for query tile 0
//   warps 4-7   the same for query tile 1
//   warp  8     tcgen05 MMA issue (one thread) and TMEM allocation
//   warp  9     TMA producer (one thread)
//   warps 10-11 idle
// The pipeline stages load -> MMA -> softmax -> correction -> epilogue of the
// FA4 design ("FlashAttention-4 de NVIDIA", "La ventaja técnica") map onto these roles;
// the correction (rescaling the output accumulator in TMEM) runs inside the
// softmax warps because threshold gating makes it rare.
//
// Tensor memory (512 columns, fp32 cells, lane = query row):
//   [  0,128) S0 = Q0 K^T   (P0 in bf16 pairs overwrites its first 64 columns)
//   [128,256) S1 = Q1 K^T   (P1 likewise)
//   [256,256+D) O0, then O1 -- the full 512-column budget at D = 128 that
//   "Contribuciones Clave" / "Puntos Clave" of the FP4 page describe.
//
// Shared memory: Q0, Q1 and a ring of NS key/value slots, each a 128 x D
// bf16 tile stored as D/64 column chunks of [128 rows][128 bytes] with the
// 128-byte swizzle that both TMA and the tcgen05 descriptors use.
//
// Template variants: EXP_MODE picks the MUFU / polynomial split of the
// exponentials; MOD (bit 0 soft-cap, bit 1 ALiBi, "El FlexAttention de
// PyTorch con FlashAttention-4", intro) transforms the scores into log2
// units before the mask and the max; PREC picks the operand precision:
// 0 bf16; 1 e4m3 Q, K, V (one 128-byte chunk per row at D = 128,
// kind::f8f6f4 MMAs) with P as four e4m3 values per TMEM column
// ("Hardware-Aware FP4 FlashAttention-4", "Precisión": the FP8 path);
// 2 and 3 the Direct-P forward of the same page ("Metodología", item 1):
// f16 operands holding NVFP4 / MXFP4 values exactly, and P built as MXFP4
// values -- E2M1 codes times one power-of-two scale per 32 keys -- by the
// affine classifier (2) or the rounded exponential (3), with the row sum
// taken from exactly those values.
//
// Online softmax in log2 units: x = s * scale * log2(e).  Each row keeps a
// running max m and sum l; a new block changes m (and rescales O and l) only
// when it raises the row max by more than `rescale_threshold` ("La ventaja
// técnica": rescale only when the max changes significantly; "为Blackwell
// 而生的性能猛兽" item 1: most rescales are skipped).  Exponentials run on
// the MUFU ex2 unit or as a cubic polynomial on the FMA pipe ("La ventaja
// técnica"; "为Blackwell而生的性能猛兽" item 2).
//
// Every wait is bounded: on expiry the kernel records a timeout in the
// device status word, lets its in-flight copies and MMAs finish, frees TMEM
// and returns.
#pragma once

#include "common.cuh"
#include "exp2_poly.cuh"
#include "ptx.cuh"

namespace tab {

constexpr int kBlockM = 128;   // query rows per tile = TMEM lanes
constexpr int kBlockN = 128;   // keys per key/value block
constexpr int kFwdThreads = 384;
constexpr int kTmemCols = 512;
// Registers: 384 threads launch with 168 each (65536 / 384, in steps of 8).
// setmaxnreg moves them from the MMA / TMA warpgroup to the two softmax
// warpgroups; the split must not exceed the launch allocation (a larger
// request would wait forever), and the host checks the compiled count.
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 216;
constexpr int kOtherRegs = 72;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kOtherRegs <= kFwdThreads * kLaunchRegs,
              "register split exceeds the launch allocation");

struct FwdParams {
    CUtensorMap tm_q;  // bf16 [B][Sq][Hq][D]: dims (D, Sq, Hq, B), box (64, 128, 1, 1)
    CUtensorMap tm_k;  // bf16 [B][Sk][Hkv][D]
    CUtensorMap tm_v;
    __nv_bfloat16 *o;
    float *lse;
    const int *doc_offsets;
    int *status;
    int num_docs;
    int B, Hq, Hkv, Sq, Sk, group;
    int causal, window_left, window_right;
    int num_qblocks;
    int head_group;  // (batch, head) pairs scheduled together (L2 reuse of K/V)
    float scale_log2;
    float rescale_threshold;
    long long *trace;  // clock64 event log (trace builds only), else null
    // Rescale statistics (counting builds only, else null): [0] blocks after
    // a row's first, [1] of those that raise the row's running maximum (each
    // a rescale of O without a threshold), [2] rescales taken under the
    // threshold, [3] warp-level O corrections executed.
    unsigned long long *rescale_counts;
    int trace_ctas;
    unsigned long long timeout_ns;  // bound of every wait
    int debug_withhold_kv;          // testing: CTA 0 skips its first K copy
    // Score modifiers (MOD != 0 kernels): soft-cap s <- cap tanh(s / cap)
    // as softcap_out * tanh(raw * softcap_in) in log2 units; ALiBi slope per
    // query head (device fp32 [Hq]) or null.
    float softcap_in;   // scale / cap
    float softcap_out;  // cap * log2(e)
    const float *alibi_slopes;
    // fp8 and Direct-P kernels: V's dequantisation factor (Q's and K's are
    // folded into scale_log2) and the integer exponent offset that puts P
    // into the range of its container (e4m3: (0, 2^8]; f16: below 2^16).
    float v_descale;
    float p_offset;
    // Block-scaled FP4 kernel: scale-factor atoms (Q per 128-row tile, K and
    // V per 128-key block; two 512-byte atoms each) and the tile counts.
    const uint8_t *sf_q, *sf_k, *sf_v;
    int nq_tiles, nk_tiles;
};

// Opt-in event trace (compile with -DATTN_TRACE): lane 0 of warps 0 and 4
// (the two softmax warpgroups) and of the MMA warp record clock64() at the
// hand-off points of each key block, for the first `trace_ctas` CTAs.
constexpr int kTraceIters = 96;
constexpr int kTraceEvents = 8;
#ifdef ATTN_TRACE
#define ATTN_TRACE_EVENT(role, iter, ev)                                                    \
    do {                                                                                  \
        if (p.trace && (int)blockIdx.x < p.trace_ctas && (iter) < kTraceIters && lane == 0) \
            p.trace[(((size_t)blockIdx.x * 3 + (role)) * kTraceIters + (iter)) *            \
                        kTraceEvents + (ev)] = clock64();                                 \
    } while (0)
#else
#define ATTN_TRACE_EVENT(role, iter, ev) \
    do {                                 \
    } while (0)
#endif

// Opt-in rescale statistics (compile with -DATTN_COUNT_RESCALES): each
// softmax thread counts for its row, per key block after the first, whether
// the block raises the running maximum and whether the threshold lets the
// rescale happen; the counts are reduced per warp and added to
// p.rescale_counts at the end.
#ifdef ATTN_COUNT_RESCALES
#define ATTN_COUNT_BLOCK(t, raises, taken) \
    do {                                   \
        if ((t) > 0) {                     \
            ++cnt_blocks;                  \
            cnt_raise += (raises) ? 1u : 0u; \
            cnt_taken += (taken) ? 1u : 0u;  \
        }                                  \
    } while (0)
#else
#define ATTN_COUNT_BLOCK(t, raises, taken) \
    do {                                   \
    } while (0)
#endif

// EB: bytes per element of Q, K, V (2 = bf16, 1 = fp8 e4m3).  A tile row of
// D elements is D*EB bytes, stored as chunks of 128-byte rows.
template <int D, int NS, int EB = 2>
struct FwdSmem {
    static constexpr int kChunkBytes = kBlockM * 128;  // 16 KB: 128 rows x 128 bytes
    static constexpr int kChunks = D * EB / 128;
    static constexpr int kChunkElems = 128 / EB;       // elements per 128-byte row
    uint8_t q[2][kChunks][kChunkBytes];
    uint8_t kv[NS][kChunks][kChunkBytes];
    uint64_t q_full;
    uint64_t kv_full[NS];
    uint64_t kv_empty[NS];
    uint64_t s_full[2];
    uint64_t p_half[2];  // P of keys [0, 64) of the block is in TMEM
    uint64_t p_full[2];  // all of P (and any O correction) is in TMEM
    uint64_t o_final[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int range[2][2];  // per query tile: first and last key block (inclusive)
};

// Column pairs that use the polynomial in EXP_MODE 1: one pair in eight,
// spread through the row so MUFU and FMA work interleave.  (Measured on
// B200 for the causal S=8192 forward: 1/8 of pairs is the fastest split; a
// quarter, two fifths, a half and a clustered 12-of-32 split are slower, and
// all-polynomial is slowest: the cubic costs more FMA-pipe cycles per element
// than one MUFU ex2, so it only pays where it fills MUFU stalls.)
template <int EXP_MODE>
__device__ __forceinline__ bool use_poly(int col) {
    if (EXP_MODE == 0) return false;
    if (EXP_MODE == 2) return true;
    return ((col >> 1) & 7) == 3;
}

// Half a row of a block: p = 2^(s*c - m) for 64 scores (packed pairs), the
// exponentials split between MUFU and the polynomial per EXP_MODE; writes
// the bf16 pairs to pk and adds to `sum` the row sum of the unrounded p (for
// the LSE) and to `sum_pv` the sum of the bf16-rounded values, the weights
// the tensor cores apply in PV.  The output is normalised by the latter, so
// O is a convex combination of V rows with exactly those weights: a row
// dominated by one key reproduces that key's V row even when its p (scaled
// by a running maximum that may lag the true one by up to the rescale
// threshold) is not a bf16 value.
template <int EXP_MODE>
__device__ __forceinline__ void exp_pack_half(const float *s, float c, float neg_m, uint32_t *pk,
                                              float &sum, float &sum_pv) {
    float sum0 = 0.0f, sum1 = 0.0f, sum2 = 0.0f, sum3 = 0.0f;
    float r0s = 0.0f, r1s = 0.0f;
#pragma unroll
    for (int e = 0; e < kBlockN / 2; e += 2) {
        float x0, x1, p0, p1;
        fma2(x0, x1, s[e], s[e + 1], c, c, neg_m, neg_m);
        if (use_poly<EXP_MODE>(e)) {
            ex2_poly2(p0, p1, x0, x1);
        } else {
            p0 = ex2_mufu(x0);
            p1 = ex2_mufu(x1);
        }
        if ((e & 2) == 0) add2(sum0, sum1, sum0, sum1, p0, p1);
        else add2(sum2, sum3, sum2, sum3, p0, p1);
        const uint32_t h = pack_bf16x2(p0, p1);
        pk[e >> 1] = h;
        add_bf16x2_f32(r0s, r1s, h);
    }
    sum += (sum0 + sum1) + (sum2 + sum3);
    sum_pv += r0s + r1s;
}

// The same for 8-bit P: 64 probabilities of a row to e4m3, four per word.
template <int EXP_MODE>
__device__ __forceinline__ float exp_pack_half_fp8(const float *s, float c, float neg_m,
                                                   uint32_t *pk) {
    float sum0 = 0.0f, sum1 = 0.0f, sum2 = 0.0f, sum3 = 0.0f;
#pragma unroll
    for (int e = 0; e < kBlockN / 2; e += 4) {
        float x0, x1, x2, x3, p0, p1, p2, p3;
        fma2(x0, x1, s[e], s[e + 1], c, c, neg_m, neg_m);
        fma2(x2, x3, s[e + 2], s[e + 3], c, c, neg_m, neg_m);
        if (use_poly<EXP_MODE>(e)) {
            ex2_poly2(p0, p1, x0, x1);
        } else {
            p0 = ex2_mufu(x0);
            p1 = ex2_mufu(x1);
        }
        if (use_poly<EXP_MODE>(e + 2)) {
            ex2_poly2(p2, p3, x2, x3);
        } else {
            p2 = ex2_mufu(x2);
            p3 = ex2_mufu(x3);
        }
        add2(sum0, sum1, sum0, sum1, p0, p1);
        add2(sum2, sum3, sum2, sum3, p2, p3);
        pk[e >> 2] = pack_e4m3x4(p0, p1, p2, p3);
    }
    return (sum0 + sum1) + (sum2 + sum3);
}

// Maximum of 32 consecutive scores.
__device__ __forceinline__ float block_max32(const float *s) {
    float a = fmax3(s[0], s[1], s[2]), b = fmax3(s[3], s[4], s[5]);
#pragma unroll
    for (int e = 6; e < 30; e += 4) {
        a = fmax3(a, s[e], s[e + 1]);
        b = fmax3(b, s[e + 2], s[e + 3]);
    }
    return fmax3(a, b, fmaxf(s[30], s[31]));
}

// Direct-P probabilities of 64 scores of a row (two 32-key blocks whose
// maxima are bm[0], bm[1]): f16 pairs to pk, returns their fp32 sum.
// base = p_offset - m (m: the row's integer anchor), so y = s*c + base is
// the log2 score relative to the anchor, raised by the container offset.
// Per block: E = floor(max y) - 2 (the OCP MX exponent rule), r = y - E;
// code = E2M1 magnitude of r by the affine classifier (PREC 2: index
// rint(2r + 2) clamped to [0, 7]) or of 2^r rounded to nearest (PREC 3);
// P = code * 2^E.  Blocks with E < -13 (far below the anchor, where
// 0.5 * 2^E would leave f16's normal range) are dropped; E is at most 13 by
// the choice of p_offset.  The codes of a block are summed exactly in f16.
constexpr float kRintMagic = 12582912.0f;  // 1.5 * 2^23: adding it rounds to an integer
template <int PREC>
__device__ __forceinline__ float direct_p_half(const float *s, const float *bm, float c,
                                               float base, uint32_t *pk) {
    float sum = 0.0f;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const float ymax = fmaf(bm[u], c, base);
        const float ef = floorf(ymax) - 2.0f;
        const bool keep = ef >= -13.0f;  // false for an all-masked block (-inf)
        const int ei = keep ? (int)fminf(ef, 13.0f) : 0;
        const float nb = keep ? base - (float)ei : -INFINITY;  // r = s*c + nb
        const uint32_t h = keep ? (uint32_t)(ei + 15) << 10 : 0u;  // f16 2^E (or 0)
        const uint32_t scale2 = h | (h << 16);
        // affine: t = 2r + 2 + magic, rounded to an integer by the FMA itself
        const float c2 = 2.0f * c, nb2 = 2.0f * nb + (2.0f + kRintMagic);
        uint32_t cs0 = 0u, cs1 = 0u;
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
            const float s0 = s[32 * u + e], s1 = s[32 * u + e + 1];
            uint32_t codes;
            if constexpr (PREC == 2) {
                float t0, t1;
                fma2(t0, t1, s0, s1, c2, c2, nb2, nb2);
                t0 = fminf(fmaxf(t0, kRintMagic), kRintMagic + 7.0f);
                t1 = fminf(fmaxf(t1, kRintMagic), kRintMagic + 7.0f);
                codes = e2m1x2_to_f16x2((__float_as_uint(t0) & 7u) |
                                        ((__float_as_uint(t1) & 7u) << 4));
            } else {
                float r0, r1;
                fma2(r0, r1, s0, s1, c, c, nb, nb);
                codes = e2m1_round_f16x2(ex2_mufu(r0), ex2_mufu(r1));
            }
            pk[(32 * u + e) >> 1] = hmul2_u32(codes, scale2);
            if ((e & 2) == 0) cs0 = hadd2_u32(cs0, codes);
            else cs1 = hadd2_u32(cs1, codes);
        }
        if (keep) sum += f16x2_sum(hadd2_u32(cs0, cs1)) * __uint_as_float((uint32_t)(ei + 127) << 23);
    }
    return sum;
}

// 2^d for an integer-valued d <= 0 (exact; 0 below fp32's normal range and
// for d = -inf).
__device__ __forceinline__ float exp2_neg_int(float d) {
    return d >= -126.0f ? __uint_as_float((uint32_t)((int)d + 127) << 23) : 0.0f;
}

// Score modifiers of n consecutive scores (n even), in log2 units, in place:
// MOD bit 0 soft-cap, bit 1 ALiBi.  v holds <q_i, k_j>; dist0 is
// i + (Sk - Sq) - j of the first as a float.
template <int MOD, int N>
__device__ __forceinline__ void modify_scores(float *v, float c, float k1, float so,
                                              float slope2, float dist0) {
#pragma unroll
    for (int e = 0; e < N; e += 2) {
        float x0, x1;
        if (MOD & 1) {
            float r0, r1;
            softcap_pair(x0, x1, r0, r1, v[e], v[e + 1], k1, so);
        } else {
            mul2(x0, x1, v[e], v[e + 1], c, c);
        }
        if (MOD & 2)
            fma2(x0, x1, -slope2, -slope2, fabsf(dist0 - (float)e), fabsf(dist0 - (float)(e + 1)),
                 x0, x1);
        v[e] = x0;
        v[e + 1] = x1;
    }
}

template <int D, int NS, int EXP_MODE, int MOD = 0, int PREC = 0>
__global__ void __launch_bounds__(kFwdThreads, 1)
attn_fwd_kernel(const __grid_constant__ FwdParams p) {
    static_assert(!(PREC && MOD), "the low-precision paths have no score modifiers");
    constexpr bool FP8 = PREC == 1;
    constexpr bool DP = PREC >= 2;  // Direct-P
    constexpr int EB = FP8 ? 1 : 2;
    using Smem = FwdSmem<D, NS, EB>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_off = smem_u32(smem_raw);
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw + ((1024u - (raw_off & 1023u)) & 1023u));

    const int warp = warp_id();
    const int lane = lane_id();

    // Work item.  (batch, head) pairs are taken in groups of head_group;
    // within a group the heaviest query blocks come first (causal load
    // balance) and consecutive CTAs cycle through the group's heads, so the
    // CTAs resident at any time share the K/V of a few heads in L2.
    const int bh_count = p.Hq * p.B;
    const int G = p.head_group;
    const int nq = p.num_qblocks;
    const int full_groups = bh_count / G;
    const int lin = (int)blockIdx.x;
    int grp, r, ge;
    if (lin < full_groups * G * nq) {
        grp = lin / (G * nq);
        r = lin % (G * nq);
        ge = G;
    } else {
        grp = full_groups;
        r = lin - full_groups * G * nq;
        ge = bh_count - full_groups * G;
    }
    const int qb = nq - 1 - r / ge;
    const int bh = grp * G + r % ge;
    const int hq = bh % p.Hq;
    const int b = bh / p.Hq;
    const int hkv = hq / p.group;
    const int q0 = qb * 2 * kBlockM;

    // ------------------------------------------------------------ prologue
    constexpr uint32_t kTileBytes = kBlockM * D * EB;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&sm.kv_full[s], 1);
            mbar_init(&sm.kv_empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.s_full[i], 1);
            mbar_init(&sm.p_half[i], kBlockM);
            mbar_init(&sm.p_full[i], kBlockM);
            mbar_init(&sm.o_final[i], 1);
        }
        mbar_init(&sm.drain, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        if (lane == 0) {
            // The Q copy needs nothing computed below, so it starts first and
            // its latency overlaps the rest of the prologue.
            mbar_init(&sm.q_full, 1);
            fence_mbar_init();
            prefetch_tensormap(&p.tm_q);
            prefetch_tensormap(&p.tm_k);
            prefetch_tensormap(&p.tm_v);
            mbar_arrive_expect_tx(&sm.q_full, 2 * kTileBytes);
            for (int i = 0; i < 2; ++i)
                for (int c = 0; c < Smem::kChunks; ++c)
                    tma_load_4d(sm.q[i][c], &p.tm_q, &sm.q_full, c * Smem::kChunkElems,
                                q0 + i * kBlockM, hq, b);
        }
        __syncwarp();
        // Key-block range of each query tile: union of its rows' key ranges.
        for (int i = 0; i < 2; ++i) {
            const int r0 = q0 + i * kBlockM;
            KeyRange kr{1, 0};
            if (r0 < p.Sq) kr = tile_key_range(p, r0, min(r0 + kBlockM - 1, p.Sq - 1), lane);
            if (lane == 0) {
                if (kr.lo > kr.hi) {
                    sm.range[i][0] = 1;
                    sm.range[i][1] = 0;
                } else {
                    sm.range[i][0] = kr.lo / kBlockN;
                    sm.range[i][1] = kr.hi / kBlockN;
                }
            }
        }
    }
    if (warp == 8) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem = sm.tmem_base;
    volatile int *abort_flag = &sm.abort_flag;
    const int lo0 = sm.range[0][0], hi0 = sm.range[0][1];
    const int lo1 = sm.range[1][0], hi1 = sm.range[1][1];
    const bool has0 = lo0 <= hi0, has1 = lo1 <= hi1;
    const int ulo = has0 ? (has1 ? min(lo0, lo1) : lo0) : lo1;
    const int uhi = has0 ? (has1 ? max(hi0, hi1) : hi0) : hi1;
    const int n_blocks = (has0 || has1) ? (uhi - ulo + 1) : 0;

    // Registers: the softmax warpgroups hold a 128-column score row per
    // thread; the MMA / TMA warpgroup needs few.  384 x 168 at launch =
    // 2 x 128 x kSoftmaxRegs + 128 x kOtherRegs.  All four warps of a
    // warpgroup execute the same setmaxnreg instruction, and each budget
    // dominates the code of its roles so the compiler allocates per role.
    if (warp >= 8) {
        setmaxnreg_dec<kOtherRegs>();
        if (warp == 9) {
            // ------------------------------------------------------ TMA producer
            if (lane == 0) {
                uint32_t it = 0;
                bool ok = true;
                for (int t = 0; t < n_blocks && ok; ++t) {
                    const int key0 = (ulo + t) * kBlockN;
                    for (int which = 0; which < 2 && ok; ++which, ++it) {
                        const uint32_t slot = it % NS;
                        ok = wait_bounded(&sm.kv_empty[slot], ((it / NS) & 1u) ^ 1u, abort_flag,
                                          p.status, true, p.timeout_ns);
                        if (!ok) break;
                        // Testing only: the first CTA withholds its first K copy (the
                        // loop increment still advances the ring position).
                        if (p.debug_withhold_kv && blockIdx.x == 0 && it == 0) continue;
                        mbar_arrive_expect_tx(&sm.kv_full[slot], kTileBytes);
                        const CUtensorMap *map = which ? &p.tm_v : &p.tm_k;
                        for (int c = 0; c < Smem::kChunks; ++c)
                            tma_load_4d(sm.kv[slot][c], map, &sm.kv_full[slot], c * Smem::kChunkElems,
                                        key0, hkv, b);
                    }
                }
                // Every copy still in flight lands before the CTA can exit (only
                // the last NS loads can be outstanding; on the normal path they
                // have been consumed already).
                wait_bounded(&sm.q_full, 0, abort_flag, p.status, false, p.timeout_ns);
                const uint32_t first = it > NS ? it - NS : 0;
                for (uint32_t L = first; L < it; ++L)
                    wait_bounded(&sm.kv_full[L % NS], (L / NS) & 1u, abort_flag, p.status, false, p.timeout_ns);
            }
            __syncwarp();
        } else if (warp == 8) {
            // --------------------------------------------------- MMA issuer
            // The whole warp runs the schedule, so control flow and descriptor
            // arithmetic stay warp-uniform; one elected lane issues the
            // tcgen05 instructions (and the commits that track them).
            if (n_blocks > 0) {
                const bool leader = elect_one();
                constexpr uint32_t kIdescQK = FP8  ? idesc_e4m3_f32(kBlockM, kBlockN, 0, 0)
                                              : DP ? idesc_f16_f32(kBlockM, kBlockN, 0, 0)
                                                   : idesc_bf16_f32(kBlockM, kBlockN, 0, 0);
                constexpr uint32_t kIdescPV = FP8  ? idesc_e4m3_f32(kBlockM, D, 0, 1)
                                              : DP ? idesc_f16_f32(kBlockM, D, 0, 1)
                                                   : idesc_bf16_f32(kBlockM, D, 0, 1);
                constexpr uint32_t kQTileBytes = Smem::kChunks * Smem::kChunkBytes;
                constexpr uint32_t kChunkBytes = Smem::kChunkBytes;
                // One MMA consumes 32 bytes of each operand row: 16 bf16 or
                // 32 fp8 elements.  PV takes kPvK keys per instruction from
                // 8 TMEM columns of P; a 64-key half of P is kPvSteps of them.
                constexpr int kKSteps = D * EB / 32;
                constexpr int kPvK = 32 / EB;
                constexpr int kPvSteps = (kBlockN / 2) / kPvK;
                // Base descriptors; a K-step or a ring slot only moves the start
                // address (bits 0-13, in 16-byte units), a constant add.
                const uint64_t q_desc = smem_desc_sw128(smem_u32(&sm.q[0][0][0]), 16, 1024);
                const uint64_t k_desc = smem_desc_sw128(smem_u32(&sm.kv[0][0][0]), 16, 1024);
                const uint64_t v_desc =
                    smem_desc_sw128(smem_u32(&sm.kv[0][0][0]), kChunkBytes, 1024);
                bool ok = __all_sync(0xffffffffu,
                                     wait_bounded(&sm.q_full, 0, abort_flag, p.status, true, p.timeout_ns));
                tc_fence_after();
                int k_ready = ulo - 1;  // last key block whose K slot was waited on
                auto ring_pos = [&](int j, int which) -> uint32_t {
                    return 2u * (uint32_t)(j - ulo) + (uint32_t)which;
                };
                auto wait_k = [&](int j) {
                    const uint32_t L = ring_pos(j, 0);
                    if (ok)
                        ok = __all_sync(0xffffffffu, wait_bounded(&sm.kv_full[L % NS],
                                                                  (L / NS) & 1u, abort_flag,
                                                                  p.status, true, p.timeout_ns));
                    tc_fence_after();
                    k_ready = j;
                };
                auto issue_s = [&](int i, int j) {
                    if (k_ready < j) wait_k(j);
                    if (!ok) return;
                    const uint64_t a0 = q_desc + ((i * kQTileBytes) >> 4);
                    const uint64_t b0 = k_desc + (((ring_pos(j, 0) % NS) * kQTileBytes) >> 4);
                    if (leader) {
#pragma unroll
                        for (int ks = 0; ks < kKSteps; ++ks) {
                            const uint32_t off = ((ks >> 2) * kChunkBytes + (ks & 3) * 32) >> 4;
                            mma_ss_k<FP8>(tmem + i * kBlockN, a0 + off, b0 + off, kIdescQK,
                                          ks > 0 ? 1u : 0u);
                        }
                        tc_commit(&sm.s_full[i]);
                    }
                    __syncwarp();
                };
                auto active = [&](int i, int j) -> bool {
                    return i == 0 ? (has0 && j >= lo0 && j <= hi0)
                                  : (has1 && j >= lo1 && j <= hi1);
                };

                for (int i = 0; i < 2; ++i)
                    if (active(i, ulo)) issue_s(i, ulo);
                if (ok && k_ready < ulo) wait_k(ulo);
                if (ok && leader) tc_commit(&sm.kv_empty[ring_pos(ulo, 0) % NS]);
                __syncwarp();

                for (int j = ulo; j <= uhi && ok; ++j) {
                    const uint32_t Lv = ring_pos(j, 1);
                    const uint32_t vslot = Lv % NS;
                    ATTN_TRACE_EVENT(2, j - ulo, 0);
                    ok = __all_sync(0xffffffffu, wait_bounded(&sm.kv_full[vslot], (Lv / NS) & 1u,
                                                              abort_flag, p.status, true, p.timeout_ns));
                    ATTN_TRACE_EVENT(2, j - ulo, 1);
                    if (!ok) break;
                    tc_fence_after();
                    const uint64_t vb = v_desc + ((vslot * kQTileBytes) >> 4);
                    for (int i = 0; i < 2 && ok; ++i) {
                        if (active(i, j)) {
                            const int lo_i = i == 0 ? lo0 : lo1;
                            const int hi_i = i == 0 ? hi0 : hi1;
                            const uint32_t par = (uint32_t)(j - lo_i) & 1u;
                            const uint32_t o_tmem = tmem + 2 * kBlockN + i * D;
                            const uint32_t p_tmem = tmem + i * kBlockN;
                            const uint32_t first = j > lo_i ? 1u : 0u;
                            // PV in two halves of 64 keys, each as soon as its P is in TMEM.
                            // V chunk: key rows of 128 bytes, 8-row groups 1024 B apart
                            // (SBO), 64-column chunks kChunkBytes apart (LBO).
                            ATTN_TRACE_EVENT(2, j - ulo, 2 + 3 * i);
                            ok = __all_sync(0xffffffffu, wait_bounded(&sm.p_half[i], par,
                                                                      abort_flag, p.status, true, p.timeout_ns));
                            if (!ok) break;
                            tc_fence_after();
                            if (leader) {
#pragma unroll
                                for (int ks = 0; ks < kPvSteps; ++ks)
                                    mma_ts_k<FP8>(o_tmem, p_tmem + ks * 8,
                                                  vb + ((ks * kPvK * 128) >> 4), kIdescPV,
                                                  ks > 0 ? 1u : first);
                            }
                            __syncwarp();
                            ok = __all_sync(0xffffffffu, wait_bounded(&sm.p_full[i], par,
                                                                      abort_flag, p.status, true, p.timeout_ns));
                            ATTN_TRACE_EVENT(2, j - ulo, 3 + 3 * i);
                            if (!ok) break;
                            tc_fence_after();
                            if (leader) {
#pragma unroll
                                for (int ks = kPvSteps; ks < 2 * kPvSteps; ++ks)
                                    mma_ts_k<FP8>(o_tmem, p_tmem + ks * 8,
                                                  vb + ((ks * kPvK * 128) >> 4), kIdescPV, 1u);
                                if (j == hi_i) tc_commit(&sm.o_final[i]);
                            }
                            __syncwarp();
                        }
                        if (j + 1 <= uhi && active(i, j + 1)) issue_s(i, j + 1);
                        ATTN_TRACE_EVENT(2, j - ulo, 4 + 3 * i);
                    }
                    if (!ok) break;
                    if (j + 1 <= uhi && k_ready < j + 1) wait_k(j + 1);
                    if (!ok) break;
                    if (leader) {
                        tc_commit(&sm.kv_empty[vslot]);
                        if (j + 1 <= uhi) tc_commit(&sm.kv_empty[ring_pos(j + 1, 0) % NS]);
                    }
                    __syncwarp();
                }
                if (!ok) {
                    // Let every MMA already issued finish before TMEM is freed.
                    if (leader) tc_commit(&sm.drain);
                    __syncwarp();
                    wait_bounded(&sm.drain, 0, abort_flag, p.status, false, p.timeout_ns);
                }
            }
            __syncwarp();
        }
        // warps 10-11: idle
    } else {
        // ------------------------------------- softmax / correction / epilogue
        setmaxnreg_inc<kSoftmaxRegs>();
        const int i = warp >> 2;
        const int row_in_tile = threadIdx.x & (kBlockM - 1);
        const int row = q0 + i * kBlockM + row_in_tile;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t s_tmem = tmem + lane_base + i * kBlockN;
        const uint32_t o_tmem = tmem + lane_base + 2 * kBlockN + i * D;
        const KeyRange kr = row_key_range(p, row);
        const int lo_b = i == 0 ? lo0 : lo1;
        const int hi_b = i == 0 ? hi0 : hi1;
        const float c = p.scale_log2;
        const float tau = p.rescale_threshold;
        // With a modifier the scores are transformed into log2 units before
        // the max, so the exponent step multiplies by 1 instead of c.
        const float c_exp = MOD ? 1.0f : c;
        const float slope2 = (MOD & 2) ? __ldg(p.alibi_slopes + hq) * kLog2eF : 0.0f;
        const float k1 = p.softcap_in * (2.0f * kLog2eF);  // soft-cap: 2 log2(e) scale / cap
        const float diag_f = (float)(row + p.Sk - p.Sq);
#ifdef ATTN_COUNT_RESCALES
        uint32_t cnt_blocks = 0, cnt_raise = 0, cnt_taken = 0, cnt_warp = 0;
#endif
        float m_run = -INFINITY;
        float l_run = 0.0f;   // row sum of the unrounded p (the LSE's normaliser)
        float l_pv = 0.0f;    // row sum of the p that PV consumes (the output's normaliser)
        bool ok = true;

        for (int j = lo_b; j <= hi_b; ++j) {
            const int t = j - lo_b;
            if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, t, 0);
            ok = wait_bounded(&sm.s_full[i], (uint32_t)t & 1u, abort_flag, p.status, true, p.timeout_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, t, 1);

            // Scores of this row: all four loads in flight together, one wait
            // (measured slightly faster than overlapping the second half's
            // load with the first half's max).
            uint32_t sr[kBlockN];
            tmem_ld32(s_tmem + 0, sr + 0);
            tmem_ld32(s_tmem + 32, sr + 32);
            tmem_ld32(s_tmem + 64, sr + 64);
            tmem_ld32(s_tmem + 96, sr + 96);
            tmem_wait_ld();
            reg_fence32(sr + 0);
            reg_fence32(sr + 32);
            reg_fence32(sr + 64);
            reg_fence32(sr + 96);
            float *s = reinterpret_cast<float *>(sr);

            const int key0 = j * kBlockN;
            const float dist0 = diag_f - (float)key0;  // distance to key0 of this block
            const bool need_mask = key0 < kr.lo || key0 + kBlockN - 1 > kr.hi;
            const bool masked = __any_sync(0xffffffffu, need_mask);
            float alpha = 1.0f;
            float neg_m;
            float bm[4];  // Direct-P: maxima of the four 32-key blocks
            if constexpr (DP) {
                // Direct-P: the anchor m is the running max rounded up to an
                // integer, so every rescale is an exact power of two and the
                // block exponents (and codes) do not depend on it.
                if (masked) {
#pragma unroll
                    for (int e = 0; e < kBlockN; ++e) {
                        const int key = key0 + e;
                        if (key < kr.lo || key > kr.hi) s[e] = -INFINITY;
                    }
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) bm[u] = block_max32(s + 32 * u);
                const float m_cand = fmax3(fmaxf(bm[0], bm[1]), bm[2], bm[3]) * c;
                ATTN_COUNT_BLOCK(t, m_cand > m_run, m_cand > m_run + tau);
                if (m_cand > m_run + tau) {
                    const float m_new = ceilf(m_cand);
                    alpha = exp2_neg_int(m_run - m_new);
                    m_run = m_new;
                }
                neg_m = m_run == -INFINITY ? 0.0f : p.p_offset - m_run;
                if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, t, 3);
            } else {
            if (MOD) modify_scores<MOD, kBlockN / 2>(s, c, k1, p.softcap_out, slope2, dist0);
            if (masked) {
#pragma unroll
                for (int e = 0; e < kBlockN / 2; ++e) {
                    const int key = key0 + e;
                    if (key < kr.lo || key > kr.hi) s[e] = -INFINITY;
                }
            }
            float mx[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) mx[u] = fmax3(s[u], s[u + 4], s[u + 8]);
#pragma unroll
            for (int e = 12; e < kBlockN / 2 - 4; e += 8)
#pragma unroll
                for (int u = 0; u < 4; ++u) mx[u] = fmax3(mx[u], s[e + u], s[e + 4 + u]);
#pragma unroll
            for (int u = 0; u < 4; ++u) mx[u] = fmaxf(mx[u], s[kBlockN / 2 - 4 + u]);
            if (MOD)
                modify_scores<MOD, kBlockN / 2>(s + kBlockN / 2, c, k1, p.softcap_out, slope2,
                                                dist0 - (float)(kBlockN / 2));
            if (masked) {
#pragma unroll
                for (int e = kBlockN / 2; e < kBlockN; ++e) {
                    const int key = key0 + e;
                    if (key < kr.lo || key > kr.hi) s[e] = -INFINITY;
                }
            }
#pragma unroll
            for (int e = kBlockN / 2; e < kBlockN; e += 8)
#pragma unroll
                for (int u = 0; u < 4; ++u) mx[u] = fmax3(mx[u], s[e + u], s[e + 4 + u]);
            if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, t, 2);
            const float row_max = fmax3(fmaxf(mx[0], mx[1]), mx[2], mx[3]);
            const float m_cand = MOD ? row_max : row_max * c;
            ATTN_COUNT_BLOCK(t, m_cand > m_run, m_cand > m_run + tau);
            if (m_cand > m_run + tau) {
                alpha = ex2_mufu(m_run - m_cand);
                m_run = m_cand;
            }
            // fp8: P = 2^(x - m + p_offset) <= 2^8 keeps e4m3's range for the
            // small probabilities (the same factor scales l, so O and LSE are
            // unchanged).
            neg_m = m_run == -INFINITY ? 0.0f : (FP8 ? p.p_offset - m_run : -m_run);
            if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, t, 3);
            }

            l_run *= alpha;
            l_pv *= alpha;

            // Correction first: rescale this row of O in TMEM (rare once the
            // max settles) before any P of this block is handed over.  PV of
            // the previous block is complete: the commit that signalled S of
            // this block covers every earlier MMA.
            if (t > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
#ifdef ATTN_COUNT_RESCALES
                ++cnt_warp;
#endif
#pragma unroll
                for (int ch = 0; ch < D / 32; ++ch) {
                    uint32_t r[32];
                    tmem_ld32(o_tmem + ch * 32, r);
                    tmem_wait_ld();
                    reg_fence32(r);
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        float a0, a1;
                        mul2(a0, a1, __uint_as_float(r[e]), __uint_as_float(r[e + 1]), alpha,
                             alpha);
                        r[e] = __float_as_uint(a0);
                        r[e + 1] = __float_as_uint(a1);
                    }
                    tmem_st32(o_tmem + ch * 32, r);
                }
            }

            // Probabilities p = 2^(s*c - m) in pairs, row sum, bf16 pairs to
            // TMEM, in two halves: the MMA warp starts PV on keys [0, 64) while
            // this warp computes keys [64, 128).  Masked blocks (-inf scores)
            // use MUFU only: ex2(-inf) = 0 exactly.
            uint32_t pk[kBlockN / 2];
            if (MOD) __syncwarp();  // converged before the warp-collective TMEM store
            if constexpr (DP) {
                l_run += direct_p_half<PREC>(s, bm, c, neg_m, pk);
                __syncwarp();  // converged before the warp-collective TMEM store
                tmem_st32(s_tmem + 0, pk + 0);
            } else if constexpr (FP8) {
                // 64 e4m3 probabilities per 16 columns.
                l_run += masked ? exp_pack_half_fp8<0>(s, c_exp, neg_m, pk)
                                : exp_pack_half_fp8<EXP_MODE>(s, c_exp, neg_m, pk);
                tmem_st16(s_tmem + 0, pk + 0);
            } else {
                if (masked) exp_pack_half<0>(s, c_exp, neg_m, pk, l_run, l_pv);
                else exp_pack_half<EXP_MODE>(s, c_exp, neg_m, pk, l_run, l_pv);
                tmem_st32(s_tmem + 0, pk + 0);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.p_half[i]);
            if constexpr (DP) {
                l_run += direct_p_half<PREC>(s + 64, bm + 2, c, neg_m, pk + 32);
                if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, t, 4);
                __syncwarp();
                tmem_st32(s_tmem + 32, pk + 32);
            } else if constexpr (FP8) {
                l_run += masked ? exp_pack_half_fp8<0>(s + 64, c_exp, neg_m, pk + 16)
                                : exp_pack_half_fp8<EXP_MODE>(s + 64, c_exp, neg_m, pk + 16);
                if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, t, 4);
                tmem_st16(s_tmem + 16, pk + 16);
            } else {
                if (masked) exp_pack_half<0>(s + 64, c_exp, neg_m, pk + 32, l_run, l_pv);
                else exp_pack_half<EXP_MODE>(s + 64, c_exp, neg_m, pk + 32, l_run, l_pv);
                if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, t, 4);
                tmem_st32(s_tmem + 32, pk + 32);
            }
            tmem_wait_st();
            if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, t, 5);
            tc_fence_before();
            mbar_arrive(&sm.p_full[i]);
        }

        // ----------------------------------------------------------- epilogue
        const bool has_blocks = lo_b <= hi_b;
        if (ok && has_blocks) {
            ok = wait_bounded(&sm.o_final[i], 0, abort_flag, p.status, true, p.timeout_ns);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
        }
        if (ok) {
            const bool row_ok = row < p.Sq;
            // bf16 P: normalise by the sum of the rounded weights PV applied;
            // fp8 and Direct-P: by the row sum (the fp8 bound is derived for
            // it; Direct-P's sum is already over the values PV consumes).
            const float l_out = PREC ? l_run : l_pv;
            const float inv_l = l_out > 0.0f ? (PREC ? p.v_descale : 1.0f) / l_out : 0.0f;
            __nv_bfloat16 *o_row =
                p.o + (((size_t)b * p.Sq + row) * p.Hq + hq) * (size_t)D;
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t r[32];
                if (has_blocks) {
                    tmem_ld32(o_tmem + ch * 32, r);
                    tmem_wait_ld();
                    reg_fence32(r);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) r[e] = 0u;
                }
                uint4 out[4];
                uint32_t *w = reinterpret_cast<uint32_t *>(out);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    w[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv_l,
                                       __uint_as_float(r[2 * e + 1]) * inv_l);
                if (row_ok) {
                    uint4 *dst = reinterpret_cast<uint4 *>(o_row + ch * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[e] = out[e];
                }
            }
            if (row_ok) {
                const float m_lse = PREC ? m_run - p.p_offset : m_run;
                const float lse = l_run > 0.0f ? (m_lse + log2f(l_run)) * 0.69314718055994531f
                                               : -INFINITY;
                p.lse[((size_t)b * p.Hq + hq) * p.Sq + row] = lse;
            }
        }
#ifdef ATTN_COUNT_RESCALES
        if (p.rescale_counts) {
            for (int o = 16; o > 0; o >>= 1) {
                cnt_blocks += __shfl_xor_sync(0xffffffffu, cnt_blocks, o);
                cnt_raise += __shfl_xor_sync(0xffffffffu, cnt_raise, o);
                cnt_taken += __shfl_xor_sync(0xffffffffu, cnt_taken, o);
            }
            if (lane == 0) {
                atomicAdd(p.rescale_counts + 0, (unsigned long long)cnt_blocks);
                atomicAdd(p.rescale_counts + 1, (unsigned long long)cnt_raise);
                atomicAdd(p.rescale_counts + 2, (unsigned long long)cnt_taken);
                atomicAdd(p.rescale_counts + 3, (unsigned long long)cnt_warp);
            }
        }
#endif
    }

    // ------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace tab
