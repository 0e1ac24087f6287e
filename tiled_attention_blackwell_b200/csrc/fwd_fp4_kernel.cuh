// Direct-P forward on the block-scaled FP4 tensor cores (sm_100a), D = 128.
//
// "Hardware-Aware FP4 FlashAttention-4", "Metodología", item 1: Q K^T as an
// NVFP4 product (E2M1 codes, one e4m3 scale per 16 elements), then the
// probabilities built directly as MXFP4 values -- E2M1 codes with one
// power-of-two scale per 32 keys, chosen by the affine classifier or the
// rounded exponential -- and P V as an MXFP4 product, the softmax
// normaliser being the sum of exactly those values.  The codes and block
// exponents are those of the f16-operand Direct-P kernel (direct_p_half in
// fwd_kernel.cuh).  The normaliser -- the sum of the represented values --
// comes from the tensor cores too: each V^T tile carries an extra row of
// E2M1 ones (scale 2^0), so P V with N = 136 leaves sum_j w_j in column 128
// of O, accumulated exactly as the output is.  The softmax warps then only
// classify and pack codes.
//
// CTA shape as in attn_fwd_kernel: two 128-row query tiles of one (batch,
// query head).  Roles: warps 0-3 / 4-7 softmax + correction + epilogue of
// tile 0 / 1, warp 8 issues Q K^T (and allocates TMEM), warp 9 is the TMA
// producer, warp 10 issues P V.  Two issuers because the two products wait
// on different things: Q K^T on the shared S region being loaded, P V on P
// being written; one in-order issuer would hold each behind the other.
//
// Tensor memory is where this kernel differs ("Contribuciones Clave":
// tensor-memory ownership bounds the overlap).  Block-scaled products read
// their scale factors from tensor memory and take P from shared memory, and
// the 512 columns cannot hold two S tiles, two O tiles and the scales, so
// the two query tiles share one S region: Q_i K^T of the other tile is
// issued once this tile's softmax has loaded its scores.  At FP4 rates the
// products are short against the softmax, which is what bounds the loop.
//   [  0,128) S (tile 0 and tile 1 in turn)
//   [128,264) O0 (column 128 of it: the row sum), [272,408) O1
//   [416,432) Q scales  (tile i, K step ks: 416 + 4 (2i + ks))
//   [432,448) K scales  (block parity, K step)
//   [448,480) V scales  (block parity, K step; 8 columns: rows 0-127, then
//             rows 128-135 -- the ones row -- written once)
//   [480,496) P scales  (tile, K step)
//
// Shared memory: Q0, Q1 and a ring of NS slots (K codes or V^T codes, each
// 128 rows x 64 bytes with the 64-byte swizzle, then 8 more rows -- the ones
// row and seven zero rows, written once -- then their two scale atoms), P0
// and P1 as codes in the same layout, and the P scale atoms the softmax
// warps write.
//
// Ordering.  Each issuer's tensor-core operations execute in its issue
// order, so a scale column or shared-memory operand that one of them
// rewrites has been read by its earlier products.  Scale columns of K and V
// alternate by block parity.  The softmax warps learn from pv_done[i] (a
// commit after P_i V(j)) that O_i may be rescaled and P_i rewritten for
// block j + 1; s_free orders the tiles' use of the S region.
#pragma once

#include "fp4_prepare.cuh"
#include "fwd_kernel.cuh"

namespace tab {

constexpr int kFp4Tile = kBlockM * 64;               // 8 KB of codes
constexpr int kFp4Extra = 8 * 64;                    // rows 128-135 of a V^T tile
constexpr int kFp4SfOff = kFp4Tile + kFp4Extra;      // the slot's two scale atoms
constexpr int kFp4Slot = 10 * 1024;                  // slot stride, 1024-aligned
static_assert(kFp4SfOff + 2 * kSfAtom <= kFp4Slot, "slot layout");
constexpr int kPvN = 136;                            // D columns of O plus the sum rows
constexpr uint32_t kColS = 0, kColO = 128, kOStride = 144, kColSfQ = 416, kColSfK = 432,
                   kColSfV = 448, kColSfP = 480;

template <int NS>
struct FwdSmemFp4 {
    alignas(1024) uint8_t q[2][kFp4Tile];
    uint8_t qsf[2][2][kSfAtom];  // [tile][K step]
    alignas(1024) uint8_t kv[NS][kFp4Slot];
    alignas(1024) uint8_t p[2][kFp4Tile];
    uint8_t psf[2][2][kSfAtom];
    uint8_t ones_sf[kSfAtom];  // scales of V^T rows 128-159 (2^0)
    uint64_t q_full;
    uint64_t kv_full[NS];
    uint64_t kv_empty[NS];
    uint64_t s_full[2];
    uint64_t s_free;     // the scores in the shared S region have been loaded
    uint64_t p_full[2];  // P_i's codes and scales are in shared memory (O_i corrected)
    uint64_t o_final[2];
    uint64_t pv_done[2];  // P_i V(j) has completed: P_i and O_i are free again
    uint64_t drain;
    uint64_t drain_pv;
    uint32_t tmem_base;
    int abort_flag;
    int range[2][2];
};

// Codes of 64 scores of a row (two 32-key blocks with maxima bm[0], bm[1]):
// per block the exponent E, the 16 bytes of E2M1 codes (key 2k in the low
// nibble of byte k) and the UE8M0 byte E + 127.  Same block exponents and
// decisions as direct_p_half, with work moved off the ALU pipe:
//   affine: index clamp(rint(2r + 2), 0, 7) as u = sat((2r + 2) / 8) (one
//     FFMA with saturation; the scaling by 1/4 and 8 is exact), rint(8u)
//     through the 1.5 * 2^23 offset (packed FFMA), the eight indices of a
//     word summed into their nibbles by shifted adds of the raw float bits
//     (the offset's bits are a known constant), then 8 -> 7;
//   exp2: 2^r rounded by the E2M1 conversion, four conversions per word.
template <int CLS>
__device__ __forceinline__ void direct_p_codes(const float *s, const float *bm, float c,
                                               float base, uint4 *codes, uint32_t &sf2) {
    constexpr uint32_t kMagicBits = 0x4B400000u;  // kRintMagic
    constexpr uint32_t kMagicNibbles = kMagicBits + (kMagicBits << 4) + (kMagicBits << 8) +
                                       (kMagicBits << 12) + (kMagicBits << 16) +
                                       (kMagicBits << 20) + (kMagicBits << 24) +
                                       (kMagicBits << 28);
    sf2 = 0u;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const float ymax = fmaf(bm[u], c, base);
        const float ef = floorf(ymax) - 2.0f;
        const bool keep = ef >= -13.0f;  // false for an all-masked block (-inf)
        const int ei = keep ? (int)fminf(ef, 13.0f) : 0;
        const float nb = keep ? base - (float)ei : -INFINITY;  // r = s*c + nb
        sf2 |= (uint32_t)(ei + 127) << (8 * u);
        uint32_t w[4];
        if constexpr (CLS == 0) {
            const float c4 = 0.25f * c, nb4 = 0.25f * (nb + 1.0f);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t word = 0u;
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    const float u0 = __saturatef(fmaf(s[32 * u + 8 * q + e], c4, nb4));
                    const float u1 = __saturatef(fmaf(s[32 * u + 8 * q + e + 1], c4, nb4));
                    float t0, t1;
                    fma2(t0, t1, u0, u1, 8.0f, 8.0f, kRintMagic, kRintMagic);
                    word += (__float_as_uint(t0) << (4 * e)) + (__float_as_uint(t1) << (4 * e + 4));
                }
                word -= kMagicNibbles;                    // nibbles k in [0, 8]
                w[q] = word - ((word >> 3) & 0x11111111u);  // 8 -> 7
            }
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float x[8];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    float r0, r1;
                    fma2(r0, r1, s[32 * u + 8 * q + e], s[32 * u + 8 * q + e + 1], c, c, nb, nb);
                    x[e] = ex2_mufu(r0);
                    x[e + 1] = ex2_mufu(r1);
                }
                w[q] = e2m1x8_round(x);
            }
        }
        codes[u] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

template <int NS, int CLS>
__global__ void __launch_bounds__(kFwdThreads, 1)
attn_fwd_fp4bs_kernel(const __grid_constant__ FwdParams p) {
    using Smem = FwdSmemFp4<NS>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_off = smem_u32(smem_raw);
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw + ((1024u - (raw_off & 1023u)) & 1023u));

    const int warp = warp_id();
    const int lane = lane_id();

    // Work item: the order of attn_fwd_kernel (head groups, heaviest query
    // blocks first).
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
    // The affine classifier's build starts the Q copy first; the exp2
    // build measured slower with it and keeps the copy after the prologue.
    constexpr bool kQFirst = CLS == 0;
    if (threadIdx.x == 0) {
        if (!kQFirst) mbar_init(&sm.q_full, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&sm.kv_full[s], 1);
            mbar_init(&sm.kv_empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.s_full[i], 1);
            mbar_init(&sm.p_full[i], kBlockM);
            mbar_init(&sm.o_final[i], 1);
        }
        mbar_init(&sm.s_free, kBlockM);
        mbar_init(&sm.pv_done[0], 1);
        mbar_init(&sm.pv_done[1], 1);
        mbar_init(&sm.drain, 1);
        mbar_init(&sm.drain_pv, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    // Rows 128-135 of every slot: row 128 all E2M1 ones (code 2), the rest
    // zero (the 64-byte swizzle permutes chunks within a row: a constant row
    // is the same either way); their scale atom: 2^0 (UE8M0 127) for the two
    // 32-key blocks of each K step.
    for (int x = threadIdx.x; x < NS * kFp4Extra / 16; x += kFwdThreads) {
        const int slot = x / (kFp4Extra / 16), off = x % (kFp4Extra / 16);
        const uint32_t v = off < 4 ? 0x22222222u : 0u;
        *reinterpret_cast<uint4 *>(sm.kv[slot] + kFp4Tile + off * 16) = make_uint4(v, v, v, v);
    }
    for (int x = threadIdx.x; x < kSfAtom / 4; x += kFwdThreads)
        reinterpret_cast<uint32_t *>(sm.ones_sf)[x] = 0x00007F7Fu;
    fence_proxy_async_smem();
    if (warp == 9) {
        if (kQFirst && lane == 0) {
            // The Q copy needs nothing computed below, so it starts first and
            // its latency overlaps the rest of the prologue.
            mbar_init(&sm.q_full, 1);
            fence_mbar_init();
            prefetch_tensormap(&p.tm_q);
            prefetch_tensormap(&p.tm_k);
            prefetch_tensormap(&p.tm_v);
            mbar_arrive_expect_tx(&sm.q_full, 2 * kFp4Tile + 4 * kSfAtom);
            for (int i = 0; i < 2; ++i)
                tma_load_4d(sm.q[i], &p.tm_q, &sm.q_full, 0, q0 + i * kBlockM, hq, b);
            // Both tiles' scale atoms (tiles 2 qb and 2 qb + 1) are adjacent.
            bulk_load(sm.qsf, p.sf_q + (((size_t)b * p.Hq + hq) * p.nq_tiles + 2 * qb) * (2 * kSfAtom),
                      4 * kSfAtom, &sm.q_full);
        }
        __syncwarp();
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

    if (warp >= 8) {
        setmaxnreg_dec<kOtherRegs>();
        if (warp == 9) {
            // ------------------------------------------------------ TMA producer
            if (lane == 0) {
                if (!kQFirst) {
                    prefetch_tensormap(&p.tm_q);
                    prefetch_tensormap(&p.tm_k);
                    prefetch_tensormap(&p.tm_v);
                    mbar_arrive_expect_tx(&sm.q_full, 2 * kFp4Tile + 4 * kSfAtom);
                    for (int i = 0; i < 2; ++i)
                        tma_load_4d(sm.q[i], &p.tm_q, &sm.q_full, 0, q0 + i * kBlockM, hq, b);
                    bulk_load(sm.qsf,
                              p.sf_q + (((size_t)b * p.Hq + hq) * p.nq_tiles + 2 * qb) * (2 * kSfAtom),
                              4 * kSfAtom, &sm.q_full);
                }
                uint32_t it = 0;
                bool ok = true;
                for (int t = 0; t < n_blocks && ok; ++t) {
                    const int j = ulo + t;
                    for (int which = 0; which < 2 && ok; ++which, ++it) {
                        const uint32_t slot = it % NS;
                        ok = wait_bounded(&sm.kv_empty[slot], ((it / NS) & 1u) ^ 1u, abort_flag,
                                          p.status, true, p.timeout_ns);
                        if (!ok) break;
                        // Testing only: the first CTA withholds its first K copy.
                        if (p.debug_withhold_kv && blockIdx.x == 0 && it == 0) continue;
                        mbar_arrive_expect_tx(&sm.kv_full[slot], kFp4Tile + 2 * kSfAtom);
                        const size_t atoms = (((size_t)b * p.Hkv + hkv) * p.nk_tiles + j) * (2 * kSfAtom);
                        if (which == 0) {
                            tma_load_4d(sm.kv[slot], &p.tm_k, &sm.kv_full[slot], 0, j * kBlockN, hkv, b);
                            bulk_load(sm.kv[slot] + kFp4SfOff, p.sf_k + atoms, 2 * kSfAtom, &sm.kv_full[slot]);
                        } else {
                            tma_load_4d(sm.kv[slot], &p.tm_v, &sm.kv_full[slot], j * 64, 0, hkv, b);
                            bulk_load(sm.kv[slot] + kFp4SfOff, p.sf_v + atoms, 2 * kSfAtom, &sm.kv_full[slot]);
                        }
                    }
                }
                wait_bounded(&sm.q_full, 0, abort_flag, p.status, false, p.timeout_ns);
                const uint32_t first = it > NS ? it - NS : 0;
                for (uint32_t L = first; L < it; ++L)
                    wait_bounded(&sm.kv_full[L % NS], (L / NS) & 1u, abort_flag, p.status, false, p.timeout_ns);
            }
            __syncwarp();
        } else if (warp == 8) {
            // ------------------------------------------- Q K^T issuer (S ring)
            // One S region serves both tiles in turn: the n-th product waits
            // until the tile that owned the region has loaded its scores.
            if (n_blocks > 0) {
                const bool leader = elect_one();
                constexpr uint32_t kIdescQK = idesc_fp4_bs(kBlockM, kBlockN, 0);  // UE4M3 scales
                const uint64_t q_desc = smem_desc_sw64(smem_u32(sm.q[0]));
                const uint64_t kv_desc = smem_desc_sw64(smem_u32(sm.kv[0]));
                bool ok = __all_sync(0xffffffffu,
                                     wait_bounded(&sm.q_full, 0, abort_flag, p.status, true, p.timeout_ns));
                tc_fence_after();
                if (ok && leader)
                    for (int i = 0; i < 2; ++i)
                        for (int ks = 0; ks < 2; ++ks)
                            tc_cp_sf(tmem + kColSfQ + 4 * (2 * i + ks),
                                     smem_desc_sf_atom(smem_u32(sm.qsf[i][ks])));
                __syncwarp();
                uint32_t n_qk = 0;
                for (int j = ulo; j <= uhi && ok; ++j) {
                    const uint32_t Lk = 2u * (uint32_t)(j - ulo);
                    const uint32_t kslot = Lk % NS;
                    ATTN_TRACE_EVENT(2, j - ulo, 0);
                    ok = __all_sync(0xffffffffu, wait_bounded(&sm.kv_full[kslot], (Lk / NS) & 1u,
                                                              abort_flag, p.status, true, p.timeout_ns));
                    if (!ok) break;
                    tc_fence_after();
                    if (leader)
                        for (int ks = 0; ks < 2; ++ks)
                            tc_cp_sf(tmem + kColSfK + 4 * (2 * (j & 1) + ks),
                                     smem_desc_sf_atom(smem_u32(sm.kv[kslot] + kFp4SfOff + ks * kSfAtom)));
                    __syncwarp();
                    const uint64_t b0 = kv_desc + ((kslot * kFp4Slot) >> 4);
                    for (int i = 0; i < 2 && ok; ++i) {
                        const bool act = i == 0 ? (has0 && j >= lo0 && j <= hi0)
                                                : (has1 && j >= lo1 && j <= hi1);
                        if (!act) continue;
                        if (n_qk > 0) {
                            ok = __all_sync(0xffffffffu, wait_bounded(&sm.s_free, (n_qk - 1) & 1u,
                                                                      abort_flag, p.status, true,
                                                                      p.timeout_ns));
                            if (!ok) break;
                            tc_fence_after();
                        }
                        ATTN_TRACE_EVENT(2, j - ulo, 1 + i);
                        const uint64_t a0 = q_desc + ((i * kFp4Tile) >> 4);
                        if (leader) {
#pragma unroll
                            for (int ks = 0; ks < 2; ++ks)
                                mma_nvf4(tmem + kColS, a0 + 2 * ks, b0 + 2 * ks, kIdescQK,
                                         tmem + kColSfQ + 4 * (2 * i + ks),
                                         tmem + kColSfK + 4 * (2 * (j & 1) + ks), ks > 0 ? 1u : 0u);
                            tc_commit(&sm.s_full[i]);
                        }
                        __syncwarp();
                        ++n_qk;
                    }
                    if (!ok) break;
                    if (leader) tc_commit(&sm.kv_empty[kslot]);
                    __syncwarp();
                }
                if (!ok) {
                    // Let every product and copy already issued finish before TMEM is freed.
                    if (leader) tc_commit(&sm.drain);
                    __syncwarp();
                    wait_bounded(&sm.drain, 0, abort_flag, p.status, false, p.timeout_ns);
                }
            }
            __syncwarp();
        } else if (warp == 10) {
            // ---------------------------------------------------- P V issuer
            // P_i V(j) as soon as P_i of block j is in shared memory;
            // pv_done[i] tells the softmax warps that P_i and O_i may be
            // touched again.
            if (n_blocks > 0) {
                const bool leader = elect_one();
                constexpr uint32_t kIdescPV = idesc_fp4_bs(kBlockM, kPvN, 1);  // UE8M0 scales
                const uint64_t kv_desc = smem_desc_sw64(smem_u32(sm.kv[0]));
                const uint64_t p_desc = smem_desc_sw64(smem_u32(sm.p[0]));
                if (leader)  // scales of the ones row, once for the four V scale groups
                    for (int g = 0; g < 4; ++g)
                        tc_cp_sf(tmem + kColSfV + 8 * g + 4, smem_desc_sf_atom(smem_u32(sm.ones_sf)));
                __syncwarp();
                bool ok = true;
                for (int j = ulo; j <= uhi && ok; ++j) {
                    const uint32_t Lv = 2u * (uint32_t)(j - ulo) + 1u;
                    const uint32_t vslot = Lv % NS;
                    ok = __all_sync(0xffffffffu, wait_bounded(&sm.kv_full[vslot], (Lv / NS) & 1u,
                                                              abort_flag, p.status, true, p.timeout_ns));
                    if (!ok) break;
                    tc_fence_after();
                    if (leader)
                        for (int ks = 0; ks < 2; ++ks)
                            tc_cp_sf(tmem + kColSfV + 8 * (2 * (j & 1) + ks),
                                     smem_desc_sf_atom(smem_u32(sm.kv[vslot] + kFp4SfOff + ks * kSfAtom)));
                    __syncwarp();
                    const uint64_t vb = kv_desc + ((vslot * kFp4Slot) >> 4);
                    for (int i = 0; i < 2 && ok; ++i) {
                        const int lo_i = i == 0 ? lo0 : lo1;
                        const int hi_i = i == 0 ? hi0 : hi1;
                        const bool act = i == 0 ? (has0 && j >= lo0 && j <= hi0)
                                                : (has1 && j >= lo1 && j <= hi1);
                        if (!act) continue;
                        const uint32_t par = (uint32_t)(j - lo_i) & 1u;
                        const uint32_t o_tmem = tmem + kColO + i * kOStride;
                        const uint64_t pa = p_desc + ((i * kFp4Tile) >> 4);
                        ok = __all_sync(0xffffffffu, wait_bounded(&sm.p_full[i], par, abort_flag, p.status,
                                                                  true, p.timeout_ns));
                        if (!ok) break;
                        tc_fence_after();
#pragma unroll
                        for (int ks = 0; ks < 2; ++ks) {
                            if (leader) {
                                tc_cp_sf(tmem + kColSfP + 4 * (2 * i + ks),
                                         smem_desc_sf_atom(smem_u32(sm.psf[i][ks])));
                                mma_mxf4(o_tmem, pa + 2 * ks, vb + 2 * ks, kIdescPV,
                                         tmem + kColSfP + 4 * (2 * i + ks),
                                         tmem + kColSfV + 8 * (2 * (j & 1) + ks),
                                         (ks > 0 || j > lo_i) ? 1u : 0u);
                            }
                            __syncwarp();
                        }
                        if (!ok) break;
                        if (leader) {
                            tc_commit(&sm.pv_done[i]);
                            if (j == hi_i) tc_commit(&sm.o_final[i]);
                        }
                        __syncwarp();
                    }
                    if (!ok) break;
                    if (leader) tc_commit(&sm.kv_empty[vslot]);
                    __syncwarp();
                }
                if (!ok) {
                    if (leader) tc_commit(&sm.drain_pv);
                    __syncwarp();
                    wait_bounded(&sm.drain_pv, 0, abort_flag, p.status, false, p.timeout_ns);
                }
            }
            __syncwarp();
        }
        // warp 11: idle
    } else {
        // ------------------------------------- softmax / correction / epilogue
        setmaxnreg_inc<kSoftmaxRegs>();
        const int i = warp >> 2;
        const int row_in_tile = threadIdx.x & (kBlockM - 1);
        const int row = q0 + i * kBlockM + row_in_tile;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t s_tmem = tmem + lane_base + kColS;
        const uint32_t o_tmem = tmem + lane_base + kColO + i * kOStride;
        const KeyRange kr = row_key_range(p, row);
        const int lo_b = i == 0 ? lo0 : lo1;
        const int hi_b = i == 0 ? hi0 : hi1;
        const float c = p.scale_log2;
        const float tau = p.rescale_threshold;
        // This row's 64 bytes of P codes: 16-byte chunk u (keys [32u, 32u + 32))
        // at chunk u ^ ((row >> 1) & 3), the 64-byte swizzle; its scale word at
        // 16 (row % 32) + 4 (row / 32) of the K step's atom.
        uint8_t *p_row = sm.p[i] + row_in_tile * 64;
        const int swz = (row_in_tile >> 1) & 3;
        const int sf_off = 16 * (row_in_tile & 31) + 4 * (row_in_tile >> 5);
#ifdef ATTN_COUNT_RESCALES
        uint32_t cnt_blocks = 0, cnt_raise = 0, cnt_taken = 0, cnt_warp = 0;
#endif
        float m_run = -INFINITY;
        bool ok = true;

        for (int j = lo_b; j <= hi_b; ++j) {
            const int t = j - lo_b;
            if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, t, 0);
            ok = wait_bounded(&sm.s_full[i], (uint32_t)t & 1u, abort_flag, p.status, true, p.timeout_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, t, 1);

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
            // The S region is free for the other tile's next product.
            tc_fence_before();
            mbar_arrive(&sm.s_free);
            if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, t, 2);
            float *s = reinterpret_cast<float *>(sr);

            const int key0 = j * kBlockN;
            const bool need_mask = key0 < kr.lo || key0 + kBlockN - 1 > kr.hi;
            if (__any_sync(0xffffffffu, need_mask)) {
#pragma unroll
                for (int e = 0; e < kBlockN; ++e) {
                    const int key = key0 + e;
                    if (key < kr.lo || key > kr.hi) s[e] = -INFINITY;
                }
            }
            float bm[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) bm[u] = block_max32(s + 32 * u);
            const float m_cand = fmax3(fmaxf(bm[0], bm[1]), bm[2], bm[3]) * c;
            float alpha = 1.0f;
            ATTN_COUNT_BLOCK(t, m_cand > m_run, m_cand > m_run + tau);
            if (m_cand > m_run + tau) {
                const float m_new = ceilf(m_cand);
                alpha = exp2_neg_int(m_run - m_new);
                m_run = m_new;
            }
            const float neg_m = m_run == -INFINITY ? 0.0f : p.p_offset - m_run;
            if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, t, 3);

            // All codes in registers, then wait until P_i V(j-1) has
            // completed: only then may O_i be rescaled (the correction, rare
            // once the maximum settles; it covers the sum column too) and P_i
            // and its scales be overwritten.  P is handed over once per block
            // (measured 7 % faster than in two halves of 64 keys: one proxy
            // fence and one hand-off fewer, and the two halves' code
            // generation interleaves).
            uint4 codes[4];
            uint32_t sf2[2];
            direct_p_codes<CLS>(s, bm, c, neg_m, codes, sf2[0]);
            direct_p_codes<CLS>(s + 64, bm + 2, c, neg_m, codes + 2, sf2[1]);
            if (t > 0) {
                ok = __all_sync(0xffffffffu, wait_bounded(&sm.pv_done[i], (uint32_t)(t - 1) & 1u,
                                                          abort_flag, p.status, true, p.timeout_ns));
                if (!ok) break;
                tc_fence_after();
            }
            if (t > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
#ifdef ATTN_COUNT_RESCALES
                ++cnt_warp;
#endif
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    uint32_t rr[32];
                    tmem_ld32(o_tmem + ch * 32, rr);
                    tmem_wait_ld();
                    reg_fence32(rr);
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        float a0, a1;
                        mul2(a0, a1, __uint_as_float(rr[e]), __uint_as_float(rr[e + 1]), alpha, alpha);
                        rr[e] = __float_as_uint(a0);
                        rr[e + 1] = __float_as_uint(a1);
                    }
                    tmem_st32(o_tmem + ch * 32, rr);
                }
                uint32_t r8[8];
                tmem_ld8(o_tmem + 128, r8);
                tmem_wait_ld();
                reg_fence8(r8);
                r8[0] = __float_as_uint(__uint_as_float(r8[0]) * alpha);
                tmem_st8(o_tmem + 128, r8);
                tmem_wait_st();
            }

            // All codes and scale bytes to shared memory, made visible to the
            // tensor cores, then signalled once.
#pragma unroll
            for (int u = 0; u < 4; ++u)
                *reinterpret_cast<uint4 *>(p_row + ((u ^ swz) << 4)) = codes[u];
            *reinterpret_cast<uint32_t *>(sm.psf[i][0] + sf_off) = sf2[0];
            *reinterpret_cast<uint32_t *>(sm.psf[i][1] + sf_off) = sf2[1];
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&sm.p_full[i]);
            if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, t, 4);
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
            float l_run = 0.0f;  // sum of the represented weights, from the ones row
            if (has_blocks) {
                uint32_t r8[8];
                tmem_ld8(o_tmem + 128, r8);
                tmem_wait_ld();
                reg_fence8(r8);
                l_run = __uint_as_float(r8[0]);
            }
            const float inv_l = l_run > 0.0f ? p.v_descale / l_run : 0.0f;
            __nv_bfloat16 *o_row = p.o + (((size_t)b * p.Sq + row) * p.Hq + hq) * (size_t)128;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                uint32_t rr[32];
                if (has_blocks) {
                    tmem_ld32(o_tmem + ch * 32, rr);
                    tmem_wait_ld();
                    reg_fence32(rr);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) rr[e] = 0u;
                }
                uint4 out[4];
                uint32_t *w = reinterpret_cast<uint32_t *>(out);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    w[e] = pack_bf16x2(__uint_as_float(rr[2 * e]) * inv_l,
                                       __uint_as_float(rr[2 * e + 1]) * inv_l);
                if (row_ok) {
                    uint4 *dst = reinterpret_cast<uint4 *>(o_row + ch * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[e] = out[e];
                }
            }
            if (row_ok) {
                const float lse = l_run > 0.0f
                                      ? (m_run - p.p_offset + log2f(l_run)) * 0.69314718055994531f
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
