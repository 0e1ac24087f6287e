// Fused exact-attention backward for B200 (sm_100a).
//
// Gradients of O = softmax(scale * Q K^T + mask) V given dO, rebuilding the
// probabilities from the forward's LSE instead of storing them
// ("Hardware-Aware FP4 FlashAttention-4", "Causal Backward Cuantizado": the
// backward reconstructs the probabilities from the saved normaliser;
// "FlashAttention-4发布", "从V1到V4", first bullet: recomputation).  With
// D_i = sum_d dO_id O_id, P = exp(s - LSE), dP = dO V^T, dS = P (dP - D):
//   dV = P^T dO,  dK = scale dS^T Q,  dQ = scale dS K.
//
// Two kernels, no atomics (deterministic), dQ first:
//   attn_bwd_dq_kernel          one CTA per (batch, query head, 128-row
//                               block): D_i of its rows (from O and dO,
//                               also stored in the caller's workspace),
//                               S = Q K^T, dP = dO V^T, dS into TMEM,
//                               dQ += dS K.
//   attn_bwd_dkdv_kernel        one CTA per (batch, kv head, 128-key block):
//                               keys in TMEM lanes, S^T = K Q^T and
//                               dP^T = V dO^T per query block, P^T and dS^T
//                               written back into TMEM as bf16, then
//                               dV += P^T dO and dK += dS^T Q (A from TMEM);
//                               the query heads of a GQA group accumulate
//                               into the same TMEM; D_i from the workspace.
// Warp roles in both main kernels (320 threads): warps 0-7 elementwise
// (warps 0-3 take columns [0, 64) of each 128-wide tile, warps 4-7 columns
// [64, 128); one TMEM lane per thread; the work is purely elementwise, so the
// halves need no exchange), warp 8 MMA issue (warp-uniform, one elected
// lane), warp 9 TMA producer.  Every wait is bounded as in the forward.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace tab {

constexpr int kBwdThreads = 320;
constexpr int kBwdMmaWarp = 8;
constexpr int kBwdLoadWarp = 9;

// TMEM column of the bf16 operand (P, P^T, dS or dS^T) for K-step ks of a
// 128-wide contraction: each elementwise warpgroup writes its 64 columns'
// pairs into the first 32 columns of its own half of the score tile, so the
// two halves never touch each other's cells.
__device__ __forceinline__ uint32_t half_operand_col(uint32_t base, int ks) {
    return base + (ks < 4 ? ks * 8 : 64 + (ks - 4) * 8);
}
constexpr float kLog2e = 1.4426950408889634f;

// 2^x for element e of a 64-wide row half: two pairs in five on the FMA pipe
// (our cubic, clamped at -125), the rest on MUFU, spread so the two units
// work side by side.  Used only where no element is masked.
__device__ __forceinline__ float bwd_ex2(float x, int e) {
    const int pair = (e >> 1) % 5;
    return (pair == 1 || pair == 3) ? ex2_poly(x) : ex2_mufu(x);
}
// The same split for the pair (e, e+1), e even, in packed f32x2 arithmetic.
__device__ __forceinline__ void bwd_ex2_pair(float &y0, float &y1, float x0, float x1, int e) {
    const int pair = (e >> 1) % 5;
    if (pair == 1 || pair == 3) {
        ex2_poly2(y0, y1, x0, x1);
    } else {
        y0 = ex2_mufu(x0);
        y1 = ex2_mufu(x1);
    }
}

struct BwdParams {
    CUtensorMap tm_q;   // bf16 [B][Sq][Hq][D] as (64, Sq, D/64, Hq, B), box = one tile
    CUtensorMap tm_do;  // bf16 [B][Sq][Hq][D]
    CUtensorMap tm_k;   // bf16 [B][Sk][Hkv][D]
    CUtensorMap tm_v;
    const __nv_bfloat16 *o;
    const __nv_bfloat16 *dout;
    const float *lse;   // [B][Hq][Sq], natural log
    float *dval;        // workspace: D_i, [B][Hq][Sq]
    float *dq;          // fp32 [B][Sq][Hq][D]
    __nv_bfloat16 *dk;  // bf16 [B][Sk][Hkv][D]
    __nv_bfloat16 *dv;
    const int *doc_offsets;
    int *status;
    int num_docs;
    int B, Hq, Hkv, Sq, Sk, group;
    int causal, window_left, window_right;
    int num_qb, num_kb;  // 128-row query blocks, 128-key blocks
    float scale;
    float scale_log2;
    long long *trace;  // clock64 event log (trace builds only), else null
    int trace_ctas;
    // Score modifiers (MOD != 0 kernels), as in the forward: soft-cap
    // softcap_out * tanh(raw * softcap_in) in log2 units; ALiBi slopes per
    // query head (device fp32 [Hq]) or null.
    float softcap_in;   // scale / cap
    float softcap_out;  // cap * log2(e)
    const float *alibi_slopes;
};

// Modified scores of a pair in log2 units (MOD bit 0 soft-cap, bit 1 ALiBi
// at distances d0, d1 = i + (Sk - Sq) - j) and their derivatives with
// respect to the scaled score scale * raw: 1 - tanh^2 = 4 r (1 - r) under
// the cap (see softcap_pair), else 1 (the ALiBi bias is constant).
template <int MOD>
__device__ __forceinline__ void bwd_modified_pair(float &x0, float &x1, float &f0, float &f1,
                                                  float raw0, float raw1, float c, float k1,
                                                  float so, float slope2, float d0, float d1) {
    if (MOD & 1) {
        float r0, r1, m0, m1;
        softcap_pair(x0, x1, r0, r1, raw0, raw1, k1, so);
        mul2(m0, m1, r0, r1, 4.0f, 4.0f);
        fma2(f0, f1, -m0, -m1, r0, r1, m0, m1);
    } else {
        mul2(x0, x1, raw0, raw1, c, c);
        f0 = f1 = 1.0f;
    }
    if (MOD & 2) fma2(x0, x1, -slope2, -slope2, fabsf(d0), fabsf(d1), x0, x1);
}

// Opt-in event trace of the dK/dV kernel (compile with -DATTN_TRACE), same
// layout as the forward's: [cta][role][item][event], roles 0 = elementwise
// warp 0, 1 = TMA producer, 2 = MMA warp.
#ifdef ATTN_TRACE
#define BWD_TRACE(role, iter, ev)                                                            \
    do {                                                                                   \
        if (p.trace && (int)blockIdx.x < p.trace_ctas && (iter) < 96 && lane == 0)            \
            p.trace[(((size_t)blockIdx.x * 3 + (role)) * 96 + (iter)) * 8 + (ev)] = clock64(); \
    } while (0)
#else
#define BWD_TRACE(role, iter, ev) \
    do {                          \
    } while (0)
#endif


// --------------------------------------------------------------- dK and dV

template <int D, int NSQ>
struct DkdvSmem {
    static constexpr int kChunks = D / 64;
    static constexpr int kChunkElems = 128 * 64;  // 16 KB
    __nv_bfloat16 k[kChunks][kChunkElems];
    __nv_bfloat16 v[kChunks][kChunkElems];
    __nv_bfloat16 q[NSQ][kChunks][kChunkElems];
    __nv_bfloat16 dout[NSQ][kChunks][kChunkElems];
    float lse2[NSQ][128];  // LSE * log2(e) of the block's rows (+inf past Sq)
    float dval[NSQ][128];  // D_i of the block's rows (0 past Sq)
    int rlo[NSQ][128];     // key interval of each row (lo > hi: none)
    int rhi[NSQ][128];
    int full[NSQ];         // every (row, key) pair of the item is allowed
    uint64_t kv_full;
    uint64_t st_full[NSQ];
    uint64_t st_empty[NSQ];
    uint64_t s_full, dp_full, p_ready, ds_ready, final_bar, drain;
    uint32_t tmem_base;
    int abort_flag;
    int qb_lo, qb_hi;
};

template <int D, int NSQ, int MOD = 0>
__global__ void __launch_bounds__(kBwdThreads, 1)
attn_bwd_dkdv_kernel(const __grid_constant__ BwdParams p) {
    using Smem = DkdvSmem<D, NSQ>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_off = smem_u32(smem_raw);
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw + ((1024u - (raw_off & 1023u)) & 1023u));
    const int warp = warp_id();
    const int lane = lane_id();

    // Work item: lowest key blocks first (under a causal mask they see the
    // most query blocks), then (batch, kv head).
    const int bh_count = p.Hkv * p.B;
    const int kb = (int)(blockIdx.x / bh_count);
    const int bh = (int)(blockIdx.x % bh_count);
    const int hkv = bh % p.Hkv;
    const int b = bh / p.Hkv;
    const int k0 = kb * 128;
    const int k1 = min(k0 + 127, p.Sk - 1);
    constexpr uint32_t kTileBytes = 128 * D * 2;

    if (threadIdx.x == 0) {
        mbar_init(&sm.kv_full, 1);
        for (int s = 0; s < NSQ; ++s) {
            mbar_init(&sm.st_full[s], 32);
            mbar_init(&sm.st_empty[s], 1);
        }
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.dp_full, 1);
        mbar_init(&sm.p_ready, 256);
        mbar_init(&sm.ds_ready, 256);
        mbar_init(&sm.final_bar, 1);
        mbar_init(&sm.drain, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kBwdLoadWarp) {
        // Query blocks whose rows can see this key block: the first and last
        // rows of a block bound its rows' key intervals (the intervals'
        // ends never decrease with the row), so a block is kept when its
        // first row's lower end is <= k1 and its last row's upper end is
        // >= k0.  Rows without keys count as (-1, -1).
        int lo = 0x7fffffff, hi = -1;
        for (int qb = lane; qb < p.num_qb; qb += 32) {
            const int r0 = qb * 128;
            const int r1 = min(r0 + 127, p.Sq - 1);
            KeyRange a = row_key_range(p, r0);
            KeyRange z = row_key_range(p, r1);
            const int a_lo = a.lo <= a.hi ? a.lo : -1;
            const int z_hi = z.lo <= z.hi ? z.hi : -1;
            if (a_lo <= k1 && z_hi >= k0) {
                lo = min(lo, qb);
                hi = max(hi, qb);
            }
        }
        for (int o = 16; o > 0; o >>= 1) {
            lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
            hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        if (lane == 0) {
            sm.qb_lo = lo;
            sm.qb_hi = hi;
        }
    }
    if (warp == kBwdMmaWarp) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem = sm.tmem_base;
    volatile int *abort_flag = &sm.abort_flag;
    const int qb_lo = sm.qb_lo, qb_hi = sm.qb_hi;
    const int n_qb = qb_hi >= qb_lo ? qb_hi - qb_lo + 1 : 0;
    const int n_items = n_qb * p.group;  // (query head in group, query block)
    // TMEM columns: S^T [0,128), dP^T [128,256), dV [256,256+D), dK [256+D,256+2D)
    constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;

    if (warp == kBwdLoadWarp) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tensormap(&p.tm_q);
            prefetch_tensormap(&p.tm_do);
            prefetch_tensormap(&p.tm_k);
            prefetch_tensormap(&p.tm_v);
            mbar_arrive_expect_tx(&sm.kv_full, 2 * kTileBytes);
            tma_load_5d(sm.k[0], &p.tm_k, &sm.kv_full, 0, k0, 0, hkv, b);
            tma_load_5d(sm.v[0], &p.tm_v, &sm.kv_full, 0, k0, 0, hkv, b);
        }
        __syncwarp();
        bool ok = true;
        int issued = 0;
        // The per-row data of the next item (LSE, D_i, key interval, whether
        // the whole item is unmasked) is computed one item ahead, while this
        // warp would otherwise wait for a free stage; after the wait only the
        // tile copies and the shared-memory stores remain.
        float nl[4], nd[4];
        int nlo[4], nhi[4];
        bool nfull = true;
        auto prefetch = [&](int it) {
            const int g = it / n_qb;
            const int qb = qb_lo + it % n_qb;
            const size_t rb = ((size_t)b * p.Hq + hkv * p.group + g) * p.Sq;
            nfull = true;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int r = qb * 128 + lane + 32 * m;
                const size_t ri = rb + (r < p.Sq ? r : 0);  // in bounds either way
                nl[m] = ld_nc_f32(p.lse + ri);
                nd[m] = ld_nc_f32(p.dval + ri);
                const KeyRange kr = r < p.Sq ? row_key_range(p, r) : KeyRange{1, 0};
                nlo[m] = kr.lo;
                nhi[m] = kr.hi;
                nfull = nfull && r < p.Sq && kr.lo <= k0 && kr.hi >= k1;
            }
            nfull = __all_sync(0xffffffffu, nfull);
        };
        if (n_items > 0) prefetch(0);
        for (int it = 0; it < n_items && ok; ++it) {
            const int s = it % NSQ;
            const int g = it / n_qb;
            const int qb = qb_lo + it % n_qb;
            const int hq = hkv * p.group + g;
            float cl[4], cd[4];
            int clo[4], chi[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                cl[m] = nl[m];
                cd[m] = nd[m];
                clo[m] = nlo[m];
                chi[m] = nhi[m];
                if (qb * 128 + lane + 32 * m >= p.Sq) {
                    cl[m] = INFINITY;
                    cd[m] = 0.0f;
                }
            }
            const bool full = nfull;
            if (it + 1 < n_items) prefetch(it + 1);
            BWD_TRACE(1, it, 0);
            ok = __all_sync(0xffffffffu, wait_bounded(&sm.st_empty[s], ((it / NSQ) & 1) ^ 1,
                                                      abort_flag, p.status));
            BWD_TRACE(1, it, 1);
            if (!ok) break;
            // The tiles go first: the copy is the long pole.
            if (lane < 2) {
                // lane 0 copies the Q tile, lane 1 the dO tile, side by side
                mbar_expect_tx(&sm.st_full[s], kTileBytes);
                if (lane == 0)
                    tma_load_5d(sm.q[s][0], &p.tm_q, &sm.st_full[s], 0, qb * 128, 0, hq, b);
                else
                    tma_load_5d(sm.dout[s][0], &p.tm_do, &sm.st_full[s], 0, qb * 128, 0, hq, b);
            }
            BWD_TRACE(1, it, 3);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int idx = lane + 32 * m;
                sm.lse2[s][idx] = cl[m] * kLog2e;
                sm.dval[s][idx] = cd[m];
                sm.rlo[s][idx] = clo[m];
                sm.rhi[s][idx] = chi[m];
            }
            if (lane == 0) sm.full[s] = full ? 1 : 0;
            BWD_TRACE(1, it, 4);
            mbar_arrive(&sm.st_full[s]);  // each lane publishes its own rows
            BWD_TRACE(1, it, 2);
            ++issued;
        }
        // Copies still in flight land before the CTA can exit.
        wait_bounded(&sm.kv_full, 0, abort_flag, p.status, false);
        for (int it = issued > NSQ ? issued - NSQ : 0; it < issued; ++it)
            wait_bounded(&sm.st_full[it % NSQ], (it / NSQ) & 1, abort_flag, p.status, false);
        __syncwarp();
    } else if (warp == kBwdMmaWarp) {
        // --------------------------------------------------------- MMA issue
        if (n_items > 0) {
            const bool leader = elect_one();
            constexpr uint32_t kIdescT = idesc_bf16_f32(128, 128, 0, 0);  // S^T, dP^T
            constexpr uint32_t kIdescG = idesc_bf16_f32(128, D, 0, 1);    // dV, dK
            constexpr uint32_t kTile = Smem::kChunks * Smem::kChunkElems * 2;
            constexpr uint32_t kChunkBytes = Smem::kChunkElems * 2;
            const uint64_t k_desc = smem_desc_sw128(smem_u32(&sm.k[0][0]), 16, 1024);
            const uint64_t v_desc = smem_desc_sw128(smem_u32(&sm.v[0][0]), 16, 1024);
            const uint64_t q_kdesc = smem_desc_sw128(smem_u32(&sm.q[0][0][0]), 16, 1024);
            const uint64_t do_kdesc = smem_desc_sw128(smem_u32(&sm.dout[0][0][0]), 16, 1024);
            const uint64_t q_mdesc = smem_desc_sw128(smem_u32(&sm.q[0][0][0]), kChunkBytes, 1024);
            const uint64_t do_mdesc =
                smem_desc_sw128(smem_u32(&sm.dout[0][0][0]), kChunkBytes, 1024);
            bool ok = __all_sync(0xffffffffu, wait_bounded(&sm.kv_full, 0, abort_flag, p.status));
            auto wait_stage = [&](int it) {
                if (ok)
                    ok = __all_sync(0xffffffffu, wait_bounded(&sm.st_full[it % NSQ],
                                                              (it / NSQ) & 1, abort_flag,
                                                              p.status));
                tc_fence_after();
            };
            // X^T = A X^T for A in {K, V} (keys in lanes), X in {Q, dO} of stage s.
            auto issue_t = [&](uint64_t a_desc, uint64_t x_desc, int s, uint32_t col,
                               uint64_t *bar) {
                const uint64_t xb = x_desc + ((s * kTile) >> 4);
                if (leader) {
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t off = ((ks >> 2) * kChunkBytes + (ks & 3) * 32) >> 4;
                        mma_ss(tmem + col, a_desc + off, xb + off, kIdescT, ks > 0 ? 1u : 0u);
                    }
                    tc_commit(bar);
                }
                __syncwarp();
            };
            // G += A_tmem Y, A = P^T or dS^T (bf16 in TMEM, keys in lanes, 128
            // rows along K), Y = dO or Q of stage s read MN-major.
            auto issue_g = [&](uint32_t a_col, uint64_t y_desc, int s, uint32_t col, bool first) {
                const uint64_t yb = y_desc + ((s * kTile) >> 4);
                if (leader) {
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_ts(tmem + col, tmem + half_operand_col(a_col, ks),
                               yb + ((ks * 16 * 128) >> 4), kIdescG,
                               (!first || ks > 0) ? 1u : 0u);
                }
                __syncwarp();
            };
            wait_stage(0);
            if (ok) {
                issue_t(k_desc, q_kdesc, 0, kColS, &sm.s_full);
                issue_t(v_desc, do_kdesc, 0, kColDP, &sm.dp_full);
            }
            for (int it = 0; it < n_items && ok; ++it) {
                const int s = it % NSQ;
                BWD_TRACE(2, it, 0);
                ok = __all_sync(0xffffffffu, wait_bounded(&sm.p_ready, it & 1, abort_flag,
                                                          p.status));
                BWD_TRACE(2, it, 1);
                if (!ok) break;
                tc_fence_after();
                issue_g(kColS, do_mdesc, s, kColDV, it == 0);
                BWD_TRACE(2, it, 2);
                if (it + 1 < n_items) {
                    wait_stage(it + 1);
                    BWD_TRACE(2, it, 3);
                    if (!ok) break;
                    issue_t(k_desc, q_kdesc, (it + 1) % NSQ, kColS, &sm.s_full);
                }
                BWD_TRACE(2, it, 4);
                ok = __all_sync(0xffffffffu, wait_bounded(&sm.ds_ready, it & 1, abort_flag,
                                                          p.status));
                BWD_TRACE(2, it, 5);
                if (!ok) break;
                tc_fence_after();
                issue_g(kColDP, q_mdesc, s, kColDK, it == 0);
                BWD_TRACE(2, it, 6);
                if (leader) tc_commit(&sm.st_empty[s]);
                __syncwarp();
                if (it + 1 < n_items) issue_t(v_desc, do_kdesc, (it + 1) % NSQ, kColDP, &sm.dp_full);
            }
            if (ok) {
                if (leader) tc_commit(&sm.final_bar);
                __syncwarp();
            } else {
                if (leader) tc_commit(&sm.drain);
                __syncwarp();
                wait_bounded(&sm.drain, 0, abort_flag, p.status, false);
            }
        }
    } else {
        // ---------------------------------------------------- elementwise
        const int key = k0 + (warp & 3) * 32 + lane;
        const int h = warp >> 2;  // this warpgroup's half of the columns
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t s_col = tmem + lane_base + kColS + h * 64;
        const uint32_t dp_col = tmem + lane_base + kColDP + h * 64;
        const float c = p.scale_log2;
        bool ok = true;
        for (int it = 0; it < n_items; ++it) {
            const int s = it % NSQ;
            if (warp == 0) BWD_TRACE(0, it, 0);
            ok = __all_sync(0xffffffffu, wait_bounded(&sm.s_full, it & 1, abort_flag, p.status));
            if (!ok) break;
            tc_fence_after();
            if (warp == 0) BWD_TRACE(0, it, 1);
            uint32_t sr[64];
            tmem_ld32(s_col, sr);
            tmem_ld32(s_col + 32, sr + 32);
            tmem_wait_ld();
            reg_fence32(sr);
            reg_fence32(sr + 32);
            float *pv = reinterpret_cast<float *>(sr);  // S^T half row, then P^T
            const bool full = sm.full[s] != 0;
            const float4 *l4 = reinterpret_cast<const float4 *>(sm.lse2[s] + h * 64);
            uint32_t pk[32];
            if (MOD) {
                // Modified scores: P from the transformed score; pv keeps
                // P * d(modified)/d(scaled) for dS, pk the plain P for dV.
                const int qb = qb_lo + it % n_qb;
                const int hq = hkv * p.group + it / n_qb;
                const float slope2 = (MOD & 2) ? __ldg(p.alibi_slopes + hq) * kLog2e : 0.0f;
                const float dist0 = (float)(qb * 128 + h * 64 + p.Sk - p.Sq - key);
                const int *rlo = sm.rlo[s] + h * 64;
                const int *rhi = sm.rhi[s] + h * 64;
                const float *l2 = sm.lse2[s] + h * 64;
                const float k1 = p.softcap_in * (2.0f * kLog2e);
#pragma unroll
                for (int e = 0; e < 64; e += 2) {
                    float x0, x1, f0, f1;
                    bwd_modified_pair<MOD>(x0, x1, f0, f1, pv[e], pv[e + 1], c, k1,
                                           p.softcap_out, slope2, dist0 + (float)e,
                                           dist0 + (float)(e + 1));
                    add2(x0, x1, x0, x1, -l2[e], -l2[e + 1]);
                    const float p0 = ex2_mufu(x0), p1 = ex2_mufu(x1);
                    const float pr0 = (full || (rlo[e] <= key && key <= rhi[e])) ? p0 : 0.0f;
                    const float pr1 = (full || (rlo[e + 1] <= key && key <= rhi[e + 1])) ? p1 : 0.0f;
                    mul2(pv[e], pv[e + 1], pr0, pr1, f0, f1);
                    pk[e >> 1] = pack_bf16x2(pr0, pr1);
                }
            } else if (full) {
#pragma unroll
                for (int e = 0; e < 64; e += 4) {
                    const float4 l = l4[e >> 2];
                    float x0, x1, x2, x3;
                    fma2(x0, x1, pv[e + 0], pv[e + 1], c, c, -l.x, -l.y);
                    fma2(x2, x3, pv[e + 2], pv[e + 3], c, c, -l.z, -l.w);
                    bwd_ex2_pair(pv[e + 0], pv[e + 1], x0, x1, e + 0);
                    bwd_ex2_pair(pv[e + 2], pv[e + 3], x2, x3, e + 2);
                    pk[(e >> 1) + 0] = pack_bf16x2(pv[e + 0], pv[e + 1]);
                    pk[(e >> 1) + 1] = pack_bf16x2(pv[e + 2], pv[e + 3]);
                }
            } else {
                const int4 *lo4 = reinterpret_cast<const int4 *>(sm.rlo[s] + h * 64);
                const int4 *hi4 = reinterpret_cast<const int4 *>(sm.rhi[s] + h * 64);
#pragma unroll
                for (int e = 0; e < 64; e += 4) {
                    const float4 l = l4[e >> 2];
                    const int4 lo = lo4[e >> 2];
                    const int4 hi = hi4[e >> 2];
                    pv[e + 0] = (lo.x <= key && key <= hi.x) ? ex2_mufu(fmaf(pv[e + 0], c, -l.x)) : 0.0f;
                    pv[e + 1] = (lo.y <= key && key <= hi.y) ? ex2_mufu(fmaf(pv[e + 1], c, -l.y)) : 0.0f;
                    pv[e + 2] = (lo.z <= key && key <= hi.z) ? ex2_mufu(fmaf(pv[e + 2], c, -l.z)) : 0.0f;
                    pv[e + 3] = (lo.w <= key && key <= hi.w) ? ex2_mufu(fmaf(pv[e + 3], c, -l.w)) : 0.0f;
                    pk[(e >> 1) + 0] = pack_bf16x2(pv[e + 0], pv[e + 1]);
                    pk[(e >> 1) + 1] = pack_bf16x2(pv[e + 2], pv[e + 3]);
                }
            }
            __syncwarp();  // tcgen05.st is warp-collective
            tmem_st32(s_col, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.p_ready);
            if (warp == 0) BWD_TRACE(0, it, 2);

            // dS^T = P^T (dP^T - D) for this key against this half's rows.
            ok = __all_sync(0xffffffffu, wait_bounded(&sm.dp_full, it & 1, abort_flag, p.status));
            if (!ok) break;
            tc_fence_after();
            if (warp == 0) BWD_TRACE(0, it, 3);
            uint32_t dr[64];
            tmem_ld32(dp_col, dr);
            tmem_ld32(dp_col + 32, dr + 32);
            tmem_wait_ld();
            reg_fence32(dr);
            reg_fence32(dr + 32);
            const float4 *d4 = reinterpret_cast<const float4 *>(sm.dval[s] + h * 64);
#pragma unroll
            for (int e = 0; e < 64; e += 4) {
                const float4 dd = d4[e >> 2];
                float a0, a1, a2, a3, g0, g1, g2, g3;
                add2(a0, a1, __uint_as_float(dr[e + 0]), __uint_as_float(dr[e + 1]), -dd.x, -dd.y);
                add2(a2, a3, __uint_as_float(dr[e + 2]), __uint_as_float(dr[e + 3]), -dd.z, -dd.w);
                mul2(g0, g1, pv[e + 0], pv[e + 1], a0, a1);
                mul2(g2, g3, pv[e + 2], pv[e + 3], a2, a3);
                pk[(e >> 1) + 0] = pack_bf16x2(g0, g1);
                pk[(e >> 1) + 1] = pack_bf16x2(g2, g3);
            }
            __syncwarp();
            tmem_st32(dp_col, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.ds_ready);
            if (warp == 0) BWD_TRACE(0, it, 4);
        }
        // ------------------------------------------------------- epilogue
        if (ok && n_items > 0) {
            ok = __all_sync(0xffffffffu, wait_bounded(&sm.final_bar, 0, abort_flag, p.status));
            tc_fence_after();
        }
        if (ok) {
            const bool key_ok = key < p.Sk;
            const size_t base = (((size_t)b * p.Sk + key) * p.Hkv + hkv) * (size_t)D + h * (D / 2);
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const uint32_t col = (which == 0 ? kColDK : kColDV) + h * (D / 2);
                const float mul = which == 0 ? p.scale : 1.0f;
                __nv_bfloat16 *dst_row = (which == 0 ? p.dk : p.dv) + base;
#pragma unroll
                for (int ch = 0; ch < D / 64; ++ch) {
                    uint32_t r[32];
                    if (n_items > 0) {
                        tmem_ld32(tmem + lane_base + col + ch * 32, r);
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
                        w[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * mul,
                                           __uint_as_float(r[2 * e + 1]) * mul);
                    if (key_ok) {
                        uint4 *dst = reinterpret_cast<uint4 *>(dst_row + ch * 32);
#pragma unroll
                        for (int e = 0; e < 4; ++e) dst[e] = out[e];
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kBwdMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// --------------------------------------------------------------------- dQ

// K and V have rings of their own: K of a block is read twice (by S and,
// after the block's dS, by dQ) while V is read once (by dP), so in one shared
// ring the next K would wait for the dQ of the block before last.
template <int D, int NK, int NV>
struct DqSmem {
    static constexpr int kChunks = D / 64;
    static constexpr int kChunkElems = 128 * 64;
    __nv_bfloat16 q[kChunks][kChunkElems];
    __nv_bfloat16 dout[kChunks][kChunkElems];
    __nv_bfloat16 k[NK][kChunks][kChunkElems];
    __nv_bfloat16 v[NV][kChunks][kChunkElems];
    uint64_t q_full;
    uint64_t k_full[NK], k_empty[NK];
    uint64_t v_full[NV], v_empty[NV];
    uint64_t s_full, dp_free, ds_ready, final_bar, drain;
    uint32_t tmem_base;
    int abort_flag;
    int range[2];
    float dpart[2][128];  // D_i of each row, per half of the columns
};

template <int D, int NK, int NV, int MOD = 0>
__global__ void __launch_bounds__(kBwdThreads, 1)
attn_bwd_dq_kernel(const __grid_constant__ BwdParams p) {
    using Smem = DqSmem<D, NK, NV>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_off = smem_u32(smem_raw);
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw + ((1024u - (raw_off & 1023u)) & 1023u));
    const int warp = warp_id();
    const int lane = lane_id();

    // Heaviest query blocks first (causal load balance), then (batch, head).
    const int bh_count = p.Hq * p.B;
    const int qb = p.num_qb - 1 - (int)(blockIdx.x / bh_count);
    const int bh = (int)(blockIdx.x % bh_count);
    const int hq = bh % p.Hq;
    const int b = bh / p.Hq;
    const int hkv = hq / p.group;
    const int q0 = qb * 128;
    constexpr uint32_t kTileBytes = 128 * D * 2;

    if (threadIdx.x == 0) {
        mbar_init(&sm.q_full, 1);
        for (int s = 0; s < NK; ++s) {
            mbar_init(&sm.k_full[s], 1);
            mbar_init(&sm.k_empty[s], 1);
        }
        for (int s = 0; s < NV; ++s) {
            mbar_init(&sm.v_full[s], 1);
            mbar_init(&sm.v_empty[s], 1);
        }
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.dp_free, 256);
        mbar_init(&sm.ds_ready, 256);
        mbar_init(&sm.final_bar, 1);
        mbar_init(&sm.drain, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kBwdLoadWarp) {
        const KeyRange kr = tile_key_range(p, q0, min(q0 + 127, p.Sq - 1), lane);
        if (lane == 0) {
            sm.range[0] = kr.lo > kr.hi ? 1 : kr.lo / 128;
            sm.range[1] = kr.lo > kr.hi ? 0 : kr.hi / 128;
        }
    }
    if (warp == kBwdMmaWarp) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem = sm.tmem_base;
    volatile int *abort_flag = &sm.abort_flag;
    const int lo_b = sm.range[0], hi_b = sm.range[1];
    const int n_blocks = hi_b >= lo_b ? hi_b - lo_b + 1 : 0;
    // TMEM columns: S of even blocks [0,128), dP [128,256), dQ [256,256+D), S of
    // odd blocks [384,512).  dS (bf16 pairs) goes over its block's S.  The
    // second S buffer lets S and dP of the next block run on the tensor
    // cores while this block's dS is computed.
    constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 256, kColS1 = 384;

    if (warp == kBwdLoadWarp) {
        if (lane == 0) {
            prefetch_tensormap(&p.tm_q);
            prefetch_tensormap(&p.tm_do);
            prefetch_tensormap(&p.tm_k);
            prefetch_tensormap(&p.tm_v);
            mbar_arrive_expect_tx(&sm.q_full, 2 * kTileBytes);
            tma_load_5d(sm.q[0], &p.tm_q, &sm.q_full, 0, q0, 0, hq, b);
            tma_load_5d(sm.dout[0], &p.tm_do, &sm.q_full, 0, q0, 0, hq, b);
            int nk = 0, nv = 0;  // K and V copies issued
            bool ok = true;
            for (int t = 0; t < n_blocks && ok; ++t) {
                const int key0 = (lo_b + t) * 128;
                ok = wait_bounded(&sm.k_empty[t % NK], ((uint32_t)(t / NK) & 1u) ^ 1u,
                                  abort_flag, p.status);
                if (!ok) break;
                mbar_arrive_expect_tx(&sm.k_full[t % NK], kTileBytes);
                tma_load_5d(sm.k[t % NK][0], &p.tm_k, &sm.k_full[t % NK], 0, key0, 0, hkv, b);
                ++nk;
                ok = wait_bounded(&sm.v_empty[t % NV], ((uint32_t)(t / NV) & 1u) ^ 1u,
                                  abort_flag, p.status);
                if (!ok) break;
                mbar_arrive_expect_tx(&sm.v_full[t % NV], kTileBytes);
                tma_load_5d(sm.v[t % NV][0], &p.tm_v, &sm.v_full[t % NV], 0, key0, 0, hkv, b);
                ++nv;
            }
            // Copies still in flight land before the CTA can exit.
            wait_bounded(&sm.q_full, 0, abort_flag, p.status, false);
            for (int t = nk > NK ? nk - NK : 0; t < nk; ++t)
                wait_bounded(&sm.k_full[t % NK], (uint32_t)(t / NK) & 1u, abort_flag, p.status, false);
            for (int t = nv > NV ? nv - NV : 0; t < nv; ++t)
                wait_bounded(&sm.v_full[t % NV], (uint32_t)(t / NV) & 1u, abort_flag, p.status, false);
        }
        __syncwarp();
    } else if (warp == kBwdMmaWarp) {
        if (n_blocks > 0) {
            const bool leader = elect_one();
            constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, 0, 0);
            constexpr uint32_t kIdescQ = idesc_bf16_f32(128, D, 0, 1);
            constexpr uint32_t kTile = Smem::kChunks * Smem::kChunkElems * 2;
            constexpr uint32_t kChunkBytes = Smem::kChunkElems * 2;
            const uint64_t q_desc = smem_desc_sw128(smem_u32(&sm.q[0][0]), 16, 1024);
            const uint64_t do_desc = smem_desc_sw128(smem_u32(&sm.dout[0][0]), 16, 1024);
            const uint64_t k_kdesc = smem_desc_sw128(smem_u32(&sm.k[0][0][0]), 16, 1024);
            const uint64_t k_mdesc = smem_desc_sw128(smem_u32(&sm.k[0][0][0]), kChunkBytes, 1024);
            const uint64_t v_kdesc = smem_desc_sw128(smem_u32(&sm.v[0][0][0]), 16, 1024);
            bool ok = __all_sync(0xffffffffu, wait_bounded(&sm.q_full, 0, abort_flag, p.status));
            tc_fence_after();
            auto wait_full = [&](uint64_t *bar, uint32_t parity) {
                if (ok)
                    ok = __all_sync(0xffffffffu, wait_bounded(bar, parity, abort_flag, p.status));
                tc_fence_after();
            };
            // S of block t into its buffer (needs K), then dP (needs V); one
            // commit signals both.
            auto issue_s = [&](int t) {
                wait_full(&sm.k_full[t % NK], (uint32_t)(t / NK) & 1u);
                if (!ok) return;
                const uint64_t kb_k = k_kdesc + (((uint32_t)(t % NK) * kTile) >> 4);
                const uint32_t col = (t & 1) ? kColS1 : kColS;
                if (leader) {
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t off = ((ks >> 2) * kChunkBytes + (ks & 3) * 32) >> 4;
                        mma_ss(tmem + col, q_desc + off, kb_k + off, kIdescS, ks > 0 ? 1u : 0u);
                    }
                }
                __syncwarp();
            };
            auto issue_dp = [&](int t) {
                wait_full(&sm.v_full[t % NV], (uint32_t)(t / NV) & 1u);
                if (!ok) return;
                const uint64_t vb_k = v_kdesc + (((uint32_t)(t % NV) * kTile) >> 4);
                if (leader) {
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t off = ((ks >> 2) * kChunkBytes + (ks & 3) * 32) >> 4;
                        mma_ss(tmem + kColDP, do_desc + off, vb_k + off, kIdescS,
                               ks > 0 ? 1u : 0u);
                    }
                    tc_commit(&sm.s_full);
                    tc_commit(&sm.v_empty[t % NV]);  // V of this block is consumed
                }
                __syncwarp();
            };
            issue_s(0);
            issue_dp(0);
            for (int t = 0; t < n_blocks && ok; ++t) {
                if (t + 1 < n_blocks) {
                    issue_s(t + 1);  // other S buffer: its last reader (dQ of t-1) is queued
                    if (!ok) break;
                    ok = __all_sync(0xffffffffu, wait_bounded(&sm.dp_free, (uint32_t)t & 1u,
                                                              abort_flag, p.status));
                    if (!ok) break;
                    tc_fence_after();
                    issue_dp(t + 1);
                    if (!ok) break;
                }
                ok = __all_sync(0xffffffffu, wait_bounded(&sm.ds_ready, (uint32_t)t & 1u,
                                                          abort_flag, p.status));
                if (!ok) break;
                tc_fence_after();
                const uint64_t kb_m = k_mdesc + (((uint32_t)(t % NK) * kTile) >> 4);
                const uint32_t col = (t & 1) ? kColS1 : kColS;
                if (leader) {
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_ts(tmem + kColDQ, tmem + half_operand_col(col, ks),
                               kb_m + ((ks * 16 * 128) >> 4), kIdescQ,
                               (t > 0 || ks > 0) ? 1u : 0u);
                    tc_commit(&sm.k_empty[t % NK]);  // K of this block is consumed
                }
                __syncwarp();
            }
            if (ok) {
                if (leader) tc_commit(&sm.final_bar);
                __syncwarp();
            } else {
                if (leader) tc_commit(&sm.drain);
                __syncwarp();
                wait_bounded(&sm.drain, 0, abort_flag, p.status, false);
            }
        }
    } else {
        // ---------------------------------------------------- elementwise
        const int row_in = (warp & 3) * 32 + lane;
        const int row = q0 + row_in;
        const int h = warp >> 2;  // this warpgroup's half of the columns
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t dp_col = tmem + lane_base + kColDP + h * 64;
        const bool row_ok = row < p.Sq;
        const KeyRange kr = row_ok ? row_key_range(p, row) : KeyRange{1, 0};
        const size_t ri = ((size_t)b * p.Hq + hq) * p.Sq + (row_ok ? row : 0);
        const float l2 = row_ok ? __ldg(p.lse + ri) * kLog2e : INFINITY;
        // D_i = sum_d dO_id O_id of this row: each warpgroup over its half of
        // the columns, the halves added in a fixed order through shared
        // memory; warpgroup 0 stores it for the dK/dV kernel, which runs after
        // this one.  (The loads overlap the first S and dP products.)
        float dval;
        {
            float a0 = 0.0f, a1 = 0.0f;
            if (row_ok) {
                const size_t off = (((size_t)b * p.Sq + row) * p.Hq + hq) * (size_t)D + h * (D / 2);
                const uint4 *o4 = reinterpret_cast<const uint4 *>(p.o + off);
                const uint4 *g4 = reinterpret_cast<const uint4 *>(p.dout + off);
#pragma unroll
                for (int ch = 0; ch < D / 16; ++ch) {
                    const uint4 ov = ld_nc_v4(o4 + ch), gv = ld_nc_v4(g4 + ch);
                    const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w};
                    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        fma2(a0, a1, __uint_as_float(ow[e] << 16), __uint_as_float(ow[e] & 0xffff0000u),
                             __uint_as_float(gw[e] << 16), __uint_as_float(gw[e] & 0xffff0000u), a0, a1);
                }
            }
            sm.dpart[h][row_in] = a0 + a1;
            named_bar_sync(1, 256);  // the 256 elementwise threads, all of which reach it
            dval = sm.dpart[0][row_in] + sm.dpart[1][row_in];
            if (h == 0 && row_ok) p.dval[ri] = dval;
        }
        const float c = p.scale_log2;
        const float slope2 = (MOD & 2) ? __ldg(p.alibi_slopes + hq) * kLog2e : 0.0f;
        bool ok = true;
        for (int t = 0; t < n_blocks; ++t) {
            const int j = lo_b + t;
            ok = __all_sync(0xffffffffu, wait_bounded(&sm.s_full, (uint32_t)t & 1u, abort_flag,
                                                      p.status));
            if (!ok) break;
            tc_fence_after();
            const uint32_t s_col = tmem + lane_base + ((t & 1) ? kColS1 : kColS) + h * 64;
            uint32_t sr[64], dr[64];
            tmem_ld32(s_col, sr);
            tmem_ld32(s_col + 32, sr + 32);
            tmem_ld32(dp_col, dr);
            tmem_ld32(dp_col + 32, dr + 32);
            tmem_wait_ld();
            reg_fence32(sr);
            reg_fence32(sr + 32);
            reg_fence32(dr);
            reg_fence32(dr + 32);
            tc_fence_before();
            mbar_arrive(&sm.dp_free);  // dP of the next block may overwrite it now
            float *pv = reinterpret_cast<float *>(sr);
            const int key0 = j * 128 + h * 64;
            const bool masked = __any_sync(0xffffffffu, key0 < kr.lo || key0 + 63 > kr.hi);
            if (MOD) {
                // pv becomes P * d(modified)/d(scaled), all dS needs.
                const float dist0 = (float)(row + p.Sk - p.Sq - key0);
                const float k1 = p.softcap_in * (2.0f * kLog2e);
#pragma unroll
                for (int e = 0; e < 64; e += 2) {
                    float x0, x1, f0, f1;
                    bwd_modified_pair<MOD>(x0, x1, f0, f1, pv[e], pv[e + 1], c, k1,
                                           p.softcap_out, slope2, dist0 - (float)e,
                                           dist0 - (float)(e + 1));
                    add2(x0, x1, x0, x1, -l2, -l2);
                    float p0 = ex2_mufu(x0), p1 = ex2_mufu(x1);
                    mul2(p0, p1, p0, p1, f0, f1);
                    const int key = key0 + e;
                    pv[e] = (!masked || (key >= kr.lo && key <= kr.hi)) ? p0 : 0.0f;
                    pv[e + 1] = (!masked || (key + 1 >= kr.lo && key + 1 <= kr.hi)) ? p1 : 0.0f;
                }
            } else if (masked) {
#pragma unroll
                for (int e = 0; e < 64; ++e) {
                    const int key = key0 + e;
                    pv[e] = (key >= kr.lo && key <= kr.hi) ? ex2_mufu(fmaf(pv[e], c, -l2)) : 0.0f;
                }
            } else {
#pragma unroll
                for (int e = 0; e < 64; e += 2) {
                    float x0, x1;
                    fma2(x0, x1, pv[e], pv[e + 1], c, c, -l2, -l2);
                    bwd_ex2_pair(pv[e], pv[e + 1], x0, x1, e);
                }
            }
            uint32_t pk[32];
#pragma unroll
            for (int e = 0; e < 64; e += 2) {
                float a0, a1, g0, g1;
                add2(a0, a1, __uint_as_float(dr[e]), __uint_as_float(dr[e + 1]), -dval, -dval);
                mul2(g0, g1, pv[e], pv[e + 1], a0, a1);
                pk[e / 2] = pack_bf16x2(g0, g1);
            }
            __syncwarp();
            tmem_st32(s_col, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.ds_ready);
        }
        if (ok && n_blocks > 0) {
            ok = __all_sync(0xffffffffu, wait_bounded(&sm.final_bar, 0, abort_flag, p.status));
            tc_fence_after();
        }
        if (ok) {
            float *dst_row = p.dq + (((size_t)b * p.Sq + row) * p.Hq + hq) * (size_t)D + h * (D / 2);
#pragma unroll
            for (int ch = 0; ch < D / 64; ++ch) {
                uint32_t r[32];
                if (n_blocks > 0) {
                    tmem_ld32(tmem + lane_base + kColDQ + h * (D / 2) + ch * 32, r);
                    tmem_wait_ld();
                    reg_fence32(r);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) r[e] = 0u;
                }
                if (row_ok) {
                    float4 *dst = reinterpret_cast<float4 *>(dst_row + ch * 32);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        dst[e] = make_float4(__uint_as_float(r[4 * e]) * p.scale,
                                             __uint_as_float(r[4 * e + 1]) * p.scale,
                                             __uint_as_float(r[4 * e + 2]) * p.scale,
                                             __uint_as_float(r[4 * e + 3]) * p.scale);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kBwdMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace tab
