// Persistent variant of the attention forward (sm_100a), used by the fp8
// forward.
//
// The per-key-block work is that of attn_fwd_kernel (fwd_kernel.cuh: the
// same roles, barriers and softmax), but one CTA per SM runs many work
// items back to back: the producer publishes each item's key-block ranges
// in a two-slot ring of shared memory, loads the next item's Q as soon as
// the last QK^T of an item has completed (q_free), and keeps loading K/V
// into the same ring; the MMA warp issues the next item's first QK^T while
// the softmax warps still store the previous item's output, and that
// item's first PV waits only until the epilogue has read O from tensor
// memory (o_free).  Every barrier phase carries over from item to item.
// This hides the fixed cost of an item -- the Q and first K/V latency, the
// pipeline fill and the epilogue -- behind the neighbouring items' work:
// the overlap of the result-storage stage with the next tile's pipeline
// ("FlashAttention-4 de NVIDIA", "La ventaja técnica"; "Hardware-Aware FP4
// FlashAttention-4", "Contribuciones Clave": overlapping the next tile's
// products with the current tile's tail).
//
// Measured on B200 (causal S=8192): 6 % faster than attn_fwd_kernel for
// e4m3 operands, but 11 % slower for bf16 operands, where the same
// structure raises the long-scoreboard and instruction-fetch stalls per
// issued instruction; the bf16, f16 and Direct-P forwards therefore keep
// the one-item-per-CTA kernel.
#pragma once

#include "fwd_kernel.cuh"

namespace tab {

// A work item: one (batch, query head) and its pair of 128-row query tiles,
// with each tile's first and last key block (lo > hi: no key).  lin < 0
// marks the end of a CTA's items.
struct FwdItem {
    int lin;
    int lo[2], hi[2];
};

// Work items are linearised in groups of `head_group` (batch, head) pairs;
// inside a group the heaviest query-tile pairs come first (causal load
// balance) and consecutive items cycle through the group's heads, so the
// items resident at one time share a few heads' K/V in L2.
struct ItemCoords {
    int b, hq, qb;
};
template <class Params>
__device__ __forceinline__ ItemCoords item_coords(const Params &p, int lin) {
    const int bh_count = p.Hq * p.B;
    const int G = p.head_group;
    const int nq = p.num_qblocks;
    const int full_groups = bh_count / G;
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
    const int bh = grp * G + r % ge;
    return {bh / p.Hq, bh % p.Hq, nq - 1 - r / ge};
}

// Persistent schedule: each CTA runs many items.  The items of a group are
// dealt to the CTAs in rounds of gridDim.x, round r left to right when r is
// even and right to left when odd (a snake, so a CTA that took a heavy item
// in one round takes a light one in the next); the dealing position carries
// over from one group to the next.  Every role of a CTA walks the same
// sequence with its own cursor.  Returns the next item's linear index, or -1.
struct ItemCursor {
    int g = 0, rnd = 0;
};
template <class Params>
__device__ __forceinline__ int next_item(const Params &p, ItemCursor &cur) {
    const int G = (int)gridDim.x, c = (int)blockIdx.x;
    const int per_group = p.head_group * p.num_qblocks;
    const int total = p.B * p.Hq * p.num_qblocks;
    for (;;) {
        const int g0 = cur.g * per_group;
        if (g0 >= total) return -1;
        const int n_g = min(per_group, total - g0);
        if (cur.rnd * G >= n_g) {
            ++cur.g;
            cur.rnd = 0;
            continue;
        }
        const int pos = (cur.rnd & 1) ? G - 1 - c : c;
        const int slot = (pos - g0 % G + G) % G;
        const int r = cur.rnd * G + slot;
        ++cur.rnd;
        if (r < n_g) return g0 + r;
    }
}

// EB: bytes per element of Q, K, V (2 = bf16, 1 = fp8 e4m3).  A tile row of
// D elements is D*EB bytes, stored as chunks of 128-byte rows.
template <int D, int NS, int EB = 2>
struct FwdSmemPersistent {
    static constexpr int kChunkBytes = kBlockM * 128;  // 16 KB: 128 rows x 128 bytes
    static constexpr int kChunks = D * EB / 128;
    static constexpr int kChunkElems = 128 / EB;       // elements per 128-byte row
    uint8_t q[2][kChunks][kChunkBytes];
    uint8_t kv[NS][kChunks][kChunkBytes];
    uint64_t q_full;
    uint64_t q_free;     // every QK^T of the item has completed: Q may be replaced
    uint64_t kv_full[NS];
    uint64_t kv_empty[NS];
    uint64_t s_full[2];
    uint64_t p_half[2];  // P of keys [0, 64) of the block is in TMEM
    uint64_t p_full[2];  // all of P (and any O correction) is in TMEM
    uint64_t o_final[2];  // the item's last PV of a tile has completed
    uint64_t o_free[2];   // the epilogue has read O of a tile: the next item may overwrite it
    uint64_t item_full[2];
    uint64_t item_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    FwdItem item[2];  // ring of the next work items and their key-block ranges
};

template <int D, int NS, int EXP_MODE, int MOD = 0, int PREC = 0>
__global__ void __launch_bounds__(kFwdThreads, 1)
attn_fwd_persistent_kernel(const __grid_constant__ FwdParams p) {
    static_assert(!(PREC && MOD), "the low-precision paths have no score modifiers");
    constexpr bool FP8 = PREC == 1;
    constexpr bool DP = PREC >= 2;  // Direct-P
    constexpr int EB = FP8 ? 1 : 2;
    using Smem = FwdSmemPersistent<D, NS, EB>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_off = smem_u32(smem_raw);
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw + ((1024u - (raw_off & 1023u)) & 1023u));

    const int warp = warp_id();
    const int lane = lane_id();

    // ------------------------------------------------------------ prologue
    // Once per CTA: barriers and the tensor-memory allocation.  The CTA then
    // runs its items back to back; every barrier's phase carries over from
    // one item to the next (each role counts its own completions).
    if (threadIdx.x == 0) {
        mbar_init(&sm.q_full, 1);
        mbar_init(&sm.q_free, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&sm.kv_full[s], 1);
            mbar_init(&sm.kv_empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.s_full[i], 1);
            mbar_init(&sm.p_half[i], kBlockM);
            mbar_init(&sm.p_full[i], kBlockM);
            mbar_init(&sm.o_final[i], 1);
            mbar_init(&sm.o_free[i], kBlockM);
            mbar_init(&sm.item_full[i], 1);
            mbar_init(&sm.item_empty[i], 1 + 8);  // the MMA warp and the 8 softmax warps
        }
        mbar_init(&sm.drain, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
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
    constexpr uint32_t kTileBytes = kBlockM * D * EB;

    // Consumers read the next item from the ring and release its slot; an
    // item with lin = -2 stands for a wait that gave up (abort).
    auto take_item = [&](uint32_t n) -> FwdItem {
        const uint32_t slot = n & 1u;
        FwdItem it;
        it.lin = -2;
        if (!__all_sync(0xffffffffu, wait_bounded<true>(&sm.item_full[slot], (n >> 1) & 1u, abort_flag,
                                                  p.status, true, p.timeout_ns)))
            return it;
        const volatile FwdItem &src = sm.item[slot];
        it.lin = src.lin;
        it.lo[0] = src.lo[0];
        it.lo[1] = src.lo[1];
        it.hi[0] = src.hi[0];
        it.hi[1] = src.hi[1];
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.item_empty[slot]);
        return it;
    };

    // Registers: the softmax warpgroups hold a 128-column score row per
    // thread; the MMA / TMA warpgroup needs few.  384 x 168 at launch =
    // 2 x 128 x kSoftmaxRegs + 128 x kOtherRegs.  All four warps of a
    // warpgroup execute the same setmaxnreg instruction, and each budget
    // dominates the code of its roles so the compiler allocates per role.
    if (warp >= 8) {
        setmaxnreg_dec<kOtherRegs>();
        if (warp == 9) {
            // ------------------------------------------------------ TMA producer
            // Per item: its key-block ranges (union of the rows' key ranges
            // of each query tile) into the item ring, then Q once the previous
            // item's QK^T products are done, then the K/V blocks into the ring.
            if (lane == 0) {
                prefetch_tensormap(&p.tm_q);
                prefetch_tensormap(&p.tm_k);
                prefetch_tensormap(&p.tm_v);
            }
            ItemCursor cur;
            uint32_t it = 0;      // K/V ring position (running over items)
            uint32_t q_loads = 0;
            bool ok = true;
            // Descriptor of item n: linear index, coordinates and each tile's
            // key-block range (union of its rows' key ranges), computed by the
            // whole warp.
            auto describe = [&](FwdItem &d, ItemCoords &ic) {
                d.lin = next_item(p, cur);
                d.lo[0] = d.lo[1] = 1;
                d.hi[0] = d.hi[1] = 0;
                ic = ItemCoords{0, 0, 0};
                if (d.lin < 0) return;
                ic = item_coords(p, d.lin);
                const int q0 = ic.qb * 2 * kBlockM;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int r0 = q0 + i * kBlockM;
                    KeyRange kr{1, 0};
                    if (r0 < p.Sq) kr = tile_key_range(p, r0, min(r0 + kBlockM - 1, p.Sq - 1), lane);
                    d.lo[i] = kr.lo > kr.hi ? 1 : kr.lo / kBlockN;
                    d.hi[i] = kr.lo > kr.hi ? 0 : kr.hi / kBlockN;
                }
            };
            // Publish item n in ring slot n & 1 (its previous user, item n - 2,
            // must have been taken by every consumer).
            auto publish = [&](uint32_t n, const FwdItem &d) {
                const uint32_t slot = n & 1u;
                if (n >= 2)
                    ok = __all_sync(0xffffffffu,
                                    wait_bounded<true>(&sm.item_empty[slot], ((n >> 1) - 1u) & 1u,
                                                 abort_flag, p.status, true, p.timeout_ns));
                if (!ok) return;
                if (lane == 0) {
                    volatile FwdItem &dst = sm.item[slot];
                    dst.lin = d.lin;
                    dst.lo[0] = d.lo[0];
                    dst.lo[1] = d.lo[1];
                    dst.hi[0] = d.hi[0];
                    dst.hi[1] = d.hi[1];
                    mbar_arrive(&sm.item_full[slot]);
                }
                __syncwarp();
            };
            FwdItem itm;
            ItemCoords ic;
            describe(itm, ic);
            publish(0, itm);
            for (uint32_t n = 0; ok && itm.lin >= 0; ++n) {
                // The next item is published before this item's loads, so the
                // consumers find it ready when they finish this one.
                FwdItem nxt;
                ItemCoords nic;
                describe(nxt, nic);
                publish(n + 1, nxt);
                if (!ok) break;
                const bool has0 = itm.lo[0] <= itm.hi[0], has1 = itm.lo[1] <= itm.hi[1];
                if (has0 || has1) {
                    const int ulo = has0 ? (has1 ? min(itm.lo[0], itm.lo[1]) : itm.lo[0]) : itm.lo[1];
                    const int uhi = has0 ? (has1 ? max(itm.hi[0], itm.hi[1]) : itm.hi[0]) : itm.hi[1];
                    const int hkv = ic.hq / p.group;
                    if (lane == 0) {
                        if (q_loads > 0)
                            ok = wait_bounded<true>(&sm.q_free, (q_loads - 1u) & 1u, abort_flag, p.status,
                                              true, p.timeout_ns);
                        if (ok) {
                            mbar_arrive_expect_tx(&sm.q_full, 2 * kTileBytes);
                            for (int i = 0; i < 2; ++i)
                                for (int c = 0; c < Smem::kChunks; ++c)
                                    tma_load_4d(sm.q[i][c], &p.tm_q, &sm.q_full, c * Smem::kChunkElems,
                                                ic.qb * 2 * kBlockM + i * kBlockM, ic.hq, ic.b);
                        }
                        for (int t = 0; t < uhi - ulo + 1 && ok; ++t) {
                            const int key0 = (ulo + t) * kBlockN;
                            for (int which = 0; which < 2 && ok; ++which, ++it) {
                                const uint32_t kslot = it % NS;
                                ok = wait_bounded<true>(&sm.kv_empty[kslot], ((it / NS) & 1u) ^ 1u,
                                                  abort_flag, p.status, true, p.timeout_ns);
                                if (!ok) break;
                                // Testing only: the first CTA withholds its first K copy
                                // (the loop increment still advances the ring position).
                                if (p.debug_withhold_kv && blockIdx.x == 0 && it == 0) continue;
                                mbar_arrive_expect_tx(&sm.kv_full[kslot], kTileBytes);
                                const CUtensorMap *map = which ? &p.tm_v : &p.tm_k;
                                for (int c = 0; c < Smem::kChunks; ++c)
                                    tma_load_4d(sm.kv[kslot][c], map, &sm.kv_full[kslot],
                                                c * Smem::kChunkElems, key0, hkv, ic.b);
                            }
                        }
                    }
                    ++q_loads;
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                }
                itm = nxt;
                ic = nic;
            }
            // Every copy still in flight lands before the CTA can exit (only
            // the last Q and the last NS K/V loads can be outstanding; on the
            // normal path they have been consumed already).
            if (lane == 0) {
                if (q_loads > 0)
                    wait_bounded<true>(&sm.q_full, (q_loads - 1u) & 1u, abort_flag, p.status, false,
                                 p.timeout_ns);
                const uint32_t first = it > NS ? it - NS : 0;
                for (uint32_t L = first; L < it; ++L)
                    wait_bounded<true>(&sm.kv_full[L % NS], (L / NS) & 1u, abort_flag, p.status, false,
                                 p.timeout_ns);
            }
            __syncwarp();
        } else if (warp == 8) {
            // --------------------------------------------------- MMA issuer
            // The whole warp runs the schedule, so control flow and descriptor
            // arithmetic stay warp-uniform; one elected lane issues the
            // tcgen05 instructions (and the commits that track them).
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
            const uint64_t v_desc = smem_desc_sw128(smem_u32(&sm.kv[0][0][0]), kChunkBytes, 1024);
            uint32_t kv_base = 0;       // ring position of this item's first K block
            uint32_t q_items = 0;       // items with key blocks (Q loads) so far
            uint32_t blocks_done0 = 0u, blocks_done1 = 0u;  // key blocks of each tile in earlier items
            uint32_t o_items0 = 0u, o_items1 = 0u;          // earlier items in which a tile had blocks
            bool ok = true;
            for (uint32_t n = 0; ok; ++n) {
                const FwdItem itm = take_item(n);
                if (itm.lin == -2) ok = false;
                if (itm.lin < 0) break;
                const int lo0 = itm.lo[0], hi0 = itm.hi[0], lo1 = itm.lo[1], hi1 = itm.hi[1];
                const bool has0 = lo0 <= hi0, has1 = lo1 <= hi1;
                if (!has0 && !has1) continue;
                const int ulo = has0 ? (has1 ? min(lo0, lo1) : lo0) : lo1;
                const int uhi = has0 ? (has1 ? max(hi0, hi1) : hi0) : hi1;
                ok = __all_sync(0xffffffffu, wait_bounded<true>(&sm.q_full, q_items & 1u, abort_flag,
                                                          p.status, true, p.timeout_ns));
                if (!ok) break;
                tc_fence_after();
                int k_ready = ulo - 1;  // last key block whose K slot was waited on
                auto ring_pos = [&](int j, int which) -> uint32_t {
                    return kv_base + 2u * (uint32_t)(j - ulo) + (uint32_t)which;
                };
                auto wait_k = [&](int j) {
                    const uint32_t L = ring_pos(j, 0);
                    if (ok)
                        ok = __all_sync(0xffffffffu, wait_bounded<true>(&sm.kv_full[L % NS],
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
                    return i == 0 ? (has0 && j >= lo0 && j <= hi0) : (has1 && j >= lo1 && j <= hi1);
                };

                for (int i = 0; i < 2; ++i)
                    if (active(i, ulo)) issue_s(i, ulo);
                if (ok && k_ready < ulo) wait_k(ulo);
                if (ok && leader) {
                    tc_commit(&sm.kv_empty[ring_pos(ulo, 0) % NS]);
                    if (ulo == uhi) tc_commit(&sm.q_free);  // no further QK^T in this item
                }
                __syncwarp();
                // The item's first PV of a tile overwrites O: the epilogue of the
                // tile's previous item must have read it.  (The first QK^T
                // products above write S only, so they do not wait for this.)
                if (ok && has0 && o_items0 > 0)
                    ok = __all_sync(0xffffffffu, wait_bounded<true>(&sm.o_free[0], (o_items0 - 1u) & 1u,
                                                              abort_flag, p.status, true, p.timeout_ns));
                if (ok && has1 && o_items1 > 0)
                    ok = __all_sync(0xffffffffu, wait_bounded<true>(&sm.o_free[1], (o_items1 - 1u) & 1u,
                                                              abort_flag, p.status, true, p.timeout_ns));
                tc_fence_after();

                for (int j = ulo; j <= uhi && ok; ++j) {
                    const uint32_t Lv = ring_pos(j, 1);
                    const uint32_t vslot = Lv % NS;
                    ATTN_TRACE_EVENT(2, blocks_done0 + (uint32_t)(j - ulo), 0);
                    ok = __all_sync(0xffffffffu, wait_bounded<true>(&sm.kv_full[vslot], (Lv / NS) & 1u,
                                                              abort_flag, p.status, true, p.timeout_ns));
                    ATTN_TRACE_EVENT(2, blocks_done0 + (uint32_t)(j - ulo), 1);
                    if (!ok) break;
                    tc_fence_after();
                    const uint64_t vb = v_desc + ((vslot * kQTileBytes) >> 4);
                    for (int i = 0; i < 2 && ok; ++i) {
                        if (active(i, j)) {
                            const int lo_i = i == 0 ? lo0 : lo1;
                            const int hi_i = i == 0 ? hi0 : hi1;
                            const uint32_t bd_i = i == 0 ? blocks_done0 : blocks_done1;
                            const uint32_t par = (bd_i + (uint32_t)(j - lo_i)) & 1u;
                            const uint32_t o_tmem = tmem + 2 * kBlockN + i * D;
                            const uint32_t p_tmem = tmem + i * kBlockN;
                            const uint32_t first = j > lo_i ? 1u : 0u;
                            // PV in two halves of 64 keys, each as soon as its P is in TMEM.
                            // V chunk: key rows of 128 bytes, 8-row groups 1024 B apart
                            // (SBO), 64-column chunks kChunkBytes apart (LBO).
                            ATTN_TRACE_EVENT(2, blocks_done0 + (uint32_t)(j - ulo), 2 + 3 * i);
                            ok = __all_sync(0xffffffffu, wait_bounded<true>(&sm.p_half[i], par,
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
                            ok = __all_sync(0xffffffffu, wait_bounded<true>(&sm.p_full[i], par,
                                                                      abort_flag, p.status, true, p.timeout_ns));
                            ATTN_TRACE_EVENT(2, blocks_done0 + (uint32_t)(j - ulo), 3 + 3 * i);
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
                        ATTN_TRACE_EVENT(2, blocks_done0 + (uint32_t)(j - ulo), 4 + 3 * i);
                    }
                    if (!ok) break;
                    if (j + 1 <= uhi && k_ready < j + 1) wait_k(j + 1);
                    if (!ok) break;
                    if (leader) {
                        tc_commit(&sm.kv_empty[vslot]);
                        if (j + 1 <= uhi) tc_commit(&sm.kv_empty[ring_pos(j + 1, 0) % NS]);
                        // The item's last QK^T products were issued just above.
                        if (j + 1 == uhi) tc_commit(&sm.q_free);
                    }
                    __syncwarp();
                }
                kv_base += 2u * (uint32_t)(uhi - ulo + 1);
                ++q_items;
                if (has0) {
                    blocks_done0 += (uint32_t)(hi0 - lo0 + 1);
                    ++o_items0;
                }
                if (has1) {
                    blocks_done1 += (uint32_t)(hi1 - lo1 + 1);
                    ++o_items1;
                }
            }
            if (!ok) {
                // Let every MMA already issued finish before TMEM is freed.
                if (leader) tc_commit(&sm.drain);
                __syncwarp();
                wait_bounded<true>(&sm.drain, 0, abort_flag, p.status, false, p.timeout_ns);
            }
            __syncwarp();
        }
        // warps 10-11: idle
    } else {
        // ------------------------------------- softmax / correction / epilogue
        setmaxnreg_inc<kSoftmaxRegs>();
        const int i = warp >> 2;
        const int row_in_tile = threadIdx.x & (kBlockM - 1);
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t s_tmem = tmem + lane_base + i * kBlockN;
        const uint32_t o_tmem = tmem + lane_base + 2 * kBlockN + i * D;
        const float c = p.scale_log2;
        const float tau = p.rescale_threshold;
        // With a modifier the scores are transformed into log2 units before
        // the max, so the exponent step multiplies by 1 instead of c.
        const float c_exp = MOD ? 1.0f : c;
        const float k1 = p.softcap_in * (2.0f * kLog2eF);  // soft-cap: 2 log2(e) scale / cap
        uint32_t blocks_done = 0;  // key blocks of this tile in earlier items
        uint32_t o_items = 0;      // earlier items in which this tile had blocks
        bool ok = true;
        for (uint32_t n = 0; ok; ++n) {
            const FwdItem itm = take_item(n);
            if (itm.lin == -2) ok = false;
            if (itm.lin < 0) break;
            const ItemCoords ic = item_coords(p, itm.lin);
            const int row = ic.qb * 2 * kBlockM + i * kBlockM + row_in_tile;
            const KeyRange kr = row_key_range(p, row);
            const int lo_b = i == 0 ? itm.lo[0] : itm.lo[1];
            const int hi_b = i == 0 ? itm.hi[0] : itm.hi[1];
            const float slope2 = (MOD & 2) ? __ldg(p.alibi_slopes + ic.hq) * kLog2eF : 0.0f;
            const float diag_f = (float)(row + p.Sk - p.Sq);
            float m_run = -INFINITY;
            float l_run = 0.0f;   // row sum of the unrounded p (the LSE's normaliser)
            float l_pv = 0.0f;    // row sum of the p that PV consumes (the output's normaliser)

            for (int j = lo_b; j <= hi_b; ++j) {
                const int t = j - lo_b;
                const uint32_t tg = blocks_done + (uint32_t)t;  // running block count of the tile
                if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, tg, 0);
                ok = wait_bounded<true>(&sm.s_full[i], tg & 1u, abort_flag, p.status, true, p.timeout_ns);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
                if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, tg, 1);
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
                    if (m_cand > m_run + tau) {
                        const float m_new = ceilf(m_cand);
                        alpha = exp2_neg_int(m_run - m_new);
                        m_run = m_new;
                    }
                    neg_m = m_run == -INFINITY ? 0.0f : p.p_offset - m_run;
                    if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, tg, 3);
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
                if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, tg, 2);
                const float row_max = fmax3(fmaxf(mx[0], mx[1]), mx[2], mx[3]);
                const float m_cand = MOD ? row_max : row_max * c;
                if (m_cand > m_run + tau) {
                    alpha = ex2_mufu(m_run - m_cand);
                    m_run = m_cand;
                }
                // fp8: P = 2^(x - m + p_offset) <= 2^8 keeps e4m3's range for the
                // small probabilities (the same factor scales l, so O and LSE are
                // unchanged).
                neg_m = m_run == -INFINITY ? 0.0f : (FP8 ? p.p_offset - m_run : -m_run);
                if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, tg, 3);
                }

                l_run *= alpha;
                l_pv *= alpha;

                // Correction first: rescale this row of O in TMEM (rare once the
                // max settles) before any P of this block is handed over.  PV of
                // the previous block is complete: the commit that signalled S of
                // this block covers every earlier MMA.
                if (t > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
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
                    if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, tg, 4);
                    __syncwarp();
                    tmem_st32(s_tmem + 32, pk + 32);
                } else if constexpr (FP8) {
                    l_run += masked ? exp_pack_half_fp8<0>(s + 64, c_exp, neg_m, pk + 16)
                                    : exp_pack_half_fp8<EXP_MODE>(s + 64, c_exp, neg_m, pk + 16);
                    if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, tg, 4);
                    tmem_st16(s_tmem + 16, pk + 16);
                } else {
                    if (masked) exp_pack_half<0>(s + 64, c_exp, neg_m, pk + 32, l_run, l_pv);
                    else exp_pack_half<EXP_MODE>(s + 64, c_exp, neg_m, pk + 32, l_run, l_pv);
                    if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, tg, 4);
                    tmem_st32(s_tmem + 32, pk + 32);
                }
                tmem_wait_st();
                if ((warp & 3) == 0) ATTN_TRACE_EVENT(i, tg, 5);
                tc_fence_before();
                mbar_arrive(&sm.p_full[i]);
            }
            if (!ok) break;

            // ------------------------------------------------------- epilogue
            // O of this tile is read from TMEM (then released for the next
            // item's first PV), normalised and stored; meanwhile the MMA warp
            // already runs the next item's first QK^T products.
            const bool has_blocks = lo_b <= hi_b;
            if (has_blocks) {
                // The last PV of this tile (and every MMA before it) is complete.
                ok = wait_bounded<true>(&sm.o_final[i], o_items & 1u, abort_flag, p.status, true,
                                  p.timeout_ns);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
            }
            const bool row_ok = row < p.Sq;
            // bf16 P: normalise by the sum of the rounded weights PV applied;
            // fp8 and Direct-P: by the row sum (the fp8 bound is derived for
            // it; Direct-P's sum is already over the values PV consumes).
            const float l_out = PREC ? l_run : l_pv;
            const float inv_l = l_out > 0.0f ? (PREC ? p.v_descale : 1.0f) / l_out : 0.0f;
            __nv_bfloat16 *o_row = p.o + (((size_t)ic.b * p.Sq + row) * p.Hq + ic.hq) * (size_t)D;
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t r[32];
                if (has_blocks) {
                    tmem_ld32(o_tmem + ch * 32, r);
                    tmem_wait_ld();
                    reg_fence32(r);
                    if (ch == D / 32 - 1) {
                        // O of this tile is in registers: the next item's first PV
                        // may overwrite it.
                        tc_fence_before();
                        mbar_arrive(&sm.o_free[i]);
                    }
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
            if (has_blocks) ++o_items;
            if (row_ok) {
                const float m_lse = PREC ? m_run - p.p_offset : m_run;
                const float lse = l_run > 0.0f ? (m_lse + log2f(l_run)) * 0.69314718055994531f
                                               : -INFINITY;
                p.lse[((size_t)ic.b * p.Hq + ic.hq) * p.Sq + row] = lse;
            }
            if (has_blocks) blocks_done += (uint32_t)(hi_b - lo_b + 1);
        }
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
