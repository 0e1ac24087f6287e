// Pieces shared by the forward and backward kernels: the per-row key
// interval every supported mask reduces to, and bounded mbarrier waits.
#pragma once

#include "exp2_poly.cuh"
#include "ptx.cuh"

namespace tab {

constexpr uint64_t kWaitTimeoutNs = 1000000000ull;  // 1 s per wait
constexpr int kStatusTimeout = 5;                   // ATTN_ERR_DEVICE_TIMEOUT
constexpr int kStatusRange = 7;                     // ATTN_ERR_RANGE

// Causal (bottom-right aligned), sliding-window and document masks each
// allow a contiguous range of keys for a query row, so their intersection is
// one interval; `Params` provides Sq, Sk, causal, window_left, window_right,
// doc_offsets and num_docs.
// Keys [lo, hi] (inclusive) that query `row` may attend to; lo > hi = none.
struct KeyRange {
    int lo, hi;
};

template <class Params>
__device__ __forceinline__ KeyRange row_key_range(const Params &p, int row) {
    long long lo = 0, hi = (long long)p.Sk - 1;
    const long long diag = (long long)row + p.Sk - p.Sq;
    if (p.causal) hi = min(hi, diag);
    if (p.window_left >= 0) lo = max(lo, diag - p.window_left);
    if (p.window_right >= 0) hi = min(hi, diag + p.window_right);
    if (p.doc_offsets != nullptr) {
        const int *off = p.doc_offsets;
        if (row < __ldg(off) || row >= __ldg(off + p.num_docs)) return {1, 0};
        int a = 0, c = p.num_docs;  // off[a] <= row < off[c]
        while (c - a > 1) {
            const int m = (a + c) >> 1;
            if (__ldg(off + m) <= row) a = m; else c = m;
        }
        lo = max(lo, (long long)__ldg(off + a));
        hi = min(hi, (long long)__ldg(off + a + 1) - 1);
    }
    if (lo > hi) return {1, 0};
    return {(int)lo, (int)hi};
}

// Union of the key intervals of rows [r0, r1] (r0 <= r1 < Sq), computed by
// one whole warp; {1, 0} when no row has a key.  Every mask here is monotone
// -- a row's interval never moves left as the row index grows, and the rows
// with a key form one contiguous run -- so when the first and the last row
// both have keys they bound the union; otherwise (a tile at the edge of the
// rows that see any key) every row is visited.
template <class Params>
__device__ __forceinline__ KeyRange tile_key_range(const Params &p, int r0, int r1, int lane) {
    const KeyRange a = row_key_range(p, r0);
    const KeyRange z = row_key_range(p, r1);
    if (a.lo <= a.hi && z.lo <= z.hi) return {a.lo, z.hi};
    int lo = 0x7fffffff, hi = -1;
    for (int row = r0 + lane; row <= r1; row += 32) {
        const KeyRange r = row_key_range(p, row);
        if (r.lo <= r.hi) {
            lo = min(lo, r.lo);
            hi = max(hi, r.hi);
        }
    }
    for (int o = 16; o > 0; o >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (hi < 0) return {1, 0};
    return {lo, hi};
}

// Bounded wait.  Returns false when the CTA is aborting (own timeout or
// another role's); `honor_abort` = false keeps waiting until the timeout only.
template <bool kHint = false>
__device__ __forceinline__ bool wait_bounded(uint64_t *bar, uint32_t parity,
                                             volatile int *abort_flag, int *status,
                                             bool honor_abort = true,
                                             uint64_t timeout_ns = kWaitTimeoutNs) {
    if (mbar_try_wait<kHint>(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait<kHint>(bar, parity)) return true;
        if ((n & 15u) == 0u) {
            if (honor_abort && *abort_flag) return false;
            if (globaltimer_ns() - t0 > timeout_ns) {
                *abort_flag = 1;
                atomicCAS(status, 0, kStatusTimeout);
                return false;
            }
        }
    }
}

constexpr float kLog2eF = 1.4426950408889634f;

// Soft-capped scores of a pair, in log2 units: with u = e^(2y), y = raw *
// scale / cap, tanh(y) = 1 - 2 / (u + 1), so cap * log2(e) * tanh(y) =
// so - 2 so r with r = 1 / (u + 1).  k1 = 2 log2(e) scale / cap, so =
// cap log2(e).  Two MUFU operations per score (ex2, rcp) and three packed
// FMA-pipe operations per pair; u = inf gives r = 0 (tanh = 1), u = 0 gives
// r = 1 (tanh = -1).  r is returned too: the backward's d tanh / dy =
// 1 - tanh^2 = 4 r (1 - r).
__device__ __forceinline__ void softcap_pair(float &x0, float &x1, float &r0, float &r1,
                                             float raw0, float raw1, float k1, float so) {
    float a0, a1;
    mul2(a0, a1, raw0, raw1, k1, k1);
    float u0 = ex2_mufu(a0), u1 = ex2_mufu(a1);
    add2(u0, u1, u0, u1, 1.0f, 1.0f);
    r0 = rcp_mufu(u0);
    r1 = rcp_mufu(u1);
    fma2(x0, x1, r0, r1, -2.0f * so, -2.0f * so, so, so);
}

// Software 2^x for the FMA pipe ("FlashAttention-4 de NVIDIA", "La ventaja técnica":
// part of the exponentials as a cubic on the CUDA cores): our minimax cubic
// (exp2_poly.cuh, fitted by fit_exp2.py) with 2^round(x) applied through the
// exponent field.
__device__ __forceinline__ float ex2_poly(float x) {
    // x = j + f, j = round(x) via the 1.5 * 2^23 trick, f in [-1/2, 1/2];
    // 2^x = p(f) * 2^j with 2^j applied through the exponent field.
    x = fmaxf(x, -125.0f);
    const float magic = 12582912.0f;
    const float t = x + magic;
    const float f = x - (t - magic);
    const float p = fmaf(fmaf(fmaf(kExp2C3, f, kExp2C2), f, kExp2C1), f, kExp2C0);
    return __uint_as_float(__float_as_uint(p) + (__float_as_uint(t) << 23));
}

// Two lanes at once with packed f32x2 arithmetic; same steps as ex2_poly.
__device__ __forceinline__ void ex2_poly2(float &y0, float &y1, float x0, float x1) {
    x0 = fmaxf(x0, -125.0f);
    x1 = fmaxf(x1, -125.0f);
    const float magic = 12582912.0f;
    float t0, t1, j0, j1, f0, f1, p0, p1;
    add2(t0, t1, x0, x1, magic, magic);
    add2(j0, j1, t0, t1, -magic, -magic);
    add2(f0, f1, x0, x1, -j0, -j1);
    fma2(p0, p1, kExp2C3, kExp2C3, f0, f1, kExp2C2, kExp2C2);
    fma2(p0, p1, p0, p1, f0, f1, kExp2C1, kExp2C1);
    fma2(p0, p1, p0, p1, f0, f1, kExp2C0, kExp2C0);
    y0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
    y1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}

}  // namespace tab
