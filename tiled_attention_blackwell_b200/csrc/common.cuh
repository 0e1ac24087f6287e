// Pieces shared by the forward and backward kernels: the per-row key
// interval every supported mask reduces to, and bounded mbarrier waits.
#pragma once

#include "ptx.cuh"

namespace tab {

constexpr uint64_t kWaitTimeoutNs = 1000000000ull;  // 1 s per wait
constexpr int kStatusTimeout = 5;                   // ATTN_ERR_DEVICE_TIMEOUT

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

// Bounded wait.  Returns false when the CTA is aborting (own timeout or
// another role's); `honor_abort` = false keeps waiting until the timeout only.
__device__ __forceinline__ bool wait_bounded(uint64_t *bar, uint32_t parity,
                                             volatile int *abort_flag, int *status,
                                             bool honor_abort = true) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((n & 15u) == 0u) {
            if (honor_abort && *abort_flag) return false;
            if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
                *abort_flag = 1;
                atomicCAS(status, 0, kStatusTimeout);
                return false;
            }
        }
    }
}

}  // namespace tab
