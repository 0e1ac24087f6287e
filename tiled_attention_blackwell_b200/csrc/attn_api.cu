// C ABI of the attention library: argument validation, TMA descriptor
// encoding, kernel selection and launch.  See include/attn.h for the
// contract of every entry point.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "../../include/attn.h"
#include "bwd_kernel.cuh"
#include "fp4_dequant.cuh"
#include "fwd_fp4_kernel.cuh"
#include "fwd_kernel.cuh"
#include "fwd_persistent.cuh"

namespace {

constexpr int kMaxDevices = 64;

thread_local char g_detail[512] = "";

attn_status_t fail(attn_status_t status, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof g_detail, fmt, ap);
    va_end(ap);
    return status;
}

attn_status_t ok() {
    g_detail[0] = '\0';
    return ATTN_OK;
}

// ------------------------------------------------------- device status word

__device__ int g_status_word;

struct DeviceState {
    std::once_flag once;
    cudaError_t init_error = cudaSuccess;
    int *status = nullptr;  // device address of g_status_word
    int num_sms = 0;
};
DeviceState g_devices[kMaxDevices];

attn_status_t device_state(DeviceState **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(ATTN_ERR_UNSUPPORTED, "device index %d", dev);
    DeviceState &st = g_devices[dev];
    std::call_once(st.once, [&]() {
        st.init_error = cudaGetSymbolAddress(reinterpret_cast<void **>(&st.status), g_status_word);
        if (st.init_error == cudaSuccess)
            st.init_error = cudaDeviceGetAttribute(&st.num_sms, cudaDevAttrMultiProcessorCount, dev);
    });
    if (st.init_error != cudaSuccess)
        return fail(ATTN_ERR_CUDA, "device %d set-up: %s", dev, cudaGetErrorString(st.init_error));
    *out = &st;
    return ATTN_OK;
}

// ----------------------------------------------------------- tensor maps

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, []() {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// bf16 tensor [B][S][H][D] as a 4-D map (D, S, H, B), box (64, 128, 1, 1),
// 128-byte swizzle, zero fill out of bounds.
// 4-D map of a [B][S][H][D] tensor with `eb`-byte elements; the box is one
// 128-byte row chunk (128 / eb elements) by kBlockM positions.
attn_status_t make_map(CUtensorMap *map, const void *base, int B, int S, int H, int D,
                       int eb = 2) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)S, (cuuint64_t)H, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)H * D * eb, (cuuint64_t)D * eb,
                                   (cuuint64_t)S * H * D * eb};
    const cuuint32_t box[4] = {(cuuint32_t)(128 / eb), (cuuint32_t)tab::kBlockM, 1, 1};
    const cuuint32_t estride[4] = {1, 1, 1, 1};
    const CUtensorMapDataType dtype =
        eb == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUresult r = fn(map, dtype, 4, const_cast<void *>(base), dims,
                    strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return ATTN_OK;
}

// 5-D map of a bf16 [B][S][H][D] tensor whose box is a whole 128-row tile:
// dims (64 columns, S, D/64 column chunks, H, B), box (64, 128, D/64, 1, 1),
// so one copy fills the tile's D/64 chunks of [128 rows][128 bytes] (the
// chunk dimension's stride, 128 bytes, is smaller than the row stride; the
// copy is still one affine box).
attn_status_t make_map_tile(CUtensorMap *map, const void *base, int B, int S, int H, int D) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const cuuint64_t dims[5] = {64, (cuuint64_t)S, (cuuint64_t)(D / 64), (cuuint64_t)H,
                                (cuuint64_t)B};
    const cuuint64_t strides[4] = {(cuuint64_t)H * D * 2, 128, (cuuint64_t)D * 2,
                                   (cuuint64_t)S * H * D * 2};
    const cuuint32_t box[5] = {64, (cuuint32_t)tab::kBlockM, (cuuint32_t)(D / 64), 1, 1};
    const cuuint32_t estride[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims,
                    strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled (tile) failed (%d)", (int)r);
    return ATTN_OK;
}

// 4-D map of packed FP4 codes, 64 bytes (128 codes) per row: dims (64,
// rows, H, B) with the given row / head / batch strides in bytes; box one
// 128-row tile, 64-byte swizzle (the layout of the block-scaled MMA
// operands), zero fill out of bounds.
attn_status_t make_map_fp4(CUtensorMap *map, const void *base, long long inner, int rows, int H,
                           int B, long long row_stride, long long head_stride,
                           long long batch_stride) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)H, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)row_stride, (cuuint64_t)head_stride,
                                   (cuuint64_t)batch_stride};
    const cuuint32_t box[4] = {64, (cuuint32_t)tab::kBlockM, 1, 1};
    const cuuint32_t estride[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void *>(base), dims, strides,
                    box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled (fp4) failed (%d)", (int)r);
    return ATTN_OK;
}

// --------------------------------------------------------------- launching

// PERSIST selects the persistent kernel (fwd_persistent.cuh: one CTA per SM
// running many items), otherwise one CTA per item.
template <int D, int NS, int EXP, int MOD = 0, int PREC = 0, bool PERSIST = false>
attn_status_t launch_fwd(const tab::FwdParams &p, int grid, cudaStream_t stream) {
    using Smem = std::conditional_t<PERSIST, tab::FwdSmemPersistent<D, NS, PREC == 1 ? 1 : 2>,
                                    tab::FwdSmem<D, NS, PREC == 1 ? 1 : 2>>;
    constexpr size_t smem = sizeof(Smem) + 1024;
    static_assert(smem <= 232448, "shared memory budget");
    auto kernel = []() {
        if constexpr (PERSIST) return tab::attn_fwd_persistent_kernel<D, NS, EXP, MOD, PREC>;
        else return tab::attn_fwd_kernel<D, NS, EXP, MOD, PREC>;
    }();
    static std::once_flag once[kMaxDevices];
    static cudaError_t attr_err[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    std::call_once(once[dev], [&]() {
        attr_err[dev] = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
    });
    if (attr_err[dev] != cudaSuccess)
        return fail(ATTN_ERR_LAUNCH, "cudaFuncSetAttribute: %s", cudaGetErrorString(attr_err[dev]));
    // The kernel moves registers between warpgroups with setmaxnreg; if the
    // compiled per-thread count does not cover the split, the increase would
    // wait forever, so never launch such a build.
    static cudaFuncAttributes attrs[kMaxDevices];
    static cudaError_t attrs_err[kMaxDevices];
    static std::once_flag attrs_once[kMaxDevices];
    std::call_once(attrs_once[dev], [&]() { attrs_err[dev] = cudaFuncGetAttributes(&attrs[dev], kernel); });
    if (attrs_err[dev] != cudaSuccess)
        return fail(ATTN_ERR_LAUNCH, "cudaFuncGetAttributes: %s", cudaGetErrorString(attrs_err[dev]));
    if (attrs[dev].numRegs < tab::kLaunchRegs)
        return fail(ATTN_ERR_LAUNCH, "kernel compiled with %d registers per thread, %d needed",
                    attrs[dev].numRegs, tab::kLaunchRegs);
    kernel<<<grid, tab::kFwdThreads, smem, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(ATTN_ERR_LAUNCH, "launch: %s", cudaGetErrorString(e));
    return ok();
}

constexpr int kStagesD128 = 4;
// Key/value heads whose query heads' CTAs are scheduled together: 8 heads of
// K/V at S = 8192, D = 128 are 32 MiB, well inside the 126 MiB L2.
// Measured on B200 (causal S=8192, outlier S=4096, GQA document S=16384):
// 8 beats 4, 16 and all heads for the first two; with 4 query heads per
// key/value head the group covers 32 query heads.
constexpr int kFwdHeadGroup = 8;

// (batch, query head) pairs per schedule group of the persistent forward.
// A group's items are dealt to the CTAs in snake rounds, so the group should
// span several rounds (a round boundary falling inside a group costs
// balance) while keeping each round's items on few heads (K/V reuse in L2):
// at least the kFwdHeadGroup key/value heads' query heads and a quarter of
// a round of pairs, rounded up to whole key/value heads.
int fwd_schedule_group(int B, int Hq, int Hkv, int ctas) {
    const int qpk = Hq / Hkv;
    int g = std::max(kFwdHeadGroup * qpk, (ctas + 3) / 4);
    g = (g + qpk - 1) / qpk * qpk;
    return std::min(B * Hq, g);
}
constexpr int kStagesD64 = 8;
constexpr int kStagesFp8 = 8;  // fp8 K/V tiles are 16 KB at D = 128

template <int D, int NS>
attn_status_t dispatch_exp(const tab::FwdParams &p, int grid, int exp_mode, int mod,
                           cudaStream_t s) {
    // With a score modifier the exponentials all run on MUFU.
    switch (mod) {
        case 1: return launch_fwd<D, NS, 0, 1>(p, grid, s);
        case 2: return launch_fwd<D, NS, 0, 2>(p, grid, s);
        case 3: return launch_fwd<D, NS, 0, 3>(p, grid, s);
        default: break;
    }
    switch (exp_mode) {
        case 0: return launch_fwd<D, NS, 0>(p, grid, s);
        case 1: return launch_fwd<D, NS, 1>(p, grid, s);
        default: return launch_fwd<D, NS, 2>(p, grid, s);
    }
}

// The fp8 forward runs persistent (measured 6 % faster than one CTA per item
// at causal S=8192; for bf16 operands the persistent kernel is slower).
attn_status_t dispatch_fp8(const tab::FwdParams &p, int grid, int exp_mode, cudaStream_t s) {
    switch (exp_mode) {
        case 0: return launch_fwd<128, kStagesFp8, 0, 0, 1, true>(p, grid, s);
        case 1: return launch_fwd<128, kStagesFp8, 1, 0, 1, true>(p, grid, s);
        default: return launch_fwd<128, kStagesFp8, 2, 0, 1, true>(p, grid, s);
    }
}

// Direct-P kernels: PREC 2 (affine classifier) or 3 (exponential).
attn_status_t dispatch_direct_p(const tab::FwdParams &p, int grid, int D, int classifier,
                                cudaStream_t s) {
    if (D == 128)
        return classifier ? launch_fwd<128, kStagesD128, 0, 0, 3>(p, grid, s)
                          : launch_fwd<128, kStagesD128, 0, 0, 2>(p, grid, s);
    return classifier ? launch_fwd<64, kStagesD64, 0, 0, 3>(p, grid, s)
                      : launch_fwd<64, kStagesD64, 0, 0, 2>(p, grid, s);
}

// The block-scaled FP4 Direct-P kernel (fwd_fp4_kernel.cuh), D = 128.
constexpr int kStagesFp4 = 8;  // K or V^T slots of 9 KB
template <int CLS>
attn_status_t launch_fp4bs(const tab::FwdParams &p, int grid, cudaStream_t stream) {
    using Smem = tab::FwdSmemFp4<kStagesFp4>;
    constexpr size_t smem = sizeof(Smem) + 1024;
    static_assert(smem <= 232448, "shared memory budget");
    auto kernel = tab::attn_fwd_fp4bs_kernel<kStagesFp4, CLS>;
    static std::once_flag once[kMaxDevices];
    static cudaError_t attr_err[kMaxDevices];
    static cudaFuncAttributes attrs[kMaxDevices];
    static cudaError_t attrs_err[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    std::call_once(once[dev], [&]() {
        attr_err[dev] = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        attrs_err[dev] = cudaFuncGetAttributes(&attrs[dev], kernel);
    });
    if (attr_err[dev] != cudaSuccess)
        return fail(ATTN_ERR_LAUNCH, "cudaFuncSetAttribute: %s", cudaGetErrorString(attr_err[dev]));
    if (attrs_err[dev] != cudaSuccess)
        return fail(ATTN_ERR_LAUNCH, "cudaFuncGetAttributes: %s", cudaGetErrorString(attrs_err[dev]));
    // setmaxnreg split: see launch_fwd.
    if (attrs[dev].numRegs < tab::kLaunchRegs)
        return fail(ATTN_ERR_LAUNCH, "kernel compiled with %d registers per thread, %d needed",
                    attrs[dev].numRegs, tab::kLaunchRegs);
    kernel<<<grid, tab::kFwdThreads, smem, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(ATTN_ERR_LAUNCH, "launch: %s", cudaGetErrorString(e));
    return ok();
}

size_t align256(size_t n) { return (n + 255) & ~(size_t)255; }

// Workspace of the block-scaled path: scale atoms of Q (tiles of both of a
// CTA's query blocks), K and V, then V^T's codes.
struct Fp4BsLayout {
    int nqt, nkt;
    size_t sf_q, sf_k, sf_v, vt, total;
};
Fp4BsLayout fp4bs_layout(int B, int Hq, int Hkv, int Sq, int Sk) {
    Fp4BsLayout L;
    L.nqt = 2 * ((Sq + 2 * tab::kBlockM - 1) / (2 * tab::kBlockM));
    L.nkt = (Sk + tab::kBlockN - 1) / tab::kBlockN;
    const size_t atoms = 2 * tab::kSfAtom;
    L.sf_q = 0;
    L.sf_k = L.sf_q + align256((size_t)B * Hq * L.nqt * atoms);
    L.sf_v = L.sf_k + align256((size_t)B * Hkv * L.nkt * atoms);
    L.vt = L.sf_v + align256((size_t)B * Hkv * L.nkt * atoms);
    L.total = L.vt + align256((size_t)B * Hkv * 128 * L.nkt * 64);
    return L;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape and mask checks shared by the forward and the backward.
attn_status_t check_common(int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale,
                           int window_left, int window_right, const int *doc_offsets,
                           int num_docs) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Sq < 1 || Sk < 1)
        return fail(ATTN_ERR_INVALID_ARG, "B, Hq, Hkv, Sq, Sk must be >= 1");
    if (Hq % Hkv != 0)
        return fail(ATTN_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
    if (D != 64 && D != 128)
        return fail(ATTN_ERR_UNSUPPORTED, "head dim %d (built: 64, 128)", D);
    if (!(scale > 0.0f) || !std::isfinite(scale))
        return fail(ATTN_ERR_INVALID_ARG, "scale must be positive and finite");
    if (window_left < -1 || window_right < -1)
        return fail(ATTN_ERR_INVALID_ARG, "window bounds must be -1 or >= 0");
    if ((doc_offsets == nullptr) != (num_docs == 0) || num_docs < 0)
        return fail(ATTN_ERR_INVALID_ARG, "doc_offsets and num_docs must be given together");
    if (doc_offsets && Sq != Sk)
        return fail(ATTN_ERR_INVALID_ARG, "a document mask requires Sq == Sk");
    const double max_stride = (double)std::max(Sq, Sk) * Hq * D * 4.0;
    if (max_stride >= 1099511627776.0)
        return fail(ATTN_ERR_UNSUPPORTED, "tensor too large for a TMA descriptor");
    return ATTN_OK;
}

template <class Kernel>
attn_status_t prepare_kernel(Kernel kernel, size_t smem, int threads, int min_regs) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess)
        return fail(ATTN_ERR_LAUNCH, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    cudaFuncAttributes attrs;
    e = cudaFuncGetAttributes(&attrs, kernel);
    if (e != cudaSuccess)
        return fail(ATTN_ERR_LAUNCH, "cudaFuncGetAttributes: %s", cudaGetErrorString(e));
    if (attrs.numRegs < min_regs || attrs.maxThreadsPerBlock < threads)
        return fail(ATTN_ERR_LAUNCH, "kernel build cannot be launched (%d regs, %d threads)",
                    attrs.numRegs, attrs.maxThreadsPerBlock);
    return ATTN_OK;
}

constexpr int kBwdStagesQ = 2;
// dQ kernel: K and V ring depths (224 KB of SMEM with Q and dO at D = 128).
constexpr int bwd_k_stages(int D) { return D == 128 ? 3 : 6; }
constexpr int bwd_v_stages(int D) { return D == 128 ? 2 : 4; }

template <int D, int MOD>
attn_status_t launch_bwd(const tab::BwdParams &p, cudaStream_t stream) {
    using DkdvS = tab::DkdvSmem<D, kBwdStagesQ>;
    using DqS = tab::DqSmem<D, bwd_k_stages(D), bwd_v_stages(D)>;
    constexpr size_t smem_dkdv = sizeof(DkdvS) + 1024;
    constexpr size_t smem_dq = sizeof(DqS) + 1024;
    static_assert(smem_dkdv <= 232448 && smem_dq <= 232448, "shared memory budget");
    auto k_dkdv = tab::attn_bwd_dkdv_kernel<D, kBwdStagesQ, MOD>;
    auto k_dq = tab::attn_bwd_dq_kernel<D, bwd_k_stages(D), bwd_v_stages(D), MOD>;
    static std::once_flag once[kMaxDevices];
    static attn_status_t prep[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    std::call_once(once[dev], [&]() {
        prep[dev] = prepare_kernel(k_dkdv, smem_dkdv, tab::kBwdThreads, 0);
        if (prep[dev] == ATTN_OK) prep[dev] = prepare_kernel(k_dq, smem_dq, tab::kBwdThreads, 0);
    });
    if (prep[dev] != ATTN_OK) return fail(prep[dev], "backward kernels could not be prepared");
    // dQ first: it also computes D_i into the workspace, which the dK/dV
    // kernel reads.
    k_dq<<<p.num_qb * p.Hq * p.B, tab::kBwdThreads, smem_dq, stream>>>(p);
    k_dkdv<<<p.num_kb * p.Hkv * p.B, tab::kBwdThreads, smem_dkdv, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(ATTN_ERR_LAUNCH, "launch: %s", cudaGetErrorString(e));
    return ok();
}

template <int D>
attn_status_t dispatch_bwd(const tab::BwdParams &p, int mod, cudaStream_t stream) {
    switch (mod) {
        case 1: return launch_bwd<D, 1>(p, stream);
        case 2: return launch_bwd<D, 2>(p, stream);
        case 3: return launch_bwd<D, 3>(p, stream);
        default: return launch_bwd<D, 0>(p, stream);
    }
}

// Shared checks of the score-modifier fields of both option structs.
attn_status_t check_modifiers(float softcap, int reserved0, const float *alibi_slopes,
                              const int *reserved, int n_reserved) {
    for (int i = 0; i < n_reserved; ++i)
        if (reserved[i] != 0) return fail(ATTN_ERR_INVALID_ARG, "reserved option fields must be zero");
    if (reserved0 != 0) return fail(ATTN_ERR_INVALID_ARG, "reserved option fields must be zero");
    if (!(softcap >= 0.0f) || !std::isfinite(softcap))
        return fail(ATTN_ERR_INVALID_ARG, "softcap must be >= 0 and finite");
    if ((reinterpret_cast<uintptr_t>(alibi_slopes) & 3u) != 0)
        return fail(ATTN_ERR_MISALIGNED, "alibi_slopes must be 4-byte aligned");
    return ATTN_OK;
}

// Checks of the backward's tensors and shapes, shared by attn_bwd_ex and
// attn_bwd_noalloc; no CUDA call.
attn_status_t check_bwd_args(const void *q, const void *k, const void *v, const void *o,
                             const float *lse, const void *dout, const float *dq, const void *dk,
                             const void *dv, int B, int Hq, int Hkv, int Sq, int Sk, int D,
                             float scale, int window_left, int window_right,
                             const int *doc_offsets, int num_docs) {
    if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv)
        return fail(ATTN_ERR_INVALID_ARG, "null pointer");
    attn_status_t s = check_common(B, Hq, Hkv, Sq, Sk, D, scale, window_left, window_right,
                                   doc_offsets, num_docs);
    if (s != ATTN_OK) return s;
    for (const void *ptr : {q, k, v, o, dout, (const void *)dq, dk, dv})
        if (!aligned16(ptr)) return fail(ATTN_ERR_MISALIGNED, "tensors must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0)
        return fail(ATTN_ERR_MISALIGNED, "lse must be 4-byte aligned");
    const long long num_qb = (Sq + 127LL) / 128, num_kb = (Sk + 127LL) / 128;
    if (num_qb * Hq * B > 0x7fffffffLL || num_kb * Hkv * B > 0x7fffffffLL)
        return fail(ATTN_ERR_UNSUPPORTED, "grid too large");
    return ATTN_OK;
}

#ifdef ATTN_TRACE
long long *g_trace = nullptr;
int g_trace_ctas = 0;
#endif
#ifdef ATTN_COUNT_RESCALES
unsigned long long *g_rescale_counts = nullptr;
#endif

// ------------------------------------------ scratch of attn_bwd_noalloc
// D_i of up to kNoAllocRows rows for callers that cannot allocate a
// workspace.  The array exists on every device that loads the library.
constexpr size_t kNoAllocRows = size_t(1) << 20;  // 4 MiB of fp32
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocRows];

struct NoAllocScratch {
    std::once_flag once;
    cudaError_t err = cudaSuccess;
    void *ptr = nullptr;  // device address of g_noalloc_scratch on this device
};
NoAllocScratch g_noalloc[kMaxDevices];

}  // namespace

extern "C" {

void attn_fwd_default_options(attn_fwd_options_t *opts) {
    if (!opts) return;
    *opts = attn_fwd_options_t{};
    opts->rescale_threshold = 8.0f;
    opts->exp2_mode = 1;
}

// The forward of both entry points.  fp8: Q, K, V are e4m3 codes with the
// given dequantisation factors (ignored for bf16).
static attn_status_t fwd_impl(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                       int Hq, int Hkv, int Sq, int Sk, int D, float scale, int causal,
                       int window_left, int window_right, const int *doc_offsets,
                       int num_docs, const attn_fwd_options_t *opts, bool fp8,
                       float q_descale, float k_descale, float v_descale, void *stream) {
    attn_fwd_options_t op;
    attn_fwd_default_options(&op);
    if (opts) op = *opts;

    // ----- validation (no CUDA call before this block completes)
    if (!q || !k || !v || !o || !lse)
        return fail(ATTN_ERR_INVALID_ARG, "null tensor pointer");
    {
        attn_status_t c = check_common(B, Hq, Hkv, Sq, Sk, D, scale, window_left, window_right,
                                       doc_offsets, num_docs);
        if (c != ATTN_OK) return c;
    }
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return fail(ATTN_ERR_MISALIGNED, "q, k, v, o must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0)
        return fail(ATTN_ERR_MISALIGNED, "lse must be 4-byte aligned");
    if (!(op.rescale_threshold >= 0.0f && op.rescale_threshold <= 16.0f))
        return fail(ATTN_ERR_INVALID_ARG, "rescale_threshold must lie in [0, 16]");
    if (op.exp2_mode < 0 || op.exp2_mode > 2)
        return fail(ATTN_ERR_INVALID_ARG, "exp2_mode must be 0, 1 or 2");
    if (op.wait_timeout_us < 0 || op.wait_timeout_us > 60000000)
        return fail(ATTN_ERR_INVALID_ARG, "wait_timeout_us must lie in [0, 60000000]");
    if (op.debug_withhold_kv != 0 && op.debug_withhold_kv != 1)
        return fail(ATTN_ERR_INVALID_ARG, "debug_withhold_kv must be 0 or 1");
    {
        attn_status_t c = check_modifiers(op.softcap, op.reserved0, op.alibi_slopes, op.reserved, 4);
        if (c != ATTN_OK) return c;
    }
    if (fp8) {
        if (D != 128) return fail(ATTN_ERR_UNSUPPORTED, "the fp8 forward supports D = 128 only");
        for (float d : {q_descale, k_descale, v_descale})
            if (!(d > 0.0f) || !std::isfinite(d))
                return fail(ATTN_ERR_INVALID_ARG, "descale factors must be > 0 and finite");
        if (op.softcap != 0.0f || op.alibi_slopes)
            return fail(ATTN_ERR_UNSUPPORTED, "the fp8 forward has no score modifiers");
        if (op.rescale_threshold > 8.0f)
            return fail(ATTN_ERR_INVALID_ARG, "the fp8 forward needs rescale_threshold <= 8");
    }
    const long long num_qblocks = (Sq + 2LL * tab::kBlockM - 1) / (2LL * tab::kBlockM);
    const long long items = num_qblocks * Hq * B;
    if (items > 0x7fffffffLL) return fail(ATTN_ERR_UNSUPPORTED, "grid too large");

    // ----- set-up
    DeviceState *st = nullptr;
    attn_status_t s = device_state(&st);
    if (s != ATTN_OK) return s;
    // One CTA per item, or (persistent fp8 kernel) one per SM.
    const int grid = fp8 ? (int)std::min<long long>(items, st->num_sms) : (int)items;

    tab::FwdParams p;
    memset(&p, 0, sizeof p);
    const int eb = fp8 ? 1 : 2;
    if ((s = make_map(&p.tm_q, q, B, Sq, Hq, D, eb)) != ATTN_OK) return s;
    if ((s = make_map(&p.tm_k, k, B, Sk, Hkv, D, eb)) != ATTN_OK) return s;
    if ((s = make_map(&p.tm_v, v, B, Sk, Hkv, D, eb)) != ATTN_OK) return s;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.lse = lse;
    p.doc_offsets = doc_offsets;
    p.num_docs = num_docs;
    p.status = st->status;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Sq = Sq;
    p.Sk = Sk;
    p.group = Hq / Hkv;
    p.causal = causal ? 1 : 0;
    p.window_left = window_left;
    p.window_right = window_right;
    p.num_qblocks = (int)num_qblocks;
    p.head_group = fp8 ? fwd_schedule_group(B, Hq, Hkv, grid)
                       : std::min(B * Hq, kFwdHeadGroup * (Hq / Hkv));
    p.scale_log2 = (float)((double)scale * 1.4426950408889634);
    if (fp8) {
        p.scale_log2 = (float)((double)scale * q_descale * k_descale * 1.4426950408889634);
        p.v_descale = v_descale;
        // P = 2^(x - m + 8 - tau) <= 2^8: e4m3 reaches 448, and the small
        // probabilities keep as many normal-range bits as tau allows.
        p.p_offset = 8.0f - op.rescale_threshold;
    }
    p.rescale_threshold = op.rescale_threshold;
    p.timeout_ns = op.wait_timeout_us > 0 ? 1000ull * (unsigned long long)op.wait_timeout_us
                                          : tab::kWaitTimeoutNs;
    p.debug_withhold_kv = op.debug_withhold_kv;
    const int mod = (op.softcap > 0.0f ? 1 : 0) | (op.alibi_slopes ? 2 : 0);
    if (op.softcap > 0.0f) {
        p.softcap_in = (float)((double)scale / op.softcap);
        p.softcap_out = (float)((double)op.softcap * 1.4426950408889634);
    }
    p.alibi_slopes = op.alibi_slopes;
#ifdef ATTN_TRACE
    p.trace = g_trace;
    p.trace_ctas = g_trace_ctas;
#endif
#ifdef ATTN_COUNT_RESCALES
    p.rescale_counts = g_rescale_counts;
#endif

    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (fp8) return dispatch_fp8(p, grid, op.exp2_mode, cs);
    if (D == 128) return dispatch_exp<128, kStagesD128>(p, grid, op.exp2_mode, mod, cs);
    return dispatch_exp<64, kStagesD64>(p, grid, op.exp2_mode, mod, cs);
}

attn_status_t attn_fwd_ex(const void *q, const void *k, const void *v, void *o, float *lse,
                          int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale,
                          int causal, int window_left, int window_right,
                          const int *doc_offsets, int num_docs,
                          const attn_fwd_options_t *opts, void *stream) {
    return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, D, scale, causal, window_left,
                    window_right, doc_offsets, num_docs, opts, false, 1.0f, 1.0f, 1.0f, stream);
}

attn_status_t attn_fwd_fp8(const void *q, const void *k, const void *v, float q_descale,
                           float k_descale, float v_descale, void *o, float *lse, int B,
                           int Hq, int Hkv, int Sq, int Sk, int D, float scale, int causal,
                           int window_left, int window_right, const int *doc_offsets,
                           int num_docs, const attn_fwd_options_t *opts, void *stream) {
    return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, D, scale, causal, window_left,
                    window_right, doc_offsets, num_docs, opts, true, q_descale, k_descale,
                    v_descale, stream);
}

attn_status_t attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                       int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale,
                       int causal, int window_left, int window_right,
                       const int *doc_offsets, int num_docs, void *stream) {
    return attn_fwd_ex(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, D, scale, causal, window_left,
                       window_right, doc_offsets, num_docs, nullptr, stream);
}

void attn_fp4_default_options(attn_fp4_options_t *opts) {
    if (!opts) return;
    *opts = attn_fp4_options_t{};
    opts->rescale_threshold = 8.0f;
    opts->classifier = ATTN_DIRECT_P_AFFINE;
    opts->mma = ATTN_FP4_MMA_AUTO;
}

size_t attn_fwd_fp4_workspace_size(int B, int Hq, int Hkv, int Sq, int Sk, int D) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Sq < 1 || Sk < 1 || D < 1) return 0;
    const size_t nq = (size_t)B * Sq * Hq * D, nkv = (size_t)B * Sk * Hkv * D;
    const size_t widened = align256(nq * 2) + 2 * align256(nkv * 2);
    // Room for either path (the options pick one per call).
    return D == 128 ? std::max(widened, fp4bs_layout(B, Hq, Hkv, Sq, Sk).total) : widened;
}

attn_status_t attn_fwd_fp4(const void *q_codes, const void *q_scales, float q_global,
                           const void *k_codes, const void *k_scales, float k_global,
                           const void *v_codes, const void *v_scales, float v_global, void *o,
                           float *lse, int B, int Hq, int Hkv, int Sq, int Sk, int D,
                           float scale, int causal, int window_left, int window_right,
                           const int *doc_offsets, int num_docs, void *workspace,
                           size_t workspace_bytes, const attn_fp4_options_t *opts,
                           void *stream) {
    attn_fp4_options_t op;
    attn_fp4_default_options(&op);
    if (opts) op = *opts;

    // ----- validation (no CUDA call before this block completes)
    const void *ptrs[] = {q_codes, q_scales, k_codes, k_scales, v_codes, v_scales, o, workspace};
    for (const void *ptr : ptrs)
        if (!ptr) return fail(ATTN_ERR_INVALID_ARG, "null pointer");
    if (!lse) return fail(ATTN_ERR_INVALID_ARG, "null pointer");
    attn_status_t s = check_common(B, Hq, Hkv, Sq, Sk, D, scale, window_left, window_right,
                                   doc_offsets, num_docs);
    if (s != ATTN_OK) return s;
    for (const void *ptr : ptrs)
        if (!aligned16(ptr))
            return fail(ATTN_ERR_MISALIGNED, "codes, scales, o and workspace must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0)
        return fail(ATTN_ERR_MISALIGNED, "lse must be 4-byte aligned");
    for (float g : {q_global, k_global, v_global})
        if (!(g > 0.0f) || !std::isfinite(g))
            return fail(ATTN_ERR_INVALID_ARG, "per-tensor factors must be > 0 and finite");
    if (!(op.rescale_threshold >= 0.0f && op.rescale_threshold <= 8.0f))
        return fail(ATTN_ERR_INVALID_ARG, "rescale_threshold must lie in [0, 8]");
    if (op.classifier != ATTN_DIRECT_P_AFFINE && op.classifier != ATTN_DIRECT_P_EXP2)
        return fail(ATTN_ERR_INVALID_ARG, "classifier must be ATTN_DIRECT_P_AFFINE or ATTN_DIRECT_P_EXP2");
    if (op.wait_timeout_us < 0 || op.wait_timeout_us > 60000000)
        return fail(ATTN_ERR_INVALID_ARG, "wait_timeout_us must lie in [0, 60000000]");
    if (op.mma < ATTN_FP4_MMA_AUTO || op.mma > ATTN_FP4_MMA_BLOCK_SCALED)
        return fail(ATTN_ERR_INVALID_ARG, "mma must be ATTN_FP4_MMA_AUTO, _F16 or _BLOCK_SCALED");
    if (op.mma == ATTN_FP4_MMA_BLOCK_SCALED && D != 128)
        return fail(ATTN_ERR_UNSUPPORTED, "the block-scaled FP4 products are built for D = 128");
    for (int r : op.reserved)
        if (r != 0) return fail(ATTN_ERR_INVALID_ARG, "reserved option fields must be zero");
    const bool block_scaled = op.mma == ATTN_FP4_MMA_BLOCK_SCALED ||
                              (op.mma == ATTN_FP4_MMA_AUTO && D == 128);
    const size_t need = attn_fwd_fp4_workspace_size(B, Hq, Hkv, Sq, Sk, D);
    if (workspace_bytes < need)
        return fail(ATTN_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed", workspace_bytes, need);
    const long long num_qblocks = (Sq + 2LL * tab::kBlockM - 1) / (2LL * tab::kBlockM);
    const long long grid = num_qblocks * Hq * B;
    if (grid > 0x7fffffffLL) return fail(ATTN_ERR_UNSUPPORTED, "grid too large");

    // ----- set-up
    DeviceState *st = nullptr;
    if ((s = device_state(&st)) != ATTN_OK) return s;
    const size_t nq = (size_t)B * Sq * Hq * D, nkv = (size_t)B * Sk * Hkv * D;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    void *q16 = ws, *k16 = ws + align256(nq * 2), *v16 = ws + align256(nq * 2) + align256(nkv * 2);
    const Fp4BsLayout L = fp4bs_layout(B, Hq, Hkv, Sq, Sk);

    tab::FwdParams p;
    memset(&p, 0, sizeof p);
    if (block_scaled) {
        // Q and K codes straight from the caller (64 bytes per row); V^T codes
        // and all scale atoms from the preparation pass.
        if ((s = make_map_fp4(&p.tm_q, q_codes, 64, Sq, Hq, B, (long long)Hq * 64, 64,
                              (long long)Sq * Hq * 64)) != ATTN_OK)
            return s;
        if ((s = make_map_fp4(&p.tm_k, k_codes, 64, Sk, Hkv, B, (long long)Hkv * 64, 64,
                              (long long)Sk * Hkv * 64)) != ATTN_OK)
            return s;
        const long long vt_row = (long long)L.nkt * 64;
        if ((s = make_map_fp4(&p.tm_v, ws + L.vt, vt_row, 128, Hkv, B, vt_row, 128 * vt_row,
                              (long long)Hkv * 128 * vt_row)) != ATTN_OK)
            return s;
        p.sf_q = ws + L.sf_q;
        p.sf_k = ws + L.sf_k;
        p.sf_v = ws + L.sf_v;
        p.nq_tiles = L.nqt;
        p.nk_tiles = L.nkt;
    } else {
        if ((s = make_map(&p.tm_q, q16, B, Sq, Hq, D)) != ATTN_OK) return s;
        if ((s = make_map(&p.tm_k, k16, B, Sk, Hkv, D)) != ATTN_OK) return s;
        if ((s = make_map(&p.tm_v, v16, B, Sk, Hkv, D)) != ATTN_OK) return s;
    }
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.lse = lse;
    p.doc_offsets = doc_offsets;
    p.num_docs = num_docs;
    p.status = st->status;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Sq = Sq;
    p.Sk = Sk;
    p.group = Hq / Hkv;
    p.causal = causal ? 1 : 0;
    p.window_left = window_left;
    p.window_right = window_right;
    p.num_qblocks = (int)num_qblocks;
    p.head_group = std::min(B * Hq, kFwdHeadGroup * (Hq / Hkv));
    p.scale_log2 = (float)((double)scale * q_global * k_global * 1.4426950408889634);
    p.v_descale = v_global;
    // P = code * 2^E with E <= 13 below the f16 maximum: with scores at most
    // rescale_threshold above the anchor, an offset of 15 - ceil(threshold)
    // keeps floor(max y) - 2 <= 13.
    p.p_offset = 15.0f - std::ceil(op.rescale_threshold);
    p.rescale_threshold = op.rescale_threshold;
    p.timeout_ns = op.wait_timeout_us > 0 ? 1000ull * (unsigned long long)op.wait_timeout_us
                                          : tab::kWaitTimeoutNs;
#ifdef ATTN_TRACE
    p.trace = g_trace;
    p.trace_ctas = g_trace_ctas;
#endif
#ifdef ATTN_COUNT_RESCALES
    p.rescale_counts = g_rescale_counts;
#endif

    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (block_scaled) {
        tab::Fp4PrepParams pp;
        memset(&pp, 0, sizeof pp);
        pp.q_codes = static_cast<const uint8_t *>(q_codes);
        pp.q_scales = static_cast<const uint8_t *>(q_scales);
        pp.k_codes = static_cast<const uint8_t *>(k_codes);
        pp.k_scales = static_cast<const uint8_t *>(k_scales);
        pp.v_codes = static_cast<const uint8_t *>(v_codes);
        pp.v_scales = static_cast<const uint8_t *>(v_scales);
        pp.sf_q = ws + L.sf_q;
        pp.sf_k = ws + L.sf_k;
        pp.sf_v = ws + L.sf_v;
        pp.vt = ws + L.vt;
        pp.B = B;
        pp.Hq = Hq;
        pp.Hkv = Hkv;
        pp.Sq = Sq;
        pp.Sk = Sk;
        pp.nqt = L.nqt;
        pp.nkt = L.nkt;
        pp.status = st->status;
        const long long v_ctas = (long long)B * Hkv * L.nkt;
        const long long rows = ((long long)B * Hq * L.nqt + (long long)B * Hkv * L.nkt) * 128;
        const long long sf_ctas = std::min<long long>((rows + 255) / 256, (long long)st->num_sms * 8);
        if (v_ctas + sf_ctas > 0x7fffffffLL) return fail(ATTN_ERR_UNSUPPORTED, "grid too large");
        pp.v_ctas = (int)v_ctas;
        tab::fp4_prepare_kernel<<<(unsigned)(v_ctas + sf_ctas), 256, 0, cs>>>(pp);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return fail(ATTN_ERR_LAUNCH, "launch: %s", cudaGetErrorString(e));
        return op.classifier ? launch_fp4bs<1>(p, (int)grid, cs) : launch_fp4bs<0>(p, (int)grid, cs);
    }
    tab::Fp4DequantParams dp;
    memset(&dp, 0, sizeof dp);
    dp.job[0] = {static_cast<const uint8_t *>(q_codes), static_cast<const uint8_t *>(q_scales),
                 static_cast<uint32_t *>(q16), (long long)(nq / 32), Sq, Hq, 0};
    dp.job[1] = {static_cast<const uint8_t *>(k_codes), static_cast<const uint8_t *>(k_scales),
                 static_cast<uint32_t *>(k16), (long long)(nkv / 32), Sk, Hkv, 0};
    dp.job[2] = {static_cast<const uint8_t *>(v_codes), static_cast<const uint8_t *>(v_scales),
                 static_cast<uint32_t *>(v16), (long long)(nkv / 32), Sk, Hkv, 1};
    dp.D = D;
    dp.status = st->status;
    const long long groups = dp.job[0].groups + dp.job[1].groups + dp.job[2].groups;
    const long long blocks = std::min<long long>((groups + 255) / 256, (long long)st->num_sms * 16);
    tab::fp4_dequant_kernel<<<(unsigned)std::max<long long>(blocks, 1), 256, 0, cs>>>(dp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(ATTN_ERR_LAUNCH, "launch: %s", cudaGetErrorString(e));
    return dispatch_direct_p(p, (int)grid, D, op.classifier, cs);
}

size_t attn_bwd_workspace_size(int B, int Hq, int Hkv, int Sq, int Sk, int D) {
    (void)Hkv;
    (void)Sk;
    (void)D;
    if (B < 1 || Hq < 1 || Sq < 1) return 0;
    const size_t n = (size_t)B * Hq * Sq * sizeof(float);
    return (n + 255) & ~(size_t)255;
}

attn_status_t attn_bwd(const void *q, const void *k, const void *v, const void *o,
                       const float *lse, const void *dout, float *dq, void *dk, void *dv,
                       int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale, int causal,
                       int window_left, int window_right, const int *doc_offsets, int num_docs,
                       void *workspace, size_t workspace_bytes, void *stream) {
    return attn_bwd_ex(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Sq, Sk, D, scale, causal,
                       window_left, window_right, doc_offsets, num_docs, workspace,
                       workspace_bytes, nullptr, stream);
}

attn_status_t attn_bwd_ex(const void *q, const void *k, const void *v, const void *o,
                          const float *lse, const void *dout, float *dq, void *dk, void *dv,
                          int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale,
                          int causal, int window_left, int window_right,
                          const int *doc_offsets, int num_docs, void *workspace,
                          size_t workspace_bytes, const attn_bwd_options_t *opts,
                          void *stream) {
    attn_status_t s = check_bwd_args(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Sq, Sk, D,
                                     scale, window_left, window_right, doc_offsets, num_docs);
    if (s != ATTN_OK) return s;
    attn_bwd_options_t op;
    memset(&op, 0, sizeof op);
    if (opts) op = *opts;
    if ((s = check_modifiers(op.softcap, op.reserved0, op.alibi_slopes, op.reserved, 4)) != ATTN_OK)
        return s;
    if (!workspace) return fail(ATTN_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(workspace)) return fail(ATTN_ERR_MISALIGNED, "workspace must be 16-byte aligned");
    const size_t need = attn_bwd_workspace_size(B, Hq, Hkv, Sq, Sk, D);
    if (workspace_bytes < need)
        return fail(ATTN_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed", workspace_bytes, need);
    const long long num_qb = (Sq + 127LL) / 128, num_kb = (Sk + 127LL) / 128;

    DeviceState *st = nullptr;
    if ((s = device_state(&st)) != ATTN_OK) return s;
    tab::BwdParams p;
    memset(&p, 0, sizeof p);
    if ((s = make_map_tile(&p.tm_q, q, B, Sq, Hq, D)) != ATTN_OK) return s;
    if ((s = make_map_tile(&p.tm_do, dout, B, Sq, Hq, D)) != ATTN_OK) return s;
    if ((s = make_map_tile(&p.tm_k, k, B, Sk, Hkv, D)) != ATTN_OK) return s;
    if ((s = make_map_tile(&p.tm_v, v, B, Sk, Hkv, D)) != ATTN_OK) return s;
    p.o = static_cast<const __nv_bfloat16 *>(o);
    p.dout = static_cast<const __nv_bfloat16 *>(dout);
    p.lse = lse;
    p.dval = static_cast<float *>(workspace);
    p.dq = dq;
    p.dk = static_cast<__nv_bfloat16 *>(dk);
    p.dv = static_cast<__nv_bfloat16 *>(dv);
    p.doc_offsets = doc_offsets;
    p.num_docs = num_docs;
    p.status = st->status;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Sq = Sq;
    p.Sk = Sk;
    p.group = Hq / Hkv;
    p.causal = causal ? 1 : 0;
    p.window_left = window_left;
    p.window_right = window_right;
    p.num_qb = (int)num_qb;
    p.num_kb = (int)num_kb;
    p.scale = scale;
    p.scale_log2 = (float)((double)scale * 1.4426950408889634);
    const int mod = (op.softcap > 0.0f ? 1 : 0) | (op.alibi_slopes ? 2 : 0);
    if (op.softcap > 0.0f) {
        p.softcap_in = (float)((double)scale / op.softcap);
        p.softcap_out = (float)((double)op.softcap * 1.4426950408889634);
    }
    p.alibi_slopes = op.alibi_slopes;
#ifdef ATTN_TRACE
    p.trace = g_trace;
    p.trace_ctas = g_trace_ctas;
#endif
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    return D == 128 ? dispatch_bwd<128>(p, mod, cs) : dispatch_bwd<64>(p, mod, cs);
}

attn_status_t attn_bwd_noalloc(const void *q, const void *k, const void *v, const void *o,
                               const float *lse, const void *dout, float *dq, void *dk,
                               void *dv, int B, int Hq, int Hkv, int Sq, int Sk, int D,
                               float scale, int causal, int window_left, int window_right,
                               const int *doc_offsets, int num_docs, void *stream) {
    // Every argument check comes before the first CUDA call.
    attn_status_t s = check_bwd_args(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Sq, Sk, D,
                                     scale, window_left, window_right, doc_offsets, num_docs);
    if (s != ATTN_OK) return s;
    const long long rows = (long long)B * Hq * Sq;
    if (rows > (long long)kNoAllocRows)
        return fail(ATTN_ERR_UNSUPPORTED,
                    "attn_bwd_noalloc: B*Hq*Sq = %lld rows exceeds the built-in scratch of "
                    "%zu rows; use attn_bwd with a workspace",
                    rows, kNoAllocRows);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(ATTN_ERR_UNSUPPORTED, "device index %d", dev);
    // Once per device, with that device current: the host-side name of the
    // array is not a device address; look the address up.
    NoAllocScratch &sc = g_noalloc[dev];
    std::call_once(sc.once, [&]() { sc.err = cudaGetSymbolAddress(&sc.ptr, g_noalloc_scratch); });
    if (sc.err != cudaSuccess || sc.ptr == nullptr)
        return fail(ATTN_ERR_CUDA, "scratch address lookup: %s", cudaGetErrorString(sc.err));
    return attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Sq, Sk, D, scale, causal,
                    window_left, window_right, doc_offsets, num_docs, sc.ptr,
                    kNoAllocRows * sizeof(float), stream);
}

attn_status_t attn_get_device_status(void *stream) {
    DeviceState *st = nullptr;
    attn_status_t s = device_state(&st);
    if (s != ATTN_OK) return s;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "stream sync: %s", cudaGetErrorString(e));
    int word = 0;
    e = cudaMemcpy(&word, st->status, sizeof word, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
    if (word != 0) {
        const int zero = 0;
        e = cudaMemcpy(st->status, &zero, sizeof zero, cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "status clear: %s", cudaGetErrorString(e));
        return fail(static_cast<attn_status_t>(word), "device reported status %d", word);
    }
    return ok();
}

const char *attn_status_string(attn_status_t status) {
    switch (status) {
        case ATTN_OK: return "ok";
        case ATTN_ERR_INVALID_ARG: return "invalid argument";
        case ATTN_ERR_UNSUPPORTED: return "unsupported configuration";
        case ATTN_ERR_MISALIGNED: return "misaligned pointer";
        case ATTN_ERR_LAUNCH: return "kernel launch failed";
        case ATTN_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
        case ATTN_ERR_CUDA: return "CUDA runtime error";
        case ATTN_ERR_RANGE: return "input value outside the representable range";
    }
    return "unknown status";
}

const char *attn_last_error_detail(void) { return g_detail; }

int attn_abi_version(void) { return ATTN_ABI_VERSION; }

#ifdef ATTN_TRACE
// Trace builds only: device buffer of trace_ctas * 3 * 96 * 8 int64 for the
// clock64 event log of the first trace_ctas CTAs (NULL disables).
ATTN_API void attn_trace_set_buffer(long long *device_buffer, int trace_ctas) {
    g_trace = device_buffer;
    g_trace_ctas = device_buffer ? trace_ctas : 0;
}
#endif
#ifdef ATTN_COUNT_RESCALES
// Counting builds only: device buffer of 4 uint64 that the bf16 / fp8 / FP4
// forward kernels add their rescale statistics to (NULL disables); see
// FwdParams::rescale_counts.
ATTN_API void attn_count_set_buffer(unsigned long long *device_buffer) {
    g_rescale_counts = device_buffer;
}
#endif

}  // extern "C"
