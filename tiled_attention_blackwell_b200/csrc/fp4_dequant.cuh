// FP4 inputs of the Direct-P forward, widened to f16.
//
// "Hardware-Aware FP4 FlashAttention-4", "Metodología", item 1, selects
// NVFP4 for Q and K and MXFP4 for V.  Every value of either format is
// exactly representable in f16 within the ranges checked below, so the
// attention kernel can run its products on the f16 tensor-core path and get
// exactly the products of the FP4 values (the per-tensor factors are applied
// outside: Q's and K's in the score scale, V's in the epilogue).
//
//   NVFP4: codes [rows][D/2] (element 2j in the low nibble), one e4m3 scale
//          byte per 16 elements of a row; value = e4m3(scale) * e2m1(code).
//          e4m3 * E2M1 has at most 6 significant bits and lies in
//          [2^-10, 2688]: exact in f16.
//   MXFP4: codes as above for V [B][S][H][D]; one UE8M0 byte u per 32 keys
//          of each (b, h, d) column, scales [B][ceil(S/32)][H][D];
//          value = 2^(u - 127) * e2m1(code), exact in f16 (and in its normal
//          range) for u - 127 in [-13, 13].
// A nonzero code whose scale is NaN, negative (NVFP4: the scale is an
// unsigned magnitude) or outside that range (MXFP4) is written as 0 and
// makes the kernel record ATTN_ERR_RANGE in the device status word.
#pragma once

#include "common.cuh"

namespace tab {

// One tensor of the widening pass.
struct Fp4DequantJob {
    const uint8_t *codes;   // [rows][D/2]
    const uint8_t *scales;  // NVFP4: [rows][D/16]; MXFP4: [B][ceil(S/32)][H][D]
    uint32_t *out;          // f16 pairs, [rows][D/2]
    long long groups;       // 32-element groups: rows * D / 32
    int S, H;               // MXFP4 scale layout
    int mx;                 // 0: NVFP4, 1: MXFP4 along keys
};

// Q, K and V in one launch: the groups of the three jobs are numbered one
// after the other.
struct Fp4DequantParams {
    Fp4DequantJob job[3];
    int D;
    int *status;
};

// Four bytes of codes (eight E2M1 values, element 2j in the low nibble of
// byte j) to four f16 pairs.
__device__ __forceinline__ void e2m1x8_to_f16x2x4(uint32_t w, uint32_t *out) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3])
        : "r"(w));
}

// f16 pair of two e4m3 bytes (low byte -> low half).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
    uint32_t r;
    asm("{\n\t.reg .b16 h;\n\t"
        "cvt.u16.u32 h, %1;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, h;\n\t}"
        : "=r"(r)
        : "r"(two));
    return r;
}

// 2^(u - 127) as f16 bits for u in [114, 140] (else 0, and *bad is set when
// the code it scales is nonzero).
__device__ __forceinline__ uint32_t ue8m0_f16(uint32_t u, bool nonzero_code, bool &bad) {
    const bool ok = u - 114u <= 26u;
    bad |= !ok && nonzero_code;
    return ok ? (u - 112u) << 10 : 0u;
}

__global__ void __launch_bounds__(256) fp4_dequant_kernel(const __grid_constant__ Fp4DequantParams p) {
    const long long g0 = p.job[0].groups, g1 = p.job[1].groups;
    const long long total = g0 + g1 + p.job[2].groups;
    const long long stride = (long long)gridDim.x * blockDim.x;
    bool bad = false;
    for (long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x; g < total; g += stride) {
        const int jb = g < g0 ? 0 : (g < g0 + g1 ? 1 : 2);
        const long long gg = g - (jb == 0 ? 0 : (jb == 1 ? g0 : g0 + g1));
        const Fp4DequantJob &J = p.job[jb];
        const uint4 cw = *reinterpret_cast<const uint4 *>(J.codes + gg * 16);
        const uint32_t cws[4] = {cw.x, cw.y, cw.z, cw.w};
        uint32_t w[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) e2m1x8_to_f16x2x4(cws[q], w + 4 * q);
        if (!J.mx) {
            // two e4m3 scales, one per 16 elements
            const uint32_t s2 = *reinterpret_cast<const uint16_t *>(J.scales + gg * 2);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const uint32_t sb = (s2 >> (8 * half)) & 0xFFu;
                const uint32_t scale2 = e4m3x2_to_f16x2(sb | (sb << 8));
                // NaN, or negative with a nonzero magnitude: outside the format
                // (the scale is an unsigned e4m3 magnitude; -0 scales to zero).
                const bool bad_scale = (sb & 0x7Fu) == 0x7Fu || sb > 0x80u;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t byte = (cws[2 * half + (k >> 2)] >> (8 * (k & 3))) & 0xFFu;
                    bad |= bad_scale && (byte & 0x77u) != 0u;
                    w[8 * half + k] = bad_scale ? 0u : hmul2_u32(w[8 * half + k], scale2);
                }
            }
        } else {
            // one UE8M0 scale per element, from the 32-key block of its column
            const long long t0 = gg * 32;
            const long long row = t0 / p.D;
            const int d0 = (int)(t0 - row * p.D);
            const int h = (int)(row % J.H);
            const long long bj = row / J.H;
            const int j = (int)(bj % J.S);
            const long long b = bj / J.S;
            const long long nblk = (J.S + 31) / 32;
            const uint4 *sp = reinterpret_cast<const uint4 *>(
                J.scales + ((b * nblk + j / 32) * J.H + h) * (long long)p.D + d0);
            const uint4 sa = sp[0], sb4 = sp[1];
            const uint32_t sw[8] = {sa.x, sa.y, sa.z, sa.w, sb4.x, sb4.y, sb4.z, sb4.w};
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const uint32_t byte = (cws[k >> 2] >> (8 * (k & 3))) & 0xFFu;
                const uint32_t u0 = (sw[k >> 1] >> (16 * (k & 1))) & 0xFFu;
                const uint32_t u1 = (sw[k >> 1] >> (16 * (k & 1) + 8)) & 0xFFu;
                const uint32_t sc = ue8m0_f16(u0, (byte & 0x07u) != 0u, bad) |
                                    (ue8m0_f16(u1, (byte & 0x70u) != 0u, bad) << 16);
                w[k] = hmul2_u32(w[k], sc);
            }
        }
        uint4 *dst = reinterpret_cast<uint4 *>(J.out + gg * 16);
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
    }
    if (bad) atomicCAS(p.status, 0, kStatusRange);
}

}  // namespace tab
