// Operand preparation of the block-scaled FP4 Direct-P forward.
//
// "Hardware-Aware FP4 FlashAttention-4", "Metodología", item 1, runs both
// products on the FP4 tensor cores: Q K^T with NVFP4 operands (E2M1 codes,
// one e4m3 scale per 16 elements along D) and P V with MXFP4 operands (one
// UE8M0 scale per 32 keys).  The tensor cores read the codes straight from
// shared memory (Q and K as the caller stores them, D contiguous) and the
// scales from tensor memory, so this pass only
//   - lays the scales out as the 512-byte atoms that tcgen05.cp copies into
//     tensor memory: per 128-row tile and K step of 64 elements, row m's
//     four scale bytes at 16 (m % 32) + 4 (m / 32);
//   - transposes V's codes so the keys are contiguous (the K dimension of
//     P V; FP4 operands must be K-major): vt [B][Hkv][D][nkt * 64 bytes],
//     zero past Sk.
// Out-of-format inputs read as 0 and record ATTN_ERR_RANGE when a nonzero
// code depends on them, as in the widening path: an NVFP4 scale that is NaN
// or negative (the tensor cores' scale is an unsigned e4m3 magnitude; -0 is
// a zero scale), a V scale with u - 127 outside [-13, 13].
#pragma once

#include "common.cuh"

namespace tab {

constexpr int kSfAtom = 512;  // bytes: 128 rows x 4 scale bytes

struct Fp4PrepParams {
    const uint8_t *q_codes, *q_scales, *k_codes, *k_scales;  // [B][S][H][64], [B][S][H][8]
    const uint8_t *v_codes, *v_scales;  // [B][Sk][Hkv][64], [B][ceil(Sk/32)][Hkv][128]
    uint8_t *sf_q;  // [B][Hq][nqt][2][512]
    uint8_t *sf_k;  // [B][Hkv][nkt][2][512]
    uint8_t *sf_v;  // [B][Hkv][nkt][2][512]
    uint8_t *vt;    // [B][Hkv][128][nkt * 64]
    int B, Hq, Hkv, Sq, Sk, nqt, nkt;
    int v_ctas;     // the first v_ctas CTAs transpose V, one (b, h, key tile) each
    int *status;
};

// An NVFP4 scale byte as the tensor cores read it (UE4M3), with the check
// of the 16 codes it scales when it is out of format.
__device__ __forceinline__ uint32_t nvfp4_scale(uint32_t sb, const uint8_t *codes16, bool &bad) {
    const bool nan = (sb & 0x7Fu) == 0x7Fu;
    const bool neg = sb > 0x80u;  // sign set, nonzero magnitude
    if (!(nan || neg)) return sb & 0x7Fu;  // -0 -> 0
    const uint2 c = *reinterpret_cast<const uint2 *>(codes16);
    bad |= ((c.x | c.y) & 0x77777777u) != 0u;
    return 0u;
}

// 4 x 4 byte transpose: out[q] byte p = x[p] byte q.
__device__ __forceinline__ void byte_transpose4(const uint32_t *x, uint32_t *out) {
    const uint32_t t0 = __byte_perm(x[0], x[1], 0x5140), t1 = __byte_perm(x[0], x[1], 0x7362);
    const uint32_t t2 = __byte_perm(x[2], x[3], 0x5140), t3 = __byte_perm(x[2], x[3], 0x7362);
    out[0] = __byte_perm(t0, t2, 0x5410);
    out[1] = __byte_perm(t0, t2, 0x7632);
    out[2] = __byte_perm(t1, t3, 0x5410);
    out[3] = __byte_perm(t1, t3, 0x7632);
}

__global__ void __launch_bounds__(256) fp4_prepare_kernel(const __grid_constant__ Fp4PrepParams p) {
    constexpr int kRow = 68;  // padded row of the key tile (bytes): 2-way bank conflicts at most
    __shared__ __align__(16) uint8_t tile[128 * kRow];
    __shared__ uint32_t us[4][128];
    bool bad = false;
    const int t = threadIdx.x;
    if ((int)blockIdx.x < p.v_ctas) {
        // ---- V: one (b, h, 128-key tile)
        const int kt = (int)blockIdx.x % p.nkt;
        const int bh = (int)blockIdx.x / p.nkt;
        const int h = bh % p.Hkv, b = bh / p.Hkv;
        const int nb32 = (p.Sk + 31) / 32;
        for (int idx = t; idx < 512; idx += 256) {
            const int key = idx >> 2, c = idx & 3;
            const int kg = kt * 128 + key;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (kg < p.Sk)
                v = *reinterpret_cast<const uint4 *>(
                    p.v_codes + (((size_t)b * p.Sk + kg) * p.Hkv + h) * 64 + c * 16);
            uint32_t *row = reinterpret_cast<uint32_t *>(tile + key * kRow + c * 16);
            row[0] = v.x;
            row[1] = v.y;
            row[2] = v.z;
            row[3] = v.w;
            const int sb = idx >> 7, d = idx & 127;
            const int blk = kt * 4 + sb;
            us[sb][d] = blk < nb32 ? p.v_scales[(((size_t)b * nb32 + blk) * p.Hkv + h) * 128 + d]
                                   : 127u;
        }
        __syncthreads();
        // Thread: keys [8 kq, 8 kq + 8) x dims [8 dq, 8 dq + 8).  Input word x:
        // dims 8 dq .. 8 dq + 7 of key 8 kq + x; per key pair a 2 x 2 nibble
        // swap gives the even-dim and odd-dim bytes, then a 4 x 4 byte
        // transpose gives output row d = 8 dq + e (keys 8 kq .. 8 kq + 7).
        const int w = t >> 5, l = t & 31;
        const int kq = 8 * (w & 1) + (l >> 2), dq = 4 * (w >> 1) + (l & 3);
        uint32_t ev[4], od[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t A = *reinterpret_cast<const uint32_t *>(tile + (8 * kq + 2 * q) * kRow + 4 * dq);
            const uint32_t B = *reinterpret_cast<const uint32_t *>(tile + (8 * kq + 2 * q + 1) * kRow + 4 * dq);
            ev[q] = (A & 0x0F0F0F0Fu) | ((B & 0x0F0F0F0Fu) << 4);
            od[q] = ((A >> 4) & 0x0F0F0F0Fu) | (B & 0xF0F0F0F0u);
        }
        uint32_t evt[4], odt[4];
        byte_transpose4(ev, evt);
        byte_transpose4(od, odt);
        const int sb = kq >> 2;  // the 32-key block of these 8 keys
        uint8_t *vrow = p.vt + (((size_t)b * p.Hkv + h) * 128 + 8 * dq) * ((size_t)p.nkt * 64) + kt * 64 + 4 * kq;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            uint32_t word = (e & 1) ? odt[e >> 1] : evt[e >> 1];
            if (us[sb][8 * dq + e] - 114u > 26u) {  // scale out of range: the codes read as 0
                bad |= (word & 0x77777777u) != 0u;
                word = 0u;
            }
            *reinterpret_cast<uint32_t *>(vrow + (size_t)e * p.nkt * 64) = word;
        }
        if (t < 128) {
            uint8_t *atom = p.sf_v + (((size_t)b * p.Hkv + h) * p.nkt + kt) * (2 * kSfAtom);
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                uint32_t u0 = us[2 * ks][t], u1 = us[2 * ks + 1][t];
                u0 = u0 - 114u <= 26u ? u0 : 127u;  // its codes were zeroed
                u1 = u1 - 114u <= 26u ? u1 : 127u;
                *reinterpret_cast<uint32_t *>(atom + ks * kSfAtom + 16 * (t & 31) + 4 * (t >> 5)) =
                    u0 | (u1 << 8);
            }
        }
    } else {
        // ---- Q and K scale atoms: one thread per (b, h, tile, row)
        const long long nq = (long long)p.B * p.Hq * p.nqt * 128;
        const long long nk = (long long)p.B * p.Hkv * p.nkt * 128;
        const long long stride = (long long)(gridDim.x - p.v_ctas) * blockDim.x;
        for (long long g = (long long)(blockIdx.x - p.v_ctas) * blockDim.x + t; g < nq + nk;
             g += stride) {
            const bool isq = g < nq;
            const long long gg = isq ? g : g - nq;
            const int H = isq ? p.Hq : p.Hkv, S = isq ? p.Sq : p.Sk, nt = isq ? p.nqt : p.nkt;
            const uint8_t *scales = isq ? p.q_scales : p.k_scales;
            const uint8_t *codes = isq ? p.q_codes : p.k_codes;
            uint8_t *out = isq ? p.sf_q : p.sf_k;
            const int m = (int)(gg & 127);
            const long long tt = gg >> 7;  // (b, h, tile)
            const int tile_i = (int)(tt % nt);
            const long long bh = tt / nt;
            const int h = (int)(bh % H), b = (int)(bh / H);
            const int r = tile_i * 128 + m;
            uint32_t w0 = 0u, w1 = 0u;
            if (r < S) {
                const size_t row = ((size_t)b * S + r) * H + h;
                const uint2 sc = *reinterpret_cast<const uint2 *>(scales + row * 8);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    w0 |= nvfp4_scale((sc.x >> (8 * e)) & 0xFFu, codes + row * 64 + e * 8, bad) << (8 * e);
                    w1 |= nvfp4_scale((sc.y >> (8 * e)) & 0xFFu, codes + row * 64 + 32 + e * 8, bad)
                          << (8 * e);
                }
            }
            uint8_t *atom = out + (size_t)tt * (2 * kSfAtom) + 16 * (m & 31) + 4 * (m >> 5);
            *reinterpret_cast<uint32_t *>(atom) = w0;
            *reinterpret_cast<uint32_t *>(atom + kSfAtom) = w1;
        }
    }
    if (bad) atomicCAS(p.status, 0, kStatusRange);
}

}  // namespace tab
