// Weight-side kernels: the int4 device format (pack / dequant) and the offline
// converter W -> (q, s, z) of T W.
#include "common.cuh"
#include "kernels.h"

namespace paro {

// ---------------------------------------------------------------------------
// pack: one thread per 32-bit word of the device format (layout in common.cuh)
// ---------------------------------------------------------------------------
__global__ void pack_q_kernel(const uint8_t* __restrict__ q, uint32_t* __restrict__ qw, int in, int64_t nwords) {
    const int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (w >= nwords) return;
    const int nkb = in / 64;
    const int j = (int)(w & 3);
    const int lane = (int)((w >> 2) & 31);
    const int64_t blk = w >> 7;
    const int kb = (int)(blk % nkb);
    const int64_t rb = blk / nkb;
    const int g = lane >> 2, qd = lane & 3;
    const int k0 = kb * 64 + j * 16 + 4 * qd;
    const uint8_t* r0 = q + (rb * 16 + g) * (int64_t)in + k0;
    const uint8_t* r1 = r0 + 8 * (int64_t)in;
    // nibble slot -> (row, k offset): 0:(r0,0) 4:(r0,1) 1:(r0,2) 5:(r0,3) 2:(r1,0) 6:(r1,1) 3:(r1,2) 7:(r1,3)
    uint32_t word = 0;
    word |= (uint32_t)(r0[0] & 0xF) << 0;
    word |= (uint32_t)(r0[1] & 0xF) << 16;
    word |= (uint32_t)(r0[2] & 0xF) << 4;
    word |= (uint32_t)(r0[3] & 0xF) << 20;
    word |= (uint32_t)(r1[0] & 0xF) << 8;
    word |= (uint32_t)(r1[1] & 0xF) << 24;
    word |= (uint32_t)(r1[2] & 0xF) << 12;
    word |= (uint32_t)(r1[3] & 0xF) << 28;
    qw[w] = word;
}

// scales and zeros of G destination groups (of 128 or 64 channels); the
// logical s, z have Gsrc = G / rep groups per row (rep = 2 for groups of 256,
// whose scale and zero are repeated for both 128-channel halves)
__global__ void pack_meta_kernel(const uint16_t* __restrict__ s, const uint8_t* __restrict__ z,
                                 uint32_t* __restrict__ sp, uint8_t* __restrict__ zp, int G, int rep, int64_t n) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;   // (rb, gi, g)
    if (i >= n) return;
    const int Gp = G + (G & 1), Gsrc = G / rep;
    const int g = (int)(i & 7);
    const int64_t rg = i >> 3;
    const int gi = (int)(rg % G);
    const int64_t rb = rg / G;
    const int64_t r0 = rb * 16 + g, r1 = r0 + 8;
    const int gs = gi / rep;
    sp[i] = (uint32_t)s[r0 * Gsrc + gs] | ((uint32_t)s[r1 * Gsrc + gs] << 16);
    const uint8_t zb = (uint8_t)((z[r0 * Gsrc + gs] & 0xF) | ((z[r1 * Gsrc + gs] & 0xF) << 4));
    zp[(rb * Gp + gi) * 8 + g] = zb;
    if ((G & 1) && gi == G - 1) zp[(rb * Gp + G) * 8 + g] = 0;   // padding group
}

cudaError_t launch_pack(const uint8_t* q, const uint16_t* sc, const uint8_t* z, int64_t in, int64_t out, int group,
                        void* qw, void* scp, void* zp, cudaStream_t s) {
    const int64_t nwords = in * out / 8;
    if (nwords > 0)
        pack_q_kernel<<<(unsigned)((nwords + 255) / 256), 256, 0, s>>>(q, static_cast<uint32_t*>(qw), (int)in, nwords);
    const int rep = group == 256 ? 2 : 1;                      // group 256: stored as group 128
    const int G = (int)(in / (group == 256 ? 128 : group));
    const int64_t nm = (out / 16) * G * 8;
    if (nm > 0)
        pack_meta_kernel<<<(unsigned)((nm + 255) / 256), 256, 0, s>>>(sc, z, static_cast<uint32_t*>(scp),
                                                                      static_cast<uint8_t*>(zp), G, rep, nm);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// dequant: device format -> w_hat fp16 [out][in], with the same per-word
// conversion the GEMV and GEMM kernels use.
// ---------------------------------------------------------------------------
__global__ void dequant_kernel(const uint32_t* __restrict__ qw, const uint32_t* __restrict__ sp,
                               const uint8_t* __restrict__ zp, __half* __restrict__ W, int in, int gshift,
                               int64_t nwords) {
    const int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (w >= nwords) return;
    const int nkb = in / 64, G = nkb >> gshift;               // quantisation groups of 64 << gshift channels
    const int j = (int)(w & 3);
    const int lane = (int)((w >> 2) & 31);
    const int64_t blk = w >> 7;
    const int kb = (int)(blk % nkb);
    const int64_t rb = blk / nkb;
    const int g = lane >> 2, qd = lane & 3;
    const int gi = kb >> gshift;
    const int64_t mi = (rb * G + gi) * 8 + g;
    const int Gp = G + (G & 1);
    uint32_t sc0, sc1, h[4];
    const Zero2 zc = zero_consts(zp[(rb * Gp + gi) * 8 + g]);
    scale_pairs(sp[mi], sc0, sc1);
    dequant_word(qw[w], zc, sc0, sc1, h);
    const int k0 = kb * 64 + j * 16 + 4 * qd;
    __half* r0 = W + (rb * 16 + g) * (int64_t)in + k0;
    *reinterpret_cast<uint2*>(r0) = make_uint2(h[0], h[1]);
    *reinterpret_cast<uint2*>(r0 + 8 * (int64_t)in) = make_uint2(h[2], h[3]);
}

cudaError_t launch_dequant(const void* qw, const void* scp, const void* zp, int64_t in, int64_t out, int group,
                           void* W, cudaStream_t s) {
    const int64_t nwords = in * out / 8;
    if (nwords > 0)
        dequant_kernel<<<(unsigned)((nwords + 255) / 256), 256, 0, s>>>(
            static_cast<const uint32_t*>(qw), static_cast<const uint32_t*>(scp), static_cast<const uint8_t*>(zp),
            static_cast<__half*>(W), (int)in, group == 64 ? 0 : 1, nwords);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Offline converter: one warp per (output row, 128-input group), fp64
// (groups of 64: each half warp quantises one).
// W'[o, c] = (T W[o, :])_c: multiply by alpha, then layers t = 1..K with
// each channel becoming a * v + b * v_partner (two rounded products and one
// rounded sum, no fused multiply-add, the order a plain fp64 evaluation of the
// 2x2 formula uses). Then the per-group asymmetric RTN.
// ---------------------------------------------------------------------------
constexpr int kRot64BlockBytes = 128 + 128 * 16;

__global__ void __launch_bounds__(128) quantize_kernel(const __half* __restrict__ W, int in, int G, int K,
                                                       int half_groups, int64_t out,
                                                       const uint8_t* __restrict__ rotp64,
                                                       const double* __restrict__ alpha64,
                                                       uint8_t* __restrict__ q, uint16_t* __restrict__ sc,
                                                       uint8_t* __restrict__ z) {
    __shared__ double buf[4][128];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t task = (int64_t)blockIdx.x * 4 + warp;
    if (task >= out * G) return;
    const int gi = (int)(task % G);
    const int64_t o = task / G;
    const int c0 = gi * 128 + 4 * lane;
    const __half* wr = W + o * in + c0;
    double v[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) v[r] = __dmul_rn((double)__half2float(wr[r]), alpha64[c0 + r]);
    double* b = buf[warp];
    for (int t = 0; t < K; ++t) {
        const uint8_t* blk = rotp64 + ((size_t)t * G + gi) * kRot64BlockBytes;
        const uint32_t pw = reinterpret_cast<const uint32_t*>(blk)[lane];
        const double2* cf = reinterpret_cast<const double2*>(blk + 128) + 4 * lane;
#pragma unroll
        for (int r = 0; r < 4; ++r) b[4 * lane + r] = v[r];
        __syncwarp();
        double p[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) p[r] = b[(pw >> (8 * r)) & 0xFF];
        __syncwarp();
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const double2 ab = cf[r];
            v[r] = __dadd_rn(__dmul_rn(ab.x, v[r]), __dmul_rn(ab.y, p[r]));
        }
    }
    // min and max over the quantisation group: the whole warp (128
    // channels), or each half warp (64 channels) when half_groups is set
    double mn = fmin(fmin(v[0], v[1]), fmin(v[2], v[3]));
    double mx = fmax(fmax(v[0], v[1]), fmax(v[2], v[3]));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        if (half_groups && off == 16) continue;
        mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, off));
        mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    __half s16 = __double2half(__ddiv_rn(__dsub_rn(mx, mn), 15.0));
    double s = (double)__half2float(s16);
    const double floor_s = 6.103515625e-05;   // 2^-14, smallest normal fp16
    if (s < floor_s) {
        s = floor_s;
        s16 = __double2half(floor_s);
    }
    const double zd = fmin(fmax(rint(__ddiv_rn(-mn, s)), 0.0), 15.0);
    uint32_t packed = 0;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const double qd = fmin(fmax(__dadd_rn(rint(__ddiv_rn(v[r], s)), zd), 0.0), 15.0);
        packed |= (uint32_t)qd << (8 * r);
    }
    *reinterpret_cast<uint32_t*>(q + o * in + c0) = packed;
    if (half_groups) {                                     // groups of 64: two per warp
        if ((lane & 15) == 0) {
            const int64_t gq = o * (2 * G) + 2 * gi + (lane >> 4);
            sc[gq] = __half_as_ushort(s16);
            z[gq] = (uint8_t)zd;
        }
    } else if (lane == 0) {
        sc[o * G + gi] = __half_as_ushort(s16);
        z[o * G + gi] = (uint8_t)zd;
    }
}

// The same for 256-channel groups: one warp per (output row, group), lane L
// holding channels 8L..8L+7; fp64 blocks of 256 partner bytes + 256 (a, b).
__global__ void __launch_bounds__(128) quantize256_kernel(const __half* __restrict__ W, int in, int G, int K,
                                                          int64_t out, const uint8_t* __restrict__ rotp64,
                                                          const double* __restrict__ alpha64,
                                                          uint8_t* __restrict__ q, uint16_t* __restrict__ sc,
                                                          uint8_t* __restrict__ z) {
    constexpr int kBlk = 256 + 256 * 16;
    __shared__ double buf[4][256];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t task = (int64_t)blockIdx.x * 4 + warp;
    if (task >= out * G) return;
    const int gi = (int)(task % G);
    const int64_t o = task / G;
    const int c0 = gi * 256 + 8 * lane;
    const __half* wr = W + o * in + c0;
    double v[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) v[r] = __dmul_rn((double)__half2float(wr[r]), alpha64[c0 + r]);
    double* b = buf[warp];
    for (int t = 0; t < K; ++t) {
        const uint8_t* blk = rotp64 + ((size_t)t * G + gi) * kBlk;
        const uint2 pw = reinterpret_cast<const uint2*>(blk)[lane];
        const double2* cf = reinterpret_cast<const double2*>(blk + 256) + 8 * lane;
#pragma unroll
        for (int r = 0; r < 8; ++r) b[8 * lane + r] = v[r];
        __syncwarp();
        double p[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) p[r] = b[((r < 4 ? pw.x : pw.y) >> (8 * (r & 3))) & 0xFF];
        __syncwarp();
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const double2 ab = cf[r];
            v[r] = __dadd_rn(__dmul_rn(ab.x, v[r]), __dmul_rn(ab.y, p[r]));
        }
    }
    double mn = v[0], mx = v[0];
#pragma unroll
    for (int r = 1; r < 8; ++r) {
        mn = fmin(mn, v[r]);
        mx = fmax(mx, v[r]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, off));
        mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    __half s16 = __double2half(__ddiv_rn(__dsub_rn(mx, mn), 15.0));
    double sd = (double)__half2float(s16);
    const double floor_s = 6.103515625e-05;   // 2^-14, smallest normal fp16
    if (sd < floor_s) {
        sd = floor_s;
        s16 = __double2half(floor_s);
    }
    const double zd = fmin(fmax(rint(__ddiv_rn(-mn, sd)), 0.0), 15.0);
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const uint32_t qd = (uint32_t)fmin(fmax(__dadd_rn(rint(__ddiv_rn(v[r], sd)), zd), 0.0), 15.0);
        if (r < 4) lo |= qd << (8 * r);
        else hi |= qd << (8 * (r - 4));
    }
    *reinterpret_cast<uint2*>(q + o * in + c0) = make_uint2(lo, hi);
    if (lane == 0) {
        sc[o * G + gi] = __half_as_ushort(s16);
        z[o * G + gi] = (uint8_t)zd;
    }
}

cudaError_t launch_quantize(const RotDev& r, const void* W, int64_t out, uint8_t* q, uint16_t* sc, uint8_t* z,
                            cudaStream_t s) {
    if (r.group == 256) {
        const int64_t tasks = out * r.G;
        if (tasks > 0)
            quantize256_kernel<<<(unsigned)((tasks + 3) / 4), 128, 0, s>>>(static_cast<const __half*>(W), (int)r.in,
                                                                           r.G, r.K, out, r.rotp64, r.alpha64, q, sc, z);
        return cudaGetLastError();
    }
    const int64_t tasks = out * r.G;
    if (tasks > 0)
        quantize_kernel<<<(unsigned)((tasks + 3) / 4), 128, 0, s>>>(static_cast<const __half*>(W), (int)r.in, r.G,
                                                                    r.K, r.group == 64 ? 1 : 0, out, r.rotp64,
                                                                    r.alpha64, q, sc, z);
    return cudaGetLastError();
}

}  // namespace paro
