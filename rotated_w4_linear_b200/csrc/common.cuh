// Shared device helpers for the sm_100a kernels of the rotated W4G128 layer.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#define PARO_GROUP 128

namespace paro {

// ---------------------------------------------------------------------------
// Prepared rotation parameters ("rotation block", host image from which the
// quad exchange blocks below are built), one per (layer t, group g), 1152
// bytes: 128 partner bytes, then 128 float2 (a, b).
// Channel c of the group becomes a * v[c] + b * v[partner[c]]:
//   first channel i of a pair (i, j, th): a = cos th, b = -sin th, partner j
//   second channel j:                     a = cos th, b = +sin th, partner i
//   channel in no pair:                   a = 1,      b = 0,       partner c
// which is the 2x2 Givens matrix of the ParoQuant CSDN article (section 2.2)
// written per output channel.
// ---------------------------------------------------------------------------
constexpr int kRotBlockBytes = 128 + 128 * 8;

// ---------------------------------------------------------------------------
// Quad exchange blocks for the decode rotation kernel, one per
// (layer t, group g), 1280 B:
//   [32 lanes][8 bytes]: float4-slot indices (0..127) in the warp's 2 KB
//     exchange buffer where lane L stores channel 4L+j (bytes 0..3, bit 7
//     set when the channel is in a pair of this layer) and where it loads
//     that channel's partner (bytes 4..7); a slot holds four tokens. A
//     channel in no pair (partial matchings) skips the exchange: its own
//     value stands in for the partner, as in the rotation block (a = 1, b = 0);
//   [32 lanes][float4]: (a, b) of channels 4L and 4L+1, as in the rotation block;
//   [32 lanes][float4]: (a, b) of channels 4L+2 and 4L+3.
// A 16-byte shared access is served a quarter-warp (8 lanes) at a time; the
// host gives the 8 lanes of every quarter distinct slots modulo 8 for each
// store and each load (a proper 8-edge-colouring of the 16 x 16 bipartite
// multigraph "store quarter-slot -> load quarter-slot", regular of degree
// 8), so no access has a bank conflict.
// ---------------------------------------------------------------------------
constexpr int kRotQBlockBytes = 32 * 8 + 128 * 8;

__device__ __forceinline__ const uint8_t* rotq_block(const uint8_t* rotq, int t, int g, int G) {
    return rotq + ((size_t)t * G + g) * kRotQBlockBytes;
}

// Two fp32 lanes in one 64-bit register pair (sm_100 packed f32x2 arithmetic).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 f2_unpack(uint64_t v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// ---------------------------------------------------------------------------
// int4 weight format (Kernel 4). For row block rb (16 output rows) and 64-wide
// k block kb, 512 bytes: lane L (g = L >> 2, q = L & 3) owns 16 bytes = 4 words,
// word j covering the 16x16 tile k in [64 kb + 16 j, +16). The word's nibbles:
//   n0 (g,   4q)   n4 (g,   4q+1)   n1 (g,   4q+2)   n5 (g,   4q+3)
//   n2 (g+8, 4q)   n6 (g+8, 4q+1)   n3 (g+8, 4q+2)   n7 (g+8, 4q+3)
// (row within the block, k within the tile). Nibbles i and i+4 sit 16 bits
// apart, so one LOP3 turns them into the fp16 pair (1024 + n_i, 1024 + n_i+4).
// Scales: uint32 [out/16][G][8], word g = (s[row g] | s[row g+8] << 16).
// Zeros:  uint8  [out/16][Gp][8] with Gp = G rounded up to even (two groups'
//         zeros form one aligned 16-byte copy), byte g = (z[row g] | z[row g+8] << 4).
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t hsub2_rn(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ uint32_t hmul2_rn(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ uint32_t hfma2_rn(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t r;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t w, uint32_t mask, uint32_t bits) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(w), "r"(mask), "r"(bits));
    return r;
}

// Per-row zero constants from the zero byte (z0 | z1 << 4), as fp16x2 pairs:
//   zb = (1024 + z, 1024 + z)   subtracted from (1024 + q)
//   zc = -(64 + z, 64 + z)      added to (1024 + 16 q) / 16
struct Zero2 {
    uint32_t zb0, zc0, zb1, zc1;
};
__device__ __forceinline__ Zero2 zero_consts(uint32_t zbyte) {
    const uint32_t t = __byte_perm(zbyte, 0u, 0x4040);     // the byte at bits 0-7 and 16-23
    Zero2 r;
    r.zb0 = lop3_and_or(t, 0x000F000Fu, 0x64006400u);
    r.zb1 = lop3_and_or(t >> 4, 0x000F000Fu, 0x64006400u);
    r.zc0 = lop3_and_or(t << 4, 0x00F000F0u, 0xD400D400u);
    r.zc1 = lop3_and_or(t, 0x00F000F0u, 0xD400D400u);
    return r;
}


// scale word (s0 | s1 << 16) -> (s0, s0) and (s1, s1)
__device__ __forceinline__ void scale_pairs(uint32_t sw, uint32_t& sc0, uint32_t& sc1) {
    sc0 = __byte_perm(sw, sw, 0x1010);
    sc1 = __byte_perm(sw, sw, 0x3232);
}

// One packed word -> four fp16x2 of w_hat = fp16((q - z) * s):
//   h[0] = (g,   k0, k0+1)   h[1] = (g,   k0+2, k0+3)
//   h[2] = (g+8, k0, k0+1)   h[3] = (g+8, k0+2, k0+3)
// Nibbles at bits 0-3 / 16-19 become 1024 + q under mask 0x000f000f, and
// (1024 + q) - (1024 + z) = q - z exactly. Nibbles at bits 4-7 / 20-23 become
// 1024 + 16 q under mask 0x00f000f0 (still inside the fp16 mantissa), and one
// fma (1024 + 16 q) * 1/16 - (64 + z) = q - z is exact as well. One shift by
// 8 serves the upper byte of each half. The product with s is rounded once.
__device__ __forceinline__ void dequant_word(uint32_t w, const Zero2& z, uint32_t sc0, uint32_t sc1,
                                             uint32_t h[4]) {
    const uint32_t kMagic = 0x64006400u, kSixteenth = 0x2C002C00u;   // fp16x2 1024, 1/16
    const uint32_t w8 = w >> 8;
    h[0] = hmul2_rn(hsub2_rn(lop3_and_or(w, 0x000F000Fu, kMagic), z.zb0), sc0);
    h[1] = hmul2_rn(hfma2_rn(lop3_and_or(w, 0x00F000F0u, kMagic), kSixteenth, z.zc0), sc0);
    h[2] = hmul2_rn(hsub2_rn(lop3_and_or(w8, 0x000F000Fu, kMagic), z.zb1), sc1);
    h[3] = hmul2_rn(hfma2_rn(lop3_and_or(w8, 0x00F000F0u, kMagic), kSixteenth, z.zc1), sc1);
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint32_t lds8(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}


__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace paro
