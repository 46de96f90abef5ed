// One warp's share of the decode rotation X' = X T^-1 (ParoQuant CSDN
// article, section 2.1; the online rotation of section 3.1): four token rows
// of one 128-channel group, divided by alpha, then K layers of independent
// Givens pairs, fp32 in registers, fp16 out (the decode rotation kernel,
// rotate.cu).
//
// Lane L holds channels 4L..4L+3 of the four rows. Each layer, channels in a
// pair store their values (one float4 slot = one channel, four tokens) into a
// warp-private 2 KB exchange buffer at a host-chosen position and load their
// partner's, with no bank conflict (the quad exchange blocks of common.cuh);
// two tokens are updated per packed f32x2 multiply and fma. The operations
// and their order do not depend on the batch, so a row's X' does not either.
#pragma once

#include "common.cuh"

namespace paro {

// X of rows t0..t0+3 (zero past T), channels g*128 + 4 lane .. +3, fp16.
__device__ __forceinline__ void givens_load_quad(const __half* __restrict__ X, int T, int in, int g, int t0, int lane,
                                                 uint2 (&raw)[4]) {
    const int c0 = g * 128 + 4 * lane;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        raw[i] = make_uint2(0u, 0u);
        if (t0 + i < T) raw[i] = __ldg(reinterpret_cast<const uint2*>(X + (size_t)(t0 + i) * in + c0));
    }
}

// Rotate the quad loaded by givens_load_quad and store rows < T of X'.
//   prm   the group's K quad exchange blocks, in shared memory
//   xbuf  the warp's 2 KB exchange buffer (shared-space address)
//   ia    1/alpha of the lane's four channels
//   PF    each layer's table entries are loaded during the layer before
//         (the exchange's asm statements are compiler barriers, so the
//         loads are placed by hand), taking their latency off the chain
//         store -> warp barrier -> load -> fma of a layer
//   lane_major  each 64-channel block of X' is written in the order the
//         decode kernel's B fragments read it: channel 16 j + 4 q + e at
//         position 16 q + 4 j + e (the same values, other places)
template <bool PF>
__device__ __forceinline__ void givens_rotate_quad(const unsigned char* prm, uint32_t xbuf, int K,
                                                   const uint2 (&raw)[4], float4 ia, __half* __restrict__ Xr, int T,
                                                   int in, int g, int t0, int lane, bool lane_major) {
    uint64_t v[4][2];                                      // [channel j][token pair]
    {
        float x[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&raw[i].x));
            const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&raw[i].y));
            x[i][0] = lo.x * ia.x;
            x[i][1] = lo.y * ia.y;
            x[i][2] = hi.x * ia.z;
            x[i][3] = hi.y * ia.w;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[j][0] = f2_pack(x[0][j], x[1][j]);
            v[j][1] = f2_pack(x[2][j], x[3][j]);
        }
    }
    uint2 pos = make_uint2(0u, 0u);
    float4 c01 = make_float4(0.f, 0.f, 0.f, 0.f), c23 = c01;
    if (PF && K > 0) {
        pos = *reinterpret_cast<const uint2*>(prm + 8 * lane);
        c01 = *reinterpret_cast<const float4*>(prm + 256 + 16 * lane);
        c23 = *reinterpret_cast<const float4*>(prm + 768 + 16 * lane);
    }
    for (int t = 0; t < K; ++t) {
        const unsigned char* blk = prm + (size_t)t * kRotQBlockBytes;
        if (!PF) {
            pos = *reinterpret_cast<const uint2*>(blk + 8 * lane);
            c01 = *reinterpret_cast<const float4*>(blk + 256 + 16 * lane);
            c23 = *reinterpret_cast<const float4*>(blk + 768 + 16 * lane);
        }
        uint2 pos_n = pos;
        float4 c01_n = c01, c23_n = c23;
        if (PF && t + 1 < K) {
            pos_n = *reinterpret_cast<const uint2*>(blk + kRotQBlockBytes + 8 * lane);
            c01_n = *reinterpret_cast<const float4*>(blk + kRotQBlockBytes + 256 + 16 * lane);
            c23_n = *reinterpret_cast<const float4*>(blk + kRotQBlockBytes + 768 + 16 * lane);
        }
        const float ca[4] = {c01.x, c01.z, c23.x, c23.z}, cb[4] = {c01.y, c01.w, c23.y, c23.w};
        uint32_t st[4], ld[4];
        bool act[4];                                       // channel in a pair of this layer
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            st[j] = 16u * ((pos.x >> (8 * j)) & 0x7Fu);
            ld[j] = 16u * ((pos.y >> (8 * j)) & 0x7Fu);
            act[j] = (pos.x >> (8 * j + 7)) & 1u;
        }
        // only channels in a pair go through shared memory (lanes with
        // inactive channels drop out of those accesses)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (act[j])
                asm volatile("st.shared.v2.b64 [%0], {%1, %2};" ::"r"(xbuf + st[j]), "l"(v[j][0]), "l"(v[j][1])
                             : "memory");
        __syncwarp();
        uint64_t p[4][2];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            p[j][0] = v[j][0];
            p[j][1] = v[j][1];
            if (act[j])
                asm volatile("ld.shared.v2.b64 {%0, %1}, [%2];" : "=l"(p[j][0]), "=l"(p[j][1]) : "r"(xbuf + ld[j])
                             : "memory");
        }
        __syncwarp();                                      // the buffer is rewritten next layer
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint64_t a2 = f2_pack(ca[j], ca[j]), b2 = f2_pack(cb[j], cb[j]);
#pragma unroll
            for (int h = 0; h < 2; ++h) v[j][h] = f2_fma(b2, p[j][h], f2_mul(a2, v[j][h]));
        }
        pos = pos_n;
        c01 = c01_n;
        c23 = c23_n;
    }
    // lane L holds channels 4L..4L+3 = 64 b + 16 j + 4 q + (0..3) with L = 16 b + 4 j + q
    const int piece = lane_major ? ((lane & 16) | ((lane & 3) << 2) | ((lane >> 2) & 3)) : lane;
    const int c0 = g * 128 + 4 * piece;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const float2 w0 = f2_unpack(v[0][h]), w1 = f2_unpack(v[1][h]);
        const float2 w2 = f2_unpack(v[2][h]), w3 = f2_unpack(v[3][h]);
        const int t = t0 + 2 * h;
        if (t < T)
            *reinterpret_cast<uint2*>(Xr + (size_t)t * in + c0) =
                make_uint2(pack_half2(w0.x, w1.x), pack_half2(w2.x, w3.x));
        if (t + 1 < T)
            *reinterpret_cast<uint2*>(Xr + (size_t)(t + 1) * in + c0) =
                make_uint2(pack_half2(w0.y, w1.y), pack_half2(w2.y, w3.y));
    }
}

}  // namespace paro
