// Activation rotation X' = X T^-1 (ParoQuant CSDN article, section 2.1; the
// online rotation kernel of section 3.1): per token row and 128-channel group,
// divide by alpha, then K layers of independent Givens pairs, fp32 in
// registers, fp16 out.
//
// Mapping: one warp owns one (group, token tile). Lane L holds channels
// 4L..4L+3 of TT tokens, loaded as one 8-byte vector per token (a warp reads
// 256 contiguous bytes per row). Partner values are exchanged through a
// warp-private shared-memory row per token each layer, at positions chosen on
// the host so that every store and load is bank-conflict-free; the next
// layer's positions and coefficients are loaded while the current one runs.
#include "common.cuh"
#include "kernels.h"

namespace paro {

template <int TT>
__global__ void __launch_bounds__(128) rotate_kernel(const __half* __restrict__ X, __half* __restrict__ Xr,
                                                     int64_t T, int in, int G, int K,
                                                     const uint8_t* __restrict__ rotx,
                                                     const float* __restrict__ inv_alpha) {
    // a kernel launched after this one on the stream may start now; it waits
    // for this grid's completion before it reads Xr
    asm volatile("griddepcontrol.launch_dependents;");
    __shared__ __align__(16) float buf[4][TT][128];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t task = (int64_t)blockIdx.x * 4 + warp;
    const int g = (int)(task % G);
    const int64_t t0 = (task / G) * TT;
    if (t0 >= T) return;
    const int c0 = g * 128 + 4 * lane;

    const float4 ia = __ldg(reinterpret_cast<const float4*>(inv_alpha + c0));
    float v[TT][4];
#pragma unroll
    for (int i = 0; i < TT; ++i) {
        uint2 raw = make_uint2(0u, 0u);
        if (t0 + i < T) raw = __ldg(reinterpret_cast<const uint2*>(X + (t0 + i) * in + c0));
        const float2 lo = __half22float2(*reinterpret_cast<__half2*>(&raw.x));
        const float2 hi = __half22float2(*reinterpret_cast<__half2*>(&raw.y));
        v[i][0] = lo.x * ia.x;
        v[i][1] = lo.y * ia.y;
        v[i][2] = hi.x * ia.z;
        v[i][3] = hi.y * ia.w;
    }

    // Each layer: every lane stores its 4 channels at the layer's positions
    // in the warp's exchange rows (one 512-byte row per token), then loads
    // the 4 partners; positions make every access bank-conflict-free.
    float* row0 = &buf[warp][0][0];
    uint4 off = make_uint4(0u, 0u, 0u, 0u);
    float4 c01 = make_float4(1.f, 0.f, 1.f, 0.f), c23 = c01;
    if (K > 0) {
        const uint8_t* blk = rotx_block(rotx, 0, g, G);
        off = __ldg(reinterpret_cast<const uint4*>(blk) + lane);
        c01 = __ldg(reinterpret_cast<const float4*>(blk + 512) + 2 * lane);
        c23 = __ldg(reinterpret_cast<const float4*>(blk + 512) + 2 * lane + 1);
    }
    for (int t = 0; t < K; ++t) {
        uint4 off_n = off;
        float4 c01_n = c01, c23_n = c23;
        if (t + 1 < K) {                                   // next layer's parameters in flight
            const uint8_t* blk = rotx_block(rotx, t + 1, g, G);
            off_n = __ldg(reinterpret_cast<const uint4*>(blk) + lane);
            c01_n = __ldg(reinterpret_cast<const float4*>(blk + 512) + 2 * lane);
            c23_n = __ldg(reinterpret_cast<const float4*>(blk + 512) + 2 * lane + 1);
        }
        // byte offsets -> float indices into the token-0 row; token i adds 128 i
        float* w0 = row0 + ((off.x & 0xFFFFu) >> 2);
        float* w1 = row0 + (off.x >> 18);
        float* w2 = row0 + ((off.y & 0xFFFFu) >> 2);
        float* w3 = row0 + (off.y >> 18);
        const float* r0 = row0 + ((off.z & 0xFFFFu) >> 2);
        const float* r1 = row0 + (off.z >> 18);
        const float* r2 = row0 + ((off.w & 0xFFFFu) >> 2);
        const float* r3 = row0 + (off.w >> 18);
#pragma unroll
        for (int i = 0; i < TT; ++i) {
            w0[i * 128] = v[i][0];
            w1[i * 128] = v[i][1];
            w2[i * 128] = v[i][2];
            w3[i * 128] = v[i][3];
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < TT; ++i) {
            const float q0 = r0[i * 128], q1 = r1[i * 128], q2 = r2[i * 128], q3 = r3[i * 128];
            v[i][0] = fmaf(c01.y, q0, c01.x * v[i][0]);
            v[i][1] = fmaf(c01.w, q1, c01.z * v[i][1]);
            v[i][2] = fmaf(c23.y, q2, c23.x * v[i][2]);
            v[i][3] = fmaf(c23.w, q3, c23.z * v[i][3]);
        }
        __syncwarp();
        off = off_n;
        c01 = c01_n;
        c23 = c23_n;
    }

#pragma unroll
    for (int i = 0; i < TT; ++i) {
        if (t0 + i < T) {
            uint2 o;
            o.x = pack_half2(v[i][0], v[i][1]);
            o.y = pack_half2(v[i][2], v[i][3]);
            *reinterpret_cast<uint2*>(Xr + (t0 + i) * in + c0) = o;
        }
    }
}

cudaError_t launch_rotate(const RotDev& r, const void* X, void* Xr, int64_t T, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    const __half* x = static_cast<const __half*>(X);
    __half* y = static_cast<__half*>(Xr);
    if (T <= 16) {   // decode batches: 4 tokens per warp for more warps in flight
        constexpr int TT = 4;
        const int64_t tasks = ((T + TT - 1) / TT) * r.G;
        rotate_kernel<TT><<<(unsigned)((tasks + 3) / 4), 128, 0, s>>>(x, y, T, (int)r.in, r.G, r.K, r.rotx, r.inv_alpha);
    } else {
        constexpr int TT = 8;
        const int64_t tasks = ((T + TT - 1) / TT) * r.G;
        rotate_kernel<TT><<<(unsigned)((tasks + 3) / 4), 128, 0, s>>>(x, y, T, (int)r.in, r.G, r.K, r.rotx, r.inv_alpha);
    }
    return cudaGetLastError();
}

}  // namespace paro
