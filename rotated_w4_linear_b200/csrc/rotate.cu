// Activation rotation X' = X T^-1 (ParoQuant CSDN article, section 2.1; the
// online rotation kernel of section 3.1): per token row and 128-channel group,
// divide by alpha, then K layers of independent Givens pairs, fp32 in
// registers, fp16 out.
//
// Mapping: one warp owns one (group, token tile). Lane L holds channels
// 4L..4L+3 of TT tokens, loaded as one 8-byte vector per token (a warp reads
// 256 contiguous bytes per row). Partner values are exchanged through a
// warp-private shared-memory slice each layer; rotation coefficients are read
// from the prepared per-(layer, group) block (L1/L2 resident).
#include "common.cuh"
#include "kernels.h"

namespace paro {

template <int TT>
__global__ void __launch_bounds__(128) rotate_kernel(const __half* __restrict__ X, __half* __restrict__ Xr,
                                                     int64_t T, int in, int G, int K,
                                                     const uint8_t* __restrict__ rotp,
                                                     const float* __restrict__ inv_alpha) {
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

    float(*b)[128] = buf[warp];
    for (int t = 0; t < K; ++t) {
        const uint8_t* blk = rot_block(rotp, t, g, G);
        const uint32_t pw = __ldg(reinterpret_cast<const uint32_t*>(blk) + lane);
        const float4 c01 = __ldg(reinterpret_cast<const float4*>(blk + 128) + 2 * lane);
        const float4 c23 = __ldg(reinterpret_cast<const float4*>(blk + 128) + 2 * lane + 1);
        const int p0 = pw & 0xFF, p1 = (pw >> 8) & 0xFF, p2 = (pw >> 16) & 0xFF, p3 = pw >> 24;
#pragma unroll
        for (int i = 0; i < TT; ++i)
            *reinterpret_cast<float4*>(&b[i][4 * lane]) = make_float4(v[i][0], v[i][1], v[i][2], v[i][3]);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < TT; ++i) {
            const float q0 = b[i][p0], q1 = b[i][p1], q2 = b[i][p2], q3 = b[i][p3];
            v[i][0] = fmaf(c01.y, q0, c01.x * v[i][0]);
            v[i][1] = fmaf(c01.w, q1, c01.z * v[i][1]);
            v[i][2] = fmaf(c23.y, q2, c23.x * v[i][2]);
            v[i][3] = fmaf(c23.w, q3, c23.z * v[i][3]);
        }
        __syncwarp();
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
    constexpr int TT = 8;
    const int64_t tasks = ((T + TT - 1) / TT) * r.G;
    const int64_t blocks = (tasks + 3) / 4;
    rotate_kernel<TT><<<(unsigned)blocks, 128, 0, s>>>(static_cast<const __half*>(X), static_cast<__half*>(Xr), T,
                                                       (int)r.in, r.G, r.K, r.rotp, r.inv_alpha);
    return cudaGetLastError();
}

}  // namespace paro
