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

    float(*b)[128] = buf[warp];
    for (int tb = 0; tb < K; tb += 8) {
        // all parameter loads of up to 8 layers are issued before any is used
        uint32_t pw[8];
        float4 c01[8], c23[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (tb + u < K) {
                const uint8_t* blk = rot_block(rotp, tb + u, g, G);
                pw[u] = __ldg(reinterpret_cast<const uint32_t*>(blk) + lane);
                c01[u] = __ldg(reinterpret_cast<const float4*>(blk + 128) + 2 * lane);
                c23[u] = __ldg(reinterpret_cast<const float4*>(blk + 128) + 2 * lane + 1);
            }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (tb + u < K) {
                const int p0 = pw[u] & 0xFF, p1 = (pw[u] >> 8) & 0xFF, p2 = (pw[u] >> 16) & 0xFF, p3 = pw[u] >> 24;
#pragma unroll
                for (int i = 0; i < TT; ++i)
                    *reinterpret_cast<float4*>(&b[i][4 * lane]) = make_float4(v[i][0], v[i][1], v[i][2], v[i][3]);
                __syncwarp();
#pragma unroll
                for (int i = 0; i < TT; ++i) {
                    const float q0 = b[i][p0], q1 = b[i][p1], q2 = b[i][p2], q3 = b[i][p3];
                    v[i][0] = fmaf(c01[u].y, q0, c01[u].x * v[i][0]);
                    v[i][1] = fmaf(c01[u].w, q1, c01[u].z * v[i][1]);
                    v[i][2] = fmaf(c23[u].y, q2, c23[u].x * v[i][2]);
                    v[i][3] = fmaf(c23[u].w, q3, c23[u].z * v[i][3]);
                }
                __syncwarp();
            }
        }
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
        rotate_kernel<TT><<<(unsigned)((tasks + 3) / 4), 128, 0, s>>>(x, y, T, (int)r.in, r.G, r.K, r.rotp, r.inv_alpha);
    } else {
        constexpr int TT = 8;
        const int64_t tasks = ((T + TT - 1) / TT) * r.G;
        rotate_kernel<TT><<<(unsigned)((tasks + 3) / 4), 128, 0, s>>>(x, y, T, (int)r.in, r.G, r.K, r.rotp, r.inv_alpha);
    }
    return cudaGetLastError();
}

}  // namespace paro
