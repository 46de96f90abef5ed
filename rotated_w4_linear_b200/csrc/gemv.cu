// Fused decode kernel for tokens <= 16:
//   Y[T][out] = (X T^-1) w_hat^T,  the weight stream dominates (HBM bound).
//
// Grid (k-chunk, row tile). A CTA of NW warps owns NW*RBW row blocks of 16
// output rows and one k-chunk of KC 128-channel groups.
//   prologue: issue the first int4 weight loads, then rotate the chunk's
//             activations (all tokens, KC groups) into shared memory as fp16;
//             the rotation of a group needs only that group (pairs never
//             leave a quantisation group), so chunks are independent;
//   mainloop: per 16-row block, dequantise each 32-bit int4 word in
//             registers (LOP3 + exact fp16 sub + one rounded fp16 mul) straight
//             into an m16n8k16 A fragment and multiply with the rotated
//             activations (B fragment from shared memory), fp32 accumulate;
//   epilogue: a single k-chunk writes fp16 Y; otherwise fp32 partial sums are
//             added into the workspace and the last CTA of a row tile (ticket
//             counter) converts them to fp16 and re-zeroes the workspace.
// The k order inside each 16x16 tile follows the packed layout: the MMA's
// logical k slot 2q+e holds channel 4q+e and slot 2q+8+e channel 4q+2+e, so
// each lane's B fragment is four consecutive channels of one token.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace paro {

struct GemvArgs {
    const __half* X;
    int T, in, out, G;
    const uint8_t* rotp;       // null: no rotation
    const float* inv_alpha;
    int K;
    const uint4* qw;
    const uint32_t* sp;
    const uint8_t* zp;
    __half* Y;
    float* acc;
    unsigned* cnt;
    int RBW;
    int nsplit;
};

__device__ __forceinline__ void mma16816(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int NT, int KC, int NW>
__global__ void __launch_bounds__(NW * 32) gemv_kernel(const GemvArgs a) {
    constexpr int KB = 2 * KC;                 // 64-wide k blocks per chunk
    constexpr int XS = KC * 128 + 16;          // smem row stride in halves (== 8 words mod 32)
    __shared__ __align__(16) __half xs[NT * 8][XS];
    __shared__ __align__(16) float rbuf[NW][128];
    __shared__ unsigned s_ticket;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int chunk = blockIdx.x, rt = blockIdx.y;
    const int g0 = chunk * KC;
    const int nkb = a.in >> 6;
    const int nrb = a.out >> 4;
    const int rb0 = (rt * NW + warp) * a.RBW;

    uint4 wq[KB];
    if (rb0 < nrb) {
        const uint4* src = a.qw + ((size_t)rb0 * nkb + 2 * g0) * 32 + lane;
#pragma unroll
        for (int i = 0; i < KB; ++i) wq[i] = ldg_stream(src + i * 32);
    }

    // ---- prologue: X' chunk -> shared memory (fp16) ----
    for (int task = warp; task < NT * 8 * KC; task += NW) {
        const int tok = task / KC, gl = task % KC;
        const int c = (g0 + gl) * 128 + 4 * lane;
        uint2 o = make_uint2(0u, 0u);
        if (tok < a.T) {
            const uint2 raw = __ldg(reinterpret_cast<const uint2*>(a.X + (size_t)tok * a.in + c));
            if (a.rotp) {
                const float4 ia = __ldg(reinterpret_cast<const float4*>(a.inv_alpha + c));
                const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
                const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
                float v[4] = {lo.x * ia.x, lo.y * ia.y, hi.x * ia.z, hi.y * ia.w};
                rotate_group_warp(v, a.rotp, g0 + gl, a.G, a.K, rbuf[warp], lane);
                o.x = pack_half2(v[0], v[1]);
                o.y = pack_half2(v[2], v[3]);
            } else {
                o = raw;
            }
        }
        *reinterpret_cast<uint2*>(&xs[tok][gl * 128 + 4 * lane]) = o;
    }
    __syncthreads();

    // ---- mainloop ----
    const int gq = lane >> 2, qd = lane & 3;
    for (int r = 0; r < a.RBW; ++r) {
        const int rb = rb0 + r;
        if (rb >= nrb) break;
        uint4 cur[KB];
#pragma unroll
        for (int i = 0; i < KB; ++i) cur[i] = wq[i];
        if (r + 1 < a.RBW && rb + 1 < nrb) {
            const uint4* src = a.qw + ((size_t)(rb + 1) * nkb + 2 * g0) * 32 + lane;
#pragma unroll
            for (int i = 0; i < KB; ++i) wq[i] = ldg_stream(src + i * 32);
        }
        float c[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) c[nt][0] = c[nt][1] = c[nt][2] = c[nt][3] = 0.f;
#pragma unroll
        for (int gl = 0; gl < KC; ++gl) {
            const size_t mi = ((size_t)rb * a.G + g0 + gl) * 8 + gq;
            uint32_t zb0, zb1, sc0, sc1;
            zero_bias(__ldg(a.zp + mi), zb0, zb1);
            scale_pairs(__ldg(a.sp + mi), sc0, sc1);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int kb = 2 * gl + h;
                const uint32_t words[4] = {cur[kb].x, cur[kb].y, cur[kb].z, cur[kb].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t hh[4];
                    dequant_word(words[j], zb0, sc0, zb1, sc1, hh);
                    const uint32_t A[4] = {hh[0], hh[2], hh[1], hh[3]};
                    const int kt = kb * 4 + j;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const uint2 bv = *reinterpret_cast<const uint2*>(&xs[nt * 8 + gq][kt * 16 + 4 * qd]);
                        mma16816(c[nt], A, bv.x, bv.y);
                    }
                }
            }
        }
        // ---- epilogue for this row block ----
        const int r0 = rb * 16 + gq, r1 = r0 + 8;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int t = nt * 8 + 2 * qd + e;
                if (t < a.T) {
                    if (a.nsplit == 1) {
                        a.Y[(size_t)t * a.out + r0] = __float2half_rn(c[nt][e]);
                        a.Y[(size_t)t * a.out + r1] = __float2half_rn(c[nt][2 + e]);
                    } else {
                        atomicAdd(a.acc + (size_t)t * a.out + r0, c[nt][e]);
                        atomicAdd(a.acc + (size_t)t * a.out + r1, c[nt][2 + e]);
                    }
                }
            }
        }
    }

    if (a.nsplit == 1) return;
    // ---- split-k completion: the last CTA of this row tile finalises ----
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_ticket = atomicAdd(a.cnt + rt, 1u);
    __syncthreads();
    if (s_ticket != (unsigned)(a.nsplit - 1)) return;
    __threadfence();
    const int rowlo = rt * NW * a.RBW * 16;
    const int rowhi = min(a.out, rowlo + NW * a.RBW * 16);
    const int nrows = rowhi - rowlo;
    const int n = a.T * nrows;
    for (int i = threadIdx.x; i < n; i += NW * 32) {
        const int t = i / nrows, row = rowlo + i % nrows;
        float* p = a.acc + (size_t)t * a.out + row;
        a.Y[(size_t)t * a.out + row] = __float2half_rn(__ldcg(p));
        __stcg(p, 0.f);
    }
    if (threadIdx.x == 0) a.cnt[rt] = 0u;
}

// workspace: fp32 accumulators for 16 tokens x out, then one counter per row block
size_t gemv_workspace_bytes(int64_t /*T*/, int64_t /*in*/, int64_t out) {
    const size_t acc = (size_t)16 * out * sizeof(float);
    const size_t cnt = (size_t)(out / 16) * sizeof(unsigned);
    return ((acc + 255) & ~(size_t)255) + ((cnt + 255) & ~(size_t)255);
}

template <int NT, int KC>
static void launch_gemv_t(const GemvArgs& a, int rowtiles, cudaStream_t s) {
    constexpr int NW = 4;
    dim3 grid(a.nsplit, rowtiles);
    gemv_kernel<NT, KC, NW><<<grid, NW * 32, 0, s>>>(a);
}

cudaError_t launch_gemv(const RotDev* rot, const void* X, const void* qw, const void* scp, const void* zp,
                        void* Y, int64_t T, int64_t in, int64_t out, void* ws, size_t /*ws_bytes*/,
                        cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    constexpr int NW = 4;
    GemvArgs a{};
    a.X = static_cast<const __half*>(X);
    a.T = (int)T;
    a.in = (int)in;
    a.out = (int)out;
    a.G = (int)(in / 128);
    a.rotp = rot ? rot->rotp : nullptr;
    a.inv_alpha = rot ? rot->inv_alpha : nullptr;
    a.K = rot ? rot->K : 0;
    a.qw = static_cast<const uint4*>(qw);
    a.sp = static_cast<const uint32_t*>(scp);
    a.zp = static_cast<const uint8_t*>(zp);
    a.Y = static_cast<__half*>(Y);
    const size_t acc_bytes = ((size_t)16 * out * sizeof(float) + 255) & ~(size_t)255;
    a.acc = static_cast<float*>(ws);
    a.cnt = reinterpret_cast<unsigned*>(static_cast<char*>(ws) + acc_bytes);
    const int KC = (a.G % 4 == 0) ? 4 : (a.G % 2 == 0) ? 2 : 1;
    a.nsplit = a.G / KC;
    const int nrb = a.out / 16;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t target = 4LL * sms;
    int64_t rbw = ((int64_t)nrb * a.nsplit) / (NW * target);
    a.RBW = (int)std::max<int64_t>(1, std::min<int64_t>(16, rbw));
    const int rowtiles = (nrb + NW * a.RBW - 1) / (NW * a.RBW);
    const bool two = T > 8;
    if (KC == 4) {
        if (two) launch_gemv_t<2, 4>(a, rowtiles, s); else launch_gemv_t<1, 4>(a, rowtiles, s);
    } else if (KC == 2) {
        if (two) launch_gemv_t<2, 2>(a, rowtiles, s); else launch_gemv_t<1, 2>(a, rowtiles, s);
    } else {
        if (two) launch_gemv_t<2, 1>(a, rowtiles, s); else launch_gemv_t<1, 1>(a, rowtiles, s);
    }
    return cudaGetLastError();
}

}  // namespace paro
