// Activation rotation X' = X T^-1 with the Givens layers themselves, for
// decode batches of at most 16 tokens (ParoQuant CSDN article, section 2.1;
// the online rotation kernel of section 3.1): per token row and 128-channel
// group, divide by alpha, then K layers of independent Givens pairs, fp32 in
// registers, fp16 out. Larger batches go to the tensor-core kernel
// (rotate_tc.cu), which applies each group's whole rotation as one matrix.
//
// Mapping: one CTA per group, one warp per quad of four tokens. Lane L holds
// channels 4L..4L+3 of the quad; partner values are exchanged through a
// warp-private shared-memory buffer each layer, at positions chosen on the
// host so that every access is bank-conflict-free.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace paro {

// Quad kernel. Work items are (128-channel group g, token tile) in
// group-major order, a tile being nw warps x QW quads of four tokens; CTA c
// takes the contiguous run [c W / n, (c + 1) W / n) of the W items, so the
// load is even and a CTA meets at most a few groups. Lane L holds channels
// 4L..4L+3. A group's K quad exchange blocks are copied into shared memory
// when the CTA reaches it (the first before the wait for the previous grid:
// tables are never written by a kernel on the path), so each layer's
// positions and coefficients come from shared memory, once per layer for all
// QW quads. Partner values are exchanged as float4 slots (one channel, four
// tokens; conflict-free for 16-byte accesses); two tokens are updated per
// packed f32x2 multiply and fma. With QW > 1 each warp uses two 2 KB
// exchange buffers alternately (one warp barrier per quad and layer) and
// loads the next item's X while it rotates the current one. The operations
// and their order do not depend on the batch, so a row's X' does not either.
// PF: each layer's table entries are loaded during the layer before.
// lane_major != 0 writes each 64-channel block of X' in the order the decode
// kernel's B fragments read it: channel 16 j + 4 q + e at position
// 16 q + 4 j + e (the values are the same, only their places change).
template <int QW, bool PF>
__global__ void __launch_bounds__(256) rotate_quad_kernel(const __half* __restrict__ X, __half* __restrict__ Xr,
                                                          int T, int in, int G, int K,
                                                          const uint8_t* __restrict__ rotq,
                                                          const float* __restrict__ inv_alpha, int lane_major) {
    constexpr int NBUF = QW > 1 ? 2 : 1;
    asm volatile("griddepcontrol.launch_dependents;");
    extern __shared__ __align__(16) unsigned char sm[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int tile_tokens = nw * 4 * QW;
    const int ntiles = (T + tile_tokens - 1) / tile_tokens;
    const int64_t W = (int64_t)G * ntiles;
    const int64_t w_lo = (int64_t)blockIdx.x * W / gridDim.x, w_hi = (int64_t)(blockIdx.x + 1) * W / gridDim.x;
    if (w_lo >= w_hi) return;
    unsigned char* prm = sm;                               // [K][kRotQBlockBytes] of the current group
    const uint32_t prm_s = (uint32_t)__cvta_generic_to_shared(prm);
    const uint32_t xbuf = prm_s + (uint32_t)K * kRotQBlockBytes + warp * (2048u * NBUF);
    auto copy_tables = [&](int g) {
        const int per_layer = kRotQBlockBytes / 16;
        for (int i = threadIdx.x; i < K * per_layer; i += blockDim.x) {
            const int t = i / per_layer, v = i - t * per_layer;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(prm_s + 16u * i),
                         "l"(rotq_block(rotq, t, g, G) + 16 * v) : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    int cur_g = (int)(w_lo / ntiles);
    copy_tables(cur_g);
    {
        // Ask L2 for the first item's X rows (two 128-byte lines per token)
        // while the previous grid finishes. A prefetch returns no data, so it
        // is safe even when X is that grid's output: the loads below still
        // come after the wait and read what the grid wrote.
        const int tile = (int)(w_lo - (int64_t)cur_g * ntiles);
        const int t = tile * tile_tokens + warp * 4 * QW + (lane >> 1);
        if (lane < 8 * QW && t < T)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(X + (size_t)t * in + cur_g * 128 + (lane & 1) * 64));
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");   // X may be the previous grid's output

    uint2 raw[QW][4];                                      // X of the item to rotate next, fp16
    auto load_item = [&](int64_t w) {
        const int g = (int)(w / ntiles), tile = (int)(w - (int64_t)g * ntiles);
        const int t0 = tile * tile_tokens + warp * 4 * QW, c0 = g * 128 + 4 * lane;
#pragma unroll
        for (int q = 0; q < QW; ++q)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = t0 + 4 * q + i;
                raw[q][i] = make_uint2(0u, 0u);
                if (t < T) raw[q][i] = __ldg(reinterpret_cast<const uint2*>(X + (size_t)t * in + c0));
            }
    };
    load_item(w_lo);
    float4 ia = __ldg(reinterpret_cast<const float4*>(inv_alpha + cur_g * 128 + 4 * lane));
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    uint32_t flip = 0;                                     // exchange buffer in use (NBUF == 2)
    for (int64_t w = w_lo; w < w_hi; ++w) {
        const int g = (int)(w / ntiles), tile = (int)(w - (int64_t)g * ntiles);
        if (g != cur_g) {                                  // next group: its tables replace the last ones
            __syncthreads();
            copy_tables(g);
            ia = __ldg(reinterpret_cast<const float4*>(inv_alpha + g * 128 + 4 * lane));
            asm volatile("cp.async.wait_all;" ::: "memory");
            __syncthreads();
            cur_g = g;
        }
        uint64_t v[QW][4][2];                              // [quad][channel j][token pair]
#pragma unroll
        for (int q = 0; q < QW; ++q) {
            float x[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 lo = __half22float2(*reinterpret_cast<__half2*>(&raw[q][i].x));
                const float2 hi = __half22float2(*reinterpret_cast<__half2*>(&raw[q][i].y));
                x[i][0] = lo.x * ia.x;
                x[i][1] = lo.y * ia.y;
                x[i][2] = hi.x * ia.z;
                x[i][3] = hi.y * ia.w;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                v[q][j][0] = f2_pack(x[0][j], x[1][j]);
                v[q][j][1] = f2_pack(x[2][j], x[3][j]);
            }
        }
        if (QW > 1 && w + 1 < w_hi) load_item(w + 1);     // in flight during the layers
        // With PF, layer t's positions and coefficients are loaded during
        // layer t - 1 (the exchange's asm statements are compiler barriers,
        // so the loads are placed by hand before them), which takes their
        // latency off the chain store -> barrier -> load -> fma of a layer.
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
            bool act[4];                                   // channel in a pair of this layer
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                st[j] = 16u * ((pos.x >> (8 * j)) & 0x7Fu);
                ld[j] = 16u * ((pos.y >> (8 * j)) & 0x7Fu);
                act[j] = (pos.x >> (8 * j + 7)) & 1u;
            }
#pragma unroll
            for (int q = 0; q < QW; ++q) {
                // with two buffers a buffer is rewritten two quads later, after
                // every lane has passed the barrier between (its reads precede it)
                const uint32_t buf = xbuf + flip;
                if (NBUF == 2) flip ^= 2048u;
                // only channels in a pair go through shared memory (lanes
                // with inactive channels drop out of those accesses)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (act[j])
                        asm volatile("st.shared.v2.b64 [%0], {%1, %2};" ::"r"(buf + st[j]), "l"(v[q][j][0]),
                                     "l"(v[q][j][1]) : "memory");
                __syncwarp();
                uint64_t p[4][2];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    p[j][0] = v[q][j][0];
                    p[j][1] = v[q][j][1];
                    if (act[j])
                        asm volatile("ld.shared.v2.b64 {%0, %1}, [%2];" : "=l"(p[j][0]), "=l"(p[j][1])
                                     : "r"(buf + ld[j]) : "memory");
                }
                if (NBUF == 1) __syncwarp();
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint64_t a2 = f2_pack(ca[j], ca[j]), b2 = f2_pack(cb[j], cb[j]);
#pragma unroll
                    for (int h = 0; h < 2; ++h) v[q][j][h] = f2_fma(b2, p[j][h], f2_mul(a2, v[q][j][h]));
                }
            }
            pos = pos_n;
            c01 = c01_n;
            c23 = c23_n;
        }
        const int t0 = tile * tile_tokens + warp * 4 * QW;
        // lane L holds channels 4L..4L+3 = 64 b + 16 j + 4 q + (0..3) with L = 16 b + 4 j + q
        const int piece = lane_major ? ((lane & 16) | ((lane & 3) << 2) | ((lane >> 2) & 3)) : lane;
        const int c0 = g * 128 + 4 * piece;
#pragma unroll
        for (int q = 0; q < QW; ++q) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float2 w0 = f2_unpack(v[q][0][h]), w1 = f2_unpack(v[q][1][h]);
                const float2 w2 = f2_unpack(v[q][2][h]), w3 = f2_unpack(v[q][3][h]);
                const int t = t0 + 4 * q + 2 * h;
                if (t < T)
                    *reinterpret_cast<uint2*>(Xr + (size_t)t * in + c0) =
                        make_uint2(pack_half2(w0.x, w1.x), pack_half2(w2.x, w3.x));
                if (t + 1 < T)
                    *reinterpret_cast<uint2*>(Xr + (size_t)(t + 1) * in + c0) =
                        make_uint2(pack_half2(w0.y, w1.y), pack_half2(w2.y, w3.y));
            }
        }
    }
}

namespace {

// above 16 tokens the tensor-core kernel (rotate_tc.cu) rotates: measured
// faster from 17 tokens on (3.0 against 3.6 us at 17 tokens, hidden 4096, K = 8)
constexpr int64_t kRotateTcMinTokens = 17;

template <int QW, bool PF>
cudaError_t launch_quad(const RotDev& r, const void* X, void* Xr, int64_t T, int warps, cudaStream_t s,
                        int lane_major) {
    constexpr int NBUF = QW > 1 ? 2 : 1;
    const size_t smem = (size_t)r.K * kRotQBlockBytes + (size_t)warps * 2048 * NBUF;
    if (smem > 48 * 1024) {
        const cudaError_t e =
            cudaFuncSetAttribute(rotate_quad_kernel<QW, PF>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const int64_t ntiles = (T + (int64_t)warps * 4 * QW - 1) / ((int64_t)warps * 4 * QW);
    int64_t ctas = ntiles * r.G;                           // one item per CTA
    if (QW > 1) {   // resident CTAs share the items evenly: one wave
        int dev = 0, sms = 148, per_sm = 1;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rotate_quad_kernel<QW, PF>, 32 * warps, smem);
        ctas = std::min<int64_t>(ctas, (int64_t)sms * std::max(per_sm, 1));
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)ctas, 1, 1);
    cfg.blockDim = dim3((unsigned)(32 * warps), 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, rotate_quad_kernel<QW, PF>, static_cast<const __half*>(X),
                                             static_cast<__half*>(Xr), (int)T, (int)r.in, r.G, r.K,
                                             (const uint8_t*)r.rotq, (const float*)r.inv_alpha, lane_major);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

size_t rotate_decode_smem(int K, int T) { return (size_t)K * kRotQBlockBytes + (size_t)((T + 3) / 4) * 2048; }

cudaError_t launch_rotate_decode(const RotDev& r, const void* X, void* Xr, int64_t T, cudaStream_t s,
                                 bool lane_major) {
    if (T <= 0) return cudaSuccess;
    if (T > 16 || r.group == 256 || !r.rotq) return cudaErrorInvalidValue;
    // prefetching the next layer's tables pays with several warps per CTA
    // (measured: 2% of the decode step at 16 tokens) but not with one or two
    const int warps = (int)((T + 3) / 4);
    return T > 8 ? launch_quad<1, true>(r, X, Xr, T, warps, s, lane_major ? 1 : 0)
                 : launch_quad<1, false>(r, X, Xr, T, warps, s, lane_major ? 1 : 0);
}

cudaError_t launch_rotate(const RotDev& r, const void* X, void* Xr, int64_t T, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    // 256-channel groups have no Givens tables: every batch on the tensor cores
    if (T < kRotateTcMinTokens && r.group != 256) return launch_rotate_decode(r, X, Xr, T, s);
    return launch_rotate_tc(r, X, Xr, T, s);
}

}  // namespace paro
