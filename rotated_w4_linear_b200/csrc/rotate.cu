// Activation rotation X' = X T^-1 with the Givens layers themselves, for
// decode batches of at most 16 tokens (ParoQuant CSDN article, section 2.1;
// the online rotation kernel of section 3.1): per token row and 128-channel
// group, divide by alpha, then K layers of independent Givens pairs, fp32 in
// registers, fp16 out. Larger batches go to the tensor-core kernel
// (rotate_tc.cu), which applies each group's whole rotation as one matrix.
// The per-warp routine is in givens.cuh.
//
// Mapping: one CTA per (group, token tile), one warp per quad of four tokens.
#include <algorithm>

#include "givens.cuh"
#include "kernels.h"

namespace paro {

// Work items are (128-channel group g, token tile) in group-major order, a
// tile being nw warps x one quad of four tokens; CTA c takes the contiguous
// run [c W / n, (c + 1) W / n) of the W items. A group's K quad exchange
// blocks are copied into shared memory when the CTA reaches it (the first
// before the wait for the previous grid: tables are never written by a
// kernel on the path), so each layer's positions and coefficients come from
// shared memory.
template <bool PF>
__global__ void __launch_bounds__(256) rotate_quad_kernel(const __half* __restrict__ X, __half* __restrict__ Xr,
                                                          int T, int in, int G, int K,
                                                          const uint8_t* __restrict__ rotq,
                                                          const float* __restrict__ inv_alpha, int lane_major) {
    asm volatile("griddepcontrol.launch_dependents;");
    extern __shared__ __align__(16) unsigned char sm[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int tile_tokens = nw * 4;
    const int ntiles = (T + tile_tokens - 1) / tile_tokens;
    const int64_t W = (int64_t)G * ntiles;
    const int64_t w_lo = (int64_t)blockIdx.x * W / gridDim.x, w_hi = (int64_t)(blockIdx.x + 1) * W / gridDim.x;
    if (w_lo >= w_hi) return;
    unsigned char* prm = sm;                               // [K][kRotQBlockBytes] of the current group
    const uint32_t prm_s = (uint32_t)__cvta_generic_to_shared(prm);
    const uint32_t xbuf = prm_s + (uint32_t)K * kRotQBlockBytes + warp * 2048u;
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
        const int t = tile * tile_tokens + warp * 4 + (lane >> 1);
        if (lane < 8 && t < T)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(X + (size_t)t * in + cur_g * 128 + (lane & 1) * 64));
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");   // X may be the previous grid's output

    float4 ia = __ldg(reinterpret_cast<const float4*>(inv_alpha + cur_g * 128 + 4 * lane));
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
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
        const int t0 = tile * tile_tokens + warp * 4;
        uint2 raw[4];
        givens_load_quad(X, T, in, g, t0, lane, raw);
        givens_rotate_quad<PF>(prm, xbuf, K, raw, ia, Xr, T, in, g, t0, lane, lane_major != 0);
    }
}

namespace {

// above 16 tokens the tensor-core kernel (rotate_tc.cu) rotates: measured
// faster from 17 tokens on (3.0 against 3.6 us at 17 tokens, hidden 4096, K = 8)
constexpr int64_t kRotateTcMinTokens = 17;

template <bool PF>
cudaError_t launch_quad(const RotDev& r, const void* X, void* Xr, int64_t T, int warps, cudaStream_t s,
                        int lane_major) {
    const size_t smem = (size_t)r.K * kRotQBlockBytes + (size_t)warps * 2048;
    if (smem > 48 * 1024) {
        const cudaError_t e =
            cudaFuncSetAttribute(rotate_quad_kernel<PF>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const int64_t ntiles = (T + (int64_t)warps * 4 - 1) / ((int64_t)warps * 4);
    const int64_t ctas = ntiles * r.G;                     // one item per CTA
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
    const cudaError_t e = cudaLaunchKernelEx(&cfg, rotate_quad_kernel<PF>, static_cast<const __half*>(X),
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
    return T > 8 ? launch_quad<true>(r, X, Xr, T, warps, s, lane_major ? 1 : 0)
                 : launch_quad<false>(r, X, Xr, T, warps, s, lane_major ? 1 : 0);
}

cudaError_t launch_rotate(const RotDev& r, const void* X, void* Xr, int64_t T, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    // 256-channel groups have no Givens tables: every batch on the tensor cores
    if (T < kRotateTcMinTokens && r.group != 256) return launch_rotate_decode(r, X, Xr, T, s);
    return launch_rotate_tc(r, X, Xr, T, s);
}

}  // namespace paro
