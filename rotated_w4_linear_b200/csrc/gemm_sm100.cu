// Prefill contraction on the 5th-generation tensor cores:
//   Y[T][out] = X'[T][in] * w_hat[out][in]^T,  X' = X T^-1 (fp16, in global
//   memory, written by the rotation kernel), w_hat dequantised on the fly.
//
// One CTA computes a 128-row x BN-token tile of Y^T = w_hat * X'^T with a
// 4-stage pipeline over 64-wide k blocks; 6 warps with fixed roles:
//   warp 0    TMA producer: per stage one 2-D tile of X' (BN tokens x 64
//             channels, 128-byte swizzle, rows past T read as zeros), one
//             tile of packed int4 codes (8 row blocks x 512 B) and the
//             group's scales and zero points of those 8 row blocks;
//   warp 1    allocates tensor memory; one lane issues tcgen05.mma
//             (kind::f16, M = 128, N = BN, K = 16) with A = w_hat read from
//             tensor memory and B = X' read from shared memory through a
//             matrix descriptor, fp32 accumulation in tensor memory, and
//             commits each stage back to the producer;
//   warps 2-5 dequantise: each thread converts one 32-bit word per 16x16
//             tile exactly as the decode kernel does (w_hat = fp16((q - z) s))
//             and writes the four fp16 pairs with tcgen05.st.16x256b, whose
//             lane/column pattern is the packed layout's (rows g, g + 8;
//             channels 4q .. 4q + 3), one store per row block and stage; then
//             they run the epilogue: tcgen05.ld of the accumulator (one row
//             per thread), fp32 -> fp16, store to Y.
// Tensor memory: columns [0, BN) hold the fp32 accumulator, then 4 stages of
// A (32 columns each: 64 fp16 per row). All waits are bounded (sm100.cuh).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace paro {

namespace {

constexpr uint32_t kWStage = 8 * 512;                   // 8 row blocks x one 64-wide k block
constexpr uint32_t kSStage = 8 * 32;                    // scales: 8 row blocks x one group (8 words)
constexpr uint32_t kZStage = 8 * 16;                    // zeros: 8 row blocks x two groups (2 x 8 bytes)

// NACC accumulators (BN columns each) + STAGES A stages of 32 columns, rounded up to a power of two
template <int BN, int STAGES, int NACC>
__host__ __device__ constexpr uint32_t tmem_cols() {
    return BN * NACC + 32 * STAGES <= 32 ? 32u : BN * NACC + 32 * STAGES <= 64 ? 64u
           : BN * NACC + 32 * STAGES <= 128 ? 128u : BN * NACC + 32 * STAGES <= 256 ? 256u : 512u;
}

struct GemmArgs {
    int T, in, out, G, Gp, nkb, nrb;   // G: quantisation groups along in (Gp: rounded up to even)
    int gshift;                 // 64-wide k block kb lies in group kb >> gshift (1: group 128, 0: group 64)
    int kb_per_split;           // 64-wide k blocks per CTA along grid z (even: splits start on a group)
    int nsplit;                 // CTAs along z = cluster size along z (split-k)
    const uint32_t* sp;
    const uint8_t* zp;
    const __half* bias;         // [out] fp16 or null
    __half* Y;                  // fp16 [T][out], or
    float* Yf;                  // fp32 [T][out] unrounded sums (row-parallel partials) when not null
};

__device__ __forceinline__ void cluster_barrier() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t local_addr, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

}  // namespace

// BN: tokens per tile (MMA N); STAGES: pipeline depth; DQG: dequant warp
// groups of 4 warps, group d handling the stages i = d, d + DQG, ...;
// NACC: accumulators the MMAs rotate over. Consecutive MMAs into one
// accumulator wait for each other's full latency, which dominates at small
// N; independent accumulators let them overlap (summed in the epilogue).
template <int BN, int STAGES, int DQG, int NACC>
__global__ void __launch_bounds__(64 + 128 * DQG, 1)
gemm_w4_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
               const __grid_constant__ CUtensorMap tm_s, const __grid_constant__ CUtensorMap tm_z, const GemmArgs a) {
    // A dequantisation group waits on its stages' mbarriers by phase parity,
    // which cannot tell phase u from u + 2: each stage must belong to one
    // group, so that a group's successive waits on it are one phase apart
    // (with 2 groups and 5 stages a group could come back to a stage while
    // the other group's use of it was still in flight, and pass on stale data).
    static_assert(STAGES % DQG == 0, "every stage must belong to one dequantisation group");
    constexpr uint32_t kBStage = BN * 128;              // BN rows x 64 fp16
    constexpr uint32_t kIdesc = umma_idesc_f16(128, BN);
    constexpr uint32_t kTmemCols = tmem_cols<BN, STAGES, NACC>();
    constexpr int kRedStride = 128 + 4;                  // floats per token row of the split-k tile
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    unsigned char* sB = smem;
    unsigned char* sW = smem + STAGES * kBStage;
    unsigned char* sS = sW + STAGES * kWStage;          // per stage: scales of the group, 8 row blocks x 32 B
    unsigned char* sZ = sS + STAGES * kSStage;          // per stage: zeros of the group pair, 8 row blocks x 16 B
    uint64_t* bars = reinterpret_cast<uint64_t*>(sZ + STAGES * kZStage);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 3 * STAGES + 1);
    // raised by a wait that ran out: every role stops issuing work (tslot[1])
    volatile uint32_t* abort = tslot + 1;
    float* red = reinterpret_cast<float*>(bars + 3 * STAGES + 2);   // split-k partial tile (BN == 16)
    const uint32_t full0 = smem_addr(bars), afull0 = full0 + 8 * STAGES, free0 = afull0 + 8 * STAGES;
    const uint32_t done = free0 + 8 * STAGES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rb0 = blockIdx.x * 8, n0 = blockIdx.y * BN;
    const int kb0 = blockIdx.z * a.kb_per_split;
    const int nk = max(0, min(a.nkb, kb0 + a.kb_per_split) - kb0);
    // CTAs walk their k-range from different starting blocks (even, so a
    // stage pair stays inside one group): concurrent requests then spread
    // over the DRAM channels instead of sharing their low address bits.
    const int kstart = nk > 2 ? (int)(((blockIdx.x * 0x9E3779B1u + blockIdx.y * 0x85EBCA77u) >> 16) % (uint32_t)(nk >> 1)) * 2 : 0;
    auto kblock = [&](int i) { int j = i + kstart; if (j >= nk) j -= nk; return kb0 + j; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(afull0 + 8 * s, 4);                 // one arrive per dequant warp of the group
            mbar_init(free0 + 8 * s, 1);
        }
        mbar_init(done, 1);
        *abort = 0u;
        mbar_fence_init();
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_w);
        tma_prefetch_desc(&tm_s);
        tma_prefetch_desc(&tm_z);
    }
    if (warp == 1) tmem_alloc(smem_addr(tslot), kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tslot;
    const uint32_t tA = tbase + BN * NACC;              // A stages after the accumulator columns
    // X' is written by the rotation grid launched just before this one
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == 0) {
        if (lane == 0) {
            // issued[s]: stage s's loads issued so far (the last one's phase
            // is issued[s] - 1); they must all have landed before the CTA exits
            int issued[STAGES];
#pragma unroll
            for (int s = 0; s < STAGES; ++s) issued[s] = 0;
            for (int i = 0; i < nk; ++i) {
                const int s = i % STAGES, u = i / STAGES;
                if (u > 0 && !mbar_wait(free0 + 8 * s, (u - 1) & 1, kFaultTmaWait, abort)) break;
                if (*abort) break;
                const int kb = kblock(i), gi = kb >> a.gshift;
                mbar_arrive_expect_tx(full0 + 8 * s, kBStage + kWStage + kSStage + kZStage);
                tma_load_2d(smem_addr(sB + s * kBStage), &tm_x, kb * 64, n0, full0 + 8 * s);
                tma_load_2d(smem_addr(sW + s * kWStage), &tm_w, kb * 128, rb0, full0 + 8 * s);
                tma_load_2d(smem_addr(sS + s * kSStage), &tm_s, gi * 8, rb0, full0 + 8 * s);
                tma_load_2d(smem_addr(sZ + s * kZStage), &tm_z, (gi & ~1) * 8, rb0, full0 + 8 * s);
#pragma unroll
                for (int t = 0; t < STAGES; ++t)
                    if (t == s) issued[t] = u + 1;
            }
            if (*abort) {   // drain: wait (bounded, not cut short) for every issued load to land
#pragma unroll
                for (int s = 0; s < STAGES; ++s)
                    if (issued[s] > 0) mbar_wait(full0 + 8 * s, (issued[s] - 1) & 1, kFaultDrainWait, nullptr);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            for (int i = 0; i < nk; ++i) {
                const int s = i % STAGES, u = i / STAGES;
                if (!mbar_wait(afull0 + 8 * s, u & 1, kFaultMmaWait, abort)) break;
                if (!mbar_wait(full0 + 8 * s, u & 1, kFaultMmaWait, abort)) break;
                tc_fence_after();
                const uint64_t bdesc = umma_desc_sw128_kmajor(smem_addr(sB + s * kBStage));
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const int n = i * 4 + kk;                 // MMA number; accumulator n % NACC
                    umma_f16_ts(tbase + (uint32_t)((n % NACC) * BN), tA + s * 32 + kk * 8,
                                bdesc + (uint64_t)(kk * 2), kIdesc, n >= NACC ? 1u : 0u);
                }
                umma_commit(free0 + 8 * s);
            }
            // always: `done` arrives once every MMA issued above has completed
            // (also after an abort, so tensor memory is released only then)
            umma_commit(done);
        }
    } else {
        // ---- dequant group dg, quarter qw of the tensor-memory lanes (rows 32 qw .. 32 qw + 31)
        const int dg = (warp - 2) >> 2;
        const int qw = warp & 3;
        const int g = lane >> 2;
        for (int i = dg; i < nk; i += DQG) {
            const int s = i % STAGES, u = i / STAGES;
            const int gi = kblock(i) >> a.gshift;
            // the tensor-memory stores below are warp-collective: the whole
            // warp goes on only if every lane saw the stage arrive
            if (!__all_sync(0xffffffffu, mbar_wait(full0 + 8 * s, u & 1, kFaultDequantWait, abort) && !*abort))
                break;
            const uint32_t wbase = smem_addr(sW + s * kWStage);
            const uint32_t sbase = smem_addr(sS + s * kSStage), zbase = smem_addr(sZ + s * kZStage);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int rbl = 2 * qw + r;
                const uint4 wv = lds128(wbase + rbl * 512 + lane * 16);
                uint32_t sc0, sc1, regs[16];
                scale_pairs(lds32(sbase + rbl * 32 + g * 4), sc0, sc1);
                const Zero2 zc = zero_consts(lds8(zbase + rbl * 16 + (gi & 1) * 8 + g));
                dequant_word(wv.x, zc, sc0, sc1, regs + 0);
                dequant_word(wv.y, zc, sc0, sc1, regs + 4);
                dequant_word(wv.z, zc, sc0, sc1, regs + 8);
                dequant_word(wv.w, zc, sc0, sc1, regs + 12);
                tmem_st_16x256b_x4(tA + s * 32 + ((uint32_t)(32 * qw + 16 * r) << 16), regs);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(afull0 + 8 * s);
        }

        // ---- epilogue (group 0): one accumulator row per thread
        // (skipped after an abort: the tile is not valid, and the fault word says so)
        if (dg == 0 && __all_sync(0xffffffffu, mbar_wait(done, 0, kFaultEpilogueWait, abort) && !*abort)) {
            tc_fence_after();
            const int rloc = 32 * qw + lane;
            const int row = rb0 * 16 + rloc;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 16) {
                uint32_t r[16];
                tmem_ld_32x32b_x16(tbase + ((uint32_t)(32 * qw) << 16) + c0, r);
                tmem_wait_ld();
#pragma unroll
                for (int ac = 1; ac < NACC; ++ac) {           // sum the independent accumulators
                    uint32_t r2[16];
                    tmem_ld_32x32b_x16(tbase + ((uint32_t)(32 * qw) << 16) + ac * BN + c0, r2);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) + __uint_as_float(r2[j]));
                }
                if (a.nsplit > 1) {                       // BN == 16: partial tile red[token][row]
#pragma unroll
                    for (int j = 0; j < 16; ++j) red[j * kRedStride + rloc] = __uint_as_float(r[j]);
                } else if (row < a.out) {
                    const float b = a.bias ? __half2float(a.bias[row]) : 0.f;
                    if (a.Yf) {                               // fp32 partial sums (row-parallel)
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int t = n0 + c0 + j;
                            if (t < a.T) a.Yf[(size_t)t * a.out + row] = __uint_as_float(r[j]) + b;
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int t = n0 + c0 + j;
                            if (t < a.T) a.Y[(size_t)t * a.out + row] = __float2half_rn(__uint_as_float(r[j]) + b);
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    if (a.nsplit > 1) {
        // split-k: CTA z of the cluster sums its slice of the 128 rows over
        // the cluster's partial tiles (distributed shared memory) and stores it
        cluster_barrier();
        const int share = (128 + a.nsplit - 1) / a.nsplit;
        const int r_lo = (int)blockIdx.z * share;
        const int n = max(0, min(share, 128 - r_lo));
        const uint32_t red_addr = smem_addr(red);
        for (int e = threadIdx.x; e < 16 * n; e += blockDim.x) {
            const int t = e / n, rl = r_lo + e % n;
            const int row = rb0 * 16 + rl;
            float sum = 0.f;
            for (int x = 0; x < a.nsplit; ++x) sum += ld_cluster_f32(red_addr + (uint32_t)(t * kRedStride + rl) * 4u, (uint32_t)x);
            if (t < a.T && row < a.out) {
                const float v = sum + (a.bias ? __half2float(a.bias[row]) : 0.f);
                if (a.Yf) a.Yf[(size_t)t * a.out + row] = v;
                else a.Y[(size_t)t * a.out + row] = __float2half_rn(v);
            }
        }
        cluster_barrier();                                // partial tiles stay alive until all reads are done
    } else {
        __syncthreads();
    }
    if (warp == 1) {
        // no MMA may still write tensor memory when it is released: `done`
        // (committed after the last MMA this CTA issued) must have arrived;
        // this wait is not cut short by the abort flag
        mbar_wait(done, 0, kFaultDrainWait, nullptr);
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
namespace {
PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {  // driver entry point, no link-time libcuda
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

}  // namespace

bool encode_tma_2d(CUtensorMap* tm, CUtensorMapDataType type, const void* base, uint64_t inner, uint64_t outer,
                   uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = get_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1u, 1u};
    return enc(tm, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


namespace {

template <int BN, int STAGES, int DQG, int NACC>
cudaError_t launch_cfg(const CUtensorMap* tm, const GemmArgs& a, int mt, int nt, cudaStream_t s) {
    constexpr size_t smem = STAGES * (BN * 128 + kWStage + kSStage + kZStage) + (3 * STAGES + 2) * 8 +
                            16 * (128 + 4) * 4 + 1024;
    // kernel attributes, set once per device (double-checked under a lock)
    static std::atomic<bool> configured[64] = {};
    static std::mutex mu;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev].load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> lock(mu);
        if (!configured[dev].load(std::memory_order_relaxed)) {
            cudaError_t e = cudaFuncSetAttribute(gemm_w4_kernel<BN, STAGES, DQG, NACC>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(gemm_w4_kernel<BN, STAGES, DQG, NACC>,
                                         cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (e != cudaSuccess) return e;
            configured[dev].store(true, std::memory_order_release);
        }
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(mt, nt, a.nsplit);
    cfg.blockDim = dim3(64 + 128 * DQG, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = a.nsplit;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, gemm_w4_kernel<BN, STAGES, DQG, NACC>, tm[0], tm[1], tm[2], tm[3], a);
}

// tm[0]: X' [T][in] fp16, box 64 channels x BN tokens, 128-byte swizzle, zero fill past T
// tm[1]: packed int4 codes as uint32 [out/16][in/64 * 128], box one k block x 8 row blocks
// tm[2]: scales uint32 [out/16][G * 8], box one group x 8 row blocks
// tm[3]: zeros uint8 [out/16][Gp * 8], box two groups x 8 row blocks
// (G quantisation groups of 128 or 64 channels)
bool encode_maps(const void* Xr, const void* qw, const void* sp, const void* zp, int64_t T, int BN,
                 const GemmArgs& a, CUtensorMap* tm) {
    return encode_tma_2d(&tm[0], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Xr, (uint64_t)a.in, (uint64_t)T, (uint64_t)a.in * 2,
                     64u, (uint32_t)BN, CU_TENSOR_MAP_SWIZZLE_128B) &&
           encode_tma_2d(&tm[1], CU_TENSOR_MAP_DATA_TYPE_UINT32, qw, (uint64_t)a.nkb * 128, (uint64_t)a.nrb,
                     (uint64_t)a.nkb * 512, 128u, 8u, CU_TENSOR_MAP_SWIZZLE_NONE) &&
           encode_tma_2d(&tm[2], CU_TENSOR_MAP_DATA_TYPE_UINT32, sp, (uint64_t)a.G * 8, (uint64_t)a.nrb,
                     (uint64_t)a.G * 32, 8u, 8u, CU_TENSOR_MAP_SWIZZLE_NONE) &&
           encode_tma_2d(&tm[3], CU_TENSOR_MAP_DATA_TYPE_UINT8, zp, (uint64_t)a.Gp * 8, (uint64_t)a.nrb,
                     (uint64_t)a.Gp * 8, 16u, 8u, CU_TENSOR_MAP_SWIZZLE_NONE);
}

GemmArgs make_args(int64_t T, int64_t in, int64_t out, int group, const void* scp, const void* zp, const void* bias,
                   void* Y, bool y_fp32) {
    GemmArgs a{};
    a.T = (int)T;
    a.in = (int)in;
    a.out = (int)out;
    a.G = (int)(in / group);
    a.gshift = group == 64 ? 0 : 1;
    a.Gp = a.G + (a.G & 1);
    a.nkb = (int)(in / 64);
    a.nrb = (int)(out / 16);
    // the kernel can split k over a cluster along z (16-token tiles, partial
    // tiles reduced through distributed shared memory); the token tiles used
    // here (64, 128, 256) need no split, so every launch runs one
    a.kb_per_split = a.nkb;
    a.nsplit = 1;
    a.sp = static_cast<const uint32_t*>(scp);
    a.zp = static_cast<const uint8_t*>(zp);
    a.bias = static_cast<const __half*>(bias);
    a.Y = y_fp32 ? nullptr : static_cast<__half*>(Y);
    a.Yf = y_fp32 ? static_cast<float*>(Y) : nullptr;
    return a;
}

}  // namespace

cudaError_t launch_gemm(const void* Xr, const void* qw, const void* scp, const void* zp, const void* bias, void* Y,
                        int64_t T, int64_t in, int64_t out, int group, cudaStream_t s, bool y_fp32) {
    if (T <= 0) return cudaSuccess;
    if (group != 64 && group != 128) return cudaErrorInvalidValue;
    const int BN = T <= 64 ? 64 : T <= 128 ? 128 : 256;
    GemmArgs a = make_args(T, in, out, group, scp, zp, bias, Y, y_fp32);
    CUtensorMap tm[4];
    if (!encode_maps(Xr, qw, scp, zp, T, BN, a, tm)) return cudaErrorInvalidValue;
    const int mt = (a.nrb + 7) / 8;
    const int nt = (int)((T + BN - 1) / BN);
    cudaError_t e;
    if (BN == 64) e = launch_cfg<64, 4, 1, 1>(tm, a, mt, nt, s);
    else if (BN == 128) e = launch_cfg<128, 4, 1, 1>(tm, a, mt, nt, s);
    else e = launch_cfg<256, 4, 1, 1>(tm, a, mt, nt, s);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// Self-test of the bounded waits: one thread waits on an mbarrier at which
// nothing ever arrives (no copy or MMA is in flight). The wait runs out after
// limit_ns, records kFaultSelfTest in the fault word and the kernel returns.
__global__ void wait_selftest_kernel(uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bar), 1);
        abort_flag = 0u;
        mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(smem_addr(&bar), 0, kFaultSelfTest, &abort_flag, limit_ns);
}

cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t s) {
    wait_selftest_kernel<<<1, 32, 0, s>>>(limit_ns);
    return cudaGetLastError();
}

cudaError_t read_fault(unsigned int* code, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(code, g_paro_fault, sizeof(unsigned int));
    if (e != cudaSuccess || !clear) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_paro_fault, &zero, sizeof(unsigned int));
}

}  // namespace paro
