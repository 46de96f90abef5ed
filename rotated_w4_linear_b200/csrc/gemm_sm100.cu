// Prefill contraction on the 5th-generation tensor cores:
//   Y[T][out] = X'[T][in] * w_hat[out][in]^T,  X' = X T^-1 (fp16, in global
//   memory, written by the rotation kernel), w_hat dequantised on the fly.
//
// One CTA computes a 128-row x BN-token tile of Y^T = w_hat * X'^T with a
// 4-stage pipeline over 64-wide k blocks; 6 warps with fixed roles:
//   warp 0    TMA producer: per stage one 2-D tile of X' (BN tokens x 64
//             channels, 128-byte swizzle, rows past T read as zeros) and one
//             tile of packed int4 codes (8 row blocks x 512 B);
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
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace paro {

namespace {

constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr uint32_t kWStage = 8 * 512;                   // 8 row blocks x one 64-wide k block

// accumulator (BN columns) + 4 A stages of 32 columns, rounded up to a power of two
template <int BN>
constexpr uint32_t tmem_cols() { return BN + 128 <= 256 ? 256u : 512u; }

struct GemmArgs {
    int T, in, out, G, Gp, nkb, nrb;
    const uint32_t* sp;
    const uint8_t* zp;
    __half* Y;
};

}  // namespace

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
gemm_w4_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w, const GemmArgs a) {
    constexpr uint32_t kBStage = BN * 128;              // BN rows x 64 fp16
    constexpr uint32_t kIdesc = umma_idesc_f16(128, BN);
    constexpr uint32_t kTmemCols = tmem_cols<BN>();
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    unsigned char* sB = smem;
    unsigned char* sW = smem + kStages * kBStage;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sW + kStages * kWStage);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 3 * kStages + 1);
    const uint32_t full0 = smem_addr(bars), afull0 = full0 + 8 * kStages, free0 = afull0 + 8 * kStages;
    const uint32_t done = free0 + 8 * kStages;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rb0 = blockIdx.x * 8, n0 = blockIdx.y * BN;
    const int nkb = a.nkb;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(afull0 + 8 * s, 4);                 // one arrive per dequant warp
            mbar_init(free0 + 8 * s, 1);
        }
        mbar_init(done, 1);
        mbar_fence_init();
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_w);
    }
    if (warp == 1) tmem_alloc(smem_addr(tslot), kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tslot;
    const uint32_t tA = tbase + BN;                     // A stages after the accumulator columns
    // X' is written by the rotation grid launched just before this one
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == 0) {
        if (lane == 0) {
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % kStages, u = kb / kStages;
                if (u > 0) mbar_wait(free0 + 8 * s, (u - 1) & 1, kFaultTmaWait);
                mbar_arrive_expect_tx(full0 + 8 * s, kBStage + kWStage);
                tma_load_2d(smem_addr(sB + s * kBStage), &tm_x, kb * 64, n0, full0 + 8 * s);
                tma_load_2d(smem_addr(sW + s * kWStage), &tm_w, kb * 128, rb0, full0 + 8 * s);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % kStages, u = kb / kStages;
                mbar_wait(afull0 + 8 * s, u & 1, kFaultMmaWait);
                mbar_wait(full0 + 8 * s, u & 1, kFaultMmaWait);
                tc_fence_after();
                const uint64_t bdesc = umma_desc_sw128_kmajor(smem_addr(sB + s * kBStage));
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16_ts(tbase, tA + s * 32 + kk * 8, bdesc + (uint64_t)(kk * 2), kIdesc,
                                (kb | kk) != 0 ? 1u : 0u);
                umma_commit(free0 + 8 * s);
            }
            umma_commit(done);
        }
    } else {
        // ---- dequant warps: quarter qw of the tensor-memory lanes = rows 32 qw .. 32 qw + 31
        const int qw = warp & 3;
        const int g = lane >> 2;
        uint32_t sw[2] = {0u, 0u}, zw[2] = {0u, 0u}, sw_n[2] = {0u, 0u}, zw_n[2] = {0u, 0u};
        auto load_meta = [&](int gi, uint32_t* so, uint32_t* zo) {
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int rb = rb0 + 2 * qw + r;
                if (rb < a.nrb && gi < a.G) {
                    so[r] = __ldg(a.sp + ((size_t)rb * a.G + gi) * 8 + g);
                    zo[r] = __ldg(a.zp + ((size_t)rb * a.Gp + gi) * 8 + g);
                } else {
                    so[r] = 0u;
                    zo[r] = 0u;
                }
            }
        };
        load_meta(0, sw, zw);
        load_meta(1, sw_n, zw_n);
        for (int kb = 0; kb < nkb; ++kb) {
            const int s = kb % kStages, u = kb / kStages;
            if (kb >= 2 && (kb & 1) == 0) {             // next group: rotate the prefetched meta
                sw[0] = sw_n[0]; sw[1] = sw_n[1]; zw[0] = zw_n[0]; zw[1] = zw_n[1];
                load_meta((kb >> 1) + 1, sw_n, zw_n);
            }
            mbar_wait(full0 + 8 * s, u & 1, kFaultDequantWait);
            const uint32_t wbase = smem_addr(sW + s * kWStage);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const uint4 wv = lds128(wbase + (2 * qw + r) * 512 + lane * 16);
                uint32_t sc0, sc1, regs[16];
                scale_pairs(sw[r], sc0, sc1);
                const Zero2 zc = zero_consts(zw[r]);
                dequant_word(wv.x, zc, sc0, sc1, regs + 0);
                dequant_word(wv.y, zc, sc0, sc1, regs + 4);
                dequant_word(wv.z, zc, sc0, sc1, regs + 8);
                dequant_word(wv.w, zc, sc0, sc1, regs + 12);
                const uint32_t taddr = tA + s * 32 + ((uint32_t)(32 * qw + 16 * r) << 16);
                tmem_st_16x256b_x4(taddr, regs);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(afull0 + 8 * s);
        }

        // ---- epilogue: one accumulator row per thread
        mbar_wait(done, 0, kFaultEpilogueWait);
        tc_fence_after();
        const int row = rb0 * 16 + 32 * qw + lane;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
            uint32_t r[16];
            tmem_ld_32x32b_x16(tbase + ((uint32_t)(32 * qw) << 16) + c0, r);
            tmem_wait_ld();
            if (row < a.out) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int t = n0 + c0 + j;
                    if (t < a.T) a.Y[(size_t)t * a.out + row] = __float2half_rn(__uint_as_float(r[j]));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
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

template <int BN>
cudaError_t launch_bn(const CUtensorMap& tx, const CUtensorMap& tw, const GemmArgs& a, int mt, int nt, cudaStream_t s) {
    constexpr size_t smem = kStages * (BN * 128 + kWStage) + (3 * kStages + 1) * 8 + 16 + 1024;
    static bool configured[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !configured[dev]) {
        cudaError_t e = cudaFuncSetAttribute(gemm_w4_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(mt, nt, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemm_w4_kernel<BN>, tx, tw, a);
}

}  // namespace

cudaError_t launch_gemm(const void* Xr, const void* qw, const void* scp, const void* zp, void* Y, int64_t T,
                        int64_t in, int64_t out, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    PFN_cuTensorMapEncodeTiled_v12000 enc = get_encoder();
    if (!enc) return cudaErrorNotSupported;
    const int BN = T <= 64 ? 64 : T <= 128 ? 128 : 256;
    GemmArgs a{};
    a.T = (int)T;
    a.in = (int)in;
    a.out = (int)out;
    a.G = (int)(in / 128);
    a.Gp = a.G + (a.G & 1);
    a.nkb = (int)(in / 64);
    a.nrb = (int)(out / 16);
    a.sp = static_cast<const uint32_t*>(scp);
    a.zp = static_cast<const uint8_t*>(zp);
    a.Y = static_cast<__half*>(Y);

    CUtensorMap tx, tw;
    {   // X' [T][in] fp16: box 64 channels x BN tokens, 128-byte swizzle, zero fill past T
        cuuint64_t dims[2] = {(cuuint64_t)in, (cuuint64_t)T};
        cuuint64_t strides[1] = {(cuuint64_t)in * 2};
        cuuint32_t box[2] = {64u, (cuuint32_t)BN};
        cuuint32_t estr[2] = {1u, 1u};
        if (enc(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(Xr), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {   // packed int4 codes as uint32 [out/16][in/64 * 128]: box 128 words (one k block) x 8 row blocks
        cuuint64_t dims[2] = {(cuuint64_t)a.nkb * 128, (cuuint64_t)a.nrb};
        cuuint64_t strides[1] = {(cuuint64_t)a.nkb * 512};
        cuuint32_t box[2] = {128u, 8u};
        cuuint32_t estr[2] = {1u, 1u};
        if (enc(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(qw), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const int mt = (a.nrb + 7) / 8;
    const int nt = (int)((T + BN - 1) / BN);
    cudaError_t e;
    if (BN == 64) e = launch_bn<64>(tx, tw, a, mt, nt, s);
    else if (BN == 128) e = launch_bn<128>(tx, tw, a, mt, nt, s);
    else e = launch_bn<256>(tx, tw, a, mt, nt, s);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t read_fault(unsigned int* code, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(code, g_paro_fault, sizeof(unsigned int));
    if (e != cudaSuccess || !clear) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_paro_fault, &zero, sizeof(unsigned int));
}

}  // namespace paro
