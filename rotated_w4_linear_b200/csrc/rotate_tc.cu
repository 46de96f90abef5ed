// Activation rotation X' = X T^-1 on the 5th-generation tensor cores, for
// batches of many tokens (ParoQuant CSDN article, section 2.1: the activation
// side of Y = (X T^-1)(T W); paper notes, "key design": T = (prod R) diag(alpha)
// is block diagonal over the 128-channel groups).
//
// Per group g, diag(1/alpha) R_1^T ... R_K^T is one dense 128 x 128 matrix M_g
// (built once on the host in fp64 by applying the K Givens layers to the
// rows of diag(1/alpha)), so a group's channels of a token row become
// x' = x M_g: a [tokens x 128] x [128 x 128] product. M_g is stored as two
// fp16 matrices, hi = fp16(M_g) and lo = fp16(M_g - hi), and the MMAs form
// x hi + x lo with fp32 accumulation: the products of the exact fp16 inputs
// are exact in fp32, and hi + lo carries M_g to about 2^-22 relative, so the
// result is the fp32-accumulated rotation whatever K is. The cost per
// element is fixed (512 flops), below the HBM time of its 4 bytes.
//
// Work items are (group g, tile of 128 tokens) in group-major order; CTA c
// (one per SM) takes the contiguous run [c W / n, (c + 1) W / n) of the W
// items, so it meets few groups. Warp roles:
//   warp 0     TMA producer: per item the X tile (128 tokens x 128 channels
//              as two 64-channel boxes, 128-byte swizzle, rows past T read as
//              zeros) into a ring of S stages;
//   warp 1     allocates tensor memory (two 128-column fp32 accumulators);
//              one lane loads M_g (hi and lo, 64 KB, one bulk copy) when the
//              run enters group g, after the MMAs on the previous group's
//              matrices have completed, and issues 16 MMAs per item
//              (M = 128 tokens, N = 128 channels, K = 16; 8 k steps x hi, lo)
//              into accumulator j mod 2, committing to the epilogue;
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (one token row per
//              thread), fp32 -> fp16 (round to nearest even) into the item's
//              X stage (its MMAs are done with it) in the same swizzled
//              layout, then one thread TMA-stores the tile to X' and returns
//              the stage to the producer once the store has read it.
// Every wait is bounded (sm100.cuh); a wait that runs out raises the CTA's
// abort flag, the roles stop issuing work, issued copies and MMAs are waited
// for, and the CTA exits without storing.
#include <cuda.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace paro {

namespace {

constexpr uint32_t kHalfTile = 128 * 128;          // 16 KB: 128 rows x 64 fp16 (one 128-byte swizzle span)
constexpr uint32_t kXStage = 2 * kHalfTile;        // 32 KB: a 128-token x 128-channel tile
constexpr uint32_t kMatBytes = 4 * kHalfTile;      // 64 KB: hi (k 0-63, 64-127), lo (k 0-63, 64-127)
constexpr int kTcThreads = 192;

struct RotTcArgs {
    int G, ntiles;
    int64_t W;                // items: G x ntiles
    const uint8_t* mats;      // [G][kMatBytes] images of the B operand (shared-memory layout)
};

}  // namespace

template <int S>
__global__ void __launch_bounds__(kTcThreads, 1)
rotate_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_y,
                 const RotTcArgs a) {
    // the next kernel may launch its prologue now; it waits for this grid
    // to complete before it reads X'
    asm volatile("griddepcontrol.launch_dependents;");
    constexpr uint32_t kIdesc = umma_idesc_f16(128, 128);
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    unsigned char* sM = smem;                               // hi | lo of the current group
    unsigned char* sX = smem + kMatBytes;                   // S stages of X, then of X'
    uint64_t* bars = reinterpret_cast<uint64_t*>(sX + S * kXStage);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 3 * S + 7);
    volatile uint32_t* abort = tslot + 1;
    const uint32_t full0 = smem_addr(bars), empty0 = full0 + 8 * S, ready0 = empty0 + 8 * S;
    const uint32_t accf0 = ready0 + 8 * S, acce0 = accf0 + 16;
    const uint32_t mfull = acce0 + 16, mfree = mfull + 8, mdone = mfree + 8;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t w_lo = (int64_t)blockIdx.x * a.W / gridDim.x;
    const int64_t w_hi = (int64_t)(blockIdx.x + 1) * a.W / gridDim.x;
    const int n = (int)(w_hi - w_lo);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
            mbar_init(ready0 + 8 * s, 4);                   // one arrive per epilogue warp
        }
        for (int c = 0; c < 2; ++c) {
            mbar_init(accf0 + 8 * c, 1);
            mbar_init(acce0 + 8 * c, 4);                    // one arrive per epilogue warp
        }
        mbar_init(mfull, 1);
        mbar_init(mfree, 1);
        mbar_init(mdone, 1);
        *abort = 0u;
        mbar_fence_init();
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_y);
    }
    if (warp == 1) tmem_alloc(smem_addr(tslot), 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tslot;

    if (warp == 0) {
        if (lane == 0) {
            // X may be the previous grid's output: read it only after this wait
            asm volatile("griddepcontrol.wait;" ::: "memory");
            int issued[S];
#pragma unroll
            for (int s = 0; s < S; ++s) issued[s] = 0;
            for (int j = 0; j < n; ++j) {
                const int64_t w = w_lo + j;
                const int g = (int)(w / a.ntiles), tt = (int)(w - (int64_t)g * a.ntiles);
                const int s = j % S, u = j / S;
                if (u > 0 && !mbar_wait(empty0 + 8 * s, (u - 1) & 1, kFaultRotate + kFaultTmaWait, abort)) break;
                if (*abort) break;
                const uint32_t dst = smem_addr(sX + s * kXStage);
                mbar_arrive_expect_tx(full0 + 8 * s, kXStage);
                tma_load_2d(dst, &tm_x, g * 128, tt * 128, full0 + 8 * s);
                tma_load_2d(dst + kHalfTile, &tm_x, g * 128 + 64, tt * 128, full0 + 8 * s);
#pragma unroll
                for (int t = 0; t < S; ++t)
                    if (t == s) issued[t] = u + 1;
            }
            if (*abort) {   // drain: every issued load must land before the CTA exits
#pragma unroll
                for (int s = 0; s < S; ++s)
                    if (issued[s] > 0) mbar_wait(full0 + 8 * s, (issued[s] - 1) & 1, kFaultRotate + kFaultDrainWait, nullptr);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int cur_g = -1;
            uint32_t m_issued = 0, m_seen = 0, f_seen = 0;
            for (int j = 0; j < n; ++j) {
                const int64_t w = w_lo + j;
                const int g = (int)(w / a.ntiles);
                if (g != cur_g) {
                    if (cur_g >= 0) {   // the previous group's MMAs must be done before sM is replaced
                        umma_commit(mfree);
                        if (!mbar_wait(mfree, f_seen & 1, kFaultRotate + kFaultMmaWait, abort)) break;
                        ++f_seen;
                    }
                    mbar_arrive_expect_tx(mfull, kMatBytes);
                    bulk_load(smem_addr(sM), a.mats + (size_t)g * kMatBytes, kMatBytes, mfull);
                    ++m_issued;
                    if ((int64_t)(g + 1) * a.ntiles < w_hi)        // the run reaches the next group
                        bulk_prefetch_l2(a.mats + (size_t)(g + 1) * kMatBytes, kMatBytes);
                    if (!mbar_wait(mfull, m_seen & 1, kFaultRotate + kFaultMmaWait, abort)) break;
                    ++m_seen;
                    cur_g = g;
                }
                const int s = j % S, u = j / S, c = j & 1, v = j >> 1;
                if (!mbar_wait(full0 + 8 * s, u & 1, kFaultRotate + kFaultMmaWait, abort)) break;
                if (v > 0 && !mbar_wait(acce0 + 8 * c, (v - 1) & 1, kFaultRotate + kFaultMmaWait, abort)) break;
                tc_fence_after();
                const uint32_t d = tbase + (uint32_t)(c * 128);
                const uint32_t xs = smem_addr(sX + s * kXStage), ms = smem_addr(sM);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (uint32_t)(kk >> 2) * kHalfTile;
                    const uint64_t koff = (uint64_t)((kk & 3) * 2);        // 32 bytes in 16-byte units
                    const uint64_t adesc = umma_desc_sw128_kmajor(xs + off) + koff;
                    umma_f16_ss(d, adesc, umma_desc_sw128_kmajor(ms + off) + koff, kIdesc, kk > 0 ? 1u : 0u);
                    umma_f16_ss(d, adesc, umma_desc_sw128_kmajor(ms + 2 * kHalfTile + off) + koff, kIdesc, 1u);
                }
                umma_commit(accf0 + 8 * c);   // the accumulator is ready and the X stage is read
            }
            if (m_issued > m_seen)            // a matrix copy still in flight (after an abort)
                mbar_wait(mfull, m_seen & 1, kFaultRotate + kFaultDrainWait, nullptr);
            umma_commit(mdone);               // arrives once every MMA issued above has completed
        }
    } else {
        // ---- epilogue: warp w reads tensor-memory lanes 32 (w mod 4) .. +31 = token rows of the tile
        const int qw = warp & 3;
        const int r = 32 * qw + lane;
        const bool storer = threadIdx.x == 64;
        int prev_s = -1;
        for (int j = 0; j < n; ++j) {
            const int64_t w = w_lo + j;
            const int g = (int)(w / a.ntiles), tt = (int)(w - (int64_t)g * a.ntiles);
            const int s = j % S, u = j / S, c = j & 1, v = j >> 1;
            // tcgen05.ld is warp-collective: the warp goes on only if every lane saw the commit
            if (!__all_sync(0xffffffffu, mbar_wait(accf0 + 8 * c, v & 1, kFaultRotate + kFaultEpilogueWait, abort) && !*abort))
                break;
            tc_fence_after();
            const uint32_t st = smem_addr(sX + s * kXStage);
#pragma unroll
            for (int c0 = 0; c0 < 128; c0 += 32) {
                uint32_t acc[32];
                tmem_ld_32x32b_x32(tbase + (uint32_t)(c * 128 + c0) + ((uint32_t)(32 * qw) << 16), acc);
                tmem_wait_ld();
                // columns c0 .. c0 + 31 = four 16-byte chunks of the row in its 64-channel half
                const uint32_t half = st + (uint32_t)(c0 >> 6) * kHalfTile + (uint32_t)r * 128u;
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int chunk = ((c0 & 63) >> 3) + m;
                    const uint32_t addr = half + (uint32_t)((chunk ^ (r & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                                 "r"(pack_half2(__uint_as_float(acc[8 * m + 0]), __uint_as_float(acc[8 * m + 1]))),
                                 "r"(pack_half2(__uint_as_float(acc[8 * m + 2]), __uint_as_float(acc[8 * m + 3]))),
                                 "r"(pack_half2(__uint_as_float(acc[8 * m + 4]), __uint_as_float(acc[8 * m + 5]))),
                                 "r"(pack_half2(__uint_as_float(acc[8 * m + 6]), __uint_as_float(acc[8 * m + 7])))
                                 : "memory");
                }
            }
            tc_fence_before();
            fence_proxy_async_smem();                     // this thread's smem writes, visible to the TMA store
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(acce0 + 8 * c);               // the accumulator may be overwritten
                mbar_arrive(ready0 + 8 * s);              // this warp's rows of the tile are written
            }
            // (a stage barrier, not a named one: a warp that stops after an
            // abort leaves the storer with a bounded wait, not a hang; a warp
            // cannot reach this stage's next item before the store has read it)
            // (a failed wait raises the abort flag; the whole warp then leaves
            // at the next item's vote, so the storer does not leave alone)
            if (storer && mbar_wait(ready0 + 8 * s, u & 1, kFaultRotate + kFaultEpilogueWait, abort)) {
                tma_store_2d(&tm_y, st, g * 128, tt * 128);
                tma_store_2d(&tm_y, st + kHalfTile, g * 128 + 64, tt * 128);
                bulk_commit();
                bulk_wait_read<1>();                       // the previous item's stores have read their stage
                if (prev_s >= 0) mbar_arrive(empty0 + 8 * prev_s);
                prev_s = s;
            }
        }
        if (storer) bulk_wait<0>();                        // every store complete before the CTA exits
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        // no MMA may still write tensor memory when it is released
        mbar_wait(mdone, 0, kFaultRotate + kFaultDrainWait, nullptr);
        tc_fence_after();
        tmem_dealloc(tbase, 256);
    }
}

// 256-channel groups. x' = x M with M 256 x 256, computed per half h of the
// output channels as [128 tokens x 256] x [256 x 128]: CTA 2p + h computes
// half h for pair p's contiguous run of (group g, 128-token tile) items,
// group-major, so one half's matrix (hi and lo of 256 x 128, 128 KB) stays in
// shared memory for a run of tiles, and the two CTAs of a pair read each X
// tile at about the same time (the second read from L2). An item's X tile arrives as two 128-channel halves in
// two of S stages of 32 KB; each half feeds 16 MMAs (8 k steps x hi, lo),
// all into one accumulator. The stage of the first half is released by an
// MMA commit; the epilogue writes the fp16 result into the stage of the
// second half and one thread stores it with TMA, releasing that stage once
// the store has read it.
template <int S>
__global__ void __launch_bounds__(kTcThreads, 1)
rotate_tc256_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_y,
                    const RotTcArgs a) {
    asm volatile("griddepcontrol.launch_dependents;");
    constexpr uint32_t kIdesc = umma_idesc_f16(128, 128);
    constexpr uint32_t kMat = 8 * kHalfTile;               // 128 KB: hi (4 k quarters), lo (4 k quarters)
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    unsigned char* sM = smem;
    unsigned char* sX = smem + kMat;                        // S stages of one 128-channel half of a tile
    uint64_t* bars = reinterpret_cast<uint64_t*>(sX + S * kXStage);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 2 * S + 11);
    volatile uint32_t* abort = tslot + 1;
    const uint32_t full0 = smem_addr(bars), empty0 = full0 + 8 * S, ready0 = empty0 + 8 * S;
    const uint32_t accf0 = ready0 + 32, acce0 = accf0 + 16;
    const uint32_t mfull = acce0 + 16, mfree = mfull + 8, mdone = mfree + 8;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // CTAs 2p and 2p + 1 take the same run of (group, tile) pairs, one half
    // of the output channels each, so they read each X tile at about the same
    // time and the second read comes from L2
    const int h_cta = blockIdx.x & 1, npairs = gridDim.x >> 1, pair = blockIdx.x >> 1;
    const int64_t Wp = a.W >> 1;                            // (group, tile) pairs
    const int64_t w_lo = (int64_t)pair * Wp / npairs;
    const int64_t w_hi = (int64_t)(pair + 1) * Wp / npairs;
    const int n = (int)(w_hi - w_lo);
    auto item = [&](int j, int& g, int& h, int& tt) {
        const int64_t w = w_lo + j;
        g = (int)(w / a.ntiles);
        tt = (int)(w - (int64_t)g * a.ntiles);
        h = h_cta;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);                   // one release per use: an MMA commit or the storer
        }
        for (int r = 0; r < 4; ++r) mbar_init(ready0 + 8 * r, 4);   // item j mod 4: one arrive per epilogue warp
        for (int c = 0; c < 2; ++c) {
            mbar_init(accf0 + 8 * c, 1);
            mbar_init(acce0 + 8 * c, 4);
        }
        mbar_init(mfull, 1);
        mbar_init(mfree, 1);
        mbar_init(mdone, 1);
        *abort = 0u;
        mbar_fence_init();
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_y);
    }
    if (warp == 1) tmem_alloc(smem_addr(tslot), 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tslot;

    if (warp == 0) {
        if (lane == 0) {
            asm volatile("griddepcontrol.wait;" ::: "memory");   // X may be the previous grid's output
            int issued[S];
#pragma unroll
            for (int s = 0; s < S; ++s) issued[s] = 0;
            for (int j = 0; j < n && !*abort; ++j) {
                int g, h, tt;
                item(j, g, h, tt);
                for (int kh = 0; kh < 2; ++kh) {
                    const int idx = 2 * j + kh, s = idx % S, u = idx / S;
                    if (u > 0 && !mbar_wait(empty0 + 8 * s, (u - 1) & 1, kFaultRotate256 + kFaultTmaWait, abort)) break;
                    if (*abort) break;
                    const uint32_t dst = smem_addr(sX + s * kXStage);
                    mbar_arrive_expect_tx(full0 + 8 * s, kXStage);
                    tma_load_2d(dst, &tm_x, g * 256 + kh * 128, tt * 128, full0 + 8 * s);
                    tma_load_2d(dst + kHalfTile, &tm_x, g * 256 + kh * 128 + 64, tt * 128, full0 + 8 * s);
#pragma unroll
                    for (int t = 0; t < S; ++t)
                        if (t == s) issued[t] = u + 1;
                }
            }
            if (*abort) {
#pragma unroll
                for (int s = 0; s < S; ++s)
                    if (issued[s] > 0) mbar_wait(full0 + 8 * s, (issued[s] - 1) & 1, kFaultRotate256 + kFaultDrainWait, nullptr);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int cur = -1;
            uint32_t m_issued = 0, m_seen = 0, f_seen = 0;
            for (int j = 0; j < n; ++j) {
                int g, h, tt;
                item(j, g, h, tt);
                const int key = 2 * g + h;
                if (key != cur) {
                    if (cur >= 0) {
                        umma_commit(mfree);
                        if (!mbar_wait(mfree, f_seen & 1, kFaultRotate256 + kFaultMmaWait, abort)) break;
                        ++f_seen;
                    }
                    mbar_arrive_expect_tx(mfull, kMat);
                    bulk_load(smem_addr(sM), a.mats + (size_t)key * kMat, kMat, mfull);
                    ++m_issued;
                    if (g + 1 < a.G && (int64_t)(g + 1) * a.ntiles < w_hi)   // the run reaches the next group
                        bulk_prefetch_l2(a.mats + (size_t)(key + 2) * kMat, kMat);
                    if (!mbar_wait(mfull, m_seen & 1, kFaultRotate256 + kFaultMmaWait, abort)) break;
                    ++m_seen;
                    cur = key;
                }
                const int c = j & 1, v = j >> 1;
                if (v > 0 && !mbar_wait(acce0 + 8 * c, (v - 1) & 1, kFaultRotate256 + kFaultMmaWait, abort)) break;
                const uint32_t d = tbase + (uint32_t)(c * 128), ms = smem_addr(sM);
                bool ok = true;
                for (int kh = 0; kh < 2 && ok; ++kh) {
                    const int idx = 2 * j + kh, s = idx % S, u = idx / S;
                    if (!mbar_wait(full0 + 8 * s, u & 1, kFaultRotate256 + kFaultMmaWait, abort)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t xs = smem_addr(sX + s * kXStage);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t q = (uint32_t)(kh * 2 + (kk >> 2));          // k quarter of M
                        const uint64_t koff = (uint64_t)((kk & 3) * 2);
                        const uint64_t adesc = umma_desc_sw128_kmajor(xs + (uint32_t)(kk >> 2) * kHalfTile) + koff;
                        umma_f16_ss(d, adesc, umma_desc_sw128_kmajor(ms + q * kHalfTile) + koff, kIdesc,
                                    (kh | kk) ? 1u : 0u);
                        umma_f16_ss(d, adesc, umma_desc_sw128_kmajor(ms + 4 * kHalfTile + q * kHalfTile) + koff,
                                    kIdesc, 1u);
                    }
                    if (kh == 0) umma_commit(empty0 + 8 * s);       // the first half's stage is free after these
                }
                if (!ok) break;
                umma_commit(accf0 + 8 * c);
            }
            if (m_issued > m_seen) mbar_wait(mfull, m_seen & 1, kFaultRotate256 + kFaultDrainWait, nullptr);
            umma_commit(mdone);
        }
    } else {
        const int qw = warp & 3;
        const int r = 32 * qw + lane;
        const bool storer = threadIdx.x == 64;
        int prev_s = -1;
        for (int j = 0; j < n; ++j) {
            int g, h, tt;
            item(j, g, h, tt);
            const int c = j & 1, v = j >> 1, s1 = (2 * j + 1) % S;
            if (!__all_sync(0xffffffffu, mbar_wait(accf0 + 8 * c, v & 1, kFaultRotate256 + kFaultEpilogueWait, abort) && !*abort))
                break;
            tc_fence_after();
            const uint32_t st = smem_addr(sX + s1 * kXStage);
#pragma unroll
            for (int c0 = 0; c0 < 128; c0 += 32) {
                uint32_t acc[32];
                tmem_ld_32x32b_x32(tbase + (uint32_t)(c * 128 + c0) + ((uint32_t)(32 * qw) << 16), acc);
                tmem_wait_ld();
                const uint32_t half = st + (uint32_t)(c0 >> 6) * kHalfTile + (uint32_t)r * 128u;
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int chunk = ((c0 & 63) >> 3) + m;
                    const uint32_t addr = half + (uint32_t)((chunk ^ (r & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                                 "r"(pack_half2(__uint_as_float(acc[8 * m + 0]), __uint_as_float(acc[8 * m + 1]))),
                                 "r"(pack_half2(__uint_as_float(acc[8 * m + 2]), __uint_as_float(acc[8 * m + 3]))),
                                 "r"(pack_half2(__uint_as_float(acc[8 * m + 4]), __uint_as_float(acc[8 * m + 5]))),
                                 "r"(pack_half2(__uint_as_float(acc[8 * m + 6]), __uint_as_float(acc[8 * m + 7])))
                                 : "memory");
                }
            }
            tc_fence_before();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(acce0 + 8 * c);
                mbar_arrive(ready0 + 8 * (j & 3));
            }
            // (items j and j + 4 share a ready barrier: no warp reaches item
            // j + 4 before every warp has read item j + 2's accumulator,
            // which comes after the storer's wait for item j)
            if (storer && mbar_wait(ready0 + 8 * (j & 3), (j >> 2) & 1, kFaultRotate256 + kFaultEpilogueWait, abort)) {
                tma_store_2d(&tm_y, st, g * 256 + h * 128, tt * 128);
                tma_store_2d(&tm_y, st + kHalfTile, g * 256 + h * 128 + 64, tt * 128);
                bulk_commit();
                bulk_wait_read<1>();
                if (prev_s >= 0) mbar_arrive(empty0 + 8 * prev_s);
                prev_s = s1;
            }
        }
        if (storer) bulk_wait<0>();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        mbar_wait(mdone, 0, kFaultRotate256 + kFaultDrainWait, nullptr);
        tc_fence_after();
        tmem_dealloc(tbase, 256);
    }
}

namespace {

constexpr int kTcStages = 5;

template <int S>
constexpr size_t tc_smem() {
    return kMatBytes + S * kXStage + (3 * S + 8) * 8 + 1024;
}

}  // namespace

namespace {

template <typename Kern>
cudaError_t configure_once(Kern kern, size_t smem, std::atomic<bool>* configured, std::mutex& mu, int dev) {
    if (!configured[dev].load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> lock(mu);
        if (!configured[dev].load(std::memory_order_relaxed)) {
            const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            configured[dev].store(true, std::memory_order_release);
        }
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_rotate_tc(const RotDev& r, const void* X, void* Xr, int64_t T, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    if (!r.mats) return cudaErrorInvalidValue;
    const bool g256 = r.group == 256;
    constexpr int S = kTcStages, S256 = 3;
    constexpr size_t smem = tc_smem<S>();
    constexpr size_t smem256 = 8 * kHalfTile + S256 * kXStage + (2 * S256 + 12) * 8 + 1024;
    static std::atomic<bool> configured[64] = {}, configured256[64] = {};
    static std::mutex mu;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    const cudaError_t ce = g256 ? configure_once(rotate_tc256_kernel<S256>, smem256, configured256, mu, dev)
                                : configure_once(rotate_tc_kernel<S>, smem, configured, mu, dev);
    if (ce != cudaSuccess) return ce;
    CUtensorMap tm[2];
    // X and X' [T][in] fp16: box 64 channels x 128 tokens, 128-byte swizzle
    if (!encode_tma_2d(&tm[0], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, X, (uint64_t)r.in, (uint64_t)T, (uint64_t)r.in * 2,
                       64u, 128u, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tma_2d(&tm[1], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Xr, (uint64_t)r.in, (uint64_t)T, (uint64_t)r.in * 2,
                       64u, 128u, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    RotTcArgs a{};
    a.G = r.G;
    a.ntiles = (int)((T + 127) / 128);
    a.W = (int64_t)a.G * a.ntiles * (g256 ? 2 : 1);
    a.mats = r.mats;
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaLaunchConfig_t cfg{};
    // group 256: an even grid of CTA pairs (one per half of the output channels)
    const int64_t ctas = g256 ? 2 * std::min<int64_t>(a.W / 2, sms / 2) : std::min<int64_t>(a.W, sms);
    cfg.gridDim = dim3((unsigned)ctas, 1, 1);
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = g256 ? smem256 : smem;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    const cudaError_t e = g256 ? cudaLaunchKernelEx(&cfg, rotate_tc256_kernel<S256>, tm[0], tm[1], a)
                               : cudaLaunchKernelEx(&cfg, rotate_tc_kernel<S>, tm[0], tm[1], a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace paro
