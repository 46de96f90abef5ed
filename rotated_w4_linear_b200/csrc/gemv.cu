// Decode kernel for tokens <= 16: Y[T][out] = X' w_hat^T with X' = X T^-1
// already in global memory (written by the rotation kernel launched just
// before on the same stream). The int4 weight stream dominates: HBM bound.
//
// Launch: a grid of (nsplit, rowtiles) CTAs of 16 warps, one per SM; CTAs with the same
// row tile form one thread-block cluster along x, each owning a k-chunk of
// KC 128-channel groups. The kernel is a programmatic dependent launch: it
// starts while the kernel before it still runs, streams its first weights,
// and waits (griddepcontrol.wait) before it reads X'. It lets the next
// kernel launch early in turn.
//
//   work split: the CTA's (row block of 16 rows, 128-channel group) units in
//     row-block-major order are cut into sixteen contiguous runs that differ
//     by at most one unit, one per warp; a warp walks its run in items of up
//     to two groups (2 KB of int4 codes + scales + zeros) that stay inside
//     one row block;
//   weight stream: each warp streams its run through a private 3-stage
//     shared-memory ring with cp.async (16-byte global->shared copies that
//     bypass the registers): one commit group per item, wait on the oldest,
//     so two items are in flight while one is consumed;
//   X': the CTA copies its X' chunk (all tokens, zero rows >= T) into shared
//     memory, one warp per token row; the decode rotation kernel writes X'
//     already in the lane-major order the B fragments read;
//   math: each 32-bit int4 word is dequantised in registers (LOP3 into the
//     1024 + q bit pattern, exact fp16 subtraction of 1024 + z, one rounded
//     fp16 multiply: w_hat = fp16((q - z) s)) straight into an m16n8k16 A
//     fragment; the B fragment (four consecutive channels of one token) comes
//     from shared memory; fp32 accumulation in two independent chains, added
//     into the CTA's partial tile [token][row] (shared-memory atomics) when
//     the warp's run leaves a row block;
//   split-k: after a cluster barrier CTA x sums its slice of the rows over
//     the cluster's tiles with distributed shared memory loads and stores it
//     as fp16. No global atomics, no workspace.
// The k order inside each 16x16 tile follows the packed layout: the MMA's
// logical k slot 2q+e holds channel 4q+e and slot 2q+8+e channel 4q+2+e.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"
#include "kernels.h"

namespace paro {

namespace {

constexpr int kWarps = 16;
constexpr int kStages = 3;
constexpr int kMaxSplit = 16;                             // largest cluster (k-chunks per row tile)
constexpr int kItemGroups = 2;                            // 128-channel groups per item
constexpr int kItemQBytes = kItemGroups * 2 * 512;        // int4 codes
// GS: quantisation groups per 128 channels (1: group 128, 2: group 64); an
// item carries codes, then GS scale words x 8 per group, then GS zero bytes x 8
template <int GS>
constexpr int item_bytes() { return kItemQBytes + kItemGroups * GS * 32 + kItemGroups * GS * 8; }

struct GemvArgs {
    const __half* Xr;     // [T][in] fp16, already rotated
    int T, in, out, G;    // G: 128-channel groups
    int Gq, Gqp;          // quantisation groups (scales and zeros) along in; Gqp rounded up to even
    int KC;               // groups per k-chunk (last chunk may be shorter)
    int RT;               // row blocks per CTA
    int nsplit;           // k-chunks = cluster size along x
    int share;            // rows of the tile each cluster CTA finalises (multiple of 16)
    const uint4* qw;
    const uint32_t* sp;
    const uint8_t* zp;
    const __half* bias;   // [out] fp16 or null
    __half* Y;            // fp16 [T][out], or
    float* Yf;            // fp32 [T][out] unrounded sums (row-parallel partials) when not null
    int xlm;              // X' already lane-major within 64-channel blocks
};

// Not volatile: the MMA reads registers only, so the compiler may schedule
// it freely against the shared-memory loads and the dequantisation.
__device__ __forceinline__ void mma16816(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// 16-byte global -> shared copies (bypassing L1) under a predicate that is
// evaluated inside the asm, so a condition costs one setp instead of a
// divergent branch around the copy.
__device__ __forceinline__ void cp_async16_if(bool pred, uint32_t dst, const void* src) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %2, 0;\n\t@p cp.async.cg.shared.global [%0], [%1], 16;\n\t}"
                 ::"r"(dst), "l"(src), "r"((int)pred) : "memory");
}
// 8 bytes, 8-byte aligned, through L1
__device__ __forceinline__ void cp_async8_if(bool pred, uint32_t dst, const void* src) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %2, 0;\n\t@p cp.async.ca.shared.global [%0], [%1], 8;\n\t}"
                 ::"r"(dst), "l"(src), "r"((int)pred) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ float4 ld_dsmem4(uint32_t addr) {   // 16-byte aligned
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Cluster barrier without memory ordering: for the last barrier, which only
// keeps each CTA's shared memory alive until the other CTAs' reads of it are
// done (their values are already used). A release here would also wait for
// this CTA's global stores of Y to complete, about a microsecond.
__device__ __forceinline__ void cluster_sync_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}

// A lane's source pointers for the items of one row block: codes (the
// lane's 16 bytes of each 512-byte k block), scales (lanes 0..2 GS - 1: 16
// bytes each) and zeros (the last 2 GS lanes: 8 bytes per quantisation
// group). Within a row block the next 128-channel group is 1 KB, 32 GS B and
// 8 GS B further on.
struct ItemSrc {
    const uint4* q;
    const uint32_t* sc;
    const uint8_t* z;
};

template <int GS>
__device__ __forceinline__ ItemSrc item_src(const GemvArgs& a, int rb, int g0, int lane) {
    const int nkb = a.in >> 6;
    ItemSrc p;
    p.q = a.qw + ((size_t)rb * nkb + 2 * g0) * 32 + lane;
    p.sc = a.sp + ((size_t)rb * a.Gq + GS * g0) * 8 + lane * 4;
    p.z = a.zp + ((size_t)rb * a.Gqp + GS * g0) * 8;
    return p;
}

// Copy one item (groups g0, g0+1 if ng == 2 of the source's row block) into
// a ring slot; `dst` is the slot address plus this lane's 16-byte offset.
// Slot layout: codes [2 ng][512 B], scales [GS ng][32 B] at kItemQBytes,
// zeros [GS ng][8 B] after the scales of kItemGroups groups.
template <int GS>
__device__ __forceinline__ void issue_item(const ItemSrc& p, uint32_t slot, uint32_t dst, int ng, int lane) {
#pragma unroll
    for (int kb = 0; kb < 2 * kItemGroups; ++kb) cp_async16_if(kb < 2 * ng, dst + kb * 512, p.q + kb * 32);
    cp_async16_if(lane < 2 * GS * ng, slot + kItemQBytes + lane * 16, p.sc);
    // zeros: 8 bytes per quantisation group from the last lanes (an item may
    // start at an odd group, so a pair need not be 16-byte aligned)
    const int zg = lane - (32 - kItemGroups * GS);
    cp_async8_if(zg >= 0 && zg < GS * ng, slot + kItemQBytes + kItemGroups * GS * 32 + 8 * zg, p.z + 8 * zg);
}

}  // namespace

template <int NT, int GS>
__global__ void __launch_bounds__(kWarps * 32, 1) gemv_kernel(const GemvArgs a) {
    constexpr int kItemBytes = item_bytes<GS>();
    // When the next kernel on the stream may launch (it prefetches only its
    // weights, or its tables, before it waits for this grid to complete):
    // at 8 tokens or fewer right away; above that once every warp of the CTA
    // has at most one item left, so that the next rotation kernel's CTAs land
    // on SMs as this grid's CTAs leave instead of crowding the few SMs this
    // grid left free (measured at 12 and 16 tokens: the trigger at the start
    // costs about 2 us per layer of four projections, the one after the
    // mainloop about 0.6 us more than this one; at 1 token the late trigger
    // costs 0.5-1 us per projection). Warps without work trigger at the end.
    if (NT == 1) asm volatile("griddepcontrol.launch_dependents;");
    extern __shared__ __align__(16) unsigned char smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int chunk = blockIdx.x, rt = blockIdx.y;
    const int g_begin = chunk * a.KC;
    const int g_end = min(a.G, g_begin + a.KC);
    const int ncg = max(0, g_end - g_begin);
    const int nrb = a.out >> 4;
    const int rb_begin = rt * a.RT;
    const int nrbt = max(0, min(nrb, rb_begin + a.RT) - rb_begin);
    // The CTA's (row block, group) units in row-block-major order, flattened
    // as f = (rb - rb_begin) ncg + (g - g_begin); warp w takes the contiguous
    // run [F w / 16, F (w + 1) / 16) of the F units (runs differ by at most
    // one group) and walks it in items of up to two groups that end at a row
    // block's last group or at the run's end.
    const int F = nrbt * ncg;
    const int f_lo = (int)(((int64_t)F * warp) / kWarps);
    const int f_hi = (int)(((int64_t)F * (warp + 1)) / kWarps);
    const int rbl_lo = ncg ? f_lo / ncg : 0;                // first row block (tile-local) and group
    const int g_lo = g_begin + (ncg ? f_lo - rbl_lo * ncg : 0);

    const int XS = a.KC * 128 + 8;                         // halves; row stride == 16 bytes mod 128
    const int SR = a.RT * 16 + 4;                          // floats per token row of the partial tile
    __half* xs = reinterpret_cast<__half*>(smem);
    float* red = reinterpret_cast<float*>(smem + (size_t)NT * 8 * XS * 2);
    unsigned char* ring = reinterpret_cast<unsigned char*>(red + NT * 8 * SR);
    const uint32_t ring_w = smem_u32(ring) + (uint32_t)(warp * kStages * kItemBytes);

    // producer cursor: position, row block and group of the next item to
    // copy and the lane's source pointers, advanced incrementally
    int p_f = f_lo, p_rb = rb_begin + rbl_lo, p_g = g_lo;
    ItemSrc src = item_src<GS>(a, p_rb, p_g, lane);
    auto issue_next = [&](int stage) {
        const int ng = min(min(kItemGroups, g_end - p_g), f_hi - p_f);
        const uint32_t slot = ring_w + stage * kItemBytes;
        issue_item<GS>(src, slot, slot + lane * 16, ng, lane);
        p_f += ng;
        p_g += ng;
        if (p_g == g_end) {
            p_g = g_begin;
            ++p_rb;
            src = item_src<GS>(a, p_rb, g_begin, lane);
        } else {
            src.q += ng * 2 * 32;
            src.sc += ng * GS * 8;
            src.z += ng * GS * 8;
        }
    };

    // ---- weight stream prologue: first kStages-1 items in flight (weights
    // are never written by the kernels this one may overlap)
#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) {
        if (p_f < f_hi) issue_next(s);
        cp_async_commit();
    }

    // ---- X' chunk and partial tile (waits for the previous grid: X' may be its output)
    // Unrotated calls: L2 prefetch of the X chunk (one 128-byte line per
    // thread and pass). A prefetch returns no data, so it may run before the
    // wait even if X is the previous grid's output; it saves the DRAM latency
    // when X is not in L2. (A rotated X' was just written by the rotation
    // kernel and sits in L2.)
    if (!a.xlm)
        for (int i = threadIdx.x; i < NT * 8 * 2 * ncg; i += kWarps * 32) {
            const int tok = i / (2 * ncg), l = i - tok * 2 * ncg;
            if (tok < a.T)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(a.Xr + (size_t)tok * a.in + (size_t)g_begin * 128 + l * 64));
        }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    {
        // all of the chunk's copies are in flight at once (cp.async; rows
        // >= T are zero-filled by a source size of 0), then one wait. Within
        // each 64-channel block the row is stored lane-major: channel
        // 16 j + 4 q + e at position 16 q + 4 j + e, so lane q of a fragment
        // row finds the four k tiles' B values in 32 contiguous bytes. Warp w
        // copies token row w mod 8 NT (two warps per row when NT == 1).
        constexpr int kRows = NT * 8, kParts = kWarps / kRows;
        const int tok = warp & (kRows - 1), part = warp / kRows;
        const bool real = tok < a.T;
        const unsigned char* srow =
            reinterpret_cast<const unsigned char*>(a.Xr + (size_t)(real ? tok : 0) * a.in + (size_t)g_begin * 128);
        const uint32_t drow = smem_u32(xs + (size_t)tok * XS);
        if (a.xlm) {                                       // the rotation wrote that order: a plain copy
            const int n16 = ncg * 16;
            for (int v = part * 32 + lane; v < n16; v += 32 * kParts)
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(drow + 16 * v), "l"(srow + 16 * v),
                             "r"(real ? 16 : 0) : "memory");
        } else {                                           // natural order: 8-byte pieces of 4 channels
            const int n8 = ncg * 32;
            for (int v = part * 32 + lane; v < n8; v += 32 * kParts) {
                const int blk = v >> 4, j = (v >> 2) & 3, q = v & 3;   // channel 64 blk + 16 j + 4 q
                asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(drow + 2 * (blk * 64 + 16 * q + 4 * j)),
                             "l"(srow + 8 * v), "r"(real ? 8 : 0) : "memory");
            }
        }
        cp_async_commit();
        for (int i = threadIdx.x; i < NT * 8 * SR; i += kWarps * 32) red[i] = 0.f;
        cp_async_wait<0>();                                // (the first weight items are in by now too)
    }
    __syncthreads();

    // ---- mainloop: fp32 sums of the current row block in registers, added
    // into the CTA's partial tile red[token][row] when the row block changes
    const int gq = lane >> 2, qd = lane & 3;
    // Shared memory is read through plain C++ loads (not asm), so the compiler
    // sees them as memory accesses: it can hoist them for latency but not
    // across the cp.async waits and warp barriers that order the ring.
    const unsigned char* xrow[NT];                         // this lane's B rows
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
        xrow[nt] = reinterpret_cast<const unsigned char*>(xs + (size_t)(nt * 8 + gq) * XS + 16 * qd);
    const unsigned char* ring_p = ring + (size_t)warp * kStages * kItemBytes;
    float acc[NT][2][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c) acc[nt][c][0] = acc[nt][c][1] = acc[nt][c][2] = acc[nt][c][3] = 0.f;
    auto flush = [&](int rbl) {
        float* base = red + rbl * 16 + gq;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int t = nt * 8 + 2 * qd + e;
                atomicAdd(base + t * SR, acc[nt][0][e] + acc[nt][1][e]);
                atomicAdd(base + t * SR + 8, acc[nt][0][2 + e] + acc[nt][1][2 + e]);
            }
#pragma unroll
            for (int c = 0; c < 2; ++c) acc[nt][c][0] = acc[nt][c][1] = acc[nt][c][2] = acc[nt][c][3] = 0.f;
        }
    };
    int c_f = f_lo, c_rbl = rbl_lo, c_g = g_lo;            // item being consumed
    bool pending = false;                                  // sums not yet flushed
    bool trig = false;
    int stage = 0, pstage = kStages - 1;
    while (c_f < f_hi) {
        if (p_f < f_hi) issue_next(pstage);
        cp_async_commit();
        pstage = (pstage + 1 == kStages) ? 0 : pstage + 1;
        cp_async_wait<kStages - 1>();
        __syncwarp();

        const unsigned char* slot = ring_p + stage * kItemBytes;
        const int ng = min(min(kItemGroups, g_end - c_g), f_hi - c_f);   // as the producer chose
        const int kb_off = (c_g - g_begin) * 128 * 2;      // bytes into the X' rows
#pragma unroll
        for (int g = 0; g < kItemGroups; ++g) {
            if (g < ng) {
                uint32_t sc0, sc1;
                Zero2 zc = zero_consts(slot[kItemQBytes + kItemGroups * GS * 32 + GS * g * 8 + gq]);
                scale_pairs(*reinterpret_cast<const uint32_t*>(slot + kItemQBytes + GS * g * 32 + gq * 4), sc0, sc1);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (GS == 2 && h == 1) {                   // group 64: the second half has its own s, z
                        zc = zero_consts(slot[kItemQBytes + kItemGroups * GS * 32 + (GS * g + 1) * 8 + gq]);
                        scale_pairs(*reinterpret_cast<const uint32_t*>(slot + kItemQBytes + (GS * g + 1) * 32 + gq * 4),
                                    sc0, sc1);
                    }
                    const uint4 wv = *reinterpret_cast<const uint4*>(slot + (2 * g + h) * 512 + lane * 16);
                    const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
                    // B values of the block's four k tiles: two 16-byte loads per token tile
                    const int bbyte = kb_off + (g * 128 + h * 64) * 2;
                    uint4 bq[NT][2];
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        bq[nt][0] = *reinterpret_cast<const uint4*>(xrow[nt] + bbyte);
                        bq[nt][1] = *reinterpret_cast<const uint4*>(xrow[nt] + bbyte + 16);
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t hh[4];
                        dequant_word(words[j], zc, sc0, sc1, hh);
                        const uint32_t A[4] = {hh[0], hh[2], hh[1], hh[3]};
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const uint4& b4 = bq[nt][j >> 1];
                            mma16816(acc[nt][j & 1], A, (j & 1) ? b4.z : b4.x, (j & 1) ? b4.w : b4.y);
                        }
                    }
                }
            }
        }
        __syncwarp();                                      // the slot may be refilled from here on
        stage = (stage + 1 == kStages) ? 0 : stage + 1;
        c_f += ng;
        c_g += ng;
        pending = true;
        if (NT == 2 && !trig && f_hi - c_f <= kItemGroups) {   // one item left at most
            asm volatile("griddepcontrol.launch_dependents;");
            trig = true;
        }
        if (c_g == g_end) {                                // row block done
            flush(c_rbl);
            pending = false;
            c_g = g_begin;
            ++c_rbl;
        }
    }
    if (pending) flush(c_rbl);                             // run ended inside a row block
    if (NT == 2) asm volatile("griddepcontrol.launch_dependents;");
    cp_async_wait<0>();
    __syncthreads();

    // ---- split-k: CTA x of the cluster sums its share of the rows over all
    // the cluster's tiles (distributed shared memory loads) and stores fp16
    const int nrows_tile = nrbt * 16;
    const int row0 = rb_begin * 16;
    if (a.nsplit == 1) {
        for (int i = threadIdx.x; i < a.T * nrows_tile; i += kWarps * 32) {
            const int t = i / nrows_tile, r = i - t * nrows_tile;
            const float b = a.bias ? __half2float(a.bias[row0 + r]) : 0.f;
            if (a.Yf) a.Yf[(size_t)t * a.out + row0 + r] = red[t * SR + r] + b;
            else a.Y[(size_t)t * a.out + row0 + r] = __float2half_rn(red[t * SR + r] + b);
        }
        return;
    }
    cluster_sync();
    const int rlo = chunk * a.share;
    const int n = max(0, min(a.share, nrows_tile - rlo));
    const uint32_t red_local = smem_u32(red);
    // four rows per thread (n is a multiple of 16); the loads from all the
    // cluster's tiles are issued before any is used, so their latencies overlap
    const int n4 = n >> 2;
    for (int i = threadIdx.x; i < a.T * n4; i += kWarps * 32) {
        const int t = i / n4, r = rlo + 4 * (i - t * n4);
        const uint32_t off = red_local + (uint32_t)(t * SR + r) * 4u;
        float4 part[kMaxSplit];
#pragma unroll
        for (int x = 0; x < kMaxSplit; ++x)
            if (x < a.nsplit) part[x] = ld_dsmem4(mapa(off, (uint32_t)x));
        float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int x = 0; x < kMaxSplit; ++x)
            if (x < a.nsplit) {
                sum.x += part[x].x;
                sum.y += part[x].y;
                sum.z += part[x].z;
                sum.w += part[x].w;
            }
        if (a.bias) {
            sum.x += __half2float(a.bias[row0 + r]);
            sum.y += __half2float(a.bias[row0 + r + 1]);
            sum.z += __half2float(a.bias[row0 + r + 2]);
            sum.w += __half2float(a.bias[row0 + r + 3]);
        }
        if (a.Yf)
            *reinterpret_cast<float4*>(a.Yf + (size_t)t * a.out + row0 + r) = sum;
        else
            *reinterpret_cast<uint2*>(a.Y + (size_t)t * a.out + row0 + r) =
                make_uint2(pack_half2(sum.x, sum.y), pack_half2(sum.z, sum.w));
    }
    cluster_sync_relaxed();                                // tiles stay alive until every reader is done
}

namespace {

struct GemvPlan {
    int KC, nsplit, RT, rowtiles, share;
    size_t smem;
};

size_t gemv_smem(int NT, int GS, int KC, int RT) {
    return (size_t)NT * 8 * (KC * 128 + 8) * 2 + (size_t)NT * 8 * (RT * 16 + 4) * 4 +
           (size_t)kWarps * kStages * (GS == 2 ? item_bytes<2>() : item_bytes<1>());
}

// CTAs of one launch that can be resident at once: clusters of `nsplit` CTAs
// must sit inside one GPC, so for nsplit > 1 this is the driver's count of
// co-resident clusters times nsplit (fewer than SMs x CTAs per SM).
template <int NT, int GS>
int gemv_slots(int dev, int nsplit, int per_sm) {
    static std::mutex mu;
    static std::map<std::tuple<int, int, int>, int> cache;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_tuple(dev, nsplit, per_sm);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int slots = sms * per_sm;
    if (nsplit > 1 && cudaFuncSetAttribute(gemv_kernel<NT, GS>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                          cudaSuccess) {
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(nsplit, 1024, 1);
        cfg.blockDim = dim3(kWarps * 32, 1, 1);
        cfg.dynamicSmemBytes = per_sm >= 2 ? 100 * 1024 : 160 * 1024;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = nsplit;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int nc = 0;
        if (cudaFuncSetAttribute(gemv_kernel<NT, GS>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) ==
                cudaSuccess &&
            cudaOccupancyMaxActiveClusters(&nc, gemv_kernel<NT, GS>, &cfg) == cudaSuccess && nc > 0)
            slots = std::min(slots, nc * nsplit);
        cudaGetLastError();   // a refused query leaves the SM-count estimate
    }
    cache[key] = slots;
    return slots;
}

// Choose (k-chunk, row tile) for one shape: minimise waves x (items per warp
// + pipeline fill), counting only CTAs that can be resident together.
template <int NT, int GS>
GemvPlan plan_gemv(int dev, int64_t in, int64_t out, int T, int K) {
    const int G = (int)(in / 128);
    const int nrb = (int)(out / 16);
    const int kc_max = NT == 2 ? 20 : 40;                 // X' chunk <= ~82 KB (one CTA per SM)
    constexpr size_t kSmemPerSm = 228 * 1024, kReserved = 1024;
    const size_t rot_reserve = K > 0 ? rotate_decode_smem(K, T) + kReserved : 0;
    GemvPlan best{};
    double best_cost = 1e30;
    for (int nsplit = 1; nsplit <= 16; ++nsplit) {
        int KC = (G + nsplit - 1) / nsplit;
        if (nsplit > 1) KC += KC & 1;
        if (KC > kc_max) continue;
        const int ns = (G + KC - 1) / KC;
        if (ns != nsplit) continue;
        for (int RT = 1; RT <= std::min(nrb, 64); ++RT) {
            const size_t smem = gemv_smem(NT, GS, KC, RT);
            if (smem > 200 * 1024) break;
            // one CTA of 16 warps per SM (one copy of the X' chunk per SM),
            // with room beside it for one CTA of the rotation kernel that
            // runs before this one
            if (smem + kReserved + rot_reserve > kSmemPerSm) break;
            const int per_sm = 1;
            const int slots = gemv_slots<NT, GS>(dev, ns, per_sm);
            const int rowtiles = (nrb + RT - 1) / RT;
            const int ctas = ns * rowtiles;
            const int waves = (ctas + slots - 1) / slots;
            // items per warp: runs of ceil(RT KC / 16) groups in items of two
            const double per_warp = std::ceil((double)RT * KC / kWarps) / kItemGroups;
            // +3: pipeline fill and epilogue per CTA; a partly empty wave
            // still costs its share of HBM time; a split-k cluster adds its
            // barrier and distributed-shared-memory reduction, measured at
            // about 1.5 items' time (plan sweeps of Qwen3- and Llama-shaped
            // layers at 1 and 8 tokens)
            const double fill = (double)ctas / ((double)waves * slots);
            const double cost = waves * (per_warp + 3.0) * (1.0 + 0.3 * (1.0 - fill)) + 0.05 * ns +
                                (ns > 1 ? 1.5 : 0.0);
            if (cost < best_cost - 1e-9) {
                best_cost = cost;
                best.KC = KC;
                best.nsplit = ns;
                best.RT = RT;
                best.rowtiles = rowtiles;
                best.smem = smem;
            }
        }
    }
    best.share = 16 * ((best.RT + best.nsplit - 1) / best.nsplit);
    return best;
}

template <int NT, int GS>
GemvPlan cached_plan(int dev, int64_t in, int64_t out, int T, int K) {
    static std::mutex mu;
    static std::map<std::tuple<int, int64_t, int64_t, int, int>, GemvPlan> cache;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_tuple(dev, in, out, T, K);
    auto it = cache.find(key);
    if (it == cache.end()) it = cache.emplace(key, plan_gemv<NT, GS>(dev, in, out, T, K)).first;
    return it->second;
}

template <int NT, int GS>
cudaError_t launch_gemv_t(const GemvArgs& a, const GemvPlan& p, int dev, cudaStream_t s) {
    // kernel attributes, set once per device (double-checked under a lock)
    static std::atomic<bool> configured[64] = {};
    static std::mutex mu;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev].load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> lock(mu);
        if (!configured[dev].load(std::memory_order_relaxed)) {
            cudaError_t e =
                cudaFuncSetAttribute(gemv_kernel<NT, GS>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(gemv_kernel<NT, GS>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (e != cudaSuccess) return e;
            configured[dev].store(true, std::memory_order_release);
        }
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(p.nsplit, p.rowtiles, 1);
    cfg.blockDim = dim3(kWarps * 32, 1, 1);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.nsplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // programmatic dependent launch: the weight prologue overlaps the tail of
    // the previous kernel; griddepcontrol.wait guards every read of X'
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, gemv_kernel<NT, GS>, a);
}

}  // namespace

// Decode: the rotation kernel writes X' = X T^-1 into ws (when rot is not
// null), then the decode kernel runs on it; both are programmatic dependent
// launches, so the decode kernel's weight stream starts during the rotation.
cudaError_t launch_gemv(const RotDev* rot, const void* X, const void* qw, const void* scp, const void* zp,
                        const void* bias, void* Y, int64_t T, int64_t in, int64_t out, int group, void* ws,
                        cudaStream_t s, bool y_fp32) {
    if (T <= 0) return cudaSuccess;
    if (group != 64 && group != 128) return cudaErrorInvalidValue;
    const bool g64 = group == 64;
    int dev = 0;
    cudaGetDevice(&dev);
    const int K = rot ? rot->K : 0;
    const void* xr = X;
    bool lane_major = false;
    if (rot && rot->group == 256) {   // no Givens tables: the tensor-core rotation, natural channel order
        cudaError_t e = launch_rotate_tc(*rot, X, ws, T, s);
        if (e != cudaSuccess) return e;
        xr = ws;
    } else if (rot) {
        cudaError_t e = launch_rotate_decode(*rot, X, ws, T, s, true);
        if (e != cudaSuccess) return e;
        xr = ws;
        lane_major = true;
    }
    const GemvPlan p = (T > 8) ? (g64 ? cached_plan<2, 2>(dev, in, out, (int)T, K) : cached_plan<2, 1>(dev, in, out, (int)T, K))
                               : (g64 ? cached_plan<1, 2>(dev, in, out, (int)T, K) : cached_plan<1, 1>(dev, in, out, (int)T, K));
    GemvArgs a{};
    a.Xr = static_cast<const __half*>(xr);
    a.T = (int)T;
    a.in = (int)in;
    a.out = (int)out;
    a.G = (int)(in / 128);
    a.Gq = (int)(in / group);
    a.Gqp = a.Gq + (a.Gq & 1);
    a.KC = p.KC;
    a.RT = p.RT;
    a.nsplit = p.nsplit;
    a.share = p.share;
    a.qw = static_cast<const uint4*>(qw);
    a.sp = static_cast<const uint32_t*>(scp);
    a.zp = static_cast<const uint8_t*>(zp);
    a.bias = static_cast<const __half*>(bias);
    a.Y = y_fp32 ? nullptr : static_cast<__half*>(Y);
    a.Yf = y_fp32 ? static_cast<float*>(Y) : nullptr;
    a.xlm = lane_major ? 1 : 0;
    cudaError_t e = (T > 8) ? (g64 ? launch_gemv_t<2, 2>(a, p, dev, s) : launch_gemv_t<2, 1>(a, p, dev, s))
                            : (g64 ? launch_gemv_t<1, 2>(a, p, dev, s) : launch_gemv_t<1, 1>(a, p, dev, s));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Decode without any allocation by the caller or by the library.
//
// Some callers cannot allocate device memory for a workspace: a serving
// engine that reserves all device memory for its own pool up front, or code
// that must not call cudaMalloc while a CUDA graph is being captured. For
// them the decode path can keep its only scratch (X T^-1, tokens x in fp16)
// in this file-scope array instead. It lives on every device that loads the
// library until the process exits. All calls share it and it keeps the last
// call's contents (X T^-1 is fully written before it is read, so nothing needs
// clearing); calls that overlap on the GPU race on it.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)1 << 20;   // 1 MiB: e.g. 16 tokens x 32768 channels
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch, looked up once per device with that
// device current (in host code the array's name is only a host-side stand-in,
// not a device address). The lookup is guarded by a lock, so threads making
// their first call on one device at once do not race. The address is kept for
// the life of the process: a context reset (cudaDeviceReset) invalidates it,
// and calls after such a reset are not supported.
cudaError_t noalloc_scratch(void** ptr) {
    static void* addr[64] = {};
    static std::atomic<bool> ready[64] = {};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!ready[dev].load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> lock(mu);
        if (!ready[dev].load(std::memory_order_relaxed)) {
            void* a = nullptr;
            e = cudaGetSymbolAddress(&a, g_noalloc_scratch);
            if (e != cudaSuccess) return e;
            addr[dev] = a;
            ready[dev].store(true, std::memory_order_release);
        }
    }
    *ptr = addr[dev];
    return cudaSuccess;
}

}  // namespace

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

cudaError_t launch_gemv_noalloc(const RotDev* rot, const void* X, const void* qw, const void* scp, const void* zp,
                                void* Y, int64_t T, int64_t in, int64_t out, cudaStream_t s) {
    void* scratch = nullptr;
    cudaError_t e = noalloc_scratch(&scratch);
    if (e != cudaSuccess) return e;
    return launch_gemv(rot, X, qw, scp, zp, nullptr, Y, T, in, out, 128, scratch, s);
}

}  // namespace paro
