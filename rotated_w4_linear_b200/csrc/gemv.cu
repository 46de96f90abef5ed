// Decode kernel for tokens <= 16: Y[T][out] = X' w_hat^T with X' = X T^-1
// already in global memory (written by the rotation kernel launched just
// before on the same stream). The int4 weight stream dominates: HBM bound.
//
// Launch: a grid of (nsplit, rowtiles) CTAs of 8 warps; CTAs with the same
// row tile form one thread-block cluster along x, each owning a k-chunk of
// KC 128-channel groups. The kernel is launched with programmatic stream
// serialisation, so it starts while the rotation kernel still runs:
//   1. every warp issues the int4 loads of its first work item;
//   2. griddepcontrol.wait: the rotation grid has completed and X' is
//      visible; the CTA copies its X' chunk (all tokens) into shared memory;
//   3. items (row block of 16 rows x 4 groups) are spread over the warps:
//      each 32-bit int4 word becomes an m16n8k16 A fragment of the exact
//      integers (q - z) in fp16 (LOP3 into the 1024 + q bit pattern, one exact
//      fp16 subtraction); the B fragment (four consecutive channels of one
//      token) comes from shared memory; each group's products are summed in
//      fp32 by the tensor core (two independent accumulator chains) and then
//      multiplied by the group's fp32 scale, i.e. the contraction uses the
//      exact product (q - z) * s; the next item's loads are in flight
//      meanwhile; per-item partial sums are added into a shared fp32 tile
//      [token][row];
//   4. split-k: the cluster's CTAs read each other's tiles through
//      distributed shared memory; CTA x sums and stores the x-th slice of
//      the rows as fp16. No global atomics and no workspace.
// The k order inside each 16x16 tile follows the packed layout: the MMA's
// logical k slot 2q+e holds channel 4q+e and slot 2q+8+e channel 4q+2+e.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace paro {

namespace {

constexpr int kWarps = 8;
constexpr int kItemGroups = 4;            // groups per work item
constexpr int kItemBlocks = 2 * kItemGroups;  // 64-wide k blocks per item

struct GemvArgs {
    const __half* Xr;     // [T][in] fp16, already rotated
    int T, in, out, G;
    int KC;               // groups per k-chunk (last chunk may be shorter)
    int RT;               // row blocks per CTA
    int nsplit;           // k-chunks = cluster size along x
    const uint4* qw;
    const uint32_t* sp;
    const uint8_t* zp;
    __half* Y;
};

__device__ __forceinline__ void mma16816(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ float ld_dsmem_f32(uint32_t local_addr, uint32_t cta_rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(cta_rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

struct Item {
    uint4 w[kItemBlocks];
    uint32_t s[kItemGroups];
    uint32_t z[kItemGroups];
};

// Issue the loads of one item: row block rb, groups [g0, g0 + ng) (ng <= 4).
__device__ __forceinline__ void load_item(Item& it, const GemvArgs& a, int rb, int g0, int ng, int lane) {
    const int nkb = a.in >> 6;
    const uint4* src = a.qw + ((size_t)rb * nkb + 2 * g0) * 32 + lane;
#pragma unroll
    for (int i = 0; i < kItemBlocks; ++i)
        if (i < 2 * ng) it.w[i] = ldg_stream(src + i * 32);
    const size_t mi = ((size_t)rb * a.G + g0) * 8 + (lane >> 2);
#pragma unroll
    for (int g = 0; g < kItemGroups; ++g) {
        if (g < ng) {
            it.s[g] = __ldg(a.sp + mi + 8 * g);
            it.z[g] = __ldg(a.zp + mi + 8 * g);
        }
    }
}

}  // namespace

template <int NT>
__global__ void __launch_bounds__(kWarps * 32, 2) gemv_kernel(const GemvArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int chunk = blockIdx.x, rt = blockIdx.y;
    const int g_begin = chunk * a.KC;
    const int g_end = min(a.G, g_begin + a.KC);
    const int ncg = g_end - g_begin;                      // groups in this chunk
    const int nsub = (ncg + kItemGroups - 1) / kItemGroups;
    const int nrb = a.out >> 4;
    const int rb_begin = rt * a.RT;
    const int rb_end = min(nrb, rb_begin + a.RT);
    const int nitems = max(0, rb_end - rb_begin) * nsub;

    const int XS = a.KC * 128 + 16;                       // halves; row stride == 8 words mod 32
    __half* xs = reinterpret_cast<__half*>(smem);
    const int RTR = a.RT * 16 + 4;                        // floats; == 4 words mod 32
    float* red = reinterpret_cast<float*>(smem + (size_t)NT * 8 * XS * 2);

    // ---- 1. first item's loads, zero the partial tile
    Item cur, nxt;
    int item = warp;
    if (item < nitems) {
        const int rb = rb_begin + item / nsub, sub = item % nsub;
        const int g0 = g_begin + sub * kItemGroups;
        load_item(cur, a, rb, g0, min(kItemGroups, g_end - g0), lane);
    }
    for (int i = threadIdx.x; i < NT * 8 * RTR; i += kWarps * 32) red[i] = 0.f;

    // ---- 2. wait for the rotation grid, stage X' chunk (zero rows >= T)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    {
        const int vec_per_row = ncg * 16;                  // 16-byte vectors per token row
        const int total = NT * 8 * vec_per_row;
        for (int i = threadIdx.x; i < total; i += kWarps * 32) {
            const int tok = i / vec_per_row, v = i % vec_per_row;
            uint4 val = make_uint4(0u, 0u, 0u, 0u);
            if (tok < a.T)
                val = __ldg(reinterpret_cast<const uint4*>(a.Xr + (size_t)tok * a.in + (size_t)g_begin * 128) + v);
            *reinterpret_cast<uint4*>(xs + (size_t)tok * XS + v * 8) = val;
        }
    }
    __syncthreads();

    // ---- 3. mainloop over this warp's items
    const int gq = lane >> 2, qd = lane & 3;
    for (; item < nitems; item += kWarps) {
        const int rbl = item / nsub, sub = item % nsub;
        const int g0 = g_begin + sub * kItemGroups;
        const int ng = min(kItemGroups, g_end - g0);
        const int nx = item + kWarps;
        if (nx < nitems) {
            const int rb2 = rb_begin + nx / nsub, sub2 = nx % nsub;
            const int g2 = g_begin + sub2 * kItemGroups;
            load_item(nxt, a, rb2, g2, min(kItemGroups, g_end - g2), lane);
        }
        // B fragment rows of this lane (token gq, gq + 8), at the item's first channel
        const __half* xb[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) xb[nt] = xs + (size_t)(nt * 8 + gq) * XS + (g0 - g_begin) * 128 + 4 * qd;
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
        for (int g = 0; g < kItemGroups; ++g) {
            if (g < ng) {
                // (q - z) is exact in fp16; s is applied to the group's fp32 partial sums
                uint32_t zb0, zb1;
                zero_bias(cur.z[g], zb0, zb1);
                float p[NT][2][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int c = 0; c < 2; ++c) p[nt][c][0] = p[nt][c][1] = p[nt][c][2] = p[nt][c][3] = 0.f;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint4 wv = cur.w[2 * g + h];
                    const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t w = words[j];
                        const uint32_t A[4] = {hsub2_rn(nib_pair_to_f16x2(w), zb0),
                                               hsub2_rn(nib_pair_to_f16x2(w >> 8), zb1),
                                               hsub2_rn(nib_pair_to_f16x2(w >> 4), zb0),
                                               hsub2_rn(nib_pair_to_f16x2(w >> 12), zb1)};
                        const int k = g * 128 + h * 64 + j * 16;
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const uint2 bv = *reinterpret_cast<const uint2*>(xb[nt] + k);
                            mma16816(p[nt][j & 1], A, bv.x, bv.y);
                        }
                    }
                }
                const float2 sf = __half22float2(*reinterpret_cast<const __half2*>(&cur.s[g]));
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    acc[nt][0] = fmaf(sf.x, p[nt][0][0] + p[nt][1][0], acc[nt][0]);
                    acc[nt][1] = fmaf(sf.x, p[nt][0][1] + p[nt][1][1], acc[nt][1]);
                    acc[nt][2] = fmaf(sf.y, p[nt][0][2] + p[nt][1][2], acc[nt][2]);
                    acc[nt][3] = fmaf(sf.y, p[nt][0][3] + p[nt][1][3], acc[nt][3]);
                }
            }
        }
        // partial sums -> shared tile red[token][row] (rows local to the CTA)
        const int r0 = rbl * 16 + gq;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int t = nt * 8 + 2 * qd + e;
                atomicAdd(red + t * RTR + r0, acc[nt][e]);
                atomicAdd(red + t * RTR + r0 + 8, acc[nt][2 + e]);
            }
        }
        cur = nxt;
    }

    // ---- 4. split-k reduction across the cluster, fp16 store
    const int nrows = max(0, rb_end - rb_begin) * 16;
    const int row0 = rb_begin * 16;
    if (a.nsplit == 1) {
        __syncthreads();
        for (int i = threadIdx.x; i < a.T * nrows; i += kWarps * 32) {
            const int t = i / nrows, r = i % nrows;
            a.Y[(size_t)t * a.out + row0 + r] = __float2half_rn(red[t * RTR + r]);
        }
        return;
    }
    cluster_sync();                                        // all partial tiles complete
    const int share = (nrows + a.nsplit - 1) / a.nsplit;
    const int rlo = chunk * share, rhi = min(nrows, rlo + share);
    const int n = max(0, rhi - rlo);
    const uint32_t red_base = smem_u32(red);
    for (int i = threadIdx.x; i < a.T * n; i += kWarps * 32) {
        const int t = i / n, r = rlo + i % n;
        const uint32_t off = red_base + (uint32_t)(t * RTR + r) * 4u;
        float sum = 0.f;
        for (int x = 0; x < a.nsplit; ++x) sum += ld_dsmem_f32(off, (uint32_t)x);
        a.Y[(size_t)t * a.out + row0 + r] = __float2half_rn(sum);
    }
    cluster_sync();                                        // keep tiles alive until every reader is done
}

struct GemvPlan {
    int KC, nsplit, RT, rowtiles;
    size_t smem;
};

static GemvPlan plan_gemv(int T, int64_t in, int64_t out, int sms) {
    const int G = (int)(in / 128);
    const int nrb = (int)(out / 16);
    const int NT = T > 8 ? 2 : 1;
    GemvPlan p{};
    const int kc_max = 20;
    int nsplit = std::max(1, (G + kc_max - 1) / kc_max);
    while (nsplit < 8 && (int64_t)nrb * nsplit < 4LL * sms && (G + nsplit) / (nsplit + 1) >= kItemGroups) ++nsplit;
    nsplit = std::min(nsplit, 8);
    p.KC = (G + nsplit - 1) / nsplit;
    p.nsplit = (G + p.KC - 1) / p.KC;
    const int want_tiles = std::max(1, (2 * sms + p.nsplit - 1) / p.nsplit);
    p.RT = std::max(1, (nrb + want_tiles - 1) / want_tiles);
    p.rowtiles = (nrb + p.RT - 1) / p.RT;
    p.smem = (size_t)NT * 8 * (p.KC * 128 + 16) * 2 + (size_t)NT * 8 * (p.RT * 16 + 4) * 4;
    return p;
}

template <int NT>
static cudaError_t launch_gemv_t(const GemvArgs& a, const GemvPlan& p, bool pdl, cudaStream_t s) {
    static bool configured[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !configured[dev]) {
        cudaError_t e = cudaFuncSetAttribute(gemv_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(p.nsplit, p.rowtiles, 1);
    cfg.blockDim = dim3(kWarps * 32, 1, 1);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = p.nsplit;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, gemv_kernel<NT>, a);
}

cudaError_t launch_gemv(const RotDev* rot, const void* X, const void* qw, const void* scp, const void* zp,
                        void* Y, int64_t T, int64_t in, int64_t out, void* ws, size_t /*ws_bytes*/,
                        cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const void* xr = X;
    if (rot) {
        // X' = X T^-1 into the workspace; the GEMV waits on this grid in-kernel
        cudaError_t e = launch_rotate(*rot, X, ws, T, s);
        if (e != cudaSuccess) return e;
        xr = ws;
    }
    const GemvPlan p = plan_gemv((int)T, in, out, sms);
    GemvArgs a{};
    a.Xr = static_cast<const __half*>(xr);
    a.T = (int)T;
    a.in = (int)in;
    a.out = (int)out;
    a.G = (int)(in / 128);
    a.KC = p.KC;
    a.RT = p.RT;
    a.nsplit = p.nsplit;
    a.qw = static_cast<const uint4*>(qw);
    a.sp = static_cast<const uint32_t*>(scp);
    a.zp = static_cast<const uint8_t*>(zp);
    a.Y = static_cast<__half*>(Y);
    cudaError_t e = (T > 8) ? launch_gemv_t<2>(a, p, rot != nullptr, s) : launch_gemv_t<1>(a, p, rot != nullptr, s);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace paro
