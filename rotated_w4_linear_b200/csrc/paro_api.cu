// Host side of the C ABI declared in include/paro.h: argument validation,
// preparation of the rotation parameters, dispatch by token count.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <new>
#include <vector>

#include "../../include/paro.h"
#include "common.cuh"
#include "kernels.h"

struct paro_rot {
    paro::RotDev dev;
    int device = 0;
    void* block = nullptr;   // single device allocation holding every table
};

namespace {

thread_local char g_err[512] = "";

paro_status fail(paro_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return st;
}

paro_status cuda_fail(cudaError_t e, const char* what) {
    return fail(PARO_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The kernels are built for sm_100a only; refuse anything else up front.
paro_status check_device() {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0)
        return fail(PARO_ERR_DEVICE, "device %d is sm_%d%d; this library is built for sm_100a", dev, major, minor);
    return PARO_OK;
}

paro_status check_shape(int64_t in, int64_t out) {
    if (in <= 0 || in % 128) return fail(PARO_ERR_ARG, "in_features=%lld must be a positive multiple of 128", (long long)in);
    if (out <= 0 || out % 16) return fail(PARO_ERR_ARG, "out_features=%lld must be a positive multiple of 16", (long long)out);
    if (in > (1LL << 20) || out > (1LL << 22)) return fail(PARO_ERR_UNSUPPORTED, "shape too large");
    return PARO_OK;
}

size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }

// Dense form of one group's activation rotation: M = diag(1/alpha) R_1^T ...
// R_K^T (x' = x M for a row x of the group's 128 channels), built in fp64 by
// applying the layers, in order, to every row of diag(1/alpha) with the 2x2
// formula. Written as the tensor-core B operand image (rotate_tc.cu): B[n][k]
// = M[k][n] for hi = fp16(M) and then lo = fp16(M - hi), each as two halves
// (k 0-63, 64-127) of 128 rows x 128 bytes, 16-byte chunk c of row n at chunk
// position c ^ (n mod 8) (the 128-byte swizzle of a K-major operand).
void dense_group_image(const int16_t* pairs, const float* theta, const float* alpha, int K, int P, int G, int g,
                       uint8_t* out) {
    std::vector<double> M(128 * 128, 0.0);                // M[k * 128 + n]
    for (int k = 0; k < 128; ++k) M[k * 128 + k] = 1.0 / (double)alpha[g * 128 + k];
    for (int t = 0; t < K; ++t)
        for (int p = 0; p < P; ++p) {
            const size_t base = (((size_t)t * G + g) * P + p);
            const int i = pairs[2 * base], j = pairs[2 * base + 1];
            const double c = std::cos((double)theta[base]), sn = std::sin((double)theta[base]);
            for (int k = 0; k < 128; ++k) {
                const double vi = M[k * 128 + i], vj = M[k * 128 + j];
                M[k * 128 + i] = c * vi - sn * vj;
                M[k * 128 + j] = sn * vi + c * vj;
            }
        }
    for (int part = 0; part < 2; ++part)
        for (int n = 0; n < 128; ++n)
            for (int k = 0; k < 128; ++k) {
                const double m = M[k * 128 + n];
                const __half hi = __double2half(m);
                const __half v = part == 0 ? hi : __double2half(m - (double)__half2float(hi));
                const int h = k >> 6, chunk = (k & 63) >> 3, e = k & 7;
                const size_t off = (size_t)part * 32768 + (size_t)h * 16384 + (size_t)n * 128 +
                                   (size_t)((chunk ^ (n & 7)) << 4) + (size_t)e * 2;
                memcpy(out + off, &v, 2);
            }
}

// Plain host memory (not allocated or registered with CUDA) that a kernel
// cannot read.
bool is_unregistered_host(const void* p) {
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return true;
    }
    return a.type == cudaMemoryTypeUnregistered;
}

// The same for a 256-channel group: M is 256 x 256; per half h of the
// output channels one 128 KB image of B[n][k] = M[k][128 h + n], n < 128,
// k < 256: hi then lo, each as four 64-channel quarters of k (128 rows x 128
// bytes, 128-byte swizzle).
void dense_group_image_256(const int16_t* pairs, const float* theta, const float* alpha, int K, int P, int G, int g,
                           uint8_t* out /* [2][128 KB] */) {
    std::vector<double> M(256 * 256, 0.0);                // M[k * 256 + n]
    for (int k = 0; k < 256; ++k) M[k * 256 + k] = 1.0 / (double)alpha[g * 256 + k];
    for (int t = 0; t < K; ++t)
        for (int p = 0; p < P; ++p) {
            const size_t base = (((size_t)t * G + g) * P + p);
            const int i = pairs[2 * base], j = pairs[2 * base + 1];
            const double c = std::cos((double)theta[base]), sn = std::sin((double)theta[base]);
            for (int k = 0; k < 256; ++k) {
                const double vi = M[k * 256 + i], vj = M[k * 256 + j];
                M[k * 256 + i] = c * vi - sn * vj;
                M[k * 256 + j] = sn * vi + c * vj;
            }
        }
    for (int h = 0; h < 2; ++h)
        for (int part = 0; part < 2; ++part)
            for (int n = 0; n < 128; ++n)
                for (int k = 0; k < 256; ++k) {
                    const double m = M[k * 256 + 128 * h + n];
                    const __half hi = __double2half(m);
                    const __half v = part == 0 ? hi : __double2half(m - (double)__half2float(hi));
                    const int q = k >> 6, chunk = (k & 63) >> 3, e = k & 7;
                    const size_t off = (size_t)h * 131072 + (size_t)part * 65536 + (size_t)q * 16384 +
                                       (size_t)n * 128 + (size_t)((chunk ^ (n & 7)) << 4) + (size_t)e * 2;
                    memcpy(out + off, &v, 2);
                }
}

}  // namespace

extern "C" {

const char* paro_last_error(void) { return g_err; }

paro_status paro_linear_noalloc(const paro_rot* r, const void* X, const void* qw, const void* sp, const void* zp,
                                void* Y, int64_t T, int64_t in, int64_t out, paro_stream stream) {
    g_err[0] = 0;
    paro_status st = check_shape(in, out);
    if (st != PARO_OK) return st;
    if (T < 0) return fail(PARO_ERR_ARG, "tokens=%lld < 0", (long long)T);
    if (T == 0) return PARO_OK;
    if (T > 16) return fail(PARO_ERR_ARG, "tokens=%lld: this entry point serves decode batches of at most 16", (long long)T);
    if ((size_t)T * (size_t)in * 2 > paro::noalloc_scratch_bytes())
        return fail(PARO_ERR_ARG, "tokens x in_features x 2 = %zu bytes exceeds the %zu-byte static scratch",
                    (size_t)T * (size_t)in * 2, paro::noalloc_scratch_bytes());
    if (r && r->dev.in != in) return fail(PARO_ERR_ARG, "rotation prepared for in=%lld, layer has in=%lld", (long long)r->dev.in, (long long)in);
    if (r && r->dev.group != 128) return fail(PARO_ERR_UNSUPPORTED, "this entry point serves group 128");
    if (!X || !qw || !sp || !zp || !Y) return fail(PARO_ERR_ARG, "null pointer");
    if (!aligned16(X) || !aligned16(qw) || !aligned16(sp) || !aligned16(zp) || !aligned16(Y))
        return fail(PARO_ERR_ARG, "pointers must be 16-byte aligned");
    cudaError_t e = paro::launch_gemv_noalloc(r ? &r->dev : nullptr, X, qw, sp, zp, Y, T, in, out,
                                              static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PARO_OK : cuda_fail(e, "decode launch (static scratch)");
}

paro_status paro_fault_status(int* code, int clear) {
    g_err[0] = 0;
    if (!code) return fail(PARO_ERR_ARG, "code is null");
    unsigned int c = 0;
    cudaError_t e = paro::read_fault(&c, clear != 0);
    if (e != cudaSuccess) return cuda_fail(e, "read fault word");
    *code = (int)c;
    return PARO_OK;
}

paro_status paro_check_wait_timeout(uint32_t limit_us, paro_stream stream) {
    g_err[0] = 0;
    if (limit_us < 1 || limit_us > 2000000) return fail(PARO_ERR_ARG, "limit_us=%u must be in 1..2000000", limit_us);
    paro_status st = check_device();
    if (st != PARO_OK) return st;
    cudaError_t e = paro::launch_wait_selftest((uint64_t)limit_us * 1000ull, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PARO_OK : cuda_fail(e, "wait self-test launch");
}

}  // extern "C"

namespace {

// The handle for 128-channel groups (group = 128 as the caller sees it, or
// pairs of 64-channel groups folded into 128-channel tables).
paro_status rot_create_128(paro_rot** out, int64_t in, int K, int P, const int16_t* pairs, const float* theta,
                           const float* alpha) {
    const int group = 128;
    if (in <= 0 || in % group) return fail(PARO_ERR_ARG, "in_features=%lld must be a positive multiple of %d", (long long)in, group);
    if (in > (1LL << 20)) return fail(PARO_ERR_UNSUPPORTED, "in_features too large");
    if (K < 0 || K > 16) return fail(PARO_ERR_ARG, "K=%d must be in 0..16", K);
    if (K > 0 && (P < 1 || P > group / 2)) return fail(PARO_ERR_ARG, "pairs_per_group=%d must be in 1..%d", P, group / 2);
    if (!alpha) return fail(PARO_ERR_ARG, "alpha is null");
    if (K > 0 && (!pairs || !theta)) return fail(PARO_ERR_ARG, "pairs/theta is null");
    paro_status st = check_device();
    if (st != PARO_OK) return st;

    const int G = (int)(in / group);
    for (int64_t c = 0; c < in; ++c)
        if (!std::isfinite(alpha[c]) || alpha[c] == 0.0f)
            return fail(PARO_ERR_ARG, "alpha[%lld] must be finite and non-zero", (long long)c);

    // host images of the tables
    std::vector<uint8_t> rot32((size_t)K * G * paro::kRotBlockBytes);
    std::vector<uint8_t> rot64((size_t)K * G * (128 + 128 * 16));
    for (int t = 0; t < K; ++t) {
        for (int g = 0; g < G; ++g) {
            uint8_t partner[128];
            float a32[128], b32[128];
            double a64[128], b64[128];
            bool used[128] = {false};
            for (int c = 0; c < 128; ++c) { partner[c] = (uint8_t)c; a32[c] = 1.f; b32[c] = 0.f; a64[c] = 1.0; b64[c] = 0.0; }
            for (int p = 0; p < P; ++p) {
                const size_t base = (((size_t)t * G + g) * P + p);
                const int i = pairs[2 * base], j = pairs[2 * base + 1];
                const float th = theta[base];
                if (i < 0 || i >= group || j < 0 || j >= group)
                    return fail(PARO_ERR_ARG, "pair (%d,%d) of layer %d group %d leaves the group", i, j, t, g);
                if (i == j || used[i] || used[j])
                    return fail(PARO_ERR_ARG, "channel reused within layer %d group %d (pair %d: %d,%d)", t, g, p, i, j);
                if (!std::isfinite(th)) return fail(PARO_ERR_ARG, "theta of layer %d group %d pair %d is not finite", t, g, p);
                used[i] = used[j] = true;
                const double c = std::cos((double)th), s = std::sin((double)th);
                partner[i] = (uint8_t)j; a64[i] = c; b64[i] = -s;
                partner[j] = (uint8_t)i; a64[j] = c; b64[j] = s;
                a32[i] = (float)c; b32[i] = (float)(-s);
                a32[j] = (float)c; b32[j] = (float)s;
            }
            uint8_t* b = &rot32[((size_t)t * G + g) * paro::kRotBlockBytes];
            memcpy(b, partner, 128);
            for (int c = 0; c < 128; ++c) {
                memcpy(b + 128 + 8 * c, &a32[c], 4);
                memcpy(b + 128 + 8 * c + 4, &b32[c], 4);
            }
            uint8_t* b6 = &rot64[((size_t)t * G + g) * (128 + 128 * 16)];
            memcpy(b6, partner, 128);
            for (int c = 0; c < 128; ++c) {
                memcpy(b6 + 128 + 16 * c, &a64[c], 8);
                memcpy(b6 + 128 + 16 * c + 8, &b64[c], 8);
            }
        }
    }
    // quad exchange blocks: 16-byte slots, 8 lanes of a quarter-warp on 8 distinct
    // slots mod 8 for every store and load (8 perfect matchings of an 8-regular
    // bipartite multigraph, found one after another by augmenting paths)
    std::vector<uint8_t> rotq((size_t)K * G * paro::kRotQBlockBytes);
    for (int t = 0; t < K; ++t) {
        for (int g = 0; g < G; ++g) {
            const uint8_t* b = &rot32[((size_t)t * G + g) * paro::kRotBlockBytes];
            const uint8_t* partner = b;
            // channel c: store class (slot c%4, quarter of lane c/4), load class
            // (slot, quarter) of the lane that owns its partner
            int sc[128], lc[128], colour[128];
            for (int c = 0; c < 128; ++c) {
                sc[c] = (c & 3) * 4 + ((c >> 2) >> 3);
                lc[c] = (partner[c] & 3) * 4 + ((partner[c] >> 2) >> 3);
                colour[c] = -1;
            }
            for (int col = 0; col < 8; ++col) {
                int match_r[16];                      // right class -> channel
                for (int v = 0; v < 16; ++v) match_r[v] = -1;
                bool vis[16];
                // augmenting path from left class u over uncoloured channels
                auto augment = [&](auto&& self, int u) -> bool {
                    for (int c = 0; c < 128; ++c) {
                        if (colour[c] >= 0 || sc[c] != u) continue;
                        const int v = lc[c];
                        if (vis[v]) continue;
                        vis[v] = true;
                        if (match_r[v] < 0 || self(self, sc[match_r[v]])) {
                            match_r[v] = c;
                            return true;
                        }
                    }
                    return false;
                };
                for (int u = 0; u < 16; ++u) {
                    for (int v = 0; v < 16; ++v) vis[v] = false;
                    if (!augment(augment, u)) return fail(PARO_ERR_ARG, "internal: no conflict-free quad exchange layout");
                }
                for (int v = 0; v < 16; ++v) colour[match_r[v]] = col;
            }
            int pos[128], used[8] = {0};
            for (int c = 0; c < 128; ++c) pos[c] = colour[c] + 8 * used[colour[c]]++;
            uint8_t* x = &rotq[((size_t)t * G + g) * paro::kRotQBlockBytes];
            for (int l = 0; l < 32; ++l) {
                for (int j = 0; j < 4; ++j) {
                    const int c = 4 * l + j;
                    // bit 7: the channel is in a pair of this layer (else it only keeps its value)
                    x[8 * l + j] = (uint8_t)(pos[c] | (partner[c] != c ? 0x80 : 0));
                    x[8 * l + 4 + j] = (uint8_t)pos[partner[c]];
                }
            }
            for (int l = 0; l < 32; ++l) {   // (a, b) of channels 4l, 4l+1 | 4l+2, 4l+3
                memcpy(x + 256 + 16 * l, b + 128 + 8 * (4 * l), 16);
                memcpy(x + 768 + 16 * l, b + 128 + 8 * (4 * l + 2), 16);
            }
        }
    }
    // dense per-group rotations for the tensor-core kernel
    std::vector<uint8_t> mats((size_t)G * paro::kRotMatBytes);
    for (int g = 0; g < G; ++g) dense_group_image(pairs, theta, alpha, K, P, G, g, &mats[(size_t)g * paro::kRotMatBytes]);
    std::vector<float> inv_alpha((size_t)in);
    std::vector<double> alpha64((size_t)in);
    for (int64_t c = 0; c < in; ++c) {
        inv_alpha[c] = (float)(1.0 / (double)alpha[c]);
        alpha64[c] = (double)alpha[c];
    }

    const size_t o_inv = 0;
    const size_t o_rot64 = o_inv + round256(inv_alpha.size() * sizeof(float));
    const size_t o_a64 = o_rot64 + round256(rot64.size());
    const size_t o_rotq = o_a64 + round256(alpha64.size() * sizeof(double));
    const size_t o_mats = o_rotq + round256(rotq.size());
    const size_t total = o_mats + round256(mats.size());

    paro_rot* r = new (std::nothrow) paro_rot();
    if (!r) return fail(PARO_ERR_ARG, "out of host memory");
    cudaGetDevice(&r->device);
    cudaError_t e = cudaMalloc(&r->block, total);
    if (e != cudaSuccess) { delete r; return cuda_fail(e, "cudaMalloc(rotation tables)"); }
    char* base = static_cast<char*>(r->block);
    e = cudaMemcpy(base + o_inv, inv_alpha.data(), inv_alpha.size() * 4, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(base + o_rot64, rot64.data(), rot64.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(base + o_a64, alpha64.data(), alpha64.size() * 8, cudaMemcpyHostToDevice);
    if (e == cudaSuccess && !rotq.empty()) e = cudaMemcpy(base + o_rotq, rotq.data(), rotq.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(base + o_mats, mats.data(), mats.size(), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) { cudaFree(r->block); delete r; return cuda_fail(e, "cudaMemcpy(rotation tables)"); }
    r->dev.in = in;
    r->dev.G = G;
    r->dev.K = K;
    r->dev.P = P;
    r->dev.inv_alpha = reinterpret_cast<float*>(base + o_inv);
    r->dev.rotp64 = reinterpret_cast<uint8_t*>(base + o_rot64);
    r->dev.alpha64 = reinterpret_cast<double*>(base + o_a64);
    r->dev.rotq = reinterpret_cast<uint8_t*>(base + o_rotq);
    r->dev.mats = reinterpret_cast<uint8_t*>(base + o_mats);
    *out = r;
    return PARO_OK;
}

// The handle for 256-channel groups: fp64 blocks for the converter (256
// partner bytes + 256 (a, b) pairs per layer and group) and the dense images
// for the tensor-core rotation; the Givens kernel's 128-channel tables are
// not built (every batch size rotates on the tensor cores).
paro_status rot_create_256(paro_rot** out, int64_t in, int K, int P, const int16_t* pairs, const float* theta,
                           const float* alpha) {
    if (in > (1LL << 20)) return fail(PARO_ERR_UNSUPPORTED, "in_features too large");
    if (!alpha) return fail(PARO_ERR_ARG, "alpha is null");
    paro_status st = check_device();
    if (st != PARO_OK) return st;
    const int G = (int)(in / 256);
    for (int64_t c = 0; c < in; ++c)
        if (!std::isfinite(alpha[c]) || alpha[c] == 0.0f)
            return fail(PARO_ERR_ARG, "alpha[%lld] must be finite and non-zero", (long long)c);
    constexpr size_t kBlk = 256 + 256 * 16;
    std::vector<uint8_t> rot64((size_t)K * G * kBlk);
    for (int t = 0; t < K; ++t)
        for (int g = 0; g < G; ++g) {
            uint8_t partner[256];
            double a64[256], b64[256];
            bool used[256] = {false};
            for (int c = 0; c < 256; ++c) { partner[c] = (uint8_t)c; a64[c] = 1.0; b64[c] = 0.0; }
            for (int p = 0; p < P; ++p) {
                const size_t base = (((size_t)t * G + g) * P + p);
                const int i = pairs[2 * base], j = pairs[2 * base + 1];
                const float th = theta[base];
                if (i < 0 || i >= 256 || j < 0 || j >= 256)
                    return fail(PARO_ERR_ARG, "pair (%d,%d) of layer %d group %d leaves the group", i, j, t, g);
                if (i == j || used[i] || used[j])
                    return fail(PARO_ERR_ARG, "channel reused within layer %d group %d (pair %d: %d,%d)", t, g, p, i, j);
                if (!std::isfinite(th)) return fail(PARO_ERR_ARG, "theta of layer %d group %d pair %d is not finite", t, g, p);
                used[i] = used[j] = true;
                const double c = std::cos((double)th), sn = std::sin((double)th);
                partner[i] = (uint8_t)j; a64[i] = c; b64[i] = -sn;
                partner[j] = (uint8_t)i; a64[j] = c; b64[j] = sn;
            }
            uint8_t* b6 = &rot64[((size_t)t * G + g) * kBlk];
            memcpy(b6, partner, 256);
            for (int c = 0; c < 256; ++c) {
                memcpy(b6 + 256 + 16 * c, &a64[c], 8);
                memcpy(b6 + 256 + 16 * c + 8, &b64[c], 8);
            }
        }
    std::vector<uint8_t> mats((size_t)G * 2 * paro::kRotMat256Bytes);
    for (int g = 0; g < G; ++g)
        dense_group_image_256(pairs, theta, alpha, K, P, G, g, &mats[(size_t)g * 2 * paro::kRotMat256Bytes]);
    std::vector<double> alpha64((size_t)in);
    for (int64_t c = 0; c < in; ++c) alpha64[c] = (double)alpha[c];
    const size_t o_rot64 = 0, o_a64 = round256(rot64.size()), o_mats = o_a64 + round256(alpha64.size() * 8);
    const size_t total = o_mats + round256(mats.size());
    paro_rot* r = new (std::nothrow) paro_rot();
    if (!r) return fail(PARO_ERR_ARG, "out of host memory");
    cudaGetDevice(&r->device);
    cudaError_t e = cudaMalloc(&r->block, total);
    if (e != cudaSuccess) { delete r; return cuda_fail(e, "cudaMalloc(rotation tables)"); }
    char* base = static_cast<char*>(r->block);
    e = cudaSuccess;
    if (!rot64.empty()) e = cudaMemcpy(base + o_rot64, rot64.data(), rot64.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(base + o_a64, alpha64.data(), alpha64.size() * 8, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(base + o_mats, mats.data(), mats.size(), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) { cudaFree(r->block); delete r; return cuda_fail(e, "cudaMemcpy(rotation tables)"); }
    r->dev.in = in;
    r->dev.G = G;
    r->dev.K = K;
    r->dev.P = P;
    r->dev.group = 256;
    r->dev.rotp64 = reinterpret_cast<uint8_t*>(base + o_rot64);
    r->dev.alpha64 = reinterpret_cast<double*>(base + o_a64);
    r->dev.mats = reinterpret_cast<uint8_t*>(base + o_mats);
    *out = r;
    return PARO_OK;
}

}  // namespace

extern "C" {

paro_status paro_rot_create(paro_rot** out, int64_t in, int group, int K, int P, const int16_t* pairs,
                            const float* theta, const float* alpha) {
    g_err[0] = 0;
    if (!out) return fail(PARO_ERR_ARG, "out is null");
    *out = nullptr;
    if (group != 128 && group != 64 && group != 256)
        return fail(PARO_ERR_UNSUPPORTED, "group=%d: 64, 128 and 256 are supported", group);
    const int unit = group == 256 ? 256 : 128;
    if (in <= 0 || in % unit)
        return fail(PARO_ERR_ARG, "in_features=%lld must be a positive multiple of %d", (long long)in, unit);
    if (K < 0 || K > 16) return fail(PARO_ERR_ARG, "K=%d must be in 0..16", K);
    if (K > 0 && (P < 1 || P > group / 2)) return fail(PARO_ERR_ARG, "pairs_per_group=%d must be in 1..%d", P, group / 2);
    if (K > 0 && (!pairs || !theta)) return fail(PARO_ERR_ARG, "pairs/theta is null");
    if (group == 128) return rot_create_128(out, in, K, P, pairs, theta, alpha);
    if (group == 256) return rot_create_256(out, in, K, P, pairs, theta, alpha);
    // groups of 64: the pairs of 64-channel groups 2h and 2h + 1 (indices
    // 0..63 each) form the 128-channel table h, the second group's indices
    // moved up by 64; a pair cannot leave its 64-channel group
    const int64_t G64 = in / 64, G = in / 128;
    std::vector<int16_t> p128((size_t)K * G * 2 * P * 2);
    std::vector<float> t128((size_t)K * G * 2 * P);
    for (int t = 0; t < K; ++t)
        for (int64_t g = 0; g < G64; ++g)
            for (int p = 0; p < P; ++p) {
                const size_t src = ((size_t)t * G64 + g) * P + p;
                const int i = pairs[2 * src], j = pairs[2 * src + 1];
                if (i < 0 || i >= 64 || j < 0 || j >= 64)
                    return fail(PARO_ERR_ARG, "pair (%d,%d) of layer %d group %lld leaves its 64-channel group", i, j,
                                t, (long long)g);
                const size_t dst = ((size_t)t * G + g / 2) * (2 * P) + (size_t)(g & 1) * P + p;
                p128[2 * dst] = (int16_t)(i + 64 * (g & 1));
                p128[2 * dst + 1] = (int16_t)(j + 64 * (g & 1));
                t128[dst] = theta[src];
            }
    paro_status st = rot_create_128(out, in, K, 2 * P, K ? p128.data() : nullptr, K ? t128.data() : nullptr, alpha);
    if (st == PARO_OK) (*out)->dev.group = 64;
    return st;
}

paro_status paro_rot_destroy(paro_rot* r) {
    g_err[0] = 0;
    if (!r) return PARO_OK;
    cudaError_t e = cudaFree(r->block);
    delete r;
    return e == cudaSuccess ? PARO_OK : cuda_fail(e, "cudaFree(rotation tables)");
}

paro_status paro_rotate(const paro_rot* r, const void* X, void* Xr, int64_t T, paro_stream stream) {
    g_err[0] = 0;
    if (!r) return fail(PARO_ERR_ARG, "rot is null");
    if (T < 0) return fail(PARO_ERR_ARG, "tokens=%lld < 0", (long long)T);
    if (T == 0) return PARO_OK;
    if (!X || !Xr) return fail(PARO_ERR_ARG, "X/Xr is null");
    if (!aligned16(X) || !aligned16(Xr)) return fail(PARO_ERR_ARG, "X/Xr must be 16-byte aligned");
    if (X == Xr) return fail(PARO_ERR_ARG, "X and Xr must not alias");
    if (T > (1LL << 31) / r->dev.in) return fail(PARO_ERR_UNSUPPORTED, "tokens too large");
    cudaError_t e = paro::launch_rotate(r->dev, X, Xr, T, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PARO_OK : cuda_fail(e, "rotate launch");
}

paro_status paro_pack_size_ex(int64_t in, int64_t out, int group, size_t* qb, size_t* sb, size_t* zb) {
    g_err[0] = 0;
    paro_status st = check_shape(in, out);
    if (st != PARO_OK) return st;
    if (group != 128 && group != 64 && group != 256)
        return fail(PARO_ERR_UNSUPPORTED, "group=%d: 64, 128 and 256 are supported", group);
    if (group == 256 && in % 256) return fail(PARO_ERR_ARG, "in_features=%lld: group 256 needs a multiple of 256", (long long)in);
    if (!qb || !sb || !zb) return fail(PARO_ERR_ARG, "null size pointer");
    const int64_t G = in / (group == 256 ? 128 : group);     // group 256: stored as group 128
    *qb = (size_t)(in * out / 2);
    *sb = (size_t)((out / 16) * G * 8 * 4);
    *zb = (size_t)((out / 16) * (G + (G & 1)) * 8);
    return PARO_OK;
}

paro_status paro_pack_size(int64_t in, int64_t out, size_t* qb, size_t* sb, size_t* zb) {
    return paro_pack_size_ex(in, out, 128, qb, sb, zb);
}

paro_status paro_pack_weights_ex(const uint8_t* q, const uint16_t* s, const uint8_t* z, int64_t in, int64_t out,
                                 int group, void* qw, void* sp, void* zp, paro_stream stream) {
    g_err[0] = 0;
    paro_status st = check_shape(in, out);
    if (st != PARO_OK) return st;
    if (group != 128 && group != 64 && group != 256)
        return fail(PARO_ERR_UNSUPPORTED, "group=%d: 64, 128 and 256 are supported", group);
    if (group == 256 && in % 256) return fail(PARO_ERR_ARG, "in_features=%lld: group 256 needs a multiple of 256", (long long)in);
    if (!q || !s || !z || !qw || !sp || !zp) return fail(PARO_ERR_ARG, "null pointer");
    if (!aligned16(qw) || !aligned16(sp) || !aligned16(zp)) return fail(PARO_ERR_ARG, "outputs must be 16-byte aligned");
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (!is_unregistered_host(q) && !is_unregistered_host(s) && !is_unregistered_host(z)) {
        cudaError_t e = paro::launch_pack(q, s, z, in, out, group, qw, sp, zp, cs);
        return e == cudaSuccess ? PARO_OK : cuda_fail(e, "pack launch");
    }
    // host inputs: stage the logical tensors in one temporary device buffer
    // (offline step; synchronous on `stream`)
    const size_t G = (size_t)(in / group);
    const size_t nq = (size_t)in * (size_t)out, ns = (size_t)out * G * 2, nz = (size_t)out * G;
    const size_t oq = 0, os_ = round256(nq), oz = os_ + round256(ns), total = oz + round256(nz);
    char* tmp = nullptr;
    cudaError_t e = cudaMalloc(&tmp, total);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(staging of host q/s/z)");
    e = cudaMemcpyAsync(tmp + oq, q, nq, cudaMemcpyDefault, cs);
    if (e == cudaSuccess) e = cudaMemcpyAsync(tmp + os_, s, ns, cudaMemcpyDefault, cs);
    if (e == cudaSuccess) e = cudaMemcpyAsync(tmp + oz, z, nz, cudaMemcpyDefault, cs);
    if (e == cudaSuccess)
        e = paro::launch_pack(reinterpret_cast<const uint8_t*>(tmp + oq), reinterpret_cast<const uint16_t*>(tmp + os_),
                              reinterpret_cast<const uint8_t*>(tmp + oz), in, out, group, qw, sp, zp, cs);
    const cudaError_t e2 = cudaStreamSynchronize(cs);
    cudaFree(tmp);
    if (e != cudaSuccess) return cuda_fail(e, "pack from host memory");
    return e2 == cudaSuccess ? PARO_OK : cuda_fail(e2, "pack from host memory (synchronize)");
}

paro_status paro_pack_weights(const uint8_t* q, const uint16_t* s, const uint8_t* z, int64_t in, int64_t out,
                              void* qw, void* sp, void* zp, paro_stream stream) {
    return paro_pack_weights_ex(q, s, z, in, out, 128, qw, sp, zp, stream);
}

paro_status paro_dequant_ex(const void* qw, const void* sp, const void* zp, int64_t in, int64_t out, int group,
                            void* W, paro_stream stream) {
    g_err[0] = 0;
    paro_status st = check_shape(in, out);
    if (st != PARO_OK) return st;
    if (group != 128 && group != 64 && group != 256)
        return fail(PARO_ERR_UNSUPPORTED, "group=%d: 64, 128 and 256 are supported", group);
    if (group == 256) group = 128;                                // stored as group 128
    if (!qw || !sp || !zp || !W) return fail(PARO_ERR_ARG, "null pointer");
    if (!aligned16(qw) || !aligned16(sp) || !aligned16(W)) return fail(PARO_ERR_ARG, "pointers must be 16-byte aligned");
    cudaError_t e = paro::launch_dequant(qw, sp, zp, in, out, group, W, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PARO_OK : cuda_fail(e, "dequant launch");
}

paro_status paro_dequant(const void* qw, const void* sp, const void* zp, int64_t in, int64_t out, void* W,
                         paro_stream stream) {
    return paro_dequant_ex(qw, sp, zp, in, out, 128, W, stream);
}

paro_status paro_quantize_weights(const paro_rot* r, const void* W, int64_t out, uint8_t* q, uint16_t* s,
                                  uint8_t* z, paro_stream stream) {
    g_err[0] = 0;
    if (!r) return fail(PARO_ERR_ARG, "rot is null");
    paro_status st = check_shape(r->dev.in, out);
    if (st != PARO_OK) return st;
    if (!W || !q || !s || !z) return fail(PARO_ERR_ARG, "null pointer");
    if (!aligned16(W) || !aligned16(q)) return fail(PARO_ERR_ARG, "W/q must be 16-byte aligned");
    cudaError_t e = paro::launch_quantize(r->dev, W, out, q, s, z, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PARO_OK : cuda_fail(e, "quantize launch");
}

paro_status paro_linear_workspace_size(int64_t T, int64_t in, int64_t out, size_t* bytes) {
    g_err[0] = 0;
    paro_status st = check_shape(in, out);
    if (st != PARO_OK) return st;
    if (T < 0 || !bytes) return fail(PARO_ERR_ARG, "bad tokens or null bytes");
    *bytes = round256((size_t)T * in * 2);   // X T^-1 (fp16), one row per token
    return PARO_OK;
}

}  // extern "C"

namespace {

// The layer: fp16 Y, or (y_fp32) the unrounded fp32 sums of a row-parallel slice.
paro_status linear_impl(const paro_rot* r, const void* X, const void* qw, const void* sp, const void* zp,
                        const void* bias, int group, void* Y, int64_t T, int64_t in, int64_t out, void* ws,
                        size_t ws_bytes, paro_stream stream, bool y_fp32) {
    g_err[0] = 0;
    paro_status st = check_shape(in, out);
    if (st != PARO_OK) return st;
    if (group != 128 && group != 64 && group != 256)
        return fail(PARO_ERR_UNSUPPORTED, "group=%d: 64, 128 and 256 are supported", group);
    if (r && r->dev.group != group)
        return fail(PARO_ERR_ARG, "rotation prepared for group %d, weights quantised with group %d", r->dev.group, group);
    if (group == 256 && in % 256) return fail(PARO_ERR_ARG, "in_features=%lld: group 256 needs a multiple of 256", (long long)in);
    // group 256 weights are stored in the group-128 format (each scale and zero repeated)
    const int fmt_group = group == 256 ? 128 : group;
    if (T < 0) return fail(PARO_ERR_ARG, "tokens=%lld < 0", (long long)T);
    if (T == 0) return PARO_OK;
    if (r && r->dev.in != in) return fail(PARO_ERR_ARG, "rotation prepared for in=%lld, layer has in=%lld", (long long)r->dev.in, (long long)in);
    if (!X || !qw || !sp || !zp || !Y || !ws) return fail(PARO_ERR_ARG, "null pointer");
    if (!aligned16(X) || !aligned16(qw) || !aligned16(sp) || !aligned16(zp) || !aligned16(Y) || !aligned16(ws))
        return fail(PARO_ERR_ARG, "pointers must be 16-byte aligned");
    if (bias && (reinterpret_cast<uintptr_t>(bias) & 1u)) return fail(PARO_ERR_ARG, "bias must be 2-byte aligned");
    if (T > (1LL << 31) / in) return fail(PARO_ERR_UNSUPPORTED, "tokens too large");
    size_t need = 0;
    paro_linear_workspace_size(T, in, out, &need);
    if (ws_bytes < need) return fail(PARO_ERR_ARG, "workspace_bytes=%zu < %zu", ws_bytes, need);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const paro::RotDev* rd = r ? &r->dev : nullptr;
    cudaError_t e;
    if (T <= 16) {   // decode rotation kernel into ws, then the int4 decode kernel
        e = paro::launch_gemv(rd, X, qw, sp, zp, bias, Y, T, in, out, fmt_group, ws, s, y_fp32);
        return e == cudaSuccess ? PARO_OK : cuda_fail(e, "decode launch");
    }
    // X' = X T^-1 into the workspace, then the tensor-core GEMM as a
    // programmatic dependent launch
    const void* src = X;
    if (rd) {
        e = paro::launch_rotate(*rd, X, ws, T, s);
        if (e != cudaSuccess) return cuda_fail(e, "rotate launch");
        src = ws;
    }
    e = paro::launch_gemm(src, qw, sp, zp, bias, Y, T, in, out, fmt_group, s, y_fp32);
    return e == cudaSuccess ? PARO_OK : cuda_fail(e, "prefill launch");
}

}  // namespace

extern "C" {

paro_status paro_linear_ex(const paro_rot* r, const void* X, const void* qw, const void* sp, const void* zp,
                           const void* bias, int group, void* Y, int64_t T, int64_t in, int64_t out, void* ws,
                           size_t ws_bytes, paro_stream stream) {
    return linear_impl(r, X, qw, sp, zp, bias, group, Y, T, in, out, ws, ws_bytes, stream, false);
}

paro_status paro_linear_partial(const paro_rot* r, const void* X, const void* qw, const void* sp, const void* zp,
                                int group, float* Yf, int64_t T, int64_t in, int64_t out, void* ws, size_t ws_bytes,
                                paro_stream stream) {
    return linear_impl(r, X, qw, sp, zp, nullptr, group, Yf, T, in, out, ws, ws_bytes, stream, true);
}

paro_status paro_finalize(const float* Yf, const void* bias, void* Y, int64_t T, int64_t out, paro_stream stream) {
    g_err[0] = 0;
    if (T < 0 || out <= 0 || out % 16) return fail(PARO_ERR_ARG, "tokens=%lld, out_features=%lld", (long long)T, (long long)out);
    if (T == 0) return PARO_OK;
    if (!Yf || !Y) return fail(PARO_ERR_ARG, "null pointer");
    if (!aligned16(Yf) || !aligned16(Y)) return fail(PARO_ERR_ARG, "pointers must be 16-byte aligned");
    if (bias && (reinterpret_cast<uintptr_t>(bias) & 1u)) return fail(PARO_ERR_ARG, "bias must be 2-byte aligned");
    cudaError_t e = paro::launch_finalize(Yf, bias, Y, T, out, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PARO_OK : cuda_fail(e, "finalize launch");
}

paro_status paro_linear_bias(const paro_rot* r, const void* X, const void* qw, const void* sp, const void* zp,
                             const void* bias, void* Y, int64_t T, int64_t in, int64_t out, void* ws,
                             size_t ws_bytes, paro_stream stream) {
    return paro_linear_ex(r, X, qw, sp, zp, bias, 128, Y, T, in, out, ws, ws_bytes, stream);
}

paro_status paro_linear(const paro_rot* r, const void* X, const void* qw, const void* sp, const void* zp, void* Y,
                        int64_t T, int64_t in, int64_t out, void* ws, size_t ws_bytes, paro_stream stream) {
    return paro_linear_bias(r, X, qw, sp, zp, nullptr, Y, T, in, out, ws, ws_bytes, stream);
}

// One-shot forms: prepare the rotation, run the call, release everything
// (allocating and synchronous; the handle calls above are the hot path).
paro_status paro_rotate_once(const void* X, void* Xr, int64_t T, int64_t in, const int16_t* pairs,
                             const float* theta, const float* alpha, int K, int group, int pairs_per_group,
                             paro_stream stream) {
    paro_rot* r = nullptr;
    paro_status st = paro_rot_create(&r, in, group, K, pairs_per_group, pairs, theta, alpha);
    if (st != PARO_OK) return st;
    st = paro_rotate(r, X, Xr, T, stream);
    if (st == PARO_OK) {
        const cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) st = cuda_fail(e, "synchronize");
    }
    const paro_status st2 = paro_rot_destroy(r);
    return st != PARO_OK ? st : st2;
}

paro_status paro_linear_once(const void* X, const int16_t* pairs, const float* theta, const float* alpha,
                             const void* qweight, const void* scales, const void* zeros, void* Y, int64_t T,
                             int64_t in, int64_t out, int K, int pairs_per_group, paro_stream stream) {
    paro_rot* r = nullptr;
    paro_status st = paro_rot_create(&r, in, 128, K, pairs_per_group, pairs, theta, alpha);
    if (st != PARO_OK) return st;
    size_t ws_bytes = 0;
    void* ws = nullptr;
    st = paro_linear_workspace_size(T, in, out, &ws_bytes);
    if (st == PARO_OK && ws_bytes > 0) {
        const cudaError_t e = cudaMalloc(&ws, ws_bytes);
        if (e != cudaSuccess) st = cuda_fail(e, "cudaMalloc(workspace)");
    }
    if (st == PARO_OK) st = paro_linear(r, X, qweight, scales, zeros, Y, T, in, out, ws ? ws : Y, ws_bytes, stream);
    const cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (st == PARO_OK && e != cudaSuccess) st = cuda_fail(e, "synchronize");
    if (ws) cudaFree(ws);
    const paro_status st2 = paro_rot_destroy(r);
    return st != PARO_OK ? st : st2;
}

}  // extern "C"
