// Host-side launchers of the sm_100a kernels (internal to libparo).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace paro {

struct RotDev {
    int64_t in = 0;         // input features
    int G = 0;              // groups of 128 (tables are built per 128 channels)
    int K = 0;              // rotation layers
    int P = 0;              // active pairs per (layer, 128-channel group)
    int group = 128;        // the layer's group size (64: two groups share each 128-channel table;
                            // 256: G counts 256-channel groups, no Givens tables, mats and rotp64
                            // hold the 256-channel forms)
    uint8_t* rotq = nullptr;       // [K][G] quad exchange blocks (decode prologue)
    float* inv_alpha = nullptr;    // [in] fp32 1/alpha
    uint8_t* rotp64 = nullptr;     // [K][G] blocks of 128 partner bytes + 128 double2 (converter)
    double* alpha64 = nullptr;     // [in] alpha as fp64
    uint8_t* mats = nullptr;       // [G][64 KB] dense per-group rotation (hi, lo fp16; tensor-core operand image)
};

// Bytes of one group's dense rotation image: hi and lo fp16 128 x 128.
constexpr size_t kRotMatBytes = 4 * 128 * 128;
// For 256-channel groups, one image per half of the output channels: hi and
// lo fp16 of 256 (k) x 128 (n).
constexpr size_t kRotMat256Bytes = 4 * 256 * 128;

// 2-D TMA descriptor of a row-major tensor [outer][inner] (driver entry point).
bool encode_tma_2d(CUtensorMap* tm, CUtensorMapDataType type, const void* base, uint64_t inner, uint64_t outer,
                   uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz);

cudaError_t launch_rotate(const RotDev& r, const void* X, void* Xr, int64_t T, cudaStream_t s);
// Tensor-core rotation (dense per-group matrices); any T >= 1.
cudaError_t launch_rotate_tc(const RotDev& r, const void* X, void* Xr, int64_t T, cudaStream_t s);
// X' = X T^-1: Givens kernel up to 16 tokens, tensor-core kernel above.
// Decode batches (1 <= T <= 16): one CTA per group, all layers' parameters in
// shared memory; launched as a programmatic dependent of the previous kernel.
// lane_major: X' is written with every 64-channel block in the decode
// kernel's B-fragment order (channel 16 j + 4 q + e at 16 q + 4 j + e).
cudaError_t launch_rotate_decode(const RotDev& r, const void* X, void* Xr, int64_t T, cudaStream_t s,
                                 bool lane_major = false);
size_t rotate_decode_smem(int K, int T);

// group: channels per quantisation group (128 or 64) of the weight format.
cudaError_t launch_pack(const uint8_t* q, const uint16_t* sc, const uint8_t* z, int64_t in, int64_t out, int group,
                        void* qw, void* scp, void* zp, cudaStream_t s);
cudaError_t launch_dequant(const void* qw, const void* scp, const void* zp, int64_t in, int64_t out, int group,
                           void* W, cudaStream_t s);
cudaError_t launch_quantize(const RotDev& r, const void* W, int64_t out, uint8_t* q, uint16_t* sc,
                            uint8_t* z, cudaStream_t s);

// Decode path (tokens <= 16): the decode rotation kernel into ws (when rot
// is not null), then the int4 decode kernel, both programmatic dependent launches.
// group: channels per quantisation group of the weights (128 or 64).
// y_fp32: Y is fp32 and receives the unrounded sums (row-parallel partials).
cudaError_t launch_gemv(const RotDev* rot, const void* X, const void* qw, const void* scp, const void* zp,
                        const void* bias, void* Y, int64_t T, int64_t in, int64_t out, int group, void* ws,
                        cudaStream_t s, bool y_fp32 = false);

// Decode with the X' scratch in a static device array (no allocation anywhere).
size_t noalloc_scratch_bytes();
cudaError_t launch_gemv_noalloc(const RotDev* rot, const void* X, const void* qw, const void* scp, const void* zp,
                                void* Y, int64_t T, int64_t in, int64_t out, cudaStream_t s);

// Prefill (tokens > 16): tcgen05 GEMM on X' (already rotated, in global memory),
// launched as a programmatic dependent of the rotation kernel.
// group: channels per quantisation group of the weights (128 or 64).
cudaError_t launch_gemm(const void* Xr, const void* qw, const void* scp, const void* zp, const void* bias, void* Y,
                        int64_t T, int64_t in, int64_t out, int group, cudaStream_t s, bool y_fp32 = false);

// Y16 = fp16(Yf + bias) (bias fp16 [out] or null): the last step of a
// row-parallel layer after the partial sums were added across ranks.
cudaError_t launch_finalize(const float* Yf, const void* bias, void* Y, int64_t T, int64_t out, cudaStream_t s);

// A kernel whose bounded wait runs out on purpose after limit_ns (fault code 6).
cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t s);

// Fault code left by a bounded wait that ran out (0 = none); optionally cleared.
cudaError_t read_fault(unsigned int* code, bool clear);

}  // namespace paro
