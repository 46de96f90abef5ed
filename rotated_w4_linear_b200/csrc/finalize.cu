// Last step of a row-parallel layer. Each rank holds a slice of the input
// channels on group boundaries (the groups rotate independently, so a rank
// rotates only its own slice) and computes the unrounded fp32 partial sums
// of Y for its slice; after the partials are added across the ranks, this
// kernel adds the bias and rounds to fp16 once, as the single-GPU layer does.
#include "common.cuh"
#include "kernels.h"

namespace paro {

// four outputs per thread (out is a multiple of 16, so a row holds whole quads)
__global__ void finalize_kernel(const float4* __restrict__ Yf, const __half* __restrict__ bias, uint2* __restrict__ Y,
                                int out4, int64_t n4) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n4) return;
    float4 v = Yf[i];
    if (bias) {
        const int c = (int)(i % out4) * 4;
        v.x += __half2float(bias[c]);
        v.y += __half2float(bias[c + 1]);
        v.z += __half2float(bias[c + 2]);
        v.w += __half2float(bias[c + 3]);
    }
    Y[i] = make_uint2(pack_half2(v.x, v.y), pack_half2(v.z, v.w));
}

cudaError_t launch_finalize(const float* Yf, const void* bias, void* Y, int64_t T, int64_t out, cudaStream_t s) {
    const int64_t n4 = T * out / 4;
    if (n4 > 0)
        finalize_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, s>>>(
            reinterpret_cast<const float4*>(Yf), static_cast<const __half*>(bias), static_cast<uint2*>(Y),
            (int)(out / 4), n4);
    return cudaGetLastError();
}

}  // namespace paro
