/*
 * paro.h - C ABI of the B200 (sm_100a) rotated W4G128 linear layer.
 *
 * The layer (ParoQuant; CSDN article "ParoQuant", section 2.1, and the ICLR
 * 2026 paper-notes page, "key design", final transform equation):
 *
 *     Y = (X T^-1) * dequant(Q(T W))^T,   T = R_K ... R_1 diag(alpha)
 *
 * R_t is a layer of independent Givens rotations over disjoint channel pairs
 * that never leave their 128-channel quantisation group (paper notes,
 * "independent rotation"); each pair (i, j) with angle th maps
 * (v_i, v_j) -> (cos th v_i - sin th v_j, sin th v_i + cos th v_j)
 * (CSDN article, section 2.2, the 2x2 matrix). Layer index 0 is applied
 * first, on the weight side and on the activation side alike:
 *     X T^-1 = X diag(1/alpha) R_1^T ... R_K^T.
 * Q is asymmetric INT4 round-to-nearest per 128-input group (W4G128) with an
 * fp16 scale s and an int4 zero z; dequant(q) = fp16((q - z) * s).
 *
 * Conventions for every entry point
 *   - Tensors are row-major and contiguous. "in" is the input-feature count
 *     (a multiple of 128), "out" the output-feature count (a multiple of 16),
 *     "tokens" the number of activation rows.
 *   - fp16 tensors are passed as void* / uint16_t* holding IEEE binary16.
 *   - Pointers named *_dev are device pointers on the current CUDA device;
 *     pointers named *_host are host pointers. The caller owns every buffer.
 *   - Calls that take a stream enqueue work on it and return without
 *     synchronising; the stream is a cudaStream_t (0 = legacy default stream).
 *     Hot-path calls (paro_rotate, paro_linear) allocate nothing.
 *   - Device pointers must be 16-byte aligned.
 *   - Every call returns a paro_status; on anything but PARO_OK,
 *     paro_last_error() returns a message for the calling thread. Argument
 *     errors are detected on the host before anything is enqueued.
 */
#ifndef PARO_H
#define PARO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PARO_OK = 0,
    PARO_ERR_ARG = 1,          /* invalid argument (null, size, alignment, pair table) */
    PARO_ERR_UNSUPPORTED = 2,  /* valid but not supported by this library (e.g. group != 128) */
    PARO_ERR_CUDA = 3,         /* a CUDA runtime call or a kernel launch failed */
    PARO_ERR_DEVICE = 4        /* no usable sm_100 device */
} paro_status;

typedef void* paro_stream;     /* a cudaStream_t */

/* Opaque prepared rotation: the device-resident form of (pairs, theta, alpha)
 * for one linear layer. */
typedef struct paro_rot paro_rot;

/* Validate and prepare the scaled pairwise rotation T of one layer and upload
 * it to the current device (setup; allocates device memory; synchronous).
 *   in_features      multiple of 128 (of 256 for group 256)
 *   group            channels per quantisation group: 128, 64 or 256 (others:
 *                    PARO_ERR_UNSUPPORTED). With 256 every batch size rotates
 *                    on the tensor cores (no Givens tables are built).
 *   K                number of rotation layers, 0..16 (K = 0: T = diag(alpha))
 *   pairs_per_group  P, 1..group/2 active pairs per (layer, group)
 *   pairs_host       int16 [K][in/group][P][2], group-local channel indices
 *                    (0..group-1); (i, j) order as in the 2x2 matrix above.
 *                    Within one (layer, group) no channel may appear twice.
 *                    (Groups of 64 are held as pairs of groups in 128-channel
 *                    tables; a pair still never leaves its 64-channel group.)
 *   theta_host       float [K][in/group][P], radians
 *   alpha_host       float [in_features], finite and non-zero
 * Paper: ICLR 2026 notes, "key design" (Givens decomposition, independent
 * rotation, K = 8 default, final transform T). */
paro_status paro_rot_create(paro_rot** out, int64_t in_features, int group, int K,
                            int pairs_per_group, const int16_t* pairs_host,
                            const float* theta_host, const float* alpha_host);

/* Free a handle from paro_rot_create (synchronous). NULL is accepted. */
paro_status paro_rot_destroy(paro_rot* rot);

/* Xr = X T^-1 (CSDN article, section 2.1: the activation side of
 * Y = (X T^-1)(T W)): divide channel c by alpha_c, then apply layers
 * t = 1..K with the 2x2 formula. fp32 arithmetic, fp16 in and out.
 *   X_dev, Xr_dev  fp16 [tokens][in_features]; may not alias.
 *   tokens >= 0 (0 is a no-op). */
paro_status paro_rotate(const paro_rot* rot, const void* X_dev, void* Xr_dev,
                        int64_t tokens, paro_stream stream);

/* Sizes in bytes of the device weight format written by paro_pack_weights. */
paro_status paro_pack_size(int64_t in_features, int64_t out_features,
                           size_t* qweight_bytes, size_t* scales_bytes, size_t* zeros_bytes);

/* The same for a quantisation group of `group` channels (128, 64 or 256;
 * the format above is group 128): one scale word and one zero byte per group
 * of each 16-row block's row pairs. Group 256 is stored in the group-128
 * format, each group's scale and zero repeated for its two 128-channel
 * halves. Paper: the group size as a speed/accuracy knob (CSDN article,
 * section 5.2). */
paro_status paro_pack_size_ex(int64_t in_features, int64_t out_features, int group,
                              size_t* qweight_bytes, size_t* scales_bytes, size_t* zeros_bytes);

/* Pack logical W4G128 tensors into the device weight format read by
 * paro_linear (the int4 layout of the weight stream; one 16x16 tile is one
 * 32-bit word per lane of a warp, nibbles ordered for a two-instruction
 * int4->fp16 conversion).
 *   q          uint8  [out][in], values 0..15
 *   s          fp16   [out][in/128], the stored scales
 *   z          uint8  [out][in/128], values 0..15
 *   q, s, z may be device memory (pinned host memory also works): the call
 *   then enqueues on `stream` and returns. If any of them is plain host
 *   memory, the three are staged through one temporary device allocation
 *   and the call is synchronous (an offline step).
 *   qweight_dev, scales_dev, zeros_dev: outputs sized by paro_pack_size.
 * Paper: W4G128 (paper notes, main-experiment table heading); s and z are the
 * quantisation parameters named in the notes' training-strategy section. */
paro_status paro_pack_weights(const uint8_t* q, const uint16_t* s, const uint8_t* z,
                              int64_t in_features, int64_t out_features,
                              void* qweight_dev, void* scales_dev, void* zeros_dev,
                              paro_stream stream);

/* paro_pack_weights for a quantisation group of `group` channels (128, 64 or
 * 256): s and z are [out][in/group]; sizes from paro_pack_size_ex. */
paro_status paro_pack_weights_ex(const uint8_t* q, const uint16_t* s, const uint8_t* z,
                                 int64_t in_features, int64_t out_features, int group,
                                 void* qweight_dev, void* scales_dev, void* zeros_dev,
                                 paro_stream stream);

/* Expand the device weight format back to w_hat = fp16((q - z) * s),
 * fp16 [out][in] (the dequantisation used inside paro_linear; exact product,
 * one rounding). */
paro_status paro_dequant(const void* qweight_dev, const void* scales_dev, const void* zeros_dev,
                         int64_t in_features, int64_t out_features, void* W_dev,
                         paro_stream stream);

/* paro_dequant for the format of paro_pack_weights_ex with `group` (128, 64 or 256). */
paro_status paro_dequant_ex(const void* qweight_dev, const void* scales_dev, const void* zeros_dev,
                            int64_t in_features, int64_t out_features, int group, void* W_dev,
                            paro_stream stream);

/* Offline converter: W' = T W along the input axis (fp64), then asymmetric
 * RTN per input group of the handle's group size (128, 64 or 256):
 * s = fp16((max-min)/15) floored at 2^-14,
 * z = clamp(rint(-min/s), 0, 15), q = clamp(rint(w/s) + z, 0, 15).
 *   W_dev  fp16 [out][in] (PyTorch orientation); outputs q_dev uint8 [out][in],
 *   s_dev fp16 [out][in/group], z_dev uint8 [out][in/group].
 * Paper: T W in the final-transform equation (paper notes, "key design");
 * the RTN rule is this library's reading of W4G128. */
paro_status paro_quantize_weights(const paro_rot* rot, const void* W_dev, int64_t out_features,
                                  uint8_t* q_dev, uint16_t* s_dev, uint8_t* z_dev,
                                  paro_stream stream);

/* Bytes of workspace paro_linear needs for this shape. */
paro_status paro_linear_workspace_size(int64_t tokens, int64_t in_features, int64_t out_features,
                                       size_t* bytes);

/* Y = (X T^-1) w_hat^T, fp32 accumulation, fp16 out (CSDN article,
 * section 2.1, without the bias).
 *   rot           prepared rotation, or NULL for the unrotated W4G128 layer
 *                 (theta = 0, alpha = 1)
 *   X_dev         fp16 [tokens][in_features]
 *   qweight_dev, scales_dev, zeros_dev   from paro_pack_weights
 *   Y_dev         fp16 [tokens][out_features]
 *   workspace_dev at least paro_linear_workspace_size bytes of scratch (no
 *                 initialisation needed); it receives X T^-1 in fp16, in an
 *                 internal order (for tokens <= 16 the channels of each
 *                 64-channel block are permuted for the decode kernel), so
 *                 its contents are not an output: use paro_rotate for X T^-1.
 *                 Calls that share a workspace must not overlap on the GPU.
 * The rotation kernel writes X T^-1 into the workspace; the contraction runs
 * as a programmatic dependent launch of it (its weight loads start before the
 * rotation has finished). tokens <= 16: the int4 decode kernel (warp MMAs fed
 * by in-register dequantisation, split-k reduced through distributed shared
 * memory inside a thread-block cluster); larger batches: the tensor-core
 * GEMM (w_hat dequantised into tensor memory, X T^-1 tiles by TMA, 64/128/256
 * tokens per tile). */
paro_status paro_linear(const paro_rot* rot, const void* X_dev,
                        const void* qweight_dev, const void* scales_dev, const void* zeros_dev,
                        void* Y_dev, int64_t tokens, int64_t in_features, int64_t out_features,
                        void* workspace_dev, size_t workspace_bytes, paro_stream stream);

/* paro_linear plus a bias: Y = (X T^-1) w_hat^T + b (CSDN article,
 * section 2.1, Y = XW + b). bias_dev is fp16 [out_features] (2-byte
 * aligned) or NULL; it is added to the fp32 sum before the single rounding
 * to fp16. Arguments, workspace and errors as paro_linear. */
paro_status paro_linear_bias(const paro_rot* rot, const void* X_dev,
                             const void* qweight_dev, const void* scales_dev, const void* zeros_dev,
                             const void* bias_dev, void* Y_dev, int64_t tokens, int64_t in_features,
                             int64_t out_features, void* workspace_dev, size_t workspace_bytes,
                             paro_stream stream);

/* The general form of the layer: paro_linear_bias with weights quantised in
 * groups of `group` channels (128, 64 or 256, packed by paro_pack_weights_ex).
 * A rotation handle, if given, must have been prepared with the same group
 * (else PARO_ERR_ARG). paro_linear and paro_linear_bias are this call with
 * group 128. Paper: CSDN article, section 2.1 (Y = (X T^-1)(T W) + b) and
 * section 5.2 (group size). */
paro_status paro_linear_ex(const paro_rot* rot, const void* X_dev,
                           const void* qweight_dev, const void* scales_dev, const void* zeros_dev,
                           const void* bias_dev, int group, void* Y_dev, int64_t tokens, int64_t in_features,
                           int64_t out_features, void* workspace_dev, size_t workspace_bytes,
                           paro_stream stream);

/* Row-parallel use (several GPUs each holding a slice of the input channels,
 * cut on 128-channel boundaries): the group-diagonal T lets every rank
 * rotate only its own channels (paper notes, "independent rotation"), so a
 * rank's share of Y is (X_r T_r^-1) w_hat_r^T over its slice. This call
 * writes that share as unrounded fp32 sums, Yf_dev fp32 [tokens][out]
 * (16-byte aligned), without a bias; the ranks add their shares (an
 * all-reduce) and paro_finalize rounds once. The rotation handle, the
 * weights and X_dev are the rank's slice (in_features = the slice's width).
 * Other arguments as paro_linear_ex. */
paro_status paro_linear_partial(const paro_rot* rot, const void* X_dev,
                                const void* qweight_dev, const void* scales_dev, const void* zeros_dev, int group,
                                float* Yf_dev, int64_t tokens, int64_t in_features, int64_t out_features,
                                void* workspace_dev, size_t workspace_bytes, paro_stream stream);

/* Y_dev fp16 [tokens][out] = fp16(Yf_dev + bias) with one rounding; bias_dev
 * fp16 [out] or NULL. The last step of a row-parallel layer (no counterpart
 * in the paper beyond Y = XW + b, CSDN article, section 2.1). */
paro_status paro_finalize(const float* Yf_dev, const void* bias_dev, void* Y_dev, int64_t tokens,
                          int64_t out_features, paro_stream stream);

/* paro_linear for decode batches (tokens <= 16) that allocates nothing and
 * takes no workspace: for callers that cannot allocate device memory, such
 * as a serving engine that hands all device memory to its own pool at start-
 * up, or code that must not call cudaMalloc while a CUDA graph is captured.
 * No counterpart in the paper: this is a deployment convenience.
 * The rotated activations X T^-1 go to a 1 MiB static device array that the
 * library holds on every device that loads it until the process exits, so
 * tokens * in_features * 2 must not exceed 1 MiB (else PARO_ERR_ARG; e.g. 16
 * tokens x 32768 channels). Every call shares that array and it keeps the
 * last call's contents (nothing in it needs clearing); calls that overlap on
 * the GPU race on it, so serialise them (one stream, or events).
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) once for that device; make that first call before
 * any stream capture. Arguments are those of paro_linear without the
 * workspace (group-128 weights); the caller still owns X, the weights and Y. */
paro_status paro_linear_noalloc(const paro_rot* rot, const void* X_dev,
                                const void* qweight_dev, const void* scales_dev, const void* zeros_dev,
                                void* Y_dev, int64_t tokens, int64_t in_features, int64_t out_features,
                                paro_stream stream);

/* One-shot form of paro_rotate with the rotation given as the pages state
 * it, X T^-1 from (pairs, theta, alpha, K, group) (CSDN article, section 2.1,
 * the activation side; paper notes, "key design", T = (prod R) diag(alpha)).
 * It runs paro_rot_create, paro_rotate and paro_rot_destroy in turn:
 * allocating and synchronous, for one-off use; repeated calls should keep a
 * handle. Arguments as in those calls (pairs/theta/alpha on the host, X and
 * Xr fp16 [tokens][in_features] on the device). */
paro_status paro_rotate_once(const void* X_dev, void* Xr_dev, int64_t tokens, int64_t in_features,
                             const int16_t* pairs_host, const float* theta_host, const float* alpha_host,
                             int K, int group, int pairs_per_group, paro_stream stream);

/* One-shot form of paro_linear, Y = (X T^-1) w_hat^T from (X, pairs, theta,
 * alpha, qweight, scales, zeros) (CSDN article, section 2.1, without the
 * bias): paro_rot_create (group 128), a workspace from cudaMalloc,
 * paro_linear, then everything is released; synchronous. Arguments as in
 * paro_rot_create and paro_linear. */
paro_status paro_linear_once(const void* X_dev, const int16_t* pairs_host, const float* theta_host,
                             const float* alpha_host, const void* qweight_dev, const void* scales_dev,
                             const void* zeros_dev, void* Y_dev, int64_t tokens, int64_t in_features,
                             int64_t out_features, int K, int pairs_per_group, paro_stream stream);

/* Fault word of the current device: 0, or the code of the first bounded wait
 * inside a tensor-core kernel that ran out (about 2 s) because a pipeline
 * stage never arrived: the kernel (0 prefill GEMM, 10 tensor-core rotation,
 * 20 its 256-channel form) plus the role (1 TMA producer, 2 MMA issuer,
 * 3 dequantisation, 4 epilogue, 5 a drain before exit); 6 is the self-test
 * below. The CTA that saw it raises an
 * abort flag in its shared memory: every role stops issuing copies and
 * MMAs, the copies and MMAs already issued are waited for (bounded), tensor
 * memory is released and the CTA exits without storing its tile. The output
 * of that call is not valid. Synchronous (copies one word); clear != 0
 * resets it to 0. */
paro_status paro_fault_status(int* code, int clear);

/* Self-test of the failure detection (no counterpart in the paper): enqueue
 * a one-thread kernel that waits, with a limit of limit_us microseconds
 * (1..2000000), on an mbarrier at which nothing arrives, with no copy or MMA
 * in flight. The wait runs out, records code 6 in the fault word and the
 * kernel returns; the context stays usable. Read and clear the code with
 * paro_fault_status. */
paro_status paro_check_wait_timeout(uint32_t limit_us, paro_stream stream);

/* Message for the last non-OK status returned on this thread ("" if none). */
const char* paro_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* PARO_H */
