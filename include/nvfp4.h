/*
 * nvfp4.h -- C ABI of the B200 (sm_100a) NVFP4 library: two-level NVFP4
 * quantization and block-scaled FP4 matrix products for the linear layers of a
 * diffusion transformer (QKV / out projections, MLP fc1 / fc2).
 *
 * Sources the operations follow (web pages, by title and section):
 *  [DiT] "NVFP4-DiT: Efficient 4-Bit Audio-Guided Video Diffusion Transformers
 *        for Low-Cost Video Generation", Methodology 1 (Definition III.1:
 *        Q_FP4(v; s) = s * clip(round(v/s)_FP4, -6, 6); E2M1 = 1 sign,
 *        2 exponent, 1 mantissa bit) and 3 (two FP4 values per byte, FP32
 *        accumulation).
 *  [RFC] "[RFC]: NVFP4 Quantization Support for Diffusion Models", Motivation
 *        (two-level scaling: an FP8 scale per 16 values plus an FP32 tensor
 *        scale; Blackwell SM100), Open Questions 1 (W4A16 and W4A4).
 *
 * Conventions shared by every call
 *  - Row-major.  Activations X are [M, K], weights W are [N, K] (nn.Linear
 *    layout), Y = X W^T is [M, N].  The 16-value quantization block runs along
 *    K, the reduction axis, for both operands.
 *  - An NVFP4 tensor of shape [rows, k] is three buffers:
 *      codes  rows * k/2 bytes, row stride k/2; element 2j of a row sits in the
 *             low nibble of byte j, element 2j+1 in the high nibble; a nibble
 *             is sign(1) exponent(2) mantissa(1).
 *      sf     nvfp4_sf_bytes(rows, k) bytes of unsigned E4M3 block scales in
 *             the tensor-core scale-factor layout: the scale of row r, block c
 *             (kb = k/16 blocks per row) sits at byte
 *               ((r/128)*(kb/4) + c/4)*512 + (r%32)*16 + ((r%128)/32)*4 + c%4,
 *             rows padded to a multiple of 128 with zero bytes.
 *      scale  one float (device memory), the tensor scale g.
 *    Element value = e2m1(code) * e4m3(sf) * g.
 *  - Every pointer is DEVICE memory unless stated; the caller allocates and
 *    owns every buffer.  Calls are asynchronous on `stream` (a cudaStream_t;
 *    NULL = legacy default stream) and never synchronize the host.
 *  - Kernels run on the calling thread's current CUDA device, and every buffer
 *    must be that device's memory (the stream too must belong to it).  Where a
 *    pointer lives is not checked: a buffer of another device is a caller
 *    error whose outcome the library does not define.
 *  - Argument checks run on the host before any launch; a failed check
 *    returns an error and launches nothing.  Launch failures return
 *    NVFP4_ERR_CUDA.
 *  - `dev_status` (nullable, device int): a kernel that gives up on a bounded
 *    internal wait writes NVFP4_ERR_TIMEOUT there and returns without hanging.
 *    The library never clears it; the caller zeroes it and reads it after the
 *    stream has synchronized.
 *  - Inputs must be finite; non-finite values give unspecified codes.  The
 *    amax pass of nvfp4_quantize (data-derived tensor scale) detects them and
 *    writes NVFP4_ERR_NONFINITE to dev_status (if no error is there yet).
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *nvfp4_stream_t;   /* same type as cudaStream_t */

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,        /* null pointer, negative size, bad flag/dtype      */
    NVFP4_ERR_UNSUPPORTED_SHAPE = 2,  /* K or N not a supported multiple (see each call) */
    NVFP4_ERR_MISALIGNED = 3,         /* pointer or row stride not 16-byte aligned        */
    NVFP4_ERR_UNSUPPORTED_DEVICE = 4, /* current device is not compute capability 10.0    */
    NVFP4_ERR_CUDA = 5,               /* a CUDA runtime/driver call failed                */
    NVFP4_ERR_TIMEOUT = 6,            /* device-side bounded wait expired (dev_status)    */
    NVFP4_ERR_WORKSPACE = 7,          /* workspace missing or too small                   */
    NVFP4_ERR_NONFINITE = 8           /* input held Inf or NaN (dev_status, amax pass)     */
} nvfp4_status;

enum { NVFP4_DTYPE_BF16 = 0, NVFP4_DTYPE_F32 = 1 };

/* nvfp4_quantize flags */
enum { NVFP4_SCALE_GIVEN = 1 };

/* GEMM epilogue activations, applied to alpha * acc before the output is
 * formed (bf16 / FP32 values, or the NVFP4 codes of the next layer):
 *   NVFP4_ACT_GELU_TANH  0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))), tanh
 *                        from the hardware approximation (relative error about
 *                        2^-11), the activation of the DiT family's MLPs. */
enum { NVFP4_ACT_NONE = 0, NVFP4_ACT_GELU_TANH = 1 };

/* Bytes of the scale buffer of a [rows, k] NVFP4 tensor:
 * ceil(rows/128)*128 * k/16.  Returns 0 for rows < 0 or k not a multiple of 64. */
size_t nvfp4_sf_bytes(int64_t rows, int64_t k);

/* Bytes of device workspace nvfp4_quantize needs when it derives the tensor
 * scale from the data (no NVFP4_SCALE_GIVEN): per-CTA partial maxima, each
 * tagged with a per-call number so that the contents need no initialisation
 * (they are not preserved).  Calls that overlap on the GPU must not share a
 * workspace.  The numbers come from a counter of this copy of the library in
 * this process: a workspace must not be shared with another process or another
 * loaded copy of the library, whose numbers can coincide. */
size_t nvfp4_quantize_workspace_bytes(int64_t rows, int64_t k);

/*
 * nvfp4_quantize -- two-level NVFP4 quantization of a bf16 tensor
 * ([DiT] Definition III.1 with the [RFC] two-level scaling):
 *   g   = amax(|x|) / (6 * 448)               (IEEE single division)
 *   per row and 16-value block along k:  a_b = max|x|,
 *         sf = E4M3_rne_satfinite(a_b / (6 g)),  s = e4m3(sf) * g
 *   per element: code = E2M1_rne(clip(x / s, -6, 6)), sign of x kept;
 *         a block with s == 0 gives codes 0.
 * x_bf16        [rows, k] bf16, row stride ld_x elements (ld_x >= k, ld_x % 8 == 0,
 *               pointer 16-byte aligned).
 * rows >= 0;    k > 0 and k % 64 == 0.  rows <= 65535 * 128 = 8,388,480 (one
 *               128-row block per grid row); larger is NVFP4_ERR_UNSUPPORTED_SHAPE.
 * codes         out, rows * k/2 bytes (16-byte aligned).
 * sf            out, nvfp4_sf_bytes(rows, k) bytes (16-byte aligned); padding rows
 *               are written as zero.
 * tensor_scale  device float.  With flags & NVFP4_SCALE_GIVEN it is read as g
 *               (for weights quantized once, or a calibrated activation scale);
 *               otherwise g is computed from the data and written there.
 * workspace     device scratch of >= nvfp4_quantize_workspace_bytes(rows, k)
 *               bytes, 16-byte aligned; unused (may be NULL) with SCALE_GIVEN.
 * One kernel on `stream`: with a data-derived scale a persistent,
 * co-resident grid reduces amax, hands it over grid-wide (a bounded wait) and
 * quantizes; when the grid cannot be co-resident, two kernels (amax pass, then
 * quantize) give the same result.  rows == 0 is a no-op (g = 0 is written when
 * not given).
 */
nvfp4_status nvfp4_quantize(const void *x_bf16, int64_t rows, int64_t k, int64_t ld_x,
                            uint8_t *codes, uint8_t *sf, float *tensor_scale,
                            unsigned flags, void *workspace, size_t workspace_bytes,
                            int *dev_status, nvfp4_stream_t stream);

/*
 * nvfp4_quantize_noalloc -- the source pages have no counterpart: this is a
 * deployment variant of nvfp4_quantize.  Same arguments, same results, bit
 * for bit, minus the workspace, for callers that cannot allocate device
 * memory (a plugin whose host application owns all device memory, a server
 * that allocates nothing after start-up, a caller without a CUDA allocator).
 * The amax pass keeps its per-CTA partial maxima in a fixed device array of
 * NVFP4_NOALLOC_SCRATCH_FLOATS floats (1 KB) that every GPU loading the
 * library holds until the process exits.  That pass never needs more entries
 * than that, whatever the tensor size; a problem that would is rejected with
 * NVFP4_ERR_WORKSPACE.  Nothing in the array has to start at zero.  Every call
 * shares the one array: calls that overlap on the GPU (for instance on two
 * streams) race and may produce wrong scales -- serialize them.  The first call
 * on each device looks up the array's device address (a runtime call, no
 * allocation); make that first call before any stream capture.  The call
 * itself allocates nothing.  The looked-up address is kept until
 * nvfp4_shutdown(): after cudaDeviceReset() (or anything else that destroys
 * and recreates the device's primary context, which may move the array) call
 * nvfp4_shutdown() before the next call.  Row limit as nvfp4_quantize.
 */
enum { NVFP4_NOALLOC_SCRATCH_FLOATS = 256 };
nvfp4_status nvfp4_quantize_noalloc(const void *x_bf16, int64_t rows, int64_t k, int64_t ld_x,
                                    uint8_t *codes, uint8_t *sf, float *tensor_scale,
                                    unsigned flags, int *dev_status, nvfp4_stream_t stream);

/*
 * nvfp4_layernorm_quantize -- the LayerNorm in front of a block's first
 * projections, emitting their NVFP4 input directly ([DiT] Abstract and
 * Methodology 3: every linear layer runs through the FP4 matmul; [RFC]
 * Motivation: two-level scaling).  The pages do not define LayerNorm; the
 * reading is the DiT pre-norm over the hidden dimension with the adaLN
 * modulation x (1 + scale) + shift of each sample written as a per-channel
 * affine shared by a group of rows:
 *   mu, var of each row from S1 = sum x_j, S2 = sum x_j^2 in double,
 *   var = max(S2 / k - mu^2, 0), rstd = 1 / sqrt(var + eps) (double, IEEE),
 *   y_j = ((x_j - (float)mu) * (float)rstd) * gamma_j + beta_j  (FP32 ops),
 * then y is quantized exactly as nvfp4_quantize quantizes an FP32 tensor (same
 * tensor-scale rule, block scales, codes and layouts).  The bf16 LayerNorm
 * output is never stored.  (Any summation order gives the same S1 and S2
 * when a row's values span fewer than about 45 binary orders of magnitude,
 * the case for activations; beyond that the statistics can differ from an
 * index-order sum in their last bit.)
 * x_bf16         [rows, k] bf16, row stride ld_x (as nvfp4_quantize).
 * gamma, beta    nullable device FP32 [groups, k], 16-byte aligned; row r uses
 *                group r / rows_per_group (rows_per_group == 0: one group);
 *                NULL reads as 1 (gamma) and 0 (beta).
 * eps            > 0 (DiT: 1e-6).
 * codes, sf, tensor_scale, flags, workspace, workspace_bytes, dev_status:
 *                as nvfp4_quantize (with NVFP4_SCALE_GIVEN the tensor scale is
 *                read; otherwise it is the largest |y| / 2688, found in the
 *                same kernel by a grid-wide handoff through the workspace).
 * rows <= 2^31, k % 64 == 0, k <= 8192 (a row is held in a warp's registers).
 * One kernel on `stream`.  Non-finite input is
 * flagged in dev_status (NVFP4_ERR_NONFINITE) when the scale is data-derived.
 */
nvfp4_status nvfp4_layernorm_quantize(const void *x_bf16, int64_t rows, int64_t k, int64_t ld_x,
                                      const float *gamma, const float *beta, int64_t rows_per_group,
                                      double eps, uint8_t *codes, uint8_t *sf, float *tensor_scale,
                                      unsigned flags, void *workspace, size_t workspace_bytes,
                                      int *dev_status, nvfp4_stream_t stream);

/*
 * Block size per layer ([DiT] Algorithmic framework, Algorithm 1 / Eq. 9:
 *   BlockSize(l) = argmin_{b in {1,2,4,8,16,32,64}} Error(l,b) + lambda Memory(b)/Memory_max).
 *
 * nvfp4_quantize_block -- nvfp4_quantize with `block` (16, 32 or 64) values per
 * E4M3 scale: the block maximum is taken over `block` values along k and the
 * scale byte is repeated in each of its block/16 slots of the block-16
 * scale layout, so nvfp4_gemm_w4a4 multiplies the result unchanged.  Other
 * arguments as nvfp4_quantize (block 16 is nvfp4_quantize itself).
 *
 * nvfp4_block_size_errors -- one pass over x computing Error(l, b) before
 * normalisation for every candidate: errors[i] = sum_j (x_j - Q_b(x)_j)^2 for
 * b = 2^i (i = 0..6), Q_b the two-level quantization with the block maximum
 * over b values and tensor scale *tensor_scale (device float, e.g. from
 * nvfp4_quantize), in double (element differences rounded once in FP32);
 * errors[7] = sum_j x_j^2.  errors: 8 device doubles, overwritten.
 * x as nvfp4_quantize (k % 64 == 0).  One kernel (after a memset of errors).
 *
 * nvfp4_select_block_size -- host function, Eq. 9 on HOST errors[8] (as
 * above, copied back): Error(b) = errors[i] / errors[7], Memory(b) = 4 + 8/b
 * bits per value (E2M1 plus one 8-bit scale per block; the tensor scale is
 * shared by the whole tensor and left out), Memory_max = Memory(1) = 12.
 * Returns the b of the first minimum, or 0 for a null pointer or a negative
 * or NaN lambda.  The pages give no value for lambda.
 */
nvfp4_status nvfp4_quantize_block(const void *x_bf16, int64_t rows, int64_t k, int64_t ld_x, int block,
                                  uint8_t *codes, uint8_t *sf, float *tensor_scale, unsigned flags,
                                  void *workspace, size_t workspace_bytes, int *dev_status,
                                  nvfp4_stream_t stream);
nvfp4_status nvfp4_block_size_errors(const void *x_bf16, int64_t rows, int64_t k, int64_t ld_x,
                                     const float *tensor_scale, double *errors, nvfp4_stream_t stream);
int nvfp4_select_block_size(const double *errors, double lambda);

/*
 * nvfp4_dequantize -- v = (e2m1(code) * e4m3(sf)) * g, rounded once (RNE) to
 * out_dtype ([DiT] Definition III.1: the quantizer returns s * round(...)).
 * codes/sf/tensor_scale as produced by nvfp4_quantize for [rows, k];
 * out: [rows, k] contiguous, NVFP4_DTYPE_BF16 or NVFP4_DTYPE_F32, 16-byte aligned.
 */
nvfp4_status nvfp4_dequantize(const uint8_t *codes, const uint8_t *sf,
                              const float *tensor_scale, int64_t rows, int64_t k,
                              void *out, int out_dtype, nvfp4_stream_t stream);

/*
 * nvfp4_fake_quantize -- fake quantization for quantization-aware training
 * ([DiT] Definition III.1 and Methodology 2, where a straight-through
 * estimator is used across the fake quantizer in training): quantization
 * exactly as nvfp4_quantize (same tensor-scale rule, block scales and
 * codes), followed in the same kernel by
 *   y = e2m1(code) * e4m3(sf) * g,  rounded once (RNE) to y_dtype,
 * the value nvfp4_dequantize would return, so that training sees in its
 * forward pass what the W4A4 product multiplies.  No codes or scales are
 * stored.
 * x_bf16, rows, k, ld_x, tensor_scale, flags, workspace, workspace_bytes,
 *               dev_status: as nvfp4_quantize (the workspace is needed unless
 *               NVFP4_SCALE_GIVEN; nvfp4_quantize_workspace_bytes gives its size).
 * y             out, [rows, k] contiguous (row stride k), NVFP4_DTYPE_BF16 or
 *               NVFP4_DTYPE_F32, 16-byte aligned.
 * clip_mask     out, nullable: rows * k/8 bytes, row stride k/8, 16-byte
 *               aligned; bit j % 8 of byte j / 8 of a row is set where
 *               element j was clipped, i.e. s > 0 and |x| > 6 s with the
 *               block's s = e4m3(sf) * g (IEEE single product), compared
 *               exactly.  A block with s == 0 clips nothing.
 * One kernel with a given scale; with a data-derived scale, one kernel when
 * the grid can be co-resident, else two (amax pass, then fake quantization).
 */
nvfp4_status nvfp4_fake_quantize(const void *x_bf16, int64_t rows, int64_t k, int64_t ld_x,
                                 void *y, int y_dtype, uint8_t *clip_mask,
                                 float *tensor_scale, unsigned flags,
                                 void *workspace, size_t workspace_bytes,
                                 int *dev_status, nvfp4_stream_t stream);

/*
 * nvfp4_ste_backward -- backward rule of the straight-through estimator with
 * the clip mask ([DiT] Methodology 2; clip's derivative is zero outside its
 * range): grad_x = grad_y where the mask bit is clear, +0 where it is set.
 * (The plain estimator, without the mask, is the identity and needs no call.)
 * grad_y, grad_x [rows, k] contiguous in dtype (NVFP4_DTYPE_BF16 or
 * NVFP4_DTYPE_F32), 16-byte aligned; grad_x may be grad_y (in place).
 * clip_mask as written by nvfp4_fake_quantize for [rows, k].
 * rows >= 0, k > 0 and k % 16 == 0.  One kernel on `stream`.
 */
nvfp4_status nvfp4_ste_backward(const void *grad_y, const uint8_t *clip_mask, int64_t rows, int64_t k,
                                int dtype, void *grad_x, nvfp4_stream_t stream);

/*
 * nvfp4_gemm_w4a4 -- block-scaled FP4 x FP4 product with FP32 accumulation
 * ([DiT] 3. Systems optimization; [RFC] Open Questions 1, W4A4):
 *   acc[m,n] = sum_k (e2m1(a)*e4m3(sfa)) * (e2m1(b)*e4m3(sfb))   (FP32, tensor cores)
 *   Y[m,n]   = alpha * acc[m,n],  alpha = g_a * g_b              (FP32)
 * A: a_codes [M, K/2], a_sf (nvfp4_sf_bytes(M, K)), a_scale (device float g_a).
 * B: b_codes [N, K/2], b_sf (nvfp4_sf_bytes(N, K)), b_scale (device float g_b).
 * M >= 0, N > 0, K > 0 with K % 64 == 0.
 * Output, one of two forms:
 *  - y != NULL: Y [M, N] row-major in y_dtype (BF16 rounded RNE, or F32);
 *    N % 8 == 0 for BF16, N % 4 == 0 for F32; y 16-byte aligned.
 *  - y == NULL and y_codes != NULL: the next layer's NVFP4 activations, Y
 *    quantized in the epilogue with the caller's tensor scale g_y (*y_scale),
 *    exactly as nvfp4_quantize with NVFP4_SCALE_GIVEN would quantize the FP32
 *    value alpha*acc: y_codes [M, N/2], y_sf nvfp4_sf_bytes(M, N); needs
 *    N % 64 == 0.  y_amax (nullable device float, caller-initialised): receives
 *    the running max of |output value| (atomic max), from which the caller can
 *    derive the next call's g_y.
 * act: NVFP4_ACT_NONE, or NVFP4_ACT_GELU_TANH to output GELU(alpha*acc) -- for
 *    an MLP's first layer with the NVFP4 output, the second layer's input is
 *    produced without writing or re-reading the activation in 16-bit form.
 * All code/scale pointers 16-byte aligned.  One persistent kernel on `stream`.
 */
nvfp4_status nvfp4_gemm_w4a4(const uint8_t *a_codes, const uint8_t *a_sf, const float *a_scale,
                             const uint8_t *b_codes, const uint8_t *b_sf, const float *b_scale,
                             int64_t M, int64_t N, int64_t K,
                             void *y, int y_dtype,
                             uint8_t *y_codes, uint8_t *y_sf, const float *y_scale, float *y_amax,
                             int act, int *dev_status, nvfp4_stream_t stream);

/*
 * nvfp4_gemm_w4a4_grouped -- up to NVFP4_MAX_GROUP independent W4A4 products
 * in one persistent launch (the product of each is nvfp4_gemm_w4a4's): the
 * linear layers of a transformer block that do not depend on each other --
 * e.g. the self-attention QKV projection of the image tokens and the
 * cross-attention K and V projections of the text tokens, which have
 * different M, N and K -- share one tile scheduler, so the small ones do not
 * each pay a launch and a partly idle wave.  ([DiT] Methodology 3 runs every
 * linear layer through the FP4-packed matmul.)
 * problems   HOST array of `count` (1 .. NVFP4_MAX_GROUP) descriptions; each
 *            field means what the argument of the same name of
 *            nvfp4_gemm_w4a4 means and is checked the same way.  Every problem
 *            has the same output kind: all y != NULL (then y_dtype applies to
 *            all), or all y == NULL with NVFP4 outputs (y_codes, y_sf, y_scale,
 *            optional y_amax), and the same act.  Problems with M == 0 are
 *            skipped.
 * One launch of the single-CTA kernel (128 x 128 tiles) for any N; the
 * array is read during the call only.
 */
typedef struct {
    const uint8_t *a_codes;
    const uint8_t *a_sf;
    const float *a_scale;
    const uint8_t *b_codes;
    const uint8_t *b_sf;
    const float *b_scale;
    int64_t M, N, K;
    void *y;
    uint8_t *y_codes;
    uint8_t *y_sf;
    const float *y_scale;
    float *y_amax;
    int act;
} nvfp4_gemm_problem;

enum { NVFP4_MAX_GROUP = 8 };

nvfp4_status nvfp4_gemm_w4a4_grouped(const nvfp4_gemm_problem *problems, int count, int y_dtype,
                                     int *dev_status, nvfp4_stream_t stream);

/*
 * nvfp4_gemm_w4a16 -- weights-only NVFP4 ([RFC] Open Questions 1, W4A16):
 *   Y[m,n] = g_w * sum_k x[m,k] * (e2m1(w[n,k]) * e4m3(sfw))
 * The weight element e2m1 * e4m3 is exact in bf16; it is formed in shared
 * memory inside the kernel and fed to bf16 tensor-core MMAs with FP32
 * accumulation; g_w is applied in the FP32 epilogue.
 * x_bf16 [M, K] contiguous bf16 (16-byte aligned); w_codes [N, K/2], w_sf,
 * w_scale as from nvfp4_quantize; K % 64 == 0; y [M, N] in y_dtype
 * (N % 8 == 0 for BF16, N % 4 == 0 for F32).
 */
nvfp4_status nvfp4_gemm_w4a16(const void *x_bf16, const uint8_t *w_codes, const uint8_t *w_sf,
                              const float *w_scale, int64_t M, int64_t N, int64_t K,
                              void *y, int y_dtype, int *dev_status, nvfp4_stream_t stream);

/*
 * MX variant (the [RFC] lists MXFP4 among related issues, as another format):
 * E2M1 elements in blocks of 32 along k, one power-of-two scale per block as
 * an unsigned E8M0 byte (value 2^(byte - 127)), no tensor scale.  The pages
 * give no scale rule; the OCP Microscaling one is used:
 *   e = floor(log2 max|x|) - 2, clamped to [-127, 127] (-127 for an all-zero
 *   block); byte = e + 127; code = E2M1_rne(clip(x / 2^e, -6, 6)), sign kept.
 * Codes [rows, k/2] as for NVFP4; scales in the same tensor-core layout with
 * kb = k/32 blocks per row:
 *   byte of (row r, block c) at ((r/128)*(kb/4) + c/4)*512 + (r%32)*16
 *                               + ((r%128)/32)*4 + c%4,
 * rows padded to 128 with zero bytes.  k must be a multiple of 128.
 */
size_t nvfp4_mx_sf_bytes(int64_t rows, int64_t k);      /* ceil(rows/128)*128 * k/32, 0 if invalid */

/* MX quantization of a bf16 [rows, k] tensor (row stride ld_x, ld_x % 8 == 0),
 * rows <= 4194240.  One kernel; pointers 16-byte aligned. */
nvfp4_status nvfp4_mx_quantize(const void *x_bf16, int64_t rows, int64_t k, int64_t ld_x,
                               uint8_t *codes, uint8_t *sf, nvfp4_stream_t stream);

/* v = e2m1(code) * 2^(byte - 127), exact in bf16 and FP32; out [rows, k]. */
nvfp4_status nvfp4_mx_dequantize(const uint8_t *codes, const uint8_t *sf, int64_t rows, int64_t k,
                                 void *out, int out_dtype, nvfp4_stream_t stream);

/*
 * nvfp4_mx_gemm -- Y = act(sum_k a^ b^), a^ = e2m1(a) * 2^(sfa - 127) (and b^),
 * with the block-32 E8M0 tensor-core MMA (kind::mxf4), FP32 accumulation.
 * A [M, K] and B [N, K] as nvfp4_mx_quantize writes them; K % 128 == 0;
 * Y [M, N] bf16 (N % 8 == 0) or FP32 (N % 4 == 0); act as nvfp4_gemm_w4a4.
 * One persistent kernel: 256 x 256 tiles on CTA pairs (cta_group::2) when
 * N % 256 == 0, else 128 x 128 tiles on single CTAs.
 */
nvfp4_status nvfp4_mx_gemm(const uint8_t *a_codes, const uint8_t *a_sf, const uint8_t *b_codes,
                           const uint8_t *b_sf, int64_t M, int64_t N, int64_t K, void *y, int y_dtype,
                           int act, int *dev_status, nvfp4_stream_t stream);

/*
 * nvfp4_attention -- attention over an NVFP4 key / value cache ([DiT]
 * Algorithmic framework, Eq. 10: softmax(Q K^T / sqrt(d) + log(s_head)) V with a
 * per-head scale s_head; Systems optimization: FP4-packed attention):
 *   Q [H*Lq, d], K and V [H*Lk, d]: NVFP4 tensors as nvfp4_quantize writes them
 *   (quantized along d), head h owning rows h*Lq .. and h*Lk .. ; tensor scales
 *   q_scale, k_scale, v_scale (device floats).
 *   S = Q K^T on the block-scaled FP4 tensor cores (FP32); online softmax in
 *   FP32 with the hardware exp2; P rounded to f16; V decoded exactly to f16
 *   (e2m1 * e4m3: at most 6 significant bits within [2^-10, 2688]); O = P V on
 *   the 16-bit tensor cores (FP32), divided by the row sum and multiplied by
 *   g_v, rounded to bf16.
 * s_head    nullable device float [H] (1 for every head).  Within one head's
 *           softmax the log(s_head) term is a constant shift of every logit.
 * out       bf16 [H*Lq, d], 16-byte aligned.
 * workspace device scratch of >= nvfp4_attention_workspace_bytes(H, Lk, d)
 *           bytes, 16-byte aligned: V decoded to f16, [H*Lk, d] (once per
 *           call, then read by every query tile), then 32 four-byte words
 *           per head that tag the head's decoded parts with a per-call
 *           number (the counter of nvfp4_quantize's workspace: the same rule
 *           on sharing); not preserved.  Calls that run at the same time need
 *           workspaces of their own.
 * d == 128, Lq and Lk multiples of 128 (no masking), H <= 65535.  When Lq / 128
 * is even, one persistent kernel (one CTA per SM, all resident) takes 256
 * queries of a head per work item and decodes V itself, each item a share of
 * its head's rows; otherwise (or when the grid cannot be co-resident) a V
 * decode kernel runs first.
 */
size_t nvfp4_attention_workspace_bytes(int64_t H, int64_t Lk, int64_t d);   /* H * d * Lk * 2 + H * 128 */
nvfp4_status nvfp4_attention(const uint8_t *q_codes, const uint8_t *q_sf, const float *q_scale,
                             const uint8_t *k_codes, const uint8_t *k_sf, const float *k_scale,
                             const uint8_t *v_codes, const uint8_t *v_sf, const float *v_scale,
                             const float *s_head, int64_t H, int64_t Lq, int64_t Lk, int64_t d, void *out,
                             void *workspace, size_t workspace_bytes, int *dev_status, nvfp4_stream_t stream);

/* Static text for a status code. */
const char *nvfp4_status_string(nvfp4_status s);

/* Number of this library's kernels launched since load (host-side counter,
 * all threads).  For accounting in benchmarks. */
uint64_t nvfp4_launch_count(void);

/* Forget the library's host-side caches (per-device capability checks and the
 * device address of nvfp4_quantize_noalloc's scratch array); the next call
 * looks them up again.  Frees nothing on the device (the library holds no
 * device allocation).  Not safe concurrently with other calls. */
void nvfp4_shutdown(void);

/*
 * nvfp4_debug_wait_timeout -- the pages have no counterpart: a check of the
 * library's failure detection.  Launches one warp that waits, through the
 * same bounded mbarrier wait the GEMM and quantize kernels use, on a barrier
 * that nothing ever arrives at.  After limit_us microseconds (1 .. 2000000)
 * the wait gives up, the kernel writes NVFP4_ERR_TIMEOUT to *dev_status and
 * returns: the stream and the context stay usable.  dev_status must be a
 * device int the caller zeroed.
 */
nvfp4_status nvfp4_debug_wait_timeout(int *dev_status, int64_t limit_us, nvfp4_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4_H_ */
