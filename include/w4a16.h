/*
 * w4a16.h -- C ABI of the B200 (sm_100a) W4A16 weight-only INT4 linear layer.
 *
 * The layer: 16-bit activations A [M, K] times a weight matrix W [K, N] that is stored as 4-bit
 * codes, eight per 32-bit word, with one FP16 scale per group of `group` consecutive input
 * channels and, for the asymmetric scheme, one 4-bit zero-point per group. The kernel reads the
 * codes, dequantizes them on chip, w = (q - z) * s, and multiplies them against the 16-bit
 * activations with FP32 accumulation.
 *   - "4.3 Weight-only INT4", section 1 "W4A16 storage and compute": eight 4-bit codes per
 *     32-bit word, one FP16 scale per group, a zero-point for asymmetric schemes, dequantized
 *     on chip to FP16/BF16, then multiplied with 16-bit activations.
 *   - "INT4 and Low-Bit Inference -- Inference Optimization", section 6-9, "the packed layout":
 *     qweight (K/8, N) int32, scales (K/g, N) fp16, qzeros (K/g, N/8) int32.
 *   - "INT4 LLMs: What 4-Bit Quantization Means and When to Use It", section "What INT4 means in
 *     an LLM": signed codes -8..7, two per byte.
 *
 * Conventions shared by every entry point
 *   - All pointers named as device buffers are CUDA device (or managed) memory of the current
 *     device. The caller allocates and frees every buffer; the library never allocates memory and
 *     never synchronises the device. Every call is asynchronous on `stream` (a cudaStream_t passed
 *     as void*, NULL = the legacy default stream).
 *   - Shapes: K % 8 == 0, N % 8 == 0, group in {32, 64, 128}, K % group == 0, M >= 1.
 *     N % 8 == 0 also makes every row of A, C and the packed arrays 16-byte aligned when the
 *     base pointers are (N = 8 with 16-bit C rows is 16 bytes).
 *   - Device pointers must be 16-byte aligned.
 *   - Arguments are checked on the host before any launch. A rejected call returns a negative
 *     w4a16_status and launches nothing. A failed launch returns W4A16_ECUDA.
 *   - Conditions found on the device are written to an optional device int `dev_status`
 *     (first error wins; the caller zeroes it). They never fault or trap the GPU.
 *   - The entry points are stateless and thread-safe, except where an entry point says otherwise.
 *
 * Packed layout ("plain", the checkpoint layout)
 *   codes  int32 [K/8, N]   word (j, n), bits [4i, 4i+4): code of (k = 8j + i, n).
 *                           symmetric: two's-complement nibble, value -8..7.
 *                           asymmetric: unsigned nibble, value 0..15.
 *   scales fp16  [K/g, N]   scale of group (g, n).
 *   zeros  int32 [K/g, N/8] asymmetric only: word (g, j), bits [4i, 4i+4): zero of (g, n = 8j + i),
 *                           unsigned 0..15. NULL for the symmetric scheme.
 *   Dequantized weight: w[k, n] = (q[k, n] - z[k/g, n]) * s[k/g, n]  (z = 0 when symmetric).
 */
#ifndef W4A16_H
#define W4A16_H

#include <stddef.h>
#include <stdint.h>

/* Symbols of this header are the only ones the shared library exports. */
#ifndef W4A16_API
#define W4A16_API __attribute__((visibility("default")))
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. Zero is success; every error is negative. */
typedef enum {
    W4A16_OK = 0,
    W4A16_EINVAL = -1,        /* bad shape, null pointer, or a value outside its enum        */
    W4A16_EALIGN = -2,        /* a device pointer is not 16-byte aligned                      */
    W4A16_EUNSUPPORTED = -3,  /* a group size, dtype, layout or kernel choice not supported   */
    W4A16_ENONFINITE = -4,    /* device: a weight group held Inf or NaN (via dev_status)      */
    W4A16_EWORKSPACE = -5,    /* workspace smaller than w4a16_workspace_bytes()               */
    W4A16_ECUDA = -6,         /* a CUDA runtime call or a kernel launch failed                */
    W4A16_ETIMEOUT = -7       /* device: a bounded wait gave up (via dev_status)              */
} w4a16_status;

/* 16-bit activation (and output) type. */
typedef enum { W4A16_F16 = 0, W4A16_BF16 = 1 } w4a16_dtype;

/* Weight layout handed to w4a16_gemm. */
typedef enum {
    W4A16_LAYOUT_PLAIN = 0,   /* codes / scales / zeros as above                              */
    W4A16_LAYOUT_TILED = 1    /* the single buffer written by w4a16_repack                    */
} w4a16_layout;

/* Kernel family chosen by the M-based dispatch (see w4a16_select_kernel). */
typedef enum {
    W4A16_KERNEL_AUTO = 0,    /* let the dispatch decide                                      */
    W4A16_KERNEL_GEMV = 1,    /* decode GEMV: split-K CUDA-core (plain layout, any M) or the
                                 persistent stream-K warp-MMA kernel (tiled layout, M <= 16, over
                                 K slices when A does not fit whole) */
    W4A16_KERNEL_TC = 2       /* tcgen05 tensor-core GEMM, TMEM accumulator (tiled layout)     */
} w4a16_kernel;

/*
 * w4a16_quantize -- round-to-nearest group quantization of an FP16 weight matrix.
 *   "INT4 LLMs: What 4-Bit Quantization Means and When to Use It", sections "What INT4 means in
 *   an LLM" and "Why mapping to 16 values still works" (16 levels, group-wise scales, symmetric
 *   grid centred on zero vs. affine grid with an offset); "4.3 Weight-only INT4", section 1.
 *   For each group (g, n) of `group` consecutive k in column n, in FP64:
 *     sym:  s = fp16(amax / 7),                              q = clamp(rne(w / s), -8, 7)
 *     asym: lo = min(0, min w), hi = max(0, max w), s = fp16((hi - lo) / 15),
 *           z = clamp(rne(-lo / s), 0, 15),                  q = clamp(rne(w / s) + z, 0, 15)
 *   rne = round half to even; every division is an IEEE FP64 division. A group whose scale rounds
 *   to zero stores s = 1, z = 0 and q = z.
 * Arguments
 *   W          device, fp16 [K, N] row-major (n fastest).
 *   K, N       input channels (rows of W) and output channels (columns).
 *   group      32, 64 or 128.
 *   sym        1 = symmetric (no zeros), 0 = asymmetric.
 *   codes      device out, int32 [K/8, N].
 *   scales     device out, fp16 [K/g, N].
 *   zeros      device out, int32 [K/g, N/8] when sym == 0; must be NULL when sym == 1.
 *   dev_status device int or NULL. Set to W4A16_ENONFINITE when a group holds Inf/NaN (that
 *              group's outputs are then unspecified).
 *   stream     cudaStream_t.
 * Returns W4A16_OK, W4A16_EINVAL, W4A16_EALIGN, W4A16_EUNSUPPORTED or W4A16_ECUDA.
 */
W4A16_API int w4a16_quantize(const void* W, int K, int N, int group, int sym, int32_t* codes, void* scales,
                   int32_t* zeros, int* dev_status, void* stream);

/*
 * w4a16_dequantize -- the packed weight expanded to a 16-bit matrix: w[k, n] = (q - z) * s,
 *   exact in FP32 and rounded once to out_dtype. This is the naive path that the fused kernels
 *   are measured against: "4.3 Weight-only INT4", section 4 (dequantize the INT4 matrix to FP16 in
 *   memory, then a standard GEMM: the weights cross HBM as 4 bits, then twice as 16 bits);
 *   "INT4 and Low-Bit Inference", section 5 "The kernel is half the story".
 * Arguments
 *   codes, scales, zeros  device, plain layout as produced by w4a16_quantize (zeros NULL iff sym).
 *   K, N, group, sym      as for w4a16_quantize.
 *   out_dtype             W4A16_F16 or W4A16_BF16.
 *   W                     device out, [K, N] row-major, out_dtype (2 K N bytes).
 *   stream                cudaStream_t.
 * Returns W4A16_OK, W4A16_EINVAL, W4A16_EALIGN, W4A16_EUNSUPPORTED or W4A16_ECUDA.
 */
W4A16_API int w4a16_dequantize(const int32_t* codes, const void* scales, const int32_t* zeros, int K, int N,
                     int group, int sym, int out_dtype, void* W, void* stream);

/*
 * w4a16_gptq_workspace_bytes -- device workspace that w4a16_gptq_quantize needs for a K x N
 * weight: 16 K^2 + 8 K N + 1024 N + 256 bytes (the damped Hessian and its factors in FP64, an FP64
 * working copy of W, one block of propagated errors). 0 on a bad shape.
 */
W4A16_API size_t w4a16_gptq_workspace_bytes(int K, int N);

/*
 * w4a16_gptq_quantize -- the GPTQ calibrated encoder: the same packed output as w4a16_quantize,
 * with every rounding error fed forward onto the input channels not yet quantized, weighted by
 * the calibration inputs' curvature. "4.3 Weight-only INT4", section 2 "GPTQ: quantize and
 * compensate as you go": objective ||X W - X W_hat||^2 with H = 2 X^T X (2.1); input channels
 * fixed in order, the free ones moved by -(w_i - w_hat_i) / [H_F^-1]_ii [H_F^-1]_{:,i} (2.2),
 * with damping, a Cholesky factorisation and block updates. Each group's RTN scale (and zero)
 * is taken from its compensated weights when its first input channel comes up. All arithmetic
 * is FP64; an offline, one-time step (not on the inference path).
 * Arguments
 *   W          device, fp16 [K, N] row-major (K input channels, N output channels).
 *   X          device, calibration inputs [S, K] row-major, 16-bit of type x_dtype.
 *   x_dtype    W4A16_F16 or W4A16_BF16.
 *   S          calibration rows, >= 1.
 *   K, N, group, sym   as for w4a16_quantize (the workspace, 16 K^2 + 8 K N bytes, is the only
 *              limit on K).
 *   damp       damping as a fraction of mean(diag H), added to the diagonal (0.01 is usual);
 *              >= 0 and finite.
 *   codes, scales, zeros   device out, the plain layout of w4a16_quantize (zeros NULL iff sym).
 *   workspace, ws_bytes    device, at least w4a16_gptq_workspace_bytes(K, N) bytes, 16-byte
 *              aligned; contents on entry do not matter.
 *   dev_status nullable device int: W4A16_ENONFINITE when W holds Inf/NaN or H + damping is not
 *              positive definite (outputs then unspecified).
 *   stream     cudaStream_t. About 3 K / 32 kernel launches.
 * Returns W4A16_OK, W4A16_EINVAL, W4A16_EALIGN, W4A16_EUNSUPPORTED, W4A16_EWORKSPACE or
 * W4A16_ECUDA (host-side checks; nothing is launched on an error).
 */
W4A16_API int w4a16_gptq_quantize(const void* W, const void* X, int x_dtype, int S, int K, int N, int group,
                                  int sym, double damp, int32_t* codes, void* scales, int32_t* zeros,
                                  void* workspace, size_t ws_bytes, int* dev_status, void* stream);

/*
 * w4a16_awq_workspace_bytes -- device workspace of w4a16_awq_quantize for a K x N weight and S
 * calibration rows: 8 (K^2 + K N + 2 K + 64 + P) + 256 bytes, P = ceil(S / 64) ceil(N / 64)
 * rounded up to even. 0 on a bad shape.
 */
W4A16_API size_t w4a16_awq_workspace_bytes(int K, int N, int S);

/*
 * w4a16_awq_quantize -- the AWQ activation-aware encoder: input channel j of W is scaled by s_j
 * before RTN quantization, and the layer's input must be divided by the same s_j (the caller
 * folds 1/s into whatever produces X). "4.3 Weight-only INT4", section 3 "AWQ: find channels to
 * protect from activations": salient channels come from the activation distribution (3.1);
 * Y = (X S^-1)(S W), Y_hat = (X S^-1) D(Q(S W)), factors searched on calibration data and
 * paired with clipping (3.2). Search (FP64): s_j = fp16(max(mean_s |x_sj|, 2^-14)^alpha),
 * alpha = i / 20 for i = 0..19, scored by ||X W - (X S^-1) D(Q(S W))||^2 over the calibration
 * rows (first minimum wins; alpha = 0 is plain RTN); then for every group and output channel
 * the RTN range of the scaled weights shrunk by r = 1 - i / 20, i = 0..10, scored by the group's
 * output error (first minimum wins; r = 1 is plain RTN). An offline, one-time step.
 * Arguments
 *   W, X, x_dtype, S, K, N, group, sym   as for w4a16_gptq_quantize.
 *   codes, scales, zeros   device out: the plain layout of w4a16_quantize, of S W.
 *   s_in       device out, fp16 [K]: the factors s_j (divide the layer's input by them).
 *   workspace, ws_bytes    device, at least w4a16_awq_workspace_bytes(K, N, S) bytes, 16-byte
 *              aligned; contents on entry do not matter.
 *   dev_status nullable device int (reserved; nothing is reported at present).
 *   stream     cudaStream_t. About 4 x 20 + 8 kernel launches.
 * Returns W4A16_OK, W4A16_EINVAL, W4A16_EALIGN, W4A16_EUNSUPPORTED, W4A16_EWORKSPACE or
 * W4A16_ECUDA (host-side checks; nothing is launched on an error).
 */
W4A16_API int w4a16_awq_quantize(const void* W, const void* X, int x_dtype, int S, int K, int N, int group,
                                 int sym, int32_t* codes, void* scales, int32_t* zeros, void* s_in,
                                 void* workspace, size_t ws_bytes, int* dev_status, void* stream);

/*
 * The W8A8 comparison path (FP8 E4M3 weights and activations, tcgen05 kind::f8f6f4 GEMM) that
 * W4A16 is measured against: "INT8 vs INT4 Quantization, in depth", section "Two regimes: waiting
 * for memory, waiting for math" (8-bit weights double the bytes read but the 8-bit tensor rate
 * doubles the math rate; the crossover batch follows from the roofline). Not a W4A16 format.
 * Codes: E4M3 round-to-nearest-even of x / s (computed in FP64), saturated to +-448; scales
 * s = fp32(amax / 448) (1 when amax = 0), per output channel (weights) and per row (activations).
 *
 * w4a16_fp8_quantize_weights -- W fp16 [K, N] (device) -> Wq uint8 [N, K] (device, one row of K
 *   codes per output channel) and w_scales fp32 [N] (device). K % 128 == 0 and N % 128 == 0
 *   (else W4A16_EUNSUPPORTED). An offline step.
 * w4a16_fp8_quantize_acts -- A [M, K] of a_dtype (device) -> Aq uint8 [M, K] and a_scales fp32 [M]
 *   (device). K % 128 == 0. Part of every W8A8 step (activations change each step).
 * w4a16_fp8_gemm -- C[m, n] = (sum_k Aq[m, k] Wq[n, k]) a_scales[m] w_scales[n], FP32
 *   accumulation, C [M, N] of c_dtype (device). M >= 1; K % 128 == 0; N % 128 == 0.
 *   dev_status (nullable) receives W4A16_ETIMEOUT if a bounded pipeline wait expired.
 * All three: every pointer 16-byte aligned (W4A16_EALIGN), the caller owns every buffer, no
 * allocation or synchronisation; W4A16_OK, W4A16_EINVAL, W4A16_EALIGN, W4A16_EUNSUPPORTED or
 * W4A16_ECUDA.
 */
W4A16_API int w4a16_fp8_quantize_weights(const void* W, int K, int N, uint8_t* Wq, float* w_scales, void* stream);
W4A16_API int w4a16_fp8_quantize_acts(const void* A, int a_dtype, int M, int K, uint8_t* Aq, float* a_scales,
                                      void* stream);
W4A16_API int w4a16_fp8_gemm(const uint8_t* Aq, const float* a_scales, int M, int K, const uint8_t* Wq,
                             const float* w_scales, int N, void* C, int c_dtype, int* dev_status, void* stream);

/*
 * w4a16_repack_bytes -- size in bytes of the tiled buffer for a K x N weight (0 on bad shape).
 */
W4A16_API size_t w4a16_repack_bytes(int K, int N, int group, int sym);

/*
 * w4a16_repack -- one-time load-time permutation of the plain packed layout into the tiled
 * layout that w4a16_gemm reads fastest. The codes, zeros and scales are moved, not changed
 * (except the scale of a group whose codes all equal its zero point, stored as 0): nothing is
 * rounded or re-quantized, and every dequantized weight is the same. "INT4 and Low-Bit Inference", section 5 "The kernel is half the story" (weights
 * pre-permuted at load so unpacking is branch-free and coalesced); "4.3 Weight-only INT4",
 * section 4 (weights pre-reordered into a layout that suits runtime reads).
 * Tiled layout: one record per unit of 128 output channels x 128 input channels; unit (t, c)
 * covers n in [128 t, 128 t + 128), k in [128 c, 128 c + 128) and has record index
 * t * (K / 128) + c. Records follow each other with no padding; a record is
 *     R = 8192 + G * 256 + (sym ? 0 : G * 64) bytes,  G = 128 / group:
 *   bytes [0, 8192)   codes: block h (h = 0..3, k in [128 c + 32 h, + 32)) at 2048 h; channel
 *                     n % 128 owns the 16 bytes at slot ((n % 128) XOR 2h) of its block, and word
 *                     w (w = 0..3) of them is plain word (j, n) with j = 16 c + 4 h + w;
 *   then G x 256 B    scales: group row c * G + gg at 256 gg, channel n % 128 at + 2 (n % 128);
 *                     a (group, channel) whose codes all equal its zero point (0 when symmetric)
 *                     stores scale 0 -- its dequantized weights are 0 with either scale;
 *   then G x 64 B     zeros (asym only): group row c * G + gg at 64 gg, plain words
 *                     [16 t, 16 t + 16) of that row.
 * Each word is re-encoded: nibble slot p (bits 4p..4p+3, p = 0..3) holds the code of element 2p
 * (k = 8j + 2p) and slot p + 4 that of element 2p + 1; symmetric codes are stored offset-binary,
 * q + 8, so that both schemes dequantize as (u - z) * s with z = 8 for the symmetric one.
 * A range of consecutive units is one contiguous range of bytes (one bulk copy), and the XOR slot
 * keeps the warp-level MMA's 16-byte reads of four blocks of one channel on different banks.
 * Requires N % 128 == 0 and K % 128 == 0 (else W4A16_EUNSUPPORTED).
 * Arguments: codes, scales, zeros as produced by w4a16_quantize (zeros NULL iff sym);
 * tiled = device out of w4a16_repack_bytes() bytes; stream.
 */
W4A16_API int w4a16_repack(const int32_t* codes, const void* scales, const int32_t* zeros, int K, int N,
                 int group, int sym, void* tiled, void* stream);

/*
 * w4a16_workspace_bytes -- device scratch that w4a16_gemm needs for an M x N x K call, large
 * enough for any kernel the call may run: 64 KiB of per-tile counters of the stream-K decode
 * kernel, followed by FP32 partial sums (the split-K sums of the plain-layout GEMV, or the decode
 * kernel's cut-tile sums and, when it runs over S slices of K, S x M x N FP32 slice outputs).
 * Depends on the SM count of the current device.
 * Returns 0 only for arguments w4a16_gemm rejects.
 */
W4A16_API size_t w4a16_workspace_bytes(int M, int N, int K, int group);

/*
 * w4a16_select_kernel -- the M-based dispatch, as a pure host function: returns the
 * w4a16_kernel that w4a16_gemm(..., W4A16_KERNEL_AUTO) runs on the tiled layout for this shape.
 * Small M is bound by the weight stream and goes to the decode GEMV (W4A16_KERNEL_GEMV); larger M
 * goes to the tensor-core GEMM ("INT8 vs INT4 Quantization, in depth", section "Two regimes:
 * waiting for memory, waiting for math"). The plain layout always runs the CUDA-core GEMV.
 * The environment variable W4A16_FORCE_KERNEL=gemv|tc overrides the choice.
 * On the tiled layout the decode GEMV is the persistent stream-K kernel (one CTA per SM, unit
 * records streamed by bulk copies, warp-level tensor-core MMA). When the M rows of A for the
 * whole K do not fit in its shared memory it runs over S equal slices of K (each served by its
 * own CTAs of one launch, FP32 slice outputs added in order by a last kernel). AUTO takes it for
 * M <= 8 (whole K or slices) and for 9 <= M <= 16 only when K fits whole; otherwise the
 * tensor-core GEMM (measured: with 9-16 rows the sliced decode kernel is slower than the
 * tensor-core GEMM).
 */
W4A16_API int w4a16_select_kernel(int M, int N, int K, int group);

/*
 * w4a16_gemm -- C[M, N] = A[M, K] . dequant(W)[K, N], FP32 accumulation, C in the dtype of A.
 *   "4.3 Weight-only INT4", section 4 (read, unpack, dequantize and multiply in one kernel, so
 *   each weight byte crosses HBM once); section 1 (dequantize on chip, 16-bit multiply inputs).
 * Arguments
 *   A          device, [M, K] row-major, fp16 or bf16 (a_dtype).
 *   a_dtype    W4A16_F16 or W4A16_BF16. C has the same type.
 *   M, K       rows of A; input channels.
 *   wq         device: codes int32 [K/8, N] (layout PLAIN) or the w4a16_repack buffer (TILED).
 *   layout     W4A16_LAYOUT_PLAIN or W4A16_LAYOUT_TILED.
 *   scales     device fp16 [K/g, N] for PLAIN; ignored (may be NULL) for TILED.
 *   zeros      device int32 [K/g, N/8] for PLAIN asymmetric; NULL for symmetric; ignored for TILED.
 *   N, group   output channels; group size.
 *   sym        1 = symmetric codes, 0 = asymmetric (must match how the weight was quantized).
 *   C          device out, [M, N] row-major, dtype a_dtype. Must not alias A or the weights.
 *   workspace  device scratch of at least w4a16_workspace_bytes(M, N, K, group) bytes, 16-byte
 *              aligned, owned by the caller. Its first 64 KiB (tile counters) must be zero before
 *              the first call that uses it; every call that completes without a device error
 *              leaves them zero, so a workspace is zeroed once, at allocation. Calls that share
 *              one workspace must be ordered on the GPU (same stream). After a call that set
 *              dev_status to W4A16_ETIMEOUT, zero the workspace again.
 *   ws_bytes   size of workspace.
 *   kernel     W4A16_KERNEL_AUTO, or a forced W4A16_KERNEL_GEMV / W4A16_KERNEL_TC. GEMV reads both
 *              layouts (TILED: M <= 16); TC reads the TILED layout only. Other combinations
 *              return W4A16_EUNSUPPORTED.
 *   dev_status device int or NULL: set to W4A16_ETIMEOUT if a bounded on-device wait gave up
 *              (the output is then unspecified; the device stays usable).
 *   stream     cudaStream_t.
 * Ordering. The decode kernel (tiled layout, M <= 16) is launched with programmatic dependent
 * launch: it may start while the kernel before it on the stream is still running, and it
 * starts streaming the tiled weight buffer before it waits for that kernel (it waits before it
 * reads A). The weight buffer must therefore not be written by the kernel that immediately
 * precedes w4a16_gemm on the stream, unless that kernel makes its writes visible device-wide
 * before its threads exit, as w4a16_repack does; a memory copy, an event or any other stream
 * operation in between also orders them. A, C and the workspace carry no such condition.
 * Returns W4A16_OK, W4A16_EINVAL, W4A16_EALIGN, W4A16_EUNSUPPORTED, W4A16_EWORKSPACE or
 * W4A16_ECUDA.
 */
W4A16_API int w4a16_gemm(const void* A, int a_dtype, int M, int K, const void* wq, int layout,
               const void* scales, const int32_t* zeros, int N, int group, int sym, void* C,
               void* workspace, size_t ws_bytes, int kernel, int* dev_status, void* stream);

/*
 * w4a16_gemm_noalloc -- w4a16_gemm for callers that cannot allocate device memory.
 *   (The pages have no counterpart: this is a convenience of this library.)
 *   w4a16_gemm needs a caller-provided workspace for its split-K partial sums. Callers that have
 *   no way to provide one -- for example a plugin inside a host application that owns every
 *   device allocation, or a latency-critical loop that must never call cudaMalloc because it can
 *   block and synchronise the device -- call this instead. It runs the plain-layout split-K
 *   CUDA-core GEMV with its partial sums in one static 8 MiB device array of this library,
 *   reserved on every GPU that loads the library until the process exits; it calls no
 *   cudaMalloc, cudaFree or other allocating routine.
 * Limits and sharing
 *   - The call's partial sums, splits x min(M, 16) x N FP32 values (see w4a16_workspace_bytes),
 *     must fit in 8 MiB; a larger call returns W4A16_EWORKSPACE and launches nothing.
 *   - Every call on a device uses the same array, which keeps the last call's contents (nothing
 *     in it needs to start at zero). Calls that can overlap on the GPU -- on different streams,
 *     or from different host threads -- race on it: order them on one stream.
 *   - Every call looks up the array's device address with cudaGetSymbolAddress (with the
 *     caller's device current); the first call on a device also loads the library's device code
 *     there, so make that first call before any stream capture begins.
 * Arguments as w4a16_gemm with layout W4A16_LAYOUT_PLAIN (codes [K/8, N], scales [K/g, N],
 * zeros [K/g, N/8] or NULL when sym), without workspace, kernel choice or dev_status.
 * Returns W4A16_OK, W4A16_EINVAL, W4A16_EALIGN, W4A16_EUNSUPPORTED, W4A16_EWORKSPACE or
 * W4A16_ECUDA.
 */
W4A16_API int w4a16_gemm_noalloc(const void* A, int a_dtype, int M, int K, const int32_t* codes,
                                 const void* scales, const int32_t* zeros, int N, int group, int sym,
                                 void* C, void* stream);

/*
 * w4a16_set_wait_limit_ns -- the time limit of every bounded wait inside the library's kernels
 *   (a pipeline barrier, or a counter another CTA of the same launch sets), in nanoseconds, for
 *   launches made after the call; 0 restores the default of 2 s. Returns the previous limit.
 *   A wait that runs out makes the kernel record W4A16_ETIMEOUT in dev_status, stop issuing work,
 *   let its copies and MMAs in flight complete, free its tensor memory and return, so the device
 *   stays usable; its outputs are then unspecified and its workspace must be zeroed again. A very
 *   short limit (say 1 ns) makes the waits run out on purpose, which is how the timeout path is
 *   tested. Not on the pages: a property of this library. Process-wide; safe to call from any
 *   thread (each launch reads the value once).
 */
W4A16_API uint64_t w4a16_set_wait_limit_ns(uint64_t ns);

/* w4a16_status_str -- a static, human-readable name for a status code. */
W4A16_API const char* w4a16_status_str(int status);

/* w4a16_version -- library version as 10000 * major + 100 * minor + patch. */
W4A16_API int w4a16_version(void);

#ifdef __cplusplus
}
#endif

#endif /* W4A16_H */
