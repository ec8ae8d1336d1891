/*
 * twq.h -- C ABI of the B200 (sm_100a) fused dual-component W4A4 + low-rank
 * linear layer of TwinQuant ("TwinQuant: Learnable Subspace Decomposition for
 * 4-Bit LLM Quantization", ICML'26).
 *
 * The layer (TwinQuant §2, Eq. (3), with the learned transforms of §4.1 folded
 * into the factors offline):
 *
 *     Y = Q(X) Q(R) + bf16( Q(X) Q(L1) ) L2      X: b x m,  W = L1 L2 + R: m x n
 *
 *   Q        symmetric 4-bit quantizer of Eq. (1): codes round(v / s) with
 *            s = max|v| / 7 (q_max = 2^(4-1) - 1), per group of 128 elements
 *            along the reduction dimension m (§5.1: group size 128 for weights
 *            and activations). Rounding is half to even; v / s is a correctly
 *            rounded float32 division; an all-zero group has s = 0, codes 0.
 *   stage 1  H = Q(X) Q(L1), b x r, exact int32 per group, scaled in fp32 per
 *            group (Eq. (2) applied group by group).
 *   stage 2  H is rounded to BF16 and multiplied by L2 (BF16, unquantized) with
 *            fp32 accumulation. H never leaves the chip (§4.3: the first
 *            low-rank GEMM's result is kept on chip and fed to the second).
 *   epilogue Y = bf16_rne(Y_res + Y_lr), one store (§4.3: a single epilogue
 *            merges both components).
 *
 * Variants (declared below): the layer with the activation quantizer inside it
 * (twq_fused_linear_x, decode batches), from host memory to host memory
 * (twq_fused_linear_x_host), with 8-bit activations (W4A8, §5.1:
 * twq_quantize_act_a8 / twq_fused_linear_a8 / twq_fused_linear_x_a8), with the
 * pages' INT4 stage 2 (twq_pack_l2_int4 / twq_fused_linear_s2q), and the offline
 * fold of the learned transforms (twq_fold_transforms).
 *
 * Memory: every pointer is a DEVICE pointer owned by the caller (except the
 * x_host / y_host buffers of twq_fused_linear_x_host); the library never
 * allocates, frees or synchronizes (except twq_device_status and the offline
 * twq_fold_transforms). Every call is asynchronous on `stream`; inputs must stay
 * live until the stream reaches the call. All base pointers must be 16-byte
 * aligned.
 *
 * Errors: arguments are validated on the host before anything is launched; a
 * failing check returns a status and launches nothing. A launch failure is
 * reported as TWQ_ERR_CUDA. Kernels never trap: every wait inside a kernel is
 * bounded, and a wait that runs out records a code that twq_device_status
 * returns.
 *
 * Formats ("K-major" = the reduction index m is contiguous):
 *   codes    two's-complement nibbles in [-7, 7], element 2p in the low nibble
 *            of byte p, element 2p+1 in the high nibble.
 *   xq, sx   b x (m/2) bytes, row-major; b x (m/128) fp32 scales, row-major.
 *   rq, sr   n x (m/2) bytes (column j of R, K-major); (m/128) x n fp32.
 *   l1q, sl1 r x (m/2) bytes (column c of L1, K-major); (m/128) x r fp32.
 *   l2t      n x r BF16: L2 transposed (K-major for stage 2).
 *   y        b x n BF16, row-major.
 * Shapes: m % 128 == 0; n % 128 == 0; r == 0 or (r % 16 == 0 and r <= 256);
 *   b >= 0 (b == 0 is a no-op).
 */
#ifndef TWQ_H_
#define TWQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TWQ_API __attribute__((visibility("default")))
#else
#define TWQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream (NULL = the legacy default stream). */
typedef struct CUstream_st* twq_stream_t;

typedef enum {
  TWQ_OK = 0,
  TWQ_ERR_INVALID_ARG = 1,     /* null pointer, bad shape or size */
  TWQ_ERR_UNSUPPORTED = 2,     /* valid but outside the library's limits (e.g. r > 256) */
  TWQ_ERR_MISALIGNED = 3,      /* a pointer or stride breaks the 16-byte rule */
  TWQ_ERR_CUDA = 4,            /* a CUDA runtime/driver call or launch failed */
  TWQ_ERR_NOT_IMPLEMENTED = 5,
  TWQ_ERR_DEVICE = 6           /* a kernel's bounded wait ran out (twq_device_status) */
} twq_status;

/* Packed weights of one layer (all device pointers, caller-allocated). */
typedef struct {
  int64_t m, n, r;
  uint8_t* rq;   /* n x m/2 */
  float* sr;     /* m/128 x n */
  uint8_t* l1q;  /* r x m/2      (may be NULL iff r == 0) */
  float* sl1;    /* m/128 x r    (may be NULL iff r == 0) */
  uint16_t* l2t; /* n x r BF16   (may be NULL iff r == 0) */
} twq_weights;

/* Library version as 10000*major + 100*minor + patch. */
TWQ_API int twq_version(void);

/* Human-readable name of a status code (static string). */
TWQ_API const char* twq_status_string(twq_status s);

/*
 * Byte sizes of the five packed-weight buffers {rq, sr, l1q, sl1, l2t} for an
 * m x n layer of rank r (TwinQuant §3, Observation 2: the low-rank part adds
 * r(m + n) parameters; here L1 is 4-bit with per-group scales, L2 is BF16).
 * Host only; returns TWQ_ERR_INVALID_ARG on a bad shape.
 */
TWQ_API twq_status twq_weights_sizes(int64_t m, int64_t n, int64_t r, size_t bytes_out[5]);

/*
 * Byte sizes of {xq, sx} for b tokens of width m. Host only; TWQ_ERR_INVALID_ARG
 * on b < 0 or m not a positive multiple of 128, TWQ_ERR_UNSUPPORTED beyond the
 * quantizer's limits (m > 2^24 or b > 2^30).
 */
TWQ_API twq_status twq_act_sizes(int64_t b, int64_t m, size_t bytes_out[2]);

/*
 * Online activation quantizer (TwinQuant Eq. (1) per token and group of 128;
 * §4.3: the activation is quantized once and reused by the residual GEMM and
 * the first low-rank GEMM).
 *   x    b x m BF16 with row stride ldx elements (ldx >= m, ldx % 8 == 0)
 *   xq   b x m/2 bytes (output), sx b x m/128 fp32 (output)
 * Bit-exact with the definition above. X must be finite.
 */
TWQ_API twq_status twq_quantize_act(const uint16_t* x, int64_t b, int64_t m, int64_t ldx, uint8_t* xq,
                            float* sx, twq_stream_t stream);

/*
 * Offline weight packing (TwinQuant §4.1: the transformed factors U', V', R'
 * are prepared offline; Eq. (1) per output column and group of 128 along m).
 *   R   m x n BF16 row-major;  L1 m x r BF16 row-major;  L2 r x n BF16 row-major
 *   out buffers and shape {m, n, r} in *w (sizes from twq_weights_sizes).
 * R and L1 are quantized (bit-exact); L2 is transposed into l2t unchanged.
 * L1 and L2 may be NULL iff w->r == 0.
 */
TWQ_API twq_status twq_pack_weights(const uint16_t* R, const uint16_t* L1, const uint16_t* L2,
                            const twq_weights* w, twq_stream_t stream);

/*
 * The fused dual-component layer (TwinQuant §4.3, Fig. 4): one persistent
 * kernel that runs the residual GEMM Q(X)Q(R) and the low-rank stage 1
 * Q(X)Q(L1) on 5th-generation tensor cores (int8 operands unpacked from the
 * 4-bit codes in shared memory, exact int32 accumulation per group in tensor
 * memory, fp32 scaling per group), keeps H on chip, rounds it to BF16, runs
 * stage 2 against L2, and writes Y once.
 *   xq, sx  from twq_quantize_act;  w  from twq_pack_weights;  y  b x n BF16 (output)
 * w->r == 0 gives exactly the twq_w4a4_only result.
 * Decode shapes (b <= 16) run a split-K kernel launched with programmatic
 * stream serialization: when the kernel just before it on the stream signals
 * programmatic completion early (twq_quantize_act does), its prologue and its
 * reads of the packed weights start while that kernel is still running, and
 * its reads of xq / sx wait until that kernel has completed. So xq / sx may come
 * from the preceding kernel, but the weights must not be written by a kernel
 * that signals early (twq_pack_weights does not). The decode kernel itself
 * signals at entry, so the next decode call's prologue and weight reads overlap
 * it; a kernel of the caller's that is launched after it with programmatic
 * serialization must wait (griddepcontrol.wait) before it reads y.
 */
TWQ_API twq_status twq_fused_linear(const uint8_t* xq, const float* sx, int64_t b, const twq_weights* w,
                            uint16_t* y, twq_stream_t stream);

/*
 * The 4-bit activation codes stored one per byte, for prefill batches. The codes and
 * scales are exactly those of twq_quantize_act (TwinQuant Eq. (1), q_max = 7, per
 * token and group of 128): only their storage differs, element k of a row in byte k
 * as a two's-complement int8 in [-7, 7], twice the bytes of the packed form
 * (b x m instead of b x m/2). The layer's tensor-core kernel reads them where its
 * copy engine puts them, so it unpacks only the weights, which halves its unpack
 * work; at prefill sizes the extra activation bytes cost far less than that work.
 *   x    b x m BF16, row stride ldx elements (ldx >= m, ldx % 8 == 0), finite
 *   xq8  b x m int8 (output);  sx  b x (m/128) fp32 (output)
 * Errors as twq_quantize_act.
 */
TWQ_API twq_status twq_quantize_act_i8(const uint16_t* x, int64_t b, int64_t m, int64_t ldx,
                                       int8_t* xq8, float* sx, twq_stream_t stream);

/*
 * The fused layer (as twq_fused_linear) on activation codes stored one per byte:
 * the 4-bit codes of twq_quantize_act_i8, or the 8-bit codes of W4A8
 * (twq_quantize_act_a8). Each group's int8 x int4 dot product is exact in the int32
 * accumulator (|sum| <= 128 * 127 * 7) and scaled per group in FP32, so with 4-bit
 * codes the result is bitwise that of twq_quantize_act + twq_fused_linear.
 *   xq8  b x m int8;  sx  b x (m/128) fp32;  w, y, shapes and errors as
 *   twq_fused_linear. Prefill batches (b > 16, m >= 256, n % 256 == 0) run the
 *   CTA-pair tensor-core kernel; decode batches the split-K decode kernel.
 * Same function as twq_fused_linear_a8 (either name).
 */
TWQ_API twq_status twq_fused_linear_i8(const int8_t* xq8, const float* sx, int64_t b,
                                       const twq_weights* w, uint16_t* y, twq_stream_t stream);

/*
 * The fused layer with the activation quantizer inside it, for decode batches
 * (TwinQuant §4.3: the activation is quantized once, on chip, and the codes feed
 * both the residual GEMM and the first low-rank GEMM). Each CTA quantizes its
 * slice of X straight into shared memory, so Q(X) never goes to HBM and the
 * whole layer is one launch.
 *   x    b x m BF16, row stride ldx elements (ldx >= m, ldx % 8 == 0), finite
 *   w    from twq_pack_weights;  y  b x n BF16 (output)
 * Result: bitwise identical to twq_quantize_act followed by twq_fused_linear.
 * Limits: 1 <= b <= 16, m <= 8192, r <= 128 (b == 0 is a no-op); other shapes
 * return TWQ_ERR_UNSUPPORTED and launch nothing (use the two-call path).
 * Launched with programmatic stream serialization like twq_fused_linear: X may
 * come from the preceding kernel; the weights must not be written by a kernel
 * that signals early.
 */
TWQ_API twq_status twq_fused_linear_x(const uint16_t* x, int64_t ldx, int64_t b,
                                      const twq_weights* w, uint16_t* y, twq_stream_t stream);

/*
 * twq_fused_linear_x from host memory to host memory (TwinQuant §4.3, one decode
 * step of the layer as a serving loop issues it). On `stream`, in order:
 *   1. copy x_host (b x m BF16, row-major, contiguous) into x_dev;
 *   2. run twq_fused_linear_x on x_dev (ldx = m), writing y_dev (b x n BF16);
 *   3. copy y_dev into y_host (b x n BF16, row-major, contiguous).
 * Nothing is synchronized: the call returns once the three operations are
 * enqueued, and y_host holds the result once the stream reaches that point (an
 * event or a stream synchronize). Host buffers should be page-locked
 * (cudaHostAlloc / cudaHostRegister), or the copies are not asynchronous. The
 * caller owns all buffers; x_dev and y_dev must not be in use by other work on
 * other streams while the step runs (a loop that overlaps steps on two streams
 * gives each stream its own x_dev, y_dev and y_host).
 * Limits and errors: those of twq_fused_linear_x, all checked before anything is
 * enqueued; TWQ_ERR_CUDA if enqueueing a copy or the launch fails.
 */
TWQ_API twq_status twq_fused_linear_x_host(const uint16_t* x_host, int64_t b, const twq_weights* w,
                                           uint16_t* x_dev, uint16_t* y_dev, uint16_t* y_host,
                                           twq_stream_t stream);

/*
 * One layer call from host memory to host memory for any batch (TwinQuant §4.3:
 * the activation is quantized once and feeds both GEMMs of the fused layer;
 * this is the call a user makes with the activations in host memory). On
 * `stream`, in order:
 *   1. copy x_host (b x m BF16, row-major, contiguous) into x_dev;
 *   2. batches that twq_fused_linear_x takes (1 <= b <= 16, r <= 128,
 *      m <= 8192): that one-launch layer on x_dev (xq, sx are not touched and
 *      may be NULL); any other batch: twq_quantize_act_i8 of x_dev into xq
 *      (b x m bytes: the 4-bit codes one per byte) and sx (b x m/128 fp32), then
 *      twq_fused_linear_i8 into y_dev (the same Y as twq_quantize_act +
 *      twq_fused_linear, bitwise);
 *   3. copy y_dev (b x n BF16) into y_host.
 * Nothing is synchronized; y_host holds the result once the stream reaches the
 * end of the call. Host buffers should be page-locked, or the copies are not
 * asynchronous. The caller owns every buffer; x_dev, xq, sx and y_dev must not
 * be in use by other streams while the call runs. Errors: the checks of the
 * calls it makes, all before anything is enqueued; TWQ_ERR_CUDA if enqueueing
 * a copy or a launch fails.
 */
TWQ_API twq_status twq_linear_host(const uint16_t* x_host, int64_t b, const twq_weights* w,
                                   uint16_t* x_dev, int8_t* xq, float* sx, uint16_t* y_dev,
                                   uint16_t* y_host, twq_stream_t stream);

/*
 * W4A8: 4-bit weights with 8-bit activations, the second quantization setting
 * of TwinQuant §5.1. The activations use Eq. (1) with k = 8 (q_max = 127), in
 * groups of 128 along m with one FP32 scale per token and group; the weights
 * and the rest of the layer are those of twq_fused_linear (same twq_weights).
 *
 * twq_quantize_act_a8: x b x m BF16 (row stride ldx, ldx % 8 == 0) ->
 *   xq8  b x m int8 codes, row-major, element k of a row in byte k;
 *   sx   b x (m/128) FP32 scales.
 * Codes and scales are bitwise those of Eq. (1) with correctly rounded float
 * divisions, round half to even. Errors as twq_quantize_act.
 */
TWQ_API twq_status twq_quantize_act_a8(const uint16_t* x, int64_t b, int64_t m, int64_t ldx,
                                       int8_t* xq8, float* sx, twq_stream_t stream);

/*
 * The fused W4A8 layer: Y = bf16(Q8(X)Q(R) + bf16(Q8(X)Q(L1)) L2), each group's
 * int8 x int4 dot product exact in the int32 accumulator (|sum| <= 128 * 127 * 7),
 * scaled per group in FP32 as in twq_fused_linear.
 *   xq8, sx  from twq_quantize_act_a8;  w  from twq_pack_weights;  y  b x n BF16.
 * w->r == 0 gives the residual component alone. Shapes and errors as
 * twq_fused_linear: decode batches (b <= 16, r <= 128, m <= 8192) run the
 * split-K decode kernel (with programmatic stream serialization), larger ones the
 * tensor-core GEMM kernel, whose MMAs read the int8 X tile where TMA stored it.
 */
TWQ_API twq_status twq_fused_linear_a8(const int8_t* xq8, const float* sx, int64_t b,
                                       const twq_weights* w, uint16_t* y, twq_stream_t stream);

/*
 * twq_fused_linear_a8 with the 8-bit activation quantizer inside the layer
 * kernel (one launch, BF16 X in). Bitwise identical to twq_quantize_act_a8
 * followed by twq_fused_linear_a8. Arguments and limits as twq_fused_linear_x.
 */
TWQ_API twq_status twq_fused_linear_x_a8(const uint16_t* x, int64_t ldx, int64_t b,
                                         const twq_weights* w, uint16_t* y, twq_stream_t stream);

/*
 * The INT4 stage 2 of TwinQuant §4.3 (H requantized on chip to 4 bits and
 * multiplied by a 4-bit V = L2). Readings: H is rounded to BF16 as in the BF16
 * stage 2, then quantized with Eq. (1) (q_max = 7) per token in groups of 128
 * along r; L2 is quantized per output column in groups of 128 along r. Stage 2 is
 * then Eq. (2) group by group:
 *     Y = bf16(Y_res + sum_g s_H[i,g] s_V[g,j] sum_{k in g} Q_H[i,k] Q_V[j,k])
 * Limits: r == 128 or r == 256.
 *
 * twq_pack_l2_int4: L2 (r x n BF16, row-major) -> l2q (n x r/2 bytes, column j of
 *   L2 contiguous along r, nibbles as the codes format above) and sl2q ((r/128) x n
 *   fp32). Offline, with twq_pack_weights; bit-exact.
 * twq_fused_linear_s2q: xq, sx from twq_quantize_act; w from twq_pack_weights (its
 *   l2t is not read); l2q, sl2q from twq_pack_l2_int4; y b x n BF16. One launch; H
 *   never leaves the chip. Decode batches (b <= 16, r == 128, m <= 8192) run the
 *   split-K decode kernel, whose CTAs exchange per-token maxima of H over the
 *   cluster; other shapes run the tensor-core prefill kernel (on CTA pairs when
 *   b > 16, m >= 256 and n % 256 == 0, else on single CTAs), where H's codes
 *   overwrite it in shared memory and feed r/128 more int8 K groups of the
 *   residual accumulation. Errors as twq_fused_linear; r outside {128, 256} returns
 *   TWQ_ERR_UNSUPPORTED (r == 0: TWQ_ERR_INVALID_ARG).
 */
TWQ_API twq_status twq_pack_l2_int4(const uint16_t* L2, int64_t r, int64_t n, uint8_t* l2q,
                                    float* sl2q, twq_stream_t stream);
TWQ_API twq_status twq_fused_linear_s2q(const uint8_t* xq, const float* sx, int64_t b,
                                        const twq_weights* w, const uint8_t* l2q,
                                        const float* sl2q, uint16_t* y, twq_stream_t stream);

/* Residual component only: Y = bf16(Q(X) Q(R)) (TwinQuant Eq. (2)); ignores l1q/sl1/l2t. */
TWQ_API twq_status twq_w4a4_only(const uint8_t* xq, const float* sx, int64_t b, const twq_weights* w,
                         uint16_t* y, twq_stream_t stream);

/* Low-rank component only: Y = bf16(bf16(Q(X) Q(L1)) L2); ignores rq/sr. Needs r > 0. */
TWQ_API twq_status twq_lowrank_only(const uint8_t* xq, const float* sx, int64_t b, const twq_weights* w,
                            uint16_t* y, twq_stream_t stream);

/*
 * Unfused comparator (the naive schedule that TwinQuant §4.3 describes and
 * rejects): four launches -- residual GEMM to fp32 Y_res in HBM, stage 1 to
 * BF16 H in HBM, stage 2 to fp32 Y_lr in HBM, then Y = bf16(Y_res + Y_lr).
 * Same arithmetic as twq_fused_linear, so the result is bitwise identical.
 * workspace: device buffer of twq_unfused_workspace_bytes(b, n, r) bytes.
 */
TWQ_API size_t twq_unfused_workspace_bytes(int64_t b, int64_t n, int64_t r);
TWQ_API twq_status twq_unfused_linear(const uint8_t* xq, const float* sx, int64_t b, const twq_weights* w,
                              uint16_t* y, void* workspace, size_t workspace_bytes,
                              twq_stream_t stream);

/*
 * twq_unfused_linear without a caller-provided workspace, for callers that
 * may not allocate device memory (for example a plugin whose host framework
 * owns the whole device-memory budget, or a service that must not let a
 * cudaMalloc synchronize the device mid-stream). The TwinQuant pages have no
 * counterpart: this is a convenience of this library.
 *   Same arguments and result as twq_unfused_linear, minus the workspace.
 *   Scratch: a fixed 16 MiB array inside the library (a file-scope __device__
 *   object that every GPU which loads the library holds until the process
 *   exits). Calls whose twq_unfused_workspace_bytes(b, n, r) exceeds 16 MiB
 *   return TWQ_ERR_UNSUPPORTED and launch nothing.
 *   With w->r == 0 the comparator is the W4A4 kernel alone (twq_w4a4_only),
 *   which uses no scratch, so the 16 MiB limit does not apply.
 *   Set-up: the first call on each device resolves the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture. The address is kept until twq_release_cache():
 *   after a cudaDeviceReset, call twq_release_cache() before the next call.
 *   Sharing: every call uses the same array, which keeps the last call's
 *   contents. No part of it needs to start at zero (each call writes every
 *   scratch byte before reading it), but calls that overlap on the GPU (two
 *   streams, or two host threads) race on it: serialize them.
 *   Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 */
TWQ_API twq_status twq_unfused_linear_noalloc(const uint8_t* xq, const float* sx, int64_t b,
                                              const twq_weights* w, uint16_t* y,
                                              twq_stream_t stream);

/*
 * Offline fold of the learned transforms into the layer's factors (TwinQuant
 * §4.1, Eq. (6) and the factors after it: U' = Q^-1 U G, V' = G^-1 V,
 * R' = Q^-1 R, absorbed offline). The layer then runs on X' = X Q with
 * L1 = U', L2 = V', R = R' (twq_pack_weights). Not on the per-token path.
 *   Q   m x m fp32 row-major, orthogonal (§4.2: Q^T Q = I), so Q^-1 = Q^T
 *   G   r x r fp32 row-major, invertible; inverted on the device by Gauss-Jordan
 *       elimination with partial pivoting in fp64
 *   U   m x r, V r x n, R m x n: BF16 row-major (the decomposed factors)
 *   L1_out m x r, L2_out r x n, R_out m x n: BF16 row-major outputs (RNE of
 *       products accumulated in fp32)
 *   workspace: device buffer of twq_fold_workspace_bytes(m, n, r) bytes,
 *       256-byte aligned
 * Limits: r <= 1024, m <= 4,194,240. This call SYNCHRONIZES `stream` (it reads
 * back whether G was singular): TWQ_ERR_INVALID_ARG if a pivot column of G
 * has no nonzero entry (the outputs are then unspecified).
 */
TWQ_API size_t twq_fold_workspace_bytes(int64_t m, int64_t n, int64_t r);
TWQ_API twq_status twq_fold_transforms(const float* Q, const float* G, const uint16_t* U,
                                       const uint16_t* V, const uint16_t* R, int64_t m, int64_t n,
                                       int64_t r, uint16_t* L1_out, uint16_t* L2_out,
                                       uint16_t* R_out, void* workspace, size_t workspace_bytes,
                                       twq_stream_t stream);

/*
 * Reads and clears the device-side status word (SYNCHRONIZES the device).
 * *code = 0 if no kernel's bounded wait has run out since the last call, else
 * a site code (which wait gave up). Returns TWQ_ERR_DEVICE if *code != 0.
 */
TWQ_API twq_status twq_device_status(int* code);

/*
 * Self-test of the kernels' bounded waits (the pages have no counterpart: this
 * checks the library's failure path without a GPU fault). Launches the prefill
 * layer kernel on the given W4A4 problem with its X copies withheld and every
 * wait limited to wait_limit_ns (1 us .. 1 s), so that the waits on X run out:
 * the kernel records the site of the first wait that gave up, its CTAs let their
 * copies in flight land, complete their MMAs, free their tensor memory and leave.
 * The launch itself succeeds; twq_device_status() then reports a nonzero site
 * code (41..52) and clears it, and later calls on the stream run normally. y is
 * left unspecified.
 *   xq, sx, b, w, y  as twq_w4a4_only, with b > 16, w->m >= 256, w->n % 256 == 0
 *   (TWQ_ERR_UNSUPPORTED otherwise: the prefill kernel does not take the shape).
 */
TWQ_API twq_status twq_selftest_wait_timeout(const uint8_t* xq, const float* sx, int64_t b,
                                             const twq_weights* w, uint16_t* y,
                                             int64_t wait_limit_ns, twq_stream_t stream);

/*
 * Drops the library's host-side caches: the encoded TMA tensor maps of the
 * decode path (a direct-mapped table of 256 entries keyed by base pointer,
 * shape, stride and box; an entry only encodes an address and a shape, so a hit
 * is always exact and the table never needs clearing for correctness) and the
 * resolved device addresses of twq_unfused_linear_noalloc's scratch array.
 * After a cudaDeviceReset in the caller's process, call this before the next
 * call into the library: the reset ends the context that the cached scratch
 * address belonged to. Host only; launches nothing; safe to call at any time
 * from any thread (calls in flight on other threads keep the entries they
 * already read).
 */
TWQ_API void twq_release_cache(void);

/* Number of kernels each entry point launches (for launch accounting). */
TWQ_API int twq_launches_per_call(const char* entry_point);

#ifdef __cplusplus
}
#endif

#endif /* TWQ_H_ */
