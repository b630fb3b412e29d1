/*
 * paro.h -- C ABI of the ParoQuant runtime hot path on NVIDIA B200 (sm_100a).
 *
 * The path (page "ParoQuant: pairwise rotations that survive deployment"):
 *   section "A rotation small enough to execute": each stage rotates disjoint
 *   channel pairs (i, j) by a Givens angle,
 *       x_i' = cos(t) x_i + sin(t) x_j,   x_j' = -sin(t) x_i + cos(t) x_j,
 *   K stages are composed and a channel-wise scale follows them; the weight
 *   transform is folded in and quantised at build time, and the activation
 *   transform x~ = diag(1/s) R_K ... R_1 x runs right before the INT4 linear;
 *   section "My reduced-calibration experiment": INT4 weights, group size 128;
 *   section "From fake quantization to a real TensorRT engine": one rotation
 *   operator and one group-wise INT4 GEMM operator per linear layer, built
 *   from weights that were transformed and packed beforehand.
 *
 * Conventions shared by every call:
 *   - Pointers named d_* are DEVICE pointers owned by the caller; the library
 *     never frees or retains them.  h_* pointers are host pointers.
 *   - bf16 and fp16 buffers are passed as uint16_t bit patterns.
 *   - Matrices are dense row-major with no padding.
 *   - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream).  Asynchronous device faults surface at the
 *     caller's next synchronisation.
 *   - Arguments are validated on the host before anything is enqueued; an
 *     invalid call enqueues nothing and returns PARO_ERR_INVALID_ARG (bad
 *     value, null or misaligned pointer) or PARO_ERR_UNSUPPORTED (a valid
 *     value outside what the kernels implement).  A failed launch returns
 *     PARO_ERR_CUDA.  paro_last_error() describes the last failure of the
 *     calling thread.
 *   - Pair tables: uint16_t pairs[K][d/2][2]; stage k = 0 (R_1) is applied
 *     first; each stage must be a set of disjoint pairs covering channels
 *     0..d-1 (a perfect matching).  Kernels check that every index is < d; an
 *     out-of-range index never addresses memory (its pair is skipped, or the
 *     index is clamped into range) and is reported through
 *     paro_get_device_status(), and that call's results are void.  Repeated
 *     channels inside a stage are not detected and give unspecified (but
 *     in-bounds) results.
 *   - cos_t[K][d/2], sin_t[K][d/2] (fp32) hold cos and sin of each pair's
 *     angle; scale[d] (fp32, > 0) is the channel scale s, NULL meaning s = 1.
 *   - Packed weights (layout version 1): qweight uint32 [d_out][d_in/8], the
 *     4-bit code of input column 8w+e in bits [4e, 4e+4) of word w;
 *     scales, zeros fp16 [d_out][d_in/128]; the zero point is an integer
 *     0..15 stored in fp16; the weight is w^ = (q - zero) * scale.
 *   - Supported sizes: d (= d_in for the rotation) even, 2 <= d <= 49152;
 *     d_in % 128 == 0 and group_size == 128 for the INT4 calls; d_out % 16 == 0;
 *     0 <= K <= 16; M >= 0 (M == 0 enqueues nothing and returns PARO_OK).
 *   - No exception crosses this boundary.  Calls are thread-safe; the only
 *     library state is one device status word per GPU and the scratch array of
 *     paro_rotate_w4_linear_noalloc.
 */
#ifndef PARO_H
#define PARO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define PARO_API __attribute__((visibility("default")))
#else
#define PARO_API
#endif

struct CUstream_st;
typedef struct CUstream_st* paro_stream_t; /* the same handle as cudaStream_t */

typedef enum {
  PARO_OK = 0,
  PARO_ERR_INVALID_ARG = 1,
  PARO_ERR_UNSUPPORTED = 2,
  PARO_ERR_CUDA = 3,
  PARO_ERR_TIMEOUT = 4,
  PARO_ERR_RANGE = 5
} paro_status;

/* Layout version of the packed weights described above. */
PARO_API int paro_weight_layout_version(void);

/* Static English name of a status code. */
PARO_API const char* paro_status_string(paro_status s);

/* Message of the last failed call on the calling thread ("" if none). */
PARO_API const char* paro_last_error(void);

/*
 * Build-time transform and packing ("transform and pack INT4 weights", page
 * "ParoQuant: pairwise rotations that survive deployment", section "From fake
 * quantization to a real TensorRT engine"; fold from section "A rotation small
 * enough to execute").
 *
 * For every output row n: w~_n = diag(s) R_K ... R_1 w_n (fp32 arithmetic),
 * so that W~ x~ = W x; then per group of 128 input columns, in fp32 IEEE
 * arithmetic with round-half-to-even:
 *   mn = min(0, min v), mx = max(0, max v), scale = fp16((mx - mn) / 15);
 *   scale == 0 -> scale = 1, zero = 0; else zero = clamp(rint(-mn / scale), 0, 15);
 *   q = clamp(rint(v / scale) + zero, 0, 15).
 * d_W:        fp32 [d_out][d_in], read only.
 * K, d_pairs, d_cos, d_sin, d_scale: the layer's transform (K == 0 and
 *             d_scale == NULL pack W itself: the plain INT4 linear).
 * d_workspace: fp32 [d_out][d_in] scratch for the folded weights; may be NULL
 *             when K == 0 and d_scale == NULL.  Must not alias d_W.
 * d_qweight, d_scales, d_zeros: outputs in layout version 1.
 */
PARO_API paro_status paro_pack_weights(const float* d_W, int d_out, int d_in, int group_size, int K,
                              const uint16_t* d_pairs, const float* d_cos, const float* d_sin,
                              const float* d_scale, float* d_workspace, uint32_t* d_qweight,
                              uint16_t* d_scales, uint16_t* d_zeros, paro_stream_t stream);

/*
 * Activation-side transform x~ = diag(1/s) R_K ... R_1 x, per token row (page
 * "ParoQuant: pairwise rotations that survive deployment", section "A
 * rotation small enough to execute").  fp32 arithmetic, bf16 in and out
 * (round to nearest even).
 * d_x:     bf16 [M][d].    d_x_rot: bf16 [M][d]; may equal d_x (in place).
 */
PARO_API paro_status paro_rotate(const uint16_t* d_x, uint16_t* d_x_rot, int M, int d, int K,
                        const uint16_t* d_pairs, const float* d_cos, const float* d_sin,
                        const float* d_scale, paro_stream_t stream);

/*
 * Gradients of the activation-side transform x~ = diag(1/s) R_K ... R_1 x for
 * an upstream gradient G = dL/dx~ (page "ParoQuant: Pairwise Rotation
 * Quantization for Efficient Reasoning LLM Inference", abstract: the Givens
 * rotations and the channel-wise scaling are optimizable; the pages print no
 * backward pass, and this is the chain rule of the forward transform):
 *   dx = dL/dx,  dtheta[k][p] = dL/dtheta of pair p of stage k,  dscale = dL/ds,
 * with (c, s) = (cos, sin) of the angle and x', h the stage's output and its
 * gradient: dtheta = sum over tokens of (h_i x_j' - h_j x_i'); the stage's
 * input gradient is the transposed rotation of h; dscale_c = -sum G_c x~_c / s_c.
 * fp32 arithmetic.  d_x: bf16 [M][d] (the forward input); d_grad: fp32 [M][d];
 * d_dx: fp32 [M][d]; d_dtheta: fp32 [K][d/2] (may be NULL when K == 0);
 * d_dscale: fp32 [d], required when d_scale is given (else ignored).  The
 * stage inputs are recovered from the outputs by the inverse rotation, so
 * nothing is stored per stage; the per-block partial sums of dtheta and
 * dscale go to d_workspace (paro_rotate_backward_workspace_bytes(M, d, K,
 * d_scale != NULL) bytes, 16-byte aligned, caller-owned) and are added in a
 * fixed order, so repeated calls give identical bits.  Needs d <= 28672
 * (PARO_ERR_UNSUPPORTED beyond); pair indices >= d are skipped and reported
 * through paro_get_device_status().
 */
PARO_API size_t paro_rotate_backward_workspace_bytes(int M, int d, int K, int with_scale);
PARO_API paro_status paro_rotate_backward(const uint16_t* d_x, const float* d_grad, int M, int d, int K,
                                          const uint16_t* d_pairs, const float* d_cos, const float* d_sin,
                                          const float* d_scale, float* d_dx, float* d_dtheta, float* d_dscale,
                                          void* d_workspace, size_t workspace_bytes, paro_stream_t stream);

/*
 * The dense learned rotation that the pairwise transform is contrasted with
 * (page "ParoQuant: pairwise rotations that survive deployment", section "Why
 * it differs from a dense learned rotation": a dense rotation puts a large
 * matrix multiply in front of every INT4 GEMM): x~ = x Q^T for a bf16 d x d
 * matrix Q, i.e. x~[m][n] = sum_k Q[n][k] x[m][k], on the tensor cores (bf16
 * operands, fp32 accumulation, bf16 out, round to nearest even).  It exists to
 * measure that cost against the pairwise transform on the same INT4 linears;
 * the result feeds paro_w4_linear like any transformed activation.
 * d_x: bf16 [M][d]; d_q: bf16 [d][d] row-major; d_out: bf16 [M][d], not
 * overlapping d_x or d_q.  Needs d a multiple of 64 (PARO_ERR_UNSUPPORTED
 * otherwise) and 16-byte aligned pointers.
 */
PARO_API paro_status paro_dense_rotate(const uint16_t* d_x, const uint16_t* d_q, uint16_t* d_out, int M, int d,
                                       paro_stream_t stream);

/*
 * Group-wise INT4 weight-only linear y = x W^T with w^ = (q - zero) * scale
 * (page "ParoQuant: pairwise rotations that survive deployment", section
 * "From fake quantization to a real TensorRT engine": the group-wise INT4 GEMM
 * operator).  fp32 accumulation, bf16 output (round to nearest even).
 * d_x: bf16 [M][d_in] (already transformed); d_y: bf16 [M][d_out]; d_y must not
 * overlap any input.
 */
PARO_API paro_status paro_w4_linear(const uint16_t* d_x, const uint32_t* d_qweight, const uint16_t* d_scales,
                           const uint16_t* d_zeros, uint16_t* d_y, int M, int d_in, int d_out,
                           int group_size, paro_stream_t stream);

/*
 * Weight-activation (W4A4) variant (page "ParoQuant: Pairwise Rotation
 * Quantization for Efficient Reasoning LLM Inference", section "Abstract
 * (arXiv)": the method also matches weight-activation quantization methods).
 * The pages give no detail of that setting; these calls take 4-bit weights
 * (the packed INT4 weights of the weight-only calls, unchanged) and 4-bit
 * activations: the transformed activations quantised per token, symmetrically,
 * to codes in -8..7.
 *
 * paro_quantize_activations: s_x[m] = max_k |x[m][k]| / 7 (1 for an all-zero
 * row) and q[m][k] = clamp(rint(x[m][k] / s_x[m]), -8, 7), in fp32 IEEE
 * arithmetic with ties to even.  d_x: bf16 [M][d], 16-byte aligned, d % 8 == 0;
 * d_q: int8 [M][d], one code per byte in column order; d_sx: fp32 [M].  The
 * outputs must not overlap d_x.
 */
PARO_API paro_status paro_quantize_activations(const uint16_t* d_x, int8_t* d_q, float* d_sx, int M, int d,
                                               paro_stream_t stream);

/*
 * Bytes of device workspace the W4A4 calls take: fp32 partial sums of the
 * linear (0 when it needs none), and with with_transform != 0 before them the
 * bf16 transformed activations, their codes and their scales of
 * paro_rotate_w4a4_linear (each part rounded up to 256 bytes).
 */
PARO_API size_t paro_w4a4_workspace_bytes(int M, int d_in, int d_out, int with_transform);

/*
 * W4A4 linear: y[m][n] = s_x[m] * sum_g s_w[n][g] * sum_{k in g}
 * (q_w[n][k] - z[n][g]) * q_x[m][k], the inner sums exact integers, the rest
 * fp32, bf16 output (round to nearest even).  d_q: int8 [M][d_in] codes in
 * -8..7, 16-byte aligned; d_sx: fp32 [M]; weights as paro_w4_linear; d_y: bf16
 * [M][d_out], overlapping no input.  d_workspace: paro_w4a4_workspace_bytes(M,
 * d_in, d_out, 0) bytes, 256-byte aligned (may be null when that is 0).
 */
PARO_API paro_status paro_w4a4_linear(const int8_t* d_q, const float* d_sx, const uint32_t* d_qweight,
                                      const uint16_t* d_scales, const uint16_t* d_zeros, uint16_t* d_y, int M,
                                      int d_in, int d_out, int group_size, void* d_workspace,
                                      size_t workspace_bytes, paro_stream_t stream);

/*
 * The whole W4A4 path of one linear: the activation transform (as
 * paro_rotate, bf16 x~ into the workspace), its per-token codes (as
 * paro_quantize_activations) and the W4A4 linear, three launches on `stream`.
 * Arguments as paro_rotate_w4_linear; d_workspace: paro_w4a4_workspace_bytes(M,
 * d_in, d_out, 1) bytes, 256-byte aligned, overlapping nothing else.
 */
PARO_API paro_status paro_rotate_w4a4_linear(const uint16_t* d_x, int K, const uint16_t* d_pairs,
                                             const float* d_cos, const float* d_sin, const float* d_scale,
                                             const uint32_t* d_qweight, const uint16_t* d_scales,
                                             const uint16_t* d_zeros, uint16_t* d_y, int M, int d_in, int d_out,
                                             int group_size, void* d_workspace, size_t workspace_bytes,
                                             paro_stream_t stream);

/*
 * Host-side, once per layer (no GPU involved): reorders the pairs inside every
 * stage, flipping some (i, j, cos, sin) into the same rotation (j, i, cos, -sin),
 * so that every aligned group of 32 consecutive pairs touches 32 different
 * shared-memory banks with its i channels and 32 with its j channels.  The
 * output tables describe exactly the same transform (the pairs of a stage are
 * disjoint, page "ParoQuant: pairwise rotations that survive deployment",
 * section "A rotation small enough to execute"), so they may replace the input
 * tables in every call, including paro_pack_weights; the transform kernels then
 * run without shared-memory bank conflicts on the rows.  Results can differ
 * from the unplanned tables by fp32 rounding only.
 * h_pairs [K][d/2][2], h_cos/h_sin [K][d/2]: host input; *_out: host output of
 * the same shapes, not overlapping the input.  Needs d % 64 == 0
 * (PARO_ERR_UNSUPPORTED otherwise: keep the original tables); every stage must
 * be a perfect matching of 0..d-1 (PARO_ERR_INVALID_ARG otherwise).
 */
PARO_API paro_status paro_plan_pair_order(const uint16_t* h_pairs, const float* h_cos, const float* h_sin, int K,
                                          int d, uint16_t* h_pairs_out, float* h_cos_out, float* h_sin_out);

/*
 * Bytes of device workspace paro_rotate_w4_linear takes for M tokens of width
 * d_in: the fp16 transformed activations (2 M d_in rounded up to 256 bytes)
 * and, for M <= 16, the partial tiles and flags of the stream-K INT4 kernel
 * (about 16.4 KB per SM at 9-16 tokens, half that up to 8).
 */
PARO_API size_t paro_workspace_bytes(int M, int d_in);

/*
 * The runtime path of one linear layer: the activation transform run right
 * before the packed INT4 linear (page "ParoQuant: pairwise rotations that
 * survive deployment", section "A rotation small enough to execute", last
 * paragraph).  y = (diag(1/s) R_K ... R_1 x) W~^T.  The transformed
 * activations never leave the GPU as bf16: they are handed to the linear in
 * fp16 through d_workspace (paro_workspace_bytes(M, d_in) bytes, 256-byte
 * aligned, caller-owned; zero before its first use, as for
 * paro_rotate_w4_linear_batched, after which the calls keep it valid; two
 * calls that run at the same time need two workspaces).  Up to 16 tokens with that full
 * workspace the call runs as paro_rotate_w4_linear_batched does for one
 * linear (one launch at one token: its first CTA transforms while the others
 * stream the weights); given only the activations' 2 M d_in bytes (rounded
 * up to 256), it runs the transform and then the INT4 linear.
 * d_x: bf16 [M][d_in]; d_y: bf16 [M][d_out], not overlapping any input.
 */
PARO_API paro_status paro_rotate_w4_linear(const uint16_t* d_x, int K, const uint16_t* d_pairs,
                                  const float* d_cos, const float* d_sin, const float* d_scale,
                                  const uint32_t* d_qweight, const uint16_t* d_scales,
                                  const uint16_t* d_zeros, uint16_t* d_y, int M, int d_in, int d_out,
                                  int group_size, void* d_workspace, size_t workspace_bytes,
                                  paro_stream_t stream);

/*
 * One linear layer of a batch for paro_rotate_w4_linear_batched: the same
 * arguments as paro_rotate_w4_linear, gathered in a host-side struct.
 */
typedef struct {
  const uint16_t* d_x;        /* bf16 [M][d_in] */
  uint16_t* d_y;              /* bf16 [M][d_out], overlapping no input of the batch */
  int M, d_in, d_out, K;
  const uint16_t* d_pairs;    /* [K][d_in/2][2] */
  const float* d_cos;         /* [K][d_in/2] */
  const float* d_sin;         /* [K][d_in/2] */
  const float* d_scale;       /* [d_in] or NULL */
  const uint32_t* d_qweight;  /* [d_out][d_in/8], layout version 1 */
  const uint16_t* d_scales;   /* fp16 [d_out][d_in/128] */
  const uint16_t* d_zeros;    /* fp16 [d_out][d_in/128] */
} paro_linear;

/* Largest number of linears one paro_rotate_w4_linear_batched call takes. */
#define PARO_MAX_BATCH 8

/*
 * Workspace bytes paro_rotate_w4_linear_batched uses for these linears: the
 * transformed activations of every linear (paro_workspace_bytes(M, d_in)
 * each, in order), then, when every M is at most 16, the partial sums of
 * the stream-K INT4 linear (2 partial 64-row tiles per CTA, every fp32 value
 * in a 64-bit word beside a launch tag), the flags of the transform's CTAs
 * (at most 128) that the INT4 linear waits on, and the workspace's launch
 * epoch (see below).
 * The second part is optional: given only the first, the call runs the older
 * per-block kernel.
 */
PARO_API size_t paro_batched_workspace_bytes(const paro_linear* h_layers, int count);

/*
 * Runs paro_rotate_w4_linear for up to PARO_MAX_BATCH independent linears,
 * e.g. the seven linears of one decoder layer, with one transform launch and
 * one INT4-linear launch up to 64 tokens (one launch in all at one token per
 * linear; one transform launch per linear beyond 64); each linear has its own
 * transform ("one rotation operator plus one group-wise INT4 GEMM operator for
 * each layer", page "ParoQuant: pairwise rotations that survive deployment",
 * section "From fake quantization to a real TensorRT engine").  h_layers is a
 * HOST array read during the call; d_workspace holds
 * paro_batched_workspace_bytes(h_layers, count) bytes (256-byte aligned,
 * caller-owned; zero before its first use, e.g. by cudaMemsetAsync, after
 * which the calls keep it valid: they leave it holding their own state, which
 * later calls rely on, so it must not be written by anything else between
 * calls).  Results equal count separate calls
 * of paro_rotate_w4_linear.  Every linear is validated before anything is
 * enqueued; the message of paro_last_error() names the failing index.  When no
 * linear has a transform (K == 0 and d_scale == NULL for all) and every M is
 * at most 64, only the INT4-linear launch runs, on the bf16 inputs, and
 * d_workspace may be NULL; with more tokens, one tensor-core launch rounds
 * the bf16 inputs to fp16 itself when every linear has at least 128 tokens,
 * else the inputs are first rounded to fp16 into the workspace, as the
 * transform does.  With many tokens the INT4 linears of all layers run as one
 * persistent tensor-core launch after the transforms.  When every linear has
 * one token (M == 1) and the full workspace is given, the call is one launch:
 * its first CTAs transform one linear each into the workspace and publish a
 * flag, and the INT4 CTAs request a linear's activations once its flag is set
 * (each linear's arithmetic waits for its own transform only).  With 2 to 16
 * tokens the transform launch's CTAs each publish such a flag, and the INT4
 * launch after it requests a linear's activations once all of that linear's
 * transform CTAs have published, not when the whole transform launch is done.
 * Every flag a launch publishes (the transforms' "x~ is written" flags)
 * holds 2E + 1 for the workspace's launch epoch E, which every CTA reads once
 * the previous kernel has completed and which the launch's last CTA advances,
 * and every value of a partial tile carries the low 32 bits of 2E + 1: a flag
 * or a value left by an earlier call, or by an earlier replay of the same
 * CUDA graph, is not taken for this launch's (a partial value left exactly a
 * multiple of 2^31 launches earlier on the same workspace, and not rewritten
 * since, would be), and calls captured in a graph may be replayed with new
 * inputs.  Two calls that may run at the same time need two workspaces.
 */
PARO_API paro_status paro_rotate_w4_linear_batched(const paro_linear* h_layers, int count, int group_size,
                                                  void* d_workspace, size_t workspace_bytes,
                                                  paro_stream_t stream);

/* Bytes of the scratch array built into the library for the call below. */
#define PARO_NOALLOC_SCRATCH_BYTES (4u << 20)

/*
 * The same computation as paro_rotate_w4_linear for callers that cannot
 * allocate device memory (the paper has no counterpart: this is an interface
 * convenience of this library).  Instead of a caller-provided workspace, the
 * call uses a scratch array built into the library: every GPU that loads
 * libparo holds PARO_NOALLOC_SCRATCH_BYTES (4 MiB) for it until the process
 * exits.  M * d_in may not exceed 262144 (PARO_ERR_UNSUPPORTED, nothing
 * enqueued).  The call allocates nothing and runs the same kernels as
 * paro_rotate_w4_linear given a workspace of PARO_NOALLOC_SCRATCH_BYTES, so
 * its results are bit-identical to that call's.  Its first call on a device
 * looks up the array's device address (cudaGetSymbolAddress) with that device
 * current and keeps it for the life of the process; make that first call
 * before any stream capture, and do not call cudaDeviceReset on that device
 * afterwards (the kept address would no longer be mapped).  All calls on a
 * device share the one array: calls that may overlap on the GPU (different
 * streams, or other work between them that is not ordered) race on it and
 * must be serialised by the caller.  Arguments, layouts and results are those
 * of paro_rotate_w4_linear.
 */
PARO_API paro_status paro_rotate_w4_linear_noalloc(const uint16_t* d_x, int K, const uint16_t* d_pairs,
                                  const float* d_cos, const float* d_sin, const float* d_scale,
                                  const uint32_t* d_qweight, const uint16_t* d_scales,
                                  const uint16_t* d_zeros, uint16_t* d_y, int M, int d_in, int d_out,
                                  int group_size, paro_stream_t stream);

/*
 * Synchronises `stream`, then returns and clears the device status word of
 * the current GPU (the first error a kernel met since the last read):
 * PARO_OK; PARO_ERR_INVALID_ARG (a kernel met a pair index >= d and skipped or
 * clamped it); PARO_ERR_TIMEOUT (a bounded wait gave up: a tensor-memory copy
 * or a hand-over flag between the transform and the INT4 linear did not come
 * within its limit; the CTAs that waited wrote none of their output tiles);
 * PARO_ERR_RANGE (a transformed activation handed to the INT4 linear in fp16
 * was beyond the fp16 range, |x~| >= 65520, and became infinite).  After any
 * of them that call's results are void.  The word's device address is looked
 * up on the first call of the library on each device and kept for the life
 * of the process, so cudaDeviceReset on a device after the library has used
 * it is not supported.
 */
PARO_API paro_status paro_get_device_status(paro_stream_t stream);

/*
 * Test hooks for the failure paths (no counterpart in the pages): they change
 * how later launches are configured and stay set until called again.
 * flag_wait_cycles > 0 bounds every wait of the decode INT4 kernel for a
 * hand-over flag (the transform's "x~ is written" flags, and the partial
 * sums of a tile split between CTAs) to about that many SM clock cycles
 * instead of about 2^31 (a second); 0 restores the default.
 * skip_ready_flags != 0 makes the decode transforms (in the fused one-token
 * launch and in the transform launch before the INT4 launch at 2-16 tokens)
 * skip publishing their "x~ is written" flags, so that the INT4 kernel's
 * waits run out: the call then reports PARO_ERR_TIMEOUT through
 * paro_get_device_status() and writes none of the output tiles of the linears
 * it waited for.  Nothing hangs: every wait is bounded.  Not thread-safe with
 * respect to calls being configured at the same time; PARO_ERR_INVALID_ARG
 * for a negative cycle count.
 */
PARO_API paro_status paro_set_test_hooks(long long flag_wait_cycles, int skip_ready_flags);

#ifdef __cplusplus
}
#endif

#endif /* PARO_H */
