// Host side of the C ABI declared in include/paro.h: argument validation,
// dispatch to the kernels, the per-device status word and error strings.
// Every check runs before anything is enqueued, so an invalid call leaves the
// stream untouched.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "paro_internal.cuh"
#include "w4_gemv.cuh"
#include "rotate_decode.cuh"
#include "w4_tc.cuh"
#include "w4_stream.cuh"

namespace {

__device__ int g_paro_status;  // first error met by a kernel on this device (0 = none)

thread_local char t_last_error[512];

paro_status fail(paro_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
  va_end(ap);
  return s;
}

paro_status ok() {
  t_last_error[0] = '\0';
  return PARO_OK;
}

paro_status from_cuda(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return ok();
  return fail(PARO_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr int kMaxDevices = 64;
std::atomic<int*> g_status_addr[kMaxDevices];

// Device address of the status word on the current device (looked up once per device).
int* status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  int* p = g_status_addr[dev].load(std::memory_order_acquire);
  if (!p) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_paro_status) != cudaSuccess) return nullptr;
    p = static_cast<int*>(a);
    g_status_addr[dev].store(p, std::memory_order_release);
  }
  return p;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return na && nb && x < y + nb && y < x + na;
}

paro_status check_tables(int K, int d, const uint16_t* pairs, const float* c, const float* s,
                         const float* scale) {
  if (K < 0) return fail(PARO_ERR_INVALID_ARG, "K = %d is negative", K);
  if (K > paro::kMaxStages) return fail(PARO_ERR_UNSUPPORTED, "K = %d exceeds %d stages", K, paro::kMaxStages);
  if (K > 0) {
    if (!pairs || !c || !s) return fail(PARO_ERR_INVALID_ARG, "K > 0 needs pair, cos and sin tables");
    if (!aligned(pairs, 4) || !aligned(c, 4) || !aligned(s, 4))
      return fail(PARO_ERR_INVALID_ARG, "pair/cos/sin tables must be 4-byte aligned");
  }
  if (scale && !aligned(scale, 4)) return fail(PARO_ERR_INVALID_ARG, "scale must be 4-byte aligned");
  (void)d;
  return PARO_OK;
}

paro_status check_width(int d) {
  if (d < 2 || (d & 1)) return fail(PARO_ERR_INVALID_ARG, "d = %d must be even and >= 2", d);
  if (d > paro::kMaxDim) return fail(PARO_ERR_UNSUPPORTED, "d = %d exceeds %d", d, paro::kMaxDim);
  return PARO_OK;
}

paro_status check_linear_shape(int M, int d_in, int d_out, int group_size) {
  if (M < 0) return fail(PARO_ERR_INVALID_ARG, "M = %d is negative", M);
  if (group_size <= 0) return fail(PARO_ERR_INVALID_ARG, "group_size = %d", group_size);
  if (group_size != paro::kGroup) return fail(PARO_ERR_UNSUPPORTED, "group_size = %d (only 128)", group_size);
  if (d_in <= 0 || d_in % paro::kGroup)
    return fail(PARO_ERR_INVALID_ARG, "d_in = %d must be a positive multiple of 128", d_in);
  if (d_out <= 0 || d_out % 16)
    return fail(d_out <= 0 ? PARO_ERR_INVALID_ARG : PARO_ERR_UNSUPPORTED,
                "d_out = %d must be a positive multiple of 16", d_out);
  return PARO_OK;
}

paro_status check_weights(const uint32_t* qweight, const uint16_t* scales, const uint16_t* zeros) {
  if (!qweight || !scales || !zeros) return fail(PARO_ERR_INVALID_ARG, "null weight pointer");
  if (!aligned(qweight, 16)) return fail(PARO_ERR_INVALID_ARG, "qweight must be 16-byte aligned");
  if (!aligned(scales, 2) || !aligned(zeros, 2))
    return fail(PARO_ERR_INVALID_ARG, "scales/zeros must be 2-byte aligned");
  return PARO_OK;
}

// Token count from which the tensor-core (tcgen05) kernel takes over.
constexpr int kTensorCoreMinM = 128;

// The INT4 linear on x (bf16, or fp16 when x_f16).  With pdl_wait the kernel is
// launched as a programmatic dependent of the previous kernel in the stream and
// waits for it before reading x or writing y (the weights may be read earlier,
// so only a previous kernel that does not write them may trigger early: in this
// library the INT4 and transform kernels trigger, the weight packing does not).
cudaError_t launch_linear(const uint16_t* x, bool x_f16, const uint32_t* qweight, const uint16_t* scales,
                          const uint16_t* zeros, uint16_t* y, int M, int d_in, int d_out, cudaStream_t s,
                          bool pdl_wait, int* status) {
  if (M >= kTensorCoreMinM && status && paro::tc_supported(M, d_in, d_out, x))
    return paro::launch_w4_tc(x, x_f16, qweight, reinterpret_cast<const __half*>(scales),
                              reinterpret_cast<const __half*>(zeros), reinterpret_cast<__nv_bfloat16*>(y), M, d_in,
                              d_out, status, s);
  if (M <= paro::kStreamMaxM && paro::stream_supported(M, d_in, d_out, x, qweight)) {
    // few tokens: the TMA stream-K kernel, each CTA on whole 64-row tiles so
    // that no partial sum crosses CTAs (this call has no workspace for them)
    const uint16_t* xs[1] = {x};
    const uint32_t* qs[1] = {qweight};
    const __half* ss[1] = {reinterpret_cast<const __half*>(scales)};
    const __half* zs[1] = {reinterpret_cast<const __half*>(zeros)};
    __nv_bfloat16* ys[1] = {reinterpret_cast<__nv_bfloat16*>(y)};
    paro::StreamBatch sb;
    int nt = 1;
    cudaError_t e = paro::plan_stream_batch(xs, qs, ss, zs, ys, &M, &d_in, &d_out, 1, x_f16, nullptr, &sb, &nt);
    if (e != cudaSuccess) return e;
    return paro::launch_stream_batch(sb, nt, x_f16, status, s, pdl_wait);
  }
  paro::GemvProblem p = {};
  p.x = x;
  p.qw = qweight;
  p.sc = reinterpret_cast<const __half*>(scales);
  p.z = reinterpret_cast<const __half*>(zeros);
  p.y = reinterpret_cast<__nv_bfloat16*>(y);
  p.M = M;
  p.d_in = d_in;
  p.d_out = d_out;
  paro::GemvBatch b;
  int nt = 1;
  cudaError_t e = paro::plan_gemv_batch(&p, 1, x_f16, &b, &nt);
  if (e != cudaSuccess) return e;
  return paro::launch_gemv_batch(b, nt, s, pdl_wait);
}

// Prefixes the current error message with the index of the failing layer.
paro_status prefix_error(paro_status st, int layer) {
  char msg[sizeof(t_last_error)];
  snprintf(msg, sizeof(msg), "%s", t_last_error);
  return fail(st, "layer %d: %s", layer, msg);
}

// Activation transform of one linear: the table-prefetching decode kernel for
// few rows, the row-block kernel otherwise.
cudaError_t launch_transform(const uint16_t* x, void* out, bool f16_out, int M, int d, int K,
                             const uint16_t* pairs, const float* c, const float* s, const float* scale,
                             int* status, cudaStream_t stream, bool pdl_trigger) {
  if (M <= 64 && (K == 0 || paro::rot_decode_supported(d, pairs, c, s))) {
    paro::RotProblem p = {};
    p.x = x;
    p.out = out;
    p.M = M;
    p.d = d;
    p.K = K;
    p.pairs = reinterpret_cast<const uint32_t*>(pairs);
    p.cos_t = c;
    p.sin_t = s;
    p.scale = scale;
    paro::RotBatch b;
    int R = 1;
    cudaError_t e = paro::plan_rot_batch(&p, 1, &b, &R);
    if (e != cudaSuccess) return e;
    return paro::launch_rot_batch(b, R, f16_out, status, stream, pdl_trigger);
  }
  return paro::launch_rotate_act(x, out, f16_out ? 1 : 0, M, d, K, pairs, c, s, scale, status, stream,
                                 pdl_trigger);
}

}  // namespace

namespace {
std::atomic<long long> g_hook_flag_wait{0};
std::atomic<int> g_hook_skip_flags{0};
}  // namespace

namespace paro {
long long hook_flag_wait() {
  const long long v = g_hook_flag_wait.load(std::memory_order_relaxed);
  return v > 0 ? v : kWaitCycles;
}
int hook_skip_ready_flags() { return g_hook_skip_flags.load(std::memory_order_relaxed); }

paro_status record_error(paro_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
  va_end(ap);
  return s;
}
}  // namespace paro

extern "C" {

int paro_weight_layout_version(void) { return 1; }

const char* paro_status_string(paro_status s) {
  switch (s) {
    case PARO_OK: return "PARO_OK";
    case PARO_ERR_INVALID_ARG: return "PARO_ERR_INVALID_ARG";
    case PARO_ERR_UNSUPPORTED: return "PARO_ERR_UNSUPPORTED";
    case PARO_ERR_CUDA: return "PARO_ERR_CUDA";
    case PARO_ERR_TIMEOUT: return "PARO_ERR_TIMEOUT";
    case PARO_ERR_RANGE: return "PARO_ERR_RANGE";
  }
  return "PARO_ERR_UNKNOWN";
}

const char* paro_last_error(void) { return t_last_error; }

paro_status paro_set_test_hooks(long long flag_wait_cycles, int skip_ready_flags) {
  if (flag_wait_cycles < 0) return fail(PARO_ERR_INVALID_ARG, "flag_wait_cycles = %lld is negative", flag_wait_cycles);
  g_hook_flag_wait.store(flag_wait_cycles, std::memory_order_relaxed);
  g_hook_skip_flags.store(skip_ready_flags != 0 ? 1 : 0, std::memory_order_relaxed);
  return ok();
}

paro_status paro_pack_weights(const float* d_W, int d_out, int d_in, int group_size, int K,
                              const uint16_t* d_pairs, const float* d_cos, const float* d_sin,
                              const float* d_scale, float* d_workspace, uint32_t* d_qweight,
                              uint16_t* d_scales, uint16_t* d_zeros, paro_stream_t stream) {
  paro_status st;
  if (d_out <= 0) return fail(PARO_ERR_INVALID_ARG, "d_out = %d must be positive", d_out);
  if (group_size <= 0) return fail(PARO_ERR_INVALID_ARG, "group_size = %d", group_size);
  if (group_size != paro::kGroup) return fail(PARO_ERR_UNSUPPORTED, "group_size = %d (only 128)", group_size);
  if (d_in <= 0 || d_in % paro::kGroup)
    return fail(PARO_ERR_INVALID_ARG, "d_in = %d must be a positive multiple of 128", d_in);
  if ((st = check_tables(K, d_in, d_pairs, d_cos, d_sin, d_scale)) != PARO_OK) return st;
  if (!d_W || !aligned(d_W, 16)) return fail(PARO_ERR_INVALID_ARG, "W must be non-null and 16-byte aligned");
  if ((st = check_weights(d_qweight, d_scales, d_zeros)) != PARO_OK) return st;
  const bool transform = K > 0 || d_scale != nullptr;
  const size_t wbytes = (size_t)d_out * d_in * sizeof(float);
  if (transform) {
    if ((st = check_width(d_in)) != PARO_OK) return st;
    if (!d_workspace || !aligned(d_workspace, 16))
      return fail(PARO_ERR_INVALID_ARG, "a transform needs a 16-byte aligned fp32 [d_out][d_in] workspace");
    if (overlap(d_workspace, wbytes, d_W, wbytes)) return fail(PARO_ERR_INVALID_ARG, "workspace overlaps W");
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const float* src = d_W;
  if (transform) {
    int* status = status_ptr();
    if (!status) return fail(PARO_ERR_CUDA, "no CUDA device / status word unavailable");
    cudaError_t e = paro::launch_fold_weights(d_W, d_workspace, d_out, d_in, K, d_pairs, d_cos, d_sin,
                                              d_scale, status, s);
    if (e != cudaSuccess) return from_cuda(e, "fold launch");
    src = d_workspace;
  }
  cudaError_t e = paro::launch_quantize_pack(src, d_out, d_in, d_qweight, reinterpret_cast<__half*>(d_scales),
                                             reinterpret_cast<__half*>(d_zeros), s);
  return from_cuda(e, "quantize/pack launch");
}

paro_status paro_rotate(const uint16_t* d_x, uint16_t* d_x_rot, int M, int d, int K,
                        const uint16_t* d_pairs, const float* d_cos, const float* d_sin,
                        const float* d_scale, paro_stream_t stream) {
  paro_status st;
  if (M < 0) return fail(PARO_ERR_INVALID_ARG, "M = %d is negative", M);
  if ((st = check_width(d)) != PARO_OK) return st;
  if ((st = check_tables(K, d, d_pairs, d_cos, d_sin, d_scale)) != PARO_OK) return st;
  if (M == 0) return ok();
  if (!d_x || !d_x_rot) return fail(PARO_ERR_INVALID_ARG, "null activation pointer");
  if (!aligned(d_x, 16) || !aligned(d_x_rot, 16)) return fail(PARO_ERR_INVALID_ARG, "x and x_rot must be 16-byte aligned");
  const size_t xb = (size_t)M * d * 2;
  if (d_x != d_x_rot && overlap(d_x, xb, d_x_rot, xb))
    return fail(PARO_ERR_INVALID_ARG, "x_rot partially overlaps x (only exact in-place is allowed)");
  int* status = status_ptr();
  if (!status) return fail(PARO_ERR_CUDA, "no CUDA device / status word unavailable");
  cudaError_t e = launch_transform(d_x, d_x_rot, false, M, d, K, d_pairs, d_cos, d_sin, d_scale, status,
                                   reinterpret_cast<cudaStream_t>(stream), false);
  return from_cuda(e, "rotate launch");
}

paro_status paro_dense_rotate(const uint16_t* d_x, const uint16_t* d_q, uint16_t* d_out, int M, int d,
                              paro_stream_t stream) {
  if (M < 0) return fail(PARO_ERR_INVALID_ARG, "M = %d is negative", M);
  if (d <= 0) return fail(PARO_ERR_INVALID_ARG, "d = %d must be positive", d);
  if (d % 64) return fail(PARO_ERR_UNSUPPORTED, "d = %d is not a multiple of 64", d);
  if (M == 0) return ok();
  if (!d_x || !d_q || !d_out) return fail(PARO_ERR_INVALID_ARG, "null pointer");
  if (!aligned(d_x, 16) || !aligned(d_q, 16) || !aligned(d_out, 16))
    return fail(PARO_ERR_INVALID_ARG, "x, Q and out must be 16-byte aligned");
  const size_t xb = (size_t)M * d * 2, qb = (size_t)d * d * 2;
  if (overlap(d_out, xb, d_x, xb) || overlap(d_out, xb, d_q, qb))
    return fail(PARO_ERR_INVALID_ARG, "out overlaps x or Q");
  int* status = status_ptr();
  if (!status) return fail(PARO_ERR_CUDA, "no CUDA device / status word unavailable");
  cudaError_t e = paro::launch_dense_tc(d_x, d_q, reinterpret_cast<__nv_bfloat16*>(d_out), M, d, status,
                                        reinterpret_cast<cudaStream_t>(stream));
  return from_cuda(e, "dense rotate launch");
}

size_t paro_rotate_backward_workspace_bytes(int M, int d, int K, int with_scale) {
  if (M <= 0 || d < 2 || (d & 1) || K < 0 || K > paro::kMaxStages) return 0;
  return paro::rot_bwd_workspace_bytes(M, d, K, with_scale != 0);
}

paro_status paro_rotate_backward(const uint16_t* d_x, const float* d_grad, int M, int d, int K,
                                 const uint16_t* d_pairs, const float* d_cos, const float* d_sin,
                                 const float* d_scale, float* d_dx, float* d_dtheta, float* d_dscale,
                                 void* d_workspace, size_t workspace_bytes, paro_stream_t stream) {
  paro_status st;
  if (M < 0) return fail(PARO_ERR_INVALID_ARG, "M = %d is negative", M);
  if ((st = check_width(d)) != PARO_OK) return st;
  if ((st = check_tables(K, d, d_pairs, d_cos, d_sin, d_scale)) != PARO_OK) return st;
  if (paro::rot_bwd_rows(d) == 0) return fail(PARO_ERR_UNSUPPORTED, "d = %d is too wide for the backward kernel", d);
  if (M == 0) return ok();
  if (!d_x || !d_grad || !d_dx) return fail(PARO_ERR_INVALID_ARG, "null x, grad or dx pointer");
  if (K > 0 && !d_dtheta) return fail(PARO_ERR_INVALID_ARG, "K > 0 needs a dtheta output");
  if (d_scale && !d_dscale) return fail(PARO_ERR_INVALID_ARG, "a scale needs a dscale output");
  if (!aligned(d_x, 4) || !aligned(d_grad, 4) || !aligned(d_dx, 4) || (d_dtheta && !aligned(d_dtheta, 4)) ||
      (d_dscale && !aligned(d_dscale, 4)))
    return fail(PARO_ERR_INVALID_ARG, "x, grad, dx, dtheta and dscale must be 4-byte aligned");
  const size_t need = paro::rot_bwd_workspace_bytes(M, d, K, d_scale != nullptr);
  if (need && (!d_workspace || workspace_bytes < need || !aligned(d_workspace, 16)))
    return fail(PARO_ERR_INVALID_ARG, "workspace must be 16-byte aligned and hold %zu bytes", need);
  const size_t gb = (size_t)M * d * 4;
  if (overlap(d_dx, gb, d_grad, gb) || overlap(d_dx, gb, d_x, (size_t)M * d * 2) ||
      (need && (overlap(d_workspace, need, d_dx, gb) || overlap(d_workspace, need, d_grad, gb))))
    return fail(PARO_ERR_INVALID_ARG, "dx or the workspace overlaps an input");
  int* status = status_ptr();
  if (!status) return fail(PARO_ERR_CUDA, "no CUDA device / status word unavailable");
  cudaError_t e = paro::launch_rot_backward(d_x, d_grad, M, d, K, reinterpret_cast<const uint32_t*>(d_pairs), d_cos,
                                            d_sin, d_scale, d_dx, d_dtheta, d_dscale, d_workspace, status,
                                            reinterpret_cast<cudaStream_t>(stream));
  return from_cuda(e, "rotate backward launch");
}

paro_status paro_w4_linear(const uint16_t* d_x, const uint32_t* d_qweight, const uint16_t* d_scales,
                           const uint16_t* d_zeros, uint16_t* d_y, int M, int d_in, int d_out,
                           int group_size, paro_stream_t stream) {
  paro_status st;
  if ((st = check_linear_shape(M, d_in, d_out, group_size)) != PARO_OK) return st;
  if (M == 0) return ok();
  if ((st = check_weights(d_qweight, d_scales, d_zeros)) != PARO_OK) return st;
  if (!d_x || !d_y) return fail(PARO_ERR_INVALID_ARG, "null activation pointer");
  if (!aligned(d_x, 16) || !aligned(d_y, 16)) return fail(PARO_ERR_INVALID_ARG, "x and y must be 16-byte aligned");
  const size_t yb = (size_t)M * d_out * 2;
  if (overlap(d_y, yb, d_x, (size_t)M * d_in * 2) || overlap(d_y, yb, d_qweight, (size_t)d_out * d_in / 2) ||
      overlap(d_y, yb, d_scales, (size_t)d_out * (d_in / 128) * 2) ||
      overlap(d_y, yb, d_zeros, (size_t)d_out * (d_in / 128) * 2))
    return fail(PARO_ERR_INVALID_ARG, "y overlaps an input");
  // a programmatic dependent of the previous kernel: only this library's INT4 and
  // transform kernels trigger early, and none of them writes weights
  cudaError_t e = launch_linear(d_x, false, d_qweight, d_scales, d_zeros, d_y, M, d_in, d_out,
                                reinterpret_cast<cudaStream_t>(stream), true, status_ptr());
  return from_cuda(e, "w4 linear launch");
}

namespace {
// fp16 transformed activations of M tokens of width d_in, rounded up to 256 bytes
size_t xt_bytes(int M, int d_in) {
  if (M <= 0 || d_in <= 0) return 0;
  const size_t b = (size_t)M * d_in * 2;
  return (b + 255) & ~(size_t)255;
}
}  // namespace

size_t paro_workspace_bytes(int M, int d_in) {
  if (M <= 0 || d_in <= 0) return 0;
  // up to 16 tokens, also the stream-K kernel's flags and partial tiles
  return xt_bytes(M, d_in) + (M <= paro::kStreamMaxM ? paro::stream_workspace_bytes(M) : 0);
}

paro_status paro_rotate_w4_linear(const uint16_t* d_x, int K, const uint16_t* d_pairs,
                                  const float* d_cos, const float* d_sin, const float* d_scale,
                                  const uint32_t* d_qweight, const uint16_t* d_scales,
                                  const uint16_t* d_zeros, uint16_t* d_y, int M, int d_in, int d_out,
                                  int group_size, void* d_workspace, size_t workspace_bytes,
                                  paro_stream_t stream) {
  paro_status st;
  if ((st = check_linear_shape(M, d_in, d_out, group_size)) != PARO_OK) return st;
  if ((st = check_width(d_in)) != PARO_OK) return st;
  if ((st = check_tables(K, d_in, d_pairs, d_cos, d_sin, d_scale)) != PARO_OK) return st;
  if (M == 0) return ok();
  if ((st = check_weights(d_qweight, d_scales, d_zeros)) != PARO_OK) return st;
  if (!d_x || !d_y) return fail(PARO_ERR_INVALID_ARG, "null activation pointer");
  if (!aligned(d_x, 16) || !aligned(d_y, 16)) return fail(PARO_ERR_INVALID_ARG, "x and y must be 16-byte aligned");
  // the transformed activations are required; up to 16 tokens, the stream-K
  // kernel's flags and partial tiles behind them are optional
  const size_t need = xt_bytes(M, d_in), full = paro_workspace_bytes(M, d_in);
  if (!d_workspace || workspace_bytes < need || !aligned(d_workspace, 256))
    return fail(PARO_ERR_INVALID_ARG, "workspace must be 256-byte aligned and hold %zu bytes", full);
  const size_t used = workspace_bytes < full ? need : full;
  const size_t yb = (size_t)M * d_out * 2;
  if (overlap(d_y, yb, d_x, (size_t)M * d_in * 2) || overlap(d_y, yb, d_workspace, used) ||
      overlap(d_workspace, used, d_x, (size_t)M * d_in * 2) ||
      overlap(d_y, yb, d_qweight, (size_t)d_out * d_in / 2))
    return fail(PARO_ERR_INVALID_ARG, "y, x and workspace must not overlap");
  int* status = status_ptr();
  if (!status) return fail(PARO_ERR_CUDA, "no CUDA device / status word unavailable");
  if (M <= paro::kStreamMaxM && used == full) {
    // few tokens with the full workspace: the batched call's decode forms for
    // this one linear (at one token a single launch whose first CTA runs the
    // transform while the others stream the weights)
    paro_linear L = {};
    L.d_x = d_x;
    L.d_y = d_y;
    L.M = M;
    L.d_in = d_in;
    L.d_out = d_out;
    L.K = K;
    L.d_pairs = d_pairs;
    L.d_cos = d_cos;
    L.d_sin = d_sin;
    L.d_scale = d_scale;
    L.d_qweight = d_qweight;
    L.d_scales = d_scales;
    L.d_zeros = d_zeros;
    return paro_rotate_w4_linear_batched(&L, 1, group_size, d_workspace, full, stream);
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_transform(d_x, d_workspace, true, M, d_in, K, d_pairs, d_cos, d_sin, d_scale, status, s,
                                   true);
  if (e != cudaSuccess) return from_cuda(e, "rotate launch");
  e = launch_linear(static_cast<const uint16_t*>(d_workspace), true, d_qweight, d_scales, d_zeros, d_y, M, d_in,
                    d_out, s, true, status);
  return from_cuda(e, "w4 linear launch");
}

namespace {
// Bytes of the stream-K kernel's publication flags and partial tiles for these
// linears (0 when some linear has more tokens than that kernel takes).
size_t batched_stream_bytes(const paro_linear* h_layers, int count) {
  int max_m = 0;
  for (int i = 0; i < count; ++i)
    if (h_layers[i].M > max_m) max_m = h_layers[i].M;
  if (max_m < 1 || max_m > paro::kStreamMaxM) return 0;
  return paro::stream_workspace_bytes(max_m);
}
}  // namespace

size_t paro_batched_workspace_bytes(const paro_linear* h_layers, int count) {
  if (!h_layers || count <= 0) return 0;
  size_t b = 0;
  for (int i = 0; i < count; ++i) b += xt_bytes(h_layers[i].M, h_layers[i].d_in);
  return b + batched_stream_bytes(h_layers, count);
}

paro_status paro_rotate_w4_linear_batched(const paro_linear* h_layers, int count, int group_size,
                                          void* d_workspace, size_t workspace_bytes, paro_stream_t stream) {
  if (count == 0) return ok();
  if (!h_layers || count < 0) return fail(PARO_ERR_INVALID_ARG, "null layer array or negative count");
  if (count > PARO_MAX_BATCH) return fail(PARO_ERR_UNSUPPORTED, "count = %d exceeds %d", count, PARO_MAX_BATCH);
  // the transformed activations are required; the stream-K kernel's flags and
  // partial tiles behind them are optional (without them the older kernel runs)
  const size_t need = paro_batched_workspace_bytes(h_layers, count);
  const size_t xt_need = need - batched_stream_bytes(h_layers, count);
  paro::RotProblem rp[PARO_MAX_BATCH];
  paro::GemvProblem gp[PARO_MAX_BATCH];
  int n = 0;
  size_t off = 0;
  bool decode_ok = true, any_transform = false;
  for (int i = 0; i < count; ++i) {
    const paro_linear& L = h_layers[i];
    paro_status st;
    if ((st = check_linear_shape(L.M, L.d_in, L.d_out, group_size)) != PARO_OK ||
        (st = check_width(L.d_in)) != PARO_OK ||
        (st = check_tables(L.K, L.d_in, L.d_pairs, L.d_cos, L.d_sin, L.d_scale)) != PARO_OK)
      return prefix_error(st, i);
    if (L.M == 0) continue;
    if ((st = check_weights(L.d_qweight, L.d_scales, L.d_zeros)) != PARO_OK)
      return prefix_error(st, i);
    if (!L.d_x || !L.d_y || !aligned(L.d_x, 16) || !aligned(L.d_y, 16))
      return fail(PARO_ERR_INVALID_ARG, "layer %d: x and y must be non-null and 16-byte aligned", i);
    const size_t yb = (size_t)L.M * L.d_out * 2;
    for (int j = 0; j < count; ++j) {
      const paro_linear& O = h_layers[j];
      if (O.M == 0) continue;
      if (overlap(L.d_y, yb, O.d_x, (size_t)O.M * O.d_in * 2) ||
          overlap(L.d_y, yb, O.d_qweight, (size_t)O.d_out * O.d_in / 2) ||
          (j != i && overlap(L.d_y, yb, O.d_y, (size_t)O.M * O.d_out * 2)))
        return fail(PARO_ERR_INVALID_ARG, "layer %d: y overlaps an input or output of layer %d", i, j);
    }
    if (L.M > 64 || (L.K > 0 && !paro::rot_decode_supported(L.d_in, L.d_pairs, L.d_cos, L.d_sin)))
      decode_ok = false;
    if (L.K > 0 || L.d_scale) any_transform = true;
    uint16_t* xt = reinterpret_cast<uint16_t*>(static_cast<char*>(d_workspace) + off);
    off += xt_bytes(L.M, L.d_in);
    rp[n] = paro::RotProblem{};
    rp[n].x = L.d_x;
    rp[n].out = xt;
    rp[n].M = L.M;
    rp[n].d = L.d_in;
    rp[n].K = L.K;
    rp[n].pairs = reinterpret_cast<const uint32_t*>(L.d_pairs);
    rp[n].cos_t = L.d_cos;
    rp[n].sin_t = L.d_sin;
    rp[n].scale = L.d_scale;
    gp[n] = paro::GemvProblem{};
    gp[n].x = xt;
    gp[n].qw = L.d_qweight;
    gp[n].sc = reinterpret_cast<const __half*>(L.d_scales);
    gp[n].z = reinterpret_cast<const __half*>(L.d_zeros);
    gp[n].y = reinterpret_cast<__nv_bfloat16*>(L.d_y);
    gp[n].M = L.M;
    gp[n].d_in = L.d_in;
    gp[n].d_out = L.d_out;
    ++n;
  }
  if (n == 0) return ok();
  if ((any_transform || !decode_ok) && (!d_workspace || workspace_bytes < xt_need || !aligned(d_workspace, 256)))
    return fail(PARO_ERR_INVALID_ARG, "workspace must be 256-byte aligned and hold %zu bytes", need);
  const size_t ws_used = d_workspace ? (workspace_bytes < need ? workspace_bytes : need) : 0;
  for (int i = 0; i < count && ws_used; ++i) {
    const paro_linear& L = h_layers[i];
    if (L.M == 0) continue;
    if (overlap(d_workspace, ws_used, L.d_x, (size_t)L.M * L.d_in * 2) ||
        overlap(d_workspace, ws_used, L.d_y, (size_t)L.M * L.d_out * 2))
      return fail(PARO_ERR_INVALID_ARG, "layer %d: workspace overlaps x or y", i);
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  // the stream-K kernel takes the INT4 linears when every linear has at most 16
  // tokens and the workspace holds its flags and partial tiles (behind the
  // transformed activations)
  const size_t xt_total = xt_need;
  bool use_stream = decode_ok && batched_stream_bytes(h_layers, count) > 0 && d_workspace &&
                    workspace_bytes >= need && aligned(d_workspace, 256);
  for (int i = 0; i < n && use_stream; ++i)
    use_stream = paro::stream_supported(gp[i].M, gp[i].d_in, gp[i].d_out, any_transform ? gp[i].x : rp[i].x,
                                        gp[i].qw);
  auto plan_stream = [&](bool x_f16, int reserved, paro::StreamBatch* sb, int* nt) -> cudaError_t {
    const uint16_t* xs[PARO_MAX_BATCH];
    const uint32_t* qs[PARO_MAX_BATCH];
    const __half *ss[PARO_MAX_BATCH], *zs[PARO_MAX_BATCH];
    __nv_bfloat16* ys[PARO_MAX_BATCH];
    int Ms[PARO_MAX_BATCH], dis[PARO_MAX_BATCH], dos[PARO_MAX_BATCH];
    for (int i = 0; i < n; ++i) {
      xs[i] = x_f16 ? gp[i].x : rp[i].x;
      qs[i] = gp[i].qw;
      ss[i] = gp[i].sc;
      zs[i] = gp[i].z;
      ys[i] = gp[i].y;
      Ms[i] = gp[i].M;
      dis[i] = gp[i].d_in;
      dos[i] = gp[i].d_out;
    }
    return paro::plan_stream_batch(xs, qs, ss, zs, ys, Ms, dis, dos, n, x_f16,
                                   static_cast<char*>(d_workspace) + xt_total, sb, nt, reserved);
  };
  auto launch_stream = [&](bool x_f16, int* st, bool pdl) -> cudaError_t {
    paro::StreamBatch sb;
    int nt = 1;
    cudaError_t err = plan_stream(x_f16, 0, &sb, &nt);
    if (err != cudaSuccess) return err;
    return paro::launch_stream_batch(sb, nt, x_f16, st, s, pdl);
  };
  if (!any_transform && decode_ok) {
    // few tokens and no layer has a transform: the INT4 linear reads the bf16 inputs directly
    if (use_stream) {
      int* status = status_ptr();
      if (!status) return fail(PARO_ERR_CUDA, "no CUDA device / status word unavailable");
      return from_cuda(launch_stream(false, status, true), "batched w4 linear launch");
    }
    for (int i = 0; i < n; ++i) gp[i].x = rp[i].x;
    paro::GemvBatch gb;
    int nt = 1;
    e = paro::plan_gemv_batch(gp, n, false, &gb, &nt);
    if (e == cudaSuccess) e = paro::launch_gemv_batch(gb, nt, s, true);
    return from_cuda(e, "batched w4 linear launch");
  }
  int* status = status_ptr();
  if (!status) return fail(PARO_ERR_CUDA, "no CUDA device / status word unavailable");
  if (!any_transform) {
    // many tokens and no layer has a transform: when the tensor-core kernel takes
    // every linear, one launch rounds every bf16 input to fp16 into the
    // workspace and the tensor-core kernel reads them by TMA (converting each
    // tile inside that kernel instead costs it a third more time: the
    // conversion competes with the dequantisation for shared memory)
    bool all_tc = true;
    paro::TcLinear tl[PARO_MAX_BATCH];
    const uint16_t* src[PARO_MAX_BATCH];
    uint16_t* dst[PARO_MAX_BATCH];
    size_t cnt[PARO_MAX_BATCH];
    for (int i = 0; i < n && all_tc; ++i) {
      all_tc = rp[i].M >= kTensorCoreMinM && paro::tc_supported(rp[i].M, rp[i].d, gp[i].d_out, gp[i].x);
      tl[i] = paro::TcLinear{gp[i].x, gp[i].qw, gp[i].sc, gp[i].z, gp[i].y, gp[i].M, gp[i].d_in, gp[i].d_out};
      src[i] = rp[i].x;
      dst[i] = static_cast<uint16_t*>(rp[i].out);
      cnt[i] = (size_t)rp[i].M * rp[i].d;
    }
    if (all_tc) {
      e = paro::launch_to_f16(src, dst, cnt, n, status, s);
      if (e == cudaSuccess) e = paro::launch_w4_tc_batch(tl, n, true, status, s);
      return from_cuda(e, "batched w4 linear launch");
    }
  }
  // the widest linear (the slowest transform) last, so that its units go to the
  // INT4 grid's last CTAs
  auto widest_last = [&]() {
    int widest = 0;
    for (int i = 1; i < n; ++i)
      if (rp[i].d > rp[widest].d) widest = i;
    if (widest == n - 1) return;
    const paro::RotProblem r = rp[widest];
    const paro::GemvProblem q = gp[widest];
    for (int i = widest; i + 1 < n; ++i) {
      rp[i] = rp[i + 1];
      gp[i] = gp[i + 1];
    }
    rp[n - 1] = r;
    gp[n - 1] = q;
  };
  if (decode_ok && use_stream && paro::fused_supported(rp, n)) {
    // one token per linear: the transforms run in the INT4 kernel's first CTAs
    // (one per linear) and each linear's arithmetic waits only for its own x~.
    // The widest linear goes to its own CTAs.
    widest_last();
    paro::RotBatch rb;
    paro::StreamBatch sb;
    int nt = 1;
    e = paro::plan_fused_rot(rp, n, &rb);
    rb.skip_flags = paro::hook_skip_ready_flags();
    if (e == cudaSuccess) e = plan_stream(true, rb.count, &sb, &nt);
    if (e == cudaSuccess) {
      paro::set_fused_split(sb, 0.6);
      e = paro::launch_fused_batch(sb, rb, status, s, true);
    }
    return from_cuda(e, "batched fused launch");
  }
  if (decode_ok && use_stream) {
    // few tokens: the transform launch publishes a flag per CTA, and the INT4
    // launch after it requests a linear's x~ once that linear's transform CTAs
    // have all published, not when the whole transform launch is done
    // The widest linear's units go last in the INT4 launch; its transform
    // (the slowest) takes the transform launch's first CTAs, which get SMs first.
    widest_last();
    paro::RotProblem rt[PARO_MAX_BATCH];
    rt[0] = rp[n - 1];
    for (int i = 0; i + 1 < n; ++i) rt[i + 1] = rp[i];
    for (int i = 0; i < n; ++i) rt[i].perm = 1;  // x~ in the stream-K kernel's operand order
    paro::RotBatch rb;
    paro::StreamBatch sb;
    int R = 1, nt = 1;
    e = paro::plan_rot_batch(rt, n, &rb, &R);
    if (e == cudaSuccess) e = plan_stream(true, 0, &sb, &nt);
    if (e == cudaSuccess && sb.total_units < 96LL * sb.ctas) {
      // a short INT4 share per CTA (Qwen2.5-1.5B's layer: about 39 units): the
      // INT4 launch leaves half as many SMs as the transform has CTAs to it,
      // so that fewer INT4 CTAs start only when a transform ends (measured:
      // the 16-token stack 1198 -> 1139 us, 4 tokens 34.1 -> 32.0 us; a long
      // share, Llama-3-8B's, loses by it: 93 -> 102 us at 16 tokens)
      const int half_sms = paro::device_sm_count() / 2, res = rb.total_ctas / 2;
      e = plan_stream(true, res < half_sms ? res : half_sms, &sb, &nt);
    }
    if (e != cudaSuccess) return from_cuda(e, "batched decode plan");
    // at most 16 rows of at most 8 linears, one row or more a CTA: the flag
    // area always suffices; checked so that no CTA could write past it
    if (rb.total_ctas > paro::kXFlagWords)
      return fail(PARO_ERR_UNSUPPORTED, "%d transform CTAs exceed the workspace's %d flags", rb.total_ctas,
                  paro::kXFlagWords);
    rb.ctl = sb.ctl;
    rb.xflags = sb.xflags;
    rb.skip_flags = paro::hook_skip_ready_flags();
    for (int i = 0; i < n; ++i) {
      const paro::RotProblem& t = rb.p[i + 1 < n ? i + 1 : 0];
      sb.p[i].xf_begin = t.cta_begin;
      sb.p[i].xf_count = (t.M + t.rows - 1) / t.rows;
    }
    // The CTAs of the widest linear, whose transform ends last, take fewer
    // units: with a long INT4 share per CTA (at least 96 units: Llama-3-8B's
    // layer has about 180) 1 - 0.9 (w - o) / w of the others' (measured at 8
    // and 16 tokens: Llama 54.3 -> 50.9 and 86.7 -> 79.5 us), with a short one
    // (Qwen2.5-1.5B's 39, beside the reserved SMs above) 1 - 0.6 (w - o) / w
    // (the 16-token stack 1114 -> 1007 us, the layer at 4 tokens 31.3 -> 29.5).
    paro::set_fused_split(sb, sb.total_units >= 96LL * sb.ctas ? 0.9 : 0.6);
    e = paro::launch_rot_batch(rb, R, true, status, s, true, true);
    if (e == cudaSuccess) e = paro::launch_stream_flagged(sb, nt, status, s);
    return from_cuda(e, "batched decode launch");
  }
  if (decode_ok) {
    paro::RotBatch rb;
    int R = 1;
    e = paro::plan_rot_batch(rp, n, &rb, &R);
    if (e == cudaSuccess) e = paro::launch_rot_batch(rb, R, true, status, s, true, true);
  } else {
    // many tokens (or tables the decode kernel cannot take): every transform, then
    // one persistent tensor-core launch over all linears it takes (their tiles
    // balanced over the SMs together); any other linear on its own
    e = cudaSuccess;
    for (int i = 0; i < n && e == cudaSuccess; ++i)
      e = launch_transform(rp[i].x, rp[i].out, true, rp[i].M, rp[i].d, rp[i].K,
                           reinterpret_cast<const uint16_t*>(rp[i].pairs), rp[i].cos_t, rp[i].sin_t, rp[i].scale,
                           status, s, false);
    paro::TcLinear tl[PARO_MAX_BATCH];
    int ntc = 0;
    for (int i = 0; i < n && e == cudaSuccess; ++i) {
      if (gp[i].M >= kTensorCoreMinM && paro::tc_supported(gp[i].M, gp[i].d_in, gp[i].d_out, gp[i].x))
        tl[ntc++] = paro::TcLinear{gp[i].x, gp[i].qw, gp[i].sc, gp[i].z, gp[i].y, gp[i].M, gp[i].d_in, gp[i].d_out};
      else
        e = launch_linear(gp[i].x, true, gp[i].qw, reinterpret_cast<const uint16_t*>(gp[i].sc),
                          reinterpret_cast<const uint16_t*>(gp[i].z), reinterpret_cast<uint16_t*>(gp[i].y), gp[i].M,
                          gp[i].d_in, gp[i].d_out, s, false, status);
    }
    if (e == cudaSuccess && ntc > 0) e = paro::launch_w4_tc_batch(tl, ntc, true, status, s);
    return from_cuda(e, "batched launch");
  }
  if (e != cudaSuccess) return from_cuda(e, "batched transform launch");
  paro::GemvBatch gb;
  int nt = 1;
  e = paro::plan_gemv_batch(gp, n, true, &gb, &nt);
  if (e == cudaSuccess) e = paro::launch_gemv_batch(gb, nt, s, true);
  return from_cuda(e, "batched w4 linear launch");
}

// ---- weight-activation (W4A4) variant ----------------------------------------------
namespace {
size_t r256(size_t b) { return (b + 255) & ~(size_t)255; }
size_t w4a4_front_bytes(int M, int d_in) {
  return r256((size_t)M * d_in * 2) + r256((size_t)M * d_in) + r256((size_t)M * 4);
}
}  // namespace

size_t paro_w4a4_workspace_bytes(int M, int d_in, int d_out, int with_transform) {
  if (M <= 0 || d_in <= 0 || d_out <= 0) return 0;
  const size_t part = paro::w4a4_partial_bytes(M, d_in, d_out, paro::device_sm_count());
  return (with_transform ? w4a4_front_bytes(M, d_in) : 0) + part;
}

paro_status paro_quantize_activations(const uint16_t* d_x, int8_t* d_q, float* d_sx, int M, int d,
                                      paro_stream_t stream) {
  if (M < 0) return fail(PARO_ERR_INVALID_ARG, "M = %d is negative", M);
  if (d <= 0 || d % 8) return fail(PARO_ERR_INVALID_ARG, "d = %d must be a positive multiple of 8", d);
  if (M == 0) return ok();
  if (!d_x || !d_q || !d_sx) return fail(PARO_ERR_INVALID_ARG, "null pointer");
  if (!aligned(d_x, 16) || !aligned(d_q, 8) || !aligned(d_sx, 4))
    return fail(PARO_ERR_INVALID_ARG, "x must be 16-byte, q 8-byte and sx 4-byte aligned");
  const size_t xb = (size_t)M * d * 2;
  if (overlap(d_q, (size_t)M * d, d_x, xb) || overlap(d_sx, (size_t)M * 4, d_x, xb) ||
      overlap(d_q, (size_t)M * d, d_sx, (size_t)M * 4))
    return fail(PARO_ERR_INVALID_ARG, "x, q and sx must not overlap");
  return from_cuda(paro::launch_quantize_act(d_x, d_q, d_sx, M, d, reinterpret_cast<cudaStream_t>(stream)),
                   "quantize launch");
}

paro_status paro_w4a4_linear(const int8_t* d_q, const float* d_sx, const uint32_t* d_qweight,
                             const uint16_t* d_scales, const uint16_t* d_zeros, uint16_t* d_y, int M, int d_in,
                             int d_out, int group_size, void* d_workspace, size_t workspace_bytes,
                             paro_stream_t stream) {
  paro_status st;
  if ((st = check_linear_shape(M, d_in, d_out, group_size)) != PARO_OK) return st;
  if (M == 0) return ok();
  if ((st = check_weights(d_qweight, d_scales, d_zeros)) != PARO_OK) return st;
  if (!d_q || !d_sx || !d_y) return fail(PARO_ERR_INVALID_ARG, "null activation pointer");
  if (!aligned(d_q, 16) || !aligned(d_sx, 4) || !aligned(d_y, 2))
    return fail(PARO_ERR_INVALID_ARG, "q must be 16-byte aligned, sx 4-byte, y 2-byte");
  const int sms = paro::device_sm_count();
  const int shares = paro::w4a4_shares(d_in, d_out, sms);
  const size_t need = paro::w4a4_partial_bytes(M, d_in, d_out, sms);
  if (need && (!d_workspace || workspace_bytes < need || !aligned(d_workspace, 256)))
    return fail(PARO_ERR_INVALID_ARG, "workspace must be 256-byte aligned and hold %zu bytes", need);
  const size_t yb = (size_t)M * d_out * 2;
  if (overlap(d_y, yb, d_q, (size_t)M * d_in) || overlap(d_y, yb, d_sx, (size_t)M * 4) ||
      overlap(d_y, yb, d_qweight, (size_t)d_out * d_in / 2) || (need && overlap(d_y, yb, d_workspace, need)))
    return fail(PARO_ERR_INVALID_ARG, "y must not overlap an input or the workspace");
  cudaError_t e = paro::launch_w4a4(d_q, d_sx, d_qweight, d_scales, d_zeros, d_y, M, d_in, d_out,
                                    static_cast<float*>(need ? d_workspace : nullptr), shares,
                                    reinterpret_cast<cudaStream_t>(stream));
  return from_cuda(e, "w4a4 linear launch");
}

paro_status paro_rotate_w4a4_linear(const uint16_t* d_x, int K, const uint16_t* d_pairs, const float* d_cos,
                                    const float* d_sin, const float* d_scale, const uint32_t* d_qweight,
                                    const uint16_t* d_scales, const uint16_t* d_zeros, uint16_t* d_y, int M,
                                    int d_in, int d_out, int group_size, void* d_workspace, size_t workspace_bytes,
                                    paro_stream_t stream) {
  paro_status st;
  if ((st = check_linear_shape(M, d_in, d_out, group_size)) != PARO_OK) return st;
  if ((st = check_width(d_in)) != PARO_OK) return st;
  if ((st = check_tables(K, d_in, d_pairs, d_cos, d_sin, d_scale)) != PARO_OK) return st;
  if (M == 0) return ok();
  if ((st = check_weights(d_qweight, d_scales, d_zeros)) != PARO_OK) return st;
  if (!d_x || !d_y) return fail(PARO_ERR_INVALID_ARG, "null activation pointer");
  if (!aligned(d_x, 16) || !aligned(d_y, 16)) return fail(PARO_ERR_INVALID_ARG, "x and y must be 16-byte aligned");
  const size_t need = paro_w4a4_workspace_bytes(M, d_in, d_out, 1);
  if (!d_workspace || workspace_bytes < need || !aligned(d_workspace, 256))
    return fail(PARO_ERR_INVALID_ARG, "workspace must be 256-byte aligned and hold %zu bytes", need);
  const size_t yb = (size_t)M * d_out * 2, xb = (size_t)M * d_in * 2;
  if (overlap(d_y, yb, d_x, xb) || overlap(d_y, yb, d_workspace, need) || overlap(d_workspace, need, d_x, xb) ||
      overlap(d_y, yb, d_qweight, (size_t)d_out * d_in / 2))
    return fail(PARO_ERR_INVALID_ARG, "y, x and workspace must not overlap");
  int* status = status_ptr();
  if (!status) return fail(PARO_ERR_CUDA, "no CUDA device / status word unavailable");
  char* ws = static_cast<char*>(d_workspace);
  uint16_t* xt = reinterpret_cast<uint16_t*>(ws);
  int8_t* q = reinterpret_cast<int8_t*>(ws + r256(xb));
  float* sx = reinterpret_cast<float*>(ws + r256(xb) + r256((size_t)M * d_in));
  float* part = reinterpret_cast<float*>(ws + w4a4_front_bytes(M, d_in));
  const int sms = paro::device_sm_count();
  const int shares = paro::w4a4_shares(d_in, d_out, sms);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_transform(d_x, xt, false, M, d_in, K, d_pairs, d_cos, d_sin, d_scale, status, s, false);
  if (e != cudaSuccess) return from_cuda(e, "rotate launch");
  e = paro::launch_quantize_act(xt, q, sx, M, d_in, s);
  if (e != cudaSuccess) return from_cuda(e, "quantize launch");
  e = paro::launch_w4a4(q, sx, d_qweight, d_scales, d_zeros, d_y, M, d_in, d_out, shares > 1 ? part : nullptr,
                        shares, s);
  return from_cuda(e, "w4a4 linear launch");
}

paro_status paro_get_device_status(paro_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return from_cuda(e, "stream synchronize");
  int* p = status_ptr();
  if (!p) return fail(PARO_ERR_CUDA, "no CUDA device / status word unavailable");
  int v = 0;
  e = cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return from_cuda(e, "status read");
  const int zero = 0;
  e = cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return from_cuda(e, "status clear");
  if (v == 0) return ok();
  return fail(static_cast<paro_status>(v), "device reported %s", paro_status_string(static_cast<paro_status>(v)));
}

}  // extern "C"
