// Internal declarations shared by the CUDA translation units of libparo.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/paro.h"

namespace paro {

// Values written into the per-device status word (first error wins).
constexpr int kStatusBadIndex = PARO_ERR_INVALID_ARG;
constexpr int kStatusTimeout = PARO_ERR_TIMEOUT;
constexpr int kStatusRange = PARO_ERR_RANGE;

// Default bound of a bounded wait, in SM clock cycles (about a second).
constexpr long long kWaitCycles = 1LL << 31;

// True when either half of a packed fp16 pair is infinite (the rounding of a
// finite value beyond the fp16 range).
__device__ __forceinline__ bool half2_inf(uint32_t u) {
  return ((u & 0x7FFFu) == 0x7C00u) | ((u & 0x7FFF0000u) == 0x7C000000u);
}

constexpr int kGroup = 128;      // quantisation group along d_in
constexpr int kMaxStages = 16;   // K
constexpr int kMaxDim = 49152;   // rotation width (one fp32 row in shared memory)

__device__ __forceinline__ void report_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Stores a printf-style message for paro_last_error() and returns s.
paro_status record_error(paro_status s, const char* fmt, ...);

// Test hooks (paro_set_test_hooks): the wait bound for hand-over flags in
// cycles, and whether the decode transforms skip publishing their flags.
long long hook_flag_wait();
int hook_skip_ready_flags();

// ---- launchers implemented in the kernel translation units --------------------
// All return a cudaError_t from the launch (cudaSuccess when nothing failed).

// Activation transform, bf16 -> bf16 (mode 0) or bf16 -> fp16 (mode 1).
// Gradients of the activation transform (rotate_backward.cu): token rows per
// block for width d (0 when d is too wide), the workspace of the per-block
// partial sums, and the two launches (blocks, then the ordered reduction).
int rot_bwd_rows(int d);
size_t rot_bwd_workspace_bytes(int M, int d, int K, bool with_scale);
cudaError_t launch_rot_backward(const uint16_t* x, const float* grad, int M, int d, int K, const uint32_t* pairs,
                                const float* cos_t, const float* sin_t, const float* scale, float* dx, float* dtheta,
                                float* dscale, void* ws, int* status, cudaStream_t stream);
cudaError_t launch_rotate_act(const uint16_t* x, void* out, int out_is_f16, int M, int d, int K,
                              const uint16_t* pairs, const float* cos_t, const float* sin_t,
                              const float* scale, int* status, cudaStream_t stream, bool pdl_trigger);

// Weight fold, fp32 -> fp32: rows of W go through the same stages, then * s.
cudaError_t launch_fold_weights(const float* W, float* out, int rows, int d, int K,
                                const uint16_t* pairs, const float* cos_t, const float* sin_t,
                                const float* scale, int* status, cudaStream_t stream);

// Group quantisation + nibble packing of fp32 rows.
cudaError_t launch_quantize_pack(const float* Wt, int d_out, int d_in, uint32_t* qweight,
                                 __half* scales, __half* zeros, cudaStream_t stream);

// The weight-activation variant (w4a4.cu): per-token INT4 codes of bf16
// activations [M][d] (d % 8 == 0, 16-byte aligned rows), and the INT4 x INT4
// linear.  The linear splits each 64-row tile's groups into w4a4_shares(...)
// shares; with more than one it needs w4a4_partial_bytes(...) of fp32 partials
// and a second, ordered reduction launch.
int w4a4_shares(int d_in, int d_out, int sms);
size_t w4a4_partial_bytes(int M, int d_in, int d_out, int sms);
cudaError_t launch_quantize_act(const uint16_t* x, int8_t* q, float* sx, int M, int d, cudaStream_t stream);
cudaError_t launch_w4a4(const int8_t* qx, const float* sx, const uint32_t* qw, const uint16_t* sw,
                        const uint16_t* zw, uint16_t* y, int M, int d_in, int d_out, float* part, int shares,
                        cudaStream_t stream);

}  // namespace paro
