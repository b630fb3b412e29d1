// Tensor-core (tcgen05) INT4 linear for many tokens (w4_tc.cu).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace paro {

// True when the tcgen05 kernel applies: M >= 128, d_in a multiple of 64,
// d_out a multiple of 16, x 16-byte aligned.
bool tc_supported(int M, int d_in, int d_out, const void* x);

cudaError_t launch_w4_tc(const uint16_t* x, bool x_f16, const uint32_t* qweight, const __half* scales,
                         const __half* zeros, __nv_bfloat16* y, int M, int d_in, int d_out, int* status,
                         cudaStream_t stream);

}  // namespace paro
