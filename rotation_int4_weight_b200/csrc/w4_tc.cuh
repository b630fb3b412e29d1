// Tensor-core (tcgen05) INT4 linear for many tokens (w4_tc.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace paro {

constexpr int kTcMaxBatch = 8;  // linears served by one launch

// One linear of a launch, as the kernel sees it.
struct TcProblem {
  CUtensorMap xmap;          // fp16 activations [M][d_in], box 64 columns x 256 tokens, 128-byte swizzle
  CUtensorMap qmap;          // packed codes uint32 [d_out][d_in / 8], box 8 words x 256 rows, 32-byte swizzle
  const uint16_t* xraw;      // bf16 activations [M][d_in] (bf16-input kernel)
  const unsigned short* sc;  // fp16 bits [d_out][d_in / 128]
  const unsigned short* z;   // fp16 bits [d_out][d_in / 128]
  __nv_bfloat16* y;          // [M][d_out]
  int M, d_in, d_out;
  int n_tiles;               // ceil(d_out / 256)
  int tile_begin;            // first tile of this linear in the launch's tile list
};

struct TcBatch {
  TcProblem p[kTcMaxBatch];
  int count;
  int total_tiles;
};

// One linear as the host describes it.
struct TcLinear {
  const uint16_t* x;  // fp16 or bf16 [M][d_in] (one type per launch)
  const uint32_t* qweight;
  const __half* scales;
  const __half* zeros;
  __nv_bfloat16* y;
  int M, d_in, d_out;
};

// True when the tcgen05 kernel applies: M >= 128, d_in a multiple of 64,
// d_out a multiple of 16, x 16-byte aligned.
bool tc_supported(int M, int d_in, int d_out, const void* x);

// One persistent launch over up to kTcMaxBatch linears: a CTA per SM walks the
// 256 x 256 output tiles of all of them, the linears with the longest K first.
cudaError_t launch_w4_tc_batch(const TcLinear* lins, int count, bool x_f16, int* status, cudaStream_t stream);
// bf16 -> fp16 (round to nearest) of up to kMaxBatch arrays in one launch,
// n[i] values each (a multiple of 8, 16-byte aligned arrays); a value beyond
// the fp16 range is reported as PARO_ERR_RANGE.  The plain (untransformed)
// linears of a batched call with many tokens take this pass into the
// workspace and the tensor-core kernel's fp16 path, rather than converting
// each tile in the kernel, where the conversion competes with the
// dequantisation for shared memory.
cudaError_t launch_to_f16(const uint16_t* const* src, uint16_t* const* dst, const size_t* n, int count, int* status,
                          cudaStream_t stream);

// The dense-rotation contrast: y = x Q^T for bf16 x [M][d] and a bf16 d x d
// matrix Q (row n = output channel n), on the same tensor-core pipeline with
// the matrix tiles copied by TMA instead of dequantised; bf16 out.
bool dense_supported(int M, int d, const void* x, const void* q);
cudaError_t launch_dense_tc(const uint16_t* x, const uint16_t* q, __nv_bfloat16* y, int M, int d, int* status,
                            cudaStream_t stream);

cudaError_t launch_w4_tc(const uint16_t* x, bool x_f16, const uint32_t* qweight, const __half* scales,
                         const __half* zeros, __nv_bfloat16* y, int M, int d_in, int d_out, int* status,
                         cudaStream_t stream);

}  // namespace paro
