// Problem descriptors of the few-token INT4 linear (w4_gemv.cu).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace paro {

constexpr int kMaxBatch = 8;  // linears served by one launch

struct GemvProblem {
  const uint16_t* x;   // activations [M][d_in], fp16 or bf16 (one type per launch)
  const uint32_t* qw;  // packed weights [d_out][d_in/8]
  const __half* sc;    // scales [d_out][d_in/128]
  const __half* z;     // zero points [d_out][d_in/128]
  __nv_bfloat16* y;    // output [M][d_out]
  int M, d_in, d_out;
  // filled by plan_gemv_batch
  int log2_chunks;     // the 8 warps of a CTA form 2^log2_chunks groups splitting d_in
  int row_blocks;      // CTAs per 16-token block
  int item_begin;      // first CTA of this linear
  int x_tok;           // token rows per activation stage (same for the whole launch)
};

struct GemvBatch {
  GemvProblem p[kMaxBatch];
  int count;
  int total_items;
  int x_f16;
};

cudaError_t plan_gemv_batch(const GemvProblem* probs, int count, bool x_f16, GemvBatch* out, int* nt_out);
cudaError_t launch_gemv_batch(const GemvBatch& b, int NT, cudaStream_t stream, bool pdl_wait);

}  // namespace paro
