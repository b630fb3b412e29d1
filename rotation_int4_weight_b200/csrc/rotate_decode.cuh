// Problem descriptors of the few-token (decode) transform kernel (rotate_decode.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "w4_gemv.cuh"  // kMaxBatch

namespace paro {

struct RotProblem {
  const uint16_t* x;      // bf16 [M][d]
  void* out;              // bf16 or fp16 [M][d] (one type per launch)
  int M, d, K;
  const uint32_t* pairs;  // [K][d/2], (i | j << 16)
  const float* cos_t;     // [K][d/2]
  const float* sin_t;     // [K][d/2]
  const float* scale;     // [d] or null
  // filled by plan_rot_batch
  int perm;               // fp16 out for the stream-K INT4 kernel: every 8-column block stored as
                          // (x0, x4, x1/16, x5/16, x2, x6, x3/16, x7/16), its MMA operand order
  int sscale;             // the channel scale in shared memory for the final pass, one bulk copy:
                          // 1 a region after the table ring, requested with the first stages;
                          // 2 the ring slot the last table refill leaves free, requested then;
                          // 0 read from global memory by the final pass (also: no scale)
  int rows;               // token rows a CTA (<= the launch's R; 0 means R)
  int ring;               // stages of tables held in shared memory at once
  int cta_begin;          // first CTA of this problem
};

struct RotBatch {
  RotProblem p[kMaxBatch];
  // optional (the INT4 linear that follows then waits per linear, not for the
  // whole grid): every CTA, once it has waited for the previous kernel, takes
  // the tag 2E + 1 from the epoch word *ctl (advanced by the last CTA of the
  // previous INT4 launch on this workspace), lets its dependents launch, and
  // sets xflags[its index] to the tag once its rows of x~ are written
  unsigned long long* ctl;
  unsigned long long* xflags;
  int skip_flags;  // test hook: publish no xflags (the INT4 linear's waits then run out)
  int count;
  int total_ctas;
};

// True when the decode kernel can run this width with these table pointers
// (d % 8 == 0 and 16-byte aligned tables, since stages are copied in 16-byte pieces).
bool rot_decode_supported(int d, const void* pairs, const void* cos_t, const void* sin_t);
cudaError_t plan_rot_batch(const RotProblem* probs, int count, RotBatch* out, int* R_out);
// RotProblem::sscale for a problem with `ring` table slots: 1 when a region
// for the scale fits beside them, else 2 when a slot frees before the end.
int scale_mode(const RotProblem& p, int ring, bool region_fits);
// pdl_trigger: let the next kernel launch early; pdl_wait: launched as a
// programmatic dependent, fetches its tables early and waits for the previous
// kernel before it reads the rows or writes the output.
cudaError_t launch_rot_batch(const RotBatch& b, int R, bool f16_out, int* status, cudaStream_t stream,
                             bool pdl_trigger, bool pdl_wait = false);

}  // namespace paro
