// Problem descriptors of the stream-K INT4 linear for few tokens (w4_stream.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "w4_gemv.cuh"  // kMaxBatch
#include "rotate_decode.cuh"

namespace paro {

constexpr int kStreamMaxM = 16;     // tokens per launch (two 8-token MMA column tiles)
constexpr int kStreamRows = 64;     // weight rows per tile (four 16-row MMA tiles)

struct StreamProblem {
  CUtensorMap qmap;            // packed weights, uint32 [d_out][d_in/8], box 16 words x 64 rows
  CUtensorMap xmap;            // activations [M][d_in] fp16/bf16, box 64 x M, 128-byte swizzle
  const unsigned short* sc;    // fp16 bits [d_out][d_in/128]
  const unsigned short* z;     // fp16 bits [d_out][d_in/128]
  __nv_bfloat16* y;            // [M][d_out]
  long long unit_begin;        // first unit (one 64-row tile x one 128-column group) of this linear
  int tile_begin;              // first tile of this linear among the tiles of the launch
  int M, d_in, d_out, G;       // G = d_in / 128
  int tiles;                   // ceil(d_out / 64)
  int xf_begin, xf_count;      // flag form: the flags of this linear's transform CTAs
};

struct StreamBatch {
  StreamProblem p[kMaxBatch];
  long long total_units;
  // two tile partials per CTA (workspace): every 64-bit word one fp32 value in
  // its low half and the low 32 bits of the publishing launch's tag in its high half
  unsigned long long* partials;
  unsigned long long* xflags;    // fused form: one per linear, set when its x~ is written (workspace);
                                 // flag form: one per CTA of the preceding transform launch
  // the workspace's launch epoch E (ctl[0]) and a wrapping count of the CTAs
  // of the current launch that have finished (the low word of ctl[1]): every
  // flag a launch publishes holds 2E + 1 for the E of that launch, and its last
  // CTA advances E, so a flag left by an earlier launch (or a replay of the
  // same CUDA graph) never matches; null in the tile-split form
  unsigned long long* ctl;
  // CTAs 0 .. ctas_a - 1 split units [0, units_a) evenly and the others the rest
  // (the fused form gives the widest linear, whose x~ comes last, fewer units a
  // CTA); ctas_a = ctas, units_a = total_units is the even split
  long long units_a;
  long long flag_wait;           // bound of a hand-over flag wait, SM clock cycles
  int ctas_a;
  // tile_split != 0: CTA c takes the whole tiles [c T / C, (c + 1) T / C) of the
  // T tiles of the launch, so no tile crosses a CTA boundary and the
  // cross-CTA flags and partials (flags, partials) are never used
  int tile_split;
  int total_tiles;
  int one;                       // every linear has one token (its activation geometry, see the kernel)
  int count;
  int ctas;                      // CTAs of the INT4 linear (after the transform CTAs in the fused form)
};

// True when a linear can run on the stream-K kernel (the caller also checks M).
bool stream_supported(int M, int d_in, int d_out, const void* x, const void* qweight);
// Workspace bytes of the kernel's publication flags and cross-CTA partial sums.
size_t stream_workspace_bytes(int max_m);
// Builds the launch descriptor: tensor maps, unit and tile offsets, the CTA count.
// x_f16 selects fp16 (else bf16) activations; ws points at stream_workspace_bytes().
// ws == nullptr plans the tile-split form (no cross-CTA partial sums).
cudaError_t plan_stream_batch(const uint16_t* const* x, const uint32_t* const* qw, const __half* const* sc,
                              const __half* const* z, __nv_bfloat16* const* y, const int* M, const int* d_in,
                              const int* d_out, int count, bool x_f16, void* ws, StreamBatch* out, int* nt_out,
                              int reserved_ctas = 0);
cudaError_t launch_stream_batch(const StreamBatch& b, int NT, bool x_f16, int* status, cudaStream_t stream,
                                bool pdl_wait);
// The flag form (fp16 x~ written by a transform launched just before with
// flags and, per problem, perm set: x~ in the kernel's operand order, see
// RotProblem): instead of waiting for the whole transform launch, the
// INT4 linear requests a linear's activations once all of that linear's
// transform CTAs have published.  b.ctl, b.xflags and every problem's
// xf_begin / xf_count must be set.
cudaError_t launch_stream_flagged(const StreamBatch& b, int NT, int* status, cudaStream_t stream);
// Workspace words of the flag form: one flag per transform CTA.
constexpr int kXFlagWords = kMaxBatch * kStreamMaxM;

// The fused form for one token per linear: the kernel's first rb.count CTAs
// each run the activation transform of one linear (writing its fp16 x~, the
// activations b reads) and then publish a flag; the other CTAs run the INT4
// linear, requesting a linear's activations once its flag is set, so their
// weight streaming and the transforms overlap and a linear's arithmetic waits
// only for its own transform.  b must come from plan_stream_batch with
// reserved_ctas = rb.count and x_f16; rb from plan_fused_rot.
bool fused_supported(const RotProblem* probs, int count);
// When the last linear is at least 1.5 times wider than any other, its
// transform finishes last: its units go to a separate group of CTAs with
// proportionally fewer units each, so that those CTAs, which start late,
// finish with the others.  A CTA of the last linear gets 1 - late (w - o) / w
// of the others' share (w, o: the widest and the next widest d_in).
void set_fused_split(StreamBatch& b, double late);
cudaError_t plan_fused_rot(const RotProblem* probs, int count, RotBatch* out);
cudaError_t launch_fused_batch(const StreamBatch& b, const RotBatch& rb, int* status, cudaStream_t stream,
                               bool pdl_wait);
// Streaming multiprocessors of the current device (cached per device).
int device_sm_count();

}  // namespace paro
