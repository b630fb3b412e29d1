// Group-wise asymmetric INT4 quantisation and nibble packing of folded weights
// (page "ParoQuant: pairwise rotations that survive deployment": INT4 with
// group size 128 in section "My reduced-calibration experiment"; real INT4
// packing in section "From fake quantization to a real TensorRT engine").
//
// Per (row, group of 128 input columns), in fp32 IEEE arithmetic with
// round-half-to-even and this exact operation order (compiled without FMA
// contraction, with IEEE division):
//   mn = min(0, min v), mx = max(0, max v), s32 = (mx - mn) / 15,
//   sc = fp16(s32); if sc == 0 { sc = 1; z = 0 } else z = clamp(rint(-mn / sc), 0, 15)
//   q  = clamp(rint(v / sc) + z, 0, 15)
// Codes are packed eight per uint32 along the input dimension: column 8w+e
// goes to bits [4e, 4e+4) of word w.
//
// One warp handles one group: lane l holds columns 4l..4l+3 of the group
// (one 16-byte load), min/max are warp reductions, and lanes 2t, 2t+1 merge
// their four codes each into word t of the group.
#include "paro_internal.cuh"

namespace paro {
namespace {

__global__ void __launch_bounds__(256)
quantize_pack_kernel(const float* __restrict__ Wt, int d_out, int d_in, uint32_t* __restrict__ qweight,
                     __half* __restrict__ scales, __half* __restrict__ zeros) {
  const int groups_per_row = d_in / kGroup;
  const long long total = (long long)d_out * groups_per_row;
  const int lane = threadIdx.x & 31;
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long gidx = warp; gidx < total; gidx += nwarps) {
    const int n = (int)(gidx / groups_per_row);
    const int g = (int)(gidx % groups_per_row);
    const float* src = Wt + (size_t)n * d_in + (size_t)g * kGroup + lane * 4;
    const float4 v4 = *reinterpret_cast<const float4*>(src);
    const float v[4] = {v4.x, v4.y, v4.z, v4.w};

    float lo = fminf(fminf(v[0], v[1]), fminf(v[2], v[3]));
    float hi = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    const float mn = fminf(lo, 0.0f);
    const float mx = fmaxf(hi, 0.0f);
    const float s32 = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
    __half sc = __float2half_rn(s32);
    float z = 0.0f;
    if (__half2float(sc) == 0.0f) {
      sc = __float2half_rn(1.0f);
    } else {
      z = fminf(fmaxf(rintf(__fdiv_rn(-mn, __half2float(sc))), 0.0f), 15.0f);
    }
    const float scf = __half2float(sc);
    uint32_t nib = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float q = fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(v[e], scf)), z), 0.0f), 15.0f);
      nib |= ((uint32_t)q & 0xFu) << (4 * e);
    }
    // lanes 2t (columns 8t..8t+3) and 2t+1 (8t+4..8t+7) form word t
    const uint32_t other = __shfl_down_sync(0xffffffffu, nib, 1);
    if ((lane & 1) == 0) {
      qweight[(size_t)n * (d_in / 8) + (size_t)g * (kGroup / 8) + (lane >> 1)] = nib | (other << 16);
    }
    if (lane == 0) {
      scales[(size_t)n * groups_per_row + g] = sc;
      zeros[(size_t)n * groups_per_row + g] = __int2half_rn((int)z);
    }
  }
}

}  // namespace

cudaError_t launch_quantize_pack(const float* Wt, int d_out, int d_in, uint32_t* qweight,
                                 __half* scales, __half* zeros, cudaStream_t stream) {
  const long long groups = (long long)d_out * (d_in / kGroup);
  const int threads = 256;
  long long blocks = (groups * 32 + threads - 1) / threads;
  if (blocks > 148LL * 16) blocks = 148LL * 16;
  quantize_pack_kernel<<<(unsigned)blocks, threads, 0, stream>>>(Wt, d_out, d_in, qweight, scales, zeros);
  return cudaPeekAtLastError();
}

}  // namespace paro
