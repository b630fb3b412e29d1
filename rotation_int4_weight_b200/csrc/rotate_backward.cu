// Gradients of the activation-side transform x~ = diag(1/s) R_K ... R_1 x:
// for an upstream gradient G = dL/dx~ (one row per token), dL/dx, dL/dtheta
// for the angle of every pair of every stage, and dL/ds for the channel scale
// (page "ParoQuant: Pairwise Rotation Quantization for Efficient Reasoning
// LLM Inference", abstract: the Givens rotations and the scaling are
// optimizable; page "ParoQuant: pairwise rotations that survive deployment",
// section "A rotation small enough to execute": the forward transform).
//
// By the chain rule, with (c, s) the pair's cos and sin, x' the stage output
// and h = dL/dx' (the pages print no backward pass; this is its plain reading):
//   dL/dtheta = sum over tokens of (h_i x_j' - h_j x_i'),
//   dL/dx_i = c h_i - s h_j,  dL/dx_j = s h_i + c h_j   (the transposed rotation),
//   dL/ds_c = -sum over tokens of G_c x~_c / s_c,  h = G / s at the last stage.
//
// rot_bwd_kernel: one CTA per block of R token rows, fp32 planes in shared
// memory for x and h.  It runs the K stages forward, applies the scale step,
// then walks the stages backward: each pair accumulates its dtheta over the
// block's rows, maps h through the transposed rotation and recovers the
// stage's input from its output by the inverse rotation (x = R_k^T x'), so no
// intermediate is stored.  Its per-block partial sums of dtheta and ds go to
// the workspace; rot_bwd_reduce_kernel adds them over the blocks in block
// order (deterministic), and dL/dx is written by the block itself.
#include "paro_internal.cuh"

namespace paro {
namespace {

constexpr int kBwdThreads = 1024;
constexpr size_t kBwdSmemBudget = 227 * 1024 - 1024;

size_t bwd_smem(int d, int R) { return (size_t)8 * R * d; }

template <int R>
__global__ void __launch_bounds__(kBwdThreads)
rot_bwd_kernel(const uint16_t* __restrict__ x, const float* __restrict__ grad, int M, int d, int K,
               const uint32_t* __restrict__ pairs, const float* __restrict__ cos_t, const float* __restrict__ sin_t,
               const float* __restrict__ scale, float* __restrict__ dx, float* __restrict__ part, int* status) {
  extern __shared__ __align__(16) float sm[];
  float* xs = sm;                   // [R][d]
  float* hs = sm + (size_t)R * d;   // [R][d]
  const int half = d >> 1, tid = threadIdx.x;
  const int row0 = blockIdx.x * R, nrows = min(R, M - row0);
  // this block's partial sums: dtheta [K][half], then ds [d] (with a scale)
  float* pth = part + (size_t)blockIdx.x * ((size_t)K * half + (scale ? d : 0));
  float* psc = pth + (size_t)K * half;

  // rows (bf16) -> fp32 planes; rows past M are zero
  for (int c = tid; c < d; c += kBwdThreads)
#pragma unroll
    for (int r = 0; r < R; ++r)
      xs[(size_t)r * d + c] =
          r < nrows ? __uint_as_float((uint32_t)x[(size_t)(row0 + r) * d + c] << 16) : 0.f;
  __syncthreads();

  auto pair_of = [&](int k, int t, int& i, int& j) -> bool {
    const uint32_t pr = __ldg(pairs + (size_t)k * half + t);
    i = (int)(pr & 0xFFFFu);
    j = (int)(pr >> 16);
    if (i < d && j < d) return true;
    report_status(status, kStatusBadIndex);
    return false;
  };
  // forward: x' = R_K ... R_1 x
#pragma unroll 1
  for (int k = 0; k < K; ++k) {
    for (int t = tid; t < half; t += kBwdThreads) {
      int i, j;
      if (!pair_of(k, t, i, j)) continue;
      const float c = __ldg(cos_t + (size_t)k * half + t), s = __ldg(sin_t + (size_t)k * half + t);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float a = xs[(size_t)r * d + i], b = xs[(size_t)r * d + j];
        xs[(size_t)r * d + i] = fmaf(c, a, s * b);
        xs[(size_t)r * d + j] = fmaf(-s, a, c * b);
      }
    }
    __syncthreads();
  }
  // scale step: h = G / s, ds partial = -sum_r G (x'/s) / s
  for (int c = tid; c < d; c += kBwdThreads) {
    const float sc = scale ? __ldg(scale + c) : 1.f;
    float acc = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float g = r < nrows ? __ldg(grad + (size_t)(row0 + r) * d + c) : 0.f;
      if (scale) {
        const float xt = xs[(size_t)r * d + c] / sc;
        acc = fmaf(-g, xt / sc, acc);
        hs[(size_t)r * d + c] = g / sc;
      } else {
        hs[(size_t)r * d + c] = g;
      }
    }
    if (scale) psc[c] = acc;
  }
  __syncthreads();
  // backward through the stages, last first
#pragma unroll 1
  for (int k = K - 1; k >= 0; --k) {
    for (int t = tid; t < half; t += kBwdThreads) {
      int i, j;
      float dt = 0.f;
      if (pair_of(k, t, i, j)) {
        const float c = __ldg(cos_t + (size_t)k * half + t), s = __ldg(sin_t + (size_t)k * half + t);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const float xi = xs[(size_t)r * d + i], xj = xs[(size_t)r * d + j];
          const float hi = hs[(size_t)r * d + i], hj = hs[(size_t)r * d + j];
          dt = fmaf(hi, xj, fmaf(-hj, xi, dt));
          hs[(size_t)r * d + i] = fmaf(c, hi, -s * hj);
          hs[(size_t)r * d + j] = fmaf(s, hi, c * hj);
          xs[(size_t)r * d + i] = fmaf(c, xi, -s * xj);
          xs[(size_t)r * d + j] = fmaf(s, xi, c * xj);
        }
      }
      pth[(size_t)k * half + t] = dt;
    }
    __syncthreads();
  }
  // dL/dx of the block's rows
  for (int c = tid; c < d; c += kBwdThreads)
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (r < nrows) dx[(size_t)(row0 + r) * d + c] = hs[(size_t)r * d + c];
}

// out[e] = sum over blocks b (in order) of part[b][e]; e < K half go to dtheta,
// the rest (with a scale) to ds
__global__ void rot_bwd_reduce_kernel(const float* __restrict__ part, int blocks, int K, int half, int d,
                                      int with_scale, float* __restrict__ dtheta, float* __restrict__ dscale) {
  const size_t n = (size_t)K * half + (with_scale ? d : 0);
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
    float acc = 0.f;
    for (int b = 0; b < blocks; ++b) acc += part[(size_t)b * n + e];
    if (e < (size_t)K * half) dtheta[e] = acc;
    else dscale[e - (size_t)K * half] = acc;
  }
}

}  // namespace

int rot_bwd_rows(int d) {
  for (int R = 4; R >= 1; R >>= 1)
    if (bwd_smem(d, R) <= kBwdSmemBudget) return R;
  return 0;
}

size_t rot_bwd_workspace_bytes(int M, int d, int K, bool with_scale) {
  const int R = rot_bwd_rows(d);
  if (R == 0 || M <= 0) return 0;
  const size_t blocks = ((size_t)M + R - 1) / R;
  return blocks * ((size_t)K * (d / 2) + (with_scale ? (size_t)d : 0)) * sizeof(float);
}

cudaError_t launch_rot_backward(const uint16_t* x, const float* grad, int M, int d, int K, const uint32_t* pairs,
                                const float* cos_t, const float* sin_t, const float* scale, float* dx, float* dtheta,
                                float* dscale, void* ws, int* status, cudaStream_t stream) {
  const int R = rot_bwd_rows(d);
  if (R == 0) return cudaErrorInvalidValue;
  const int blocks = (M + R - 1) / R;
  const size_t smem = bwd_smem(d, R);
  float* part = static_cast<float*>(ws);
  cudaError_t e;
#define PARO_BWD_LAUNCH(r)                                                                              \
  {                                                                                                     \
    e = cudaFuncSetAttribute(rot_bwd_kernel<r>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
    if (e != cudaSuccess) return e;                                                                     \
    rot_bwd_kernel<r><<<blocks, kBwdThreads, smem, stream>>>(x, grad, M, d, K, pairs, cos_t, sin_t, scale, dx, \
                                                             part, status);                            \
  }
  if (R == 4) PARO_BWD_LAUNCH(4) else if (R == 2) PARO_BWD_LAUNCH(2) else PARO_BWD_LAUNCH(1)
#undef PARO_BWD_LAUNCH
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t n = (size_t)K * (d / 2) + (scale ? d : 0);
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  const int grid = (int)((n + threads - 1) / threads < 4096 ? (n + threads - 1) / threads : 4096);
  rot_bwd_reduce_kernel<<<grid, threads, 0, stream>>>(part, blocks, K, d / 2, d, scale ? 1 : 0, dtheta, dscale);
  return cudaGetLastError();
}

}  // namespace paro
