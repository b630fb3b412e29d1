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
// the workspace; rot_bwd_reduce_kernel adds them over the blocks in a fixed
// order (deterministic), and dL/dx is written by the block itself.
#include "paro_internal.cuh"

namespace paro {
namespace {

constexpr size_t kBwdSmemBudget = 227 * 1024 - 1024;

// shared memory: the rows and their gradients (8 R d bytes) and NB stage
// tables (pairs, cos, sin: 6 d bytes each)
size_t bwd_smem(int d, int R, int NB) { return (size_t)8 * R * d + (size_t)NB * 6 * d; }

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}

template <int R> struct Vec;
template <> struct Vec<1> { using T = float; };
template <> struct Vec<2> { using T = float2; };
template <> struct Vec<4> { using T = float4; };
__device__ __forceinline__ float& el(float& v, int) { return v; }
__device__ __forceinline__ float& el(float2& v, int r) { return r == 0 ? v.x : v.y; }
__device__ __forceinline__ float& el(float4& v, int r) { return r == 0 ? v.x : (r == 1 ? v.y : (r == 2 ? v.z : v.w)); }

// NB > 0: the tables of the stage steps (forward k = 0 .. K-1, then backward
// k = K-1 .. 0) are copied into a ring of NB shared-memory buffers (cp.async,
// 16 bytes a thread and copy), NB - 1 steps ahead of their use; NB = 0: every
// pair reads its table entries from global memory.  NTH threads a CTA.
template <int R, int NB, int NTH>
__global__ void __launch_bounds__(NTH)
rot_bwd_kernel(const uint16_t* __restrict__ x, const float* __restrict__ grad, int M, int d, int K,
               const uint32_t* __restrict__ pairs, const float* __restrict__ cos_t, const float* __restrict__ sin_t,
               const float* __restrict__ scale, float* __restrict__ dx, float* __restrict__ part, int* status) {
  using VT = typename Vec<R>::T;
  extern __shared__ __align__(16) float sm[];
  // channel-major: channel c of the R rows is one VT, so a pair moves its two
  // channels of x and of h with four vector loads and four vector stores
  VT* xs = reinterpret_cast<VT*>(sm);                 // [d] x R
  VT* hs = reinterpret_cast<VT*>(sm + (size_t)R * d);  // [d] x R
  float* tb = sm + (size_t)2 * R * d;  // NB x (pairs [half] | cos [half] | sin [half])
  constexpr bool STAGED = NB > 0;
  const int half = d >> 1, tid = threadIdx.x;
  const int row0 = blockIdx.x * R, nrows = min(R, M - row0);
  // this block's partial sums: dtheta [K][half], then ds [d] (with a scale)
  float* pth = part + (size_t)blockIdx.x * ((size_t)K * half + (scale ? d : 0));
  float* psc = pth + (size_t)K * half;

  // rows (bf16) -> fp32, channel-major; rows past M are zero
  for (int c = tid; c < d; c += NTH) {
    VT v;
#pragma unroll
    for (int r = 0; r < R; ++r)
      el(v, r) = r < nrows ? __uint_as_float((uint32_t)x[(size_t)(row0 + r) * d + c] << 16) : 0.f;
    xs[c] = v;
  }
  __syncthreads();

  // table step q (0 .. 2K-1) is stage q (forward) or 2K-1-q (backward)
  auto stage_of = [&](int q) { return q < K ? q : 2 * K - 1 - q; };
  auto stage_copy = [&](int q) {  // step q's table into buffer q % NB
    if constexpr (STAGED) {
      if (q < 2 * K) {
        const int k = stage_of(q);
        float* dst = tb + (size_t)(q % (NB > 0 ? NB : 1)) * 3 * half;
        const int chunks = half / 4;  // 16-byte pieces of each of the three arrays
        for (int u = tid; u < 3 * chunks; u += NTH) {
          const int a = u / chunks, o = (u - a * chunks) * 4;
          const void* src = a == 0 ? (const void*)(pairs + (size_t)k * half + o)
                                   : (a == 1 ? (const void*)(cos_t + (size_t)k * half + o)
                                             : (const void*)(sin_t + (size_t)k * half + o));
          cp_async16(dst + (size_t)a * half + o, src);
        }
      }
      asm volatile("cp.async.commit_group;\n" ::: "memory");
    }
  };
  auto stage_ready = [&]() {  // the current step's copies have landed, for every thread
    if constexpr (STAGED) asm volatile("cp.async.wait_group %0;\n" ::"n"(NB > 0 ? NB - 1 : 0) : "memory");
    __syncthreads();
  };
  // the pair and angle of pair t in table step q
  auto pair_of = [&](int q, int t, int& i, int& j, float& c, float& s) -> bool {
    uint32_t pr;
    if constexpr (STAGED) {
      const float* b = tb + (size_t)(q % (NB > 0 ? NB : 1)) * 3 * half;
      pr = __float_as_uint(b[t]);
      c = b[half + t];
      s = b[2 * half + t];
    } else {
      const int k = stage_of(q);
      pr = __ldg(pairs + (size_t)k * half + t);
      c = __ldg(cos_t + (size_t)k * half + t);
      s = __ldg(sin_t + (size_t)k * half + t);
    }
    i = (int)(pr & 0xFFFFu);
    j = (int)(pr >> 16);
    if (i < d && j < d) return true;
    report_status(status, kStatusBadIndex);
    return false;
  };
#pragma unroll
  for (int q = 0; q + 1 < NB; ++q) stage_copy(q);
  // forward: x' = R_K ... R_1 x
#pragma unroll 1
  for (int k = 0; k < K; ++k) {
    stage_copy(k + NB - 1);
    stage_ready();
    for (int t = tid; t < half; t += NTH) {
      int i, j;
      float c, s;
      if (!pair_of(k, t, i, j, c, s)) continue;
      VT a = xs[i], b = xs[j], na, nb;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        el(na, r) = fmaf(c, el(a, r), s * el(b, r));
        el(nb, r) = fmaf(-s, el(a, r), c * el(b, r));
      }
      xs[i] = na;
      xs[j] = nb;
    }
    __syncthreads();
  }
  // scale step: h = G / s, ds partial = -sum_r G (x'/s) / s
  for (int c = tid; c < d; c += NTH) {
    const float sc = scale ? __ldg(scale + c) : 1.f;
    const VT xv = xs[c];
    VT hv;
    float acc = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float g = r < nrows ? __ldg(grad + (size_t)(row0 + r) * d + c) : 0.f;
      if (scale) {
        const float xt = el(const_cast<VT&>(xv), r) / sc;
        acc = fmaf(-g, xt / sc, acc);
        el(hv, r) = g / sc;
      } else {
        el(hv, r) = g;
      }
    }
    hs[c] = hv;
    if (scale) psc[c] = acc;
  }
  __syncthreads();
  // backward through the stages, last first
#pragma unroll 1
  for (int k = K - 1; k >= 0; --k) {
    const int q = 2 * K - 1 - k;  // table step
    stage_copy(q + NB - 1);
    stage_ready();
    for (int t = tid; t < half; t += NTH) {
      int i, j;
      float dt = 0.f, c, s;
      if (pair_of(q, t, i, j, c, s)) {
        VT xi = xs[i], xj = xs[j], hi = hs[i], hj = hs[j], nxi, nxj, nhi, nhj;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          dt = fmaf(el(hi, r), el(xj, r), fmaf(-el(hj, r), el(xi, r), dt));
          el(nhi, r) = fmaf(c, el(hi, r), -s * el(hj, r));
          el(nhj, r) = fmaf(s, el(hi, r), c * el(hj, r));
          el(nxi, r) = fmaf(c, el(xi, r), -s * el(xj, r));
          el(nxj, r) = fmaf(s, el(xi, r), c * el(xj, r));
        }
        hs[i] = nhi;
        hs[j] = nhj;
        xs[i] = nxi;
        xs[j] = nxj;
      }
      pth[(size_t)k * half + t] = dt;
    }
    __syncthreads();
  }
  // dL/dx of the block's rows
  for (int c = tid; c < d; c += NTH) {
    VT hv = hs[c];
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (r < nrows) dx[(size_t)(row0 + r) * d + c] = el(hv, r);
  }
}

// out[e] = sum over blocks b of part[b][e], in a fixed order.  A CTA of 32 x 32
// threads takes 32 consecutive outputs (threadIdx.x, coalesced) and cuts the
// blocks into 32 contiguous ranges (threadIdx.y); the range sums are then added
// in range order.  e < K half go to dtheta, the rest (with a scale) to ds.
__global__ void __launch_bounds__(1024)
rot_bwd_reduce_kernel(const float* __restrict__ part, int blocks, int K, int half, int d, int with_scale,
                      float* __restrict__ dtheta, float* __restrict__ dscale) {
  __shared__ float sums[32][33];
  const size_t n = (size_t)K * half + (with_scale ? d : 0);
  const size_t e = blockIdx.x * (size_t)32 + threadIdx.x;
  const int b0 = (int)((long long)threadIdx.y * blocks / 32), b1 = (int)((long long)(threadIdx.y + 1) * blocks / 32);
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;  // four running sums, blocks b = q (mod 4) of the range
  if (e < n) {
    int b = b0;
#pragma unroll 1
    for (; b + 4 <= b1; b += 4) {
      a0 += part[(size_t)b * n + e];
      a1 += part[(size_t)(b + 1) * n + e];
      a2 += part[(size_t)(b + 2) * n + e];
      a3 += part[(size_t)(b + 3) * n + e];
    }
    if (b < b1) a0 += part[(size_t)b * n + e];
    if (b + 1 < b1) a1 += part[(size_t)(b + 1) * n + e];
    if (b + 2 < b1) a2 += part[(size_t)(b + 2) * n + e];
  }
  sums[threadIdx.y][threadIdx.x] = (a0 + a1) + (a2 + a3);
  __syncthreads();
  if (threadIdx.y == 0 && e < n) {
    float t = 0.f;
#pragma unroll 1
    for (int y = 0; y < 32; ++y) t += sums[y][threadIdx.x];
    if (e < (size_t)K * half) dtheta[e] = t;
    else dscale[e - (size_t)K * half] = t;
  }
}

}  // namespace

namespace {
// Launch shape for width d: rows a CTA, table buffers, threads.  Two CTAs of
// 512 threads an SM when their rows and two tables fit in half the shared
// memory (each covers the other's table latency); else one CTA of 1024 threads
// with up to four rows and as many table buffers as fit (three: the copies run
// two steps ahead); the widest rows read their tables from global memory.
struct BwdPlan {
  int R, NB, NTH;
};
BwdPlan bwd_plan(int d) {
  const bool al = d % 8 == 0;
  for (int R = 4; R >= 1; R >>= 1)
    if (al && 2 * bwd_smem(d, R, 2) + 2048 <= kBwdSmemBudget) return {R, 2, 512};
  for (int R = 4; R >= 1; R >>= 1) {
    if (al && bwd_smem(d, R, 3) <= kBwdSmemBudget) return {R, 3, 1024};
    if (al && bwd_smem(d, R, 2) <= kBwdSmemBudget) return {R, 2, 1024};
    if (bwd_smem(d, R, 0) <= kBwdSmemBudget) return {R, 0, 1024};
  }
  return {0, 0, 0};
}
}  // namespace

int rot_bwd_rows(int d) { return bwd_plan(d).R; }

size_t rot_bwd_workspace_bytes(int M, int d, int K, bool with_scale) {
  const int R = rot_bwd_rows(d);
  if (R == 0 || M <= 0) return 0;
  const size_t blocks = ((size_t)M + R - 1) / R;
  return blocks * ((size_t)K * (d / 2) + (with_scale ? (size_t)d : 0)) * sizeof(float);
}

cudaError_t launch_rot_backward(const uint16_t* x, const float* grad, int M, int d, int K, const uint32_t* pairs,
                                const float* cos_t, const float* sin_t, const float* scale, float* dx, float* dtheta,
                                float* dscale, void* ws, int* status, cudaStream_t stream) {
  BwdPlan pl = bwd_plan(d);
  if (pl.R == 0) return cudaErrorInvalidValue;
  if (pl.NB > 0 && K > 0 &&
      ((reinterpret_cast<uintptr_t>(pairs) | reinterpret_cast<uintptr_t>(cos_t) | reinterpret_cast<uintptr_t>(sin_t)) &
       15) != 0) {
    pl.NB = 0;  // the tables are copied in 16-byte pieces
    pl.NTH = 1024;
  }
  const int blocks = (M + pl.R - 1) / pl.R;
  const size_t smem = bwd_smem(d, pl.R, pl.NB);
  float* part = static_cast<float*>(ws);
  cudaError_t e = cudaErrorInvalidValue;
#define PARO_BWD_LAUNCH(r, nb, nth)                                                                             \
  if (pl.R == r && pl.NB == nb && pl.NTH == nth) {                                                              \
    e = cudaFuncSetAttribute(rot_bwd_kernel<r, nb, nth>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
    if (e != cudaSuccess) return e;                                                                             \
    rot_bwd_kernel<r, nb, nth><<<blocks, nth, smem, stream>>>(x, grad, M, d, K, pairs, cos_t, sin_t, scale, dx,   \
                                                              part, status);                                    \
    e = cudaGetLastError();                                                                                     \
  }
  PARO_BWD_LAUNCH(4, 2, 512)
  PARO_BWD_LAUNCH(2, 2, 512)
  PARO_BWD_LAUNCH(1, 2, 512)
  PARO_BWD_LAUNCH(4, 3, 1024)
  PARO_BWD_LAUNCH(2, 3, 1024)
  PARO_BWD_LAUNCH(1, 3, 1024)
  PARO_BWD_LAUNCH(4, 2, 1024)
  PARO_BWD_LAUNCH(2, 2, 1024)
  PARO_BWD_LAUNCH(1, 2, 1024)
  PARO_BWD_LAUNCH(4, 0, 1024)
  PARO_BWD_LAUNCH(2, 0, 1024)
  PARO_BWD_LAUNCH(1, 0, 1024)
#undef PARO_BWD_LAUNCH
  if (e != cudaSuccess) return e;
  const size_t n = (size_t)K * (d / 2) + (scale ? d : 0);
  if (n == 0) return cudaSuccess;
  rot_bwd_reduce_kernel<<<(unsigned)((n + 31) / 32), dim3(32, 32), 0, stream>>>(part, blocks, K, d / 2, d,
                                                                               scale ? 1 : 0, dtheta, dscale);
  return cudaGetLastError();
}

}  // namespace paro
