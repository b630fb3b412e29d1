// Givens-stage transform kernels: the activation-side transform
//   x~ = diag(1/s) R_K ... R_1 x                       (runtime, per token row)
// and the build-time weight fold
//   w~ = diag(s)   R_K ... R_1 w                       (per output row of W)
// Page "ParoQuant: pairwise rotations that survive deployment", section "A
// rotation small enough to execute": a stage rotates disjoint channel pairs
// (i, j) with x_i' = c x_i + s x_j, x_j' = -s x_i + c x_j, so every pair of a
// stage can be updated in parallel without write conflicts.
//
// One CTA owns R whole rows.  It stages them in shared memory as fp32, one
// plane per row (channel c of every row in bank c % 32, so pair tables ordered
// by paro_plan_pair_order make every access of a warp conflict-free),
// applies all K stages there with a barrier between stages, and writes the
// result once.  HBM sees one read and one write of the rows; the pair and
// cos/sin tables stream from L2, each thread fetching its entries of the next
// stage while it works on the current one.
#include "paro_internal.cuh"

namespace paro {
namespace {

enum Mode { kActBf16 = 0, kActF16 = 1, kFoldF32 = 2 };

// UP: upper bound on the pairs (and channel pairs) one thread handles per stage.
template <int R, int MODE, int UP>
__global__ void __launch_bounds__(512, 2)
givens_rows_kernel(const void* __restrict__ in, void* __restrict__ out, int M, int d, int K,
                   const uint32_t* __restrict__ pairs, const float* __restrict__ cos_t,
                   const float* __restrict__ sin_t, const float* __restrict__ scale, int* status,
                   int pdl_trigger) {
  extern __shared__ __align__(16) float xs[];  // [R][d]
  if (pdl_trigger) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int row0 = blockIdx.x * R;
  const int nrows = min(R, M - row0);
  const int tid = threadIdx.x, nth = blockDim.x;
  const int half = d >> 1;

  // this thread's pairs of a stage: t = tid + u * nth, u < UP; their table
  // entries are fetched one stage ahead into registers
  uint32_t pr[UP];
  float cs[UP], sn[UP];
  auto fetch = [&](int k, uint32_t (&p)[UP], float (&c)[UP], float (&s_)[UP]) {
#pragma unroll
    for (int u = 0; u < UP; ++u) {
      const int t = tid + u * nth;
      if (k < K && t < half) {
        p[u] = __ldg(pairs + (size_t)k * half + t);
        c[u] = __ldg(cos_t + (size_t)k * half + t);
        s_[u] = __ldg(sin_t + (size_t)k * half + t);
      }
    }
  };
  fetch(0, pr, cs, sn);

  // ---- load: rows -> xs[r][c].  A thread issues the loads of four channel
  // pairs before their shared stores, so their latencies overlap.
#pragma unroll
  for (int u0 = 0; u0 < UP; u0 += 4) {
    float v0[4][R], v1[4][R];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int cp = tid + (u0 + q) * nth;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        v0[q][r] = 0.f; v1[q][r] = 0.f;
        if (u0 + q < UP && cp < half && r < nrows) {
          const size_t off = (size_t)(row0 + r) * d + 2 * cp;
          if constexpr (MODE == kFoldF32) {
            const float2 f = *reinterpret_cast<const float2*>(static_cast<const float*>(in) + off);
            v0[q][r] = f.x; v1[q][r] = f.y;
          } else {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(
                static_cast<const __nv_bfloat16*>(in) + off));
            v0[q][r] = f.x; v1[q][r] = f.y;
          }
        }
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int cp = tid + (u0 + q) * nth;
      if (u0 + q < UP && cp < half) {
#pragma unroll
        for (int r = 0; r < R; ++r)
          *reinterpret_cast<float2*>(xs + (size_t)r * d + 2 * cp) = make_float2(v0[q][r], v1[q][r]);
      }
    }
  }
  __syncthreads();

  // ---- K stages.  The pairs of a stage are disjoint, so a batch's loads may
  // all be issued before its stores.
  constexpr int B = R == 4 ? 2 : 4;
#pragma unroll 1
  for (int k = 0; k < K; ++k) {
    uint32_t npr[UP];
    float ncs[UP], nsn[UP];
    fetch(k + 1, npr, ncs, nsn);
#pragma unroll
    for (int u0 = 0; u0 < UP; u0 += B) {
      int ii[B], jj[B];
      float a[B][R], b[B][R];
#pragma unroll
      for (int q = 0; q < B; ++q) {
        const int u = u0 + q;
        ii[q] = -1;
        if (u < UP && tid + u * nth < half) {
          const int i = pr[u] & 0xFFFF, j = pr[u] >> 16;
          if (i < d && j < d) { ii[q] = i; jj[q] = j; }
          else report_status(status, kStatusBadIndex);
        }
      }
#pragma unroll
      for (int q = 0; q < B; ++q)
        if (ii[q] >= 0) {
#pragma unroll
          for (int r = 0; r < R; ++r) {
            a[q][r] = xs[(size_t)r * d + ii[q]];
            b[q][r] = xs[(size_t)r * d + jj[q]];
          }
        }
#pragma unroll
      for (int q = 0; q < B; ++q)
        if (ii[q] >= 0) {
          const float c = cs[u0 + q], s_ = sn[u0 + q];
          float na[R], nb[R];
#pragma unroll
          for (int r = 0; r < R; ++r) {
            na[r] = fmaf(c, a[q][r], s_ * b[q][r]);
            nb[r] = fmaf(-s_, a[q][r], c * b[q][r]);
          }
#pragma unroll
          for (int r = 0; r < R; ++r) {
            xs[(size_t)r * d + ii[q]] = na[r];
            xs[(size_t)r * d + jj[q]] = nb[r];
          }
        }
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < UP; ++u) { pr[u] = npr[u]; cs[u] = ncs[u]; sn[u] = nsn[u]; }
  }

  // ---- channel scale and store -------------------------------------------------
#pragma unroll
  for (int u = 0; u < UP; ++u) {
    const int cp = tid + u * nth;
    if (cp >= half) break;
    const int c = 2 * cp;
    float f0 = 1.0f, f1 = 1.0f;
    if (scale) {
      const float s0 = __ldg(scale + c), s1 = __ldg(scale + c + 1);
      if constexpr (MODE == kFoldF32) { f0 = s0; f1 = s1; }
      else { f0 = 1.0f / s0; f1 = 1.0f / s1; }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (r < nrows) {
        const float2 v = *reinterpret_cast<const float2*>(xs + (size_t)r * d + c);
        const size_t off = (size_t)(row0 + r) * d + c;
        const float a = v.x * f0, b = v.y * f1;
        if constexpr (MODE == kFoldF32) {
          *reinterpret_cast<float2*>(static_cast<float*>(out) + off) = make_float2(a, b);
        } else if constexpr (MODE == kActBf16) {
          *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(out) + off) = __floats2bfloat162_rn(a, b);
        } else {
          *reinterpret_cast<__half2*>(static_cast<__half*>(out) + off) = __floats2half2_rn(a, b);
        }
      }
    }
  }
}

// Plain variant for wide rows (more than 4 pairs per thread and stage):
// table entries are read when used.
template <int R, int MODE>
__global__ void __launch_bounds__(512)
givens_rows_simple(const void* __restrict__ in, void* __restrict__ out, int M, int d, int K,
                   const uint32_t* __restrict__ pairs, const float* __restrict__ cos_t,
                   const float* __restrict__ sin_t, const float* __restrict__ scale, int* status,
                   int pdl_trigger) {
  extern __shared__ __align__(16) float xs[];  // [R][d]
  if (pdl_trigger) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int row0 = blockIdx.x * R;
  const int nrows = min(R, M - row0);
  const int tid = threadIdx.x, nth = blockDim.x;

  // ---- load: rows -> xs[r][c] ------------------------------------------------
  // Each thread takes two adjacent channels of every row (4-byte bf16 pairs or
  // 8-byte fp32 pairs: a warp reads 128 or 256 contiguous bytes per row) and
  // writes the 2 x R values with vector stores to consecutive channel slots.
  const int npairs_ch = d >> 1;
  for (int cp = tid; cp < npairs_ch; cp += nth) {
    float v0[R], v1[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (r < nrows) {
        const size_t off = (size_t)(row0 + r) * d + 2 * cp;
        if constexpr (MODE == kFoldF32) {
          const float2 f = *reinterpret_cast<const float2*>(static_cast<const float*>(in) + off);
          v0[r] = f.x; v1[r] = f.y;
        } else {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(
              static_cast<const __nv_bfloat16*>(in) + off));
          v0[r] = f.x; v1[r] = f.y;
        }
      } else {
        v0[r] = 0.f; v1[r] = 0.f;
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) *reinterpret_cast<float2*>(xs + (size_t)r * d + 2 * cp) = make_float2(v0[r], v1[r]);
  }
  __syncthreads();

  // ---- K stages of disjoint pair rotations -------------------------------------
  const int half = d >> 1;
  for (int k = 0; k < K; ++k) {
    const uint32_t* pk = pairs + (size_t)k * half;
    const float* ck = cos_t + (size_t)k * half;
    const float* sk = sin_t + (size_t)k * half;
    for (int t = tid; t < half; t += nth) {
      const uint32_t pr = __ldg(pk + t);
      const int i = pr & 0xFFFF, j = pr >> 16;
      const float c = __ldg(ck + t), s = __ldg(sk + t);
      if (i >= d || j >= d) {
        report_status(status, kStatusBadIndex);
        continue;
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float a = xs[(size_t)r * d + i], b = xs[(size_t)r * d + j];
        xs[(size_t)r * d + i] = fmaf(c, a, s * b);
        xs[(size_t)r * d + j] = fmaf(-s, a, c * b);
      }
    }
    __syncthreads();
  }

  // ---- channel scale and store -------------------------------------------------
  for (int cp = tid; cp < npairs_ch; cp += nth) {
    const int c = 2 * cp;
    float f0 = 1.0f, f1 = 1.0f;
    if (scale) {
      const float s0 = __ldg(scale + c), s1 = __ldg(scale + c + 1);
      if constexpr (MODE == kFoldF32) { f0 = s0; f1 = s1; }
      else { f0 = 1.0f / s0; f1 = 1.0f / s1; }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (r < nrows) {
        const float2 v = *reinterpret_cast<const float2*>(xs + (size_t)r * d + c);
        const size_t off = (size_t)(row0 + r) * d + c;
        const float a = v.x * f0, b = v.y * f1;
        if constexpr (MODE == kFoldF32) {
          *reinterpret_cast<float2*>(static_cast<float*>(out) + off) = make_float2(a, b);
        } else if constexpr (MODE == kActBf16) {
          *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(out) + off) = __floats2bfloat162_rn(a, b);
        } else {
          *reinterpret_cast<__half2*>(static_cast<__half*>(out) + off) = __floats2half2_rn(a, b);
        }
      }
    }
  }
}

int pick_rows_per_cta(int M, int d) {
  int R = 1;
  if (d <= 6144) R = 4;
  else if (d <= 12288) R = 2;
  while (R > 1 && R > M) R >>= 1;
  return R;
}

template <int MODE, int R, int UP>
cudaError_t launch_rup(const void* in, void* out, int M, int d, int K, const uint32_t* p32, const float* cos_t,
                       const float* sin_t, const float* scale, int* status, cudaStream_t stream, int trig) {
  const size_t smem = (size_t)R * d * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(givens_rows_kernel<R, MODE, UP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  givens_rows_kernel<R, MODE, UP><<<(M + R - 1) / R, 512, smem, stream>>>(in, out, M, d, K, p32, cos_t, sin_t, scale,
                                                                          status, trig);
  return cudaPeekAtLastError();
}

template <int MODE, int R>
cudaError_t launch_r(const void* in, void* out, int M, int d, int K, const uint32_t* p32, const float* cos_t,
                     const float* sin_t, const float* scale, int* status, cudaStream_t stream, int trig) {
  const int per = (d / 2 + 511) / 512;  // pairs per thread and stage
  if (per <= 1) return launch_rup<MODE, R, 1>(in, out, M, d, K, p32, cos_t, sin_t, scale, status, stream, trig);
  if (per <= 2) return launch_rup<MODE, R, 2>(in, out, M, d, K, p32, cos_t, sin_t, scale, status, stream, trig);
  if (per <= 4) return launch_rup<MODE, R, 4>(in, out, M, d, K, p32, cos_t, sin_t, scale, status, stream, trig);
  // wider rows: the register prefetch would spill at two CTAs per SM; read the tables when used
  const int threads = d >= 2048 ? 512 : 256;
  const size_t smem = (size_t)R * d * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(givens_rows_simple<R, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  givens_rows_simple<R, MODE><<<(M + R - 1) / R, threads, smem, stream>>>(in, out, M, d, K, p32, cos_t, sin_t,
                                                                          scale, status, trig);
  return cudaPeekAtLastError();
}

template <int MODE>
cudaError_t launch_givens(const void* in, void* out, int M, int d, int K, const uint16_t* pairs,
                          const float* cos_t, const float* sin_t, const float* scale, int* status,
                          cudaStream_t stream, bool pdl_trigger) {
  const int R = pick_rows_per_cta(M, d);
  const uint32_t* p32 = reinterpret_cast<const uint32_t*>(pairs);
  const int trig = pdl_trigger ? 1 : 0;
  if (R == 4) return launch_r<MODE, 4>(in, out, M, d, K, p32, cos_t, sin_t, scale, status, stream, trig);
  if (R == 2) return launch_r<MODE, 2>(in, out, M, d, K, p32, cos_t, sin_t, scale, status, stream, trig);
  return launch_r<MODE, 1>(in, out, M, d, K, p32, cos_t, sin_t, scale, status, stream, trig);
}

}  // namespace

cudaError_t launch_rotate_act(const uint16_t* x, void* out, int out_is_f16, int M, int d, int K,
                              const uint16_t* pairs, const float* cos_t, const float* sin_t,
                              const float* scale, int* status, cudaStream_t stream, bool pdl_trigger) {
  if (out_is_f16)
    return launch_givens<kActF16>(x, out, M, d, K, pairs, cos_t, sin_t, scale, status, stream, pdl_trigger);
  return launch_givens<kActBf16>(x, out, M, d, K, pairs, cos_t, sin_t, scale, status, stream, pdl_trigger);
}

cudaError_t launch_fold_weights(const float* W, float* out, int rows, int d, int K,
                                const uint16_t* pairs, const float* cos_t, const float* sin_t,
                                const float* scale, int* status, cudaStream_t stream) {
  return launch_givens<kFoldF32>(W, out, rows, d, K, pairs, cos_t, sin_t, scale, status, stream, false);
}

}  // namespace paro
