// Givens-stage transform kernels: the activation-side transform
//   x~ = diag(1/s) R_K ... R_1 x                       (runtime, per token row)
// and the build-time weight fold
//   w~ = diag(s)   R_K ... R_1 w                       (per output row of W)
// Page "ParoQuant: pairwise rotations that survive deployment", section "A
// rotation small enough to execute": a stage rotates disjoint channel pairs
// (i, j) with x_i' = c x_i + s x_j, x_j' = -s x_i + c x_j, so every pair of a
// stage can be updated in parallel without write conflicts.
//
// One CTA owns R whole rows.  It stages them in shared memory as fp32 with
// the R values of a channel side by side, applies all K stages there with a
// barrier between stages, and writes the result once.  HBM sees one read and
// one write of the rows; the pair and cos/sin tables stream from L2, each
// thread fetching its entries of the next stage while it works on the
// current one.
#include "paro_internal.cuh"

namespace paro {
namespace {

enum Mode { kActBf16 = 0, kActF16 = 1, kFoldF32 = 2 };

template <int R> struct VecT;
template <> struct VecT<1> { using T = float; };
template <> struct VecT<2> { using T = float2; };
template <> struct VecT<4> { using T = float4; };

__device__ __forceinline__ float vget(const float& v, int) { return v; }
__device__ __forceinline__ float vget(const float2& v, int r) { return r == 0 ? v.x : v.y; }
__device__ __forceinline__ float vget(const float4& v, int r) { return r == 0 ? v.x : r == 1 ? v.y : r == 2 ? v.z : v.w; }
__device__ __forceinline__ void vset(float& v, int, float x) { v = x; }
__device__ __forceinline__ void vset(float2& v, int r, float x) { if (r == 0) v.x = x; else v.y = x; }
__device__ __forceinline__ void vset(float4& v, int r, float x) {
  if (r == 0) v.x = x; else if (r == 1) v.y = x; else if (r == 2) v.z = x; else v.w = x;
}

// Packed pairs of fp32 (sm_100 f32x2 arithmetic: two IEEE operations per
// instruction, each rounded exactly like its scalar form).
__device__ __forceinline__ uint64_t pk2(float x, float y) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(x), "f"(y));
  return r;
}
__device__ __forceinline__ void up2(uint64_t v, float& x, float& y) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(x), "=f"(y) : "l"(v));
}
// (x, y) rows of channels i and j: x' = c x + s y, y' = -s x + c y, as
// fmaf(c, x, s * y) and fmaf(-s, x, c * y) elementwise
__device__ __forceinline__ void rot2(uint64_t& x, uint64_t& y, uint64_t c2, uint64_t s2, uint64_t ns2) {
  uint64_t sy, cy, nx, ny;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(sy) : "l"(s2), "l"(y));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(cy) : "l"(c2), "l"(y));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(nx) : "l"(c2), "l"(x), "l"(sy));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(ny) : "l"(ns2), "l"(x), "l"(cy));
  x = nx;
  y = ny;
}

// One pair of one stage on R rows at once: a = channel i, b = channel j.
__device__ __forceinline__ void rotate_pair(float& a, float& b, float c, float s) {
  const float x = a, y = b;
  a = fmaf(c, x, s * y);
  b = fmaf(-s, x, c * y);
}
__device__ __forceinline__ void rotate_pair(float2& a, float2& b, float c, float s) {
  uint64_t x = pk2(a.x, a.y), y = pk2(b.x, b.y);
  rot2(x, y, pk2(c, c), pk2(s, s), pk2(-s, -s));
  up2(x, a.x, a.y);
  up2(y, b.x, b.y);
}
__device__ __forceinline__ void rotate_pair(float4& a, float4& b, float c, float s) {
  const uint64_t c2 = pk2(c, c), s2 = pk2(s, s), ns2 = pk2(-s, -s);
  uint64_t x0 = pk2(a.x, a.y), y0 = pk2(b.x, b.y), x1 = pk2(a.z, a.w), y1 = pk2(b.z, b.w);
  rot2(x0, y0, c2, s2, ns2);
  rot2(x1, y1, c2, s2, ns2);
  up2(x0, a.x, a.y);
  up2(x1, a.z, a.w);
  up2(y0, b.x, b.y);
  up2(y1, b.z, b.w);
}

// Channel-major transform kernel.  One CTA owns R whole rows (R = 1, 2 or 4)
// and keeps them in shared memory with the R values of a channel side by side
// (one float, float2 or float4 per channel), so a pair of a stage costs two
// vector loads and two vector stores for all R rows.  A warp's 32 lanes take
// 32 consecutive pairs; with tables ordered by paro_plan_pair_order every
// phase of those vector accesses (8 lanes for float4, 16 for float2, 32 for
// float) touches distinct banks.  UP > 0: every thread handles at most UP
// pairs per stage and fetches their table entries one stage ahead into
// registers; UP == 0: any width, table entries read when used.
template <int R, int MODE, int UP, int NTH>
__global__ void __launch_bounds__(NTH, NTH <= 512 ? 2 : 1)
givens_cm_kernel(const void* __restrict__ in, void* __restrict__ out, int M, int d, int K,
                 const uint32_t* __restrict__ pairs, const float* __restrict__ cos_t,
                 const float* __restrict__ sin_t, const float* __restrict__ scale, int* status,
                 int pdl_trigger) {
  using V = typename VecT<R>::T;
  extern __shared__ __align__(16) unsigned char smem_cm[];
  V* xs = reinterpret_cast<V*>(smem_cm);  // [d + 2] channels, R rows each (d, d + 1 spare)
  if (pdl_trigger) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int row0 = blockIdx.x * R;
  const int nrows = min(R, M - row0);
  const int tid = threadIdx.x;
  const int half = d >> 1;

  constexpr int UPR = UP > 0 ? UP : 1;
  // pair slots of this thread (the same in every stage) and its table pointers
  bool valid[UPR];
#pragma unroll
  for (int u = 0; u < UPR; ++u) valid[u] = UP > 0 && tid + u * NTH < half;
  const uint32_t* pk = pairs + tid;
  const float* ck = cos_t + tid;
  const float* sk = sin_t + tid;
  uint32_t pr[UPR];
  float cs[UPR], sn[UPR];
  auto fetch = [&](uint32_t (&p)[UPR], float (&c)[UPR], float (&s_)[UPR]) {
#pragma unroll
    for (int u = 0; u < UPR; ++u)
      if (valid[u]) {
        p[u] = __ldg(pk + u * NTH);
        c[u] = __ldg(ck + u * NTH);
        s_[u] = __ldg(sk + u * NTH);
      }
  };
  if (K > 0) fetch(pr, cs, sn);

  // ---- load: two adjacent channels of every row per thread (a warp reads 128
  // or 256 contiguous bytes of each row), stored as two channel vectors.  The
  // loads of LB consecutive channel pairs are issued before their stores, so
  // their DRAM latencies overlap.
  constexpr int LB = MODE == kFoldF32 ? 2 : 4;
#pragma unroll 1
  for (int cp0 = tid; cp0 < half; cp0 += LB * NTH) {
    float2 f[LB][R];
#pragma unroll
    for (int q = 0; q < LB; ++q) {
      const int cp = cp0 + q * NTH;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        f[q][r] = make_float2(0.f, 0.f);
        if (cp < half && r < nrows) {
          const size_t off = (size_t)(row0 + r) * d + 2 * cp;
          if constexpr (MODE == kFoldF32) {
            f[q][r] = __ldg(reinterpret_cast<const float2*>(static_cast<const float*>(in) + off));
          } else {
            f[q][r] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(
                static_cast<const __nv_bfloat16*>(in) + off));
          }
        }
      }
    }
#pragma unroll
    for (int q = 0; q < LB; ++q) {
      const int cp = cp0 + q * NTH;
      if (cp < half) {
        V v0, v1;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          vset(v0, r, f[q][r].x);
          vset(v1, r, f[q][r].y);
        }
        xs[2 * cp] = v0;
        xs[2 * cp + 1] = v1;
      }
    }
  }
  __syncthreads();

  // ---- K stages.  The pairs of a stage are disjoint: all loads of a thread's
  // pairs are issued before any of its stores.
  bool bad = false;
#pragma unroll 1
  for (int k = 0; k < K; ++k) {
    if constexpr (UP > 0) {
      uint32_t npr[UPR];
      float ncs[UPR], nsn[UPR];
      if (k + 1 < K) {
        pk += half;
        ck += half;
        sk += half;
        fetch(npr, ncs, nsn);
      }
      // CH pairs at a time keep the row vectors' registers few.  A slot
      // without a pair, or a pair with an index >= d, reads and writes the two
      // spare channels d and d + 1 instead (nothing else reads them).
      constexpr int CH = (R == 4 || UP >= 7) ? 2 : (UP < 4 ? UP : 4);
#pragma unroll
      for (int u0 = 0; u0 < UPR; u0 += CH) {
        int ii[CH], jj[CH];
        V a[CH], b[CH];
#pragma unroll
        for (int q = 0; q < CH; ++q) {
          const int u = u0 + q;
          if (u < UPR) {
            const int i = pr[u] & 0xFFFF, j = pr[u] >> 16;
            const bool in_range = i < d && j < d;
            bad |= valid[u] && !in_range;
            const bool use = valid[u] && in_range;
            ii[q] = use ? i : d;
            jj[q] = use ? j : d + 1;
            a[q] = xs[ii[q]];
            b[q] = xs[jj[q]];
          }
        }
#pragma unroll
        for (int q = 0; q < CH; ++q)
          if (u0 + q < UPR) {
            rotate_pair(a[q], b[q], cs[u0 + q], sn[u0 + q]);
            xs[ii[q]] = a[q];
            xs[jj[q]] = b[q];
          }
      }
      __syncthreads();
#pragma unroll
      for (int u = 0; u < UPR; ++u) { pr[u] = npr[u]; cs[u] = ncs[u]; sn[u] = nsn[u]; }
    } else {
      const uint32_t* pk0 = pairs + (size_t)k * half;
      const float* ck0 = cos_t + (size_t)k * half;
      const float* sk0 = sin_t + (size_t)k * half;
#pragma unroll 1
      for (int t = tid; t < half; t += NTH) {
        const uint32_t p = __ldg(pk0 + t);
        const int i = p & 0xFFFF, j = p >> 16;
        const float c = __ldg(ck0 + t), s_ = __ldg(sk0 + t);
        if (i >= d || j >= d) {
          bad = true;
          continue;
        }
        V a = xs[i], b = xs[j];
        rotate_pair(a, b, c, s_);
        xs[i] = a;
        xs[j] = b;
      }
      __syncthreads();
    }
  }

  if (bad) report_status(status, kStatusBadIndex);

  // ---- channel scale and store (an fp16 value that rounds to infinity is
  // reported once: PARO_ERR_RANGE) ------------------------------------------------
  bool ovf = false;
#pragma unroll 1
  for (int cp = tid; cp < half; cp += NTH) {
    const int c = 2 * cp;
    float f0 = 1.0f, f1 = 1.0f;
    if (scale) {
      const float s0 = __ldg(scale + c), s1 = __ldg(scale + c + 1);
      if constexpr (MODE == kFoldF32) { f0 = s0; f1 = s1; }
      else { f0 = 1.0f / s0; f1 = 1.0f / s1; }
    }
    const V v0 = xs[c], v1 = xs[c + 1];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (r < nrows) {
        const size_t off = (size_t)(row0 + r) * d + c;
        const float a = vget(v0, r) * f0, b = vget(v1, r) * f1;
        if constexpr (MODE == kFoldF32) {
          *reinterpret_cast<float2*>(static_cast<float*>(out) + off) = make_float2(a, b);
        } else if constexpr (MODE == kActBf16) {
          *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(out) + off) = __floats2bfloat162_rn(a, b);
        } else {
          const __half2 h = __floats2half2_rn(a, b);
          ovf |= half2_inf(*reinterpret_cast<const uint32_t*>(&h));
          *reinterpret_cast<__half2*>(static_cast<__half*>(out) + off) = h;
        }
      }
    }
  }
  if (ovf) report_status(status, kStatusRange);
}

// Rows per CTA: the widest channel vector whose rows fit in shared memory
// (two CTAs per SM up to 6656 channels with four rows), never more than M.
int pick_rows_per_cta(int M, int d) {
  int R = 1;
  if (d <= 6656) R = 4;
  else if (d <= 28672) R = 2;
  while (R > 1 && R > M) R >>= 1;
  return R;
}

template <int MODE, int R, int UP, int NTH>
cudaError_t launch_cm(const void* in, void* out, int M, int d, int K, const uint32_t* p32, const float* cos_t,
                      const float* sin_t, const float* scale, int* status, cudaStream_t stream, int trig) {
  const size_t smem = (size_t)R * (d + 2) * sizeof(float);
  auto kern = givens_cm_kernel<R, MODE, UP, NTH>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<(M + R - 1) / R, NTH, smem, stream>>>(in, out, M, d, K, p32, cos_t, sin_t, scale, status, trig);
  return cudaPeekAtLastError();
}

template <int MODE, int R>
cudaError_t launch_r(const void* in, void* out, int M, int d, int K, const uint32_t* p32, const float* cos_t,
                     const float* sin_t, const float* scale, int* status, cudaStream_t stream, int trig) {
  const int half = d / 2;
  if (half <= 512) return launch_cm<MODE, R, 1, 512>(in, out, M, d, K, p32, cos_t, sin_t, scale, status, stream, trig);
  if (half <= 1024) return launch_cm<MODE, R, 2, 512>(in, out, M, d, K, p32, cos_t, sin_t, scale, status, stream, trig);
  if (half <= 2048) return launch_cm<MODE, R, 4, 512>(in, out, M, d, K, p32, cos_t, sin_t, scale, status, stream, trig);
  if (half <= 4096) return launch_cm<MODE, R, 4, 1024>(in, out, M, d, K, p32, cos_t, sin_t, scale, status, stream, trig);
  if (half <= 7168) return launch_cm<MODE, R, 7, 1024>(in, out, M, d, K, p32, cos_t, sin_t, scale, status, stream, trig);
  if (half <= 8192) return launch_cm<MODE, R, 8, 1024>(in, out, M, d, K, p32, cos_t, sin_t, scale, status, stream, trig);
  return launch_cm<MODE, R, 0, 1024>(in, out, M, d, K, p32, cos_t, sin_t, scale, status, stream, trig);
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
