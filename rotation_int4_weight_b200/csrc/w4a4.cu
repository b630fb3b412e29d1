// Weight-activation (W4A4) variant of the linear: per-token symmetric INT4
// codes of the transformed activations, and the INT4 x INT4 linear on the
// packed INT4 weights of the weight-only path (page "ParoQuant: Pairwise
// Rotation Quantization for Efficient Reasoning LLM Inference", section
// "Abstract (arXiv)": the method also matches weight-activation quantization
// methods; the pages give no detail of that setting, so this is the plainest
// reading of 4-bit weights and 4-bit activations on top of the weight-only path).
//
//   codes:  s_x[m] = max_k |x~[m][k]| / 7 (1 for an all-zero row),
//           q_x[m][k] = clamp(rint(x~[m][k] / s_x[m]), -8, 7), fp32, ties to even;
//   linear: y[m][n] = s_x[m] * sum_g s_w[n][g] * sum_{k in g} (q_w[n][k] - z[n][g]) q_x[m][k].
//
// The inner sums are exact integers: the nibbles of a packed weight word become
// bytes (the even columns in one register, the odd ones in another) and meet
// the activation codes, rearranged the same way with a byte permute, in
// mma.sync m16n8k32 with u8 x s8 operands and int32 accumulation.  One more MMA
// with an all-ones A gives sum_k q_x per token and group for the zero-point
// term.  Each CTA takes 64 weight rows and a contiguous share of the groups;
// its warps take every 8th group of that share and are summed in shared memory
// in warp order, the shares of several CTAs of one tile in a second launch in
// share order, so the result does not depend on timing.
#include "paro_internal.cuh"

namespace paro {
namespace {

constexpr int kQuantThreads = 256;
constexpr int kW4a4Warps = 8;
constexpr int kW4a4Rows = 64;
constexpr int kW4a4Tokens = 16;  // tokens a CTA takes (two 8-column MMA tiles)

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  return red[0];
}

// One CTA per token row: the row's largest magnitude, its scale, then the codes.
__global__ void __launch_bounds__(kQuantThreads)
quantize_act_kernel(const __nv_bfloat16* __restrict__ x, int8_t* __restrict__ q, float* __restrict__ sx, int d) {
  __shared__ float red[32];
  const size_t row = (size_t)blockIdx.x * d;
  float amax = 0.0f;
  for (int c = threadIdx.x * 8; c < d; c += kQuantThreads * 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(x + row + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
      amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
  amax = block_max(amax, red);
  const float s = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 7.0f);
  if (threadIdx.x == 0) sx[blockIdx.x] = s;
  for (int c = threadIdx.x * 8; c < d; c += kQuantThreads * 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(x + row + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
      const int q0 = (int)fminf(fmaxf(rintf(__fdiv_rn(f.x, s)), -8.0f), 7.0f);
      const int q1 = (int)fminf(fmaxf(rintf(__fdiv_rn(f.y, s)), -8.0f), 7.0f);
      const uint32_t pair = ((uint32_t)q0 & 0xFFu) | (((uint32_t)q1 & 0xFFu) << 8);
      out[e >> 1] |= pair << (16 * (e & 1));
    }
    *reinterpret_cast<uint2*>(q + row + c) = make_uint2(out[0], out[1]);
  }
}

__device__ __forceinline__ void mma_u8s8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// CTA (tile, share, token block): rows tile*64 .. +63, groups [g0, g1), tokens
// m0 .. m0 + 15.  out: y (bf16, scaled by s_x) when the tile has one share,
// else the share's fp32 partial [share][M][d_out].
template <int NT>
__global__ void __launch_bounds__(kW4a4Warps * 32)
w4a4_kernel(const int8_t* __restrict__ qx, const float* __restrict__ sx, const uint32_t* __restrict__ qw,
            const __half* __restrict__ sw, const __half* __restrict__ zw, __nv_bfloat16* __restrict__ y,
            float* __restrict__ part, int M, int d_in, int d_out, int shares) {
  __shared__ float red[kW4a4Warps][kW4a4Rows][kW4a4Tokens];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gq = lane >> 2, t = lane & 3;
  const int tile = blockIdx.x, share = blockIdx.y, m0 = blockIdx.z * kW4a4Tokens;
  const int G = d_in / kGroup, W8 = d_in / 8;
  const int g0 = (int)((long long)share * G / shares), g1 = (int)((long long)(share + 1) * G / shares);
  float acc[4][NT][4];
#pragma unroll
  for (int rt = 0; rt < 4; ++rt)
#pragma unroll
    for (int m = 0; m < NT; ++m)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[rt][m][e] = 0.0f;
  const uint32_t ones[4] = {0x01010101u, 0x01010101u, 0x01010101u, 0x01010101u};

#pragma unroll 1
  for (int g = g0 + warp; g < g1; g += kW4a4Warps) {
    // activation codes of token m0 + m*8 + gq, columns 32t .. 32t + 31 of the
    // group: word kk (8 columns) as its even and its odd columns
    uint32_t b[NT][4][2];
    int xs[NT][4];
#pragma unroll
    for (int m = 0; m < NT; ++m) {
      const int tok = m0 + m * 8 + gq;
      uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
      if (tok < M) {
        const uint4* p = reinterpret_cast<const uint4*>(qx + (size_t)tok * d_in + (size_t)g * kGroup + 32 * t);
        v0 = p[0];
        v1 = p[1];
      }
      const uint32_t lo[4] = {v0.x, v0.z, v1.x, v1.z}, hi[4] = {v0.y, v0.w, v1.y, v1.w};
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        b[m][kk][0] = __byte_perm(lo[kk], hi[kk], 0x6420);
        b[m][kk][1] = __byte_perm(lo[kk], hi[kk], 0x7531);
      }
      // sum of the codes per token: xs[m][0] token 2t, xs[m][1] token 2t + 1
#pragma unroll
      for (int e = 0; e < 4; ++e) xs[m][e] = 0;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) mma_u8s8(xs[m], ones, b[m][kk][0], b[m][kk][1]);
    }
#pragma unroll
    for (int rt = 0; rt < 4; ++rt) {
      const int rg = tile * kW4a4Rows + rt * 16 + gq, rh = rg + 8;
      uint4 wg = make_uint4(0u, 0u, 0u, 0u), wh = wg;
      if (rg < d_out) wg = __ldg(reinterpret_cast<const uint4*>(qw + (size_t)rg * W8 + (size_t)g * 16 + 4 * t));
      if (rh < d_out) wh = __ldg(reinterpret_cast<const uint4*>(qw + (size_t)rh * W8 + (size_t)g * 16 + 4 * t));
      const uint32_t wgv[4] = {wg.x, wg.y, wg.z, wg.w}, whv[4] = {wh.x, wh.y, wh.z, wh.w};
      int c[NT][4];
#pragma unroll
      for (int m = 0; m < NT; ++m)
#pragma unroll
        for (int e = 0; e < 4; ++e) c[m][e] = 0;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        // a0 / a1: the even columns of rows g / g + 8, a2 / a3 the odd ones
        const uint32_t a[4] = {wgv[kk] & 0x0F0F0F0Fu, whv[kk] & 0x0F0F0F0Fu, (wgv[kk] >> 4) & 0x0F0F0F0Fu,
                               (whv[kk] >> 4) & 0x0F0F0F0Fu};
#pragma unroll
        for (int m = 0; m < NT; ++m) mma_u8s8(c[m], a, b[m][kk][0], b[m][kk][1]);
      }
      const float sg = rg < d_out ? __half2float(sw[(size_t)rg * G + g]) : 0.0f;
      const float sh = rh < d_out ? __half2float(sw[(size_t)rh * G + g]) : 0.0f;
      const int zg = rg < d_out ? (int)__half2float(zw[(size_t)rg * G + g]) : 0;
      const int zh = rh < d_out ? (int)__half2float(zw[(size_t)rh * G + g]) : 0;
#pragma unroll
      for (int m = 0; m < NT; ++m) {
        acc[rt][m][0] += sg * (float)(c[m][0] - zg * xs[m][0]);
        acc[rt][m][1] += sg * (float)(c[m][1] - zg * xs[m][1]);
        acc[rt][m][2] += sh * (float)(c[m][2] - zh * xs[m][0]);
        acc[rt][m][3] += sh * (float)(c[m][3] - zh * xs[m][1]);
      }
    }
  }
  // the warps' sums in warp order
#pragma unroll
  for (int rt = 0; rt < 4; ++rt)
#pragma unroll
    for (int m = 0; m < NT; ++m)
#pragma unroll
      for (int e = 0; e < 4; ++e) red[warp][rt * 16 + gq + (e >> 1) * 8][m * 8 + 2 * t + (e & 1)] = acc[rt][m][e];
  __syncthreads();
  for (int i = threadIdx.x; i < kW4a4Rows * NT * 8; i += kW4a4Warps * 32) {
    const int r = i / (NT * 8), tl = i % (NT * 8);
    const int row = tile * kW4a4Rows + r, tok = m0 + tl;
    if (row >= d_out || tok >= M) continue;
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < kW4a4Warps; ++w) v += red[w][r][tl];
    if (shares == 1) y[(size_t)tok * d_out + row] = __float2bfloat16_rn(sx[tok] * v);
    else part[((size_t)share * M + tok) * d_out + row] = v;
  }
}

// y = s_x * (the shares' partials summed in share order)
__global__ void w4a4_reduce_kernel(const float* __restrict__ part, const float* __restrict__ sx,
                                   __nv_bfloat16* __restrict__ y, int M, int d_out, int shares) {
  const size_t n = (size_t)M * d_out;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    float v = 0.0f;
    for (int s = 0; s < shares; ++s) v += part[(size_t)s * n + i];
    y[i] = __float2bfloat16_rn(sx[i / d_out] * v);
  }
}

}  // namespace

int w4a4_shares(int d_in, int d_out, int sms) {
  const int tiles = (d_out + kW4a4Rows - 1) / kW4a4Rows, G = d_in / kGroup;
  int s = (2 * sms + tiles - 1) / tiles;
  return s < 1 ? 1 : (s > G ? G : s);
}

size_t w4a4_partial_bytes(int M, int d_in, int d_out, int sms) {
  const int s = w4a4_shares(d_in, d_out, sms);
  return s > 1 ? (size_t)s * M * d_out * 4 : 0;
}

cudaError_t launch_quantize_act(const uint16_t* x, int8_t* q, float* sx, int M, int d, cudaStream_t stream) {
  quantize_act_kernel<<<M, kQuantThreads, 0, stream>>>(reinterpret_cast<const __nv_bfloat16*>(x), q, sx, d);
  return cudaGetLastError();
}

cudaError_t launch_w4a4(const int8_t* qx, const float* sx, const uint32_t* qw, const uint16_t* sw,
                        const uint16_t* zw, uint16_t* y, int M, int d_in, int d_out, float* part, int shares,
                        cudaStream_t stream) {
  const dim3 grid((d_out + kW4a4Rows - 1) / kW4a4Rows, shares, (M + kW4a4Tokens - 1) / kW4a4Tokens);
  auto* yy = reinterpret_cast<__nv_bfloat16*>(y);
  auto* s16 = reinterpret_cast<const __half*>(sw);
  auto* z16 = reinterpret_cast<const __half*>(zw);
  if (M <= 8)
    w4a4_kernel<1><<<grid, kW4a4Warps * 32, 0, stream>>>(qx, sx, qw, s16, z16, yy, part, M, d_in, d_out, shares);
  else
    w4a4_kernel<2><<<grid, kW4a4Warps * 32, 0, stream>>>(qx, sx, qw, s16, z16, yy, part, M, d_in, d_out, shares);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || shares == 1) return e;
  const size_t n = (size_t)M * d_out;
  const int blocks = (int)((n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184);
  w4a4_reduce_kernel<<<blocks, 256, 0, stream>>>(part, sx, yy, M, d_out, shares);
  return cudaGetLastError();
}

}  // namespace paro
