// Group-wise INT4 weight-only linear y[m][n] = sum_k w^[n][k] x[m][k],
// w^ = (q - zero) * scale per group of 128 input columns (page "ParoQuant:
// pairwise rotations that survive deployment", section "From fake
// quantization to a real TensorRT engine": the group-wise INT4 GEMM operator).
//
// Skinny-M kernel (decode, any M; used for M <= 64).  The weight matrix plays
// the MMA's M side (16 output rows per tile) and the tokens its N side (8 per
// tile), so a single token still fills whole tensor-core tiles
// (mma.sync.m16n8k16, fp16 operands, fp32 accumulation).  Per group of 128
// input columns:
//   * lane (g, t) = (lane / 4, lane % 4) loads 16 bytes (four words = 32
//     columns 32t..32t+31 of the group) of rows g and g+8 of its tile;
//   * every word is dequantised in registers to four fp16 pairs holding the
//     exact small integers q - zero (columns (e, e+4) of the word), using the
//     0x6400 exponent-bias trick (1024 + q is exact in fp16) followed by one
//     subtract or one fused multiply-add;
//   * the activation fragments are the same 32 columns of the lane's token,
//     permuted with byte-permutes into the same (e, e+4) pairing: the order
//     of k inside an MMA is free as long as A and B agree;
//   * eight MMAs accumulate sum (q - zero) x over the group in fp32, and the
//     group's scale is applied once: acc += scale * partial.
// Groups are split round-robin over the warps of a CTA and over the CTAs of
// a thread-block cluster; partial sums are reduced through shared memory and
// then through distributed shared memory into the cluster's rank-0 CTA,
// which writes bf16.  No global scratch is used.
#include <cooperative_groups.h>

#include "paro_internal.cuh"

namespace cg = cooperative_groups;

namespace paro {
namespace {

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// Four fp16 pairs (q - z) of one packed word: P[0] = cols (0,4), P[1] = (1,5),
// P[2] = (2,6), P[3] = (3,7).  zc = 1024 + z, zh = -(64 + z), both exact in fp16.
__device__ __forceinline__ void dequant_word(uint32_t w, __half2 zc, __half2 zh, uint32_t (&P)[4]) {
  const __half2 sixteenth = __float2half2_rn(0.0625f);
  const uint32_t w2 = w >> 8;
  const uint32_t l0 = (w & 0x000F000Fu) | 0x64006400u;
  const uint32_t h0 = (w & 0x00F000F0u) | 0x64006400u;
  const uint32_t l1 = (w2 & 0x000F000Fu) | 0x64006400u;
  const uint32_t h1 = (w2 & 0x00F000F0u) | 0x64006400u;
  P[0] = h2_as_u32(__hsub2(u32_as_h2(l0), zc));
  P[1] = h2_as_u32(__hfma2(u32_as_h2(h0), sixteenth, zh));
  P[2] = h2_as_u32(__hsub2(u32_as_h2(l1), zc));
  P[3] = h2_as_u32(__hfma2(u32_as_h2(h1), sixteenth, zh));
}

// 8 consecutive activation values (as fp16 in 4 words) -> pairs (0,4),(1,5),(2,6),(3,7)
__device__ __forceinline__ void pair_act(const uint4& u, uint32_t (&B)[4]) {
  B[0] = __byte_perm(u.x, u.z, 0x5410);
  B[1] = __byte_perm(u.x, u.z, 0x7632);
  B[2] = __byte_perm(u.y, u.w, 0x5410);
  B[3] = __byte_perm(u.y, u.w, 0x7632);
}

__device__ __forceinline__ uint32_t bf2_to_h2(uint32_t v) {
  const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&v));
  return h2_as_u32(__floats2half2_rn(f.x, f.y));
}

template <bool X_F16>
__device__ __forceinline__ uint4 load_act8(const uint16_t* p) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  if constexpr (!X_F16) {
    u.x = bf2_to_h2(u.x); u.y = bf2_to_h2(u.y); u.z = bf2_to_h2(u.z); u.w = bf2_to_h2(u.w);
  }
  return u;
}

// RT row tiles of 16 weight rows, NT token tiles of 8 tokens per warp.
template <int RT, int NT, bool X_F16>
__global__ void __launch_bounds__(256)
w4_mma_kernel(const uint16_t* __restrict__ x, const uint32_t* __restrict__ qweight,
              const __half* __restrict__ scales, const __half* __restrict__ zeros,
              __nv_bfloat16* __restrict__ y, int M, int d_in, int d_out, int pdl_wait) {
  constexpr int ROWS = RT * 16, TOKS = NT * 8;
  extern __shared__ __align__(16) float red[];  // [KW][ROWS][TOKS]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int KW = blockDim.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int S = gridDim.y, rank = blockIdx.y;
  const int n0 = blockIdx.x * ROWS;
  const int m0 = blockIdx.z * TOKS;
  const int G = d_in / kGroup;
  const int wpr = d_in / 8;  // words per weight row
  const int split = S * KW, first = rank * KW + warp;

  float acc[RT][NT][4];
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[r][n][e] = 0.f;

  // prefetch the first group's weights before waiting on the producer grid
  uint4 wq[RT][2];
  auto load_w = [&](int grp) {
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const uint32_t* base = qweight + (size_t)(n0 + r * 16 + g) * wpr + (size_t)grp * 16 + t * 4;
      wq[r][0] = __ldcs(reinterpret_cast<const uint4*>(base));
      wq[r][1] = __ldcs(reinterpret_cast<const uint4*>(base + (size_t)8 * wpr));
    }
  };
  if (first < G) load_w(first);
  if (pdl_wait) asm volatile("griddepcontrol.wait;" ::: "memory");

  for (int grp = first; grp < G; grp += split) {
    // activation fragments of this group: token m0 + n*8 + g, columns 32t..32t+31
    uint32_t Bf[NT][4][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int m = m0 + n * 8 + g;
      if (m < M) {
        const uint16_t* xp = x + (size_t)m * d_in + (size_t)grp * kGroup + t * 32;
#pragma unroll
        for (int j = 0; j < 4; ++j) pair_act(load_act8<X_F16>(xp + j * 8), Bf[n][j]);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) Bf[n][j][e] = 0u;
      }
    }
    uint4 cur[RT][2];
#pragma unroll
    for (int r = 0; r < RT; ++r) { cur[r][0] = wq[r][0]; cur[r][1] = wq[r][1]; }
    const int nxt = grp + split;
    if (nxt < G) load_w(nxt);

#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const size_t srow = (size_t)(n0 + r * 16 + g) * G + grp;
      const float sc0 = __half2float(scales[srow]);
      const float sc1 = __half2float(scales[srow + (size_t)8 * G]);
      const float z0 = __half2float(zeros[srow]);
      const float z1 = __half2float(zeros[srow + (size_t)8 * G]);
      const __half2 zc0 = __float2half2_rn(1024.f + z0), zh0 = __float2half2_rn(-(64.f + z0));
      const __half2 zc1 = __float2half2_rn(1024.f + z1), zh1 = __float2half2_rn(-(64.f + z1));
      float part[NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) part[n][e] = 0.f;
      const uint32_t w0[4] = {cur[r][0].x, cur[r][0].y, cur[r][0].z, cur[r][0].w};
      const uint32_t w1[4] = {cur[r][1].x, cur[r][1].y, cur[r][1].z, cur[r][1].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t P0[4], P1[4];
        dequant_word(w0[j], zc0, zh0, P0);   // row g
        dequant_word(w1[j], zc1, zh1, P1);   // row g + 8
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          mma_16816(part[n], P0[0], P1[0], P0[1], P1[1], Bf[n][j][0], Bf[n][j][1]);
          mma_16816(part[n], P0[2], P1[2], P0[3], P1[3], Bf[n][j][2], Bf[n][j][3]);
        }
      }
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        acc[r][n][0] = fmaf(sc0, part[n][0], acc[r][n][0]);
        acc[r][n][1] = fmaf(sc0, part[n][1], acc[r][n][1]);
        acc[r][n][2] = fmaf(sc1, part[n][2], acc[r][n][2]);
        acc[r][n][3] = fmaf(sc1, part[n][3], acc[r][n][3]);
      }
    }
  }

  // ---- reduce over the warps of the CTA ------------------------------------------
  float* mine = red + (size_t)warp * ROWS * TOKS;
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int row = r * 16 + g, tok = n * 8 + 2 * t;
      mine[row * TOKS + tok] = acc[r][n][0];
      mine[row * TOKS + tok + 1] = acc[r][n][1];
      mine[(row + 8) * TOKS + tok] = acc[r][n][2];
      mine[(row + 8) * TOKS + tok + 1] = acc[r][n][3];
    }
  __syncthreads();
  for (int idx = threadIdx.x; idx < ROWS * TOKS; idx += blockDim.x) {
    float s = 0.f;
    for (int w = 0; w < KW; ++w) s += red[(size_t)w * ROWS * TOKS + idx];
    red[idx] = s;  // each idx is read and written by one thread only
  }

  // ---- reduce over the CTAs of the cluster (distributed shared memory) ---------
  if (S > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (rank == 0) {
      for (int idx = threadIdx.x; idx < ROWS * TOKS; idx += blockDim.x) {
        float s = red[idx];
        for (int q = 1; q < S; ++q) s += cluster.map_shared_rank(red, q)[idx];
        red[idx] = s;
      }
    }
    cluster.sync();
    if (rank != 0) return;
  } else {
    __syncthreads();
  }
  // ---- write bf16: consecutive threads take consecutive rows of one token ------
  for (int idx = threadIdx.x; idx < ROWS * TOKS; idx += blockDim.x) {
    const int tok = idx / ROWS, row = idx % ROWS;
    const int m = m0 + tok;
    if (m < M) y[(size_t)m * d_out + n0 + row] = __float2bfloat16_rn(red[row * TOKS + tok]);
  }
}

template <int RT, int NT, bool X_F16>
cudaError_t launch_cfg(const void* x, const uint32_t* qweight, const __half* scales, const __half* zeros,
                       __nv_bfloat16* y, int M, int d_in, int d_out, int KW, int S, cudaStream_t stream,
                       bool pdl_wait) {
  constexpr int ROWS = RT * 16, TOKS = NT * 8;
  const size_t smem = (size_t)KW * ROWS * TOKS * sizeof(float);
  auto kern = w4_mma_kernel<RT, NT, X_F16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (S > 1) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(d_out / ROWS, S, (M + TOKS - 1) / TOKS);
  cfg.blockDim = dim3(32 * KW);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeClusterDimension;
  attr[na].val.clusterDim.x = 1;
  attr[na].val.clusterDim.y = S;
  attr[na].val.clusterDim.z = 1;
  ++na;
  if (pdl_wait) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<const uint16_t*>(x), qweight, scales, zeros, y, M, d_in,
                            d_out, pdl_wait ? 1 : 0);
}

}  // namespace

cudaError_t launch_w4_linear_mma(const void* x, int x_is_f16, const uint32_t* qweight,
                                 const __half* scales, const __half* zeros, __nv_bfloat16* y,
                                 int M, int d_in, int d_out, cudaStream_t stream, bool pdl_wait) {
  const int G = d_in / kGroup;
  const int NT = M <= 8 ? 1 : 2;
  int RT = (M <= 8) ? 2 : 4;
  while (RT > 1 && d_out % (16 * RT)) RT >>= 1;
  const int row_blocks = d_out / (16 * RT);
  const int tok_blocks = (M + 8 * NT - 1) / (8 * NT);
  // enough warps in flight to cover HBM latency: about 1536 warps per launch
  int T = (1536 + row_blocks * tok_blocks - 1) / (row_blocks * tok_blocks);
  if (T > G) T = G;
  if (T > 64) T = 64;
  if (T < 1) T = 1;
  int KW = T < 8 ? T : 8;
  int S = (T + KW - 1) / KW;
  if (S > 8) S = 8;
  const bool f16 = x_is_f16 != 0;
#define PARO_W4_CASE(rt, nt)                                                                          \
  if (RT == rt && NT == nt)                                                                           \
    return f16 ? launch_cfg<rt, nt, true>(x, qweight, scales, zeros, y, M, d_in, d_out, KW, S, stream, pdl_wait) \
               : launch_cfg<rt, nt, false>(x, qweight, scales, zeros, y, M, d_in, d_out, KW, S, stream, pdl_wait);
  PARO_W4_CASE(1, 1)
  PARO_W4_CASE(2, 1)
  PARO_W4_CASE(1, 2)
  PARO_W4_CASE(2, 2)
  PARO_W4_CASE(4, 2)
#undef PARO_W4_CASE
  return cudaErrorInvalidConfiguration;
}

}  // namespace paro
