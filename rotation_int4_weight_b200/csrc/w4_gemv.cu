// Group-wise INT4 weight-only linear for few tokens (decode):
//   y[m][n] = sum_k w^[n][k] x[m][k],  w^ = (q - zero) * scale per group of 128 input columns
// (page "ParoQuant: pairwise rotations that survive deployment", section "From fake
// quantization to a real TensorRT engine": the group-wise INT4 GEMM operator).
//
// Tensor-core mapping.  The weights are the MMA's 16-row side and the tokens
// its 8-column side (mma.sync m16n8k16, fp32 accumulation), so one token still
// fills whole tiles.  Lane (g, t) = (lane / 4, lane % 4) holds, per 128-column
// group, 16 bytes (32 columns) of weight rows g and g + 8 of its tile.  A word
// becomes MMA operands with four bit operations and one shift: OR-ing a nibble
// into the mantissa of 1024 (fp16) or 128 (bf16) gives bias + q exactly, and
// the odd nibbles are left where they sit (x16, or moved one bit: x8), with the
// matching activations pre-divided by 16 (or 8) once per stage.  The order of k
// inside an MMA is free when both operands agree, so the activations are
// byte-permuted into the order the nibbles unpack to.  Per group and token, two
// MMAs with constant operands give Tb = sum(bias x) and Sx = sum x, shared by all
// rows, so sum (q - z) x = R - Tb - z Sx with R the weight MMAs' result, and the
// group scale multiplies that once (all in fp32).  fp16 activations (the fused
// path's transformed x) use fp16 MMAs, bf16 activations bf16 MMAs: the codes are
// exact in both, so no rounding is added to the weights.
//
// Work decomposition.  One launch serves up to kMaxBatch independent linears.
// A CTA (8 warps) takes one item = (linear, block of rows, block of <= 16
// tokens); its warps form 2^c chunk groups that split the item's groups of 128
// columns, each warp of a chunk group owning one 16-row tile.  Partial sums of
// the chunk groups meet in shared memory at the end of the item (no global
// scratch, no atomics, a fixed summation order).
//
// Memory pipeline.  Every warp streams its weights through a private ring of D
// stages in shared memory with cp.async (16 bytes per lane, read back by the
// same lane, so a wait on the lane's own copies is enough); the activations of
// a stage are copied once per chunk group and published with a named barrier.
// Scales and zeros ride in registers, D - 1 stages ahead.  With programmatic
// dependent launch, the weights of the first D - 1 stages are requested before
// the kernel waits for the grid that produces the activations.
#include "paro_internal.cuh"
#include "w4_gemv.cuh"

namespace paro {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = 4;
constexpr int kRowTiles = 2;     // 16-row weight tiles per warp
constexpr int kTokStride = 320;  // bytes per token row of an activation stage (256 + 64 pad: no bank conflicts)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }
__device__ __forceinline__ void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

template <bool F16>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (F16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

// One packed word -> four operand pairs of exponent-biased codes, exact in the
// operand type: P[0] = columns (0,4), P[1] = (1,5), P[2] = (2,6), P[3] = (3,7).
//   fp16: even nibbles give 1024 + q, odd nibbles (left in bits 4..7) 1024 + 16 q;
//   bf16: even nibbles give 128 + q, odd nibbles (moved to bits 3..6) 128 + 8 q.
// The odd columns' activations are pre-divided by 16 (fp16) or 8 (bf16), so every
// product is (bias + q) x for the matching bias, and the bias and zero point are
// removed once per group with two constant-operand MMAs (see the kernel).
template <bool F16>
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t (&P)[4]) {
  if constexpr (F16) {
    const uint32_t w2 = w >> 8;
    P[0] = (w & 0x000F000Fu) | 0x64006400u;
    P[1] = (w & 0x00F000F0u) | 0x64006400u;
    P[2] = (w2 & 0x000F000Fu) | 0x64006400u;
    P[3] = (w2 & 0x00F000F0u) | 0x64006400u;
  } else {
    P[0] = (w & 0x000F000Fu) | 0x43004300u;
    P[1] = ((w >> 1) & 0x00780078u) | 0x43004300u;
    P[2] = ((w >> 8) & 0x000F000Fu) | 0x43004300u;
    P[3] = ((w >> 9) & 0x00780078u) | 0x43004300u;
  }
}

template <bool F16>
__device__ __forceinline__ uint32_t mul2(uint32_t a, uint32_t b) {
  uint32_t r;
  if constexpr (F16) asm("mul.rn.f16x2 %0, %1, %2;\n" : "=r"(r) : "r"(a), "r"(b));
  else asm("mul.rn.bf16x2 %0, %1, %2;\n" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// 8 consecutive activations (4 words) -> pairs (0,4), (1,5), (2,6), (3,7)
__device__ __forceinline__ void pair_act(const uint4& u, uint32_t (&B)[4]) {
  B[0] = __byte_perm(u.x, u.z, 0x5410);
  B[1] = __byte_perm(u.x, u.z, 0x7632);
  B[2] = __byte_perm(u.y, u.w, 0x5410);
  B[3] = __byte_perm(u.y, u.w, 0x7632);
}

template <bool F16, int NT>
__global__ void __launch_bounds__(kThreads, 2)
w4_gemv_kernel(const __grid_constant__ GemvBatch batch, int pdl_wait) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int D = kStages;
  constexpr int RT = kRowTiles;         // 16-row tiles per warp
  constexpr int WSTAGE = RT * 1024;     // weight bytes per warp and stage
  constexpr int TOK = 8 * NT;

  // ---- which linear and which item ------------------------------------------------
  const int item = blockIdx.x;
  int pi = 0;
#pragma unroll 1
  while (pi + 1 < batch.count && item >= batch.p[pi + 1].item_begin) ++pi;
  const GemvProblem& P = batch.p[pi];
  const int local = item - P.item_begin;
  const int tb = local / P.row_blocks, rb = local % P.row_blocks;
  const int lg = P.log2_chunks;
  const int n_chunks = 1 << lg, wpc = kWarps >> lg;  // chunk groups, warps per chunk group
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int chunk = warp / wpc, rt = warp % wpc;
  const int G = P.d_in >> 7;
  const int g_lo = chunk * G / n_chunks, g_hi = (chunk + 1) * G / n_chunks;
  const int nst = g_hi - g_lo;
  const int row0 = (rb * wpc + rt) * 16 * RT;   // first of this warp's RT x 16 rows
  const int ntile = max(0, min(RT, (P.d_out - row0) >> 4));
  const int m0 = tb * TOK;
  const int mt = min(P.M - m0, TOK);       // tokens of this item
  const int xtok = P.x_tok;                // token rows reserved per activation stage

  // ---- shared memory: weight rings | activation rings | reduction --------------------
  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_w = s_base + (uint32_t)(warp * D * WSTAGE);                 // [warp][D][RT][2][32][16]
  const uint32_t x_stage = (uint32_t)xtok * kTokStride;
  const uint32_t s_x = s_base + (uint32_t)(kWarps * D * WSTAGE) + (uint32_t)(chunk * D) * x_stage;
  float* red = reinterpret_cast<float*>(smem + kWarps * D * WSTAGE + n_chunks * D * x_stage);

  const size_t wpr = (size_t)(P.d_in >> 3);  // words per weight row
  const uint32_t* qbase = P.qw + (size_t)(row0 + g) * wpr + t * 4;
  // lane (g, t) fetches one 16-bit value per row tile and stage: t = 0 scale of row
  // g, t = 1 scale of row g + 8, t = 2 zero of row g, t = 3 zero of row g + 8; the
  // four are gathered with shuffles only when the stage is computed, so the loads
  // stay in flight D - 1 stages like the weights
  const unsigned short* szb = reinterpret_cast<const unsigned short*>((t & 2) ? P.z : P.sc) +
                              (size_t)(row0 + g + (t & 1) * 8) * G;
  const int cthreads = wpc * 32, ctid = rt * 32 + lane;  // threads of this chunk group

  auto issue_w = [&](int i, int slot) {
    if (i < nst) {
      const int grp = g_lo + i;
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        if (r < ntile) {
          const uint32_t d = s_w + (uint32_t)(slot * WSTAGE + r * 1024) + (uint32_t)lane * 16u;
          const uint32_t* src = qbase + (size_t)(r * 16) * wpr + grp * 16;
          cp_async16(d, src);
          cp_async16(d + 512u, src + 8 * wpr);
        }
      }
    }
  };
  auto issue_x = [&](int i, int slot) {
    if (i < nst) {
      const int grp = g_lo + i;
      // 16-byte pieces (token, p): p = 0..15 covers columns 8p..8p+7 of the group;
      // lane t's 64 bytes are pieces 4t..4t+3 and land at [token][j = p % 4][t = p / 4]
      for (int idx = ctid; idx < mt * 16; idx += cthreads) {
        const int tok = idx >> 4, p = idx & 15;
        const uint16_t* src = P.x + (size_t)(m0 + tok) * P.d_in + (size_t)grp * kGroup + p * 8;
        const uint32_t d = s_x + (uint32_t)slot * x_stage + (uint32_t)tok * kTokStride +
                           (uint32_t)((p & 3) * 64 + (p >> 2) * 16);
        cp_async16(d, src);
      }
    }
  };
  uint32_t szr[D][RT];  // raw 16-bit scale or zero per slot and row tile (see szb)
  auto issue_sz = [&](int i, uint32_t (&r1)[RT]) {
    if (i < nst) {
      const int grp = g_lo + i;
#pragma unroll
      for (int r = 0; r < RT; ++r)
        if (r < ntile) r1[r] = __ldg(szb + (size_t)(r * 16) * G + grp);
    }
  };

  // ---- prologue: weights first, then (after the producer grid) activations ------------
#pragma unroll
  for (int s = 0; s < D - 1; ++s) {
    issue_w(s, s);
    cp_commit();
    issue_sz(s, szr[s]);
  }
  if (pdl_wait) asm volatile("griddepcontrol.wait;\n" ::: "memory");
#pragma unroll
  for (int s = 0; s < D - 1; ++s) {
    issue_x(s, s);
    cp_commit();
  }

  float acc[RT][NT][4];
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[r][n][e] = 0.f;

  for (int base = 0; base < nst; base += D) {
#pragma unroll
    for (int s = 0; s < D; ++s) {
      const int i = base + s;
      if (i >= nst) break;
      cp_wait<D - 2>();
      named_sync(1 + chunk, cthreads);
      {  // refill the slot freed by the previous iteration
        const int ns = (s + D - 1) % D;
        issue_w(i + D - 1, ns);
        issue_x(i + D - 1, ns);
        cp_commit();
        issue_sz(i + D - 1, szr[ns]);
      }
      if (ntile == 0) continue;
      // activation fragments of this stage (shared by the warp's row tiles); the odd
      // columns (second register of each pair) are pre-divided to match the codes
      constexpr uint32_t kOddScale = F16 ? 0x2C002C00u : 0x3E003E00u;  // 1/16 or 1/8
      uint32_t Bf[NT][4][4];
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int tok = n * 8 + g;
        if (tok < mt) {
          const uint32_t xa = s_x + (uint32_t)s * x_stage + (uint32_t)tok * kTokStride + (uint32_t)t * 16u;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            pair_act(lds128(xa + j * 64), Bf[n][j]);
            Bf[n][j][1] = mul2<F16>(Bf[n][j][1], kOddScale);
            Bf[n][j][3] = mul2<F16>(Bf[n][j][3], kOddScale);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) Bf[n][j][e] = 0u;
        }
      }
      // per token: Tb = sum (bias x) over the group's products, Sx = sum x
      //   fp16: Tb = 1024 S_even + 64 S_odd;  bf16: Tb = 128 S_even + 16 S_odd
      constexpr uint32_t kBias = F16 ? 0x64006400u : 0x43004300u;     // 1024 / 128
      constexpr uint32_t kOne = F16 ? 0x3C003C00u : 0x3F803F80u;      // 1
      constexpr uint32_t kOddUp = F16 ? 0x4C004C00u : 0x41004100u;    // 16 / 8
      const uint32_t aT[4] = {kBias, kBias, kBias, kBias};
      const uint32_t aS[4] = {kOne, kOne, kOddUp, kOddUp};
      float Tb[NT][4], Sx[NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) { Tb[n][e] = 0.f; Sx[n][e] = 0.f; }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          mma16816<F16>(Tb[n], aT, Bf[n][j][0], Bf[n][j][1]);
          mma16816<F16>(Tb[n], aT, Bf[n][j][2], Bf[n][j][3]);
          mma16816<F16>(Sx[n], aS, Bf[n][j][0], Bf[n][j][1]);
          mma16816<F16>(Sx[n], aS, Bf[n][j][2], Bf[n][j][3]);
        }
      }
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        if (r >= ntile) break;
        const uint32_t wa = s_w + (uint32_t)(s * WSTAGE + r * 1024) + (uint32_t)lane * 16u;
        const uint4 wg = lds128(wa), wh = lds128(wa + 512u);
        const int q0 = lane & ~3;
        const float scg = __half2float(__ushort_as_half((unsigned short)__shfl_sync(0xffffffffu, szr[s][r], q0)));
        const float sch = __half2float(__ushort_as_half((unsigned short)__shfl_sync(0xffffffffu, szr[s][r], q0 | 1)));
        const float zg = __half2float(__ushort_as_half((unsigned short)__shfl_sync(0xffffffffu, szr[s][r], q0 | 2)));
        const float zh = __half2float(__ushort_as_half((unsigned short)__shfl_sync(0xffffffffu, szr[s][r], q0 | 3)));
        float R[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) R[n][e] = 0.f;
        const uint32_t wgv[4] = {wg.x, wg.y, wg.z, wg.w};
        const uint32_t whv[4] = {wh.x, wh.y, wh.z, wh.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t Pg[4], Ph[4];
          unpack_word<F16>(wgv[j], Pg);
          unpack_word<F16>(whv[j], Ph);
          const uint32_t a0[4] = {Pg[0], Ph[0], Pg[1], Ph[1]};
          const uint32_t a1[4] = {Pg[2], Ph[2], Pg[3], Ph[3]};
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            mma16816<F16>(R[n], a0, Bf[n][j][0], Bf[n][j][1]);
            mma16816<F16>(R[n], a1, Bf[n][j][2], Bf[n][j][3]);
          }
        }
        // sum (q - z) x = R - Tb - z Sx; then the group scale
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          acc[r][n][0] = fmaf(scg, fmaf(-zg, Sx[n][0], R[n][0] - Tb[n][0]), acc[r][n][0]);
          acc[r][n][1] = fmaf(scg, fmaf(-zg, Sx[n][1], R[n][1] - Tb[n][1]), acc[r][n][1]);
          acc[r][n][2] = fmaf(sch, fmaf(-zh, Sx[n][2], R[n][2] - Tb[n][2]), acc[r][n][2]);
          acc[r][n][3] = fmaf(sch, fmaf(-zh, Sx[n][3], R[n][3] - Tb[n][3]), acc[r][n][3]);
        }
      }
    }
  }
  cp_wait<0>();

  // ---- combine the chunk groups and write bf16 --------------------------------------
  constexpr int WROWS = RT * 16;
  float* mine = red + warp * (WROWS * TOK);
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int tok = n * 8 + 2 * t, row = r * 16 + g;
      mine[row * TOK + tok] = acc[r][n][0];
      mine[row * TOK + tok + 1] = acc[r][n][1];
      mine[(row + 8) * TOK + tok] = acc[r][n][2];
      mine[(row + 8) * TOK + tok + 1] = acc[r][n][3];
    }
  __syncthreads();
  const int rows_item = wpc * WROWS;
  for (int idx = threadIdx.x; idx < rows_item * TOK; idx += kThreads) {
    const int tok = idx / rows_item, r = idx % rows_item;
    const int w = r / WROWS, rr = r % WROWS;
    const int n = rb * rows_item + r;
    if (tok >= mt || n >= P.d_out) continue;
    float sum = 0.f;
    for (int c = 0; c < n_chunks; ++c) sum += red[(c * wpc + w) * (WROWS * TOK) + rr * TOK + tok];
    P.y[(size_t)(m0 + tok) * P.d_out + n] = __float2bfloat16_rn(sum);
  }
}

size_t smem_bytes(int log2_chunks, int x_tok, int NT) {
  return (size_t)kWarps * kStages * kRowTiles * 1024 + (size_t)(1 << log2_chunks) * kStages * x_tok * kTokStride +
         (size_t)kWarps * kRowTiles * 16 * 8 * NT * sizeof(float);
}

}  // namespace

// Chooses the split of every linear and lays the items out.
cudaError_t plan_gemv_batch(const GemvProblem* probs, int count, bool x_f16, GemvBatch* out, int* nt_out) {
  if (count < 1 || count > kMaxBatch) return cudaErrorInvalidValue;
  int maxM = 0;
  for (int i = 0; i < count; ++i) maxM = probs[i].M > maxM ? probs[i].M : maxM;
  const int NT = maxM <= 8 ? 1 : 2;
  const int x_tok = maxM < 8 * NT ? maxM : 8 * NT;
  *out = GemvBatch{};
  int items = 0;
  for (int i = 0; i < count; ++i) {
    GemvProblem p = probs[i];
    const int G = p.d_in / kGroup;
    // split the groups over as many chunk groups as keeps >= 2 groups each and
    // the shared memory of two CTAs per SM
    // two CTAs per SM when one token tile is staged; with two token tiles the
    // activation stages are larger and one CTA per SM keeps more row groups busy
    const size_t limit = NT == 1 ? 110 * 1024 : 220 * 1024;
    int lg = 3;
    while (lg > 0 && ((1 << lg) * 2 > G || smem_bytes(lg, x_tok, NT) > limit)) --lg;
    p.log2_chunks = lg;
    const int rows_item = (kWarps >> lg) * 16 * kRowTiles;
    p.row_blocks = (p.d_out + rows_item - 1) / rows_item;
    p.item_begin = items;
    p.x_tok = x_tok;
    const int tok_blocks = (p.M + 8 * NT - 1) / (8 * NT);
    items += p.row_blocks * tok_blocks;
    out->p[i] = p;
  }
  out->count = count;
  out->total_items = items;
  out->x_f16 = x_f16 ? 1 : 0;
  *nt_out = NT;
  return cudaSuccess;
}

cudaError_t launch_gemv_batch(const GemvBatch& b, int NT, cudaStream_t stream, bool pdl_wait) {
  int lgmax = 0;
  for (int i = 0; i < b.count; ++i) lgmax = b.p[i].log2_chunks > lgmax ? b.p[i].log2_chunks : lgmax;
  const size_t smem = smem_bytes(lgmax, b.p[0].x_tok, NT);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(b.total_items);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_wait ? 1 : 0;
  const int wait = pdl_wait ? 1 : 0;
  cudaError_t e;
#define PARO_GEMV_LAUNCH(f16, nt)                                                                         \
  {                                                                                                       \
    auto k = w4_gemv_kernel<f16, nt>;                                                                     \
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);                  \
    if (e != cudaSuccess) return e;                                                                       \
    return cudaLaunchKernelEx(&cfg, k, b, wait);                                                          \
  }
  if (b.x_f16) {
    if (NT == 1) PARO_GEMV_LAUNCH(true, 1) else PARO_GEMV_LAUNCH(true, 2)
  } else {
    if (NT == 1) PARO_GEMV_LAUNCH(false, 1) else PARO_GEMV_LAUNCH(false, 2)
  }
#undef PARO_GEMV_LAUNCH
}

}  // namespace paro
