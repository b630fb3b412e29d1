// Group-wise INT4 weight-only linear for many tokens (prefill) on the 5th-
// generation tensor cores: y[m][n] = sum_k x[m][k] w^[n][k],
// w^ = (q - zero) * scale per group of 128 input columns (page "ParoQuant:
// pairwise rotations that survive deployment", section "From fake
// quantization to a real TensorRT engine": the group-wise INT4 GEMM operator).
//
// One CTA computes a 256-token x 256-output tile, K in steps of 64 through a
// ring of kStages shared-memory stages:
//   warp 16, lane 0 TMA: the stage's packed codes (256 rows x 32 bytes, 32-byte
//                   swizzle), completing on full_c[s], and the 256 x 64 fp16
//                   activation tile (128-byte swizzle), completing on
//                   full_a[s]; bf16 activations land the same way (on
//                   full_raw[s]) and warps 18-25 round them to fp16 in place
//                   (fp16 operands keep the product error an order of
//                   magnitude below bf16 ones);
//   warps 0-15      dequantisation: thread (row t, half h) reads its 16 bytes
//                   of the stage's codes from shared memory, holds its row's
//                   scale and zero bits (loaded once per 128-column group, a
//                   few groups ahead), turns every word into eight fp16 values
//                   (q - zero) * scale in column order and stores them in the
//                   128-byte-swizzled K-major layout the tensor core reads;
//                   then arrives on full_b[s] after a proxy fence;
//   warp 17, lane 0 MMA: four tcgen05.mma (kind::f16, K = 16, N = 256) per step
//                   and token half into two 128 x 256 fp32 accumulators in tensor
//                   memory, then tcgen05.commit to empty[s] (the stage may be
//                   refilled once the MMAs that read it are done) and, after
//                   the last step, to acc_full;
//   warps 0-15      epilogue: tcgen05.ld of their 32 lanes (tokens) and 128
//                   columns of one accumulator, bf16 round, 64-byte stores.
// A 256 x 256 tile reads each activation tile once per 256 outputs: the
// tensor core's shared-memory operand traffic per flop is 3/4 of that of a
// 256 x 128 tile.
// Every mbarrier wait is bounded; a wait that gives up sets PARO_ERR_TIMEOUT,
// stops the pipeline and still releases the tensor memory.
#include <cuda.h>

#include "paro_internal.cuh"
#include "w4_tc.cuh"
#include "w4_stream.cuh"  // device_sm_count

namespace paro {
namespace {

constexpr int BM = 256, BN = 256, BK = 64;  // two 128-token MMA halves share each B tile
constexpr int MH = 128;                       // tokens per MMA (M of one tcgen05.mma)
constexpr int kStages = 3;
constexpr int kDqWarps = 16;      // warps 0-15: dequantisation (one weight row per thread), then epilogue
constexpr int kWarpTma = 16;      // TMA producer, tensor-memory allocation
constexpr int kWarpMma = 17;      // MMA issuer
constexpr int kWarpConv = 18;     // warps 18-25: bf16 activations -> fp16 tiles (bf16 input only)
constexpr int kThreadsTma = 576;
constexpr int kThreadsConv = 832;
constexpr int A_BYTES = BM * BK * 2;  // 32 KB
constexpr int B_BYTES = BN * BK * 2;  // 32 KB
constexpr int C_BYTES = BN * BK / 2;  // 8 KB of packed codes (256 rows x 32 bytes, 32-byte swizzle)
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + C_BYTES;
constexpr int SMEM_BYTES = kStages * STAGE_BYTES + 1024;  // + alignment slack
constexpr uint32_t kTmemCols = 512;  // two 128 x 256 fp32 accumulators (all of tensor memory)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}
// Bounded wait on an mbarrier phase (about a second of SM clock).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_test(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_test(bar, parity))
    if (clock64() - t0 > (1LL << 31)) return false;
  return true;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

// K-major operand in the 128-byte swizzle: rows of 128 bytes (64 fp16), 8-row
// atoms of 1024 bytes (stride byte offset), start address 1024-aligned per tile.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFF);  // start address
  d |= (uint64_t)1 << 16;                 // leading byte offset (unused by swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;       // stride byte offset: one 8-row atom
  d |= (uint64_t)1 << 46;                 // descriptor version (Blackwell)
  d |= (uint64_t)2 << 61;                 // layout: 128-byte swizzle
  return d;
}

// fp32 accumulate, A and B both fp16 (bf16 = false) or both bf16, both K-major,
// N = BN = 256, M = 128
__host__ __device__ constexpr uint32_t instr_desc(bool bf16 = false) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((uint32_t)(BN >> 3) << 17) |
         ((uint32_t)(MH >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
               : "memory");
}

// Eight consecutive 4-bit codes of one word -> eight 16-bit (q - zero) * scale,
// in column order, as four packed pairs.
template <bool F16>
__device__ __forceinline__ void dequant8(uint32_t w, uint32_t zc, uint32_t sc, uint32_t (&out)[4]) {
  const uint32_t lo = w & 0x0F0F0F0Fu;          // codes 0, 2, 4, 6 in bytes 0..3
  const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;   // codes 1, 3, 5, 7
  const uint32_t c0123 = __byte_perm(lo, hi, 0x5140);  // bytes: q0 q1 q2 q3
  const uint32_t c4567 = __byte_perm(lo, hi, 0x7362);  // bytes: q4 q5 q6 q7
  constexpr uint32_t kMagic = F16 ? 0x64646464u : 0x43434343u;  // high byte of 1024 (fp16) / 128 (bf16)
  const uint32_t p01 = __byte_perm(c0123, kMagic, 0x4140);
  const uint32_t p23 = __byte_perm(c0123, kMagic, 0x4342);
  const uint32_t p45 = __byte_perm(c4567, kMagic, 0x4140);
  const uint32_t p67 = __byte_perm(c4567, kMagic, 0x4342);
  const uint32_t p[4] = {p01, p23, p45, p67};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t d;
    if constexpr (F16) {
      asm("sub.rn.f16x2 %0, %1, %2;\n" : "=r"(d) : "r"(p[i]), "r"(zc));
      asm("mul.rn.f16x2 %0, %1, %2;\n" : "=r"(out[i]) : "r"(d), "r"(sc));
    } else {
      asm("sub.rn.bf16x2 %0, %1, %2;\n" : "=r"(d) : "r"(p[i]), "r"(zc));
      asm("mul.rn.bf16x2 %0, %1, %2;\n" : "=r"(out[i]) : "r"(d), "r"(sc));
    }
  }
}

// Per-linear scalars of a launch, copied into shared memory at kernel start
// (the tile walk indexes linears by a runtime number).
struct TcMeta {
  const uint16_t* xraw;
  const unsigned short* sc;
  const unsigned short* z;
  __nv_bfloat16* y;
  int M, d_in, d_out, n_tiles, tile_begin;
};

// The j-th tile of this CTA, or -1: tiles go out in rounds of gridDim.x, in
// ascending CTA order on even rounds and descending order on odd ones, so that
// the CTAs given the first (longest) tiles get the last partial round least.
__device__ __forceinline__ int tile_of(int j, int total) {
  const int G = (int)gridDim.x, c = (int)blockIdx.x;
  const int t = j * G + ((j & 1) ? (G - 1 - c) : c);
  return t < total ? t : -1;
}
struct TileInfo {
  int pi, m0, n0, nk;
};
__device__ __forceinline__ TileInfo tile_info(const TcMeta* mt, int count, int t) {
  int pi = 0;
#pragma unroll 1
  while (pi + 1 < count && t >= mt[pi + 1].tile_begin) ++pi;
  const int local = t - mt[pi].tile_begin;
  const int mtile = local / mt[pi].n_tiles, ntile = local - mtile * mt[pi].n_tiles;
  return TileInfo{pi, mtile * BM, ntile * BN, mt[pi].d_in / BK};
}

// DENSE: the dense-rotation contrast (a d x d bf16 matrix instead of INT4
// weights): the TMA producer also loads the B tile (256 rows x 64 columns of
// the matrix, 128-byte swizzle) straight into the tensor core's layout, A is
// bf16 as given, and warps 0-15 only run the epilogue.
template <bool XF16, bool DENSE = false>
__global__ void __launch_bounds__(XF16 ? kThreadsTma : kThreadsConv, 1)
w4_tc_kernel(const __grid_constant__ TcBatch b, int* status) {
  static_assert(XF16 || !DENSE, "the dense form takes its A tile as given");
  constexpr bool F16 = true;  // tensor-core operands are fp16 in both INT4 variants
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t bars[5 * kStages + 2];
  __shared__ uint32_t tmem_base_slot;
  __shared__ int abort_flag;
  __shared__ int s_issued, s_committed;  // stages the TMA thread issued / the MMA thread committed
  __shared__ TcMeta meta[kTcMaxBatch];

  // the 128-byte swizzle needs every tile at a 1024-byte aligned shared address
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t s_base = smem_u32(smem);
  const uint32_t b_full_a = smem_u32(&bars[0]);
  const uint32_t b_full_b = smem_u32(&bars[kStages]);
  const uint32_t b_empty = smem_u32(&bars[2 * kStages]);
  const uint32_t b_full_c = smem_u32(&bars[3 * kStages]);    // codes of a stage landed
  const uint32_t b_acc_full = smem_u32(&bars[4 * kStages]);  // a tile's accumulator is complete
  const uint32_t b_acc_empty = smem_u32(&bars[4 * kStages + 1]);  // ... and has been read out
  const uint32_t b_full_raw = smem_u32(&bars[4 * kStages + 2]);   // bf16 activation tile landed

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = b.total_tiles, count = b.count;

  if (threadIdx.x < count) {
    const TcProblem& P = b.p[threadIdx.x];
    meta[threadIdx.x] = TcMeta{P.xraw, P.sc, P.z, P.y, P.M, P.d_in, P.d_out, P.n_tiles, P.tile_begin};
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&P.qmap)) : "memory");
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&P.xmap)) : "memory");
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(b_full_a + 8 * s, XF16 ? 1 : BM);
      mbar_init(b_full_b + 8 * s, DENSE ? 1 : kDqWarps * 32);
      mbar_init(b_empty + 8 * s, 1);
      mbar_init(b_full_c + 8 * s, 1);
      mbar_init(b_full_raw + 8 * s, 1);
    }
    mbar_init(b_acc_full, 1);
    mbar_init(b_acc_empty, kDqWarps * 32);
    abort_flag = 0;
    s_issued = 0;
    s_committed = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == kWarpTma) {  // tensor memory for the accumulators
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(&tmem_base_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  const uint32_t tmem = tmem_base_slot;

  auto fail = [&]() {
    report_status(status, kStatusTimeout);
    atomicExch(&abort_flag, 1);
  };
  auto aborted = [&]() { return *(volatile int*)&abort_flag != 0; };

  if (warp >= kWarpConv) {
    // ---------------- bf16 activations -> fp16, in place (bf16 input only) -----------
    // The TMA put the stage's bf16 tile in the A slot in the same swizzled layout
    // the tensor core reads; every 16-byte chunk holds 8 consecutive columns of
    // one token, so converting each chunk where it lies keeps the layout.
    if constexpr (!XF16) {
      const int t = threadIdx.x - kWarpConv * 32;  // 0 .. 255
      int it = 0;
      bool stop = false, ovf = false;
#pragma unroll 1
      for (int j = 0; !stop; ++j) {
        const int T = tile_of(j, total);
        if (T < 0) break;
        const TileInfo ti = tile_info(meta, count, T);
#pragma unroll 1
        for (int k = 0; k < ti.nk; ++k, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(b_full_raw + 8 * s, (it / kStages) & 1)) { fail(); stop = true; break; }
          if (aborted()) { stop = true; break; }
          const uint32_t a0 = s_base + (uint32_t)(s * STAGE_BYTES);
          uint32_t v[A_BYTES / 16 / (BM)][4];  // the chunks of this thread
#pragma unroll
          for (int q = 0; q < A_BYTES / 16 / BM; ++q) {
            const uint32_t a = a0 + (uint32_t)((t + q * BM) * 16);
            asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                         : "=r"(v[q][0]), "=r"(v[q][1]), "=r"(v[q][2]), "=r"(v[q][3]) : "r"(a) : "memory");
          }
#pragma unroll
          for (int q = 0; q < A_BYTES / 16 / BM; ++q) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v[q][e]));
              const __half2 h = __floats2half2_rn(f.x, f.y);
              v[q][e] = *reinterpret_cast<const uint32_t*>(&h);
              ovf |= half2_inf(v[q][e]);
            }
            const uint32_t a = a0 + (uint32_t)((t + q * BM) * 16);
            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(a), "r"(v[q][0]), "r"(v[q][1]), "r"(v[q][2]),
                         "r"(v[q][3])
                         : "memory");
          }
          asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
          mbar_arrive(b_full_a + 8 * s);
        }
      }
      // a bf16 input beyond the fp16 range became infinite (the rows past M are
      // zero-filled by the copy, so this is always a real input)
      if (ovf) report_status(status, kStatusRange);
    }
  } else if (warp == kWarpTma) {
    // ---------------- TMA producer: packed codes (both variants), fp16 activations ---
    if (lane == 0) {
      int it = 0;
      bool stop = false;
#pragma unroll 1
      for (int j = 0; !stop; ++j) {
        const int T = tile_of(j, total);
        if (T < 0) break;
        const TileInfo ti = tile_info(meta, count, T);
        const TcProblem& P = b.p[ti.pi];
#pragma unroll 1
        for (int k = 0; k < ti.nk; ++k, ++it) {
          const int s = it % kStages;
          if (it >= kStages && !mbar_wait(b_empty + 8 * s, ((it / kStages) - 1) & 1)) { fail(); stop = true; break; }
          if (aborted()) { stop = true; break; }
          if constexpr (DENSE) {
            // the matrix tile goes straight into the B slot
            mbar_expect_tx(b_full_b + 8 * s, B_BYTES);
            tma_load_2d(s_base + s * STAGE_BYTES + A_BYTES, &P.qmap, k * BK, ti.n0, b_full_b + 8 * s);
          } else {
            mbar_expect_tx(b_full_c + 8 * s, C_BYTES);
            tma_load_2d(s_base + s * STAGE_BYTES + A_BYTES + B_BYTES, &P.qmap, k * (BK / 8), ti.n0,
                        b_full_c + 8 * s);
          }
          // fp16 activations complete the stage's A tile; bf16 ones land first and
          // are converted in place by the conversion warps
          const uint32_t bar_a = XF16 ? b_full_a + 8 * s : b_full_raw + 8 * s;
          mbar_expect_tx(bar_a, A_BYTES);
          tma_load_2d(s_base + s * STAGE_BYTES, &P.xmap, k * BK, ti.m0, bar_a);
        }
      }
      s_issued = it;
    }
  } else if (warp == kWarpMma) {
    // ---------------- MMA issuer ---------------------------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc(DENSE);
      int it = 0;
      bool ok = true;
#pragma unroll 1
      for (int j = 0; ok; ++j) {
        const int T = tile_of(j, total);
        if (T < 0) break;
        const TileInfo ti = tile_info(meta, count, T);
        // the previous tile's accumulators must have been read out
        if (j > 0 && !mbar_wait(b_acc_empty, (j - 1) & 1)) { fail(); ok = false; break; }
        asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
#pragma unroll 1
        for (int k = 0; k < ti.nk; ++k, ++it) {
          const int s = it % kStages;
          const uint32_t par = (it / kStages) & 1;
          if (!mbar_wait(b_full_a + 8 * s, par) || !mbar_wait(b_full_b + 8 * s, par)) { fail(); ok = false; break; }
          if (aborted()) { ok = false; break; }
          asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
          const uint32_t a_addr = s_base + s * STAGE_BYTES, b_addr = a_addr + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 32);
#pragma unroll
            for (int h = 0; h < BM / MH; ++h)  // token half h -> accumulator columns [h * BN, (h + 1) * BN)
              mma_f16(tmem + h * BN, smem_desc_sw128(a_addr + h * (MH * 128) + kk * 32), bdesc, idesc,
                      (k > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(b_empty + 8 * s);
        }
        if (ok) mma_commit(b_acc_full);  // arrives once every MMA of the tile has completed
      }
      s_committed = it;
    }
  } else {
    // ---------------- dequantisation (warps 0-15), then each tile's epilogue ----------
    const int t = threadIdx.x & (BN - 1);  // row of the tile
    const int hw = threadIdx.x / BN;        // which half of the row's 64 columns (4 words)
    // this thread's 16 bytes of a stage's codes: row t holds 32 bytes, its
    // 16-byte halves swapped on rows with bit 2 set (the 32-byte swizzle)
    const uint32_t c_off = (uint32_t)(A_BYTES + B_BYTES + t * 32 + ((hw ^ ((t >> 2) & 1)) << 4));
    constexpr int SPG = kGroup / BK;  // steps per group
    constexpr int PD = 4;             // groups of scale/zero bits in flight
    int it = 0;
    bool stop = false;
#pragma unroll 1
    for (int j = 0; !stop; ++j) {
      const int T = tile_of(j, total);
      if (T < 0) break;
      const TileInfo ti = tile_info(meta, count, T);
      const TcMeta& P = meta[ti.pi];
      if constexpr (!DENSE) {
      const int G = P.d_in / kGroup;
      const int rA = ti.n0 + t;
      const bool okA = rA < P.d_out;
      const unsigned short* sA = P.sc + (size_t)(okA ? rA : 0) * G;
      const unsigned short* zA = P.z + (size_t)(okA ? rA : 0) * G;
      uint32_t sz[PD][2];
      auto load_group = [&](int g, uint32_t (&z)[2]) {
        if (g < G && okA) {
          z[0] = __ldg(sA + g);
          z[1] = __ldg(zA + g);
        }
      };
#pragma unroll
      for (int q = 0; q < PD - 1; ++q) load_group(q, sz[q]);
#pragma unroll 1
      for (int kb = 0; kb < ti.nk && !stop; kb += PD * SPG) {
#pragma unroll
        for (int q = 0; q < PD * SPG; ++q) {
          const int k = kb + q;
          if (k >= ti.nk) break;
          const int gj = q / SPG;  // ring slot of this step's group
          if (q % SPG == 0) load_group(k / SPG + PD - 1, sz[(gj + PD - 1) % PD]);
          const int s = it % kStages;
          const uint32_t par = (it / kStages) & 1;
          if (it >= kStages && !mbar_wait(b_empty + 8 * s, par ^ 1)) fail();
          if (!mbar_wait(b_full_c + 8 * s, par)) fail();
          if (aborted()) { stop = true; break; }
          uint32_t zc = 0, sc = 0;
          if (okA) {
            const float z = __half2float(__ushort_as_half((unsigned short)sz[gj][1]));
            const __half2 zz = __float2half2_rn(1024.f + z);
            zc = *reinterpret_cast<const uint32_t*>(&zz);
            sc = (sz[gj][0] & 0xFFFFu) * 0x00010001u;
          }
          uint32_t wv[4];
          {
            const uint32_t a = s_base + (uint32_t)(s * STAGE_BYTES) + c_off;
            asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                         : "=r"(wv[0]), "=r"(wv[1]), "=r"(wv[2]), "=r"(wv[3]) : "r"(a) : "memory");
          }
          unsigned char* rowp = smem + s * STAGE_BYTES + A_BYTES + t * 128;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {  // 16-byte chunk = 8 columns = one word
            const int c = hw * 4 + c4;
            uint32_t o[4] = {0u, 0u, 0u, 0u};
            if (okA) dequant8<F16>(wv[c4], zc, sc, o);
            *reinterpret_cast<uint4*>(rowp + ((c ^ (t & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
          }
          asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // generic writes -> tensor core reads
          mbar_arrive(b_full_b + 8 * s);
          ++it;
        }
      }
      }  // !DENSE
      if (stop) break;

      // ---------------- epilogue of this tile --------------------------------------
      if (!mbar_wait(b_acc_full, j & 1)) { fail(); break; }
      asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
      if (!aborted()) {
        const int q = warp & 3;                 // TMEM lane quarter this warp may access
        const int h = (warp >> 2) & 1;          // token half (accumulator) this warp drains
        const int cb = (warp >> 3) * (BN / 2);  // and which half of its columns
        const int m = ti.m0 + h * MH + q * 32 + lane;  // token of this thread's TMEM lane
        const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * BN + cb);
#pragma unroll 1
        for (int c0 = 0; c0 < BN / 2; c0 += 32) {
          uint32_t v[32];
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
              "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
              : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
                "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
                "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
                "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
              : "r"(taddr + c0));
          asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
          const int n = ti.n0 + cb + c0;  // first output column of this chunk
          if (m < P.M && n < P.d_out) {
            __nv_bfloat16* dst = P.y + (size_t)m * P.d_out + n;
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const __nv_bfloat162 b2 =
                  __floats2bfloat162_rn(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
              pk[i] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            // d_out is a multiple of 16: the last 32-column chunk may hold only 16
            const int nq = (n + 32 <= P.d_out) ? 4 : 2;
#pragma unroll
            for (int i = 0; i < 4; ++i)
              if (i < nq)
                reinterpret_cast<uint4*>(dst)[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
      }
      asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
      mbar_arrive(b_acc_empty);  // the MMA warp may overwrite the accumulators
    }
  }

  // ---------------- teardown --------------------------------------------------------
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  if (abort_flag && threadIdx.x == 0) {
    // let the copies and MMAs still in flight land before the memory goes away:
    // per slot, the phase of the last copy issued into it and of the last MMA
    // commit that read it (earlier phases have completed before those could be
    // issued); a wait that gives up again is reported again
    const uint32_t bar_a = XF16 ? b_full_a : b_full_raw;
    const uint32_t bar_w = DENSE ? b_full_b : b_full_c;  // the weight tile's copy
    auto last_of = [](int n, int slot) { return n > slot ? slot + ((n - 1 - slot) / kStages) * kStages : -1; };
    for (int s = 0; s < kStages; ++s) {
      const int jt = last_of(s_issued, s), jm = last_of(s_committed, s);
      bool landed = true;
      if (jt >= 0) {
        const uint32_t par = (uint32_t)((jt / kStages) & 1);
        landed = mbar_wait(bar_a + 8 * s, par) && mbar_wait(bar_w + 8 * s, par);
      }
      if (jm >= 0) landed = mbar_wait(b_empty + 8 * s, (uint32_t)((jm / kStages) & 1)) && landed;
      if (!landed) report_status(status, kStatusTimeout);
    }
  }
  __syncthreads();
  if (warp == kWarpTma) {
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
  static EncodeTiled fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(p);
  }
  return fn;
}

}  // namespace

bool tc_supported(int M, int d_in, int d_out, const void* x) {
  return M >= 128 && d_in % BK == 0 && d_out % 16 == 0 && (reinterpret_cast<uintptr_t>(x) & 15) == 0 &&
         ((size_t)d_in * 2) % 16 == 0;
}

namespace {
struct ConvBatch {
  const uint4* src[kMaxBatch];
  uint4* dst[kMaxBatch];
  size_t begin[kMaxBatch + 1];  // prefix sums of the arrays' 8-value chunks
  int count;
};

__global__ void __launch_bounds__(256) to_f16_kernel(const __grid_constant__ ConvBatch b, int* status) {
  // every thread takes four chunks 'stride' apart per round, their loads issued
  // before any is converted, so that enough bytes are in flight
  const size_t total = b.begin[b.count], stride = (size_t)gridDim.x * blockDim.x;
  bool ovf = false;
  for (size_t i0 = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i0 < total; i0 += 4 * stride) {
    uint4 v[4];
    int a[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const size_t i = i0 + u * stride;
      a[u] = 0;
      v[u] = make_uint4(0u, 0u, 0u, 0u);
      if (i < total) {
        while (a[u] + 1 < b.count && i >= b.begin[a[u] + 1]) ++a[u];
        v[u] = __ldcs(b.src[a[u]] + (i - b.begin[a[u]]));
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const size_t i = i0 + u * stride;
      if (i >= total) continue;
      uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
        const __half2 h = __floats2half2_rn(f.x, f.y);
        w[e] = *reinterpret_cast<const uint32_t*>(&h);
        ovf |= half2_inf(w[e]);
      }
      b.dst[a[u]][i - b.begin[a[u]]] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  if (ovf) report_status(status, kStatusRange);
}
}  // namespace

cudaError_t launch_to_f16(const uint16_t* const* src, uint16_t* const* dst, const size_t* n, int count, int* status,
                          cudaStream_t stream) {
  if (count < 1 || count > kMaxBatch) return cudaErrorInvalidValue;
  ConvBatch b = {};
  b.count = count;
  for (int i = 0; i < count; ++i) {
    if (n[i] % 8 || (reinterpret_cast<uintptr_t>(src[i]) | reinterpret_cast<uintptr_t>(dst[i])) & 15)
      return cudaErrorInvalidValue;
    b.src[i] = reinterpret_cast<const uint4*>(src[i]);
    b.dst[i] = reinterpret_cast<uint4*>(dst[i]);
    b.begin[i + 1] = b.begin[i] + n[i] / 8;
  }
  const size_t chunks = b.begin[count];
  if (chunks == 0) return cudaSuccess;
  const size_t want = (chunks + 1023) / 1024, cap = (size_t)device_sm_count() * 8;
  to_f16_kernel<<<(unsigned)(want < cap ? want : cap), 256, 0, stream>>>(b, status);
  return cudaGetLastError();
}

cudaError_t launch_w4_tc_batch(const TcLinear* lins, int count, bool x_f16, int* status, cudaStream_t stream) {
  if (count < 1 || count > kTcMaxBatch) return cudaErrorInvalidValue;
  EncodeTiled enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  // the linears with the longest K (slowest tiles) first, otherwise in call order
  int order[kTcMaxBatch];
  for (int i = 0; i < count; ++i) {
    int j = i;
    while (j > 0 && lins[order[j - 1]].d_in < lins[i].d_in) {
      order[j] = order[j - 1];
      --j;
    }
    order[j] = i;
  }
  TcBatch b{};
  int tiles = 0;
  const cuuint32_t elem[2] = {1, 1};
  for (int oi = 0; oi < count; ++oi) {
    const TcLinear& L = lins[order[oi]];
    if (!tc_supported(L.M, L.d_in, L.d_out, L.x)) return cudaErrorInvalidValue;
    TcProblem& P = b.p[oi];
    {  // activations [M][d_in]: box 64 columns x 256 tokens, 128-byte swizzle
      const cuuint64_t dims[2] = {(cuuint64_t)L.d_in, (cuuint64_t)L.M};
      const cuuint64_t strides[1] = {(cuuint64_t)L.d_in * 2};
      const cuuint32_t box[2] = {BK, BM};
      if (enc(&P.xmap, x_f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
              const_cast<uint16_t*>(L.x), dims, strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
    {  // packed codes uint32 [d_out][d_in / 8]: box 8 words x 256 rows, 32-byte swizzle
      const cuuint64_t dims[2] = {(cuuint64_t)(L.d_in / 8), (cuuint64_t)L.d_out};
      const cuuint64_t strides[1] = {(cuuint64_t)L.d_in / 2};
      const cuuint32_t box[2] = {BK / 8, BN};
      if (enc(&P.qmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(L.qweight), dims, strides, box,
              elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
    P.xraw = L.x;
    P.sc = reinterpret_cast<const unsigned short*>(L.scales);
    P.z = reinterpret_cast<const unsigned short*>(L.zeros);
    P.y = L.y;
    P.M = L.M;
    P.d_in = L.d_in;
    P.d_out = L.d_out;
    P.n_tiles = (L.d_out + BN - 1) / BN;
    P.tile_begin = tiles;
    tiles += ((L.M + BM - 1) / BM) * P.n_tiles;
  }
  b.count = count;
  b.total_tiles = tiles;
  const int sms = device_sm_count();
  const int grid = tiles < sms ? tiles : sms;
  cudaError_t e;
  if (x_f16) {
    e = cudaFuncSetAttribute(w4_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    w4_tc_kernel<true><<<grid, kThreadsTma, SMEM_BYTES, stream>>>(b, status);
  } else {
    e = cudaFuncSetAttribute(w4_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    w4_tc_kernel<false><<<grid, kThreadsConv, SMEM_BYTES, stream>>>(b, status);
  }
  return cudaPeekAtLastError();
}

bool dense_supported(int M, int d, const void* x, const void* q) {
  return M >= 1 && d >= BK && d % BK == 0 && (reinterpret_cast<uintptr_t>(x) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(q) & 15) == 0;
}

cudaError_t launch_dense_tc(const uint16_t* x, const uint16_t* q, __nv_bfloat16* y, int M, int d, int* status,
                            cudaStream_t stream) {
  if (!dense_supported(M, d, x, q)) return cudaErrorInvalidValue;
  EncodeTiled enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  TcBatch b{};
  TcProblem& P = b.p[0];
  const cuuint32_t elem[2] = {1, 1};
  {  // bf16 activations [M][d]: box 64 columns x 256 tokens, 128-byte swizzle
    const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    const cuuint32_t box[2] = {BK, BM};
    if (enc(&P.xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(x), dims, strides, box, elem,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {  // bf16 matrix [d][d] (row n = output channel n): box 64 columns x 256 rows, 128-byte swizzle
    const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)d};
    const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    const cuuint32_t box[2] = {BK, BN};
    if (enc(&P.qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(q), dims, strides, box, elem,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  P.xraw = x;
  P.y = y;
  P.M = M;
  P.d_in = d;
  P.d_out = d;
  P.n_tiles = (d + BN - 1) / BN;
  P.tile_begin = 0;
  b.count = 1;
  b.total_tiles = ((M + BM - 1) / BM) * P.n_tiles;
  const int sms = device_sm_count();
  const int grid = b.total_tiles < sms ? b.total_tiles : sms;
  cudaError_t e = cudaFuncSetAttribute(w4_tc_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       SMEM_BYTES);
  if (e != cudaSuccess) return e;
  w4_tc_kernel<true, true><<<grid, kThreadsTma, SMEM_BYTES, stream>>>(b, status);
  return cudaPeekAtLastError();
}

cudaError_t launch_w4_tc(const uint16_t* x, bool x_f16, const uint32_t* qweight, const __half* scales,
                         const __half* zeros, __nv_bfloat16* y, int M, int d_in, int d_out, int* status,
                         cudaStream_t stream) {
  const TcLinear L{x, qweight, scales, zeros, y, M, d_in, d_out};
  return launch_w4_tc_batch(&L, 1, x_f16, status, stream);
}

}  // namespace paro
