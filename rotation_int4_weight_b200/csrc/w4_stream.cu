// Group-wise INT4 weight-only linear for few tokens (decode), stream-K form:
//   y[m][n] = sum_k w^[n][k] x[m][k],  w^ = (q - zero) * scale per group of 128 input columns
// (page "ParoQuant: pairwise rotations that survive deployment", section "From fake
// quantization to a real TensorRT engine": the group-wise INT4 GEMM operator).
//
// With one to sixteen tokens a linear is a stream of packed weights, and a
// decoder layer's worth of them (tens of MB) lasts only a few microseconds on
// the whole GPU, so the time goes to filling the memory pipeline and to uneven
// work.  This kernel therefore splits the weight bytes of all the linears of
// a launch evenly:
//   unit   = one 64-row tile x one 128-column group (4 KB of codes), numbered
//            linear by linear, tile by tile, group by group;
//   CTA c  = the contiguous units [c U / C, (c + 1) U / C), one CTA per SM;
//   warp w = a contiguous eighth of its CTA's units.
// Every warp streams its units through a private ring of D slots: one elected
// lane issues a TMA tile load of the unit's codes (64 rows x 64 bytes) and two
// of its activations (the 128 columns of every token, 128-byte swizzle), all
// completing on the slot's mbarrier; scales and zeros come into registers with
// the loads of the same unit.  So a warp keeps D units (16 KB of codes) in
// flight and an SM about 128 KB.
//
// Arithmetic, per unit and warp: the codes are the MMA's 16-row side and the
// tokens its 8-column side (mma.sync m16n8k16, fp32 accumulation).  OR-ing a
// nibble into the mantissa of 1024 (fp16) or 128 (bf16) gives bias + q exactly;
// odd nibbles stay in place (x16, or moved one bit: x8) and their activations
// are pre-divided to match.  One MMA per k-step with constant operands yields,
// per token, Tb = sum(bias x) in its upper rows and Sx = sum x in its lower
// rows, shared by the four 16-row tiles of the unit, so
//   sum (q - z) x = R - Tb - z Sx,  R = the code MMAs' result,
// and the group scale multiplies that once, all in fp32.
//
// Partial sums.  A tile wholly inside one warp's units is written by that warp.
// A tile split between warps of a CTA is summed in shared memory at the end, in
// warp order.  A tile split between CTAs goes through the workspace: every CTA
// holding part of it but the last writes its partial tile, each fp32 value in
// a 64-bit word beside this launch's tag (the low 32 bits of 2E + 1 for the
// workspace's launch epoch E: a word left by another launch or by an earlier
// replay of the same CUDA graph, or never written, holds another tag, since
// the last CTA of every launch advances E; the workspace needs clearing only
// once, before its first use); the tile's last CTA reads the earlier CTAs'
// partials, which were launched no later than it, until every word carries
// the tag (bounded), and sums them in CTA order.  A word is written and read
// as a whole, so its tag vouches for its value: no flag after the values and
// no fence between them, which would cost two more round trips to memory at
// the end of a launch.  (A word left exactly a multiple of 2^31 launches
// earlier would pass for current; a workspace never sees that many launches
// between two uses of a slot in practice.)  Every sum has a fixed order, so
// the result does not depend on timing.
#include "paro_internal.cuh"
#include "w4_stream.cuh"
#include "rotate_decode_cta.cuh"

#ifdef PARO_TIMELINE
// Instrumented build only: per CTA of the fused one-token launch, global-timer
// stamps in ns, in one of two slots chosen by the launch epoch's parity (so the
// last two launches on a workspace are kept).  A transform CTA writes
// {entry, wait done, rows staged, stages done, flag published, 1, 0, 0}; an
// INT4 CTA {entry, wait done, warp 0's first unit landed, units done, end
// (latest warp), 2, warp 0's units, linear of its last tile}.
constexpr int kTimelineCtas = 256;
__device__ unsigned long long g_paro_timeline[2][kTimelineCtas][8];
extern "C" PARO_API int paro_timeline_read(void* host, size_t bytes) {
  if (bytes < sizeof(g_paro_timeline)) return (int)PARO_ERR_INVALID_ARG;
  return cudaMemcpyFromSymbol(host, g_paro_timeline, sizeof(g_paro_timeline)) == cudaSuccess ? 0 : (int)PARO_ERR_CUDA;
}
#define PARO_TL_NOW(v) v = rotdec::tl_now()
#else
#define PARO_TL_NOW(v)
#endif

namespace paro {
namespace {

// Warps per CTA and ring slots per warp, for one (NT = 1) and two (NT = 2)
// 8-token column tiles; a CTA's registers and shared memory bound both.  One
// token tile: 16 warps of two slots (128 registers a thread) hide the
// latency of the dequantise-and-MMA chains better than 12 warps of three
// (Llama-3-8B layer at M = 1: 47.3 against 50.6 us; Qwen2.5-1.5B: 19.3 against 21.4).
#ifndef PARO_STREAM_W1
#define PARO_STREAM_W1 16
#endif
#ifndef PARO_STREAM_D1
#define PARO_STREAM_D1 2
#endif
#ifndef PARO_STREAM_W2
#define PARO_STREAM_W2 8
#endif
#ifndef PARO_STREAM_D2
#define PARO_STREAM_D2 3
#endif
// CTAs of the one-token-tile kernel resident per SM (their registers and rings
// must fit together)
#ifndef PARO_STREAM_CPS1
#define PARO_STREAM_CPS1 1
#endif
// ring slots per warp when every linear of the launch has one token, and
// whether that geometry is used at all
#ifndef PARO_STREAM_D0
#define PARO_STREAM_D0 2
#endif
#ifndef PARO_STREAM_ONE
#define PARO_STREAM_ONE 1
#endif
constexpr int kUnitBytes = kStreamRows * 64;  // 64 rows x 128 codes

// ONE: every linear has a single token.  Its activations for a unit are then
// one unswizzled 128-column box of 256 bytes (the 128-byte swizzle only
// spreads 8 token rows over the banks): one copy instead of two, and a slot of
// 4352 bytes instead of 6144.  (Three slots a warp were measured slower than
// two on the Llama-3-8B-shaped layer: 45.7 against 39.2 us.)
template <int NT, bool ONE = false>
struct Geo {
  static_assert(!ONE || NT == 1, "one token is one token tile");
  static constexpr int W = NT == 1 ? PARO_STREAM_W1 : PARO_STREAM_W2;  // warps per CTA
  static constexpr int D = ONE ? PARO_STREAM_D0 : (NT == 1 ? PARO_STREAM_D1 : PARO_STREAM_D2);  // ring slots
  // bytes per activation half-box slot (>= 128 M, 1024-aligned under the swizzle)
  static constexpr int XB = ONE ? 128 : (NT == 1 ? 1024 : 2048);
  static constexpr int SLOT = kUnitBytes + 2 * XB;
  static constexpr int PF = 4 * NT * 32 * 4;        // floats of one tile partial (fragment order)
  static constexpr int SMEM = W * D * SLOT + 1024;
  static constexpr int CPS = NT == 1 ? PARO_STREAM_CPS1 : 1;  // CTAs per SM
  static_assert(2 * PF * 4 <= D * SLOT, "a warp's two partial tiles fit in its ring");
  static_assert(SMEM * CPS <= 227 * 1024, "rings exceed shared memory");
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
// adds expected transaction bytes to the current phase without arriving
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
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
// the same with an L2 eviction policy (the packed weights: read once per call,
// fetched evict-first so that they do not push the layer tables out of L2)
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint32_t bar,
                                            uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, "
      "%3}], [%4], %5;\n"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar), "l"(pol)
      : "memory");
}
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ float4 lds128f(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];\n" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts128f(uint32_t addr, float4 v) {
  asm volatile("st.shared.v4.f32 [%0], {%1,%2,%3,%4};\n" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
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
// (a & mask) | bias as one three-input logic operation
template <uint32_t MASK, uint32_t BIAS>
__device__ __forceinline__ uint32_t and_or(uint32_t a) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;\n" : "=r"(d) : "r"(a), "n"(MASK), "n"(BIAS));
  return d;
}
template <bool F16>
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t (&P)[4]) {
  if constexpr (F16) {
    const uint32_t w2 = w >> 8;
    P[0] = and_or<0x000F000Fu, 0x64006400u>(w);
    P[1] = and_or<0x00F000F0u, 0x64006400u>(w);
    P[2] = and_or<0x000F000Fu, 0x64006400u>(w2);
    P[3] = and_or<0x00F000F0u, 0x64006400u>(w2);
  } else {
    P[0] = and_or<0x000F000Fu, 0x43004300u>(w);
    P[1] = and_or<0x00780078u, 0x43004300u>(w >> 1);
    P[2] = and_or<0x000F000Fu, 0x43004300u>(w >> 8);
    P[3] = and_or<0x00780078u, 0x43004300u>(w >> 9);
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

// ---- the unit sequence ----------------------------------------------------------
struct Cur {
  int pi, tile, grp;
};
// The scalar fields of a StreamProblem, copied into shared memory at kernel
// start: the unit walk indexes problems by a runtime number, and shared memory
// serves such loads without the dependent round trips of kernel parameters.
struct Meta {
  long long unit_begin;
  const unsigned short* sc;
  const unsigned short* z;
  __nv_bfloat16* y;
  int M, d_out, G, tiles, tile_begin;
};
__device__ __forceinline__ void cur_at(const Meta* mp, int count, long long u, Cur& c) {
  int pi = 0;
#pragma unroll 1
  while (pi + 1 < count && u >= mp[pi + 1].unit_begin) ++pi;
  const uint32_t local = (uint32_t)(u - mp[pi].unit_begin);
  c.pi = pi;
  c.tile = (int)(local / (uint32_t)mp[pi].G);
  c.grp = (int)(local - (uint32_t)c.tile * (uint32_t)mp[pi].G);
}
__device__ __forceinline__ void cur_next(const Meta* mp, Cur& c) {
  if (++c.grp == mp[c.pi].G) {
    c.grp = 0;
    if (++c.tile == mp[c.pi].tiles) {
      c.tile = 0;
      ++c.pi;
    }
  }
}
// first unit of part i when U units are cut into P contiguous parts (32-bit:
// a launch has fewer than 2^31 / 2^12 units, and i, P are at most a few hundred)
__device__ __forceinline__ long long part_start(long long i, long long P, long long U) {
  return (long long)((uint32_t)i * (uint32_t)U / (uint32_t)P);
}
// the part holding unit x
__device__ __forceinline__ long long part_of(long long x, long long P, long long U) {
  return (long long)((((uint32_t)x + 1u) * (uint32_t)P - 1u) / (uint32_t)U);
}

// lane (g, t) fetches one 16-bit value per row tile: t = 0 scale of row g, t = 1
// scale of row g + 8, t = 2 zero of row g, t = 3 zero of row g + 8 (rows past
// d_out read as 0); the four are gathered with shuffles when the unit is computed
__device__ __forceinline__ void load_sz(const Meta& P, const Cur& c, int g, int t, uint32_t (&r)[4]) {
  const unsigned short* src = (t & 2) ? P.z : P.sc;
#pragma unroll
  for (int rt = 0; rt < 4; ++rt) {
    const int row = c.tile * kStreamRows + rt * 16 + g + (t & 1) * 8;
    r[rt] = row < P.d_out ? (uint32_t)__ldg(src + (size_t)row * P.G + c.grp) : 0u;
  }
}

template <int NT>
__device__ __forceinline__ void store_tile(const Meta& P, int tile, int g, int t,
                                           const float (&v)[4][NT][4]) {
#pragma unroll
  for (int rt = 0; rt < 4; ++rt) {
    const int r0 = tile * kStreamRows + rt * 16 + g;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int m0 = n * 8 + 2 * t;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = r0 + (e >> 1) * 8, m = m0 + (e & 1);
        if (row < P.d_out && m < P.M) P.y[(size_t)m * P.d_out + row] = __float2bfloat16_rn(v[rt][n][e]);
      }
    }
  }
}

// This launch's tag, 2E + 1 for the workspace's launch epoch E read after the
// launch's dependency point (the previous launch on the workspace has then
// completed, and no CTA of this launch advances E before every CTA has read
// it): a flag holding it was written by this launch; a word left by an earlier
// launch, by an earlier replay of the same graph, or never written (zero)
// holds another value.
__device__ __forceinline__ unsigned long long launch_tag(const unsigned long long* ctl) {
  unsigned long long e;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];\n" : "=l"(e) : "l"(ctl) : "memory");
  return 2ull * e + 1ull;
}
// Every CTA of a launch that has a workspace counts itself once, after it has
// read the epoch: the CTA that completes the count advances the epoch (the
// count wraps back to zero).  The INT4 CTAs count themselves after their units
// (inline in the kernel, so that the count's round trip overlaps their
// combine); a transform CTA of the fused form, or a CTA that gave up, calls
// this at its end.
__device__ __forceinline__ void finish_cta(unsigned long long* ctl) {
  if (!ctl) return;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned old = atomicInc(reinterpret_cast<unsigned*>(ctl + 1), gridDim.x - 1);
    if (old == gridDim.x - 1) atomicAdd(ctl, 1ull);
  }
}
__device__ __forceinline__ void st_flag(unsigned long long* f, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;\n" ::"l"(f), "l"(v) : "memory");
}
// Bounded wait (at most `limit` SM clock cycles; about a second by default)
// for a flag to hold v.
__device__ bool wait_flag(const unsigned long long* f, unsigned long long v, long long limit) {
  const long long t0 = clock64();
#pragma unroll 1
  while (true) {
    unsigned long long x;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];\n" : "=l"(x) : "l"(f) : "memory");
    if (x == v) return true;
    if (clock64() - t0 > limit) return false;
    __nanosleep(64);
  }
}

// Two tagged values (a 16-byte store of two 64-bit words, each written as a whole).
__device__ __forceinline__ void st_tagged(unsigned long long* p, float a, float b, uint32_t tag) {
  const unsigned long long wa = ((unsigned long long)tag << 32) | __float_as_uint(a);
  const unsigned long long wb = ((unsigned long long)tag << 32) | __float_as_uint(b);
  asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %2};\n" ::"l"(p), "l"(wa), "l"(wb) : "memory");
}
// Adds another CTA's tagged partial tile (this lane's 4 NT words of 4 values) to
// tot once every word of every lane carries `tag`; reads again (bounded by
// `limit` SM cycles, lane 0's clock deciding for the warp) until then.
template <int NT>
__device__ bool add_tagged(const unsigned long long* src, int lane, uint32_t tag, long long limit,
                           float (&tot)[4][NT][4]) {
  const long long t0 = clock64();
#pragma unroll 1
  while (true) {
    unsigned long long w[4][NT][4];
    bool mine = true;
#pragma unroll
    for (int rt = 0; rt < 4; ++rt)
#pragma unroll
      for (int m = 0; m < NT; ++m) {
        const unsigned long long* q = src + (size_t)(((rt * NT + m) * 32 + lane) * 4);
        asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];\n"
                     : "=l"(w[rt][m][0]), "=l"(w[rt][m][1]) : "l"(q) : "memory");
        asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];\n"
                     : "=l"(w[rt][m][2]), "=l"(w[rt][m][3]) : "l"(q + 2) : "memory");
      }
#pragma unroll
    for (int rt = 0; rt < 4; ++rt)
#pragma unroll
      for (int m = 0; m < NT; ++m)
#pragma unroll
        for (int e = 0; e < 4; ++e) mine = mine && (uint32_t)(w[rt][m][e] >> 32) == tag;
    if (__all_sync(0xffffffffu, mine)) {
#pragma unroll
      for (int rt = 0; rt < 4; ++rt)
#pragma unroll
        for (int m = 0; m < NT; ++m)
#pragma unroll
          for (int e = 0; e < 4; ++e) tot[rt][m][e] += __uint_as_float((uint32_t)w[rt][m][e]);
      return true;
    }
    int late = clock64() - t0 > limit ? 1 : 0;
    if (__shfl_sync(0xffffffffu, late, 0)) return false;
    __nanosleep(64);
  }
}

// FU > 0: the fused form (one token per linear): CTAs 0 .. rb.count - 1 run the
// activation transform of one linear each, FU pairs per thread and round, and
// publish a flag holding this launch's tag once its x~ is written; the INT4
// CTAs request a linear's activations only after its flag.
// FU < 0: the flag form: the transform ran in the launch just before and its
// CTAs publish flags holding the same launch tag (read from the workspace's
// epoch after the previous INT4 launch completed); the INT4 CTAs request a
// linear's activations once all its transform CTAs have published (and do not
// wait for the whole launch).
// XPERM: the fp16 activations were written by this library's decode transform
// in the MMA's operand order (every 8-column block as x0, x4, x1/16, x5/16, x2,
// x6, x3/16, x7/16), so a 16-byte chunk is a ready B fragment; the fused and
// flag forms always take them so.
template <bool F16, int NT, int FU, bool XPERM, bool ONE>
__global__ void __launch_bounds__(Geo<NT, ONE>::W * 32, Geo<NT, ONE>::CPS)
w4_stream_kernel(const __grid_constant__ StreamBatch b, const __grid_constant__ RotBatch rb, int* status,
                 int pdl_wait) {
  static_assert(!XPERM || F16, "the operand-order layout is fp16");
  using Gm = Geo<NT, ONE>;
  constexpr int W = Gm::W, D = Gm::D, SLOT = Gm::SLOT, XB = Gm::XB, PF = Gm::PF;
  extern __shared__ unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t bars[W * D];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#ifdef PARO_TIMELINE
  unsigned long long tl_entry = 0, tl_wait = 0, tl_first = 0, tl_loop = 0;
  PARO_TL_NOW(tl_entry);
#endif
  // flag form: the preceding transform let this grid launch only after it had
  // waited for the previous launch, so the epoch is already this launch's
  unsigned long long ltag = 0;
  if constexpr (FU < 0) ltag = launch_tag(b.ctl);
  // a programmatic dependent (the next call's transform) may start its table
  // fetches as SMs free up; it waits for this grid before touching its data
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  const int T = FU > 0 ? rb.count : 0;  // transform CTAs
  if constexpr (FU > 0) {
    if ((int)blockIdx.x < T) {
      __shared__ __align__(8) uint64_t tbars[rotdec::kRotBars];
      // pairs per thread and round: enough that a stage of this linear is one
      // round of loads and stores where the registers allow (wider ones take two)
      const RotProblem& Pt = rb.p[blockIdx.x];
      unsigned char* ts = smem_raw + (sbase - smem_u32(smem_raw));
      const int rounds = (Pt.d / 2 + W * 32 - 33) / (W * 32 - 32);
      // the launch epoch for the flag, read by thread 0 right after the wait
      // for the previous launch
      const unsigned long long* ep = b.ctl && !rb.skip_flags ? b.ctl : nullptr;
      unsigned long long e = 0;
      bool done;
      if (rounds <= 2)
        done = rotdec::rot_decode_cta<1, true, 2, W * 32>(Pt, 0, ts, tbars, status, pdl_wait != 0, false, ep, &e);
      else if (rounds <= 5)
        done = rotdec::rot_decode_cta<1, true, 5, W * 32>(Pt, 0, ts, tbars, status, pdl_wait != 0, false, ep, &e);
      else if (rounds <= 10)
        done = rotdec::rot_decode_cta<1, true, 10, W * 32>(Pt, 0, ts, tbars, status, pdl_wait != 0, false, ep, &e);
      else
        done = rotdec::rot_decode_cta<1, true, 8, W * 32>(Pt, 0, ts, tbars, status, pdl_wait != 0, false, ep, &e);
      if (done) {
        // every thread's x~ stores, then the flag (the INT4 CTAs read x~ through
        // the asynchronous proxy after seeing it)
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0 && !rb.skip_flags) st_flag(b.xflags + blockIdx.x, 2ull * e + 1ull);
#ifdef PARO_TIMELINE
        if (threadIdx.x == 0 && b.ctl && blockIdx.x < kTimelineCtas) {
          unsigned long long* o = g_paro_timeline[e & 1][blockIdx.x];
          o[0] = tl_entry; o[1] = rotdec::tl_rot[1]; o[2] = rotdec::tl_rot[2]; o[3] = rotdec::tl_rot[3];
          o[4] = rotdec::tl_now(); o[5] = 1; o[6] = 0; o[7] = 0;
        }
#endif
      }
      finish_cta(b.ctl);
      return;
    }
  }
  __shared__ Meta meta[kMaxBatch];
  if (threadIdx.x < b.count) {
    const StreamProblem& P = b.p[threadIdx.x];
    meta[threadIdx.x] = Meta{P.unit_begin, P.sc, P.z, P.y, P.M, P.d_out, P.G, P.tiles, P.tile_begin};
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&P.qmap)) : "memory");
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&P.xmap)) : "memory");
  }
  __syncthreads();

  // ---- this CTA's and this warp's units --------------------------------------------
  const long long U = b.total_units, C = b.ctas, cta = (long long)blockIdx.x - T;
  // CTA ranges: CTAs 0 .. CA - 1 split units [0, UA) evenly, the others [UA, U)
  const long long CA = b.ctas_a, UA = b.units_a;
  auto cta_start = [&](long long c) -> long long {
    if (b.tile_split) {
      // whole tiles: the first unit of tile c T / C of the launch
      const int tt = (int)part_start(c, C, b.total_tiles);
      int pi = 0;
#pragma unroll 1
      while (pi + 1 < b.count && tt >= meta[pi + 1].tile_begin) ++pi;
      return tt >= b.total_tiles ? U
                                 : meta[pi].unit_begin + (long long)(tt - meta[pi].tile_begin) * meta[pi].G;
    }
    return c <= CA ? part_start(c, CA, UA) : UA + part_start(c - CA, C - CA, U - UA);
  };
  auto cta_of = [&](long long x) -> long long {
    return x < UA ? part_of(x, CA, UA) : CA + part_of(x - UA, C - CA, U - UA);
  };
  const long long c0 = cta_start(cta), c1 = cta_start(cta + 1), nC = c1 - c0;
  const long long w0 = c0 + part_start(warp, W, nC), w1 = c0 + part_start(warp + 1, W, nC);
  const int n = (int)(w1 - w0);
  const uint32_t ring = sbase + (uint32_t)(warp * D * SLOT);
  const uint32_t bar0 = smem_u32(&bars[warp * D]);

  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < D; ++s) mbar_init(bar0 + 8u * s, 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  __syncwarp();

  // ---- prologue: codes of the first D units, the scales of the first, then, once
  // the grid that writes the activations is done, their activations ------------------
  Cur ic = {0, 0, 0};
  if (n > 0) cur_at(meta, b.count, w0, ic);
  Cur cc = ic;  // the unit being computed
  if (lane == 0) {
    Cur c = ic;
#pragma unroll 1
    for (int s = 0; s < D && s < n; ++s) {
      mbar_expect_tx(bar0 + 8u * s, (uint32_t)kUnitBytes);
      tma_load_2d(ring + (uint32_t)(s * SLOT), &b.p[c.pi].qmap, c.grp * 16, c.tile * kStreamRows, bar0 + 8u * s,
                  l2_evict_first());
      cur_next(meta, c);
    }
  }
  uint32_t szc[4] = {0u, 0u, 0u, 0u};  // scale and zero bits of the unit being computed
  if (n > 0) load_sz(meta[cc.pi], cc, g, t, szc);
  // (the flag form orders everything after the transform's flags instead: the
  // transform waited for the previous launch before it published any)
  if (FU >= 0 && pdl_wait) asm volatile("griddepcontrol.wait;\n" ::: "memory");
  // the fused form compares the transforms' flags with the launch tag from the
  // start; the plain form needs it only for its partial tiles and reads it
  // after the units (one round trip less before its first activations)
  if (FU > 0 && b.ctl) ltag = launch_tag(b.ctl);
  PARO_TL_NOW(tl_wait);
  // the activations of the unit in slot s (with the slot's arrival; its codes
  // were requested without one)
  auto issue_x = [&](const Cur& c, int s) {
    const CUtensorMap* xm = &b.p[c.pi].xmap;
    const uint32_t sx = ring + (uint32_t)(s * SLOT + kUnitBytes), bar = bar0 + 8u * s;
    mbar_arrive_expect_tx(bar, (uint32_t)(256 * meta[c.pi].M));
    tma_load_2d(sx, xm, c.grp * 128, 0, bar);
    if constexpr (!ONE) tma_load_2d(sx + XB, xm, c.grp * 128 + 64, 0, bar);
  };
  // fused form (lane 0): linears whose x~ flag was seen, and slots whose
  // activations are still to be requested
  uint32_t xready = 0u, xpend = 0u;
  const unsigned long long xtag = ltag;
  auto x_ready = [&](int pi, bool block) -> bool {
    if (FU == 0 || ((xready >> pi) & 1u)) return true;
    const unsigned long long* f = FU > 0 ? b.xflags + pi : b.xflags + b.p[pi].xf_begin;
    const int nf = FU > 0 ? 1 : b.p[pi].xf_count;
    bool seen = true;
#pragma unroll 1
    for (int q = 0; q < nf && seen; ++q) {
      if (block) {
        seen = wait_flag(f + q, xtag, b.flag_wait);
        if (!seen) report_status(status, kStatusTimeout);
      } else {
        unsigned long long v;
        asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];\n" : "=l"(v) : "l"(f + q) : "memory");
        seen = v == xtag;
      }
    }
    if (!seen) return false;
    // acquire the transform CTA's x~, then order the TMA reads after it
    __threadfence();
    asm volatile("fence.proxy.async.global;\n" ::: "memory");
    xready |= 1u << pi;
    return true;
  };
#pragma unroll 1
  for (int s = 0; s < D && s < n; ++s) {
    if (lane == 0) {
      if (x_ready(ic.pi, false)) issue_x(ic, s);
      else xpend |= 1u << s;
    }
    cur_next(meta, ic);
  }

  // ---- the units ------------------------------------------------------------------
  float acc[4][NT][4], first[4][NT][4];
#pragma unroll
  for (int rt = 0; rt < 4; ++rt)
#pragma unroll
    for (int m = 0; m < NT; ++m)
#pragma unroll
      for (int e = 0; e < 4; ++e) { acc[rt][m][e] = 0.f; first[rt][m][e] = 0.f; }

  int cur_pi = cc.pi, cur_tile = cc.tile;
  bool ok = true;
  int done = 0;  // units consumed
  int slot = 0;
  uint32_t phase = 0;

  constexpr uint32_t kOddScale = F16 ? 0x2C002C00u : 0x3E003E00u;  // 1/16 or 1/8
  constexpr uint32_t kBias = F16 ? 0x64006400u : 0x43004300u;      // 1024 / 128
  constexpr uint32_t kOne = F16 ? 0x3C003C00u : 0x3F803F80u;       // 1
  constexpr uint32_t kOddUp = F16 ? 0x4C004C00u : 0x41004100u;     // 16 / 8
  // rows 0-7 of this operand weigh the activations by their codes' bias (Tb),
  // rows 8-15 by one, undoing the odd columns' pre-division (Sx)
  const uint32_t aTS[4] = {kBias, kOne, kBias, kOddUp};

#pragma unroll 1
  for (int i = 0; i < n; ++i) {
    const Meta& P = meta[cc.pi];
    if (cc.pi != cur_pi || cc.tile != cur_tile) {
      // leaving a tile: write it when it lies wholly in this warp's units, else
      // keep it as this warp's first (split) tile
      const long long Ub = meta[cur_pi].unit_begin + (long long)cur_tile * meta[cur_pi].G;
      if (Ub >= w0) {
        store_tile<NT>(meta[cur_pi], cur_tile, g, t, acc);
      } else {
#pragma unroll
        for (int rt = 0; rt < 4; ++rt)
#pragma unroll
          for (int m = 0; m < NT; ++m)
#pragma unroll
            for (int e = 0; e < 4; ++e) first[rt][m][e] = acc[rt][m][e];
      }
#pragma unroll
      for (int rt = 0; rt < 4; ++rt)
#pragma unroll
        for (int m = 0; m < NT; ++m)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[rt][m][e] = 0.f;
      cur_pi = cc.pi;
      cur_tile = cc.tile;
    }
    // scales and zeros of the next unit, one unit ahead of their use
    Cur nx = cc;
    uint32_t szn[4] = {0u, 0u, 0u, 0u};
    if (i + 1 < n) {
      cur_next(meta, nx);
      load_sz(meta[nx.pi], nx, g, t, szn);
    }
    if constexpr (FU != 0) {
      // the unit's activations were deferred: wait (bounded) for its linear's x~
      int xfail = 0;
      if (lane == 0 && ((xpend >> slot) & 1u)) {
        // on a timeout the slot still gets its arrival, so that its phase
        // completes once the codes have landed, and the warp stops: the
        // status says the result is void and no tile it holds is written
        if (x_ready(cc.pi, true)) {
          issue_x(cc, slot);
        } else {
          mbar_arrive(bar0 + 8u * slot);
          xfail = 1;
        }
        xpend &= ~(1u << slot);
      }
      if (__shfl_sync(0xffffffffu, xfail, 0)) {
        ok = false;
        break;
      }
    }
    if (!mbar_wait(bar0 + 8u * slot, phase)) {
      report_status(status, kStatusTimeout);
      ok = false;
      break;
    }
    ++done;
#ifdef PARO_TIMELINE
    if (i == 0) PARO_TL_NOW(tl_first);
#endif
    const uint32_t sw = ring + (uint32_t)slot * SLOT, sx = sw + kUnitBytes;
    const int mt = P.M;

    // activation fragments: token n*8 + g, columns 32t + 8j .. + 7 of the group,
    // read from the box of columns 64 (t >> 1) .. + 63 (128-byte swizzle)
    uint32_t Bf[NT][4][4];
#pragma unroll
    for (int m = 0; m < NT; ++m) {
      const int tok = m * 8 + g;
      if (tok < mt) {
        const uint32_t row = sx + (uint32_t)((t >> 1) * XB + tok * 128);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t ch = (uint32_t)(4 * (t & 1) + j) ^ (uint32_t)(tok & 7);
          const uint4 u = lds128(row + (ch << 4));
          if constexpr (XPERM) {
            Bf[m][j][0] = u.x;
            Bf[m][j][1] = u.y;
            Bf[m][j][2] = u.z;
            Bf[m][j][3] = u.w;
          } else {
            pair_act(u, Bf[m][j]);
            Bf[m][j][1] = mul2<F16>(Bf[m][j][1], kOddScale);
            Bf[m][j][3] = mul2<F16>(Bf[m][j][3], kOddScale);
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) Bf[m][j][e] = 0u;
      }
    }
    // TS[m] = {Tb(token 2t), Tb(2t + 1), Sx(2t), Sx(2t + 1)} of token tile m
    float TS[NT][4];
#pragma unroll
    for (int m = 0; m < NT; ++m) {
#pragma unroll
      for (int e = 0; e < 4; ++e) TS[m][e] = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        mma16816<F16>(TS[m], aTS, Bf[m][j][0], Bf[m][j][1]);
        mma16816<F16>(TS[m], aTS, Bf[m][j][2], Bf[m][j][3]);
      }
    }
    const int q0 = lane & ~3;
#pragma unroll
    for (int rt = 0; rt < 4; ++rt) {
      // rows rt*16 + g and + 8 of the unit: 64 bytes per row, lane t's 16 bytes
      const uint32_t wa = sw + (uint32_t)((rt * 16 + g) * 64 + t * 16);
      const uint4 wg = lds128(wa), wh = lds128(wa + 512u);
      const float scg = __half2float(__ushort_as_half((unsigned short)__shfl_sync(0xffffffffu, szc[rt], q0)));
      const float sch = __half2float(__ushort_as_half((unsigned short)__shfl_sync(0xffffffffu, szc[rt], q0 | 1)));
      const float zg = __half2float(__ushort_as_half((unsigned short)__shfl_sync(0xffffffffu, szc[rt], q0 | 2)));
      const float zh = __half2float(__ushort_as_half((unsigned short)__shfl_sync(0xffffffffu, szc[rt], q0 | 3)));
      float R[NT][4];
#pragma unroll
      for (int m = 0; m < NT; ++m)
#pragma unroll
        for (int e = 0; e < 4; ++e) R[m][e] = 0.f;
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
        for (int m = 0; m < NT; ++m) {
          mma16816<F16>(R[m], a0, Bf[m][j][0], Bf[m][j][1]);
          mma16816<F16>(R[m], a1, Bf[m][j][2], Bf[m][j][3]);
        }
      }
#pragma unroll
      for (int m = 0; m < NT; ++m) {
        acc[rt][m][0] = fmaf(scg, fmaf(-zg, TS[m][2], R[m][0] - TS[m][0]), acc[rt][m][0]);
        acc[rt][m][1] = fmaf(scg, fmaf(-zg, TS[m][3], R[m][1] - TS[m][1]), acc[rt][m][1]);
        acc[rt][m][2] = fmaf(sch, fmaf(-zh, TS[m][2], R[m][2] - TS[m][0]), acc[rt][m][2]);
        acc[rt][m][3] = fmaf(sch, fmaf(-zh, TS[m][3], R[m][3] - TS[m][1]), acc[rt][m][3]);
      }
    }

    // refill this slot with unit i + D (the generic-proxy reads above are done
    // before the asynchronous copy may overwrite the slot)
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    __syncwarp();
    if (i + D < n) {
      if (lane == 0) {
        const StreamProblem& Q = b.p[ic.pi];
        const uint32_t bar = bar0 + 8u * slot;
        if (x_ready(ic.pi, false)) {
          mbar_arrive_expect_tx(bar, (uint32_t)(kUnitBytes + 256 * meta[ic.pi].M));
          tma_load_2d(sw, &Q.qmap, ic.grp * 16, ic.tile * kStreamRows, bar, l2_evict_first());
          tma_load_2d(sx, &Q.xmap, ic.grp * 128, 0, bar);
          if constexpr (!ONE) tma_load_2d(sx + XB, &Q.xmap, ic.grp * 128 + 64, 0, bar);
        } else {
          // fused form, x~ not written yet: the codes now, the activations (and
          // the slot's arrival) when the unit comes up
          mbar_expect_tx(bar, (uint32_t)kUnitBytes);
          tma_load_2d(sw, &Q.qmap, ic.grp * 16, ic.tile * kStreamRows, bar, l2_evict_first());
          xpend |= 1u << slot;
        }
      }
      cur_next(meta, ic);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) szc[e] = szn[e];
    cc = nx;
    if (++slot == D) {
      slot = 0;
      phase ^= 1u;
    }
  }
  if (!ok) {
    // let the copies still in flight land (each wait bounded) before leaving the
    // ring; slots whose activations were never requested get their arrival first
    if (lane == 0)
      for (int q = 0; q < D; ++q)
        if ((xpend >> q) & 1u) mbar_arrive(bar0 + 8u * q);
    __syncwarp();
    for (int j = done; j < n && j < done + D; ++j) mbar_wait(bar0 + 8u * (j % D), (uint32_t)((j / D) & 1));
  }
  // a warp that gave up voids the CTA's result: none of its remaining tiles is
  // written and no partial is published (a CTA waiting for one gives up too)
  if (__syncthreads_or(!ok)) {
    finish_cta(b.ctl);
    return;
  }
  if (FU == 0 && b.ctl) ltag = launch_tag(b.ctl);
  PARO_TL_NOW(tl_loop);

  // ---- the last tile, and the partial tiles in shared memory -------------------------
  // slot 0: the warp's first tile when it began before the warp's units;
  // slot 1: its last tile when it goes on after them (a tile that does both is slot 0)
  long long fUb = 0, fUe = 0, lUb = 0, lUe = 0;  // unit ranges of the first and last tile
  int f_pi = 0, f_tile = 0, l_pi = 0, l_tile = 0;
  bool f_split = false, l_split = false;
  if (n > 0) {
    Cur f;
    cur_at(meta, b.count, w0, f);
    f_pi = f.pi;
    f_tile = f.tile;
    fUb = meta[f.pi].unit_begin + (long long)f.tile * meta[f.pi].G;
    fUe = fUb + meta[f.pi].G;
    l_pi = cur_pi;
    l_tile = cur_tile;
    lUb = meta[cur_pi].unit_begin + (long long)cur_tile * meta[cur_pi].G;
    lUe = lUb + meta[cur_pi].G;
    f_split = fUb < w0;
    const bool same = (f_pi == l_pi && f_tile == l_tile);
    l_split = !same && lUe > w1;
    if (same) {
      if (fUb < w0 || fUe > w1) {
        f_split = true;
#pragma unroll
        for (int rt = 0; rt < 4; ++rt)
#pragma unroll
          for (int m = 0; m < NT; ++m)
#pragma unroll
            for (int e = 0; e < 4; ++e) first[rt][m][e] = acc[rt][m][e];
      } else {
        store_tile<NT>(meta[l_pi], l_tile, g, t, acc);
      }
    } else if (!l_split) {
      store_tile<NT>(meta[l_pi], l_tile, g, t, acc);
    }
  }
  // the ring is drained: it now holds this warp's partial tiles
#pragma unroll
  for (int rt = 0; rt < 4; ++rt)
#pragma unroll
    for (int m = 0; m < NT; ++m) {
      const uint32_t off = (uint32_t)(((rt * NT + m) * 32 + lane) * 16);
      if (f_split) sts128f(ring + off, make_float4(first[rt][m][0], first[rt][m][1], first[rt][m][2], first[rt][m][3]));
      if (l_split)
        sts128f(ring + (uint32_t)(PF * 4) + off, make_float4(acc[rt][m][0], acc[rt][m][1], acc[rt][m][2], acc[rt][m][3]));
    }
  __syncthreads();
  // every thread of this CTA has read the launch epoch (before the barrier
  // above), so the CTA counts itself as finished now, for the last CTA of the
  // launch to advance the epoch; the count's round trip overlaps the combine
  // (nothing in this launch reads the epoch again, and the next launch reads
  // it only once this one has completed)
  unsigned checkin = 0u;
  if (threadIdx.x == 0 && b.ctl) checkin = atomicInc(reinterpret_cast<unsigned*>(b.ctl + 1), gridDim.x - 1);

  // ---- combine: the warp holding a split tile's first unit in this CTA sums the
  // warps' partials in warp order.  A tile that crosses the CTA's bounds then
  // goes through the workspace: every CTA but the tile's last publishes its
  // partial and a flag (this launch's tag) and moves on; the tile's last
  // CTA waits for the flags of the earlier CTAs, which started no later than
  // it did, and sums the partials in CTA order.  Publishing comes first (the
  // warp's last tile), so no warp waits while holding back a partial. ------------
  const uint32_t tag32 = (uint32_t)ltag;  // the tag's low half, carried by every partial value
#pragma unroll 1
  for (int pass = 0; pass < 2; ++pass) {
    const int which = 1 - pass;
    const bool split = which == 0 ? f_split : l_split;
    if (!split) continue;
    const int pi = which == 0 ? f_pi : l_pi, tile = which == 0 ? f_tile : l_tile;
    const long long Ub = which == 0 ? fUb : lUb, Ue = which == 0 ? fUe : lUe;
    const long long lo = Ub > c0 ? Ub : c0, hi = Ue < c1 ? Ue : c1;  // the tile's units in this CTA
    if (c0 + part_of(lo - c0, W, nC) != c0 + warp) continue;     // not the owner
    const int wlast = (int)part_of(hi - 1 - c0, W, nC);
    float sum[4][NT][4];
#pragma unroll
    for (int rt = 0; rt < 4; ++rt)
#pragma unroll
      for (int m = 0; m < NT; ++m)
#pragma unroll
        for (int e = 0; e < 4; ++e) sum[rt][m][e] = 0.f;
#pragma unroll 1
    for (int w = warp; w <= wlast; ++w) {
      const long long ws0 = c0 + part_start(w, W, nC), ws1 = c0 + part_start(w + 1, W, nC);
      if (ws1 <= ws0) continue;                  // a warp without units
      const int e = (Ub <= ws0) ? 0 : 1;         // the tile is that warp's first or its last
      const uint32_t src = sbase + (uint32_t)(w * D * SLOT) + (uint32_t)(e * PF * 4);
#pragma unroll
      for (int rt = 0; rt < 4; ++rt)
#pragma unroll
        for (int m = 0; m < NT; ++m) {
          const float4 v = lds128f(src + (uint32_t)(((rt * NT + m) * 32 + lane) * 16));
          sum[rt][m][0] += v.x; sum[rt][m][1] += v.y; sum[rt][m][2] += v.z; sum[rt][m][3] += v.w;
        }
    }
    const Meta& P = meta[pi];
    if (Ub >= c0 && Ue <= c1) {
      store_tile<NT>(P, tile, g, t, sum);
      continue;
    }
    if (Ue > c1) {
      // the tile goes on in a later CTA: publish this CTA's partial, every
      // value tagged
      const int eC = (Ub <= c0) ? 0 : 1;
      unsigned long long* mine = b.partials + ((size_t)cta * 2 + eC) * PF;
#pragma unroll
      for (int rt = 0; rt < 4; ++rt)
#pragma unroll
        for (int m = 0; m < NT; ++m) {
          unsigned long long* q = mine + (size_t)(((rt * NT + m) * 32 + lane) * 4);
          st_tagged(q, sum[rt][m][0], sum[rt][m][1], tag32);
          st_tagged(q + 2, sum[rt][m][2], sum[rt][m][3], tag32);
        }
      continue;
    }
    // the tile began in an earlier CTA and ends here: add the earlier partials
    // in CTA order, then this CTA's
    float tot[4][NT][4];
#pragma unroll
    for (int rt = 0; rt < 4; ++rt)
#pragma unroll
      for (int m = 0; m < NT; ++m)
#pragma unroll
        for (int e = 0; e < 4; ++e) tot[rt][m][e] = 0.f;
    const long long ca = cta_of(Ub);
    bool got = true;  // every earlier CTA's partial arrived
#pragma unroll 1
    for (long long cx = ca; cx < cta; ++cx) {
      const long long s0 = cta_start(cx);
      if (cta_start(cx + 1) <= s0) continue;  // a CTA without units
      const int e = (Ub <= s0) ? 0 : 1;
      if (!add_tagged<NT>(b.partials + ((size_t)cx * 2 + e) * PF, lane, tag32, b.flag_wait, tot)) {
        if (lane == 0) report_status(status, kStatusTimeout);
        got = false;
        break;
      }
    }
    if (!got) continue;  // the tile stays unwritten: the status says the result is void
#pragma unroll
    for (int rt = 0; rt < 4; ++rt)
#pragma unroll
      for (int m = 0; m < NT; ++m)
#pragma unroll
        for (int e = 0; e < 4; ++e) tot[rt][m][e] += sum[rt][m][e];
    store_tile<NT>(P, tile, g, t, tot);
  }
  if (threadIdx.x == 0 && b.ctl && checkin == gridDim.x - 1) atomicAdd(b.ctl, 1ull);
#ifdef PARO_TIMELINE
  if (FU > 0 && b.ctl && blockIdx.x < kTimelineCtas) {
    unsigned long long* o = g_paro_timeline[(ltag >> 1) & 1][blockIdx.x];
    if (threadIdx.x == 0) {
      o[0] = tl_entry; o[1] = tl_wait; o[2] = tl_first; o[3] = tl_loop; o[5] = 2;
      o[6] = (unsigned long long)n; o[7] = (unsigned long long)cur_pi;
    }
    if (lane == 0) atomicMax(o + 4, rotdec::tl_now());
  }
#endif
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

size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }

}  // namespace

int device_sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cache[dev] = v;
  }
  return cache[dev];
}

bool stream_supported(int M, int d_in, int d_out, const void* x, const void* qweight) {
  return M >= 1 && M <= kStreamMaxM && d_in % kGroup == 0 && d_out >= kStreamRows && d_out % 16 == 0 &&
         (reinterpret_cast<uintptr_t>(x) & 15) == 0 && (reinterpret_cast<uintptr_t>(qweight) & 15) == 0;
}

// most INT4 CTAs a launch of that token-tile count has (a flag pair and two
// partial tiles each in the workspace)
static int max_ctas(int NT) { return device_sm_count() * (NT == 1 ? Geo<1>::CPS : Geo<2>::CPS); }

// two partial tiles per CTA (a 64-bit tagged word per value), the transforms'
// flags, the launch epoch and the finished-CTA count
size_t stream_workspace_bytes(int max_m) {
  const int NT = max_m <= 8 ? 1 : 2;
  const size_t C = (size_t)max_ctas(NT);
  return round256(C * 2 * (4 * NT * 32 * 4) * 8) + round256((size_t)kXFlagWords * 8) + 256;
}

cudaError_t plan_stream_batch(const uint16_t* const* x, const uint32_t* const* qw, const __half* const* sc,
                              const __half* const* z, __nv_bfloat16* const* y, const int* M, const int* d_in,
                              const int* d_out, int count, bool x_f16, void* ws, StreamBatch* out, int* nt_out,
                              int reserved_ctas) {
  if (count < 1 || count > kMaxBatch) return cudaErrorInvalidValue;
  EncodeTiled enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  *out = StreamBatch{};
  int maxM = 0, tiles = 0;
  long long units = 0;
  bool all_one = PARO_STREAM_ONE != 0;
  for (int i = 0; i < count; ++i) all_one = all_one && M[i] == 1;
  for (int i = 0; i < count; ++i) {
    if (!stream_supported(M[i], d_in[i], d_out[i], x[i], qw[i])) return cudaErrorInvalidValue;
    maxM = M[i] > maxM ? M[i] : maxM;
    StreamProblem& p = out->p[i];
    p.sc = reinterpret_cast<const unsigned short*>(sc[i]);
    p.z = reinterpret_cast<const unsigned short*>(z[i]);
    p.y = y[i];
    p.M = M[i];
    p.d_in = d_in[i];
    p.d_out = d_out[i];
    p.G = d_in[i] / kGroup;
    p.tiles = (d_out[i] + kStreamRows - 1) / kStreamRows;
    p.unit_begin = units;
    p.tile_begin = tiles;
    units += (long long)p.tiles * p.G;
    tiles += p.tiles;
    const cuuint32_t unit_strides[2] = {1, 1};
    {  // codes: uint32 [d_out][d_in / 8], one box = 16 words x 64 rows
      const cuuint64_t dims[2] = {(cuuint64_t)(d_in[i] / 8), (cuuint64_t)d_out[i]};
      const cuuint64_t strides[1] = {(cuuint64_t)d_in[i] / 2};
      const cuuint32_t box[2] = {16, (cuuint32_t)kStreamRows};
      if (enc(&p.qmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(qw[i]), dims, strides, box,
              unit_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
    {  // activations [M][d_in]: one box = 64 columns x all M tokens, 128-byte swizzle;
       // with one token in every linear, one unswizzled box of 128 columns
      const bool one = all_one;
      const cuuint64_t dims[2] = {(cuuint64_t)d_in[i], (cuuint64_t)M[i]};
      const cuuint64_t strides[1] = {(cuuint64_t)d_in[i] * 2};
      const cuuint32_t box[2] = {one ? 128u : 64u, (cuuint32_t)M[i]};
      if (enc(&p.xmap, x_f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
              const_cast<uint16_t*>(x[i]), dims, strides, box, unit_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
              one ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
  }
  // the kernel's unit arithmetic is 32-bit: units times CTAs stays below 2^32
  if (units >= (1LL << 23)) return cudaErrorInvalidValue;
  out->count = count;
  out->one = all_one ? 1 : 0;
  out->total_units = units;
  out->total_tiles = tiles;
  const int W = maxM <= 8 ? Geo<1>::W : Geo<2>::W;
  const long long want = (units + W - 1) / W;
  const int sms = device_sm_count();
  const int avail = sms * (maxM <= 8 ? Geo<1>::CPS : Geo<2>::CPS) - reserved_ctas;
  if (avail < 1) return cudaErrorInvalidValue;
  out->ctas = (int)(want < avail ? want : avail);
  out->ctas_a = out->ctas;
  out->units_a = units;
  out->flag_wait = hook_flag_wait();
  *nt_out = maxM <= 8 ? 1 : 2;
  if (!ws) {
    // no workspace: whole tiles per CTA, so no partial sum crosses a CTA
    if (reserved_ctas) return cudaErrorInvalidValue;
    out->tile_split = 1;
    if (out->ctas > tiles) out->ctas = tiles;
    out->ctas_a = out->ctas;
    return cudaSuccess;
  }
  const size_t C = (size_t)max_ctas(maxM <= 8 ? 1 : 2);
  out->partials = static_cast<unsigned long long*>(ws);
  out->xflags = reinterpret_cast<unsigned long long*>(static_cast<char*>(ws) +
                                                      round256(C * 2 * (4 * (maxM <= 8 ? 1 : 2) * 32 * 4) * 8));
  out->ctl = out->xflags + round256((size_t)kXFlagWords * 8) / 8;
  return cudaSuccess;
}

cudaError_t launch_stream_batch(const StreamBatch& b, int NT, bool x_f16, int* status, cudaStream_t stream,
                                bool pdl_wait) {
  const bool one = b.one != 0;
  const size_t smem = NT == 1 ? (one ? Geo<1, true>::SMEM : Geo<1>::SMEM) : Geo<2>::SMEM;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(b.ctas);
  cfg.blockDim = dim3((NT == 1 ? Geo<1>::W : Geo<2>::W) * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_wait ? 1 : 0;
  const int wait = pdl_wait ? 1 : 0;
  cudaError_t e;
  const RotBatch none{};
#define PARO_STREAM_LAUNCH(f16, nt, one)                                                                  \
  {                                                                                                       \
    auto k = w4_stream_kernel<f16, nt, 0, false, one>;                                                    \
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);                  \
    if (e != cudaSuccess) return e;                                                                       \
    return cudaLaunchKernelEx(&cfg, k, b, none, status, wait);                                            \
  }
  if (x_f16) {
    if (NT == 1) {
      if (one) PARO_STREAM_LAUNCH(true, 1, true) else PARO_STREAM_LAUNCH(true, 1, false)
    } else PARO_STREAM_LAUNCH(true, 2, false)
  } else {
    if (NT == 1) {
      if (one) PARO_STREAM_LAUNCH(false, 1, true) else PARO_STREAM_LAUNCH(false, 1, false)
    } else PARO_STREAM_LAUNCH(false, 2, false)
  }
#undef PARO_STREAM_LAUNCH
}

cudaError_t launch_stream_flagged(const StreamBatch& b, int NT, int* status, cudaStream_t stream) {
  const bool one = b.one != 0 && NT == 1;
  const size_t smem = NT == 1 ? (one ? Geo<1, true>::SMEM : Geo<1>::SMEM) : Geo<2>::SMEM;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(b.ctas);
  cfg.blockDim = dim3((NT == 1 ? Geo<1>::W : Geo<2>::W) * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const RotBatch none{};
  cudaError_t e;
  if (NT == 1 && one) {
    e = cudaFuncSetAttribute(w4_stream_kernel<true, 1, -1, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, w4_stream_kernel<true, 1, -1, true, true>, b, none, status, 1);
  }
  if (NT == 1) {
    e = cudaFuncSetAttribute(w4_stream_kernel<true, 1, -1, true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, w4_stream_kernel<true, 1, -1, true, false>, b, none, status, 1);
  }
  e = cudaFuncSetAttribute(w4_stream_kernel<true, 2, -1, true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, w4_stream_kernel<true, 2, -1, true, false>, b, none, status, 1);
}

// ---- fused form -----------------------------------------------------------------------
namespace {
// dynamic shared memory of the fused kernel: the INT4 CTAs' rings, or a
// transform CTA's row and stage slots after the 1024-byte alignment, whichever
// is larger, within 227 KB less the kernel's static shared memory
constexpr size_t kFusedSmemBudget = 227 * 1024 - 2048;
size_t fused_rot_smem(int d, int ring, bool region = false) {
  return 1024 + (size_t)d * 4 + (size_t)ring * 6 * d + (region ? (size_t)d * 4 : 0);
}
}  // namespace

void set_fused_split(StreamBatch& b, double late) {
  b.ctas_a = b.ctas;
  b.units_a = b.total_units;
  if (b.count < 2 || b.ctas < 4) return;
  int other = 0;
  for (int i = 0; i + 1 < b.count; ++i) other = b.p[i].d_in > other ? b.p[i].d_in : other;
  const int wide = b.p[b.count - 1].d_in;
  if (2 * wide < 3 * other) return;
  // units a CTA of the last linear gets, relative to the others: the later its
  // x~ comes (the wider it is than the rest), the fewer (fitted to the arrival
  // times of the transforms on B200 for Qwen2.5-1.5B and Llama-3-8B layers)
  double rho = 1.0 - late * (double)(wide - other) / wide;
  rho = rho < 0.25 ? 0.25 : rho;  // (a share near zero would leave those CTAs nearly idle)
  const long long UA = b.p[b.count - 1].unit_begin, UB = b.total_units - UA;
  long long CA = (long long)((double)b.ctas / (1.0 + (double)UB / (rho * (double)UA)) + 0.5);
  CA = CA < 1 ? 1 : (CA > b.ctas - 1 ? b.ctas - 1 : CA);
  b.ctas_a = (int)CA;
  b.units_a = UA;
}

bool fused_supported(const RotProblem* probs, int count) {
  if (count < 1 || count > kMaxBatch) return false;
  for (int i = 0; i < count; ++i) {
    const RotProblem& p = probs[i];
    if (p.M != 1 || p.d % 8 != 0 || p.K < 0 || p.K > 16 || fused_rot_smem(p.d, 1) > kFusedSmemBudget) return false;
    if (p.K > 0 && ((reinterpret_cast<uintptr_t>(p.pairs) | reinterpret_cast<uintptr_t>(p.cos_t) |
                     reinterpret_cast<uintptr_t>(p.sin_t)) & 15) != 0)
      return false;
  }
  return true;
}

cudaError_t plan_fused_rot(const RotProblem* probs, int count, RotBatch* out) {
  if (!fused_supported(probs, count)) return cudaErrorInvalidValue;
  *out = RotBatch{};
  for (int i = 0; i < count; ++i) {
    RotProblem p = probs[i];
    // as many stages of tables as fit beside a region for 1/scale, as long as
    // that leaves at least two slots (a stage's table then lands while the
    // previous stage is rotated); else as many as fit without it, the scale
    // then going into the slot that the last refill leaves free
    const int want = p.K < 1 ? 1 : (p.K > rotdec::kRotMaxRing ? rotdec::kRotMaxRing : p.K);
    int ring = want;
    while (ring > 1 && fused_rot_smem(p.d, ring, true) > kFusedSmemBudget) --ring;
    const bool region = fused_rot_smem(p.d, ring, true) <= kFusedSmemBudget && ring >= (want < 2 ? want : 2);
    if (!region) {
      ring = want;
      while (ring > 1 && fused_rot_smem(p.d, ring) > kFusedSmemBudget) --ring;
    }
    p.sscale = scale_mode(p, ring, region);
    p.rows = 1;
    p.ring = ring;
    p.cta_begin = i;
    p.perm = 1;  // the INT4 CTAs read x~ in their operand order
    out->p[i] = p;
  }
  out->count = count;
  out->total_ctas = count;
  return cudaSuccess;
}

cudaError_t launch_fused_batch(const StreamBatch& b, const RotBatch& rb, int* status, cudaStream_t stream,
                               bool pdl_wait) {
  static_assert(sizeof(StreamBatch) + sizeof(RotBatch) + 16 <= 4096, "kernel parameters");

  size_t smem = b.one ? Geo<1, true>::SMEM : Geo<1>::SMEM;
  for (int i = 0; i < rb.count; ++i) {
    const size_t s = fused_rot_smem(rb.p[i].d, rb.p[i].ring, rb.p[i].sscale == 1);
    smem = s > smem ? s : smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rb.count + b.ctas);
  cfg.blockDim = dim3(Geo<1>::W * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_wait ? 1 : 0;
  const int wait = pdl_wait ? 1 : 0;
  auto k = b.one ? w4_stream_kernel<true, 1, 1, true, true> : w4_stream_kernel<true, 1, 1, true, false>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, k, b, rb, status, wait);
}

}  // namespace paro
