// One CTA of the few-token activation transform x~ = diag(1/s) R_K ... R_1 x
// (page "ParoQuant: pairwise rotations that survive deployment", section "A
// rotation small enough to execute": disjoint channel pairs per stage, each
// rotated by x_i' = c x_i + s x_j, x_j' = -s x_i + c x_j; channel scale last),
// shared by the transform kernel (rotate_decode.cu) and the decode INT4 linear
// that runs the transform in its own first CTAs (w4_stream.cu).
//
// The CTA stages its R rows as fp32 planes (channel c in bank c % 32 for every
// row).  Its last warp streams the stage tables (pairs, cos, sin: 12 bytes a
// pair) by bulk copies through a ring of mbarrier slots, L2-prefetches the
// stages beyond the ring, and waits for each stage's table before the CTA
// barrier that starts the stage, so the barrier also tells the other warps that
// the table has landed; they rotate the pairs, U per thread and round, loads
// before stores.  The same thread brings the channel scale into shared memory
// with one more bulk copy (into a region of its own, or into the slot the last
// table refill leaves free), so the final pass, which divides by it, reads no
// global memory.  Waits are bounded: a stage or scale that never lands is
// reported as PARO_ERR_TIMEOUT and the CTA returns false without writing.
#pragma once

#include "paro_internal.cuh"
#include "rotate_decode.cuh"

namespace paro {
namespace rotdec {

#ifdef PARO_TIMELINE
// Instrumented build only (rotation_int4_weight_b200/_build.py --timeline): the
// global timer in ns, and the moments this CTA's transform passed its phases
// (1 wait for the previous kernel done, 2 rows staged, 3 stages done), kept by
// thread 0 for the caller to publish.
__device__ __forceinline__ unsigned long long tl_now() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
  return t;
}
__shared__ unsigned long long tl_rot[4];
#define PARO_TL_ROT(k) \
  if (threadIdx.x == 0) tl_rot[k] = tl_now()
#else
#define PARO_TL_ROT(k)
#endif

constexpr int kRotMaxRing = 8;
constexpr int kRotBars = kRotMaxRing + 1;  // one mbarrier per ring slot, one for the channel scale

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
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
// non-blocking test of the same phase (cheaper than try_wait when the phase has
// long completed, the usual case for the stages after the first)
__device__ __forceinline__ bool mbar_done(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}
// Waits for phase `parity` of an mbarrier; gives up after about a second of
// SM clock (then returns false and the caller reports PARO_ERR_TIMEOUT).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_done(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_test(bar, parity))
    if (clock64() - t0 > (1LL << 31)) return false;
  return true;
}
// plain shared-memory accesses at 32-bit shared-window addresses (volatile:
// they keep their order with each other; the stage barrier orders them with
// everything else)
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];\n" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ float lds_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];\n" : "=f"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts_f32(uint32_t a, float v) {
  asm volatile("st.shared.f32 [%0], %1;\n" ::"r"(a), "f"(v) : "memory");
}
// An L2 policy that keeps the lines it fetches past lines of normal and
// evict-first priority: the stage tables and scales are layer constants, read
// once per call like the weights but a fraction of their size, so they stay in
// L2 from one token to the next while the weights (fetched evict-first by the
// INT4 kernels) stream through
__device__ __forceinline__ uint64_t l2_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;\n" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, size_t bytes, uint64_t pol) {
  asm volatile("cp.async.bulk.prefetch.L2.global.L2::cache_hint [%0], %1, %2;\n"
               ::"l"(src), "r"((uint32_t)bytes), "l"(pol) : "memory");
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar, uint64_t pol) {
  asm volatile("cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;\n"
               ::"r"(dst), "l"(src), "r"(bytes), "r"(bar), "l"(pol) : "memory");
}


// Transforms rows row0 .. row0 + RP - 1 of problem P with NTHR threads, RP =
// P.rows (at most R; 0 means R); smem holds d RP 4 + ring 6 d (+ 4 d with
// P.sscale == 1) bytes (16-byte aligned), bars kRotBars mbarriers.
// Returns true when the rows were written (uniform over the CTA).
// trigger_after_wait: let the grid's dependents launch right after the wait
// for the previous kernel (rather than earlier).
// epoch, epoch_out: when given, thread 0 reads the launch epoch *epoch right
// after that wait into *epoch_out, for the caller's flag.
template <int R, bool F16OUT, int U, int NTHR>
__device__ __forceinline__ bool rot_decode_cta(const RotProblem& P, int row0, unsigned char* smem, uint64_t* bars,
                                               int* status, bool pdl_wait, bool trigger_after_wait = false,
                                               const unsigned long long* epoch = nullptr,
                                               unsigned long long* epoch_out = nullptr) {
  constexpr int kProd = NTHR - 32;  // the table-fetching thread (lane 0 of the last warp)
  constexpr int kComp = NTHR - 32;  // rotating threads
  const int d = P.d, K = P.K, half = d >> 1, ring = P.ring;
  const int RP = P.rows > 0 && P.rows < R ? P.rows : R;  // row planes (uniform)
  const int nrows = min(RP, P.M - row0);
  const int tid = threadIdx.x;

  // shared memory: xs [RP][d] fp32 (one plane per row: channel c in bank c % 32) |
  // ring [ring][6d] of stage tables
  float* xs = reinterpret_cast<float*>(smem);
  unsigned char* tab = reinterpret_cast<unsigned char*>(xs + (size_t)d * RP);
  const size_t stage_bytes = (size_t)6 * d;  // pairs | cos | sin
  const uint32_t s_tab = static_cast<uint32_t>(__cvta_generic_to_shared(tab));
  const uint32_t s_bar = static_cast<uint32_t>(__cvta_generic_to_shared(bars));
  const uint64_t pol = tid == kProd ? l2_evict_last() : 0;  // (used by the producer only)

  // one thread requests whole stages with bulk copies (three per stage); the
  // stage's mbarrier completes when all 6d bytes have landed
  auto issue_stage = [&](int k) {
    if (k < K) {
      const int slot = k % ring;
      const uint32_t base = s_tab + (uint32_t)(slot * stage_bytes), bar = s_bar + 8u * slot;
      mbar_expect_tx(bar, (uint32_t)stage_bytes);
      bulk_g2s(base, P.pairs + (size_t)k * half, 2u * d, bar, pol);
      bulk_g2s(base + 2u * d, P.cos_t + (size_t)k * half, 2u * d, bar, pol);
      bulk_g2s(base + 4u * d, P.sin_t + (size_t)k * half, 2u * d, bar, pol);
    }
  };
  // the channel scale in shared memory (fp32, read by the final pass):
  // sscale 1, a region after the ring, requested with the first stages and
  // turned into 1/s in place before the wait for the previous kernel; sscale 2,
  // s in the ring slot that the last refill leaves free, requested once that
  // slot is free (while the last stages run).  It lands on bars[kRotMaxRing].
  const uint32_t s_sbar = s_bar + 8u * kRotMaxRing;
  const int ks = K - ring + 1 > 1 ? K - ring + 1 : 1;  // sscale 2: the stage that requests it
  const float* ssm = nullptr;
  if (P.sscale == 1) ssm = reinterpret_cast<const float*>(tab + (size_t)ring * stage_bytes);
  else if (P.sscale == 2) ssm = reinterpret_cast<const float*>(tab + (size_t)((ks - 1) % ring) * stage_bytes);
  auto issue_scale = [&]() {
    mbar_expect_tx(s_sbar, 4u * (uint32_t)d);
    bulk_g2s(static_cast<uint32_t>(__cvta_generic_to_shared(ssm)), P.scale, 4u * (uint32_t)d, s_sbar, pol);
  };
  if (tid == kProd) {
    for (int k = 0; k < kRotBars; ++k) mbar_init(s_bar + 8u * k, 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    for (int k = 0; k < ring; ++k) issue_stage(k);
    if (P.sscale == 1) issue_scale();
    // then the stages beyond the ring go to L2, so that their copies into the
    // ring later wait for L2 rather than HBM
    if (K > ring) {
      const size_t off = (size_t)ring * half, bytes = (size_t)(K - ring) * 2 * d;
      bulk_prefetch_l2(P.pairs + off, bytes, pol);
      bulk_prefetch_l2(P.cos_t + off, bytes, pol);
      bulk_prefetch_l2(P.sin_t + off, bytes, pol);
    }
    if (P.sscale != 1 && P.scale && (reinterpret_cast<uintptr_t>(P.scale) & 15) == 0)
      bulk_prefetch_l2(P.scale, (size_t)4 * d, pol);
  }
  if (P.sscale == 1) __syncthreads();  // the mbarriers are initialised before anyone waits
  // sscale 1: 1/s in place, each thread its channels, once the copy has landed
  // (the scale is a layer constant, so this may overlap the previous kernel;
  // the barrier after the rows are staged orders it before the final pass)
  bool ok = true;
  if (P.sscale == 1) {
    ok = mbar_wait_bounded(s_sbar, 0u);
    float* r = const_cast<float*>(ssm);
    if (ok)
      for (int c = tid; c < d; c += NTHR) r[c] = 1.0f / r[c];
  }
  // launched as a programmatic dependent: the tables above may be fetched while
  // the previous kernel finishes; the rows (which it may have written) and the
  // output (which it may still read) wait for it to complete
  if (pdl_wait) asm volatile("griddepcontrol.wait;\n" ::: "memory");
  if (trigger_after_wait) asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  // the epoch is final once the previous kernel has completed, so it is read
  // now and used only when the flag is written, its latency hidden by the work
  // between (relaxed: the wait made that kernel's writes visible, and an
  // acquire would hold back this thread's row loads until it returned)
  if (epoch && tid == 0)
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];\n" : "=l"(*epoch_out) : "l"(epoch) : "memory");
  PARO_TL_ROT(1);
  // rows -> xs as fp32: each thread two adjacent channels of every row, the
  // loads of LB channel pairs issued before their stores so that their
  // latencies overlap
  constexpr int LB = R == 4 ? 2 : (R == 2 ? 4 : 8);
#pragma unroll 1
  for (int cp0 = tid; cp0 < half; cp0 += LB * NTHR) {
    __nv_bfloat162 v[LB][R];
#pragma unroll
    for (int q = 0; q < LB; ++q)
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int cp = cp0 + q * NTHR;
        v[q][r] = __floats2bfloat162_rn(0.f, 0.f);
        if (cp < half && r < nrows)
          v[q][r] = *reinterpret_cast<const __nv_bfloat162*>(P.x + (size_t)(row0 + r) * d + 2 * cp);
      }
#pragma unroll
    for (int q = 0; q < LB; ++q) {
      const int cp = cp0 + q * NTHR;
      if (cp < half) {
#pragma unroll
        for (int r = 0; r < R; ++r)
          if (r < RP) *reinterpret_cast<float2*>(xs + (size_t)r * d + 2 * cp) = __bfloat1622float2(v[q][r]);
      }
    }
  }
  // The producer waits for each stage's table before the CTA barrier that
  // starts the stage, so that the barrier also tells the other threads that
  // the table has landed; it refills a slot as soon as the barrier after its
  // stage has passed.  With one slot the next stage can only be requested once
  // the current one is done, which costs a second barrier per stage.
  if (tid == kProd && K > 0 && ok) ok = mbar_wait_bounded(s_bar, 0u);
  int failed = __syncthreads_or(!ok);  // also: rows staged
  PARO_TL_ROT(2);
  int issued = ring < K ? ring : K;    // stages requested so far (producer)
  bool scale_issued = P.sscale == 1;   // (producer)

  // K stages.  The pairs of a stage are disjoint, so the loads of a batch of
  // pairs may all be issued before any of its stores.  Addresses are 32-bit
  // shared-window offsets worked out once; a channel index outside 0..d-1 is
  // clamped into range (so every access stays inside the rows) and reported
  // once (PARO_ERR_INVALID_ARG) after the stages, the result then being void.
  const uint32_t s_xs = static_cast<uint32_t>(__cvta_generic_to_shared(xs));
  const uint32_t ud = (uint32_t)d, plane = 4u * ud;
  uint32_t slot_off = 0;  // this stage's ring slot, bytes from s_tab
  bool bad = false;
#pragma unroll 1
  for (int k = 0; k < K && !failed; ++k) {
    if (tid < kComp) {
      const uint32_t st = s_tab + slot_off;
      for (int t0 = tid; t0 < half; t0 += U * kComp) {
        uint32_t ai[U], aj[U];
        float c[U], sn[U], a[U][R], b[U][R];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int t = t0 + u * kComp;
          if (t < half) {
            const uint32_t off = st + 4u * (uint32_t)t;
            const uint32_t pr = lds_u32(off);
            c[u] = lds_f32(off + 2u * ud);
            sn[u] = lds_f32(off + 4u * ud);
            uint32_t i = pr & 0xFFFFu, j = pr >> 16;
            bad |= (i >= ud) | (j >= ud);
            i = min(i, ud - 1u);
            j = min(j, ud - 1u);
            ai[u] = s_xs + 4u * i;
            aj[u] = s_xs + 4u * j;
          }
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
          if (t0 + u * kComp < half) {
#pragma unroll
            for (int r = 0; r < R; ++r)
              if (r < RP) {
                a[u][r] = lds_f32(ai[u] + r * plane);
                b[u][r] = lds_f32(aj[u] + r * plane);
              }
          }
#pragma unroll
        for (int u = 0; u < U; ++u)
          if (t0 + u * kComp < half) {
#pragma unroll
            for (int r = 0; r < R; ++r)
              if (r < RP) {
                sts_f32(ai[u] + r * plane, fmaf(c[u], a[u][r], sn[u] * b[u][r]));
                sts_f32(aj[u] + r * plane, fmaf(-sn[u], a[u][r], c[u] * b[u][r]));
              }
          }
      }
    } else if (tid == kProd) {
      if (ring > 1) {
        // stage k - 1's slot is free since the barrier that started this stage:
        // it takes the next table, or, once none is left, the scale (sscale 2)
        if (k >= 1 && k - 1 + ring < K) {
          issue_stage(k - 1 + ring);
          ++issued;
        } else if (P.sscale == 2 && k == ks) {
          issue_scale();
          scale_issued = true;
        }
        if (k + 1 < K) ok = mbar_wait_bounded(s_bar + 8u * ((k + 1) % ring), (uint32_t)(((k + 1) / ring) & 1));
      }
      // the scale (sscale 2) before the barrier that ends the last stage
      if (k == K - 1 && P.sscale == 2 && ok) ok = mbar_wait_bounded(s_sbar, 0u);
    }
    failed = __syncthreads_or(!ok);
    slot_off += (uint32_t)stage_bytes;
    if (slot_off == (uint32_t)(ring * stage_bytes)) slot_off = 0;
    if (ring == 1 && k + 1 < K && !failed) {
      if (tid == kProd) {
        issue_stage(k + 1);
        ++issued;
        ok = mbar_wait_bounded(s_bar, (uint32_t)((k + 1) & 1));
      }
      failed = __syncthreads_or(!ok);
    }
  }
  PARO_TL_ROT(3);
  if (bad) report_status(status, kStatusBadIndex);
  if (failed) {
    // a stage never arrived: report, let the latest copy of every slot land
    // (each wait bounded again), then leave
    if (tid == kProd) {
      report_status(status, kStatusTimeout);
      for (int q = issued > ring ? issued - ring : 0; q < issued; ++q)
        mbar_wait_bounded(s_bar + 8u * (q % ring), (uint32_t)((q / ring) & 1));
      if (scale_issued) mbar_wait_bounded(s_sbar, 0u);
    }
    __syncthreads();
    return false;
  }

  // channel scale and store: the scales of LB channel pairs are loaded (from
  // L2, where the prologue put them) before any of them is used.  An fp16
  // value that rounds to infinity is reported once (PARO_ERR_RANGE).
  bool ovf = false;
  if constexpr (F16OUT) {
    if (P.perm) {
      // operand order of the stream-K INT4 kernel: one 16-byte store per
      // 8-column block, (x0, x4, x1/16, x5/16, x2, x6, x3/16, x7/16), the odd
      // columns divided by 16 to match its codes' exponent bias
#pragma unroll 1
      for (int b0 = tid; b0 < (d >> 3); b0 += NTHR) {
        float f[8];
        if (ssm) {
          const float4 r0 = *reinterpret_cast<const float4*>(ssm + 8 * b0);
          const float4 r1 = *reinterpret_cast<const float4*>(ssm + 8 * b0 + 4);
          f[0] = r0.x; f[1] = r0.y; f[2] = r0.z; f[3] = r0.w;
          f[4] = r1.x; f[5] = r1.y; f[6] = r1.z; f[7] = r1.w;
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = P.scale ? __ldg(P.scale + 8 * b0 + e) : 1.0f;
        }
        if (P.sscale != 1) {
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = 1.0f / f[e];
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
          if (r < nrows) {
            const float4 lo = *reinterpret_cast<const float4*>(xs + (size_t)r * d + 8 * b0);
            const float4 hi = *reinterpret_cast<const float4*>(xs + (size_t)r * d + 8 * b0 + 4);
            const __half2 h0 = __floats2half2_rn(lo.x * f[0], hi.x * f[4]);
            const __half2 h1 = __floats2half2_rn(lo.y * f[1] * 0.0625f, hi.y * f[5] * 0.0625f);
            const __half2 h2 = __floats2half2_rn(lo.z * f[2], hi.z * f[6]);
            const __half2 h3 = __floats2half2_rn(lo.w * f[3] * 0.0625f, hi.w * f[7] * 0.0625f);
            uint4 u;
            u.x = *reinterpret_cast<const uint32_t*>(&h0);
            u.y = *reinterpret_cast<const uint32_t*>(&h1);
            u.z = *reinterpret_cast<const uint32_t*>(&h2);
            u.w = *reinterpret_cast<const uint32_t*>(&h3);
            ovf |= half2_inf(u.x) | half2_inf(u.y) | half2_inf(u.z) | half2_inf(u.w);
            *reinterpret_cast<uint4*>(static_cast<__half*>(P.out) + (size_t)(row0 + r) * d + 8 * b0) = u;
          }
        }
      }
      if (ovf) report_status(status, kStatusRange);
      return true;
    }
  }
#pragma unroll 1
  for (int cp0 = tid; cp0 < half; cp0 += LB * NTHR) {
    float2 sc[LB];
#pragma unroll
    for (int q = 0; q < LB; ++q) {
      const int cp = cp0 + q * NTHR;
      sc[q] = make_float2(1.0f, 1.0f);
      if (cp < half) {
        if (ssm) sc[q] = *reinterpret_cast<const float2*>(ssm + 2 * cp);
        else if (P.scale) sc[q] = make_float2(__ldg(P.scale + 2 * cp), __ldg(P.scale + 2 * cp + 1));
      }
    }
#pragma unroll
    for (int q = 0; q < LB; ++q) {
      const int cp = cp0 + q * NTHR;
      if (cp >= half) continue;
      const int c = 2 * cp;
      const float f0 = P.sscale == 1 ? sc[q].x : 1.0f / sc[q].x, f1 = P.sscale == 1 ? sc[q].y : 1.0f / sc[q].y;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (r < nrows) {
          const float2 v = *reinterpret_cast<const float2*>(xs + (size_t)r * d + c);
          const size_t off = (size_t)(row0 + r) * d + c;
          if constexpr (F16OUT) {
            const __half2 h = __floats2half2_rn(v.x * f0, v.y * f1);
            ovf |= half2_inf(*reinterpret_cast<const uint32_t*>(&h));
            *reinterpret_cast<__half2*>(static_cast<__half*>(P.out) + off) = h;
          } else
            *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(P.out) + off) =
                __floats2bfloat162_rn(v.x * f0, v.y * f1);
        }
      }
    }
  }
  if (ovf) report_status(status, kStatusRange);
  return true;
}

}  // namespace rotdec
}  // namespace paro
