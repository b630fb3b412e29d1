// Activation-side transform for few tokens (decode), several linears per launch:
//   x~ = diag(1/s) R_K ... R_1 x
// (page "ParoQuant: pairwise rotations that survive deployment", section "A
// rotation small enough to execute": disjoint channel pairs per stage, each
// rotated by x_i' = c x_i + s x_j, x_j' = -s x_i + c x_j; channel scale last).
//
// With one or a few token rows the work per stage is tiny and the time goes
// into fetching the stage tables (12 bytes per pair and stage), so the tables
// are requested up front: one thread of every CTA issues bulk (TMA) copies of
// as many whole stages (pairs, cos, sin) as fit in shared memory, each stage
// completing on its own mbarrier, and a bulk L2 prefetch of all later stages,
// so that the refill of a slot, issued as soon as its stage is done, waits for
// L2 rather than HBM.  Waits are bounded: a stage that never lands is reported
// as PARO_ERR_TIMEOUT.  The rows live in shared memory as fp32 (one plane per
// row, so channel c sits in bank c % 32 for every row), and each stage is one
// pass over its disjoint pairs followed by one barrier.
#include "paro_internal.cuh"
#include "rotate_decode.cuh"

namespace paro {
namespace {

constexpr int kRotThreads = 1024;
// warp 31 fetches the stage tables; the other 31 warps rotate
constexpr int kProducer = kRotThreads - 32;
constexpr int kCompute = kRotThreads - 32;
constexpr int kMaxRing = 8;
constexpr size_t kRotSmemBudget = 227 * 1024 - 256;

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
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, size_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(src), "r"((uint32_t)bytes) : "memory");
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n"
               ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

// R token rows per CTA; UP pairs per thread and round of a stage (0: the
// default for R, 4 for one or two rows and 2 for four)
template <int R, bool F16OUT, int UP>
__global__ void __launch_bounds__(kRotThreads)
rot_decode_kernel(const __grid_constant__ RotBatch batch, int* status, int pdl_trigger, int pdl_wait) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ __align__(8) uint64_t bars[kMaxRing + 1];
  if (pdl_trigger) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  int pi = 0;
#pragma unroll 1
  while (pi + 1 < batch.count && (int)blockIdx.x >= batch.p[pi + 1].cta_begin) ++pi;
  const RotProblem& P = batch.p[pi];
  const int d = P.d, K = P.K, half = d >> 1, ring = P.ring;
  const int row0 = ((int)blockIdx.x - P.cta_begin) * R;
  const int nrows = min(R, P.M - row0);
  const int tid = threadIdx.x;

  // shared memory: xs [R][d] fp32 (one plane per row: channel c in bank c % 32) |
  // ring [ring][6d] of stage tables
  float* xs = reinterpret_cast<float*>(smem);
  unsigned char* tab = reinterpret_cast<unsigned char*>(xs + (size_t)d * R);
  const size_t stage_bytes = (size_t)6 * d;  // pairs | cos | sin
  const uint32_t s_tab = static_cast<uint32_t>(__cvta_generic_to_shared(tab));
  const uint32_t s_bar = static_cast<uint32_t>(__cvta_generic_to_shared(bars));

  // one thread requests whole stages with bulk copies (three per stage); the
  // stage's mbarrier completes when all 6d bytes have landed
  auto issue_stage = [&](int k) {
    if (k < K) {
      const int slot = k % ring;
      const uint32_t base = s_tab + (uint32_t)(slot * stage_bytes), bar = s_bar + 8u * slot;
      mbar_expect_tx(bar, (uint32_t)stage_bytes);
      bulk_g2s(base, P.pairs + (size_t)k * half, 2u * d, bar);
      bulk_g2s(base + 2u * d, P.cos_t + (size_t)k * half, 2u * d, bar);
      bulk_g2s(base + 4u * d, P.sin_t + (size_t)k * half, 2u * d, bar);
    }
  };
  if (tid == kProducer) {
    for (int k = 0; k < kMaxRing; ++k) mbar_init(s_bar + 8u * k, 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    for (int k = 0; k < ring; ++k) issue_stage(k);
    // then the stages beyond the ring go to L2, so that their copies into the
    // ring later wait for L2 rather than HBM
    if (K > ring) {
      const size_t off = (size_t)ring * half, bytes = (size_t)(K - ring) * 2 * d;
      bulk_prefetch_l2(P.pairs + off, bytes);
      bulk_prefetch_l2(P.cos_t + off, bytes);
      bulk_prefetch_l2(P.sin_t + off, bytes);
    }
    if (P.scale && (reinterpret_cast<uintptr_t>(P.scale) & 15) == 0) bulk_prefetch_l2(P.scale, (size_t)4 * d);
  }
  // launched as a programmatic dependent: the tables above may be fetched while
  // the previous kernel finishes; the rows (which it may have written) and the
  // output (which it may still read) wait for it to complete
  if (pdl_wait) asm volatile("griddepcontrol.wait;\n" ::: "memory");
  // rows -> xs as fp32: each thread two adjacent channels of every row, the
  // loads of LB channel pairs issued before their stores so that their
  // latencies overlap
  constexpr int LB = R == 4 ? 2 : (R == 2 ? 4 : 8);
#pragma unroll 1
  for (int cp0 = tid; cp0 < half; cp0 += LB * kRotThreads) {
    __nv_bfloat162 v[LB][R];
#pragma unroll
    for (int q = 0; q < LB; ++q)
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int cp = cp0 + q * kRotThreads;
        v[q][r] = __floats2bfloat162_rn(0.f, 0.f);
        if (cp < half && r < nrows)
          v[q][r] = *reinterpret_cast<const __nv_bfloat162*>(P.x + (size_t)(row0 + r) * d + 2 * cp);
      }
#pragma unroll
    for (int q = 0; q < LB; ++q) {
      const int cp = cp0 + q * kRotThreads;
      if (cp < half) {
#pragma unroll
        for (int r = 0; r < R; ++r)
          *reinterpret_cast<float2*>(xs + (size_t)r * d + 2 * cp) = __bfloat1622float2(v[q][r]);
      }
    }
  }
  // The producer waits for each stage's table before the CTA barrier that
  // starts the stage, so that the barrier also tells the other threads that
  // the table has landed; it refills a slot as soon as the barrier after its
  // stage has passed.  With one slot the next stage can only be requested once
  // the current one is done, which costs a second barrier per stage.
  bool ok = true;
  if (tid == kProducer && K > 0) ok = mbar_wait_bounded(s_bar, 0u);
  int failed = __syncthreads_or(!ok);  // also: rows staged
  int issued = ring < K ? ring : K;    // stages requested so far (producer)

  // K stages.  The pairs of a stage are disjoint, so the loads of a batch of
  // pairs may all be issued before any of its stores.
  constexpr int U = UP > 0 ? UP : (R == 4 ? 2 : 4);
#pragma unroll 1
  for (int k = 0; k < K && !failed; ++k) {
    if (tid < kCompute) {
      const unsigned char* st = tab + (size_t)(k % ring) * stage_bytes;
      const uint32_t* pk = reinterpret_cast<const uint32_t*>(st);
      const float* ck = reinterpret_cast<const float*>(st + 2 * d);
      const float* sk = reinterpret_cast<const float*>(st + 4 * d);
      for (int t0 = tid; t0 < half; t0 += U * kCompute) {
        int ii[U], jj[U];
        float c[U], sn[U], a[U][R], b[U][R];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int t = t0 + u * kCompute;
          ii[u] = -1;
          if (t < half) {
            const uint32_t pr = pk[t];
            const int i = pr & 0xFFFF, j = pr >> 16;
            if (i < d && j < d) { ii[u] = i; jj[u] = j; c[u] = ck[t]; sn[u] = sk[t]; }
            else report_status(status, kStatusBadIndex);
          }
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
          if (ii[u] >= 0) {
#pragma unroll
            for (int r = 0; r < R; ++r) {
              a[u][r] = xs[(size_t)r * d + ii[u]];
              b[u][r] = xs[(size_t)r * d + jj[u]];
            }
          }
#pragma unroll
        for (int u = 0; u < U; ++u)
          if (ii[u] >= 0) {
            float na[R], nb[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
              na[r] = fmaf(c[u], a[u][r], sn[u] * b[u][r]);
              nb[r] = fmaf(-sn[u], a[u][r], c[u] * b[u][r]);
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
              xs[(size_t)r * d + ii[u]] = na[r];
              xs[(size_t)r * d + jj[u]] = nb[r];
            }
          }
      }
    } else if (tid == kProducer && ring > 1) {
      // stage k - 1's slot is free since the barrier that started this stage
      if (k >= 1 && k - 1 + ring < K) {
        issue_stage(k - 1 + ring);
        ++issued;
      }
      if (k + 1 < K) ok = mbar_wait_bounded(s_bar + 8u * ((k + 1) % ring), (uint32_t)(((k + 1) / ring) & 1));
    }
    failed = __syncthreads_or(!ok);
    if (ring == 1 && k + 1 < K && !failed) {
      if (tid == kProducer) {
        issue_stage(k + 1);
        ++issued;
        ok = mbar_wait_bounded(s_bar, (uint32_t)((k + 1) & 1));
      }
      failed = __syncthreads_or(!ok);
    }
  }
  if (failed) {
    // a stage never arrived: report, let the latest copy of every slot land
    // (each wait bounded again), then leave
    if (tid == kProducer) {
      report_status(status, kStatusTimeout);
      for (int q = issued > ring ? issued - ring : 0; q < issued; ++q)
        mbar_wait_bounded(s_bar + 8u * (q % ring), (uint32_t)((q / ring) & 1));
    }
    __syncthreads();
    return;
  }

  // channel scale and store: the scales of LB channel pairs are loaded (from
  // L2, where the prologue put them) before any of them is used
#pragma unroll 1
  for (int cp0 = tid; cp0 < half; cp0 += LB * kRotThreads) {
    float2 sc[LB];
#pragma unroll
    for (int q = 0; q < LB; ++q) {
      const int cp = cp0 + q * kRotThreads;
      sc[q] = make_float2(1.0f, 1.0f);
      if (P.scale && cp < half) sc[q] = make_float2(__ldg(P.scale + 2 * cp), __ldg(P.scale + 2 * cp + 1));
    }
#pragma unroll
    for (int q = 0; q < LB; ++q) {
      const int cp = cp0 + q * kRotThreads;
      if (cp >= half) continue;
      const int c = 2 * cp;
      const float f0 = 1.0f / sc[q].x, f1 = 1.0f / sc[q].y;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (r < nrows) {
          const float2 v = *reinterpret_cast<const float2*>(xs + (size_t)r * d + c);
          const size_t off = (size_t)(row0 + r) * d + c;
          if constexpr (F16OUT)
            *reinterpret_cast<__half2*>(static_cast<__half*>(P.out) + off) = __floats2half2_rn(v.x * f0, v.y * f1);
          else
            *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(P.out) + off) =
                __floats2bfloat162_rn(v.x * f0, v.y * f1);
        }
      }
    }
  }
}

size_t rot_smem(int d, int R, int ring) { return (size_t)d * R * 4 + (size_t)ring * 6 * d; }

}  // namespace

bool rot_decode_supported(int d, const void* pairs, const void* c, const void* s) {
  auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  return (d % 8) == 0 && rot_smem(d, 1, 1) <= kRotSmemBudget && al(pairs) && al(c) && al(s);
}

cudaError_t plan_rot_batch(const RotProblem* probs, int count, RotBatch* out, int* R_out) {
  if (count < 1 || count > kMaxBatch) return cudaErrorInvalidValue;
  int maxM = 0;
  for (int i = 0; i < count; ++i) maxM = probs[i].M > maxM ? probs[i].M : maxM;
  int R = maxM >= 4 ? 4 : (maxM >= 2 ? 2 : 1);
  // the widest problem must still hold its rows and two stages (one copy in
  // flight while the other is used)
  for (int i = 0; i < count; ++i)
    while (R > 1 && rot_smem(probs[i].d, R, probs[i].K > 1 ? 2 : 1) > kRotSmemBudget) R >>= 1;
  *out = RotBatch{};
  int ctas = 0;
  for (int i = 0; i < count; ++i) {
    RotProblem p = probs[i];
    int ring = p.K < 1 ? 1 : p.K;
    if (ring > 8) ring = 8;
    while (ring > 1 && rot_smem(p.d, R, ring) > kRotSmemBudget) --ring;
    p.ring = ring;
    p.cta_begin = ctas;
    ctas += (p.M + R - 1) / R;
    out->p[i] = p;
  }
  out->count = count;
  out->total_ctas = ctas;
  *R_out = R;
  return cudaSuccess;
}

cudaError_t launch_rot_batch(const RotBatch& b, int R, bool f16_out, int* status, cudaStream_t stream,
                             bool pdl_trigger, bool pdl_wait) {
  size_t smem = 0;
  for (int i = 0; i < b.count; ++i) {
    const size_t s = rot_smem(b.p[i].d, R, b.p[i].ring);
    smem = s > smem ? s : smem;
  }
  const int trig = pdl_trigger ? 1 : 0, wait = pdl_wait ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(b.total_ctas);
  cfg.blockDim = dim3(kRotThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_wait ? 1 : 0;
  cudaError_t e;
#define PARO_ROT_LAUNCH(r, f16, up)                                                                 \
  {                                                                                                 \
    auto k = rot_decode_kernel<r, f16, up>;                                                         \
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);            \
    if (e != cudaSuccess) return e;                                                                 \
    return cudaLaunchKernelEx(&cfg, k, b, status, trig, wait);                                      \
  }
  // enough pairs per thread that a stage of the widest problem is one round of
  // loads and stores, within the registers each row count leaves (one row: up
  // to 8; two rows: 5; four rows: 3)
  int max_half = 0;
  for (int i = 0; i < b.count; ++i) max_half = b.p[i].d / 2 > max_half ? b.p[i].d / 2 : max_half;
  const int rounds = (max_half + kCompute - 1) / kCompute;  // pairs per thread in one round
  if (f16_out) {
    if (R == 4) {
      if (rounds == 3) PARO_ROT_LAUNCH(4, true, 3) else PARO_ROT_LAUNCH(4, true, 0)
    } else if (R == 2) {
      if (rounds == 5) PARO_ROT_LAUNCH(2, true, 5) else PARO_ROT_LAUNCH(2, true, 0)
    } else {
      if (rounds == 5) PARO_ROT_LAUNCH(1, true, 5)
      else if (rounds == 6 || rounds == 7) PARO_ROT_LAUNCH(1, true, 7)
      else if (rounds >= 8) PARO_ROT_LAUNCH(1, true, 8)
      else PARO_ROT_LAUNCH(1, true, 0)
    }
  } else {
    if (R == 4) {
      if (rounds == 3) PARO_ROT_LAUNCH(4, false, 3) else PARO_ROT_LAUNCH(4, false, 0)
    } else if (R == 2) {
      if (rounds == 5) PARO_ROT_LAUNCH(2, false, 5) else PARO_ROT_LAUNCH(2, false, 0)
    } else {
      if (rounds == 5) PARO_ROT_LAUNCH(1, false, 5)
      else if (rounds == 6 || rounds == 7) PARO_ROT_LAUNCH(1, false, 7)
      else if (rounds >= 8) PARO_ROT_LAUNCH(1, false, 8)
      else PARO_ROT_LAUNCH(1, false, 0)
    }
  }
#undef PARO_ROT_LAUNCH
}

}  // namespace paro
