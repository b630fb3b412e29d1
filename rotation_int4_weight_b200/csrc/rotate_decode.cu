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
#include "rotate_decode_cta.cuh"

namespace paro {
namespace {

constexpr int kRotThreads = 1024;
// warp 31 fetches the stage tables; the other 31 warps rotate
constexpr int kCompute = kRotThreads - 32;
constexpr size_t kRotSmemBudget = 227 * 1024 - 256;

// R token rows per CTA; UP pairs per thread and round of a stage (0: the
// default for R, 4 for one or two rows and 2 for four)
template <int R, bool F16OUT, int UP>
__global__ void __launch_bounds__(kRotThreads)
rot_decode_kernel(const __grid_constant__ RotBatch batch, int* status, int pdl_trigger, int pdl_wait) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ __align__(8) uint64_t bars[rotdec::kRotBars];
  // with flags, the INT4 launch that follows may start only once this grid has
  // waited for the previous kernel (it takes the launch epoch at its start, which
  // the previous INT4 launch on the workspace advanced at its end): the CTAs
  // let it launch right after that wait, inside the transform
  const bool flagged = batch.xflags != nullptr;
  if (pdl_trigger && !flagged) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  int pi = 0;
#pragma unroll 1
  while (pi + 1 < batch.count && (int)blockIdx.x >= batch.p[pi + 1].cta_begin) ++pi;
  const RotProblem& P = batch.p[pi];
  constexpr int U = UP > 0 ? UP : (R == 4 ? 2 : 4);
  const int rp = P.rows > 0 && P.rows < R ? P.rows : R;
  const int row0 = ((int)blockIdx.x - P.cta_begin) * rp;
  bool done;
  const bool trig_late = pdl_trigger && flagged;
  if (R > 1 && rp == 1) {
    // a linear too wide for more than one row a CTA (its stage tables need the
    // room): the one-row body, whose registers allow 7 pairs a thread and
    // round, so a stage of up to 13888 channels is one round, not several
    done = rotdec::rot_decode_cta<1, F16OUT, 7, kRotThreads>(P, row0, smem, bars, status, pdl_wait != 0,
                                                             trig_late);
  } else {
    done = rotdec::rot_decode_cta<R, F16OUT, U, kRotThreads>(P, row0, smem, bars, status, pdl_wait != 0,
                                                             trig_late);
  }
  if (flagged && done && !batch.skip_flags) {
    // every thread's x~ stores, then this CTA's flag (the tag of the launch
    // epoch, read after this grid's wait for the previous kernel)
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned long long e;
      asm volatile("ld.acquire.gpu.global.u64 %0, [%1];\n" : "=l"(e) : "l"(batch.ctl) : "memory");
      asm volatile("st.relaxed.gpu.global.u64 [%0], %1;\n" ::"l"(batch.xflags + blockIdx.x), "l"(2ull * e + 1ull)
                   : "memory");
    }
  }
}

size_t rot_smem(int d, int R, int ring, bool region = false) {
  return (size_t)d * R * 4 + (size_t)ring * 6 * d + (region ? (size_t)d * 4 : 0);
}

}  // namespace

int scale_mode(const RotProblem& p, int ring, bool region_fits) {
  if (!p.scale || (reinterpret_cast<uintptr_t>(p.scale) & 15) != 0) return 0;
  if (region_fits) return 1;
  return ring >= 2 && p.K >= 2 ? 2 : 0;
}

bool rot_decode_supported(int d, const void* pairs, const void* c, const void* s) {
  auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  return (d % 8) == 0 && rot_smem(d, 1, 1) <= kRotSmemBudget && al(pairs) && al(c) && al(s);
}

cudaError_t plan_rot_batch(const RotProblem* probs, int count, RotBatch* out, int* R_out) {
  if (count < 1 || count > kMaxBatch) return cudaErrorInvalidValue;
  int maxM = 0;
  for (int i = 0; i < count; ++i) maxM = probs[i].M > maxM ? probs[i].M : maxM;
  const int R = maxM >= 4 ? 4 : (maxM >= 2 ? 2 : 1);
  *out = RotBatch{};
  int ctas = 0;
  for (int i = 0; i < count; ++i) {
    RotProblem p = probs[i];
    // rows a CTA for this problem: as many as R while its rows and min(K, 3)
    // stages of tables fit.  A stage's rotation is shorter than the refill of
    // a table slot (issued when the slot frees), so a wide problem with a
    // shallower ring would wait on its tables every stage; it takes fewer rows
    // (more CTAs) instead.
    const int want = p.K < 1 ? 1 : (p.K < 3 ? p.K : 3);
    int rows = R;
    while (rows > 1 && rot_smem(p.d, rows, want) > kRotSmemBudget) rows >>= 1;
    // table slots: as many as fit beside a region for 1/scale while that
    // leaves two (or all K), else as many as fit without it
    const int all = p.K < 1 ? 1 : (p.K > 8 ? 8 : p.K);
    int ring = all;
    while (ring > 1 && rot_smem(p.d, rows, ring, true) > kRotSmemBudget) --ring;
    const bool region = rot_smem(p.d, rows, ring, true) <= kRotSmemBudget && ring >= (all < 2 ? all : 2);
    if (!region) {
      ring = all;
      while (ring > 1 && rot_smem(p.d, rows, ring) > kRotSmemBudget) --ring;
    }
    p.sscale = scale_mode(p, ring, region);
    p.rows = rows;
    p.ring = ring;
    p.cta_begin = ctas;
    ctas += (p.M + rows - 1) / rows;
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
    const int rows = b.p[i].rows > 0 && b.p[i].rows < R ? b.p[i].rows : R;
    const size_t s = rot_smem(b.p[i].d, rows, b.p[i].ring, b.p[i].sscale == 1);
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
