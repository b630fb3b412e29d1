// paro_rotate_w4_linear_noalloc: the fused rotate + INT4 linear for callers
// that cannot allocate device memory.
//
// Who cannot allocate: code that runs where cudaMalloc/cudaFree are off
// limits, e.g. a plugin hosted by an inference engine that owns every byte of
// device memory and hands its plugins no workspace, a latency-critical path
// that must not take the implicit device synchronisation cudaFree can cause,
// or a program that reserves all of its memory at start-up and forbids any
// allocation afterwards.  Those callers still own their inputs and outputs;
// only the fused call's scratch is provided here, by a fixed device array
// that the library carries: the transformed activations in fp16 and, up to 16
// tokens, the stream-K INT4 kernel's publication flags and partial tiles.
//
// The array is a file-scope __device__ variable: every GPU that loads this
// library holds PARO_NOALLOC_SCRATCH_BYTES (4 MiB) until the process exits.
// Host code cannot use the array's name as a device address (it is a
// host-side stand-in), so the entry point looks the address up once per
// device with cudaGetSymbolAddress, with that device current, and passes it
// to the kernels as their workspace.
#include <atomic>

#include "paro_internal.cuh"

namespace {

// M * d_in of one call may not exceed this many fp16 elements (e.g. M = 16
// tokens of width 16384, or one token of width 49152); the rest of the array
// holds the stream-K kernel's partial tiles and flags, which need about
// 16.4 KB per SM at 9-16 tokens (the call runs the stream-K kernel on whole
// tiles per CTA, without partials, on a GPU with so many SMs that they do not
// fit)
constexpr size_t kNoAllocMaxElems = size_t(1) << 18;
constexpr size_t kScratchBytes = PARO_NOALLOC_SCRATCH_BYTES;
static_assert(kScratchBytes >= kNoAllocMaxElems * sizeof(__half), "scratch holds the transformed activations");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of the scratch array on the current device; looked up on the
// first call made on each device.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (!p) {
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return cudaSuccess;
}

}  // namespace

extern "C" paro_status paro_rotate_w4_linear_noalloc(const uint16_t* d_x, int K, const uint16_t* d_pairs,
                                                     const float* d_cos, const float* d_sin, const float* d_scale,
                                                     const uint32_t* d_qweight, const uint16_t* d_scales,
                                                     const uint16_t* d_zeros, uint16_t* d_y, int M, int d_in,
                                                     int d_out, int group_size, paro_stream_t stream) {
  if (M > 0 && d_in > 0 && (size_t)M * (size_t)d_in > kNoAllocMaxElems) {
    return paro::record_error(PARO_ERR_UNSUPPORTED,
                              "paro_rotate_w4_linear_noalloc: M * d_in = %zu exceeds the built-in scratch of %zu "
                              "fp16 values; use paro_rotate_w4_linear with a caller-provided workspace",
                              (size_t)M * (size_t)d_in, kNoAllocMaxElems);
  }
  void* scratch = nullptr;
  if (M > 0) {
    cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess)
      return paro::record_error(PARO_ERR_CUDA, "paro_rotate_w4_linear_noalloc: scratch address lookup: %s",
                                cudaGetErrorString(e));
  }
  // Same validation and kernels as the workspace-taking call given a workspace
  // of kScratchBytes.  That workspace must be zero before its first use: the
  // array is, as a __device__ variable without initializer is zero when the
  // module loads, and every call leaves it in the state the next call expects
  // (the transform overwrites every activation it hands to the linear; the
  // stream-K flags hold a launch epoch that each launch advances).
  return paro_rotate_w4_linear(d_x, K, d_pairs, d_cos, d_sin, d_scale, d_qweight, d_scales, d_zeros, d_y, M,
                               d_in, d_out, group_size, scratch, kScratchBytes, stream);
}
