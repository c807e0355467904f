// quantize_noalloc.cu — the NF4 quantiser for callers that cannot allocate.
//
// qlora_quantize() asks the caller for a workspace (the per-block absmax values
// and the per-group float64 sums the fixed-order mean is built from).  Some
// callers have no way to provide one: a plugin or custom-op interface that
// hands the library its input and output buffers but no allocator, code that
// runs while a framework's allocator forbids new device allocations (for
// example mid-step under a fixed memory plan), or runtimes where cudaMalloc is
// off limits because it can synchronise the device.  For them this entry point
// keeps that scratch in a file-scope __device__ array instead, so the call
// itself allocates nothing: no cudaMalloc, no cudaFree, no allocating library
// routine.
//
// Cost and limits: the array is part of the loaded module, so every GPU that
// loads this library holds kScratchBytes (about 4 MiB) until the process exits.
// The weight may have at most kMaxWeights elements (N*K <= 2^26, e.g. 8192 x
// 8192); larger weights are rejected with QLORA_ERR_TOO_LARGE before anything
// is launched.  All calls share the one array: two calls whose kernels overlap
// on the GPU (different streams, or different host threads) race on it and give
// undefined results; calls on one stream are ordered and safe.  The array keeps
// the previous call's contents; nothing in it needs to start at zero (every
// absmax slot and group sum used is written before it is read, and the padding
// of the mean's summation tree is cleared by the kernel that reads it).
//
// Host code cannot use the array's name as a device address (it is a host-side
// stand-in for the symbol), so each call looks the address up with
// cudaGetSymbolAddress on the current device and remembers it per device.  A
// call made while its stream is being captured into a CUDA graph uses the
// remembered address instead (looking a symbol up can load the module, which
// capture does not allow), so the first call on each device should come before
// any stream capture.  Looking the address up again on every other call keeps it
// valid after cudaDeviceReset or a new primary context, which reload the module
// at another address.
#include <cstdint>
#include <cstring>
#include <mutex>
#include <cuda_runtime.h>
#include "internal.h"

namespace qlora {
namespace {

constexpr int64_t kMaxWeights = int64_t(1) << 26;           // N*K limit
constexpr int64_t kMaxBlocks = kMaxWeights / 64;             // absmax slots (float32)
constexpr int64_t kMaxGroupSlots = kMaxBlocks / 256;         // group sums, already a power of two (float64)
constexpr size_t kAbsmaxBytes = static_cast<size_t>(kMaxBlocks) * 4;
constexpr size_t kScratchBytes = kAbsmaxBytes + static_cast<size_t>(kMaxGroupSlots) * 8;
static_assert((kMaxGroupSlots & (kMaxGroupSlots - 1)) == 0, "tree size must be a power of two");
static_assert(kAbsmaxBytes % 256 == 0, "group sums stay 256-byte aligned");

static __device__ __align__(256) unsigned char g_quant_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_quant_scratch on the current device: looked up afresh unless
// `stream` is capturing, when the address remembered from an earlier call is used.
cudaError_t scratch_for_current_device(cudaStream_t stream, void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(stream, &cs);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mu);
  if (cs == cudaStreamCaptureStatusNone) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_quant_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  } else if (!g_scratch_ptr[dev]) {
    return cudaErrorStreamCaptureUnsupported;  // no earlier call on this device to take the address from
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace qlora

using namespace qlora;

extern "C" qlora_status qlora_quantize_noalloc(const uint16_t *W, const qlora_nf4_weight *out, int *dev_err,
                                               void *stream) {
  if (!W || !out || !out->codes || !out->c2q || !out->c1 || !out->mean) return QLORA_ERR_INVALID_ARG;
  if (out->N < 1 || out->K < 64) return QLORA_ERR_INVALID_ARG;
  if (out->K % 64 != 0) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (out->N > kMaxWeights || out->K > kMaxWeights || out->N * out->K > kMaxWeights) return QLORA_ERR_TOO_LARGE;
  if (!aligned16(W) || !aligned16(out->codes) || !aligned16(out->c2q) || !aligned16(out->c1) ||
      !aligned16(out->mean))
    return QLORA_ERR_MISALIGNED;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10)
    return QLORA_ERR_NO_DEVICE;
  void *scratch = nullptr;
  const cudaError_t es = scratch_for_current_device(static_cast<cudaStream_t>(stream), &scratch);
  if (es != cudaSuccess) return cuda_status(es);
  float levels[16];
  Nf4Thresholds thr;
  build_codebook_f32(levels, thr.t);
  const int64_t nb = out->N * out->K / 64;
  const int64_t ng = (nb + 255) / 256;
  int64_t tree = 1;
  while (tree < ng) tree *= 2;
  unsigned char *base = static_cast<unsigned char *>(scratch);
  const cudaError_t e =
      launch_quantize(W, nb, out->codes, out->c2q, out->c1, out->mean, reinterpret_cast<float *>(base),
                      reinterpret_cast<double *>(base + kAbsmaxBytes), tree, thr, dev_err,
                      static_cast<cudaStream_t>(stream));
  return cuda_status(e);
}
