// NF4 quantisation entry point that allocates no device memory.
//
// lst_k_nf4_quantize needs two scratch arrays (the per-block absmax values and the per-group fp64
// partial sums of the double-quantisation mean) and gets them with cudaMalloc / cudaFree. Some
// callers cannot do that: code whose device memory is entirely reserved by its own caching
// allocator (a framework that has taken the GPU's memory up front), and code that must not
// trigger the device-wide synchronisation cudaFree implies while other streams are busy (for
// example a host-to-device weight copy running next to compute). This variant takes its scratch
// from one file-scope device array instead, sized for tensors of up to kNoAllocMaxElems elements.
// Every GPU that loads the library holds that array (4 MiB + 32 KiB) until the process exits.
#include "../../include/lst_kernels.h"
#include "common.cuh"
#include "nf4.cuh"

namespace {

constexpr int64_t kNoAllocMaxElems = int64_t(1) << 26;           // 67,108,864 elements per call
constexpr int64_t kAbsmaxFloats = kNoAllocMaxElems / 64;         // one fp32 absmax per 64 elements
constexpr int64_t kGsumDoubles = (kAbsmaxFloats + 255) / 256;    // one fp64 sum per 256 blocks
constexpr size_t kScratchBytes = (size_t)kAbsmaxFloats * 4 + (size_t)kGsumDoubles * 8;

// The scratch itself. In host code this name only stands in for the device array: its address on
// a device comes from cudaGetSymbolAddress below and is what the kernels receive.
static __device__ __align__(256) unsigned char g_nf4_noalloc_scratch[kScratchBytes];

}  // namespace

extern "C" lst_status lst_k_nf4_quantize_noalloc(const float* w, int64_t n, uint8_t* packed, int8_t* qabs,
                                                 float* gscale, float* mean, void* stream) {
  if (!w || !packed || !qabs || !gscale || !mean || n <= 0 || n % 64) return LST_ERR_ARG;
  if (n > kNoAllocMaxElems) return LST_ERR_ARG;  // beyond the fixed scratch: rejected, nothing launched
  // The array's address on the current device, looked up on every call (cheap, allocates
  // nothing): a cached address would go stale if the device's primary context were recreated
  // (cudaDeviceReset), which may place the module's arrays elsewhere.
  void* base = nullptr;
  if (cudaGetSymbolAddress(&base, g_nf4_noalloc_scratch) != cudaSuccess || !base) {
    cudaGetLastError();
    return LST_ERR_CUDA;
  }
  // Both scratch arrays are fully written by the quantiser before they are read, so nothing has
  // to be cleared between calls.
  float* absmax = static_cast<float*>(base);
  double* gsum = reinterpret_cast<double*>(static_cast<unsigned char*>(base) + kAbsmaxFloats * 4);
  lst::Nf4Out o{packed, qabs, gscale, mean};
  const cudaError_t e = lst::nf4_quantize(w, n, o, absmax, gsum, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    cudaGetLastError();
    return e == cudaErrorInvalidValue ? LST_ERR_ARG : LST_ERR_CUDA;
  }
  return LST_OK;
}
