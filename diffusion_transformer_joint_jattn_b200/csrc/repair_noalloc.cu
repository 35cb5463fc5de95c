// FP8 attention with token repair for callers that cannot allocate device
// memory: the same path as jattn_fwd_fp8_repair, with its workspace in a
// file-scope device array instead of a caller buffer.
//
// Who needs it: code that runs where cudaMalloc is unavailable or must not
// be called -- inside a region being captured into a CUDA graph with a
// memory policy that forbids allocation, in a plug-in whose host framework
// owns every device allocation, or in a real-time loop that may not block
// on the allocator.  Such a caller still passes its inputs and outputs; the
// scratch comes from this file.
//
// The array lives in this translation unit alone.  With the CUDA runtime's
// default lazy module loading its memory is reserved only once a process
// first calls this entry point on a device; with CUDA_MODULE_LOADING=EAGER
// every process that loads the library reserves it on each device when the
// context is created.  Either way the device holds it until the process
// exits.  Its address is looked up once per device and context (the first
// call on a device does it; make that call before any stream capture) and
// looked up again after a cudaDeviceReset.  Calls on one device share the
// array: calls that overlap on the GPU race on it, so use one stream per
// device or serialise them.  Nothing in the array needs clearing between
// calls: every segment is written by the path before it is read.
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "jattn.h"
#include "jattn_internal.h"

namespace {

constexpr size_t kScratchBytes = JATTN_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) uint8_t g_repair_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};
unsigned long long g_ctx[kMaxDevices] = {};

// The array's device address for the current device (nullptr on failure).
// In host code the name g_repair_scratch is only a host-side stand-in; the
// kernels must be given this address.
void* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  const unsigned long long ctx = jattn::current_context_id();
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_addr[dev] == nullptr || ctx == 0 || g_ctx[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_repair_scratch) != cudaSuccess) return nullptr;
    g_addr[dev] = p;
    g_ctx[dev] = jattn::current_context_id();
  }
  return g_addr[dev];
}

}  // namespace

extern "C" jattn_status jattn_fwd_fp8_repair_noalloc(const jattn_shape* shape, const void* qkv_txt,
                                                     const void* qkv_img, const void* qkv_ref, const int32_t* pos,
                                                     float theta, const int32_t split[3], const float* norm_w,
                                                     float eps, float rho, void* o, float* lse, int32_t* repaired,
                                                     float softmax_scale, void* stream) {
  const size_t need = jattn_fwd_fp8_repair_workspace(shape, rho);
  if (need == 0)   // invalid shape or rho: the full entry point reports which, before any launch
    return jattn_fwd_fp8_repair(shape, qkv_txt, qkv_img, qkv_ref, pos, theta, split, norm_w, eps, rho, nullptr, 0,
                                o, lse, repaired, softmax_scale, stream);
  if (need > kScratchBytes) return JATTN_ERR_UNSUPPORTED;
  void* ws = scratch_address();
  if (ws == nullptr) return JATTN_ERR_CUDA;
  return jattn_fwd_fp8_repair(shape, qkv_txt, qkv_img, qkv_ref, pos, theta, split, norm_w, eps, rho, ws,
                              kScratchBytes, o, lse, repaired, softmax_scale, stream);
}
