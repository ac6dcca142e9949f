// Stream-K scratch that lives in a file-scope device array, for lbm_attend_frame_noalloc.
//
// Some callers of this library may not allocate device memory while frames stream: a
// serving runtime that owns every byte of the GPU through its own pool and budget, or a
// real-time frame loop where cudaMalloc / cudaFree would synchronise the device and stall
// the stream.  lbm_attend_frame_noalloc serves them: its stream-K partial results go to the
// array below, which the CUDA runtime places when the library is loaded, so the call itself
// allocates nothing.
//
// The array is shared by every call on a device and keeps the last call's contents.  No
// part of it needs to start at zero: each call writes every partial row it later reads.
// Calls that overlap on the GPU (two streams, or two caches at once) race on it.
#include <atomic>
#include <mutex>

#include "../../include/lbm.h"
#include "lbm_internal.h"

namespace lbm {
namespace {

constexpr size_t kNoallocScratchFloats = LBM_NOALLOC_SCRATCH_BYTES / sizeof(float);

static __device__ __align__(256) float g_noalloc_scratch[kNoallocScratchFloats];

// Device address of the array, per device, once looked up.  In host code the array's name
// is only a host-side stand-in: the address a kernel may be given comes from
// cudaGetSymbolAddress with that device current.  Host threads may make their first call on a
// device at the same time: the lookup runs under a mutex, the result is published with
// release / acquire order.
constexpr int kMaxDevices = 64;
std::atomic<float*> g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_lookup;

}  // namespace

// Device address of the scratch array on `device`, which must be the current device.  The
// first call on a device looks the address up (cudaGetSymbolAddress) and remembers it.
int noalloc_scratch(int device, float** ptr, size_t* floats) {
  if (device < 0 || device >= kMaxDevices || !ptr || !floats) return LBM_ERR_INVALID;
  float* p = g_scratch_ptr[device].load(std::memory_order_acquire);
  if (!p) {
    std::lock_guard<std::mutex> lock(g_scratch_lookup);
    p = g_scratch_ptr[device].load(std::memory_order_relaxed);
    if (!p) {
      void* addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr) {
        cudaGetLastError();
        return LBM_ERR_CUDA;
      }
      p = static_cast<float*>(addr);
      g_scratch_ptr[device].store(p, std::memory_order_release);
    }
  }
  *ptr = p;
  *floats = kNoallocScratchFloats;
  return LBM_OK;
}

}  // namespace lbm
