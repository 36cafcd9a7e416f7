// hlwq_gemm_noalloc: the small-M GEMM for callers that cannot allocate device
// memory.  Some callers cannot call cudaMalloc: code running inside a captured
// stream region that must not allocate, plug-ins embedded in a host that owns
// every allocation, and allocator-less runtimes that only hand out input and
// output buffers.  hlwq_gemm needs a scratch workspace for the rotated
// activations when it runs on the tensor cores (M >= 5 and rows of at most
// 8192 inputs); this entry point takes that scratch from a
// fixed-size array in device memory that belongs to the library instead.
//
// The array is a file-scope static __device__ object: every GPU that loads the
// library holds kNoallocScratchBytes of it until the process exits.  Host code
// cannot use the array's name as a device address, so the first call on each
// device looks the address up with cudaGetSymbolAddress (with that device
// current) and caches it; that first call should therefore come before any
// stream capture.  All calls on a device share the array and it keeps the last
// call's contents; nothing in it needs to start at zero (every call rewrites
// the part it reads), but calls whose executions overlap on the GPU race on it.

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>

#include "hlwq.h"

namespace hlwq {
size_t gemm_tc_workspace_min_bytes(int64_t O, int64_t in, int64_t M);
int gemm_check_args(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t out, int64_t in,
                    int64_t M, const uint16_t* X, int64_t ldx, const void* Y, int64_t ldy, int ydtype);
}  // namespace hlwq

namespace {

constexpr size_t kNoallocScratchBytes = HLWQ_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_setup_mutex;
std::atomic<void*> g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device (set up once per device).
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HLWQ_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return HLWQ_EUNSUPPORTED;
  void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (!p) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
    if (!p) {
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return HLWQ_ECUDA;
      g_scratch_ptr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return HLWQ_OK;
}

}  // namespace

extern "C" int hlwq_gemm_noalloc(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t out,
                                 int64_t in, int64_t M, const uint16_t* X, int64_t ldx, void* Y, int64_t ldy,
                                 int ydtype, void* stream) {
  // the same argument checks as hlwq_gemm, before any size is derived from them
  if (const int st = hlwq::gemm_check_args(packed, norms, codebook, out, in, M, X, ldx, Y, ldy, ydtype)) return st;
  // the tensor-core path runs with its smallest workspace here (it uses the K
  // split of its last tiles only when the scratch also holds the partials);
  // shapes that hlwq_gemm serves without a workspace need none
  const size_t need = hlwq_workspace_bytes(HLWQ_OP_GEMM, out, in, M, 1, 0)
                          ? hlwq::gemm_tc_workspace_min_bytes(out, in, M) : 0;
  if (need > kNoallocScratchBytes) return HLWQ_ESCRATCH;
  void* scratch = nullptr;
  if (need > 0) {
    const int st = scratch_for_current_device(&scratch);
    if (st != HLWQ_OK) return st;
  }
  return hlwq_gemm(packed, norms, codebook, out, in, M, X, ldx, Y, ldy, ydtype, scratch,
                   need > 0 ? kNoallocScratchBytes : 0, stream);
}
