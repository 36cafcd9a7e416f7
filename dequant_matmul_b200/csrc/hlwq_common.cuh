// Shared device helpers for the HLWQ Q5 kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "hlwq.h"

namespace hlwq {

constexpr int kBlock = 128;      // weights per block (Method step [1])
constexpr int kBlockBytes = 80;  // 128 codes x 5 bits (Method step [5])
constexpr int kLevels = 32;      // centroids (Method step [4])

// Device error word (see hlwq_device_error in hlwq.h).
__device__ unsigned int g_device_error = 0u;

__device__ __forceinline__ void raise_device_error(unsigned bits) { atomicOr(&g_device_error, bits); }

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b16) { return __uint_as_float(b16 << 16); }

// Two bf16 values packed in a 32-bit word -> fp32 (exact).
__device__ __forceinline__ float bf16x2_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16x2_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ uint32_t float_to_bf16_bits(float f) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(f)));
}

__device__ __forceinline__ float half_bits_to_float(uint16_t h) { return __half2float(__ushort_as_half(h)); }

// Streaming 128-bit load that does not allocate in L1 (data read once).
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Packed fp32 pair arithmetic (sm_100 f32x2 instructions).
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 r;
  asm("{ .reg .b64 pa, pb, pd; mov.b64 pa, {%2, %3}; mov.b64 pb, {%4, %5};\n\t"
      "add.rn.f32x2 pd, pa, pb; mov.b64 {%0, %1}, pd; }"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  float2 r;
  asm("{ .reg .b64 pa, pb, pd; mov.b64 pa, {%2, %3}; mov.b64 pb, {%4, %5};\n\t"
      "sub.rn.f32x2 pd, pa, pb; mov.b64 {%0, %1}, pd; }"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 r;
  asm("{ .reg .b64 pa, pb, pc, pd; mov.b64 pa, {%2, %3}; mov.b64 pb, {%4, %5}; mov.b64 pc, {%6, %7};\n\t"
      "fma.rn.f32x2 pd, pa, pb, pc; mov.b64 {%0, %1}, pd; }"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return r;
}

// Extract 10 bits starting at bit `sh` of the 64-bit pair (lo, hi).
template <int SH>
__device__ __forceinline__ uint32_t bits10(uint32_t lo, uint32_t hi) {
  if constexpr (SH <= 22) {
    return (lo >> SH) & 0x3ffu;
  } else {
    return __funnelshift_r(lo, hi, SH) & 0x3ffu;
  }
}

template <int SH>
__device__ __forceinline__ uint32_t bits5(uint32_t lo, uint32_t hi) {
  if constexpr (SH <= 27) {
    return (lo >> SH) & 0x1fu;
  } else {
    return __funnelshift_r(lo, hi, SH) & 0x1fu;
  }
}

// Host-side set-up done once per device (kernel attributes belong to the
// device that was current when they were set).  Thread-safe; a device index
// at or above kMaxDevices is refused with HLWQ_EUNSUPPORTED.
constexpr int kMaxDevices = 64;

struct PerDeviceOnce {
  std::atomic<bool> done[kMaxDevices];
  std::mutex mu;
  // Runs f() (returning true on success) on the current device unless it has
  // succeeded there before; HLWQ_OK, HLWQ_ECUDA or HLWQ_EUNSUPPORTED.
  template <class F>
  int operator()(F&& f) {
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess) return HLWQ_ECUDA;
    if (d < 0 || d >= kMaxDevices) return HLWQ_EUNSUPPORTED;
    if (done[d].load(std::memory_order_acquire)) return HLWQ_OK;
    std::lock_guard<std::mutex> lock(mu);
    if (done[d].load(std::memory_order_relaxed)) return HLWQ_OK;
    if (!f()) return HLWQ_ECUDA;
    done[d].store(true, std::memory_order_release);
    return HLWQ_OK;
  }
};

// Number of SMs of the current device (cached per device; 148 if the query fails).
inline int sm_count() {
  static std::atomic<int> n[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int v = n[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    n[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

__host__ __device__ constexpr int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace hlwq
