#pragma once
// HLWQ Q5 quantizer and dequantizer kernels (sm_100a).
//
// Quantizer ("Qwen3.6-35B-A3B -- HLWQ Q5" model card, Method steps [1]-[5]).
// Four lanes own one 128-weight block, 32 consecutive weights each, so a warp
// covers 8 consecutive blocks and its loads and stores are contiguous.  The
// Walsh-Hadamard rotation is seven butterfly stages in natural (Sylvester)
// order: the five stages within a lane's 32 values run in registers, the two
// that pair values 32 and 64 apart exchange registers between the block's four
// lanes with shuffles.  The per-lane code is small (no 128-way unrolling), which
// keeps the kernel inside the instruction cache.
//
// Nearest-centroid assignment (step [4]) uses a bucket table: y is mapped to a
// bucket of width 1/64 by one FFMA whose rounding leaves the bucket index in the
// low mantissa bits; each bucket holds at most one decision midpoint, stored as
// an fp32 threshold whose low 5 bits carry the code of the bucket's lower edge,
// so one compare finishes the search.  y is clamped to the table's range
// [-3, 3] first; values beyond it land in the edge buckets, which send them to
// the exact path below when a midpoint lies beyond the table on their side
// (never for the Lloyd-Max codebook).  The table is replicated once per lane
// (lane l reads bank l), so lookups never conflict.  A grid shift sigma keeps every midpoint at least 4e-5 from a
// bucket edge.
//
// Exactness.  The fp32 rotation differs from the exact value by at most ~7.5e-6
// (seven rounded additions of terms whose magnitudes sum to <= sqrt(128), plus
// the scaling), and a stored threshold differs from its midpoint by at most
// 31 ulps; every element within 2e-5 of a threshold is re-decided exactly: the
// warp recomputes that one rotated value in fp64 from the original weights
// (32 lanes x 4 terms, shuffle reduction) and compares it with the fp64
// midpoints.  The norm is treated the same way: a block whose fp32 norm lies
// within 2e-6 (relative) of a binary16 rounding midpoint gets its norm
// recomputed in fp64 by the warp.  The result is the nearest-centroid encoding
// of the exactly rotated block, ties to the lower index.
//
// Dequantizer ("Qwopus3.6-27B-v2 . HLWQ Q5", Pipeline: dequantize per-Linear).
// The inverse is the same rotation (H symmetric, H H = 128 I): same lane layout,
// centroid lookups from a 32-entry shared table, butterflies, scale n16 / 128.

#include "hlwq_common.cuh"

namespace hlwq {

namespace {

constexpr int kQThreads = 256;
constexpr int kQCtasPerSm = 3;  // 85 registers per thread: the code group and the rotation stay in registers
constexpr int kQBuckets = 385;           // clamped shifted value in [-3, 3] at 1/64 resolution
constexpr float kQGuard = 2e-5f;
constexpr float kQMagic = 12583104.0f;   // 1.5 * 2^23 + 192: fmaf(y, 64, kQMagic) -> round(64 y + 192) in the low bits
constexpr int kQTabWords = kQBuckets * 32;
constexpr int kQSmemBytes = kQTabWords * 4 + 31 * 8 + 16;

struct QuantShared {
  uint32_t* tab;  // [kQBuckets][32] lane-replicated entries
  double* mid;    // [31] exact midpoints
  float* sigma;
};

__device__ __forceinline__ QuantShared quant_shared(uint8_t* smem) {
  QuantShared q;
  q.tab = reinterpret_cast<uint32_t*>(smem);
  q.mid = reinterpret_cast<double*>(smem + kQTabWords * 4);
  q.sigma = reinterpret_cast<float*>(smem + kQTabWords * 4 + 31 * 8);
  return q;
}

// All-15 code pattern (the code of y = 0 under ties-to-lower) for a lane's
// 32 codes (160 bits, 5 words): fields of 0b01111.
__host__ __device__ constexpr uint32_t code15_word(int w) {
  uint32_t r = 0;
  for (int bit = 0; bit < 32; ++bit)
    if (((w * 32 + bit) % 5) < 4) r |= 1u << bit;
  return r;
}

__device__ void build_quant_tables(const QuantShared& s, const float* __restrict__ codebook) {
  const int tid = threadIdx.x;
  if (tid < kLevels - 1) {
    const float a = __ldg(codebook + tid), b = __ldg(codebook + tid + 1);
    s.mid[tid] = 0.5 * (static_cast<double>(a) + static_cast<double>(b));
    if (!(a < b) || !isfinite(a) || !isfinite(b)) raise_device_error(HLWQ_DEVERR_CODEBOOK);
  }
  __syncthreads();
  if (tid < 32) {
    // lane q tests the shift q/1024; a midpoint m lands at position 64 (m + sigma) + 192,
    // bucket edges at half-integers.
    const double sig = tid < 16 ? tid * (1.0 / 1024.0) : 0.0;
    bool ok = tid < 16;
    for (int k = 0; k < kLevels - 1 && ok; ++k) {
      const double p = 64.0 * (s.mid[k] + sig) + 192.0;
      if (fabs(p - floor(p) - 0.5) < 64.0 * 4e-5) ok = false;
    }
    const unsigned good = __ballot_sync(0xffffffffu, ok);
    if (tid == 0) *s.sigma = good ? static_cast<float>((__ffs(good) - 1) * (1.0 / 1024.0)) : -1.0f;
  }
  __syncthreads();
  const bool shifted = *s.sigma >= 0.0f;
  const double sig = shifted ? static_cast<double>(*s.sigma) : 0.0;
  for (int i = tid; i < kQBuckets; i += blockDim.x) {
    const double lo = (i - 192.5) / 64.0, hi = (i - 191.5) / 64.0;
    int below = 0, inside = 0, inside_k = -1;
    bool risky = false;
    for (int k = 0; k < kLevels - 1; ++k) {
      const double m = s.mid[k] + sig;
      if (m < lo) ++below;
      else if (m <= hi) { ++inside; inside_k = k; }
      if (!shifted && (fabs(m - lo) < 4e-5 || fabs(m - hi) < 4e-5)) risky = true;
    }
    // values beyond the table's range land in the edge buckets: those take
    // the exact path when a midpoint (ascending) lies beyond the range on
    // their side
    const bool beyond = (i == 0 && s.mid[0] + sig < lo) || (i == kQBuckets - 1 && s.mid[kLevels - 2] + sig > hi);
    uint32_t thr;
    if (inside >= 2 || risky || beyond) thr = 0x7fc00000u;            // NaN: always the exact path
    else if (inside == 1) thr = __float_as_uint(static_cast<float>(s.mid[inside_k] + sig));
    else thr = __float_as_uint(3.0e38f);
    const uint32_t e = (thr & ~31u) | static_cast<uint32_t>(below);
    for (int l = 0; l < 32; ++l) s.tab[i * 32 + l] = e;
  }
  __syncthreads();
  if (tid == 0 && !shifted) *s.sigma = 0.0f;
  __syncthreads();
}

// Butterfly stage over a lane's 32 values (pairs H apart); for H >= 2 the
// pairs (v[i], v[i+1]) are processed as packed f32x2.
template <int H>
__device__ __forceinline__ void stage32(float (&v)[32]) {
  if constexpr (H == 1) {
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float a = v[i], b = v[i + 1];
      v[i] = a + b;
      v[i + 1] = a - b;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; i += 2)
      if ((i & H) == 0) {
        const float2 a = make_float2(v[i], v[i + 1]), b = make_float2(v[i + H], v[i + H + 1]);
        const float2 s = add2(a, b), d = sub2(a, b);
        v[i] = s.x; v[i + 1] = s.y;
        v[i + H] = d.x; v[i + H + 1] = d.y;
      }
  }
}

// Cross-lane butterfly stage: values 32*LM apart live in lanes LM apart.
template <int LM>
__device__ __forceinline__ void stage_x(float (&v)[32], int lane) {
  const float sg = (lane & LM) ? -1.0f : 1.0f;
  const float2 sgn = make_float2(sg, sg);
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float2 p = make_float2(__shfl_xor_sync(0xffffffffu, v[i], LM), __shfl_xor_sync(0xffffffffu, v[i + 1], LM));
    const float2 r = fma2(make_float2(v[i], v[i + 1]), sgn, p);  // lower lane: v + p; upper lane: p - v
    v[i] = r.x;
    v[i + 1] = r.y;
  }
}

// The full 128-point transform of the block held by 4 lanes (32 values each).
__device__ __forceinline__ void fwht_4lanes(float (&v)[32], int lane) {
  stage32<1>(v);
  stage32<2>(v);
  stage32<4>(v);
  stage32<8>(v);
  stage32<16>(v);
  stage_x<1>(v, lane);
  stage_x<2>(v, lane);
}

template <bool kBf16, bool kVec>
__device__ __forceinline__ void load_quarter(const void* __restrict__ base, int qlen, float (&v)[32]) {
  if constexpr (kVec && kBf16) {
    const uint4* p = static_cast<const uint4*>(base);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint4 u = make_uint4(0, 0, 0, 0);
      if (8 * c < qlen) u = ldg_stream(p + c);
      v[8 * c + 0] = bf16x2_lo(u.x); v[8 * c + 1] = bf16x2_hi(u.x);
      v[8 * c + 2] = bf16x2_lo(u.y); v[8 * c + 3] = bf16x2_hi(u.y);
      v[8 * c + 4] = bf16x2_lo(u.z); v[8 * c + 5] = bf16x2_hi(u.z);
      v[8 * c + 6] = bf16x2_lo(u.w); v[8 * c + 7] = bf16x2_hi(u.w);
    }
  } else if constexpr (kVec && !kBf16) {
    const uint4* p = static_cast<const uint4*>(base);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint4 u = make_uint4(0, 0, 0, 0);
      if (4 * c < qlen) u = ldg_stream(p + c);
      v[4 * c + 0] = __uint_as_float(u.x); v[4 * c + 1] = __uint_as_float(u.y);
      v[4 * c + 2] = __uint_as_float(u.z); v[4 * c + 3] = __uint_as_float(u.w);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      float f = 0.0f;
      if (e < qlen) {
        if constexpr (kBf16) f = bf16_bits_to_float(__ldg(static_cast<const uint16_t*>(base) + e));
        else f = __ldg(static_cast<const float*>(base) + e);
      }
      v[e] = f;
    }
  }
}

__device__ __forceinline__ uint32_t lds_u32_q(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

template <bool kBf16>
__device__ __forceinline__ double load_elem64(const void* base, int i, int len) {
  if (i >= len) return 0.0;
  if constexpr (kBf16) return static_cast<double>(bf16_bits_to_float(static_cast<const uint16_t*>(base)[i]));
  else return static_cast<double>(static_cast<const float*>(base)[i]);
}

__device__ __forceinline__ double warp_sum64(double x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  return x + __shfl_xor_sync(0xffffffffu, x, 2);
}

// Reductions over the 4 lanes of one block; `mask` names those lanes only, so
// they may be called where other blocks of the warp took another branch.
__device__ __forceinline__ float quad_max(float x, unsigned mask) {
  x = fmaxf(x, __shfl_xor_sync(mask, x, 1));
  return fmaxf(x, __shfl_xor_sync(mask, x, 2));
}

__device__ __forceinline__ float quad_sum_m(float x, unsigned mask) {
  x += __shfl_xor_sync(mask, x, 1);
  return x + __shfl_xor_sync(mask, x, 2);
}

// Replaces the 5-bit field of code e (0..31) in a lane's 160-bit group p[5].
__device__ __forceinline__ void patch_code(uint32_t (&p)[5], int e, uint32_t code) {
  // the field's bits are written into each word they overlap, with shift
  // amounts computed at run time (a runtime index into p would put the whole
  // group in local memory)
  const int bit = 5 * e;
#pragma unroll
  for (int q = 0; q < 5; ++q) {
    const int rel = bit - 32 * q;  // field position relative to word q
    if (rel > -5 && rel < 32) {
      const uint64_t m64 = rel >= 0 ? (31ull << rel) : (31ull >> -rel);
      const uint64_t c64 = rel >= 0 ? (static_cast<uint64_t>(code) << rel) : (static_cast<uint64_t>(code) >> -rel);
      p[q] = (p[q] & ~static_cast<uint32_t>(m64)) | static_cast<uint32_t>(c64);
    }
  }
}

template <bool kBf16, bool kVec>
__global__ void __launch_bounds__(kQThreads, kQCtasPerSm)
quantize_kernel(const void* __restrict__ W, int64_t rows, int in, int nb, const float* __restrict__ codebook,
                uint8_t* __restrict__ packed, uint16_t* __restrict__ norms) {
  extern __shared__ __align__(16) uint8_t smem[];
  const QuantShared s = quant_shared(smem);
  build_quant_tables(s, codebook);
  const float sigma = *s.sigma;
  constexpr int kEsz = kBf16 ? 2 : 4;

  const int lane = threadIdx.x & 31, q = lane & 3;
  const uint32_t lane_base = static_cast<uint32_t>(__cvta_generic_to_shared(s.tab)) + 4u * lane;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kQThreads + threadIdx.x) >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kQThreads / 32);
  const int64_t nblocks = rows * nb;

  for (int64_t first = warp * 8; first < nblocks; first += nwarps * 8) {
    const int64_t F = first + (lane >> 2);
    const bool active = F < nblocks;
    int len = 0;
    const char* wblk = static_cast<const char*>(W);
    if (active) {
      // (row, block) of F; 32-bit division whenever the block count allows it
      int64_t o;
      if (nblocks <= 0xffffffffll) o = static_cast<uint32_t>(F) / static_cast<uint32_t>(nb);
      else o = F / nb;
      const int b = static_cast<int>(F - o * nb);
      len = min(kBlock, in - kBlock * b);
      wblk += (o * static_cast<int64_t>(in) + static_cast<int64_t>(kBlock) * b) * kEsz;
    }
    const int qlen = max(0, min(32, len - 32 * q));

    float v[32];
    load_quarter<kBf16, kVec>(wblk + 32 * q * kEsz, qlen, v);

    float2 s01 = make_float2(0.0f, 0.0f), s23 = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
      const float2 x01 = make_float2(v[e], v[e + 1]), x23 = make_float2(v[e + 2], v[e + 3]);
      s01 = fma2(x01, x01, s01);
      s23 = fma2(x23, x23, s23);
    }
    float ssum = quad_sum((s01.x + s01.y) + (s23.x + s23.y));
    float a0;

    bool zero_block = false, norm_exact = false;
    if (!(ssum >= 0x1p-100f && ssum <= 0x1p100f)) {
      // Zero, tiny, huge or non-finite block: rescale by a power of two (codes
      // are scale-invariant) and take the norm on the exact path.
      float mx = 0.0f;
#pragma unroll
      for (int e = 0; e < 32; ++e) mx = fmaxf(mx, fabsf(v[e]));
      const unsigned qmask = 0xfu << (lane & ~3);
      mx = quad_max(mx, qmask);
      if (mx == 0.0f) {
        zero_block = true;
      } else if (isfinite(mx)) {
        int ex;
        frexpf(mx, &ex);
        const float sc = ldexpf(1.0f, -ex);
        a0 = 0.0f;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          v[e] *= sc;
          a0 = fmaf(v[e], v[e], a0);
        }
        ssum = quad_sum_m(a0, qmask);
      }
      norm_exact = !zero_block;
    }
    const float n32 = sqrtf(ssum);
    uint16_t h16 = zero_block ? 0 : __half_as_ushort(__float2half_rn(n32));
    if (!norm_exact && !zero_block) {
      // Norm within ~2e-6 relative of a binary16 rounding midpoint -> exact path.
      const uint16_t lo16 = __half_as_ushort(__float2half_rn(n32 * (1.0f - 2e-6f)));
      const uint16_t hi16 = __half_as_ushort(__float2half_rn(n32 * (1.0f + 2e-6f)));
      norm_exact = lo16 != hi16;
    }
    norm_exact = norm_exact && active && q == 0;
    const float inv = zero_block ? 0.0f : 1.0f / n32;

    uint32_t p[5] = {0u, 0u, 0u, 0u, 0u};
    uint32_t fm = 0u;
    fwht_4lanes(v, lane);  // every lane takes part in the shuffles
    if (zero_block || !active) {
#pragma unroll
      for (int w = 0; w < 5; ++w) p[w] = code15_word(w);
    } else {
      const float2 inv2 = make_float2(inv, inv), sig2 = make_float2(sigma, sigma);
      const float2 k64 = make_float2(64.0f, 64.0f), mag2 = make_float2(kQMagic, kQMagic);
#pragma unroll
      for (int e2 = 0; e2 < 32; e2 += 2) {
        const float2 y2 = fma2(make_float2(v[e2], v[e2 + 1]), inv2, sig2);
        const float2 c2 = make_float2(fminf(fmaxf(y2.x, -3.0f), 3.0f), fminf(fmaxf(y2.y, -3.0f), 3.0f));
        const float2 t2 = fma2(c2, k64, mag2);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int e = e2 + h;
          const float ys = h ? c2.y : c2.x;
          const uint32_t idx = __float_as_uint(h ? t2.y : t2.x) & 511u;
          const uint32_t ent = lds_u32_q(idx * 128u + lane_base);
          const float thr = __uint_as_float(ent);
          const uint32_t code = (ent & 31u) + (ys > thr ? 1u : 0u);
          if (!(fabsf(ys - thr) >= kQGuard)) fm |= 1u << e;
          const int bit = 5 * e, w = bit >> 5, sh = bit & 31;
          p[w] += code << sh;  // fields are disjoint: + lets shift and add be one instruction
          if (sh > 27) p[w + 1] += code >> (32 - sh);
        }
      }
    }

    // Exact path for norms near a binary16 rounding midpoint.
    for (unsigned bal = __ballot_sync(0xffffffffu, norm_exact); bal; bal &= bal - 1) {
      const int src = __ffs(bal) - 1;
      const char* base =
          reinterpret_cast<const char*>(__shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(wblk), src));
      const int slen = __shfl_sync(0xffffffffu, len, src);
      double qq = 0.0;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const double w = load_elem64<kBf16>(base, lane + 32 * t, slen);
        qq = fma(w, w, qq);
      }
      qq = warp_sum64(qq);
      if (lane == src) h16 = __half_as_ushort(__double2half(sqrt(qq)));
    }

    // Exact path for codes within the guard band of a threshold.
    for (;;) {
      const unsigned bal = __ballot_sync(0xffffffffu, fm != 0u);
      if (!bal) break;
      const int src = __ffs(bal) - 1;
      const int el = __shfl_sync(0xffffffffu, __ffs(fm) - 1, src);
      const int j = 32 * (src & 3) + el;
      const char* base =
          reinterpret_cast<const char*>(__shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(wblk), src));
      const int slen = __shfl_sync(0xffffffffu, len, src);
      double sy = 0.0, qq = 0.0;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int i = lane + 32 * t;
        const double w = load_elem64<kBf16>(base, i, slen);
        qq = fma(w, w, qq);
        sy += (__popc(i & j) & 1) ? -w : w;
      }
      sy = warp_sum64(sy);
      qq = warp_sum64(qq);
      const double y = qq > 0.0 ? sy / sqrt(qq) : 0.0;
      uint32_t code = 0;
#pragma unroll
      for (int k = 0; k < kLevels - 1; ++k) code += (y > s.mid[k]) ? 1u : 0u;
      if (lane == src) {
        patch_code(p, el, code);
        fm &= fm - 1u;
      }
    }

    if (active) {
      uint32_t* dst = reinterpret_cast<uint32_t*>(packed + F * kBlockBytes + 20 * q);
#pragma unroll
      for (int w = 0; w < 5; ++w) dst[w] = p[w];
      if (q == 0) norms[F] = h16;
    }
  }
}

// ---------------------------------------------------------------- dequantize
constexpr int kDequantThreads = 256;

template <bool kOutBf16, bool kVec>
__global__ void __launch_bounds__(kDequantThreads)
dequantize_kernel(const uint8_t* __restrict__ packed, const uint16_t* __restrict__ norms,
                  const float* __restrict__ codebook, int64_t rows, int in, int nb, void* __restrict__ out) {
  __shared__ float cb[kLevels];
  if (threadIdx.x < kLevels) cb[threadIdx.x] = __ldg(codebook + threadIdx.x);
  __syncthreads();
  const int lane = threadIdx.x & 31, q = lane & 3;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kDequantThreads + threadIdx.x) >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kDequantThreads / 32);
  const int64_t nblocks = rows * nb;
  for (int64_t first = warp * 8; first < nblocks; first += nwarps * 8) {
    const int64_t F = first + (lane >> 2);
    const bool active = F < nblocks;
    int64_t o = 0;
    int b = 0, len = 0;
    uint32_t w[5] = {0u, 0u, 0u, 0u, 0u};
    float scale = 0.0f;
    if (active) {
      if (nblocks <= 0xffffffffll) o = static_cast<uint32_t>(F) / static_cast<uint32_t>(nb);
      else o = F / nb;
      b = static_cast<int>(F - o * nb);
      len = min(kBlock, in - kBlock * b);
      const uint32_t* src = reinterpret_cast<const uint32_t*>(packed + F * kBlockBytes + 20 * q);
#pragma unroll
      for (int k = 0; k < 5; ++k) w[k] = __ldg(src + k);
      scale = half_bits_to_float(__ldg(norms + F)) * (1.0f / 128.0f);
    }
    float v[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int bit = 5 * e, k = bit >> 5, sh = bit & 31;
      const uint32_t code = (sh <= 27) ? ((w[k] >> sh) & 31u) : (__funnelshift_r(w[k], w[k + 1], sh) & 31u);
      v[e] = cb[code];
    }
    fwht_4lanes(v, lane);
    const int qlen = max(0, min(32, len - 32 * q));
    if (!active || qlen == 0) continue;
    const int64_t off = o * static_cast<int64_t>(in) + static_cast<int64_t>(kBlock) * b + 32 * q;
    if constexpr (!kOutBf16) {
      float* dst = static_cast<float*>(out) + off;
      if constexpr (kVec) {
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (4 * c < qlen)
            reinterpret_cast<float4*>(dst)[c] =
                make_float4(v[4 * c] * scale, v[4 * c + 1] * scale, v[4 * c + 2] * scale, v[4 * c + 3] * scale);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (e < qlen) dst[e] = v[e] * scale;
      }
    } else {
      uint16_t* dst = static_cast<uint16_t*>(out) + off;
      if constexpr (kVec) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (8 * c < qlen) {
            uint4 u;
            u.x = float_to_bf16_bits(v[8 * c] * scale) | (float_to_bf16_bits(v[8 * c + 1] * scale) << 16);
            u.y = float_to_bf16_bits(v[8 * c + 2] * scale) | (float_to_bf16_bits(v[8 * c + 3] * scale) << 16);
            u.z = float_to_bf16_bits(v[8 * c + 4] * scale) | (float_to_bf16_bits(v[8 * c + 5] * scale) << 16);
            u.w = float_to_bf16_bits(v[8 * c + 6] * scale) | (float_to_bf16_bits(v[8 * c + 7] * scale) << 16);
            reinterpret_cast<uint4*>(dst)[c] = u;
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (e < qlen) dst[e] = static_cast<uint16_t>(float_to_bf16_bits(v[e] * scale));
      }
    }
  }
}

template <typename K>
bool quant_attr(K kernel) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmemBytes) == cudaSuccess;
}

}  // namespace

int launch_quantize(const void* W, bool bf16, int64_t rows, int in, const float* codebook, uint8_t* packed,
                    uint16_t* norms, cudaStream_t stream) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  const int64_t nblocks = rows * nb;
  const int64_t warps_needed = ceil_div(nblocks, 8);
  const int64_t max_ctas = static_cast<int64_t>(sm_count()) * kQCtasPerSm;  // persistent: one wave
  const int grid = static_cast<int>(std::min<int64_t>(max_ctas, ceil_div(warps_needed, kQThreads / 32)));
  const bool vec = (reinterpret_cast<uintptr_t>(W) % 16 == 0) &&
                   ((static_cast<int64_t>(in) * (bf16 ? 2 : 4)) % 16 == 0);
  static PerDeviceOnce attrs;
  if (const int st = attrs([&] {
        return quant_attr(quantize_kernel<true, true>) &&
               quant_attr(quantize_kernel<true, false>) &&
               quant_attr(quantize_kernel<false, true>) &&
               quant_attr(quantize_kernel<false, false>);
      }))
    return st;
  if (bf16) {
    if (vec) quantize_kernel<true, true><<<grid, kQThreads, kQSmemBytes, stream>>>(W, rows, in, nb, codebook, packed, norms);
    else quantize_kernel<true, false><<<grid, kQThreads, kQSmemBytes, stream>>>(W, rows, in, nb, codebook, packed, norms);
  } else {
    if (vec) quantize_kernel<false, true><<<grid, kQThreads, kQSmemBytes, stream>>>(W, rows, in, nb, codebook, packed, norms);
    else quantize_kernel<false, false><<<grid, kQThreads, kQSmemBytes, stream>>>(W, rows, in, nb, codebook, packed, norms);
  }
  return cudaGetLastError() == cudaSuccess ? HLWQ_OK : HLWQ_ECUDA;
}

int launch_dequantize(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t rows, int in,
                      void* out, bool bf16, cudaStream_t stream) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  const int64_t nblocks = rows * nb;
  const int64_t max_ctas = static_cast<int64_t>(sm_count()) * 8;
  const int grid = static_cast<int>(std::min<int64_t>(max_ctas, ceil_div(nblocks, kDequantThreads / 4)));
  const bool vec = (reinterpret_cast<uintptr_t>(out) % 16 == 0) &&
                   ((static_cast<int64_t>(in) * (bf16 ? 2 : 4)) % 16 == 0);
  if (bf16) {
    if (vec) dequantize_kernel<true, true><<<grid, kDequantThreads, 0, stream>>>(packed, norms, codebook, rows, in, nb, out);
    else dequantize_kernel<true, false><<<grid, kDequantThreads, 0, stream>>>(packed, norms, codebook, rows, in, nb, out);
  } else {
    if (vec) dequantize_kernel<false, true><<<grid, kDequantThreads, 0, stream>>>(packed, norms, codebook, rows, in, nb, out);
    else dequantize_kernel<false, false><<<grid, kDequantThreads, 0, stream>>>(packed, norms, codebook, rows, in, nb, out);
  }
  return cudaGetLastError() == cudaSuccess ? HLWQ_OK : HLWQ_ECUDA;
}

}  // namespace hlwq
