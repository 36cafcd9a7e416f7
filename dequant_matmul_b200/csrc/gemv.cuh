#pragma once
// Fused dequant-GEMV / small-M GEMM on CUDA cores (sm_100a).
//
// y[m][o] = sum_i X[m][i] * w_hat[o][i] with w_hat the HLWQ Q5 weights
// ("Qwen3.6-35B-A3B -- HLWQ Q5", Method), evaluated in the rotated domain by
// the decode engine (engine.cuh): the CTA rotates its tokens' activations once
// (FWHT per 128-block, binary16 in shared memory), then every pair of weights
// costs one table lookup and two fp32-accumulating FMAs per token.
//
// One persistent CTA of 512 threads per SM (the 128 KiB lane-replicated pair
// table fills most of the SM's shared memory); the O rows are split into equal
// contiguous ranges of whole row groups, one per CTA, so every SM streams the
// same number of code bytes.  Tokens are processed MT (1, 2 or 4) at a time;
// the chunk partial sums are added in a fixed order, so results are
// deterministic.

#include <algorithm>
#include <mutex>
#include <utility>

#include "engine.cuh"
#include "sm100.cuh"

namespace hlwq {

namespace {

template <int C, int MT>
__global__ void __launch_bounds__(kEngineThreads, 1)
dense_kernel(const uint8_t* __restrict__ packed, const uint16_t* __restrict__ norms,
             const float* __restrict__ codebook, int64_t O, int in, int nb,
             const uint16_t* __restrict__ X, int64_t ldx, int M, void* __restrict__ Y, int64_t ldy,
             int out_bf16, int max_rows) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int G = 32 / C;
  const int nch = (nb + C - 1) / C;
  const EngineLayout L = engine_layout(MT, nb, max_rows, nch);
  uint32_t* tab = reinterpret_cast<uint32_t*>(smem);
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + L.xs_off);
  float* xinv = reinterpret_cast<float*>(smem + L.xinv_off);
  float* slots = reinterpret_cast<float*>(smem + L.slot_off);
  float* misc = reinterpret_cast<float*>(smem + L.misc_off);
  uint16_t* c16 = reinterpret_cast<uint16_t*>(misc + 64);

  const int64_t ngroups = (O + G - 1) / G;
  const int64_t g0 = static_cast<int64_t>(blockIdx.x) * ngroups / gridDim.x;
  const int64_t g1 = static_cast<int64_t>(blockIdx.x + 1) * ngroups / gridDim.x;
  const int64_t row0 = g0 * G;
  const int nvrows = static_cast<int>(std::min<int64_t>(g1 * G, O) - row0);
  auto rowfn = [=](int v) { return row0 + v; };

  for (int m0 = 0; m0 < M; m0 += MT) {
    const int ntok = std::min(MT, M - m0);
    auto eng = make_engine<C, MT>(packed, norms, nb, nvrows, rowfn);
    eng.prefetch();  // code loads in flight while the tables and activations are prepared
    if (m0 == 0) build_pair_table(tab, c16, codebook);
    rotate_tokens_bf16(X + m0 * ldx, ldx, in, nb, ntok, MT, xs, xinv);
    __syncthreads();
    eng.run(tab, xs, xinv, slots);
    __syncthreads();
    for (int idx = threadIdx.x; idx < ntok * nvrows; idx += blockDim.x) {
      const int m = idx / nvrows, v = idx - m * nvrows;
      const float* sl = slots + (m * nvrows + v) * nch;
      float sum = 0.0f;
      for (int ch = 0; ch < nch; ++ch) sum += sl[ch];
      const int64_t off = (m0 + m) * ldy + row0 + v;
      if (out_bf16) static_cast<uint16_t*>(Y)[off] = static_cast<uint16_t>(float_to_bf16_bits(sum));
      else static_cast<float*>(Y)[off] = sum;
    }
    __syncthreads();
  }
}


// Single-token GEMV.  One CTA of 512 threads per SM (the 128 KiB lane-
// replicated pair table).  An item is 2G rows (G = 16 / C) x one chunk of C
// blocks (always 32 blocks, 2560 bytes of codes); lane (r, s, h) = (lane / 2C,
// (lane % 2C) / 2, lane % 2) takes rows r and r + G, block s of the chunk and
// half h of that block (2 x 64 codes), so the two rows share the lane's 64
// rotated activations (32 half2 registers) and the per-item costs (wait,
// refill, reduction) are paid once per 64 code pairs.  A CTA owns a contiguous
// range of rows; its items are ordered chunk-major and split into 16
// contiguous warp ranges, so a lane reloads its activations only when its
// range crosses into the next chunk.
//
// Codes are streamed by TMA: every warp owns a ring of S item slots in shared
// memory (one 3-D box {80 bytes, C blocks, 2G rows} per item, one mbarrier per
// slot) and keeps S items in flight; lane 0 refills a slot as soon as the warp
// has read it.  Norms travel in a register ring beside it.
//
// Per pair of codes: one shift that puts the 10-bit pair index at bit 7, one
// and-or that forms the byte offset of (entry, lane) in the table, one shared
// load and two mixed-precision FMAs that add the binary16 products to fp32
// accumulators.  A lane's row sums are scaled by n16 / 128 and the block's
// activation scale and summed over the row's 2C lanes (the two rows of a lane
// are reduced together: log2(2C) shuffles); the row sums over chunks are
// formed at the end in a fixed order (deterministic).
//
// Launched with programmatic stream serialisation (HLWQ_FLAG_WEIGHTS_STATIC),
// the first code boxes and their norms (issued first) and the codebook load
// do not wait for the previous kernel on the stream (griddepcontrol.wait); x
// is read and y written only after that wait.
constexpr int kG1Threads = 512;
constexpr int kG1Warps = kG1Threads / 32;
constexpr int kG1ItemBytes = 32 * kBlockBytes;  // 2G rows x C blocks = 32 blocks for every C
// Rotated activation: 256 bytes per block, its sixteen 16-byte chunks stored
// at chunk (j ^ (b & 7)) so that the lanes of a row (blocks b, b + 1, ...)
// reload their halves from different banks.
constexpr int kG1XsBytes = 256;
__host__ __device__ inline int g1_xs_chunk(int b, int j) { return b * 16 + (j ^ (b & 7)); }

struct G1Layout {
  int ring_off, xs_off, xinv_off, part_off, c16_off, bar_off, total;
};

__host__ __device__ inline int round16(int v) { return (v + 15) & ~15; }

__host__ __device__ inline G1Layout g1_layout(int nb, int pass_rows, int nch, int S) {
  G1Layout L;
  L.ring_off = kPairTabBytes;  // the table sits at offset 0
  L.xs_off = L.ring_off + kG1Warps * S * kG1ItemBytes;
  L.xinv_off = L.xs_off + nb * kG1XsBytes;
  L.part_off = L.xinv_off + round16(nb * 4);
  L.c16_off = L.part_off + round16(pass_rows * nch * 4);
  L.bar_off = L.c16_off + 64;
  L.total = L.bar_off + kG1Warps * S * 8;
  return L;
}

// Byte offset of pair P's table entry for this lane: the 10-bit field at bit
// 10 P of the half block's 10 words, moved to bit 7, or-ed with lane * 4.
template <int P>
__device__ __forceinline__ uint32_t g1_off(const uint2 (&cw)[5], uint32_t lane4) {
  constexpr int bit = 10 * P, wi = bit >> 5, sh = bit & 31;
  const uint32_t lo = word10(cw, wi);
  uint32_t t;
  if constexpr (sh > 22) {
    t = __funnelshift_r(lo, word10(cw, wi + 1), sh - 7);
  } else if constexpr (sh >= 7) {
    t = lo >> (sh - 7);
  } else {
    t = lo << (7 - sh);
  }
  return (t & 0x1ff80u) | lane4;
}

// Pair P: one table lookup gives the binary16 centroids (c[k_2P], c[k_2P+1]),
// each multiplied by its binary16 rotated activation and added to an fp32
// accumulator (exact products, one fp32 rounding per term).  Four
// accumulators (pair parity x half) keep the dependent chains short.
template <int P>
__device__ __forceinline__ void g1_pair(const uint8_t* tab, const uint2 (&cw)[5], uint32_t lane4,
                                        const uint32_t (&xr)[32], float (&acc)[4]) {
  const uint32_t e = *reinterpret_cast<const uint32_t*>(tab + g1_off<P>(cw, lane4));
  acc[2 * (P & 1)] = fma_lo(e, xr[P], acc[2 * (P & 1)]);
  acc[2 * (P & 1) + 1] = fma_hi(e, xr[P], acc[2 * (P & 1) + 1]);
}

template <int... P>
__device__ __forceinline__ float g1_dot(const uint8_t* tab, const uint2 (&cw)[5], uint32_t lane4,
                                        const uint32_t (&xr)[32], std::integer_sequence<int, P...>) {
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  (g1_pair<P>(tab, cw, lane4, xr, acc), ...);
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// Lane l's centroid c = c[l] as binary16 (a warp with `check` set, warp 0 in
// g1_codebook_lane, also checks that the codebook is strictly ascending and
// raises HLWQ_DEVERR_CODEBOOK otherwise).
__device__ __forceinline__ uint32_t g1_codebook_half(float c, bool check) {
  const int lane = threadIdx.x & 31;
  if (check) {
    const float next = __shfl_down_sync(0xffffffffu, c, 1);
    if (lane + 1 < kLevels && !(c < next)) raise_device_error(HLWQ_DEVERR_CODEBOOK);
  }
  return static_cast<uint32_t>(__half_as_ushort(__float2half_rn(c)));
}

__device__ __forceinline__ uint32_t g1_codebook_lane(const float* __restrict__ codebook) {
  return g1_codebook_half(__ldg(codebook + (threadIdx.x & 31)), threadIdx.x < 32);
}

// The binary16 centroids the pair table is expected to hold, passed by value
// as a kernel parameter (two per word, c[2i] in the low half), so that the
// table can be built at once instead of after the codebook's memory latency.
// The host fills it with the Lloyd-Max N(0,1) codebook; every CTA still loads
// the caller's codebook and rebuilds the table from it when any centroid
// differs, so the result never depends on this guess.
struct G1Centroids {
  uint32_t c16[kLevels / 2];
};

__device__ __forceinline__ uint32_t g1_expected_half(const G1Centroids& e) {
  const int lane = threadIdx.x & 31;
  return (e.c16[lane >> 1] >> (16 * (lane & 1))) & 0xffffu;
}

// Warps [w0, w0 + nw) write the lane-replicated pair table, word (v * 32 +
// lane) = half2(c[v & 31], c[v >> 5]), from the centroids in their lanes (no
// shared copy of the codebook, so no CTA barrier before the table is built).
// One 16-byte store per lane covers four entries (lane l: entry 4m + l / 8,
// words 4 (l & 7) .. + 3), so the low halves c[4 (m & 7) + l / 8] repeat with
// period 8 in m and are shuffled once when the warp count is a multiple of 8.
__device__ __forceinline__ void g1_build_table(uint8_t* smem, uint32_t c16r, int w0, int nw) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp < w0 || warp >= w0 + nw) return;
  uint4* t4 = reinterpret_cast<uint4*>(smem);
  const int k = warp - w0;
  uint32_t lo = __shfl_sync(0xffffffffu, c16r, 4 * (k & 7) + (lane >> 3));
  for (int m = k; m < 256; m += nw) {
    if (nw & 7) lo = __shfl_sync(0xffffffffu, c16r, 4 * (m & 7) + (lane >> 3));
    const uint32_t e = lo | (__shfl_sync(0xffffffffu, c16r, m >> 3) << 16);
    t4[m * 32 + lane] = make_uint4(e, e, e, e);
  }
}

// Rotation of activation vectors with eight lanes per 128-block (16
// consecutive values per lane: four butterfly stages in registers, three
// across lanes).  Blocks are numbered gb = vector * nb + block over nvec
// vectors of `in` values (row pitch ld); a warp covers blocks gb0 .. gb0 + 3.
// Block gb is scaled by 2^k so that max |x_tilde| * 2^k lies in [2^9, 2^10)
// and stored as binary16 at chunks g1_xs_chunk(gb, .); xinv[gb] = 2^-k.  The
// load is a separate step so that its latency can overlap other set-up work.
struct RotBlock {
  int gb, vec, b, i0;
  bool act;
};

__device__ __forceinline__ RotBlock g1_rot_block(int nb, int nblocks, int gb0) {
  const int lane = threadIdx.x & 31;
  RotBlock B;
  B.gb = gb0 + (lane >> 3);
  B.act = B.gb < nblocks;
  B.vec = B.act ? B.gb / nb : 0;
  B.b = B.gb - B.vec * nb;
  B.i0 = kBlock * B.b + 16 * (lane & 7);
  return B;
}

// bf16 source: the 16 values as 8 words (kept packed while other work runs).
__device__ __forceinline__ void g1_rot_load(const uint16_t* __restrict__ x, int64_t ld, int in, int nb, int nblocks,
                                            bool xvec, int gb0, uint32_t (&w)[8]) {
  const RotBlock B = g1_rot_block(nb, nblocks, gb0);
  const uint16_t* row = x + B.vec * ld;
  if (xvec) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      uint4 t = make_uint4(0, 0, 0, 0);
      if (B.act && B.i0 + 8 * j < in) t = __ldg(reinterpret_cast<const uint4*>(row + B.i0 + 8 * j));
      w[4 * j] = t.x; w[4 * j + 1] = t.y; w[4 * j + 2] = t.z; w[4 * j + 3] = t.w;
    }
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t lo = (B.act && B.i0 + 2 * e < in) ? __ldg(row + B.i0 + 2 * e) : 0u;
      const uint32_t hi = (B.act && B.i0 + 2 * e + 1 < in) ? __ldg(row + B.i0 + 2 * e + 1) : 0u;
      w[e] = lo | (hi << 16);
    }
  }
}

// Butterflies of one block held 16 values per lane by 8 lanes; returns the
// power-of-two exponent k with max |x_tilde| * 2^k in [2^9, 2^10).
__device__ __forceinline__ int g1_rot_compute(float (&v)[16]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int e = 0; e < 16; ++e)
      if ((e & h) == 0) {
        const float a = v[e], c = v[e + h];
        v[e] = a + c;
        v[e + h] = a - c;
      }
  }
#pragma unroll
  for (int lm = 1; lm < 8; lm <<= 1) {
    const float sgn = (lane & lm) ? -1.0f : 1.0f;
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = fmaf(v[e], sgn, __shfl_xor_sync(0xffffffffu, v[e], lm));
  }
  float mx = 0.0f;
#pragma unroll
  for (int e = 0; e < 16; ++e) mx = fmaxf(mx, fabsf(v[e]));
#pragma unroll
  for (int lm = 1; lm < 8; lm <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, lm));
  int ex = 0;
  if (mx > 0.0f && isfinite(mx)) frexpf(mx, &ex);
  return max(-120, min(120, 10 - ex));
}

__device__ __forceinline__ void g1_rot_core(float (&v)[16], int nb, int nblocks, int gb0, uint16_t* xs,
                                            float* xinv) {
  const int q = threadIdx.x & 7;
  const RotBlock B = g1_rot_block(nb, nblocks, gb0);
  const int k = g1_rot_compute(v);
  const float sc = ldexpf(1.0f, k);
  if (B.act) {
    uint4* dst = reinterpret_cast<uint4*>(xs);
#pragma unroll
    for (int c = 0; c < 2; ++c)
      dst[g1_xs_chunk(B.gb, 2 * q + c)] =
          make_uint4(pack_half2(v[8 * c] * sc, v[8 * c + 1] * sc), pack_half2(v[8 * c + 2] * sc, v[8 * c + 3] * sc),
                     pack_half2(v[8 * c + 4] * sc, v[8 * c + 5] * sc), pack_half2(v[8 * c + 6] * sc, v[8 * c + 7] * sc));
    if (q == 0) xinv[B.gb] = ldexpf(1.0f, -k);
  }
}

__device__ __forceinline__ void g1_rot_store(const uint32_t (&w)[8], int nb, int nblocks, int gb0, uint16_t* xs,
                                             float* xinv) {
  float v[16];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    v[2 * k] = __uint_as_float(w[k] << 16);
    v[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
  }
  g1_rot_core(v, nb, nblocks, gb0, xs, xinv);
}

// fp32 source (the MoE intermediate h), loaded and rotated in one step.
__device__ __forceinline__ void g1_rot_f32(const float* __restrict__ x, int64_t ld, int in, int nb, int nblocks,
                                           int gb0, uint16_t* xs, float* xinv) {
  const RotBlock B = g1_rot_block(nb, nblocks, gb0);
  const float* row = x + B.vec * ld;
  float v[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) v[e] = (B.act && B.i0 + e < in) ? row[B.i0 + e] : 0.0f;
  g1_rot_core(v, nb, nblocks, gb0, xs, xinv);
}

template <int C, int S>
__global__ void __launch_bounds__(kG1Threads, 1)
gemv1_kernel(const __grid_constant__ CUtensorMap cmap, const uint16_t* __restrict__ norms,
             const float* __restrict__ codebook, const __grid_constant__ G1Centroids expect, int64_t O, int in,
             int nb, const uint16_t* __restrict__ x, void* __restrict__ Y, int out_bf16, int pass_rows, int xvec) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int L2C = 2 * C;   // lanes per row
  constexpr int G = 32 / L2C;  // rows of one half item
  constexpr int RG = 2 * G;    // rows per item
  const int nch = (nb + C - 1) / C;
  const G1Layout L = g1_layout(nb, pass_rows, nch, S);
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + L.xs_off);
  float* xinv = reinterpret_cast<float*>(smem + L.xinv_off);
  float* part = reinterpret_cast<float*>(smem + L.part_off);
  const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(smem));

  const int64_t ngroups = (O + RG - 1) / RG;
  const int64_t g0 = static_cast<int64_t>(blockIdx.x) * ngroups / gridDim.x;
  const int64_t g1 = static_cast<int64_t>(blockIdx.x + 1) * ngroups / gridDim.x;
  const int64_t row0 = g0 * RG;
  const int nrows = static_cast<int>(std::min<int64_t>(g1 * RG, O) - row0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = lane / L2C, u = lane % L2C, s = u >> 1, hh = u & 1;
  const uint32_t lane4 = static_cast<uint32_t>(lane) << 2;

  // this warp's ring: S slots of one item each, one mbarrier per slot
  const uint32_t ring = sbase + L.ring_off + warp * (S * kG1ItemBytes);
  const uint32_t bar = sbase + L.bar_off + warp * (S * 8);
  const uint8_t* my_codes = smem + L.ring_off + warp * (S * kG1ItemBytes) + 40 * lane;  // slot layout [2G][C][80]
  if (lane == 0) {
#pragma unroll
    for (int d = 0; d < S; ++d) mbar_init(bar + 8 * d, 1);
    fence_barrier_init();
  }
  __syncwarp();
  const uint64_t deadline = globaltimer_ns() + wait_limit_ns();
  bool ok = true;
  uint32_t phase = 0;    // parity of the next completion, one bit per slot
  uint32_t pending = 0;  // slots with a box in flight

  for (int p0 = 0; p0 < nrows; p0 += pass_rows) {
    const int prow = min(pass_rows, nrows - p0);
    const int ngr = (prow + RG - 1) / RG;
    const int nitems = ngr * nch;
    const int it0 = warp * nitems / kG1Warps, it1 = (warp + 1) * nitems / kG1Warps;
    const int nw = it1 - it0;
    const int64_t prow0 = row0 + p0;

    // issue cursor: item (ich, ig) goes to the slot being refilled; nptr
    // points at the norm of (row ig * RG + r, block ich * C + s)
    int ich = it0 / ngr, ig = it0 - (it0 / ngr) * ngr;
    const uint16_t* nptr = norms + (prow0 + ig * RG + r) * nb + ich * C + s;
    uint32_t nlo[S], nhi[S];  // the two rows' norms, kept apart so that no instruction waits on them before use
    auto issue = [&](int d) {
      if (lane == 0 && !fault_skip_tma()) {
        mbar_arrive_expect_tx(bar + 8 * d, kG1ItemBytes);
        tma_load_3d(ring + d * kG1ItemBytes, &cmap, 0, ich * C, static_cast<int>(prow0 + ig * RG), bar + 8 * d);
      }
      const int v = ig * RG + r;
      const bool bok = ich * C + s < nb;
      uint32_t n0 = 0u;
      if (bok && v < prow) n0 = __ldg(nptr);
      uint32_t n1 = 0u;
      if (bok && v + G < prow) n1 = __ldg(nptr + G * nb);
      nlo[d] = n0;
      nhi[d] = n1;
      pending |= 1u << d;
      if (++ig == ngr) {
        ig = 0;
        ++ich;
        nptr = norms + (prow0 + r) * nb + ich * C + s;
      } else {
        nptr += RG * nb;
      }
    };
#pragma unroll
    for (int d = 0; d < S; ++d)
      if (d < nw) issue(d);

    if (p0 == 0) {
      // set-up while the first boxes are in flight.  x may be produced by the
      // previous kernel on the stream: every thread passes the dependency
      // wait before it touches x or y.  The x loads are then in flight while
      // the pair table is built from the expected centroids (a kernel
      // parameter, no memory latency); the caller's codebook, loaded first,
      // is compared with them at the barrier that publishes table and x, and
      // a codebook that differs rebuilds the table before any lookup.
      const float cl = __ldg(codebook + lane);
      const uint32_t c16x = g1_expected_half(expect);
      pdl_wait();
      uint32_t xw[8];
      const int rb0 = 4 * warp;
      if (rb0 < nb) g1_rot_load(x, in, in, nb, nb, xvec != 0, rb0, xw);
      g1_build_table(smem, c16x, 0, kG1Warps);
      if (rb0 < nb) g1_rot_store(xw, nb, nb, rb0, xs, xinv);
      for (int b0 = rb0 + 4 * kG1Warps; b0 < nb; b0 += 4 * kG1Warps) {
        g1_rot_load(x, in, in, nb, nb, xvec != 0, b0, xw);
        g1_rot_store(xw, nb, nb, b0, xs, xinv);
      }
      const uint32_t c16 = g1_codebook_half(cl, warp == 0);
      if (__syncthreads_or(c16 != c16x)) {
        g1_build_table(smem, c16, 0, kG1Warps);
        __syncthreads();
      }
      pdl_trigger();
    }

    int cch = it0 / ngr, cg = it0 - (it0 / ngr) * ngr, xch = -1;
    uint32_t xr[32];
    float xi = 0.0f;
    for (int base = 0; base < nw; base += S) {
#pragma unroll
      for (int d = 0; d < S; ++d) {
        const int k = base + d;
        if (k < nw) {
          const uint32_t nr0 = nlo[d], nr1 = nhi[d];
          if (ok && ((pending >> d) & 1u)) {
            ok = __all_sync(0xffffffffu, mbar_wait(bar + 8 * d, (phase >> d) & 1u, deadline));
            if (ok) {
              phase ^= 1u << d;
              pending &= ~(1u << d);
            }
          }
          uint2 cw0[5], cw1[5];
          const uint2* src = reinterpret_cast<const uint2*>(my_codes + d * kG1ItemBytes);
#pragma unroll
          for (int q = 0; q < 5; ++q) {
            cw0[q] = src[q];
            cw1[q] = src[q + kG1ItemBytes / 16];  // row r + G: half a slot further
          }
          __syncwarp();
          if (ok && k + S < nw) {
            if (lane == 0) fence_proxy_async();  // the slot's reads precede the refill
            issue(d);
          }
          if (cch != xch) {
            xch = cch;
            const int b = cch * C + s;
            if (b < nb) {
              const uint4* xsrc = reinterpret_cast<const uint4*>(xs);
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const uint4 w = xsrc[g1_xs_chunk(b, 8 * hh + q)];
                xr[4 * q] = w.x; xr[4 * q + 1] = w.y; xr[4 * q + 2] = w.z; xr[4 * q + 3] = w.w;
              }
              xi = xinv[b] * (1.0f / 128.0f);
            } else {
#pragma unroll
              for (int q = 0; q < 32; ++q) xr[q] = 0u;
              xi = 0.0f;
            }
          }
          const float a0 = g1_dot(smem, cw0, lane4, xr, std::make_integer_sequence<int, 32>{}) *
                           (half_bits_to_float(static_cast<uint16_t>(nr0)) * xi);
          const float a1 = g1_dot(smem, cw1, lane4, xr, std::make_integer_sequence<int, 32>{}) *
                           (half_bits_to_float(static_cast<uint16_t>(nr1)) * xi);
          // reduce both rows over the 2C lanes: the first exchange leaves row
          // r's partial on lanes with bit C clear and row r + G's on the others
          const bool hi = (u & C) != 0;
          float acc = (hi ? a1 : a0) + __shfl_xor_sync(0xffffffffu, hi ? a0 : a1, C);
#pragma unroll
          for (int off = C / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
          const int v = cg * RG + r + (hi ? G : 0);
          if ((u & (C - 1)) == 0 && v < prow) part[v * nch + cch] = acc;
          if (++cg == ngr) { cg = 0; ++cch; }
        }
      }
    }
    if (!ok) {
      // a box never arrived: drain what is still in flight (bounded), then stop
      const uint64_t dl = globaltimer_ns() + wait_limit_ns();
      for (int d = 0; d < S; ++d)
        if ((pending >> d) & 1u) mbar_wait(bar + 8 * d, (phase >> d) & 1u, dl);
      if (lane == 0) raise_device_error(HLWQ_DEVERR_TIMEOUT);
    }
    __syncthreads();
    for (int v = threadIdx.x; v < prow; v += kG1Threads) {
      const float* pr = part + v * nch;
      float sum = 0.0f;
      for (int ch = 0; ch < nch; ++ch) sum += pr[ch];
      const int64_t o = prow0 + v;
      if (out_bf16) static_cast<uint16_t*>(Y)[o] = static_cast<uint16_t>(float_to_bf16_bits(sum));
      else static_cast<float*>(Y)[o] = sum;
    }
    __syncthreads();
    if (__syncthreads_or(!ok)) break;
  }
}

// Tensor map of the codes viewed as a 3-D byte tensor {80, NB, O}.  Encoding
// costs host time, so the last few maps are kept (a map depends only on the
// pointer, the shape and the box).
struct CodesMapEntry {
  const void* ptr;
  int64_t O;
  int nb, C, rows;
  CUtensorMap map;
};

// box = {80 bytes, C blocks, box_rows rows}
inline int codes_map(const uint8_t* packed, int64_t O, int nb, int C, int box_rows, CUtensorMap* out) {
  static std::mutex mu;
  static CodesMapEntry cache[8];
  static int used = 0, next = 0;
  std::lock_guard<std::mutex> lock(mu);
  for (int k = 0; k < used; ++k) {
    const CodesMapEntry& e = cache[k];
    if (e.ptr == packed && e.O == O && e.nb == nb && e.C == C && e.rows == box_rows) {
      *out = e.map;
      return HLWQ_OK;
    }
  }
  PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode_fn();
  if (!encode) return HLWQ_ECUDA;
  const cuuint64_t dim[3] = {static_cast<cuuint64_t>(kBlockBytes), static_cast<cuuint64_t>(nb),
                             static_cast<cuuint64_t>(O)};
  const cuuint64_t stride[2] = {static_cast<cuuint64_t>(kBlockBytes), static_cast<cuuint64_t>(nb) * kBlockBytes};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(kBlockBytes), static_cast<cuuint32_t>(C),
                             static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUtensorMap m;
  if (encode(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(packed), dim, stride, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return HLWQ_ECUDA;
  CodesMapEntry& e = cache[next];
  e.ptr = packed;
  e.O = O;
  e.nb = nb;
  e.C = C;
  e.rows = box_rows;
  e.map = m;
  next = (next + 1) % 8;
  used = std::min(used + 1, 8);
  *out = m;
  return HLWQ_OK;
}

// Rows of a CTA handled per pass for ring depth S (0 if the layout does not fit).
inline int g1_pass_rows(int nb, int C, int S, int rows_cta) {
  const int RG = 32 / C, nch = (nb + C - 1) / C;
  const int fixed = g1_layout(nb, 0, nch, S).total;
  const int cap = (227 * 1024 - fixed - 16) / (nch * 4) / RG * RG;
  return cap < RG ? 0 : std::min(rows_cta, cap);
}

// Binary16 bits of the Lloyd-Max N(0,1) codebook (hlwq_lloyd_codebook),
// computed once per process.
inline const G1Centroids& g1_lloyd_max_centroids() {
  static const G1Centroids e = [] {
    G1Centroids r{};
    float c[kLevels];
    if (hlwq_lloyd_codebook(kLevels, c, nullptr, nullptr) == HLWQ_OK)
      for (int i = 0; i < kLevels; ++i)
        r.c16[i >> 1] |= static_cast<uint32_t>(__half_as_ushort(__float2half_rn(c[i]))) << (16 * (i & 1));
    return r;
  }();
  return e;
}

template <int C, int S>
int launch_gemv1_cs(const CUtensorMap& map, const uint16_t* norms, const float* codebook, int64_t O, int in,
                    int nb, const uint16_t* x, void* Y, bool out_bf16, unsigned flags, int grid, int pass_rows,
                    cudaStream_t stream) {
  const G1Layout L = g1_layout(nb, pass_rows, (nb + C - 1) / C, S);
  static PerDeviceOnce attr_set;
  if (const int st = attr_set([&] {
        return cudaFuncSetAttribute(gemv1_kernel<C, S>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    227 * 1024) == cudaSuccess;
      }))
    return st;
  const int xvec = (reinterpret_cast<uintptr_t>(x) % 16 == 0 && in % 8 == 0) ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kG1Threads);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (flags & HLWQ_FLAG_WEIGHTS_STATIC) ? 1 : 0;
  const int ob = out_bf16 ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, gemv1_kernel<C, S>, map, norms, codebook, g1_lloyd_max_centroids(), O, in, nb, x, Y,
                         ob, pass_rows, xvec) != cudaSuccess)
    return HLWQ_ECUDA;
  return HLWQ_OK;
}

template <int C>
int launch_gemv1_c(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                   const uint16_t* x, void* Y, bool out_bf16, unsigned flags, cudaStream_t stream) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  constexpr int RG = 32 / C;
  const int64_t ngroups = ceil_div(O, RG);
  const int grid = static_cast<int>(std::min<int64_t>(sm_count(), ngroups));
  const int rows_cta = static_cast<int>(ceil_div(ngroups, grid) * RG);
  CUtensorMap map;
  const int st = codes_map(packed, O, nb, C, RG, &map);
  if (st != HLWQ_OK) return st;
  // deepest ring that fits beside the table and the rotated activation
  if (const int pr = g1_pass_rows(nb, C, 2, rows_cta))
    return launch_gemv1_cs<C, 2>(map, norms, codebook, O, in, nb, x, Y, out_bf16, flags, grid, pr, stream);
  if (const int pr = g1_pass_rows(nb, C, 1, rows_cta))
    return launch_gemv1_cs<C, 1>(map, norms, codebook, O, in, nb, x, Y, out_bf16, flags, grid, pr, stream);
  return HLWQ_EUNSUPPORTED;
}

}  // namespace

int launch_dense_m1(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                    const uint16_t* x, void* Y, bool out_bf16, cudaStream_t stream);

int launch_gemv1(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                 const uint16_t* x, void* Y, bool out_bf16, cudaStream_t stream, unsigned flags) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  int st;
  switch (pick_chunk(nb)) {
    case 8: st = launch_gemv1_c<8>(packed, norms, codebook, O, in, x, Y, out_bf16, flags, stream); break;
    case 4: st = launch_gemv1_c<4>(packed, norms, codebook, O, in, x, Y, out_bf16, flags, stream); break;
    default: st = launch_gemv1_c<2>(packed, norms, codebook, O, in, x, Y, out_bf16, flags, stream); break;
  }
  // rows too long for the code ring beside the table and the activation:
  // the CUDA-core decode kernel (no ring) takes them
  if (st == HLWQ_EUNSUPPORTED) st = launch_dense_m1(packed, norms, codebook, O, in, x, Y, out_bf16, stream);
  return st;
}

namespace {

template <int C, int MT>
int launch_dense_t(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                   const uint16_t* X, int64_t ldx, int M, void* Y, int64_t ldy, bool out_bf16,
                   cudaStream_t stream) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  constexpr int G = 32 / C;
  const int64_t ngroups = ceil_div(O, G);
  const int grid = static_cast<int>(std::min<int64_t>(sm_count(), ngroups));
  const int max_rows = static_cast<int>(ceil_div(ngroups, grid) * G);
  const int nch = (nb + C - 1) / C;
  const EngineLayout L = engine_layout(MT, nb, max_rows, nch);
  if (L.total > 227 * 1024) return HLWQ_EUNSUPPORTED;
  static PerDeviceOnce attr_set;
  if (const int st = attr_set([&] {
        return cudaFuncSetAttribute(dense_kernel<C, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    227 * 1024) == cudaSuccess;
      }))
    return st;
  dense_kernel<C, MT><<<grid, kEngineThreads, L.total, stream>>>(packed, norms, codebook, O, in, nb, X, ldx, M, Y,
                                                                  ldy, out_bf16 ? 1 : 0, max_rows);
  return cudaGetLastError() == cudaSuccess ? HLWQ_OK : HLWQ_ECUDA;
}

template <int C>
int launch_dense_c(int mt, const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                   const uint16_t* X, int64_t ldx, int M, void* Y, int64_t ldy, bool out_bf16,
                   cudaStream_t stream) {
  switch (mt) {
    case 1: return launch_dense_t<C, 1>(packed, norms, codebook, O, in, X, ldx, M, Y, ldy, out_bf16, stream);
    case 2: return launch_dense_t<C, 2>(packed, norms, codebook, O, in, X, ldx, M, Y, ldy, out_bf16, stream);
    default: return launch_dense_t<C, 4>(packed, norms, codebook, O, in, X, ldx, M, Y, ldy, out_bf16, stream);
  }
}

}  // namespace

// Shared-memory bytes the dense kernel needs for a given shape and token tile.
int dense_smem_bytes(int64_t O, int in, int mt) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  const int C = pick_chunk(nb), G = 32 / C;
  const int64_t ngroups = ceil_div(O, G);
  const int grid = static_cast<int>(std::min<int64_t>(sm_count(), ngroups));
  const int max_rows = static_cast<int>(ceil_div(ngroups, grid) * G);
  return engine_layout(mt, nb, max_rows, (nb + C - 1) / C).total;
}

int launch_dense_m1(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                    const uint16_t* x, void* Y, bool out_bf16, cudaStream_t stream) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  if (dense_smem_bytes(O, in, 1) > 227 * 1024) return HLWQ_EUNSUPPORTED;
  switch (pick_chunk(nb)) {
    case 8: return launch_dense_c<8>(1, packed, norms, codebook, O, in, x, in, 1, Y, O, out_bf16, stream);
    case 4: return launch_dense_c<4>(1, packed, norms, codebook, O, in, x, in, 1, Y, O, out_bf16, stream);
    default: return launch_dense_c<2>(1, packed, norms, codebook, O, in, x, in, 1, Y, O, out_bf16, stream);
  }
}

int launch_gemvm(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                 const uint16_t* X, int64_t ldx, int M, void* Y, int64_t ldy, bool out_bf16, cudaStream_t stream);

int launch_dense(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                 const uint16_t* X, int64_t ldx, int M, void* Y, int64_t ldy, bool out_bf16, cudaStream_t stream) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  if (M == 1) return launch_gemv1(packed, norms, codebook, O, in, X, Y, out_bf16, stream, 0u);
  if (M <= 8) {
    // few tokens: the TMA-fed multi-token kernel (falls through when its
    // shared memory does not fit, e.g. very long rows)
    const int st = launch_gemvm(packed, norms, codebook, O, in, X, ldx, M, Y, ldy, out_bf16, stream);
    if (st != HLWQ_EUNSUPPORTED) return st;
  }
  int mt = M >= 3 ? 4 : M;
  while (mt > 1 && dense_smem_bytes(O, in, mt) > 227 * 1024) mt >>= 1;
  switch (pick_chunk(nb)) {
    case 8: return launch_dense_c<8>(mt, packed, norms, codebook, O, in, X, ldx, M, Y, ldy, out_bf16, stream);
    case 4: return launch_dense_c<4>(mt, packed, norms, codebook, O, in, X, ldx, M, Y, ldy, out_bf16, stream);
    default: return launch_dense_c<2>(mt, packed, norms, codebook, O, in, X, ldx, M, Y, ldy, out_bf16, stream);
  }
}

}  // namespace hlwq
