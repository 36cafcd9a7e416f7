#pragma once
// Small-M GEMM on the 5th-generation tensor cores (tcgen05 / TMEM / TMA), sm_100a.
//
// Y[m][o] = sum_i X[m][i] w_hat[o][i] for M >= 5 tokens, evaluated in the
// rotated domain ("Qwen3.6-35B-A3B -- HLWQ Q5", Method step [3]; H symmetric,
// H H = 128 I):
//     Y[m][o] = 2^e_o / (128 s_m) * sum_K A[o][K] B[m][K],
//     A[o][128 b + j] = c[k_obj] * n16[o][b] * 2^-e_o   (binary16),
//     B[m][128 b + j] = x_tilde[m][128 b + j] * s_m     (binary16),
// with x_tilde_b = x_b @ H, e_o a per-row power of two (so that every A entry is
// at most max|c|) and s_m a per-token power of two (max |B| in [2^14, 2^15)).
//
// Kernel 1 (rotate_x_kernel): one CTA per token rotates X once per call into
// the workspace (binary16 B matrix, K-major) and records 1/s_m.
// Kernel 2 (gemm_tc_kernel<F, NG>): one CTA per 128-row tile of W (and up to
// 256-token tile of X); F is the weight format (HLWQ Q5 or TQ3).  The same
// kernel runs the routed MoE layer's grouped GEMMs (TcGroup, launch_moe_tc).
// Roles, D = 8 NG decode warps plus three:
//   warps 0..D-1 decode, in NG groups of 8 taking blocks b = g (mod NG): each
//              lane owns one weight row of the tile and decodes one half block
//              (code -> fp32 centroid from a shared table, times the block
//              scale, rounded to binary16) and writes it straight into tensor
//              memory with tcgen05.st (the A operand lives in TMEM, so
//              decoding costs no shared-memory bandwidth that the MMA needs
//              for B);
//   warp D     initialises the barriers, then TMA producer of the code tiles
//              (128 rows x one block); its first boxes go out before the
//              CTA-wide barrier;
//   warp D + 2 TMA producer of B: two 64 x N boxes per block, 128-byte
//              swizzled (no multicast);
//   warp D + 1 allocates TMEM and issues tcgen05.mma (kind::f16, M = 128,
//              N = tokens, K = 16) into an fp32 accumulator in TMEM;
//   warps 0..D-1 epilogue (split by TMEM lane quarter and columns):
//              tcgen05.ld of the accumulator, scaling, bf16/fp32 store.
// The single MMA-issuing thread paces a CTA: a tcgen05.mma takes about as
// long to issue as a 64-token MMA takes to run, and the decode warps on its
// scheduler slow it further.  Token tiles of at most 128 therefore run with
// one decode group (NG = 1, 352 threads, 256 TMEM columns) and two CTAs per
// SM, so that two threads issue MMAs on every SM; 256-token tiles, whose MMAs
// are long, use two groups (NG = 2) and the whole TMEM of the SM.
// Stages are handed over with mbarriers; every wait is bounded (2 s), after
// which the kernel raises HLWQ_DEVERR_TIMEOUT, drains and frees TMEM.

#include "engine.cuh"
#include "sm100.cuh"

namespace hlwq {

namespace {

// Warp roles of a CTA with NG decode groups of 8 warps.
template <int NG>
struct TcRoles {
  static constexpr int kDecWarps = 8 * NG;
  static constexpr int kWCodes = kDecWarps, kWMma = kDecWarps + 1, kWB = kDecWarps + 2;
  static constexpr int kThreads = 32 * (kDecWarps + 3);
};
constexpr int kTcTileRows = 128;
constexpr int kTcKChunk = 64;  // K elements per B box (one half block)
constexpr int kTcStages = 2;   // A/B stages (A: 64 TMEM columns each, after the accumulator)

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tc_ld8(uint32_t taddr, uint32_t (&v)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "r"(taddr)
               : "memory");
}

__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row atoms of
// 1024 bytes stacked along the non-K dimension (stride byte offset 1024).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3fffu);
  d |= static_cast<uint64_t>(1u) << 16;                 // leading byte offset (unused for swizzled K-major)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;         // stride byte offset
  d |= static_cast<uint64_t>(1u) << 46;                 // descriptor version
  d |= static_cast<uint64_t>(2u) << 61;                 // 128-byte swizzle
  return d;
}

// Instruction descriptor: kind::f16, A and B binary16, K-major, D fp32, M = 128.
__host__ __device__ constexpr uint32_t idesc_f16(int n) {
  return (1u << 4) | (0u << 7) | (0u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(128 >> 4) << 24);
}

// Weight formats the kernel decodes.  HLWQ Q5: 5-bit codes, 80-byte blocks,
// binary16 norms, 32 centroids.  TQ3 (the scalar case of HIGGS,
// "Qwen3.6-35B-A3B-TQ3-native", "What TQ3 actually does"): 3-bit codes,
// 48-byte groups, fp32 shape-gain norms, 8 centroids.  Both are dotted in the
// rotated domain, sum_b scale_b / 128 * sum_j c[k_bj] x_tilde_bj; only the
// rotation of x differs (TQ3: x_tilde = s2 * H128 (s1 * x) per group).
struct TcQ5 {
  static constexpr int kBits = 5, kLevels = 32, kBytes = 80;
  using Norm = uint16_t;
  __device__ static float norm(Norm v) { return half_bits_to_float(v); }
};
struct TcTq3 {
  static constexpr int kBits = 3, kLevels = 8, kBytes = 48;
  using Norm = float;
  __device__ static float norm(Norm v) { return v; }
};

template <int NW>
__device__ __forceinline__ uint32_t code_word(const uint2 (&c)[NW], int i) {
  const uint2 u = c[i >> 1];
  return (i & 1) ? u.y : u.x;
}

// Shared address of the fp32 centroid of the code at bit POS of a half block
// (NW 8-byte words): the field moved to bit 2 with one shift, masked and
// or-ed with the (1024-byte aligned) table address.
// (pos is a compile-time constant after unrolling.)
template <class F, int NW>
__device__ __forceinline__ uint32_t code_addr(const uint2 (&cw)[NW], int pos, uint32_t tab) {
  const int wi = pos >> 5, sh = pos & 31;
  const uint32_t lo = code_word(cw, wi);
  uint32_t t;
  if (sh + F::kBits > 32) {
    t = __funnelshift_r(lo, code_word(cw, wi + 1), sh - 2);
  } else if (sh >= 2) {
    t = lo >> (sh - 2);
  } else {
    t = lo << (2 - sh);
  }
  return (t & (4u * (F::kLevels - 1))) | tab;  // tab is 1024-byte aligned: or == add, one and-or instruction
}

__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 r;
  asm("{ .reg .b64 pa, pb, pd; mov.b64 pa, {%2, %3}; mov.b64 pb, {%4, %5};\n\t"
      "mul.rn.f32x2 pd, pa, pb; mov.b64 {%0, %1}, pd; }"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

// (lo, hi) -> binary16 pair, round to nearest even.
__device__ __forceinline__ uint32_t cvt_half2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// ---------------------------------------------------------------- rotation
constexpr int kRotThreads = 256;

// One CTA per B row m: B[m][:] = binary16(x_tilde[m][:] * s_m), inv_s[m] = 1 / s_m,
// for the activation row rows[m] (rows == nullptr: row m; the MoE layer's
// gather of each assignment's token); CTA 0 also clears the GEMM's K-split
// counters.  x_tilde_b = x_b @ H128, or with signs (TQ3; int8 [2][128],
// negative = -1): s2 * (H128 (s1 * x_b)).
__global__ void __launch_bounds__(kRotThreads)
rotate_x_kernel(const uint16_t* __restrict__ X, int64_t ldx, int in, int nb, const int8_t* __restrict__ signs,
                const int* __restrict__ rows, uint16_t* __restrict__ B, float* __restrict__ inv_s,
                unsigned* __restrict__ part_cnt, int nsplit) {
  extern __shared__ __align__(16) float buf[];  // [nb * 128]
  __shared__ float red[kRotThreads / 32];
  const int m = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (m == 0)  // the K-split counters of the GEMM that follows start at zero
    for (int i = threadIdx.x; i < nsplit; i += kRotThreads) part_cnt[i] = 0u;
  const uint16_t* x = X + static_cast<int64_t>(rows ? __ldg(rows + m) : m) * ldx;
  float s1[4] = {1.0f, 1.0f, 1.0f, 1.0f}, s2[4] = {1.0f, 1.0f, 1.0f, 1.0f};
  if (signs) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      s1[k] = __ldg(signs + 4 * lane + k) < 0 ? -1.0f : 1.0f;
      s2[k] = __ldg(signs + kBlock + 4 * lane + k) < 0 ? -1.0f : 1.0f;
    }
  }
  float mx = 0.0f;
  for (int b = warp; b < nb; b += kRotThreads / 32) {
    float e4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = kBlock * b + 4 * lane + k;
      e4[k] = i < in ? bf16_bits_to_float(__ldg(x + i)) * s1[k] : 0.0f;  // sign flips are exact
    }
    float a = e4[0] + e4[1], bb = e4[0] - e4[1], c = e4[2] + e4[3], d = e4[2] - e4[3];
    e4[0] = a + c; e4[1] = bb + d; e4[2] = a - c; e4[3] = bb - d;
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float p = __shfl_xor_sync(0xffffffffu, e4[k], h);
        e4[k] = (lane & h) ? p - e4[k] : e4[k] + p;
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      buf[kBlock * b + 4 * lane + k] = e4[k] * s2[k];
      mx = fmaxf(mx, fabsf(e4[k]));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  float t = 0.0f;
#pragma unroll
  for (int w = 0; w < kRotThreads / 32; ++w) t = fmaxf(t, red[w]);
  int e = 0;
  if (t > 0.0f && isfinite(t)) frexpf(t, &e);
  const int k = max(-120, min(120, 15 - e));
  const float sc = ldexpf(1.0f, k);
  if (threadIdx.x == 0) inv_s[m] = ldexpf(1.0f, -k);
  uint16_t* dst = B + static_cast<int64_t>(m) * nb * kBlock;
  for (int i = threadIdx.x; i < nb * kBlock; i += kRotThreads) dst[i] = __half_as_ushort(__float2half_rn(buf[i] * sc));
}

// The MoE layer's down-projection operand: one CTA per assignment row a of
// G [NA][2F] (gate columns [0, F), up columns [F, 2F), fp32):
// h = SiLU(g) * u = g / (1 + e^-g) * u, zero past F; then as rotate_x_kernel,
// Bh[a][:] = binary16(h_tilde * s_a) with h_tilde_b = h_b @ H128, and
// inv_s[a] = weight[a] / s_a (the down GEMM's output comes out weighted).
__global__ void __launch_bounds__(kRotThreads)
silu_rotate_kernel(const float* __restrict__ Gm, int F, int nb, const float* __restrict__ weight,
                   uint16_t* __restrict__ Bh, float* __restrict__ inv_s) {
  extern __shared__ __align__(16) float buf[];  // [nb * 128]
  __shared__ float red[kRotThreads / 32];
  const int a = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float* g = Gm + static_cast<int64_t>(a) * 2 * F;
  float mx = 0.0f;
  for (int b = warp; b < nb; b += kRotThreads / 32) {
    float e4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = kBlock * b + 4 * lane + k;
      float h = 0.0f;
      if (i < F) {
        const float gv = g[i], up = g[F + i];
        h = gv / (1.0f + expf(-gv)) * up;
      }
      e4[k] = h;
    }
    float p = e4[0] + e4[1], q = e4[0] - e4[1], r = e4[2] + e4[3], t = e4[2] - e4[3];
    e4[0] = p + r; e4[1] = q + t; e4[2] = p - r; e4[3] = q - t;
#pragma unroll
    for (int hs = 1; hs < 32; hs <<= 1) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float o = __shfl_xor_sync(0xffffffffu, e4[k], hs);
        e4[k] = (lane & hs) ? o - e4[k] : e4[k] + o;
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      buf[kBlock * b + 4 * lane + k] = e4[k];
      mx = fmaxf(mx, fabsf(e4[k]));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  float tmax = 0.0f;
#pragma unroll
  for (int w = 0; w < kRotThreads / 32; ++w) tmax = fmaxf(tmax, red[w]);
  int e = 0;
  if (tmax > 0.0f && isfinite(tmax)) frexpf(tmax, &e);
  const int k = max(-120, min(120, 15 - e));
  const float sc = ldexpf(1.0f, k);
  if (threadIdx.x == 0) inv_s[a] = ldexpf(1.0f, -k) * __ldg(weight + a);  // the routing weight rides on the scale
  uint16_t* dst = Bh + static_cast<int64_t>(a) * nb * kBlock;
  for (int i = threadIdx.x; i < nb * kBlock; i += kRotThreads) dst[i] = __half_as_ushort(__float2half_rn(buf[i] * sc));
}

// ---------------------------------------------------------------- main kernel
// Rings: codes (one 128-row x 80-byte block column per stage, TMA) and A/B
// stages (one 128-wide K block: A decoded into 64 TMEM columns, B as two
// 64-wide TMA boxes with 128-byte swizzle); see tc_groups for the mapping.
template <class F>
__host__ __device__ constexpr int tc_code_bytes() { return kTcTileRows * F::kBytes; }  // one code stage

constexpr int kTcSmemMax = 227 * 1024;
constexpr int kTcSmemFixed = 1024 /*align slack*/ + 1024 /*centroid table, barriers, misc*/;
static_assert(4 * TcQ5::kLevels + 8 * (2 * kTcStages + 2 * 4 + 1) + 16 <= 512, "barrier block overflows into the row maxima");
constexpr int kTcMaxNb = 64;  // tile norms in shared memory: 128 x nb (in <= 8192)

// Decode groups: G groups of 8 warps take blocks b = g (mod G).  Every ring
// stage belongs to exactly one group, so each stage is consumed in order by a
// single consumer and mbarrier parity waits are never ambiguous:
//   A/B stage of block b   = b mod S (S = 2 stages: one per group when G = 2,
//                            both of the one group when G = 1)
//   code stage of block b  = 2 (b mod G) + (b / G) mod 2   (two per group)
// TMEM: the accumulator (128 columns for token tiles <= 128, else 256), then
// the S A stages; 256 or 512 columns allocated.
__host__ __device__ inline int tc_groups(int n_box) { return n_box > 128 ? 2 : 1; }
__host__ __device__ inline int tc_cstages(int n_box) { return 2 * tc_groups(n_box); }
__host__ __device__ inline int tc_stages(int, int) { return kTcStages; }
__host__ __device__ inline uint32_t tc_acc_cols(int n_box) { return n_box > 128 ? 256u : 128u; }
__host__ __device__ inline uint32_t tc_alloc_cols(int n_box) { return n_box > 128 ? 512u : 256u; }

template <class F>
__host__ __device__ inline int tc_norm_bytes(int nb) {
  return (kTcTileRows * nb * static_cast<int>(sizeof(typename F::Norm)) + 15) & ~15;
}

template <class F>
__host__ __device__ inline int tc_smem_bytes(int n_box, int nb) {
  return kTcSmemFixed + tc_stages(n_box, nb) * n_box * 256 + tc_cstages(n_box) * tc_code_bytes<F>() +
         tc_norm_bytes<F>(nb);
}

__host__ __device__ inline int tc_ab_stage(int b, int S) { return b % S; }
__host__ __device__ inline uint32_t tc_ab_parity(int b, int S) { return static_cast<uint32_t>(b / S) & 1u; }
__host__ __device__ inline int tc_code_stage(int b, int G) { return 2 * (b % G) + ((b / G) & 1); }
__host__ __device__ inline uint32_t tc_code_parity(int b, int G) { return static_cast<uint32_t>(b / G / 2) & 1u; }

// Grouped mode (the routed MoE layer): the weights are E experts stacked by
// rows (rows_e rows each) and B holds one row per (token, expert) assignment,
// grouped by expert.  CTA (slot, row tile j, token tile nt) multiplies the
// rows of expert active[slot] with the B rows offsets[slot] ..
// offsets[slot + 1] - 1 and writes Y[assignment][j * 128 + r].  The expert
// id shared_id (the shared expert) reads its own matrix (second code map,
// norms2).  Slots past the active count (meta[0]) and token tiles past an
// expert's assignments exit at once.  active == nullptr: plain mode.
struct TcGroup {
  const int* meta;
  const int* active;
  const int* offsets;
  const void* norms2;
  int rows_e, tiles_e, n_tiles, shared_id;
};

template <class F, int NG>
__global__ void __launch_bounds__(TcRoles<NG>::kThreads, NG == 1 ? 2 : 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap bmap, const __grid_constant__ CUtensorMap cmap,
               const __grid_constant__ CUtensorMap cmap2,
               const typename F::Norm* __restrict__ norms, const float* __restrict__ codebook, int64_t O, int nb, int M,
               const float* __restrict__ inv_s, void* __restrict__ Y, int64_t ldy, int out_bf16, int n_box,
               int row_tiles, int nfull, float* __restrict__ part, unsigned* __restrict__ part_cnt,
               const TcGroup grp) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw));
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  constexpr int kTcDecWarps = TcRoles<NG>::kDecWarps, kTcWCodes = TcRoles<NG>::kWCodes, kTcWMma = TcRoles<NG>::kWMma,
                kTcWB = TcRoles<NG>::kWB;
  constexpr int G = NG, S = kTcStages, CS = 2 * NG;
  const uint32_t acc_cols = tc_acc_cols(n_box), alloc_cols = tc_alloc_cols(n_box);
  const uint32_t tab = base;                 // 32 fp32 centroids
  const uint32_t bst = base + 1024;
  const uint32_t cst = bst + S * n_box * 256;
  constexpr int kCode = tc_code_bytes<F>();
  using Norm = typename F::Norm;
  const uint32_t nst = cst + CS * kCode;                 // tile norms [128][nb]
  const uint32_t bars = base + 4 * TcQ5::kLevels;        // after the table, inside the first 1 KiB
  // barrier block: full[S] empty[S] c_full[CS] c_empty[CS] accum, then misc
  // (TMEM base, abort flag, split count): at most 128 + 8 (2 S + 2 CS + 1) + 16 = 296 bytes
  const uint32_t full0 = bars, empty0 = full0 + 8 * S, c_full0 = empty0 + 8 * S, c_empty0 = c_full0 + 8 * CS,
                 accum = c_empty0 + 8 * CS;
  const uint32_t misc = accum + 8;
  volatile uint32_t* misc_g = reinterpret_cast<volatile uint32_t*>(gbase + (misc - base));
  float* c32 = reinterpret_cast<float*>(gbase);
  const uint8_t* codes_g = gbase + (cst - base);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // CTA -> tile and K range: CTAs [0, nfull) take whole tiles; the rest take
  // the two K halves of the tiles after them (tile nfull + j / 2, half j % 2)
  int tt = blockIdx.x, half = -1, kb0 = 0, kb1 = nb;
  if (tt >= nfull) {
    const int j = tt - nfull;
    tt = nfull + (j >> 1);
    half = j & 1;
    kb0 = half ? nb / 2 : 0;
    kb1 = half ? nb : nb / 2;
  }
  int64_t o0 = static_cast<int64_t>(tt % row_tiles) * kTcTileRows;  // first weight row of the tile
  int64_t oend = O;                                                  // end of the rows the tile may read
  int64_t oy0 = o0;                                                  // output column of the tile's first row
  int n0 = (tt / row_tiles) * n_box;                                 // first B row of the tile
  int mend = M;                                                      // end of the tile's valid B rows
  bool use2 = false;                                                 // the shared expert's own matrix
  if (grp.active) {
    // grouped mode: a CTA-uniform early exit, before any barrier or TMEM
    const int per = grp.tiles_e * grp.n_tiles;
    const int slot = static_cast<int>(blockIdx.x) / per, rem = static_cast<int>(blockIdx.x) - slot * per;
    if (slot >= __ldg(grp.meta)) return;
    const int e = __ldg(grp.active + slot);
    use2 = e == grp.shared_id;
    const int a0 = __ldg(grp.offsets + slot), cnt = __ldg(grp.offsets + slot + 1) - a0;
    const int j = rem / grp.n_tiles, nt = rem - j * grp.n_tiles;
    if (nt * n_box >= cnt) return;
    oy0 = static_cast<int64_t>(j) * kTcTileRows;
    const int64_t er = use2 ? 0 : static_cast<int64_t>(e) * grp.rows_e;  // the expert's first row
    o0 = er + oy0;
    oend = er + grp.rows_e;
    n0 = a0 + nt * n_box;
    mend = a0 + cnt;
  }
  const uint64_t deadline = globaltimer_ns() + wait_limit_ns();

  // ---- set-up: barriers, TMEM, row maxima cleared (the codebook is loaded
  // by the decode warps, whose own barrier publishes it)
  uint32_t* rowmax = reinterpret_cast<uint32_t*>(gbase + 512);  // [128] fp32 bits, inside the first 1 KiB
  if (threadIdx.x < kTcTileRows) rowmax[threadIdx.x] = 0u;
  // The code producer initialises the barriers and requests the first code
  // boxes (one per code stage) before the CTA barrier, so that their memory
  // latency overlaps the TMEM allocation and the norm loads.
  const int early = std::min(kb1 - kb0, CS);
  if (warp == kTcWCodes && lane == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 9);   // 8 decode warps + the B producer (plus its TMA bytes)
      mbar_init(empty0 + 8 * s, 1);  // the MMA commit
    }
    for (int s = 0; s < CS; ++s) {
      mbar_init(c_full0 + 8 * s, 1);
      mbar_init(c_empty0 + 8 * s, 8);
    }
    mbar_init(accum, 1);
    misc_g[1] = 0u;  // abort flag
    fence_barrier_init();
    for (int lb = 0; lb < early; ++lb) {
      const int cs = tc_code_stage(lb, G);
      if (fault_skip_tma()) continue;
      mbar_arrive_expect_tx(c_full0 + 8 * cs, kCode);
      tma_load_2d(cst + cs * kCode, use2 ? &cmap2 : &cmap, F::kBytes * (kb0 + lb), static_cast<int>(o0),
                  c_full0 + 8 * cs);
    }
  }
  if (warp == kTcWMma) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(misc), "r"(alloc_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc_g[0];
  Norm* nrm_s = reinterpret_cast<Norm*>(gbase + (nst - base));

  if (warp < kTcDecWarps) {
    // The tile's norms [128][nb] are one contiguous run of the norm array
    // (rows past O read as zero); they are staged while the producers start
    // on the first code and B boxes, then a barrier of the decode warps only.
    const int64_t nvalid = std::min<int64_t>(kTcTileRows, oend - o0) * nb;
    const Norm* nsrc = (use2 ? static_cast<const Norm*>(grp.norms2) : norms) + o0 * nb;
    // Each row's largest norm is gathered on the way (shared-memory atomic
    // max on the fp32 bits: the norms are >= 0; NaN is left out).
    if (threadIdx.x < F::kLevels) {
      const float c = __ldg(codebook + threadIdx.x);
      c32[threadIdx.x] = c;
      if (threadIdx.x + 1 < F::kLevels && !(c < __ldg(codebook + threadIdx.x + 1)))
        raise_device_error(HLWQ_DEVERR_CODEBOOK);
    }
    auto row_max = [&](int k, float v) {
      if (!(v != v)) atomicMax(rowmax + k / nb, __float_as_uint(v));
    };
    const int ntot = kTcTileRows * nb;                                   // a multiple of 8
    constexpr int kPer16 = 16 / static_cast<int>(sizeof(Norm));          // norms per 16-byte load
    if ((reinterpret_cast<uintptr_t>(nsrc) & 15u) == 0) {
      for (int q = threadIdx.x; q < ntot / kPer16; q += 32 * kTcDecWarps) {
        if (kPer16 * q + kPer16 <= nvalid) {
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(nsrc) + q);
          reinterpret_cast<uint4*>(nrm_s)[q] = u;
          const Norm* e = reinterpret_cast<const Norm*>(&u);
          if (nb % kPer16 == 0) {  // the 16 bytes lie in one row: one atomic
            float m = 0.0f;
#pragma unroll
            for (int k = 0; k < kPer16; ++k) m = fmaxf(m, F::norm(e[k]));
            row_max(kPer16 * q, m);
          } else {
#pragma unroll
            for (int k = 0; k < kPer16; ++k) row_max(kPer16 * q + k, F::norm(e[k]));
          }
        } else {
          for (int k = kPer16 * q; k < kPer16 * q + kPer16; ++k) {
            const Norm v = k < nvalid ? __ldg(nsrc + k) : Norm(0);
            nrm_s[k] = v;
            row_max(k, F::norm(v));
          }
        }
      }
    } else {
      for (int q = threadIdx.x; q < ntot; q += 32 * kTcDecWarps) {
        const Norm v = q < nvalid ? __ldg(nsrc + q) : Norm(0);
        nrm_s[q] = v;
        row_max(q, F::norm(v));
      }
    }
    asm volatile("bar.sync 1, %0;" ::"r"(32 * kTcDecWarps) : "memory");

    // ---------------------------------------------------------- decode
    // two groups of 8 warps take alternate blocks; in a group, warp (q4, hh)
    // decodes half block hh of rows 32 q4 + lane
    const int dg = warp >> 3, q4 = warp & 3, hh = (warp >> 2) & 1;  // group dg takes blocks b = dg mod G
    const int r = 32 * q4 + lane;
    const Norm* rown = nrm_s + r * nb;
    const float nmax = __uint_as_float(rowmax[r]);
    int erow = 0;
    if (nmax > 0.0f && isfinite(nmax)) frexpf(nmax, &erow);
    const float rs = ldexpf(1.0f, -erow);
    const uint32_t tm_row = tmem + (static_cast<uint32_t>(32 * q4) << 16);
    bool ok = true;
    for (int b = kb0 + dg; b < kb1 && dg < G; b += G) {
      const int lb = b - kb0;
      const int cs = tc_code_stage(lb, G), as = tc_ab_stage(lb, S);
      const float nsc = F::norm(rown[b]) * rs;
      constexpr int NW = F::kBytes / 16;  // 8-byte words of a half block
      uint2 cw[NW];
      if (ok) ok = mbar_wait(c_full0 + 8 * cs, tc_code_parity(lb, G), deadline);
      const uint2* src = reinterpret_cast<const uint2*>(codes_g + cs * kCode + r * F::kBytes + (F::kBytes / 2) * hh);
#pragma unroll
      for (int k = 0; k < NW; ++k) cw[k] = src[k];
      __syncwarp();
      if (lane == 0) mbar_arrive(c_empty0 + 8 * cs);
      const float2 sc2 = make_float2(nsc, nsc);
      uint32_t v[32];
#pragma unroll
      for (int p = 0; p < 32; ++p) {
        const float2 c = make_float2(__uint_as_float(lds_u32(code_addr<F>(cw, 2 * F::kBits * p, tab))),
                                     __uint_as_float(lds_u32(code_addr<F>(cw, 2 * F::kBits * p + F::kBits, tab))));
        const float2 a = fmul2(c, sc2);
        v[p] = cvt_half2(a.x, a.y);
      }
      if (ok) ok = mbar_wait(empty0 + 8 * as, tc_ab_parity(lb, S) ^ 1u, deadline);
      if (ok && misc_g[1] == 0u) {
        const uint32_t ta = tm_row + acc_cols + 64 * as + 32 * hh;
        uint32_t v0[16], v1[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) { v0[k] = v[k]; v1[k] = v[16 + k]; }
        tc_st16(ta, v0);
        tc_st16(ta + 16, v1);
        tc_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(full0 + 8 * as);
    }
    if (!ok) {
      misc_g[1] = 1u;
      raise_device_error(HLWQ_DEVERR_TIMEOUT);
    }

    // ---------------------------------------------------------- epilogue
    // every decode warp: warp w reads TMEM lanes 32 (w mod 4) .. + 31 (its own
    // rows) and columns 16 (w / 4) + 96 j, so six warps share a lane quarter
    {
      const bool done = mbar_wait(accum, 0, deadline);
      tc_fence_after();
      if (!done) {
        misc_g[1] = 1u;
        raise_device_error(HLWQ_DEVERR_TIMEOUT);
      }
      const float rscale = ldexpf(1.0f, erow - 7);  // 2^erow / 128 (no overflow for fp32 norms)
      constexpr int kCStep = 16 * (kTcDecWarps / 4);
      bool write_tile = true;
      const float* p0 = nullptr;
      const float* p1 = nullptr;
      if (half >= 0) {
        // K-split tile: both halves write their fp32 partial ([column][row],
        // so a warp's stores are contiguous), then count themselves in; the
        // half that arrives second adds the two partials in the fixed order
        // (K half 0) + (K half 1), so the result does not depend on which
        // half finished first.  No CTA waits for another.
        const int slot = tt - nfull;
        float* q0 = part + static_cast<int64_t>(2 * slot) * n_box * kTcTileRows;
        float* mine = q0 + (half ? static_cast<int64_t>(n_box) * kTcTileRows : 0);
        p0 = q0;
        p1 = q0 + static_cast<int64_t>(n_box) * kTcTileRows;
        for (int c0 = 16 * (warp >> 2); c0 < n_box; c0 += kCStep) {
          uint32_t acc[16];
          tc_ld16(tm_row + c0, acc);
          tc_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) mine[(c0 + j) * kTcTileRows + r] = __uint_as_float(acc[j]);
        }
        __threadfence();
        asm volatile("bar.sync 2, %0;" ::"r"(32 * kTcDecWarps) : "memory");
        if (threadIdx.x == 0) misc_g[2] = atomicAdd(part_cnt + slot, 1u);
        asm volatile("bar.sync 2, %0;" ::"r"(32 * kTcDecWarps) : "memory");
        write_tile = misc_g[2] == 1u;
        if (write_tile) __threadfence();
      }
      if (write_tile) {
        // The scaled tile is staged in shared memory as [token][row] (the B
        // stages are free once the accumulator is complete: n_box x 128 x 4
        // bytes at most, within S >= 2 stages of n_box x 256), then written
        // out as contiguous runs of every token's 128 outputs.
        const int es = out_bf16 ? 2 : 4;
        uint8_t* stage = gbase + (bst - base);
        for (int c0 = 16 * (warp >> 2); c0 < n_box; c0 += kCStep) {
#pragma unroll
          for (int h8 = 0; h8 < 16; h8 += 8) {  // eight columns at a time (register budget)
            float v[8];
            if (half < 0) {
              uint32_t acc[8];
              tc_ld8(tm_row + c0 + h8, acc);
              tc_wait_ld();
#pragma unroll
              for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(acc[j]);
            } else {
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const int idx = (c0 + h8 + j) * kTcTileRows + r;
                v[j] = __ldcg(p0 + idx) + __ldcg(p1 + idx);
              }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int m = n0 + c0 + h8 + j;
              const float yv = m < mend ? v[j] * rscale * __ldg(inv_s + m) : 0.0f;
              const int si = (c0 + h8 + j) * kTcTileRows + r;
              if (out_bf16) reinterpret_cast<uint16_t*>(stage)[si] = static_cast<uint16_t>(float_to_bf16_bits(yv));
              else reinterpret_cast<float*>(stage)[si] = yv;
            }
          }
        }
        asm volatile("bar.sync 2, %0;" ::"r"(32 * kTcDecWarps) : "memory");
        if (done && misc_g[1] == 0u) {
          const int ncols = static_cast<int>(std::min<int64_t>(kTcTileRows, oend - o0));  // outputs of the tile
          const int mrows = std::min(n_box, mend - n0);                                   // tokens of the tile
          char* yb = static_cast<char*>(Y);
          if (ncols == kTcTileRows && ((ldy * es) & 15) == 0) {
            const int sh = out_bf16 ? 4 : 5;  // 16-byte pieces per token: 128 x es / 16
            const int64_t pitch = ldy * es;
            char* yt = yb + (static_cast<int64_t>(n0) * ldy + oy0) * es;
            for (int q = threadIdx.x; q < (mrows << sh); q += 32 * kTcDecWarps) {
              const int ml = q >> sh, pc = q & ((1 << sh) - 1);
              *reinterpret_cast<uint4*>(yt + ml * pitch + 16 * pc) = reinterpret_cast<const uint4*>(stage)[q];
            }
          } else {
            for (int q = threadIdx.x; q < mrows * kTcTileRows; q += 32 * kTcDecWarps) {
              const int ml = q >> 7, oc = q & (kTcTileRows - 1);
              if (oc >= ncols) continue;
              const int64_t off = (n0 + ml) * ldy + oy0 + oc;
              if (out_bf16) reinterpret_cast<uint16_t*>(yb)[off] = reinterpret_cast<const uint16_t*>(stage)[q];
              else reinterpret_cast<float*>(yb)[off] = reinterpret_cast<const float*>(stage)[q];
            }
          }
        }
      }
    }
  } else if (warp == kTcWCodes) {
    // ---------------------------------------------------------- TMA producer: code tiles
    if (lane == 0) {
      bool ok = true;
      int last = early > 0 && !fault_skip_tma() ? kb0 + early - 1 : -1;  // last block whose copy was issued
      for (int b = kb0 + early; b < kb1; ++b) {
        const int cs = tc_code_stage(b - kb0, G);
        ok = mbar_wait(c_empty0 + 8 * cs, tc_code_parity(b - kb0, G) ^ 1u, deadline) && misc_g[1] == 0u;
        if (!ok) break;
        if (fault_skip_tma()) continue;
        mbar_arrive_expect_tx(c_full0 + 8 * cs, kCode);
        tma_load_2d(cst + cs * kCode, use2 ? &cmap2 : &cmap, F::kBytes * b, static_cast<int>(o0), c_full0 + 8 * cs);
        last = b;
      }
      if (!ok) {
        misc_g[1] = 1u;
        raise_device_error(HLWQ_DEVERR_TIMEOUT);
      }
      // no copy may still be landing when the CTA exits: wait (bounded) for
      // the last copy issued into each code stage
      const uint64_t dl = globaltimer_ns() + wait_limit_ns();
      for (int b = std::max(kb0, last - CS + 1); b <= last; ++b)
        mbar_wait(c_full0 + 8 * tc_code_stage(b - kb0, G), tc_code_parity(b - kb0, G), dl);
    }
  } else if (warp == kTcWB) {
    // ---------------------------------------------------------- TMA producer: B tiles
    if (lane == 0) {
      const uint32_t half_bytes = static_cast<uint32_t>(n_box) * 128u;
      bool ok = true;
      int last = -1;  // last block whose copies were issued
      for (int b = kb0; b < kb1; ++b) {
        const int st = tc_ab_stage(b - kb0, S);
        ok = mbar_wait(empty0 + 8 * st, tc_ab_parity(b - kb0, S) ^ 1u, deadline) && misc_g[1] == 0u;
        if (!ok) break;
        if (fault_skip_tma()) continue;
        mbar_arrive_expect_tx(full0 + 8 * st, 2 * half_bytes);
        const uint32_t dst = bst + st * n_box * 256;
        tma_load_2d(dst, &bmap, kTcKChunk * (2 * b), n0, full0 + 8 * st);
        tma_load_2d(dst + half_bytes, &bmap, kTcKChunk * (2 * b + 1), n0, full0 + 8 * st);
        last = b;
      }
      if (!ok) {
        misc_g[1] = 1u;
        raise_device_error(HLWQ_DEVERR_TIMEOUT);
      }
      // wait (bounded) for the last copies issued into each A/B stage (the
      // decode warps arrive on every stage they take, so a stage's phase
      // completes once its bytes have landed)
      const uint64_t dl = globaltimer_ns() + wait_limit_ns();
      for (int b = std::max(kb0, last - S + 1); b <= last; ++b)
        mbar_wait(full0 + 8 * tc_ab_stage(b - kb0, S), tc_ab_parity(b - kb0, S), dl);
    }
  } else if (warp == kTcWMma) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(n_box);
      bool ok = true;
      // The MMA thread paces the whole CTA (one tcgen05.mma costs about as
      // much to issue as a 64-token MMA takes to run), so its loop carries
      // the stage and parity instead of dividing by G, and does not poll the
      // abort flag: when another role gives up, this thread's own bounded
      // wait on the stage it needs runs out.
      int st = 0;
      uint32_t par = 0u;
      for (int b = kb0; b < kb1; ++b, st = (st + 1 == S) ? 0 : st + 1, par ^= (st == 0) ? 1u : 0u) {
        ok = mbar_wait(full0 + 8 * st, par, deadline);
        if (!ok) break;
        tc_fence_after();
        const uint32_t bstage = bst + st * n_box * 256;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint64_t bdesc = smem_desc_sw128(bstage + h * n_box * 128);
#pragma unroll
          for (int kk = 0; kk < kTcKChunk / 16; ++kk)
            tc_mma_f16(tmem, tmem + acc_cols + 64 * st + 32 * h + 8 * kk, bdesc + static_cast<uint64_t>(2 * kk),
                       idesc, (b > kb0 || h > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(empty0 + 8 * st);  // frees both the A stage (TMEM) and the B stage (shared memory)
      }
      if (!ok) {
        misc_g[1] = 1u;
        raise_device_error(HLWQ_DEVERR_TIMEOUT);
      }
      tc_commit(accum);  // fires once every MMA issued above has completed
      // the commit's arrival lands before the CTA can exit (bounded)
      mbar_wait(accum, 0, globaltimer_ns() + wait_limit_ns());
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kTcWMma) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(alloc_cols) : "memory");
  }
}

}  // namespace

// Launch plan for a shape on the current device.  Tiles are 128 rows x n_box
// tokens.  When the tiles fill the SMs once and leave a partial second wave
// of at most half the SMs, those last tiles are split into two K halves (two
// CTAs each), so the second wave takes half a tile's time on up to all SMs.
// Workspace: B (binary16 rotated activations) | 1/s_m | split counters |
// split partials (fp32, two per split tile).  A workspace of base_bytes
// runs without the split.
struct TcPlan {
  int nb, n_box, row_tiles, n_tiles, nsplit;
  size_t inv_off, cnt_off, part_off, base_bytes, split_bytes;
};

template <class F>
TcPlan tc_plan(int64_t O, int64_t in, int64_t M) {
  auto r256 = [](size_t v) { return (v + 255) & ~static_cast<size_t>(255); };
  TcPlan P;
  P.nb = static_cast<int>(ceil_div(in, kBlock));
  int n_box = static_cast<int>(std::min<int64_t>(256, (std::min<int64_t>(M, 256) + 15) / 16 * 16));
  while (n_box > 16 && tc_smem_bytes<F>(n_box, P.nb) > kTcSmemMax) n_box = (n_box / 2 + 15) / 16 * 16;
  P.n_box = n_box;
  P.row_tiles = static_cast<int>(ceil_div(O, kTcTileRows));
  P.n_tiles = static_cast<int>(ceil_div(M, n_box));
  const int64_t tiles = static_cast<int64_t>(P.row_tiles) * P.n_tiles;
  const int64_t sms = sm_count();
  P.nsplit = (P.nb >= 2 && tiles > sms && 2 * (tiles - sms) <= sms) ? static_cast<int>(tiles - sms) : 0;
  P.inv_off = r256(static_cast<size_t>(M) * P.nb * kBlock * 2);
  P.base_bytes = P.inv_off + static_cast<size_t>(M) * 4 + 256;
  P.cnt_off = r256(P.inv_off + static_cast<size_t>(M) * 4);
  P.part_off = r256(P.cnt_off + static_cast<size_t>(P.nsplit) * 4);
  P.split_bytes = P.part_off + static_cast<size_t>(P.nsplit) * 2 * kTcTileRows * n_box * 4;
  return P;
}

// Rows longer than kTcMaxNb blocks do not fit the tile-norm staging and run
// on the CUDA-core kernels, which need no workspace.
inline bool gemm_tc_takes(int64_t in) { return ceil_div(in, kBlock) <= kTcMaxNb; }

template <class F>
size_t tc_workspace_bytes(int64_t O, int64_t in, int64_t M) {
  if (!gemm_tc_takes(in)) return 0;
  const TcPlan P = tc_plan<F>(O, in, M);
  return P.nsplit ? std::max(P.split_bytes, P.base_bytes) : P.base_bytes;
}

template <class F>
size_t tc_workspace_min_bytes(int64_t O, int64_t in, int64_t M) {
  return gemm_tc_takes(in) ? tc_plan<F>(O, in, M).base_bytes : 0;
}

size_t gemm_tc_workspace_bytes(int64_t O, int64_t in, int64_t M) { return tc_workspace_bytes<TcQ5>(O, in, M); }
size_t gemm_tc_workspace_min_bytes(int64_t O, int64_t in, int64_t M) {
  return tc_workspace_min_bytes<TcQ5>(O, in, M);
}
size_t tq3_tc_workspace_bytes(int64_t O, int64_t in, int64_t M) { return tc_workspace_bytes<TcTq3>(O, in, M); }
size_t tq3_tc_workspace_min_bytes(int64_t O, int64_t in, int64_t M) {
  return tc_workspace_min_bytes<TcTq3>(O, in, M);
}

// The tensor-core kernel on a prepared B operand: binary16 [b_rows][nb * 128]
// (K-major, 16-byte aligned rows), scales inv_s per B row.  Plain mode:
// row_tiles x token tiles (the last partial wave split in K over nsplit tile
// pairs); grouped mode: grp.active != nullptr, grid CTAs of the group mapping.
template <class F>
int launch_tc_core(const uint8_t* packed, const typename F::Norm* norms, const float* codebook, int64_t O, int nb,
                   const uint16_t* B, int64_t b_rows, int M, const float* inv_s, void* Y, int64_t ldy, bool out_bf16,
                   int n_box, int row_tiles, int nfull, int nsplit, float* part, unsigned* part_cnt,
                   const TcGroup& grp, cudaStream_t stream, const uint8_t* packed2 = nullptr, int64_t O2 = 0) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode_fn();
  if (!encode) return HLWQ_ECUDA;
  CUtensorMap map;
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(nb) * kBlock, static_cast<cuuint64_t>(b_rows)};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(nb) * kBlock * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTcKChunk), static_cast<cuuint32_t>(n_box)};
  const cuuint32_t estr[2] = {1, 1};
  if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(B), gdim, gstride, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return HLWQ_ECUDA;
  // Codes viewed as a 2-D byte tensor [O][NB * bytes]; one box = 128 rows x
  // one block (80 or 48 bytes: multiples of 16, as is every box's x offset).
  CUtensorMap cmap, cmap2;
  const cuuint64_t cstride[1] = {static_cast<cuuint64_t>(nb) * F::kBytes};
  const cuuint32_t cbox[2] = {static_cast<cuuint32_t>(F::kBytes), static_cast<cuuint32_t>(kTcTileRows)};
  static_assert(F::kBytes % 16 == 0, "code boxes start on 16-byte boundaries");
  for (int k = 0; k < 2; ++k) {
    const uint8_t* src = k == 0 ? packed : (packed2 ? packed2 : packed);
    const cuuint64_t cdim[2] = {static_cast<cuuint64_t>(nb) * F::kBytes,
                                static_cast<cuuint64_t>(k == 0 || !packed2 ? O : O2)};
    if (encode(k == 0 ? &cmap : &cmap2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(src), cdim, cstride,
               cbox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return HLWQ_ECUDA;
  }
  const int smem = tc_smem_bytes<F>(n_box, nb);
  static PerDeviceOnce attr;
  if (const int st = attr([&] {
        return cudaFuncSetAttribute(gemm_tc_kernel<F, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    227 * 1024) == cudaSuccess &&
               cudaFuncSetAttribute(gemm_tc_kernel<F, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    227 * 1024) == cudaSuccess;
      }))
    return st;
  if (smem > kTcSmemMax) return HLWQ_EUNSUPPORTED;
  const int grid = nfull + 2 * nsplit, ob = out_bf16 ? 1 : 0;
  if (grid <= 0) return HLWQ_OK;
  if (tc_groups(n_box) == 1)
    gemm_tc_kernel<F, 1><<<grid, TcRoles<1>::kThreads, smem, stream>>>(map, cmap, cmap2, norms, codebook, O, nb, M, inv_s, Y,
                                                                       ldy, ob, n_box, row_tiles, nfull, part,
                                                                       part_cnt, grp);
  else
    gemm_tc_kernel<F, 2><<<grid, TcRoles<2>::kThreads, smem, stream>>>(map, cmap, cmap2, norms, codebook, O, nb, M, inv_s, Y,
                                                                       ldy, ob, n_box, row_tiles, nfull, part,
                                                                       part_cnt, grp);
  return cudaGetLastError() == cudaSuccess ? HLWQ_OK : HLWQ_ECUDA;
}

inline int set_rot_attrs() {
  static PerDeviceOnce rot_attr;
  return rot_attr([&] {
    return cudaFuncSetAttribute(rotate_x_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) ==
               cudaSuccess &&
           cudaFuncSetAttribute(silu_rotate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) ==
               cudaSuccess;
  });
}

// Rotation of X into the workspace, then the tensor-core kernel (in <= 8192;
// the workspace holds at least the plan's base_bytes).  signs: TQ3's sign
// vectors, or nullptr for Q5.
template <class F>
int launch_tc(const uint8_t* packed, const typename F::Norm* norms, const float* codebook, const int8_t* signs,
              int64_t O, int in, const uint16_t* X, int64_t ldx, int M, void* Y, int64_t ldy, bool out_bf16,
              void* workspace, size_t ws_bytes, cudaStream_t stream) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  const TcPlan P = tc_plan<F>(O, in, M);
  if (ws_bytes < P.base_bytes) return HLWQ_EWORKSPACE;
  const int nsplit = ws_bytes >= P.split_bytes ? P.nsplit : 0;
  char* ws = static_cast<char*>(workspace);
  uint16_t* B = reinterpret_cast<uint16_t*>(ws);
  float* inv_s = reinterpret_cast<float*>(ws + P.inv_off);
  unsigned* part_cnt = reinterpret_cast<unsigned*>(ws + P.cnt_off);
  float* part = nsplit ? reinterpret_cast<float*>(ws + P.part_off) : nullptr;
  const int rot_smem = nb * kBlock * 4;
  if (rot_smem > 200 * 1024) return HLWQ_EUNSUPPORTED;
  if (const int st = set_rot_attrs()) return st;
  rotate_x_kernel<<<M, kRotThreads, rot_smem, stream>>>(X, ldx, in, nb, signs, nullptr, B, inv_s, part_cnt, nsplit);
  if (cudaGetLastError() != cudaSuccess) return HLWQ_ECUDA;
  const int nfull = P.row_tiles * P.n_tiles - nsplit;
  return launch_tc_core<F>(packed, norms, codebook, O, nb, B, M, M, inv_s, Y, ldy, out_bf16, P.n_box, P.row_tiles,
                           nfull, nsplit, part, part_cnt, TcGroup{}, stream);
}

// The routed MoE layer on the tensor cores (the grouped path): after the
// router has grouped the (token, expert) assignments by expert,
//   1. rotate_x_kernel gathers and rotates each assignment's token (Bg);
//   2. the grouped kernel multiplies every active expert's gate_up rows with
//      its assignments' rows of Bg (each expert's codes decoded once for all
//      its tokens; the shared expert, the last slot, from its own matrix);
//   3. silu_rotate_kernel forms h = SiLU(g) * u and rotates it (Bh), with the
//      routing weight folded into the row scale;
//   4. the same for the down rows into the per-assignment partial outputs;
// the caller then adds the partials per token in a fixed order.
// EUNSUPPORTED when the rows' tile norms do not fit the shared memory.
int launch_moe_tc(const uint8_t* gu_packed, const uint16_t* gu_norms, const uint8_t* dn_packed,
                  const uint16_t* dn_norms, const uint8_t* sh_gu_packed, const uint16_t* sh_gu_norms,
                  const uint8_t* sh_dn_packed, const uint16_t* sh_dn_norms, const float* codebook, int E, int H, int F,
                  int topk, int T, const uint16_t* X, const MoeWs& ws, cudaStream_t stream) {
  const int nbh = static_cast<int>(ceil_div(H, kBlock)), nbf = static_cast<int>(ceil_div(F, kBlock));
  const bool shared = sh_gu_packed != nullptr;
  const int na = T * topk + (shared ? T : 0);
  int n_box = static_cast<int>(std::min<int64_t>(256, (static_cast<int64_t>(T) + 15) / 16 * 16));
  while (n_box > 16 && tc_smem_bytes<TcQ5>(n_box, std::max(nbh, nbf)) > kTcSmemMax) n_box = (n_box / 2 + 15) / 16 * 16;
  const int n_tiles = static_cast<int>(ceil_div(T, n_box));  // an expert has at most T assignments
  if (const int st = set_rot_attrs()) return st;
  rotate_x_kernel<<<na, kRotThreads, nbh * kBlock * 4, stream>>>(X, H, H, nbh, nullptr, ws.asg_token, ws.bg, ws.inv_g,
                                                                   nullptr, 0);
  if (cudaGetLastError() != cudaSuccess) return HLWQ_ECUDA;
  const int two_f = 2 * F;
  const int nslots = E + (shared ? 1 : 0);
  TcGroup gu{ws.meta, ws.active, ws.offsets, sh_gu_norms, two_f, static_cast<int>(ceil_div(two_f, kTcTileRows)),
             n_tiles, shared ? E : -1};
  int st = launch_tc_core<TcQ5>(gu_packed, gu_norms, codebook, static_cast<int64_t>(E) * two_f, nbh, ws.bg, na, na,
                                ws.inv_g, ws.g2, two_f, false, n_box, 1, nslots * gu.tiles_e * n_tiles, 0, nullptr,
                                nullptr, gu, stream, sh_gu_packed, two_f);
  if (st) return st;
  silu_rotate_kernel<<<na, kRotThreads, nbf * kBlock * 4, stream>>>(ws.g2, F, nbf, ws.asg_weight, ws.bh, ws.inv_h);
  if (cudaGetLastError() != cudaSuccess) return HLWQ_ECUDA;
  TcGroup dn{ws.meta, ws.active, ws.offsets, sh_dn_norms, H, static_cast<int>(ceil_div(H, kTcTileRows)), n_tiles,
             shared ? E : -1};
  st = launch_tc_core<TcQ5>(dn_packed, dn_norms, codebook, static_cast<int64_t>(E) * H, nbf, ws.bh, na, na, ws.inv_h,
                            ws.part, H, false, n_box, 1, nslots * dn.tiles_e * n_tiles, 0, nullptr, nullptr, dn, stream,
                            sh_dn_packed, H);
  if (st) return st;
  return HLWQ_OK;
}

int launch_dense(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                 const uint16_t* X, int64_t ldx, int M, void* Y, int64_t ldy, bool out_bf16, cudaStream_t stream);

int launch_gemm_tc(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                   const uint16_t* X, int64_t ldx, int M, void* Y, int64_t ldy, bool out_bf16, void* workspace,
                   size_t ws_bytes, cudaStream_t stream) {
  if (!gemm_tc_takes(in)) return launch_dense(packed, norms, codebook, O, in, X, ldx, M, Y, ldy, out_bf16, stream);
  return launch_tc<TcQ5>(packed, norms, codebook, nullptr, O, in, X, ldx, M, Y, ldy, out_bf16, workspace, ws_bytes,
                         stream);
}

int launch_tq3_gemv(const uint8_t* packed, const float* norms, const int8_t* signs, const float* codebook,
                    int64_t O, int in, const uint16_t* x, void* y, bool out_bf16, cudaStream_t stream);

// TQ3 for M tokens: the tensor-core kernel when M >= 2 and in <= 8192,
// otherwise one TQ3 GEMV launch per token (no workspace).
int launch_tq3_gemm(const uint8_t* packed, const float* norms, const int8_t* signs, const float* codebook,
                    int64_t O, int in, const uint16_t* X, int64_t ldx, int M, void* Y, int64_t ldy, bool out_bf16,
                    void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (M >= 2 && gemm_tc_takes(in))
    return launch_tc<TcTq3>(packed, norms, codebook, signs, O, in, X, ldx, M, Y, ldy, out_bf16, workspace, ws_bytes,
                            stream);
  const int es = out_bf16 ? 2 : 4;
  for (int m = 0; m < M; ++m)
    if (const int st = launch_tq3_gemv(packed, norms, signs, codebook, O, in, X + static_cast<int64_t>(m) * ldx,
                                       static_cast<char*>(Y) + static_cast<int64_t>(m) * ldy * es, out_bf16, stream))
      return st;
  return HLWQ_OK;
}

}  // namespace hlwq
