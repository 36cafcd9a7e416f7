#pragma once
// Small-M GEMM on the 5th-generation tensor cores (tcgen05 / TMEM / TMA), sm_100a.
//
// Y[m][o] = sum_i X[m][i] w_hat[o][i] for M >= 16 tokens, evaluated in the
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
// Kernel 2 (gemm_tc_kernel): one CTA per 128-row tile of W (and 256-token tile
// of X).  Roles, 320 threads:
//   warps 0-7  decode: each lane owns one weight row of the tile and decodes 32
//              codes of each 64-wide K chunk (code pair -> binary16 centroid
//              pair from a lane-replicated table, times the block scale) and
//              writes them straight into tensor memory with tcgen05.st (the A
//              operand lives in TMEM, so decoding costs no shared-memory
//              bandwidth that the MMA needs for B);
//   warp 8     TMA producer: 64 x N tiles of B, 128-byte swizzled, into a
//              3-4 stage shared-memory ring (no multicast);
//   warp 9     allocates TMEM and issues tcgen05.mma (kind::f16, M = 128,
//              N = tokens, K = 16) into an fp32 accumulator in TMEM;
//   warps 0-3  epilogue: tcgen05.ld of the accumulator, scaling, bf16/fp32 store.
// Stages are handed over with mbarriers; every wait is bounded (2 s), after
// which the kernel raises HLWQ_DEVERR_TIMEOUT, drains and frees TMEM.

#include <cuda.h>
#include <cudaTypedefs.h>

#include "engine.cuh"

namespace hlwq {

namespace {

constexpr int kTcThreads = 320;
constexpr int kTcTileRows = 128;
constexpr int kTcKChunk = 64;                 // K elements per pipeline stage (one half block)
constexpr int kTcAccCols = 256;               // TMEM columns reserved for the accumulator
constexpr int kTcAllocCols = 512;
constexpr uint64_t kTcTimeoutNs = 2000000000ull;

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// Bounded wait for the phase of `parity` to complete; false on timeout.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t deadline) {
  for (;;) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    if (ok) return true;
    if (globaltimer_ns() > deadline) return false;
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

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

// ---------------------------------------------------------------- rotation
constexpr int kRotThreads = 256;

// One CTA per token: B[m][:] = binary16(x_tilde[m][:] * s_m), inv_s[m] = 1 / s_m.
__global__ void __launch_bounds__(kRotThreads)
rotate_x_kernel(const uint16_t* __restrict__ X, int64_t ldx, int in, int nb, uint16_t* __restrict__ B,
                float* __restrict__ inv_s) {
  extern __shared__ __align__(16) float buf[];  // [nb * 128]
  __shared__ float red[kRotThreads / 32];
  const int m = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint16_t* x = X + static_cast<int64_t>(m) * ldx;
  float mx = 0.0f;
  for (int b = warp; b < nb; b += kRotThreads / 32) {
    float e4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = kBlock * b + 4 * lane + k;
      e4[k] = i < in ? bf16_bits_to_float(__ldg(x + i)) : 0.0f;
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
      buf[kBlock * b + 4 * lane + k] = e4[k];
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

// ---------------------------------------------------------------- main kernel
struct TcSmem {
  uint32_t tab;     // pair table (128 KiB)
  uint32_t bstage;  // B stages, each n_box * 128 bytes
  uint32_t bars;    // full_a[S], full_b[S], empty[S], accum, 8 bytes each
  uint32_t misc;    // tmem base (4 B), abort flag (4 B), c16 (64 B)
};

__host__ __device__ inline int tc_stages(int n_box) { return n_box > 128 ? 3 : 4; }

__host__ __device__ inline int tc_smem_bytes(int n_box) {
  return 1024 /*align slack*/ + kPairTabBytes + tc_stages(n_box) * n_box * 128 + 256 + 128;
}

__global__ void __launch_bounds__(kTcThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap bmap, const uint8_t* __restrict__ packed,
               const uint16_t* __restrict__ norms, const float* __restrict__ codebook, int64_t O, int nb, int M,
               const float* __restrict__ inv_s, void* __restrict__ Y, int64_t ldy, int out_bf16, int n_box) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw));
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int S = tc_stages(n_box);
  const uint32_t tab = base;
  const uint32_t bst = base + kPairTabBytes;
  const uint32_t bars = bst + S * n_box * 128;
  const uint32_t misc = bars + 8 * (3 * S + 1);
  uint32_t* tab_g = reinterpret_cast<uint32_t*>(gbase);
  volatile uint32_t* misc_g = reinterpret_cast<volatile uint32_t*>(gbase + (misc - base));
  uint16_t* c16 = reinterpret_cast<uint16_t*>(gbase + (misc - base) + 16);
  auto full_a = [&](int s) { return bars + 8u * s; };
  auto full_b = [&](int s) { return bars + 8u * (S + s); };
  auto empty = [&](int s) { return bars + 8u * (2 * S + s); };
  const uint32_t accum = bars + 8u * (3 * S);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t o0 = static_cast<int64_t>(blockIdx.x) * kTcTileRows;
  const int n0 = blockIdx.y * n_box;
  const int nchunks = 2 * nb;
  const uint64_t deadline = globaltimer_ns() + kTcTimeoutNs;

  // ---- set-up: codebook, barriers, TMEM, pair table
  if (threadIdx.x < kLevels) {
    const float c = __ldg(codebook + threadIdx.x);
    c16[threadIdx.x] = __half_as_ushort(__float2half_rn(c));
    if (threadIdx.x + 1 < kLevels && !(c < __ldg(codebook + threadIdx.x + 1))) raise_device_error(HLWQ_DEVERR_CODEBOOK);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_a(s), 8);
      mbar_init(full_b(s), 1);
      mbar_init(empty(s), 1);
    }
    mbar_init(accum, 1);
    misc_g[1] = 0u;  // abort flag
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(misc), "r"(kTcAllocCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  __syncthreads();
  if (warp < 8) {
    uint4* t4 = reinterpret_cast<uint4*>(tab_g);
    for (int q = threadIdx.x; q < 1024 * 8; q += 256) {
      const int v = q >> 3;
      const uint32_t e = static_cast<uint32_t>(c16[v & 31]) | (static_cast<uint32_t>(c16[v >> 5]) << 16);
      t4[q] = make_uint4(e, e, e, e);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc_g[0];

  if (warp < 8) {
    // ---------------------------------------------------------- decode
    const int q4 = warp & 3, hh = warp >> 2;
    const int r = 32 * q4 + lane;
    const int64_t o = o0 + r;
    const bool row_ok = o < O;
    // per-row power of two so that n * 2^-e <= 1
    float nmax = 0.0f;
    if (row_ok)
      for (int b = 0; b < nb; ++b) nmax = fmaxf(nmax, half_bits_to_float(__ldg(norms + o * nb + b)));
    int erow = 0;
    if (nmax > 0.0f && isfinite(nmax)) frexpf(nmax, &erow);
    const float rs = ldexpf(1.0f, -erow);
    const uint32_t lane_base = tab + 4u * lane;
    const uint32_t tm_row = tmem + (static_cast<uint32_t>(32 * q4) << 16);
    const uint8_t* rowp = packed + (row_ok ? o : 0) * static_cast<int64_t>(nb) * kBlockBytes + 20 * hh;
    const uint16_t* rown = norms + (row_ok ? o : 0) * static_cast<int64_t>(nb);

    constexpr int kD = 4;
    uint32_t cw[kD][5];
    float nsc[kD];
    auto fetch = [&](int i, int d) {
      if (i < nchunks && row_ok) {
        const uint32_t* src = reinterpret_cast<const uint32_t*>(rowp + (i >> 1) * kBlockBytes + 40 * (i & 1));
#pragma unroll
        for (int k = 0; k < 5; ++k) cw[d][k] = __ldg(src + k);
        nsc[d] = half_bits_to_float(__ldg(rown + (i >> 1))) * rs;
      } else {
#pragma unroll
        for (int k = 0; k < 5; ++k) cw[d][k] = 0u;
        nsc[d] = 0.0f;
      }
    };
#pragma unroll
    for (int d = 0; d < kD; ++d) fetch(d, d);
    bool ok = true;
    for (int i0 = 0; i0 < nchunks; i0 += kD) {
#pragma unroll
      for (int d = 0; d < kD; ++d) {
        const int i = i0 + d;
        if (i < nchunks) {
          const int s = i % S;
          const uint32_t h2 = pack_half2(nsc[d], nsc[d]);
          uint32_t v[16];
#pragma unroll
          for (int p = 0; p < 16; ++p) {
            const int bit = 10 * p, wi = bit >> 5, sh = bit & 31;
            const uint32_t lo = cw[d][wi];
            const uint32_t hi = (wi + 1 < 5) ? cw[d][wi + 1] : 0u;
            const uint32_t v10 = (sh <= 22) ? ((lo >> sh) & 0x3ffu) : (__funnelshift_r(lo, hi, sh) & 0x3ffu);
            v[p] = hmul2(lds_u32(lane_base + (v10 << 7)), h2);
          }
          fetch(i + kD, d);
          if (ok) ok = mbar_wait(empty(s), ((i / S) & 1) ^ 1, deadline);
          if (ok && misc_g[1] == 0u) {
            tc_st16(tm_row + kTcAccCols + 32 * s + 16 * hh, v);
            tc_wait_st();
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(full_a(s));
        }
      }
    }
    if (!ok) {
      misc_g[1] = 1u;
      raise_device_error(HLWQ_DEVERR_TIMEOUT);
    }

    // ---------------------------------------------------------- epilogue (warps 0-3)
    if (warp < 4) {
      const bool done = mbar_wait(accum, 0, deadline);
      tc_fence_after();
      if (!done) {
        misc_g[1] = 1u;
        raise_device_error(HLWQ_DEVERR_TIMEOUT);
      }
      const float rscale = ldexpf(1.0f, erow) * (1.0f / 128.0f);
      const bool store = done && misc_g[1] == 0u && row_ok;
      for (int c0 = 0; c0 < n_box; c0 += 16) {
        uint32_t acc[16];
        tc_ld16(tm_row + c0, acc);
        tc_wait_ld();
        if (store) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int m = n0 + c0 + j;
            if (m < M) {
              const float yv = __uint_as_float(acc[j]) * rscale * __ldg(inv_s + m);
              const int64_t off = static_cast<int64_t>(m) * ldy + o;
              if (out_bf16) static_cast<uint16_t*>(Y)[off] = static_cast<uint16_t>(float_to_bf16_bits(yv));
              else static_cast<float*>(Y)[off] = yv;
            }
          }
        }
      }
    }
  } else if (warp == 8) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      const uint32_t bytes = static_cast<uint32_t>(n_box) * 128u;
      for (int i = 0; i < nchunks; ++i) {
        const int s = i % S;
        if (!mbar_wait(empty(s), ((i / S) & 1) ^ 1, deadline) || misc_g[1] != 0u) {
          misc_g[1] = 1u;
          raise_device_error(HLWQ_DEVERR_TIMEOUT);
          break;
        }
        mbar_arrive_expect_tx(full_b(s), bytes);
        tma_load_2d(bst + s * n_box * 128, &bmap, kTcKChunk * i, n0, full_b(s));
      }
    }
  } else {
    // ---------------------------------------------------------- MMA issuer (warp 9)
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(n_box);
      bool ok = true;
      for (int i = 0; i < nchunks && ok; ++i) {
        const int s = i % S;
        const uint32_t par = (i / S) & 1;
        ok = mbar_wait(full_a(s), par, deadline) && mbar_wait(full_b(s), par, deadline) && misc_g[1] == 0u;
        if (!ok) break;
        tc_fence_after();
        const uint64_t bdesc = smem_desc_sw128(bst + s * n_box * 128);
#pragma unroll
        for (int kk = 0; kk < kTcKChunk / 16; ++kk)
          tc_mma_f16(tmem, tmem + kTcAccCols + 32 * s + 8 * kk, bdesc + static_cast<uint64_t>(2 * kk), idesc,
                     (i > 0 || kk > 0) ? 1u : 0u);
        tc_commit(empty(s));
      }
      if (!ok) {
        misc_g[1] = 1u;
        raise_device_error(HLWQ_DEVERR_TIMEOUT);
      }
      tc_commit(accum);  // fires once every MMA issued above has completed
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcAllocCols) : "memory");
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

}  // namespace

size_t gemm_tc_workspace_bytes(int64_t O, int64_t in, int64_t M) {
  (void)O;
  const int64_t nb = ceil_div(in, kBlock);
  const size_t b_bytes = static_cast<size_t>(M) * nb * kBlock * 2;
  return ((b_bytes + 255) & ~static_cast<size_t>(255)) + static_cast<size_t>(M) * 4 + 256;
}

int launch_gemm_tc(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                   const uint16_t* X, int64_t ldx, int M, void* Y, int64_t ldy, bool out_bf16, void* workspace,
                   size_t ws_bytes, cudaStream_t stream) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  if (ws_bytes < gemm_tc_workspace_bytes(O, in, M)) return HLWQ_EWORKSPACE;
  uint16_t* B = static_cast<uint16_t*>(workspace);
  const size_t b_bytes = static_cast<size_t>(M) * nb * kBlock * 2;
  float* inv_s = reinterpret_cast<float*>(static_cast<char*>(workspace) + ((b_bytes + 255) & ~static_cast<size_t>(255)));
  const int rot_smem = nb * kBlock * 4;
  if (rot_smem > 200 * 1024) return HLWQ_EUNSUPPORTED;
  static bool rot_attr = false;
  if (!rot_attr) {
    if (cudaFuncSetAttribute(rotate_x_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) != cudaSuccess)
      return HLWQ_ECUDA;
    rot_attr = true;
  }
  rotate_x_kernel<<<M, kRotThreads, rot_smem, stream>>>(X, ldx, in, nb, B, inv_s);
  if (cudaGetLastError() != cudaSuccess) return HLWQ_ECUDA;

  const int n_box = static_cast<int>(std::min<int64_t>(256, (std::min<int64_t>(M, 256) + 15) / 16 * 16));
  PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode_fn();
  if (!encode) return HLWQ_ECUDA;
  CUtensorMap map;
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(nb) * kBlock, static_cast<cuuint64_t>(M)};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(nb) * kBlock * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTcKChunk), static_cast<cuuint32_t>(n_box)};
  const cuuint32_t estr[2] = {1, 1};
  if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, B, gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return HLWQ_ECUDA;
  const int smem = tc_smem_bytes(n_box);
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess)
      return HLWQ_ECUDA;
    attr = true;
  }
  if (smem > 227 * 1024) return HLWQ_EUNSUPPORTED;
  dim3 grid(static_cast<unsigned>(ceil_div(O, kTcTileRows)), static_cast<unsigned>(ceil_div(M, n_box)));
  gemm_tc_kernel<<<grid, kTcThreads, smem, stream>>>(map, packed, norms, codebook, O, nb, M, inv_s, Y, ldy,
                                                     out_bf16 ? 1 : 0, n_box);
  return cudaGetLastError() == cudaSuccess ? HLWQ_OK : HLWQ_ECUDA;
}

}  // namespace hlwq
