#pragma once
// Fused dequant-matmul for a few tokens (M = 2..8) on the TMA-fed decode
// engine of the single-token GEMV (sm_100a).
//
// Y[m][o] = sum_i X[m][i] w_hat[o][i] ("Qwen3.6-35B-A3B -- HLWQ Q5", Method:
// the rotated-domain product, as in gemv.cuh), MT = 2 or 4 tokens per pass.
// Items, lanes, code ring and pair table are those of gemv1_kernel: a lane
// decodes the same half block of two rows per item, every pair of codes costs
// a shift, an and-or and one shared load per row, and each table entry then
// feeds two fp32-accumulating mixed-precision FMAs per token.  The tokens' rotated activations live in
// shared memory interleaved by token: for (block b, pair pp of the block) the
// MT half2 values sit side by side, so one 8- or 16-byte load gives a lane all
// tokens' values for a pair; each half block's units are padded by one so
// that the lanes of a warp (different blocks and halves, same pair) hit
// different banks.  Each (row, token) accumulates in two fp32 sums (the
// pair's halves); the two rows of a lane are reduced over the
// row's 2C lanes together, per token, and the chunk partials are summed at the
// end in a fixed order (deterministic).

#include "gemv.cuh"

namespace hlwq {

namespace {

// Unit (MT half2 values) of pair pp (0..63) of block b.  Each half block's 32
// units are padded by one, so the lanes of a warp (blocks b, b + 1, ..., both
// halves, same pair) fall in different banks.
__host__ __device__ inline int gm_unit(int b, int pp) { return (2 * b + (pp >> 5)) * 33 + (pp & 31); }

struct GmLayout {
  int ring_off, xs_off, xinv_off, part_off, bar_off, total;
};

__host__ __device__ inline GmLayout gm_layout(int nb, int pass_rows, int nch, int S, int MT) {
  GmLayout L;
  L.ring_off = kPairTabBytes;
  L.xs_off = L.ring_off + kG1Warps * S * kG1ItemBytes;
  L.xinv_off = L.xs_off + round16(nb * 66 * MT * 4);
  L.part_off = L.xinv_off + round16(MT * nb * 4);
  L.bar_off = L.part_off + round16(pass_rows * MT * nch * 4);
  L.total = L.bar_off + kG1Warps * S * 8;
  return L;
}

template <int MT>
struct XVec;
template <>
struct XVec<2> {
  using T = uint2;
  __device__ static void get(const T& v, uint32_t (&o)[2]) { o[0] = v.x; o[1] = v.y; }
};
template <>
struct XVec<4> {
  using T = uint4;
  __device__ static void get(const T& v, uint32_t (&o)[4]) { o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w; }
};

// Pair P of both rows against all tokens: every binary16 product is added to
// an fp32 accumulator (two per row and token: the pair's halves).
template <int MT, int P>
__device__ __forceinline__ void gm_pair(const uint8_t* tab, const uint2 (&cw0)[5], const uint2 (&cw1)[5],
                                        uint32_t lane4, const typename XVec<MT>::T* xrow,
                                        float (&h0)[MT][2], float (&h1)[MT][2]) {
  const uint32_t e0 = *reinterpret_cast<const uint32_t*>(tab + g1_off<P>(cw0, lane4));
  const uint32_t e1 = *reinterpret_cast<const uint32_t*>(tab + g1_off<P>(cw1, lane4));
  uint32_t x[MT];
  XVec<MT>::get(xrow[P], x);
#pragma unroll
  for (int t = 0; t < MT; ++t) {
    h0[t][0] = fma_lo(e0, x[t], h0[t][0]);
    h0[t][1] = fma_hi(e0, x[t], h0[t][1]);
    h1[t][0] = fma_lo(e1, x[t], h1[t][0]);
    h1[t][1] = fma_hi(e1, x[t], h1[t][1]);
  }
}

template <int MT, int... P>
__device__ __forceinline__ void gm_dot(const uint8_t* tab, const uint2 (&cw0)[5], const uint2 (&cw1)[5],
                                       uint32_t lane4, const typename XVec<MT>::T* xrow, float (&a0)[MT],
                                       float (&a1)[MT], std::integer_sequence<int, P...>) {
  float h0[MT][2], h1[MT][2];
#pragma unroll
  for (int t = 0; t < MT; ++t) h0[t][0] = h0[t][1] = h1[t][0] = h1[t][1] = 0.0f;
  (gm_pair<MT, P>(tab, cw0, cw1, lane4, xrow, h0, h1), ...);
#pragma unroll
  for (int t = 0; t < MT; ++t) {
    a0[t] = h0[t][0] + h0[t][1];
    a1[t] = h1[t][0] + h1[t][1];
  }
}

// Rotation of token t's block b into the interleaved layout (8 lanes per block).
template <int MT>
__device__ __forceinline__ void gm_rot_store(const uint32_t (&w)[8], int nb, int nblocks, int gb0, uint32_t* xs32,
                                             float* xinv) {
  float v[16];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    v[2 * k] = __uint_as_float(w[k] << 16);
    v[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
  }
  const RotBlock B = g1_rot_block(nb, nblocks, gb0);  // vec = token, b = block
  const int q = threadIdx.x & 7;
  const int k = g1_rot_compute(v);
  const float sc = ldexpf(1.0f, k);
  if (B.act) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      xs32[gm_unit(B.b, 8 * q + j) * MT + B.vec] = pack_half2(v[2 * j] * sc, v[2 * j + 1] * sc);
    if (q == 0) xinv[B.vec * nb + B.b] = ldexpf(1.0f, -k);
  }
}

template <int C, int S, int MT>
__global__ void __launch_bounds__(kG1Threads, 1)
gemvm_kernel(const __grid_constant__ CUtensorMap cmap, const uint16_t* __restrict__ norms,
             const float* __restrict__ codebook, int64_t O, int in, int nb, const uint16_t* __restrict__ X,
             int64_t ldx, int ntok, void* __restrict__ Y, int64_t ldy, int out_bf16, int pass_rows, int xvec) {
  extern __shared__ __align__(16) uint8_t smem[];
  using XV = typename XVec<MT>::T;
  constexpr int L2C = 2 * C;   // lanes per row
  constexpr int G = 32 / L2C;  // rows of one half item
  constexpr int RG = 2 * G;    // rows per item
  const int nch = (nb + C - 1) / C;
  const GmLayout L = gm_layout(nb, pass_rows, nch, S, MT);
  uint32_t* xs32 = reinterpret_cast<uint32_t*>(smem + L.xs_off);
  const XV* xsv = reinterpret_cast<const XV*>(smem + L.xs_off);
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
  uint32_t phase = 0, pending = 0;

  for (int p0 = 0; p0 < nrows; p0 += pass_rows) {
    const int prow = min(pass_rows, nrows - p0);
    const int ngr = (prow + RG - 1) / RG;
    const int nitems = ngr * nch;
    const int it0 = warp * nitems / kG1Warps, it1 = (warp + 1) * nitems / kG1Warps;
    const int nw = it1 - it0;
    const int64_t prow0 = row0 + p0;

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
    if (p0 > 0 && lane == 0) fence_proxy_async();  // the previous pass's reads of the slots precede the refills
#pragma unroll
    for (int d = 0; d < S; ++d)
      if (ok && d < nw) issue(d);

    if (p0 == 0) {
      // pair table before the dependency wait; the tokens' activations after it
      const uint32_t c16r = g1_codebook_lane(codebook);
      g1_build_table(smem, c16r, 0, kG1Warps);
      pdl_wait();
      const int nblk = MT * nb;  // tokens beyond ntok are rotated as zeros
      for (int gb0 = 4 * warp; gb0 < nblk; gb0 += 4 * kG1Warps) {
        uint32_t xw[8];
        g1_rot_load(X, ldx, in, nb, ntok * nb, xvec != 0, gb0, xw);
        gm_rot_store<MT>(xw, nb, nblk, gb0, xs32, xinv);
      }
      __syncthreads();
      pdl_trigger();
    }

    int cch = it0 / ngr, cg = it0 - (it0 / ngr) * ngr, xch = -1;
    const XV* xrow = xsv;
    float xi[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) xi[t] = 0.0f;
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
            cw1[q] = src[q + kG1ItemBytes / 16];
          }
          __syncwarp();
          if (ok && k + S < nw) {
            if (lane == 0) fence_proxy_async();
            issue(d);
          }
          if (cch != xch) {
            xch = cch;
            const int b = cch * C + s;
            const bool bv = b < nb;
            xrow = xsv + (bv ? (2 * b + hh) * 33 : 0);  // a block past the end reads block 0 and weighs it 0
#pragma unroll
            for (int t = 0; t < MT; ++t) xi[t] = bv ? xinv[t * nb + b] * (1.0f / 128.0f) : 0.0f;
          }
          float a0[MT], a1[MT];
          gm_dot<MT>(smem, cw0, cw1, lane4, xrow, a0, a1, std::make_integer_sequence<int, 32>{});
          const float n0f = half_bits_to_float(static_cast<uint16_t>(nr0));
          const float n1f = half_bits_to_float(static_cast<uint16_t>(nr1));
          const bool hi = (u & C) != 0;
          const int v = cg * RG + r + (hi ? G : 0);
#pragma unroll
          for (int t = 0; t < MT; ++t) {
            const float b0 = a0[t] * (n0f * xi[t]), b1 = a1[t] * (n1f * xi[t]);
            float acc = (hi ? b1 : b0) + __shfl_xor_sync(0xffffffffu, hi ? b0 : b1, C);
#pragma unroll
            for (int off = C / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if ((u & (C - 1)) == 0 && v < prow) part[(v * MT + t) * nch + cch] = acc;
          }
          if (++cg == ngr) { cg = 0; ++cch; }
        }
      }
    }
    if (!ok) {
      const uint64_t dl = globaltimer_ns() + wait_limit_ns();
      for (int d = 0; d < S; ++d)
        if ((pending >> d) & 1u) mbar_wait(bar + 8 * d, (phase >> d) & 1u, dl);
      pending = 0;
      if (lane == 0) raise_device_error(HLWQ_DEVERR_TIMEOUT);
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < prow * ntok; idx += kG1Threads) {
      const int t = idx / prow, v = idx - t * prow;
      const float* pv = part + (v * MT + t) * nch;
      float sum = 0.0f;
      for (int ch = 0; ch < nch; ++ch) sum += pv[ch];
      const int64_t off = static_cast<int64_t>(t) * ldy + prow0 + v;
      if (out_bf16) static_cast<uint16_t*>(Y)[off] = static_cast<uint16_t>(float_to_bf16_bits(sum));
      else static_cast<float*>(Y)[off] = sum;
    }
    __syncthreads();
    if (__syncthreads_or(!ok)) break;
  }
}

template <int C, int S, int MT>
int launch_gemvm_cs(const CUtensorMap& map, const uint16_t* norms, const float* codebook, int64_t O, int in, int nb,
                    const uint16_t* X, int64_t ldx, int ntok, void* Y, int64_t ldy, bool out_bf16, int grid,
                    int pass_rows, cudaStream_t stream) {
  const GmLayout L = gm_layout(nb, pass_rows, (nb + C - 1) / C, S, MT);
  static PerDeviceOnce attr_set;
  if (const int st = attr_set([&] {
        return cudaFuncSetAttribute(gemvm_kernel<C, S, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    227 * 1024) == cudaSuccess;
      }))
    return st;
  const int xvec = (reinterpret_cast<uintptr_t>(X) % 16 == 0 && in % 8 == 0 && ldx % 8 == 0) ? 1 : 0;
  gemvm_kernel<C, S, MT><<<grid, kG1Threads, L.total, stream>>>(map, norms, codebook, O, in, nb, X, ldx, ntok, Y, ldy,
                                                                out_bf16 ? 1 : 0, pass_rows, xvec);
  return cudaGetLastError() == cudaSuccess ? HLWQ_OK : HLWQ_ECUDA;
}

template <int C, int MT>
int launch_gemvm_c(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                   const uint16_t* X, int64_t ldx, int ntok, void* Y, int64_t ldy, bool out_bf16,
                   cudaStream_t stream) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  const int nch = (nb + C - 1) / C;
  constexpr int RG = 32 / C;
  const int64_t ngroups = ceil_div(O, RG);
  const int grid = static_cast<int>(std::min<int64_t>(sm_count(), ngroups));
  const int rows_cta = static_cast<int>(ceil_div(ngroups, grid) * RG);
  CUtensorMap map;
  const int st = codes_map(packed, O, nb, C, RG, &map);
  if (st != HLWQ_OK) return st;
  for (int S : {2, 1}) {
    const int fixed = gm_layout(nb, 0, nch, S, MT).total;
    const int cap = (227 * 1024 - fixed - 16) / (MT * nch * 4) / RG * RG;
    if (cap < RG) continue;
    const int pr = std::min(rows_cta, cap);
    return S == 2 ? launch_gemvm_cs<C, 2, MT>(map, norms, codebook, O, in, nb, X, ldx, ntok, Y, ldy, out_bf16, grid,
                                              pr, stream)
                  : launch_gemvm_cs<C, 1, MT>(map, norms, codebook, O, in, nb, X, ldx, ntok, Y, ldy, out_bf16, grid,
                                              pr, stream);
  }
  return HLWQ_EUNSUPPORTED;
}

template <int MT>
int launch_gemvm_mt(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                    const uint16_t* X, int64_t ldx, int ntok, void* Y, int64_t ldy, bool out_bf16,
                    cudaStream_t stream) {
  switch (pick_chunk(static_cast<int>(ceil_div(in, kBlock)))) {
    case 8: return launch_gemvm_c<8, MT>(packed, norms, codebook, O, in, X, ldx, ntok, Y, ldy, out_bf16, stream);
    case 4: return launch_gemvm_c<4, MT>(packed, norms, codebook, O, in, X, ldx, ntok, Y, ldy, out_bf16, stream);
    default: return launch_gemvm_c<2, MT>(packed, norms, codebook, O, in, X, ldx, ntok, Y, ldy, out_bf16, stream);
  }
}

}  // namespace

// M = 2..8 tokens: groups of four (two for a remainder of one or two), one
// launch per group; each launch streams the weights once.
int launch_gemvm(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                 const uint16_t* X, int64_t ldx, int M, void* Y, int64_t ldy, bool out_bf16, cudaStream_t stream) {
  const size_t esz = out_bf16 ? 2 : 4;
  for (int m0 = 0; m0 < M; m0 += 4) {
    const int n = std::min(4, M - m0);
    const uint16_t* Xg = X + static_cast<int64_t>(m0) * ldx;
    void* Yg = static_cast<char*>(Y) + static_cast<size_t>(m0) * ldy * esz;
    const int st = n > 2 ? launch_gemvm_mt<4>(packed, norms, codebook, O, in, Xg, ldx, n, Yg, ldy, out_bf16, stream)
                         : launch_gemvm_mt<2>(packed, norms, codebook, O, in, Xg, ldx, n, Yg, ldy, out_bf16, stream);
    if (st != HLWQ_OK) return st;
  }
  return HLWQ_OK;
}

}  // namespace hlwq
