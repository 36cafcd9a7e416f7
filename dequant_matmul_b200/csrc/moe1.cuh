#pragma once
// Routed MoE layer for few tokens on the TMA-fed decode engine of the
// single-token GEMV (sm_100a).
//
// Same computation as moe.cuh ("Qwen3.6-35B-A3B -- HLWQ Q5": 8 routed + 1
// shared expert per token; each expert quantized independently), as two
// kernels over (token, expert slot) pairs p = t * KP + s (KP = k routed slots,
// plus the shared expert last when present):
//
//   moe_gu1_kernel  every CTA routes all tokens itself (top-k + softmax of the
//                   logits, the routine of the router kernel), rotates the
//                   tokens' activations, and decodes a balanced range of
//                   (pair, group of G intermediate columns) x chunk items: one
//                   item carries gate rows j .. j + G - 1 and up rows F + j ..
//                   in the two halves of a TMA slot, so a lane's two rows are
//                   gate and up of the same column; the epilogue writes
//                   h[p][j] = SiLU(g) * u (fp32).
//   moe_dn1_kernel  every CTA routes the tokens again (same result), owns a
//                   balanced range of output-row groups for all pairs, issues
//                   its first down-projection boxes and builds the pair table
//                   before griddepcontrol.wait (launched with programmatic
//                   stream serialisation after moe_gu1_kernel, whose output h
//                   it reads only after the wait), rotates h of every pair
//                   and decodes; the epilogue forms
//                   Y[t][i] = sum_s p_ts * (W_dn[e_ts] h_ts)[i] in a fixed
//                   order (the shared expert with weight 1).
//
// Each pair streams its expert's codes once; for few tokens the pairs are
// almost always distinct experts, so this is the layer's distinct-expert
// traffic.  No atomics; deterministic.

#include "gemv.cuh"
#include "moe.cuh"

namespace hlwq {

namespace {

struct Moe1Params {
  const float* logits;  // [T][E]
  const uint16_t* X;    // [T][H] bf16
  const uint16_t* gu_norms;
  const uint16_t* sh_gu_norms;
  const uint16_t* dn_norms;
  const uint16_t* sh_dn_norms;
  const float* codebook;
  float* h;  // [NP][F]
  int32_t* ids_out;
  float* w_out;
  void* Y;
  int E, H, F, T, topk, has_shared, out_bf16;
};

struct Moe1Layout {
  int ring_off, xs_off, xinv_off, part_off, c16_off, rid_off, rw_off, bar_off, total;
};

// nvec activation vectors of nb blocks; part_floats partial sums; np pairs.
__host__ __device__ inline Moe1Layout moe1_layout(int S, int nvec, int nb, int part_floats, int np) {
  Moe1Layout L;
  L.ring_off = kPairTabBytes;
  L.xs_off = L.ring_off + kG1Warps * S * kG1ItemBytes;
  L.xinv_off = L.xs_off + nvec * nb * kG1XsBytes;
  L.part_off = L.xinv_off + round16(nvec * nb * 4);
  L.c16_off = L.part_off + round16(part_floats * 4);
  L.rid_off = L.c16_off + 64;
  L.rw_off = L.rid_off + round16(np * 4);
  L.bar_off = L.rw_off + round16(np * 4);
  L.total = L.bar_off + kG1Warps * S * 8;
  return L;
}

// Routes tokens t_lo .. t_hi into rid / rw: pair t * KP + s holds the expert
// id (E = the shared expert) and weight.  Warps 0 .. min(count, 15) - 1 route
// (t = t_lo + warp, + that count, ...); the other warps return at once.
__device__ __forceinline__ void moe1_route(const Moe1Params& P, int* rid, float* rw, bool write_out, int t_lo,
                                           int t_hi) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KP = P.topk + P.has_shared;
  const int nroute = min(t_hi - t_lo + 1, kG1Warps - 1);
  if (warp >= nroute) return;
  for (int t = t_lo + warp; t <= t_hi; t += nroute) {
    route_token_warp(P.logits + static_cast<int64_t>(t) * P.E, P.E, P.topk, rid + t * KP, rw + t * KP);
    if (lane == 0 && P.has_shared) {
      rid[t * KP + P.topk] = P.E;
      rw[t * KP + P.topk] = 1.0f;
    }
    if (write_out && lane < P.topk) {
      if (P.ids_out) P.ids_out[t * P.topk + lane] = rid[t * KP + lane];
      if (P.w_out) P.w_out[t * P.topk + lane] = rw[t * KP + lane];
    }
  }
}

// Reloads a lane's 64 rotated activations (block gb, half hh) into registers.
__device__ __forceinline__ void moe1_load_x(const uint16_t* xs, const float* xinv, int gb, bool valid, int hh,
                                            uint32_t (&xr)[32], float& xi) {
  if (valid) {
    const uint4* xsrc = reinterpret_cast<const uint4*>(xs);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint4 w = xsrc[g1_xs_chunk(gb, 8 * hh + q)];
      xr[4 * q] = w.x; xr[4 * q + 1] = w.y; xr[4 * q + 2] = w.z; xr[4 * q + 3] = w.w;
    }
    xi = xinv[gb] * (1.0f / 128.0f);
  } else {
#pragma unroll
    for (int q = 0; q < 32; ++q) xr[q] = 0u;
    xi = 0.0f;
  }
}

// ----------------------------------------------------------------- gate_up
template <int C, int S>
__global__ void __launch_bounds__(kG1Threads, 1)
moe_gu1_kernel(const __grid_constant__ CUtensorMap gmap, const __grid_constant__ CUtensorMap smap, Moe1Params P,
               int part_rows, int tok_max) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int L2C = 2 * C, G = 32 / L2C;
  const int nb = (P.H + kBlock - 1) / kBlock, nch = (nb + C - 1) / C;
  const int KP = P.topk + P.has_shared, NP = P.T * KP;
  const int F = P.F, F2 = 2 * P.F;
  const int ngj = (F + G - 1) / G;  // column groups per pair
  const int nq_all = NP * ngj;
  const int q0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * nq_all / gridDim.x);
  const int q1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * nq_all / gridDim.x);
  const int nq = q1 - q0;
  // the tokens this CTA's pairs belong to (its range is contiguous in pairs)
  const int t_lo = nq > 0 ? (q0 / ngj) / KP : 0, t_hi = nq > 0 ? ((q1 - 1) / ngj) / KP : 0;
  const int ntok = t_hi - t_lo + 1;
  const Moe1Layout L = moe1_layout(S, tok_max, nb, part_rows * nch * 2, NP);
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + L.xs_off);
  float* xinv = reinterpret_cast<float*>(smem + L.xinv_off);
  float* part = reinterpret_cast<float*>(smem + L.part_off);  // [nq * G][nch][2] (gate, up)
  int* rid = reinterpret_cast<int*>(smem + L.rid_off);
  float* rw = reinterpret_cast<float*>(smem + L.rw_off);
  const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = lane / L2C, u = lane % L2C, s = u >> 1, hh = u & 1;
  const uint32_t lane4 = static_cast<uint32_t>(lane) << 2;
  const uint32_t ring = sbase + L.ring_off + warp * (S * kG1ItemBytes);
  const uint32_t bar = sbase + L.bar_off + warp * (S * 8);
  const uint8_t* my_codes = smem + L.ring_off + warp * (S * kG1ItemBytes) + 40 * lane;

  const uint32_t c16r = g1_codebook_lane(P.codebook);
  if (lane == 0) {
#pragma unroll
    for (int d = 0; d < S; ++d) mbar_init(bar + 8 * d, 1);
    fence_barrier_init();
  }
  // the tokens' activations are loaded now and rotated once the boxes are on
  // their way; the routing warps run while the other warps build the table
  const int nblk = ntok * nb;
  const uint16_t* Xc = P.X + static_cast<int64_t>(t_lo) * P.H;
  const bool xvec = (reinterpret_cast<uintptr_t>(P.X) % 16 == 0) && (P.H % 8 == 0);
  uint32_t xw[8];
  if (4 * warp < nblk) g1_rot_load(Xc, P.H, P.H, nb, nblk, xvec, 4 * warp, xw);
  const int nroute = min(ntok, kG1Warps - 1);
  moe1_route(P, rid, rw, true, t_lo, t_hi);  // CTAs sharing a token write the same ids / weights
  g1_build_table(smem, c16r, nroute, kG1Warps - nroute);
  __syncthreads();  // routing, table, barriers

  const uint64_t deadline = globaltimer_ns() + wait_limit_ns();
  bool ok = true;
  uint32_t phase = 0, pending = 0;
  const int nitems = nq * nch;  // chunk-major: item k = (chunk k / nq, group q0 + k % nq)
  const int it0 = warp * nitems / kG1Warps, it1 = (warp + 1) * nitems / kG1Warps;
  const int nw = it1 - it0;
  int ich = nq ? it0 / nq : 0, iq = it0 - ich * nq;
  uint32_t nlo[S], nhi[S];  // the two rows' norms, kept apart so that no instruction waits on them before use
  auto issue = [&](int d) {
    const int q = q0 + iq, p = q / ngj, j0 = (q - p * ngj) * G;
    const int e = rid[p];
    const bool sh = e == P.E;
    const int64_t rbase = sh ? 0 : static_cast<int64_t>(e) * F2;
    if (lane == 0 && !fault_skip_tma()) {
      mbar_arrive_expect_tx(bar + 8 * d, kG1ItemBytes);
      const CUtensorMap* m = sh ? &smap : &gmap;
      tma_load_3d(ring + d * kG1ItemBytes, m, 0, ich * C, static_cast<int>(rbase + j0), bar + 8 * d);
      tma_load_3d(ring + d * kG1ItemBytes + kG1ItemBytes / 2, m, 0, ich * C, static_cast<int>(rbase + F + j0),
                  bar + 8 * d);
    }
    const int j = j0 + r, b = ich * C + s;
    const uint16_t* nm = sh ? P.sh_gu_norms : P.gu_norms;
    const bool v = j < F && b < nb;
    uint32_t n0 = 0u;
    if (v) n0 = __ldg(nm + (rbase + j) * nb + b);
    uint32_t n1 = 0u;
    if (v) n1 = __ldg(nm + (rbase + F + j) * nb + b);
    nlo[d] = n0;
    nhi[d] = n1;
    pending |= 1u << d;
    if (++iq == nq) { iq = 0; ++ich; }
  };
#pragma unroll
  for (int d = 0; d < S; ++d)
    if (d < nw) issue(d);

  if (4 * warp < nblk) g1_rot_store(xw, nb, nblk, 4 * warp, xs, xinv);
  for (int gb0 = 4 * warp + 4 * kG1Warps; gb0 < nblk; gb0 += 4 * kG1Warps) {
    g1_rot_load(Xc, P.H, P.H, nb, nblk, xvec, gb0, xw);
    g1_rot_store(xw, nb, nblk, gb0, xs, xinv);
  }
  __syncthreads();
  pdl_trigger();

  int cch = nq ? it0 / nq : 0, cq = it0 - cch * nq, xkey = -1;
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
          cw1[q] = src[q + kG1ItemBytes / 16];
        }
        __syncwarp();
        if (ok && k + S < nw) {
          if (lane == 0) fence_proxy_async();
          issue(d);
        }
        const int q = q0 + cq, p = q / ngj, t = p / KP;
        const int key = t * nch + cch;
        if (key != xkey) {
          xkey = key;
          const int b = cch * C + s;
          moe1_load_x(xs, xinv, (t - t_lo) * nb + b, b < nb, hh, xr, xi);
        }
        const float a0 = g1_dot(smem, cw0, lane4, xr, std::make_integer_sequence<int, 32>{}) *
                         (half_bits_to_float(static_cast<uint16_t>(nr0)) * xi);
        const float a1 = g1_dot(smem, cw1, lane4, xr, std::make_integer_sequence<int, 32>{}) *
                         (half_bits_to_float(static_cast<uint16_t>(nr1)) * xi);
        const bool hi = (u & C) != 0;
        float acc = (hi ? a1 : a0) + __shfl_xor_sync(0xffffffffu, hi ? a0 : a1, C);
#pragma unroll
        for (int off = C / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if ((u & (C - 1)) == 0) part[((cq * G + r) * nch + cch) * 2 + (hi ? 1 : 0)] = acc;
        if (++cq == nq) { cq = 0; ++cch; }
      }
    }
  }
  if (!ok) {
    const uint64_t dl = globaltimer_ns() + wait_limit_ns();
    for (int d = 0; d < S; ++d)
      if ((pending >> d) & 1u) mbar_wait(bar + 8 * d, (phase >> d) & 1u, dl);
    if (lane == 0) raise_device_error(HLWQ_DEVERR_TIMEOUT);
  }
  __syncthreads();
  for (int v = threadIdx.x; v < nq * G; v += kG1Threads) {
    const int q = q0 + v / G, p = q / ngj, j = (q - p * ngj) * G + v % G;
    if (j >= F) continue;
    const float* pv = part + v * nch * 2;
    float g = 0.0f, up = 0.0f;
    for (int ch = 0; ch < nch; ++ch) {
      g += pv[2 * ch];
      up += pv[2 * ch + 1];
    }
    P.h[static_cast<int64_t>(p) * F + j] = g / (1.0f + expf(-g)) * up;
  }
}

// -------------------------------------------------------------------- down
// The pairs are taken in groups of at most pg_max whose rotated h fit in
// shared memory; every pair's partial sums stay in shared memory until the
// fixed-order combine at the end.
template <int C, int S>
__global__ void __launch_bounds__(kG1Threads, 1)
moe_dn1_kernel(const __grid_constant__ CUtensorMap dmap, const __grid_constant__ CUtensorMap smap, Moe1Params P,
               int rows_max, int pg_max) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int L2C = 2 * C, G = 32 / L2C, RG = 2 * G;
  const int H = P.H, F = P.F;
  const int nb = (F + kBlock - 1) / kBlock, nch = (nb + C - 1) / C;
  const int KP = P.topk + P.has_shared, NP = P.T * KP;
  const int ngr_all = (H + RG - 1) / RG;
  const int g0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * ngr_all / gridDim.x);
  const int g1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * ngr_all / gridDim.x);
  const int ngr = g1 - g0, row0 = g0 * RG, nr = min(g1 * RG, H) - row0;
  const Moe1Layout L = moe1_layout(S, pg_max, nb, NP * rows_max * nch, NP);
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + L.xs_off);
  float* xinv = reinterpret_cast<float*>(smem + L.xinv_off);
  float* part = reinterpret_cast<float*>(smem + L.part_off);  // [NP][rows_max][nch]
  int* rid = reinterpret_cast<int*>(smem + L.rid_off);
  float* rw = reinterpret_cast<float*>(smem + L.rw_off);
  const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = lane / L2C, u = lane % L2C, s = u >> 1, hh = u & 1;
  const uint32_t lane4 = static_cast<uint32_t>(lane) << 2;
  const uint32_t ring = sbase + L.ring_off + warp * (S * kG1ItemBytes);
  const uint32_t bar = sbase + L.bar_off + warp * (S * 8);
  const uint8_t* my_codes = smem + L.ring_off + warp * (S * kG1ItemBytes) + 40 * lane;

  // Before the dependency wait: only the logits, the codebook and the down
  // weights are read (written before the gate_up kernel started).
  const uint32_t c16r = g1_codebook_lane(P.codebook);
  if (lane == 0) {
#pragma unroll
    for (int d = 0; d < S; ++d) mbar_init(bar + 8 * d, 1);
    fence_barrier_init();
  }
  const int nroute = min(P.T, kG1Warps - 1);
  moe1_route(P, rid, rw, false, 0, P.T - 1);
  g1_build_table(smem, c16r, nroute, kG1Warps - nroute);
  __syncthreads();  // routing, table, barriers

  const uint64_t deadline = globaltimer_ns() + wait_limit_ns();
  bool ok = true;
  uint32_t phase = 0, pending = 0;
  for (int pg0 = 0; pg0 < NP; pg0 += pg_max) {
    const int npg = min(pg_max, NP - pg0);
    const int nitems = npg * nch * ngr;  // item k = (pair, chunk, row group), row group fastest
    const int it0 = warp * nitems / kG1Warps, it1 = (warp + 1) * nitems / kG1Warps;
    const int nw = it1 - it0;
    int ilg = it0 % ngr, ich = (it0 / ngr) % nch, ip = pg0 + it0 / (ngr * nch);
    uint32_t nlo[S], nhi[S];  // the two rows' norms, kept apart so that no instruction waits on them before use
    auto issue = [&](int d) {
      const int e = rid[ip];
      const bool sh = e == P.E;
      const int64_t rbase = sh ? 0 : static_cast<int64_t>(e) * H;
      const int lrow = (g0 + ilg) * RG;  // first output row of the item
      if (lane == 0 && !fault_skip_tma()) {
        mbar_arrive_expect_tx(bar + 8 * d, kG1ItemBytes);
        tma_load_3d(ring + d * kG1ItemBytes, sh ? &smap : &dmap, 0, ich * C, static_cast<int>(rbase + lrow),
                    bar + 8 * d);
      }
      const int b = ich * C + s;
      const uint16_t* nm = (sh ? P.sh_dn_norms : P.dn_norms) + (rbase + lrow + r) * nb + b;
      uint32_t n0 = 0u;
      if (b < nb && lrow + r < H) n0 = __ldg(nm);
      uint32_t n1 = 0u;
      if (b < nb && lrow + r + G < H) n1 = __ldg(nm + G * nb);
      nlo[d] = n0;
      nhi[d] = n1;
      pending |= 1u << d;
      if (++ilg == ngr) {
        ilg = 0;
        if (++ich == nch) { ich = 0; ++ip; }
      }
    };
    if (lane == 0) fence_proxy_async();  // the previous group's reads of the slots precede the refills
#pragma unroll
    for (int d = 0; d < S; ++d)
      if (ok && d < nw) issue(d);

    if (pg0 == 0) pdl_wait();  // h is written by the gate_up kernel
    const int nblk = npg * nb;
    for (int gb0 = 4 * warp; gb0 < nblk; gb0 += 4 * kG1Warps)
      g1_rot_f32(P.h + static_cast<int64_t>(pg0) * F, F, F, nb, nblk, gb0, xs, xinv);
    __syncthreads();
    if (pg0 == 0) pdl_trigger();

    int clg = it0 % ngr, cch = (it0 / ngr) % nch, cp = pg0 + it0 / (ngr * nch), xkey = -1;
    uint32_t xr[32];
    float xi = 0.0f;
    for (int base = 0; base < nw; base += S) {
#pragma unroll
      for (int d = 0; d < S; ++d) {
        const int k = base + d;
        if (k < nw) {
          const uint32_t nq0 = nlo[d], nq1 = nhi[d];
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
          const int key = cp * nch + cch;
          if (key != xkey) {
            xkey = key;
            const int b = cch * C + s;
            moe1_load_x(xs, xinv, (cp - pg0) * nb + b, b < nb, hh, xr, xi);
          }
          const float a0 = g1_dot(smem, cw0, lane4, xr, std::make_integer_sequence<int, 32>{}) *
                           (half_bits_to_float(static_cast<uint16_t>(nq0)) * xi);
          const float a1 = g1_dot(smem, cw1, lane4, xr, std::make_integer_sequence<int, 32>{}) *
                           (half_bits_to_float(static_cast<uint16_t>(nq1)) * xi);
          const bool hi = (u & C) != 0;
          float acc = (hi ? a1 : a0) + __shfl_xor_sync(0xffffffffu, hi ? a0 : a1, C);
#pragma unroll
          for (int off = C / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
          if ((u & (C - 1)) == 0) part[(cp * rows_max + clg * RG + r + (hi ? G : 0)) * nch + cch] = acc;
          if (++clg == ngr) {
            clg = 0;
            if (++cch == nch) { cch = 0; ++cp; }
          }
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
    __syncthreads();  // the next group overwrites the rotated h
  }
  for (int idx = threadIdx.x; idx < P.T * nr; idx += kG1Threads) {
    const int t = idx / nr, i = idx - t * nr;
    float y = 0.0f;
    for (int sl = 0; sl < KP; ++sl) {
      const int p = t * KP + sl;
      const float* pv = part + (p * rows_max + i) * nch;
      float z = 0.0f;
      for (int ch = 0; ch < nch; ++ch) z += pv[ch];
      y += rw[p] * z;
    }
    const int64_t off = static_cast<int64_t>(t) * H + row0 + i;
    if (P.out_bf16) static_cast<uint16_t*>(P.Y)[off] = static_cast<uint16_t>(float_to_bf16_bits(y));
    else static_cast<float*>(P.Y)[off] = y;
  }
}

// ------------------------------------------------------------------- host
template <typename K>
bool moe1_attr(K kernel) {
  static_assert(sizeof(K) > 0, "");
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) == cudaSuccess;
}

template <int C, int S>
int moe1_launch_gu(const CUtensorMap& gm, const CUtensorMap& sm, const Moe1Params& P, int grid, int part_rows,
                   int tok_max, int smem, cudaStream_t stream) {
  static PerDeviceOnce attr;
  if (const int st = attr([&] {
        return moe1_attr(moe_gu1_kernel<C, S>);
      }))
    return st;
  moe_gu1_kernel<C, S><<<grid, kG1Threads, smem, stream>>>(gm, sm, P, part_rows, tok_max);
  return cudaGetLastError() == cudaSuccess ? HLWQ_OK : HLWQ_ECUDA;
}

template <int C, int S>
int moe1_launch_dn(const CUtensorMap& dm, const CUtensorMap& sm, const Moe1Params& P, int grid, int rows_max,
                   int pg_max, int smem, cudaStream_t stream) {
  static PerDeviceOnce attr;
  if (const int st = attr([&] {
        return moe1_attr(moe_dn1_kernel<C, S>);
      }))
    return st;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kG1Threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, moe_dn1_kernel<C, S>, dm, sm, P, rows_max, pg_max) == cudaSuccess ? HLWQ_OK
                                                                                              : HLWQ_ECUDA;
}

template <int C>
int moe1_gu_c(int S, const CUtensorMap& gm, const CUtensorMap& sm, const Moe1Params& P, int grid, int part_rows,
              int tok_max, int smem, cudaStream_t stream) {
  return S == 2 ? moe1_launch_gu<C, 2>(gm, sm, P, grid, part_rows, tok_max, smem, stream)
                : moe1_launch_gu<C, 1>(gm, sm, P, grid, part_rows, tok_max, smem, stream);
}

template <int C>
int moe1_dn_c(int S, const CUtensorMap& dm, const CUtensorMap& sm, const Moe1Params& P, int grid, int rows_max,
              int pg_max, int smem, cudaStream_t stream) {
  return S == 2 ? moe1_launch_dn<C, 2>(dm, sm, P, grid, rows_max, pg_max, smem, stream)
                : moe1_launch_dn<C, 1>(dm, sm, P, grid, rows_max, pg_max, smem, stream);
}

}  // namespace

// Few-token MoE path.  Returns HLWQ_EUNSUPPORTED (nothing launched) when the
// pairs' activations do not fit beside the table and a code ring.
int launch_moe1(const uint8_t* gu_packed, const uint16_t* gu_norms, const uint8_t* dn_packed,
                const uint16_t* dn_norms, const uint8_t* sh_gu_packed, const uint16_t* sh_gu_norms,
                const uint8_t* sh_dn_packed, const uint16_t* sh_dn_norms, const float* codebook, int E, int H, int F,
                int topk, int T, const float* logits, const uint16_t* X, void* Y, bool out_bf16, int32_t* ids_out,
                float* w_out, float* h_ws, cudaStream_t stream) {
  const bool shared = sh_gu_packed != nullptr;
  const int KP = topk + (shared ? 1 : 0), NP = T * KP;
  const int nbh = static_cast<int>(ceil_div(H, kBlock)), nbf = static_cast<int>(ceil_div(F, kBlock));
  const int cg = pick_chunk(nbh), cd = pick_chunk(nbf);
  const int Gg = 16 / cg, RGd = 32 / cd;
  const int nchg = (nbh + cg - 1) / cg, nchd = (nbf + cd - 1) / cd;
  const int sms = sm_count();
  // gate_up: groups of Gg columns per pair
  const int64_t ngj = ceil_div(F, Gg);
  const int64_t nq_all = static_cast<int64_t>(NP) * ngj;
  // one CTA per SM when its partial sums fit; otherwise more CTAs (in waves),
  // each with a shorter range of column groups
  int grid_g = 0, part_rows = 0, tok_max = 0, Sg = 0, smem_g = 0;
  for (int waves = 1; waves <= 4 && !Sg; ++waves) {
    grid_g = static_cast<int>(std::min<int64_t>(static_cast<int64_t>(sms) * waves, nq_all));
    const int64_t nq_max = ceil_div(nq_all, grid_g);
    part_rows = static_cast<int>(nq_max) * Gg;
    // tokens one CTA's contiguous range of pairs can touch
    tok_max = static_cast<int>(std::min<int64_t>(T, (ceil_div(nq_max, ngj) + 1 + KP - 1) / KP + 1));
    for (int S : {2, 1}) {
      const int t = moe1_layout(S, tok_max, nbh, part_rows * nchg * 2, NP).total;
      if (t <= 227 * 1024) { Sg = S; smem_g = t; break; }
    }
    if (grid_g == nq_all) break;
  }
  // down: groups of RGd output rows, all pairs
  const int64_t ngr_all = ceil_div(H, RGd);
  const int grid_d = static_cast<int>(std::min<int64_t>(sms, ngr_all));
  const int rows_max = static_cast<int>(ceil_div(ngr_all, grid_d)) * RGd;
  // pairs per group: as many rotated h as fit beside the ring and all partials
  int Sd = 0, smem_d = 0, pg_max = 0;
  for (int S : {2, 1}) {
    int pg = NP;
    while (pg > 0 && moe1_layout(S, pg, nbf, NP * rows_max * nchd, NP).total > 227 * 1024) pg = pg > 8 ? pg * 3 / 4 : pg - 1;
    if (pg > 0 && (pg >= std::min(NP, KP) || S == 1)) {
      Sd = S;
      pg_max = pg;
      smem_d = moe1_layout(S, pg, nbf, NP * rows_max * nchd, NP).total;
      break;
    }
  }
  if (!Sg || !Sd) return HLWQ_EUNSUPPORTED;

  CUtensorMap gm, gsm, dm, dsm;
  int st = codes_map(gu_packed, static_cast<int64_t>(E) * 2 * F, nbh, cg, Gg, &gm);
  if (st == HLWQ_OK) st = codes_map(dn_packed, static_cast<int64_t>(E) * H, nbf, cd, RGd, &dm);
  if (st == HLWQ_OK && shared) st = codes_map(sh_gu_packed, 2 * static_cast<int64_t>(F), nbh, cg, Gg, &gsm);
  if (st == HLWQ_OK && shared) st = codes_map(sh_dn_packed, H, nbf, cd, RGd, &dsm);
  if (st != HLWQ_OK) return st;
  if (!shared) {
    gsm = gm;
    dsm = dm;
  }
  Moe1Params P;
  P.logits = logits;
  P.X = X;
  P.gu_norms = gu_norms;
  P.sh_gu_norms = shared ? sh_gu_norms : gu_norms;
  P.dn_norms = dn_norms;
  P.sh_dn_norms = shared ? sh_dn_norms : dn_norms;
  P.codebook = codebook;
  P.h = h_ws;
  P.ids_out = ids_out;
  P.w_out = w_out;
  P.Y = Y;
  P.E = E;
  P.H = H;
  P.F = F;
  P.T = T;
  P.topk = topk;
  P.has_shared = shared ? 1 : 0;
  P.out_bf16 = out_bf16 ? 1 : 0;
  switch (cg) {
    case 8: st = moe1_gu_c<8>(Sg, gm, gsm, P, grid_g, part_rows, tok_max, smem_g, stream); break;
    case 4: st = moe1_gu_c<4>(Sg, gm, gsm, P, grid_g, part_rows, tok_max, smem_g, stream); break;
    default: st = moe1_gu_c<2>(Sg, gm, gsm, P, grid_g, part_rows, tok_max, smem_g, stream); break;
  }
  if (st != HLWQ_OK) return st;
  switch (cd) {
    case 8: return moe1_dn_c<8>(Sd, dm, dsm, P, grid_d, rows_max, pg_max, smem_d, stream);
    case 4: return moe1_dn_c<4>(Sd, dm, dsm, P, grid_d, rows_max, pg_max, smem_d, stream);
    default: return moe1_dn_c<2>(Sd, dm, dsm, P, grid_d, rows_max, pg_max, smem_d, stream);
  }
}

}  // namespace hlwq
