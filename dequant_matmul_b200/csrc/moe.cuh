#pragma once
// Routed mixture-of-experts layer on HLWQ Q5 experts (sm_100a).
//
// "Qwen3.6-35B-A3B -- HLWQ Q5" model card: 256 experts per layer, 8 routed +
// 1 shared per token; "Gemma-4-26B-A4B-it-HLWQ-Q5", Technical Details: 3-D
// expert tensors (128, 1408, 2816) and (128, 2816, 704), each expert quantized
// independently.  Per token t:
//   ids, p = top-k of the router logits (ties: lower id), p = softmax over the
//            k selected logits;
//   g || u = w_hat_gu[e] @ x_t (rows [0, F) gate, [F, 2F) up), h = SiLU(g) * u;
//   Y[t]   = sum_s p_s * w_hat_dn[ids_s] @ h_s  (+ shared expert with weight 1).
//
// The grouped path (the fused two-kernel path for few tokens is moe1.cuh):
//   1. router_kernel (one CTA): top-k + softmax per token, then the
//      per-expert assignment lists (shared-memory atomics and a block scan);
//   2. gate_up, SiLU and down on the tensor cores, each active expert's codes
//      decoded once for all its tokens (launch_moe_tc, gemm_tc.cuh);
//   3. combine: Y[t] = sum over the token's assignment slots in a fixed order.
// Deterministic: the order of an expert's assignments varies with the
// atomics, but each assignment is computed on its own.

#include <algorithm>

#include "engine.cuh"

namespace hlwq {

namespace {

constexpr int kRouterThreads = 1024;
constexpr int kMoeMaxIn = 16384;  // H and F of the grouped path (tile norms of up to 128 blocks)

struct MoeWs {
  int* meta;          // [0] = number of active experts (shared expert last)
  int* active;        // [E + 1] expert id per active slot (E = shared expert)
  int* offsets;       // [E + 2] assignment range per active slot
  int* asg_token;     // [NA]
  float* asg_weight;  // [NA]
  int* tok_asg;       // [T][topk + 1] assignment index per (token, slot), -1 = none
  int* sel_id;        // [T][topk]
  float* sel_w;       // [T][topk]
  float* h;           // [NA][F]
  float* part;        // [NA][H]
  // tensor-core grouped path
  uint16_t* bg;       // [NA][NBh * 128] rotated activation of each assignment's token (binary16)
  float* inv_g;       // [NA] its scale
  float* g2;          // [NA][2F] gate and up outputs (fp32)
  uint16_t* bh;       // [NA][NBf * 128] rotated SiLU(g) * u (binary16)
  float* inv_h;       // [NA] its scale times the assignment's routing weight
};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

size_t moe_layout(int64_t E, int64_t H, int64_t F, int64_t T, int64_t topk, char* base, MoeWs* ws) {
  const int64_t nbh = ceil_div(H, kBlock);
  const int64_t na = T * topk + T;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off += align256(bytes);
    return p;
  };
  MoeWs w;
  w.meta = reinterpret_cast<int*>(take(16));
  w.active = reinterpret_cast<int*>(take(sizeof(int) * (E + 1)));
  w.offsets = reinterpret_cast<int*>(take(sizeof(int) * (E + 2)));
  w.asg_token = reinterpret_cast<int*>(take(sizeof(int) * na));
  w.asg_weight = reinterpret_cast<float*>(take(sizeof(float) * na));
  w.tok_asg = reinterpret_cast<int*>(take(sizeof(int) * T * (topk + 1)));
  w.sel_id = reinterpret_cast<int*>(take(sizeof(int) * T * topk));
  w.sel_w = reinterpret_cast<float*>(take(sizeof(float) * T * topk));
  w.h = reinterpret_cast<float*>(take(sizeof(float) * na * F));
  w.part = reinterpret_cast<float*>(take(sizeof(float) * na * H));
  const int64_t nbf = ceil_div(F, kBlock);
  w.bg = reinterpret_cast<uint16_t*>(take(sizeof(uint16_t) * na * nbh * kBlock));
  w.inv_g = reinterpret_cast<float*>(take(sizeof(float) * na));
  w.g2 = reinterpret_cast<float*>(take(sizeof(float) * na * 2 * F));
  w.bh = reinterpret_cast<uint16_t*>(take(sizeof(uint16_t) * na * nbf * kBlock));
  w.inv_h = reinterpret_cast<float*>(take(sizeof(float) * na));
  if (ws) *ws = w;
  return off;
}

// Top-k routing of one token by one warp: the k largest logits (ties: lower
// expert id) and softmax weights over the k selected logits, accumulated in
// selection order.  ids / wts get k entries; every lane of the warp must call
// it.  Each logit (expert lane + 32 i, E <= 1024) is held as an unsigned key
// whose order is the float order (-0 counted as +0; logits must not be NaN),
// so one selection round is a warp max-reduction of the keys and a min-
// reduction of the indices that hold the maximum (a real key is never 0: the
// smallest, that of -NaN payloads aside, is the key of -inf, 0x007fffff).
__device__ __forceinline__ uint32_t logit_key(float f) {
  uint32_t b = __float_as_uint(f);
  if ((b & 0x7fffffffu) == 0u) b = 0u;  // -0 == +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key_logit(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// NL keys per lane (E <= 32 NL); per-lane maxima and minima as pairwise trees.
template <int NL>
__device__ __forceinline__ void route_token_warp_n(const float* __restrict__ lg, int E, int topk, int* ids,
                                                   float* wts) {
  const int lane = threadIdx.x & 31;
  uint32_t key[NL];
#pragma unroll
  for (int i = 0; i < NL; ++i) {
    const int e = lane + 32 * i;
    key[i] = e < E ? logit_key(__ldg(lg + e)) : 0u;  // key 0: absent or taken (real keys are > 0)
  }
  float vmax = 0.0f, wsum = 0.0f;
  for (int s = 0; s < topk; ++s) {
    uint32_t t[NL];
#pragma unroll
    for (int i = 0; i < NL; ++i) t[i] = key[i];
#pragma unroll
    for (int w = NL / 2; w > 0; w >>= 1)
#pragma unroll
      for (int i = 0; i < w; ++i) t[i] = max(t[i], t[i + w]);
    const uint32_t gm = __reduce_max_sync(0xffffffffu, t[0]);
#pragma unroll
    for (int i = 0; i < NL; ++i) t[i] = key[i] == gm ? static_cast<uint32_t>(lane + 32 * i) : 0xffffffffu;
#pragma unroll
    for (int w = NL / 2; w > 0; w >>= 1)
#pragma unroll
      for (int i = 0; i < w; ++i) t[i] = min(t[i], t[i + w]);
    const int bi = static_cast<int>(__reduce_min_sync(0xffffffffu, t[0]));
#pragma unroll
    for (int i = 0; i < NL; ++i)
      if (lane + 32 * i == bi) key[i] = 0u;
    const float bv = key_logit(gm);
    if (s == 0) vmax = bv;
    const float ex = expf(bv - vmax);
    wsum += ex;
    if (lane == 0) {
      ids[s] = bi;
      wts[s] = ex;
    }
  }
  __syncwarp();
  if (lane < topk) wts[lane] = wts[lane] / wsum;
  __syncwarp();
}

__device__ __forceinline__ void route_token_warp(const float* __restrict__ lg, int E, int topk, int* ids,
                                                 float* wts) {
  if (E <= 256) route_token_warp_n<8>(lg, E, topk, ids, wts);
  else route_token_warp_n<32>(lg, E, topk, ids, wts);
}

__global__ void __launch_bounds__(kRouterThreads, 1)
router_kernel(const float* __restrict__ logits, int E, int T, int topk, int has_shared,
              int32_t* __restrict__ ids_out, float* __restrict__ w_out, MoeWs ws) {
  __shared__ int s_count[1025], s_cursor[1025], s_wsum[32], s_wact[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  // 1. top-k + softmax, one warp per token.
  for (int t = warp; t < T; t += kRouterThreads / 32) {
    route_token_warp(logits + static_cast<int64_t>(t) * E, E, topk, ws.sel_id + t * topk, ws.sel_w + t * topk);
    if (lane < topk) {
      if (ids_out) ids_out[t * topk + lane] = ws.sel_id[t * topk + lane];
      if (w_out) w_out[t * topk + lane] = ws.sel_w[t * topk + lane];
    }
  }
  __syncthreads();

  // 2. assignments per expert (id E = shared expert, every token): counts by
  // shared-memory atomics, active slots and offsets by a block-wide scan,
  // then every selection placed at its expert's cursor.  The order of an
  // expert's assignments is not fixed, and nothing depends on it: every
  // assignment is computed on its own and each token's partials are added
  // through tok_asg in slot order.
  const int nexp = E + (has_shared ? 1 : 0);
  const int nsel = T * topk;
  for (int e = threadIdx.x; e < nexp; e += kRouterThreads) s_count[e] = (e == E) ? T : 0;
  __syncthreads();
  for (int q = threadIdx.x; q < nsel; q += kRouterThreads) atomicAdd(&s_count[ws.sel_id[q]], 1);
  __syncthreads();
  {
    // thread t owns experts 2t and 2t + 1 (nexp <= 1025 <= 2 * kRouterThreads)
    const int e0 = 2 * threadIdx.x, e1 = e0 + 1;
    const int c0 = e0 < nexp ? s_count[e0] : 0, c1 = e1 < nexp ? s_count[e1] : 0;
    int cnt = c0 + c1, act = (c0 > 0) + (c1 > 0);
    // inclusive warp scans, then the warps' totals
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, cnt, off), b = __shfl_up_sync(0xffffffffu, act, off);
      if (lane >= off) { cnt += a; act += b; }
    }
    if (lane == 31) { s_wsum[warp] = cnt; s_wact[warp] = act; }
    __syncthreads();
    if (warp == 0) {
      int wc = s_wsum[lane], wa = s_wact[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int a = __shfl_up_sync(0xffffffffu, wc, off), b = __shfl_up_sync(0xffffffffu, wa, off);
        if (lane >= off) { wc += a; wa += b; }
      }
      s_wsum[lane] = wc - s_wsum[lane];  // exclusive
      s_wact[lane] = wa - s_wact[lane];
      if (lane == 31) { ws.offsets[wa] = wc; ws.meta[0] = wa; }
    }
    __syncthreads();
    int off = s_wsum[warp] + cnt - c0 - c1, slot = s_wact[warp] + act - (c0 > 0) - (c1 > 0);
    if (c0 > 0) { ws.active[slot] = e0; ws.offsets[slot] = off; s_cursor[e0] = off; off += c0; ++slot; }
    if (c1 > 0) { ws.active[slot] = e1; ws.offsets[slot] = off; s_cursor[e1] = off; }
  }
  __syncthreads();
  for (int q = threadIdx.x; q < nsel; q += kRouterThreads) {
    const int pos = atomicAdd(&s_cursor[ws.sel_id[q]], 1);
    ws.asg_token[pos] = q / topk;
    ws.asg_weight[pos] = ws.sel_w[q];
    ws.tok_asg[(q / topk) * (topk + 1) + (q % topk)] = pos;
  }
  if (has_shared) {
    const int base = s_cursor[E];
    for (int t = threadIdx.x; t < T; t += kRouterThreads) {
      ws.asg_token[base + t] = t;
      ws.asg_weight[base + t] = 1.0f;
      ws.tok_asg[t * (topk + 1) + topk] = base + t;
    }
  }
  if (!has_shared)
    for (int t = threadIdx.x; t < T; t += kRouterThreads) ws.tok_asg[t * (topk + 1) + topk] = -1;
}

__global__ void combine_kernel(int H, int T, int topk, MoeWs ws, void* __restrict__ Y, int out_bf16) {
  const int t = blockIdx.y;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T || i >= H) return;
  float acc = 0.0f;
  for (int s = 0; s <= topk; ++s) {
    const int asg = ws.tok_asg[t * (topk + 1) + s];
    if (asg >= 0) acc += ws.part[static_cast<int64_t>(asg) * H + i];
  }
  const int64_t off = static_cast<int64_t>(t) * H + i;
  if (out_bf16) static_cast<uint16_t*>(Y)[off] = static_cast<uint16_t>(float_to_bf16_bits(acc));
  else static_cast<float*>(Y)[off] = acc;
}


}  // namespace

size_t moe_workspace_bytes(int64_t E, int64_t H, int64_t F, int64_t T, int64_t topk) {
  return moe_layout(E, H, F, T, topk, nullptr, nullptr);
}

// gemm_tc.cuh: gate_up and down of the grouped path on the tensor cores.
int launch_moe_tc(const uint8_t* gu_packed, const uint16_t* gu_norms, const uint8_t* dn_packed,
                  const uint16_t* dn_norms, const uint8_t* sh_gu_packed, const uint16_t* sh_gu_norms,
                  const uint8_t* sh_dn_packed, const uint16_t* sh_dn_norms, const float* codebook, int E, int H, int F,
                  int topk, int T, const uint16_t* X, const MoeWs& ws, cudaStream_t stream);

int launch_moe(const uint8_t* gu_packed, const uint16_t* gu_norms, const uint8_t* dn_packed,
               const uint16_t* dn_norms, const uint8_t* sh_gu_packed, const uint16_t* sh_gu_norms,
               const uint8_t* sh_dn_packed, const uint16_t* sh_dn_norms, const float* codebook, int E, int H, int F,
               int topk, int T, const float* logits, const uint16_t* X, void* Y, bool out_bf16, int32_t* ids_out,
               float* w_out, void* workspace, cudaStream_t stream) {
  MoeWs ws;
  moe_layout(E, H, F, T, topk, static_cast<char*>(workspace), &ws);
  const bool shared = sh_gu_packed != nullptr;
  // one CTA routes and builds the lists; gate_up and down on the tensor cores
  // (H and F up to kMoeMaxIn), then the fixed-order combine
  if (H > kMoeMaxIn || F > kMoeMaxIn) return HLWQ_EUNSUPPORTED;
  router_kernel<<<1, kRouterThreads, 0, stream>>>(logits, E, T, topk, shared ? 1 : 0, ids_out, w_out, ws);
  if (cudaGetLastError() != cudaSuccess) return HLWQ_ECUDA;
  if (const int st = launch_moe_tc(gu_packed, gu_norms, dn_packed, dn_norms, sh_gu_packed, sh_gu_norms, sh_dn_packed,
                                   sh_dn_norms, codebook, E, H, F, topk, T, X, ws, stream))
    return st;
  dim3 cgrid(static_cast<unsigned>(ceil_div(H, 256)), static_cast<unsigned>(T));
  combine_kernel<<<cgrid, 256, 0, stream>>>(H, T, topk, ws, Y, out_bf16 ? 1 : 0);
  return cudaGetLastError() == cudaSuccess ? HLWQ_OK : HLWQ_ECUDA;
}

}  // namespace hlwq
