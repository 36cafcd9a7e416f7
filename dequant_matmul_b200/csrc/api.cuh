#pragma once
// extern "C" entry points of libhlwq (declared and documented in include/hlwq.h).
// Every argument is validated on the host; nothing is launched on an error.

#include <algorithm>
#include <cstdint>

#include "hlwq_common.cuh"

namespace hlwq {



int launch_quantize(const void* W, bool bf16, int64_t rows, int in, const float* codebook, uint8_t* packed,
                    uint16_t* norms, cudaStream_t stream);
int launch_dequantize(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t rows, int in,
                      void* out, bool bf16, cudaStream_t stream);
int launch_codes_unpack(const uint8_t* packed, int64_t nblocks, uint8_t* codes, cudaStream_t stream);
int launch_codes_pack(const uint8_t* codes, int64_t nblocks, uint8_t* packed, cudaStream_t stream);
int launch_tq3_quantize(const uint16_t* W, int64_t rows, int in, const int8_t* signs, const float* codebook,
                        uint8_t* packed, float* norms, cudaStream_t stream);
int launch_tq3_dequantize(const uint8_t* packed, const float* norms, const int8_t* signs, const float* codebook,
                          int64_t rows, int in, void* out, bool bf16, cudaStream_t stream);
int launch_tq3_gemv(const uint8_t* packed, const float* norms, const int8_t* signs, const float* codebook,
                    int64_t O, int in, const uint16_t* x, void* y, bool out_bf16, cudaStream_t stream);
int launch_requantize_int4(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t rows,
                           int in, uint8_t* q4, uint16_t* scale, uint16_t* zero, cudaStream_t stream);
int launch_kv_quantize(const uint16_t* X, int64_t n, int64_t ldx, const float* codebook, uint8_t* packed,
                       uint16_t* norms, cudaStream_t stream);
int launch_kv_dequantize(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t n, void* out,
                         bool bf16, cudaStream_t stream);
int launch_kv_scores(const uint16_t* Q, int64_t m, int64_t ldq, const uint8_t* packed, const uint16_t* norms,
                     const float* codebook, int64_t n_enc, const uint16_t* window, int64_t R, int64_t n_total,
                     float* S, int64_t lds, cudaStream_t stream);
int launch_kv_window_append(const uint16_t* X, int64_t t, int64_t ldx, uint16_t* window, int64_t R, int64_t n_enc,
                            int64_t n_total, const float* codebook, uint8_t* packed, uint16_t* norms,
                            int64_t* n_enc_out, cudaStream_t stream);
int launch_dense(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                 const uint16_t* X, int64_t ldx, int M, void* Y, int64_t ldy, bool out_bf16, cudaStream_t stream);
int launch_gemm_tc(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                   const uint16_t* X, int64_t ldx, int M, void* Y, int64_t ldy, bool out_bf16, void* workspace,
                   size_t ws_bytes, cudaStream_t stream);
size_t gemm_tc_workspace_bytes(int64_t O, int64_t in, int64_t M);
size_t gemm_tc_workspace_min_bytes(int64_t O, int64_t in, int64_t M);
size_t tq3_tc_workspace_bytes(int64_t O, int64_t in, int64_t M);
size_t tq3_tc_workspace_min_bytes(int64_t O, int64_t in, int64_t M);
int launch_tq3_gemm(const uint8_t* packed, const float* norms, const int8_t* signs, const float* codebook,
                    int64_t O, int in, const uint16_t* X, int64_t ldx, int M, void* Y, int64_t ldy, bool out_bf16,
                    void* workspace, size_t ws_bytes, cudaStream_t stream);
size_t moe_workspace_bytes(int64_t E, int64_t H, int64_t F, int64_t T, int64_t topk);
int launch_moe(const uint8_t* gu_packed, const uint16_t* gu_norms, const uint8_t* dn_packed,
               const uint16_t* dn_norms, const uint8_t* sh_gu_packed, const uint16_t* sh_gu_norms,
               const uint8_t* sh_dn_packed, const uint16_t* sh_dn_norms, const float* codebook, int E, int H, int F,
               int topk, int T, const float* logits, const uint16_t* X, void* Y, bool out_bf16, int32_t* ids_out,
               float* w_out, void* workspace, cudaStream_t stream);

}  // namespace hlwq

namespace {

constexpr int64_t kMaxIn = 1 << 20;  // in-features limit (int indexing inside blocks)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned2(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 1u) == 0; }
cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// Threshold between the CUDA-core decode path and the tensor-core path.
constexpr int64_t kTensorCoreMinM = 5;  // M = 2..4: the multi-token CUDA-core kernel; M >= 5: tcgen05

}  // namespace

extern "C" int hlwq_quantize(const void* W, int wdtype, int64_t rows, int64_t in, const float* codebook,
                             uint8_t* packed, uint16_t* norms, void* stream) {
  if (!W || !codebook || !packed || !norms || rows <= 0 || in <= 0 || in > kMaxIn) return HLWQ_EINVAL;
  if (wdtype != HLWQ_F32 && wdtype != HLWQ_BF16) return HLWQ_EUNSUPPORTED;
  if (!aligned16(packed) || !aligned2(norms) || !aligned2(W) || (wdtype == HLWQ_F32 && (reinterpret_cast<uintptr_t>(W) & 3u)))
    return HLWQ_EALIGN;
  return hlwq::launch_quantize(W, wdtype == HLWQ_BF16, rows, static_cast<int>(in), codebook, packed, norms,
                               as_stream(stream));
}

extern "C" int hlwq_dequantize(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t rows,
                               int64_t in, void* W_out, int odtype, void* stream) {
  if (!W_out || !codebook || !packed || !norms || rows <= 0 || in <= 0 || in > kMaxIn) return HLWQ_EINVAL;
  if (odtype != HLWQ_F32 && odtype != HLWQ_BF16) return HLWQ_EUNSUPPORTED;
  if (!aligned16(packed) || !aligned2(norms) || !aligned2(W_out) ||
      (odtype == HLWQ_F32 && (reinterpret_cast<uintptr_t>(W_out) & 3u)))
    return HLWQ_EALIGN;
  return hlwq::launch_dequantize(packed, norms, codebook, rows, static_cast<int>(in), W_out, odtype == HLWQ_BF16,
                                 as_stream(stream));
}

extern "C" int hlwq_codes_unpack(const uint8_t* packed, int64_t nblocks, uint8_t* codes, void* stream) {
  if (!packed || !codes || nblocks <= 0 || nblocks > (int64_t(1) << 40)) return HLWQ_EINVAL;
  if (!aligned16(packed) || !aligned16(codes)) return HLWQ_EALIGN;
  return hlwq::launch_codes_unpack(packed, nblocks, codes, as_stream(stream));
}

extern "C" int hlwq_codes_pack(const uint8_t* codes, int64_t nblocks, uint8_t* packed, void* stream) {
  if (!packed || !codes || nblocks <= 0 || nblocks > (int64_t(1) << 40)) return HLWQ_EINVAL;
  if (!aligned16(packed) || !aligned16(codes)) return HLWQ_EALIGN;
  return hlwq::launch_codes_pack(codes, nblocks, packed, as_stream(stream));
}

extern "C" int hlwq_tq3_quantize(const uint16_t* W, int64_t rows, int64_t in, const int8_t* signs,
                                 const float* codebook8, uint8_t* packed, float* norms, void* stream) {
  if (!W || !signs || !codebook8 || !packed || !norms || rows <= 0 || in <= 0 || in > kMaxIn) return HLWQ_EINVAL;
  if (!aligned2(W) || (reinterpret_cast<uintptr_t>(packed) & 3u) || (reinterpret_cast<uintptr_t>(norms) & 3u))
    return HLWQ_EALIGN;
  return hlwq::launch_tq3_quantize(W, rows, static_cast<int>(in), signs, codebook8, packed, norms, as_stream(stream));
}

extern "C" int hlwq_tq3_dequantize(const uint8_t* packed, const float* norms, const int8_t* signs,
                                   const float* codebook8, int64_t rows, int64_t in, void* W_out, int odtype,
                                   void* stream) {
  if (!packed || !norms || !signs || !codebook8 || !W_out || rows <= 0 || in <= 0 || in > kMaxIn)
    return HLWQ_EINVAL;
  if (odtype != HLWQ_F32 && odtype != HLWQ_BF16) return HLWQ_EUNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(packed) & 3u) || (reinterpret_cast<uintptr_t>(norms) & 3u) || !aligned2(W_out) ||
      (odtype == HLWQ_F32 && (reinterpret_cast<uintptr_t>(W_out) & 3u)))
    return HLWQ_EALIGN;
  return hlwq::launch_tq3_dequantize(packed, norms, signs, codebook8, rows, static_cast<int>(in), W_out,
                                     odtype == HLWQ_BF16, as_stream(stream));
}

extern "C" int hlwq_tq3_gemv(const uint8_t* packed, const float* norms, const int8_t* signs, const float* codebook8,
                             int64_t out, int64_t in, const uint16_t* x, void* y, int ydtype, void* stream) {
  if (!packed || !norms || !signs || !codebook8 || !x || !y || out <= 0 || in <= 0 || in > kMaxIn ||
      out > (int64_t(1) << 40))
    return HLWQ_EINVAL;
  if (ydtype != HLWQ_F32 && ydtype != HLWQ_BF16) return HLWQ_EUNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(packed) & 3u) || (reinterpret_cast<uintptr_t>(norms) & 3u) || !aligned2(x) ||
      !aligned2(y) || (ydtype == HLWQ_F32 && (reinterpret_cast<uintptr_t>(y) & 3u)))
    return HLWQ_EALIGN;
  return hlwq::launch_tq3_gemv(packed, norms, signs, codebook8, out, static_cast<int>(in), x, y, ydtype == HLWQ_BF16,
                               as_stream(stream));
}

extern "C" int hlwq_tq3_gemm(const uint8_t* packed, const float* norms, const int8_t* signs,
                             const float* codebook8, int64_t out, int64_t in, int64_t M, const uint16_t* X,
                             int64_t ldx, void* Y, int64_t ldy, int ydtype, void* workspace, size_t ws_bytes,
                             void* stream) {
  if (!packed || !norms || !signs || !codebook8 || !X || !Y || out <= 0 || in <= 0 || in > kMaxIn ||
      out > (int64_t(1) << 40) || M <= 0 || M > (1 << 20))
    return HLWQ_EINVAL;
  if (ldx < in || ldy < out) return HLWQ_EINVAL;
  if (ydtype != HLWQ_F32 && ydtype != HLWQ_BF16) return HLWQ_EUNSUPPORTED;
  if (!aligned16(packed) || (reinterpret_cast<uintptr_t>(norms) & 3u) || !aligned2(X) || !aligned2(Y) ||
      (ydtype == HLWQ_F32 && (reinterpret_cast<uintptr_t>(Y) & 3u)))
    return HLWQ_EALIGN;
  const size_t need = M >= 2 ? hlwq::tq3_tc_workspace_min_bytes(out, in, M) : 0;
  if (need && (!workspace || ws_bytes < need)) return HLWQ_EWORKSPACE;
  if (need && !aligned16(workspace)) return HLWQ_EALIGN;
  return hlwq::launch_tq3_gemm(packed, norms, signs, codebook8, out, static_cast<int>(in), X, ldx,
                               static_cast<int>(M), Y, ldy, ydtype == HLWQ_BF16, workspace, ws_bytes,
                               as_stream(stream));
}

extern "C" int hlwq_requantize_int4(const uint8_t* packed, const uint16_t* norms, const float* codebook,
                                    int64_t rows, int64_t in, uint8_t* q4, uint16_t* scale, uint16_t* zero,
                                    void* stream) {
  if (!packed || !norms || !codebook || !q4 || !scale || !zero || rows <= 0 || in <= 0 || in > kMaxIn)
    return HLWQ_EINVAL;
  if (in % hlwq::kBlock) return HLWQ_EUNSUPPORTED;  // non-aligned rows stay in the Q5 / dequantized form
  if (!aligned16(packed) || !aligned16(q4) || !aligned2(norms) || !aligned2(scale) || !aligned2(zero))
    return HLWQ_EALIGN;
  return hlwq::launch_requantize_int4(packed, norms, codebook, rows, static_cast<int>(in), q4, scale, zero,
                                      as_stream(stream));
}

extern "C" int hlwq_kv_quantize(const uint16_t* x, int64_t n, int64_t ldx, const float* codebook8, uint8_t* packed,
                                uint16_t* norms, void* stream) {
  if (!x || !codebook8 || !packed || !norms || n <= 0 || n > (int64_t(1) << 40) || ldx < 256) return HLWQ_EINVAL;
  if (!aligned2(x) || (reinterpret_cast<uintptr_t>(packed) & 3u) || !aligned2(norms)) return HLWQ_EALIGN;
  return hlwq::launch_kv_quantize(x, n, ldx, codebook8, packed, norms, as_stream(stream));
}

extern "C" int hlwq_kv_dequantize(const uint8_t* packed, const uint16_t* norms, const float* codebook8, int64_t n,
                                  void* out, int odtype, void* stream) {
  if (!packed || !norms || !codebook8 || !out || n <= 0 || n > (int64_t(1) << 40)) return HLWQ_EINVAL;
  if (odtype != HLWQ_F32 && odtype != HLWQ_BF16) return HLWQ_EUNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(packed) & 3u) || !aligned2(norms) || !aligned16(out)) return HLWQ_EALIGN;
  return hlwq::launch_kv_dequantize(packed, norms, codebook8, n, out, odtype == HLWQ_BF16, as_stream(stream));
}

extern "C" int hlwq_kv_scores(const uint16_t* q, int64_t m, int64_t ldq, const uint8_t* packed,
                              const uint16_t* norms, const float* codebook8, int64_t n, float* scores, int64_t lds,
                              void* stream) {
  if (!q || !packed || !norms || !codebook8 || !scores || m <= 0 || n <= 0 || n > (int64_t(1) << 40) ||
      ldq < 256 || lds < n)
    return HLWQ_EINVAL;
  if (m > 64) return HLWQ_EUNSUPPORTED;
  if (!aligned2(q) || (reinterpret_cast<uintptr_t>(packed) & 3u) || !aligned2(norms) ||
      (reinterpret_cast<uintptr_t>(scores) & 3u))
    return HLWQ_EALIGN;
  return hlwq::launch_kv_scores(q, m, ldq, packed, norms, codebook8, n, nullptr, 1, n, scores, lds,
                                as_stream(stream));
}

extern "C" int hlwq_kv_scores_window(const uint16_t* q, int64_t m, int64_t ldq, const uint8_t* packed,
                                     const uint16_t* norms, const float* codebook8, int64_t n_enc,
                                     const uint16_t* window, int64_t R, int64_t n_total, float* scores, int64_t lds,
                                     void* stream) {
  constexpr int64_t kMaxTokens = int64_t(1) << 40;
  if (!q || !codebook8 || !scores || m <= 0 || ldq < 256 || n_enc < 0 || n_total > kMaxTokens || n_total <= 0 ||
      n_enc > n_total || lds < n_total || R < 1 || R > kMaxIn || n_total - n_enc > R)
    return HLWQ_EINVAL;
  if (n_enc > 0 && (!packed || !norms)) return HLWQ_EINVAL;
  if (n_total > n_enc && !window) return HLWQ_EINVAL;
  if (m > 64) return HLWQ_EUNSUPPORTED;
  if (!aligned2(q) || (reinterpret_cast<uintptr_t>(packed) & 3u) || !aligned2(norms) || !aligned16(window) ||
      (reinterpret_cast<uintptr_t>(scores) & 3u))
    return HLWQ_EALIGN;
  return hlwq::launch_kv_scores(q, m, ldq, packed, norms, codebook8, n_enc, window, R, n_total, scores, lds,
                                as_stream(stream));
}

extern "C" int hlwq_kv_window_append(const uint16_t* x, int64_t t, int64_t ldx, uint16_t* window, int64_t R,
                                     int64_t n_enc, int64_t n_total, const float* codebook8, uint8_t* packed,
                                     uint16_t* norms, int64_t* n_enc_out, void* stream) {
  constexpr int64_t kMaxTokens = int64_t(1) << 40;
  if (!window || !codebook8 || !packed || !norms || t < 0 || (t > 0 && !x) || ldx < 256 || R < 1 || R > kMaxIn ||
      n_enc < 0 || n_enc > n_total || n_total - n_enc > R || n_total > kMaxTokens || t > kMaxTokens - n_total)
    return HLWQ_EINVAL;
  if (!aligned2(x) || !aligned16(window) || (reinterpret_cast<uintptr_t>(packed) & 3u) || !aligned2(norms))
    return HLWQ_EALIGN;
  return hlwq::launch_kv_window_append(x, t, ldx, window, R, n_enc, n_total, codebook8, packed, norms, n_enc_out,
                                       as_stream(stream));
}

extern "C" int hlwq_gemv(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t out,
                         int64_t in, const uint16_t* x, void* y, int ydtype, void* stream) {
  if (!packed || !norms || !codebook || !x || !y || out <= 0 || in <= 0 || in > kMaxIn) return HLWQ_EINVAL;
  if (ydtype != HLWQ_F32 && ydtype != HLWQ_BF16) return HLWQ_EUNSUPPORTED;
  if (!aligned16(packed) || !aligned2(norms) || !aligned2(x) || !aligned2(y) ||
      (ydtype == HLWQ_F32 && (reinterpret_cast<uintptr_t>(y) & 3u)))
    return HLWQ_EALIGN;
  return hlwq::launch_dense(packed, norms, codebook, out, static_cast<int>(in), x, in, 1, y, out,
                            ydtype == HLWQ_BF16, as_stream(stream));
}

extern "C" int hlwq_gemv_ex(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t out,
                            int64_t in, const uint16_t* x, void* y, int ydtype, unsigned flags, void* stream) {
  if (flags & ~static_cast<unsigned>(HLWQ_FLAG_WEIGHTS_STATIC)) return HLWQ_EINVAL;
  if (!packed || !norms || !codebook || !x || !y || out <= 0 || in <= 0 || in > kMaxIn) return HLWQ_EINVAL;
  if (ydtype != HLWQ_F32 && ydtype != HLWQ_BF16) return HLWQ_EUNSUPPORTED;
  if (!aligned16(packed) || !aligned2(norms) || !aligned2(x) || !aligned2(y) ||
      (ydtype == HLWQ_F32 && (reinterpret_cast<uintptr_t>(y) & 3u)))
    return HLWQ_EALIGN;
  return hlwq::launch_gemv1(packed, norms, codebook, out, static_cast<int>(in), x, y, ydtype == HLWQ_BF16,
                            as_stream(stream), flags);
}

namespace hlwq {
// Host checks of hlwq_gemm's arguments other than the workspace (shared with
// hlwq_gemm_noalloc, which runs them before it sizes its scratch).
int gemm_check_args(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t out, int64_t in,
                    int64_t M, const uint16_t* X, int64_t ldx, const void* Y, int64_t ldy, int ydtype) {
  if (!packed || !norms || !codebook || !X || !Y || out <= 0 || in <= 0 || in > kMaxIn || M <= 0 || M > (1 << 20))
    return HLWQ_EINVAL;
  if (ldx < in || ldy < out) return HLWQ_EINVAL;
  if (ydtype != HLWQ_F32 && ydtype != HLWQ_BF16) return HLWQ_EUNSUPPORTED;
  if (!aligned16(packed) || !aligned2(norms) || !aligned2(X) || !aligned2(Y) ||
      (ydtype == HLWQ_F32 && (reinterpret_cast<uintptr_t>(Y) & 3u)))
    return HLWQ_EALIGN;
  return HLWQ_OK;
}
}  // namespace hlwq

extern "C" int hlwq_gemm(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t out,
                         int64_t in, int64_t M, const uint16_t* X, int64_t ldx, void* Y, int64_t ldy, int ydtype,
                         void* workspace, size_t ws_bytes, void* stream) {
  if (const int st = hlwq::gemm_check_args(packed, norms, codebook, out, in, M, X, ldx, Y, ldy, ydtype)) return st;
  // the tensor-core path accepts its smallest workspace (no K split of the
  // last wave) up to the size hlwq_workspace_bytes reports
  const size_t need = M >= kTensorCoreMinM ? hlwq::gemm_tc_workspace_min_bytes(out, in, M) : 0;
  if (need && (!workspace || ws_bytes < need)) return HLWQ_EWORKSPACE;
  if (need && !aligned16(workspace)) return HLWQ_EALIGN;
  if (M >= kTensorCoreMinM)
    return hlwq::launch_gemm_tc(packed, norms, codebook, out, static_cast<int>(in), X, ldx, static_cast<int>(M), Y,
                                ldy, ydtype == HLWQ_BF16, workspace, ws_bytes, as_stream(stream));
  return hlwq::launch_dense(packed, norms, codebook, out, static_cast<int>(in), X, ldx, static_cast<int>(M), Y, ldy,
                            ydtype == HLWQ_BF16, as_stream(stream));
}

extern "C" int hlwq_moe_gemv_ex(const uint8_t* gu_packed, const uint16_t* gu_norms, const uint8_t* dn_packed,
                                const uint16_t* dn_norms, const uint8_t* sh_gu_packed, const uint16_t* sh_gu_norms,
                                const uint8_t* sh_dn_packed, const uint16_t* sh_dn_norms, const float* codebook,
                                int64_t E, int64_t H, int64_t F, int64_t topk, int64_t T, const float* router_logits,
                                const uint16_t* X, void* Y, int ydtype, int32_t* topk_ids, float* topk_weights,
                                void* workspace, size_t ws_bytes, unsigned flags, void* stream) {
  if (flags & ~static_cast<unsigned>(HLWQ_FLAG_MOE_GROUPED)) return HLWQ_EINVAL;
  if (!gu_packed || !gu_norms || !dn_packed || !dn_norms || !codebook || !router_logits || !X || !Y)
    return HLWQ_EINVAL;
  if (E <= 0 || E > 1024 || H <= 0 || H > kMaxIn || F <= 0 || F > kMaxIn || T <= 0 || T > 65535 || topk <= 0 ||
      topk > 32 || topk > E)
    return HLWQ_EINVAL;
  const int shared_given = (sh_gu_packed != nullptr) + (sh_gu_norms != nullptr) + (sh_dn_packed != nullptr) +
                           (sh_dn_norms != nullptr);
  if (shared_given != 0 && shared_given != 4) return HLWQ_EINVAL;
  if (ydtype != HLWQ_F32 && ydtype != HLWQ_BF16) return HLWQ_EUNSUPPORTED;
  if (!aligned16(gu_packed) || !aligned16(dn_packed) || (sh_gu_packed && !aligned16(sh_gu_packed)) ||
      (sh_dn_packed && !aligned16(sh_dn_packed)) || !aligned2(gu_norms) || !aligned2(dn_norms) || !aligned2(X) ||
      !aligned2(Y) || (reinterpret_cast<uintptr_t>(router_logits) & 3u) ||
      (ydtype == HLWQ_F32 && (reinterpret_cast<uintptr_t>(Y) & 3u)))
    return HLWQ_EALIGN;
  const size_t need = hlwq_workspace_bytes(HLWQ_OP_MOE, H, F, T, E, topk);
  if (!workspace || ws_bytes < need) return HLWQ_EWORKSPACE;
  if (!aligned16(workspace)) return HLWQ_EALIGN;
  // The grouped path (tensor cores, H and F up to 16384) reads each active
  // expert once for all its tokens; it pays off once the assignments reach
  // about three quarters of the experts (measured on the 256- and 128-expert
  // layers: the fused path is faster below, the grouped path from there on).
  // The fused path also runs when the grouped path cannot; the grouped path
  // when the fused one's shared memory does not fit.
  const bool grouped_ok = H <= 16384 && F <= 16384;
  if ((flags & HLWQ_FLAG_MOE_GROUPED) && !grouped_ok) return HLWQ_EUNSUPPORTED;
  hlwq::MoeWs ws;
  hlwq::moe_layout(E, H, F, T, topk, static_cast<char*>(workspace), &ws);
  const bool grouped = (flags & HLWQ_FLAG_MOE_GROUPED) || (4 * T * topk >= 3 * E && grouped_ok);
  const int st = grouped ? HLWQ_EUNSUPPORTED : hlwq::launch_moe1(gu_packed, gu_norms, dn_packed, dn_norms, sh_gu_packed, sh_gu_norms, sh_dn_packed,
                                   sh_dn_norms, codebook, static_cast<int>(E), static_cast<int>(H),
                                   static_cast<int>(F), static_cast<int>(topk), static_cast<int>(T), router_logits, X,
                                   Y, ydtype == HLWQ_BF16, topk_ids, topk_weights, ws.h, as_stream(stream));
  if (st != HLWQ_EUNSUPPORTED) return st;
  return hlwq::launch_moe(gu_packed, gu_norms, dn_packed, dn_norms, sh_gu_packed, sh_gu_norms, sh_dn_packed,
                          sh_dn_norms, codebook, static_cast<int>(E), static_cast<int>(H), static_cast<int>(F),
                          static_cast<int>(topk), static_cast<int>(T), router_logits, X, Y, ydtype == HLWQ_BF16,
                          topk_ids, topk_weights, workspace, as_stream(stream));
}

extern "C" int hlwq_moe_gemv(const uint8_t* gu_packed, const uint16_t* gu_norms, const uint8_t* dn_packed,
                             const uint16_t* dn_norms, const uint8_t* sh_gu_packed, const uint16_t* sh_gu_norms,
                             const uint8_t* sh_dn_packed, const uint16_t* sh_dn_norms, const float* codebook,
                             int64_t E, int64_t H, int64_t F, int64_t topk, int64_t T, const float* router_logits,
                             const uint16_t* X, void* Y, int ydtype, int32_t* topk_ids, float* topk_weights,
                             void* workspace, size_t ws_bytes, void* stream) {
  return hlwq_moe_gemv_ex(gu_packed, gu_norms, dn_packed, dn_norms, sh_gu_packed, sh_gu_norms, sh_dn_packed,
                          sh_dn_norms, codebook, E, H, F, topk, T, router_logits, X, Y, ydtype, topk_ids, topk_weights,
                          workspace, ws_bytes, 0u, stream);
}

extern "C" size_t hlwq_workspace_bytes(int op, int64_t a, int64_t b, int64_t c, int64_t E, int64_t topk) {
  if (a <= 0 || b <= 0 || c <= 0) return 0;
  if (op == HLWQ_OP_GEMM) return c >= kTensorCoreMinM ? hlwq::gemm_tc_workspace_bytes(a, b, c) : 0;
  if (op == HLWQ_OP_TQ3_GEMM) return c >= 2 ? hlwq::tq3_tc_workspace_bytes(a, b, c) : 0;
  if (op == HLWQ_OP_MOE) {
    if (E <= 0 || topk <= 0) return 0;
    return hlwq::moe_workspace_bytes(E, a, b, c, topk);
  }
  return 0;
}

extern "C" int hlwq_fault_inject(unsigned int skip_tma, unsigned long long wait_ns) {
#ifdef HLWQ_FAULT_INJECTION
  if (wait_ns == 0 || wait_ns > hlwq::kWaitTimeoutNs) return HLWQ_EINVAL;
  const unsigned int skip = skip_tma ? 1u : 0u;
  if (cudaDeviceSynchronize() != cudaSuccess) return HLWQ_ECUDA;
  if (cudaMemcpyToSymbol(hlwq::g_fault_skip_tma, &skip, sizeof(skip)) != cudaSuccess) return HLWQ_ECUDA;
  if (cudaMemcpyToSymbol(hlwq::g_fault_wait_ns, &wait_ns, sizeof(wait_ns)) != cudaSuccess) return HLWQ_ECUDA;
  return HLWQ_OK;
#else
  (void)skip_tma;
  (void)wait_ns;
  return HLWQ_EUNSUPPORTED;
#endif
}

extern "C" int hlwq_device_error(uint32_t* bits) {
  if (!bits) return HLWQ_EINVAL;
  if (cudaDeviceSynchronize() != cudaSuccess) return HLWQ_ECUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, hlwq::g_device_error, sizeof(v)) != cudaSuccess) return HLWQ_ECUDA;
  if (cudaMemcpyToSymbol(hlwq::g_device_error, &zero, sizeof(zero)) != cudaSuccess) return HLWQ_ECUDA;
  *bits = v;
  return HLWQ_OK;
}

extern "C" const char* hlwq_status_string(int status) {
  switch (status) {
    case HLWQ_OK: return "ok";
    case HLWQ_EINVAL: return "invalid argument";
    case HLWQ_EALIGN: return "misaligned pointer or leading dimension";
    case HLWQ_EUNSUPPORTED: return "unsupported size or dtype";
    case HLWQ_ECUDA: return "CUDA runtime error";
    case HLWQ_EWORKSPACE: return "workspace missing or too small";
    case HLWQ_ESCRATCH: return "request exceeds the static scratch of hlwq_gemm_noalloc";
    default: return "unknown status";
  }
}

extern "C" int hlwq_version(void) { return 100; }
