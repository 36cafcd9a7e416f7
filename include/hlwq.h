/*
 * hlwq.h -- C ABI of libhlwq, a CUDA (sm_100a) implementation of HLWQ Q5
 * (Hadamard-Lloyd Weight Quantization, 5 bits) and of the dequant-matmul that
 * consumes its packed codes directly.
 *
 * The method (as described on the "Qwen3.6-35B-A3B -- HLWQ Q5" model card,
 * section "Method", and restated on the "Qwopus3.6-27B-v2 . HLWQ Q5" card,
 * "Methodology notes"):
 *   [1] view W (out x in) as (out, NB, 128), NB = ceil(in / 128), the tail block
 *       zero-padded;
 *   [2] n = ||block||_2, stored as fp16;
 *   [3] y = (block / n) @ H, H the 128 x 128 +-1 Sylvester-Hadamard matrix
 *       H[i][j] = (-1)^popcount(i & j) (the orthonormal Hadamard x sqrt(128));
 *   [4] code = index of the nearest of 32 Lloyd-Max centroids for N(0,1), ties
 *       to the lower index;
 *   [5] pack 8 codes into 5 bytes: code j of a block occupies bits [5j, 5j+5)
 *       of the block's 80-byte little-endian bit string, least significant bit
 *       first.
 * Dequantisation: w_hat[o][128b + i] = n16[o][b] / 128 * sum_j c[k_obj] H[j][i].
 *
 * Also declared here: the Q5 -> INT4 re-encoder, the Q3 KV-cache encoding
 * with its residual window, the TQ3 (scalar HIGGS) weight format with its
 * fused GEMV and small-M GEMM, and the conversion between the packed codes
 * and one code per byte.
 *
 * Storage contract (all row-major, caller-owned):
 *   packed  uint8  [rows][NB][80]   (0.625 byte per weight, including the pad)
 *   norms   binary16 bit patterns, uint16 [rows][NB]
 *   codebook float32 [32], strictly ascending (as hlwq_lloyd_codebook returns)
 * Activations are bfloat16 bit patterns (uint16).  Output dtype is chosen per
 * call with hlwq_dtype.
 *
 * Conventions for every call:
 *   - Device pointers are CUDA device (or managed) memory on the current
 *     device; "stream" is a cudaStream_t passed as void* (NULL = the legacy
 *     default stream).  Device calls are asynchronous on that stream; errors
 *     detected on the host are returned before anything is launched.
 *   - The library allocates no memory at run time.  Calls that need scratch take a
 *     caller-provided device workspace sized by hlwq_workspace_bytes(), except
 *     hlwq_gemm_noalloc, which uses a static device array of the library.
 *   - Alignment: packed, W, W_out, X, Y and workspace must be 16-byte aligned
 *     (torch allocations are); leading dimensions are in elements.
 *   - Return value: HLWQ_OK (0) or a negative hlwq_status.
 *   - A kernel never traps.  Conditions it can only see on the device (e.g. a
 *     codebook that is not ascending) set bits in a device error word that
 *     hlwq_device_error() reads (synchronously) and clears.
 */
#ifndef HLWQ_H
#define HLWQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HLWQ_OK = 0,
  HLWQ_EINVAL = -1,       /* null pointer, non-positive size, bad levels / topk */
  HLWQ_EALIGN = -2,       /* a pointer or leading dimension breaks the alignment rule */
  HLWQ_EUNSUPPORTED = -3, /* a size or dtype combination this build does not handle */
  HLWQ_ECUDA = -4,        /* a CUDA runtime call (launch, attribute) failed */
  HLWQ_EWORKSPACE = -5,   /* workspace is NULL or below the call's minimum (hlwq_workspace_bytes; hlwq_gemm) */
  HLWQ_ESCRATCH = -6      /* request needs more than the static scratch of hlwq_gemm_noalloc */
} hlwq_status;

typedef enum { HLWQ_F32 = 0, HLWQ_BF16 = 1, HLWQ_F16 = 2 } hlwq_dtype;

/* Operations whose scratch size hlwq_workspace_bytes() reports. */
typedef enum { HLWQ_OP_GEMM = 1, HLWQ_OP_MOE = 2, HLWQ_OP_TQ3_GEMM = 3 } hlwq_op;

/* Launch flags of the *_ex calls. */
typedef enum { HLWQ_FLAG_WEIGHTS_STATIC = 1, HLWQ_FLAG_MOE_GROUPED = 2 } hlwq_flags;

/* Device error bits (hlwq_device_error). */
#define HLWQ_DEVERR_CODEBOOK 0x1u  /* codebook not strictly ascending or not finite */
#define HLWQ_DEVERR_TIMEOUT  0x2u  /* a bounded in-kernel wait gave up */
#define HLWQ_DEVERR_CODE_RANGE 0x4u  /* hlwq_codes_pack met a code above 31 */

/*
 * Lloyd-Max codebook for N(0,1) (Method step [4]: "Lloyd-Max 5-bit quantization
 * (32 centroids, N(0,1))").  Host-only, synchronous.
 *   levels      2, 4, 8, 16 or 32 (the device calls use 32)
 *   centroids   host float[levels], ascending, symmetric (c[L-1-k] = -c[k]):
 *               the fixed point of Lloyd's conditions rounded to nearest fp32
 *   midpoints   host float[levels-1] or NULL: (c[k] + c[k+1]) / 2 rounded to fp32
 *   mse         host double* or NULL: E[(Z - q(Z))^2] of the fp64 fixed point
 * Errors: HLWQ_EINVAL for another `levels` or a NULL centroids pointer.
 */
int hlwq_lloyd_codebook(int levels, float* centroids, float* midpoints, double* mse);

/*
 * Quantize `rows` x `in` weights (Method steps [1]-[5]); experts are stacked
 * rows ("Gemma-4-26B-A4B-it-HLWQ-Q5", Technical Details: each expert is
 * quantized independently -- rows never mix, so E experts of O rows are simply
 * rows = E * O).
 *   W         device, wdtype (HLWQ_F32 or HLWQ_BF16), [rows][in], row pitch = in
 *   codebook  device float[32]
 *   packed    device uint8 [rows][NB][80]   (output)
 *   norms     device uint16 [rows][NB]      (output, binary16 bits)
 * The norm is the exact L2 norm rounded to nearest binary16; codes are the
 * nearest centroid of the exactly rotated value (decisions within 1e-5 of a
 * midpoint are re-taken in fp64 on the device).
 * Errors: HLWQ_EINVAL (NULL, rows/in <= 0), HLWQ_EUNSUPPORTED (wdtype),
 *         HLWQ_EALIGN (W or packed not 16-byte aligned), HLWQ_ECUDA.
 */
int hlwq_quantize(const void* W, int wdtype, int64_t rows, int64_t in,
                  const float* codebook, uint8_t* packed, uint16_t* norms, void* stream);

/*
 * Dequantize ("Qwopus3.6-27B-v2 . HLWQ Q5", Pipeline: dequantize per-Linear).
 *   W_out  device, odtype (HLWQ_F32 or HLWQ_BF16), [rows][in]; pad dropped.
 * Errors: as hlwq_quantize.
 */
int hlwq_dequantize(const uint8_t* packed, const uint16_t* norms, const float* codebook,
                    int64_t rows, int64_t in, void* W_out, int odtype, void* stream);

/*
 * One-code-per-byte layout ("Gemma-4-26B-A4B-it-HLWQ-Q5", Technical Details:
 * codes stored as int8, one per byte) <-> the packed 5-bit stream (Method
 * step [5]).  nblocks = rows * NB blocks of 128 codes.
 *   codes   device uint8 [nblocks][128], values 0..31 (16-byte aligned)
 *   packed  device uint8 [nblocks][80] (16-byte aligned)
 * hlwq_codes_unpack writes codes from packed; hlwq_codes_pack writes packed
 * from codes, storing the low five bits of a code above 31 and setting
 * HLWQ_DEVERR_CODE_RANGE.  The norms are the same array in both layouts.
 * Errors: HLWQ_EINVAL (NULL, nblocks <= 0 or above 2^40), HLWQ_EALIGN, HLWQ_ECUDA.
 */
int hlwq_codes_unpack(const uint8_t* packed, int64_t nblocks, uint8_t* codes, void* stream);
int hlwq_codes_pack(const uint8_t* codes, int64_t nblocks, uint8_t* packed, void* stream);

/*
 * Q5 -> INT4 re-encoding ("Qwopus3.6-27B-v2 . HLWQ Q5", Pipeline: dequantize
 * per Linear, then INT4 weight-only with groups of 128 on 128-aligned Linears).
 * Per row and group b of 128 inputs (= the Q5 block), with w the dequantized
 * weights (as hlwq_dequantize, evaluated exactly in fp64):
 *   s = bf16((max w - min w) / 15),  z = bf16(min w)   (round to nearest even
 *       from the fp64 value; magnitudes below 2^-126 give a signed zero; a
 *       zero minimum is stored as +0)
 *   q_i = clamp(rint((w_i - z) / s), 0, 15) in fp64 (q = 0 when s = 0)
 *   q4     device uint8 [rows][in/128][64]: element 2k in bits 0-3 of byte k,
 *          element 2k+1 in bits 4-7 (16-byte aligned)
 *   scale  device uint16 [rows][in/128]: bfloat16 bits of s
 *   zero   device uint16 [rows][in/128]: bfloat16 bits of z
 * The INT4 weights are z + q * s.  in must be a multiple of 128 (non-aligned
 * rows stay in the Q5 form): otherwise HLWQ_EUNSUPPORTED.
 * Errors: HLWQ_EINVAL, HLWQ_EALIGN, HLWQ_EUNSUPPORTED, HLWQ_ECUDA.
 */
int hlwq_requantize_int4(const uint8_t* packed, const uint16_t* norms, const float* codebook,
                         int64_t rows, int64_t in, uint8_t* q4, uint16_t* scale, uint16_t* zero, void* stream);

/*
 * Q3 KV-cache encoding ("Qwopus3.6-27B-v2 . HLWQ Q5", Methodology notes,
 * KV-cache bullet: per-head Hadamard 256x256, 8-centroid Lloyd-Max, 3 bits per
 * value; head_dim = 256).  One vector = one (token, head) key or value.
 *   codebook8  device float32 [8], strictly ascending (hlwq_lloyd_codebook(8))
 *   packed     [N][96]: code j of a vector at bits [3j, 3j+3), LSB first
 *   norms      [N]: binary16 bits of ||x||_2 (round to nearest even from fp64)
 * hlwq_kv_quantize: x bf16 [N][ldx] (ldx >= 256) -> packed, norms; code_j =
 *   number of midpoints of the codebook below y_j = (x @ H256)_j / ||x||, all
 *   in fp64 (ties to the lower index; a zero vector gets code 3).
 * hlwq_kv_dequantize: -> out [N][256] (HLWQ_F32 or HLWQ_BF16, 16-byte
 *   aligned) = n16 * (c[code] @ H256) / 256.
 * hlwq_kv_scores: S[m][i] = q_m . x_hat_i for M <= 64 bf16 queries [M][ldq]
 *   (fp32, row pitch lds >= N); evaluated with each query rotated once.
 * Errors: HLWQ_EINVAL, HLWQ_EALIGN (packed 4-byte, norms / x / q 2-byte
 * alignment), HLWQ_EUNSUPPORTED (dtype; M > 64), HLWQ_ECUDA.
 *
 * The residual window (same card and bullet: the most recent 128 tokens stay
 * unquantized).  A cache of one head holds n_total tokens: tokens
 * 0 .. n_enc - 1 encoded (packed / norms rows), tokens n_enc .. n_total - 1 in
 * the window, a bf16 ring of R slots [R][256] (token i in slot i % R,
 * n_total - n_enc <= R; R = 128 for the cards' buffer).  The caller owns
 * every buffer and gives packed / norms room for the rows that get encoded.
 * hlwq_kv_window_append: appends t bf16 tokens x [t][ldx]; with
 *   n_total' = n_total + t and n_enc' = max(n_enc, n_total' - R), tokens
 *   n_enc .. n_enc' - 1 (oldest first, from the window or, when t > R, from
 *   x) are encoded into rows n_enc .. n_enc' - 1 exactly as hlwq_kv_quantize
 *   would, and the new tokens that stay are copied into their slots.
 *   *n_enc_out (host, may be NULL) receives n_enc'.  Asynchronous on stream;
 *   window, packed and norms must not be used by other streams meanwhile.
 * hlwq_kv_scores_window: S[m][i] for every cached token i < n_total: the
 *   decoded key for i < n_enc (as hlwq_kv_scores), the exact window key
 *   otherwise (q . k in fp32); one launch.  window may be NULL when
 *   n_total == n_enc, packed / norms when n_enc == 0.
 * Errors: HLWQ_EINVAL (counts out of range: n_enc > n_total, more than R
 * tokens in the window, lds < n_total), HLWQ_EALIGN (window 16-byte,
 * packed 4-byte, norms / x / q 2-byte), HLWQ_EUNSUPPORTED (M > 64),
 * HLWQ_ECUDA.
 */
int hlwq_kv_quantize(const uint16_t* x, int64_t n, int64_t ldx, const float* codebook8, uint8_t* packed,
                     uint16_t* norms, void* stream);
int hlwq_kv_dequantize(const uint8_t* packed, const uint16_t* norms, const float* codebook8, int64_t n,
                       void* out, int odtype, void* stream);
int hlwq_kv_scores(const uint16_t* q, int64_t m, int64_t ldq, const uint8_t* packed, const uint16_t* norms,
                   const float* codebook8, int64_t n, float* scores, int64_t lds, void* stream);
int hlwq_kv_window_append(const uint16_t* x, int64_t t, int64_t ldx, uint16_t* window, int64_t R,
                          int64_t n_enc, int64_t n_total, const float* codebook8, uint8_t* packed,
                          uint16_t* norms, int64_t* n_enc_out, void* stream);
int hlwq_kv_scores_window(const uint16_t* q, int64_t m, int64_t ldq, const uint8_t* packed,
                          const uint16_t* norms, const float* codebook8, int64_t n_enc,
                          const uint16_t* window, int64_t R, int64_t n_total, float* scores, int64_t lds,
                          void* stream);

/*
 * TQ3 weights, the scalar case of HIGGS ("Qwen3.6-35B-A3B-TQ3-native", "What
 * TQ3 actually does" and "Files").  Per row and group g of 128 inputs (the
 * tail zero-padded), with one pair of sign vectors for every group:
 *   y      = s2 * (H128 (s1 * g)) / ||g||       (H128 the +-1 Sylvester matrix)
 *   code_j = nearest of the 8 Lloyd-Max centroids (ties to the lower index),
 *            decided in fp64
 *   gamma  = ||g|| / sqrt(||c[code]||^2 / 128)   (shape-gain norm; 0 for a zero
 *            group; ||c[code]||^2 = sum over levels l = 0..7 of
 *            count_l * c_l^2 in fp64, in that order), rounded to fp32
 *   w_hat  = gamma * s1 * (H128 (s2 * c[code])) / 128
 *   signs     device int8 [2][128]: row 0 = s1, row 1 = s2; a negative byte
 *             is -1, any other value +1
 *   codebook8 device float32 [8] (hlwq_lloyd_codebook(8))
 *   packed    [rows][NB][48]: code j of a group at bits [3j, 3j+3), LSB first
 *   norms     float32 [rows][NB] (gamma)
 * hlwq_tq3_quantize: W bf16 [rows][in] (row pitch in) -> packed, norms.
 * hlwq_tq3_dequantize: -> W_out [rows][in] (HLWQ_F32 or HLWQ_BF16).
 * hlwq_tq3_gemv: y[o] = sum_i x[i] w_hat[o][i] for one bf16 activation
 *   x [in], fp32 accumulation, evaluated in the rotated domain (x rotated
 *   once); one launch of thread-block clusters, no workspace.
 * Errors: HLWQ_EINVAL, HLWQ_EALIGN (packed / norms 4-byte, W / x / y 2-byte,
 * f32 outputs 4-byte alignment), HLWQ_EUNSUPPORTED (dtype), HLWQ_ECUDA.
 */
int hlwq_tq3_quantize(const uint16_t* W, int64_t rows, int64_t in, const int8_t* signs, const float* codebook8,
                      uint8_t* packed, float* norms, void* stream);
int hlwq_tq3_dequantize(const uint8_t* packed, const float* norms, const int8_t* signs, const float* codebook8,
                        int64_t rows, int64_t in, void* W_out, int odtype, void* stream);
int hlwq_tq3_gemv(const uint8_t* packed, const float* norms, const int8_t* signs, const float* codebook8,
                  int64_t out, int64_t in, const uint16_t* x, void* y, int ydtype, void* stream);

/*
 * TQ3 small-M GEMM (the same weights as hlwq_tq3_gemv, "a second encoding on
 * the same kernels"): Y[m][o] = sum_i X[m][i] w_hat[o][i], fp32 accumulation,
 * evaluated in the rotated domain, sum over groups b of gamma_b / 128 *
 * sum_j c[code_bj] xt_bj with xt_b = s2 * (H128 (s1 * x_b)).
 *   X  device bf16 [M][in], row pitch ldx >= in elements
 *   Y  device ydtype [M][out] (HLWQ_F32 or HLWQ_BF16), row pitch ldy >= out
 *   packed must be 16-byte aligned (its 48-byte groups are tensor-memory-
 *   access boxes); norms 4-byte; X, Y as hlwq_gemm.
 *   workspace  device, 16-byte aligned, ws_bytes >=
 *              hlwq_workspace_bytes(HLWQ_OP_TQ3_GEMM, out, in, M, 1, 0) when
 *              that is non-zero (a smaller workspace of at least the
 *              tensor-core path's minimum runs without its K split)
 * Paths: M >= 2 and in <= 8192 run the tcgen05 tensor-core kernel of
 * hlwq_gemm with the TQ3 decode (3-bit codes, fp32 gammas, 8 centroids, the
 * sign-vector rotation of X); M = 1, and rows longer than 8192, run the TQ3
 * GEMV once per token and need no workspace.
 * Errors: HLWQ_EINVAL, HLWQ_EALIGN, HLWQ_EUNSUPPORTED, HLWQ_EWORKSPACE,
 * HLWQ_ECUDA.
 */
int hlwq_tq3_gemm(const uint8_t* packed, const float* norms, const int8_t* signs, const float* codebook8,
                  int64_t out, int64_t in, int64_t M, const uint16_t* X, int64_t ldx, void* Y, int64_t ldy,
                  int ydtype, void* workspace, size_t ws_bytes, void* stream);

/*
 * Decode GEMV: y[o] = sum_i x[i] * w_hat[o][i], fp32 accumulation, without
 * materialising w_hat (the activation is rotated once per 128-block and dotted
 * with centroid values in the rotated domain).
 *   x  device bf16 [in];   y  device ydtype [out] (HLWQ_F32 or HLWQ_BF16)
 * Errors: HLWQ_EINVAL, HLWQ_EALIGN, HLWQ_EUNSUPPORTED, HLWQ_ECUDA.
 */
int hlwq_gemv(const uint8_t* packed, const uint16_t* norms, const float* codebook,
              int64_t out, int64_t in, const uint16_t* x, void* y, int ydtype, void* stream);

/*
 * hlwq_gemv with launch flags (bitwise or of hlwq_flags; 0 = hlwq_gemv).
 *   HLWQ_FLAG_WEIGHTS_STATIC: the caller guarantees that packed, norms and
 *     codebook are not written by any work enqueued earlier on `stream` that
 *     may still be running (true of the weights of a decode loop).  The kernel
 *     is then launched with programmatic stream serialisation: its set-up
 *     (first code loads, codebook, decode table) may run while the previous
 *     kernel on the stream is finishing; x is read and y written only after
 *     that kernel has completed and its writes are visible.
 * Errors: as hlwq_gemv; unknown flag bits -> HLWQ_EINVAL.
 */
int hlwq_gemv_ex(const uint8_t* packed, const uint16_t* norms, const float* codebook,
                 int64_t out, int64_t in, const uint16_t* x, void* y, int ydtype,
                 unsigned flags, void* stream);

/*
 * Small-M GEMM: Y[m][o] = sum_i X[m][i] * w_hat[o][i], fp32 accumulation.
 *   X  device bf16 [M][ldx] (ldx >= in, ldx % 8 == 0)
 *   Y  device ydtype [M][ldy] (ldy >= out)
 *   workspace  device, ws_bytes >= hlwq_workspace_bytes(HLWQ_OP_GEMM, out, in, M, 1, 0)
 * M = 1..4 runs on the CUDA-core decode path (one launch streams the weights for
 * up to four tokens); M >= 5 on the tensor-core path (workspace needed) when
 * in <= 8192.  Longer rows run on the CUDA-core path at every M and need no
 * workspace (hlwq_workspace_bytes reports 0 for them).
 * On the tensor-core path the reported size includes fp32 partials for
 * splitting the K range of the tiles of a partial last wave over two CTAs
 * each (added in a fixed order, so results do not depend on timing).  Any
 * workspace of at least 2 * M * 128 * ceil(in / 128) + 4 * M + 512 bytes is
 * accepted; below the reported size the call runs without that split.
 */
int hlwq_gemm(const uint8_t* packed, const uint16_t* norms, const float* codebook,
              int64_t out, int64_t in, int64_t M, const uint16_t* X, int64_t ldx,
              void* Y, int64_t ldy, int ydtype, void* workspace, size_t ws_bytes, void* stream);

/*
 * Routed MoE layer ("Qwen3.6-35B-A3B -- HLWQ Q5": 8 routed + 1 shared expert):
 *   ids, p   = top-k of router_logits[t] (ties: lower expert id), p = softmax
 *              over the k selected logits;
 *   g || u   = w_hat_gu[e] @ x_t  (rows [0,F) gate, [F,2F) up);
 *   h        = SiLU(g) * u (kept fp32);
 *   Y[t]     = sum_s p_s * w_hat_dn[ids_s] @ h  (+ shared expert, weight 1).
 *   gu_*  [E][2F][NBh][80] / [E][2F][NBh],  NBh = ceil(H / 128)
 *   dn_*  [E][H][NBf][80]  / [E][H][NBf],   NBf = ceil(F / 128)
 *   sh_*  the shared expert's matrices, or all four NULL for none
 *   router_logits device f32 [T][E];  X device bf16 [T][H];  Y device ydtype [T][H]
 *   topk_ids / topk_weights  device int32 / f32 [T][topk], or NULL
 * Errors: HLWQ_EINVAL (sizes, topk > E, topk > 32), HLWQ_EWORKSPACE, ...
 */
int hlwq_moe_gemv(const uint8_t* gu_packed, const uint16_t* gu_norms,
                  const uint8_t* dn_packed, const uint16_t* dn_norms,
                  const uint8_t* sh_gu_packed, const uint16_t* sh_gu_norms,
                  const uint8_t* sh_dn_packed, const uint16_t* sh_dn_norms,
                  const float* codebook, int64_t E, int64_t H, int64_t F, int64_t topk,
                  int64_t T, const float* router_logits, const uint16_t* X,
                  void* Y, int ydtype, int32_t* topk_ids, float* topk_weights,
                  void* workspace, size_t ws_bytes, void* stream);

/*
 * hlwq_moe_gemv with launch flags.  flags = 0 is hlwq_moe_gemv: the fused
 * two-kernel path while 4 * T * topk < 3 * E (fewer assignments than about
 * three quarters of the experts) and its shared memory fits, else the
 * grouped path.
 * HLWQ_FLAG_MOE_GROUPED selects the grouped path at any T.  The grouped path
 * (H and F up to 16384) reads each active expert's codes once for all its
 * tokens: routing and per-expert assignment lists; each assignment's token
 * gathered and rotated; gate_up as one grouped tcgen05 GEMM over (active
 * expert, 128-row tile), the shared expert from its own matrix in the same
 * launch; SiLU(g) * u rotated with the routing weight on its scale; down as a
 * grouped GEMM; a fixed-order combine of each token's partial outputs.
 * Same arguments, results (to rounding) and workspace; other flag bits are
 * HLWQ_EINVAL; HLWQ_EUNSUPPORTED when the grouped path is asked for with H or
 * F above 16384, or when neither path fits (very long rows and many tokens).
 */
int hlwq_moe_gemv_ex(const uint8_t* gu_packed, const uint16_t* gu_norms,
                     const uint8_t* dn_packed, const uint16_t* dn_norms,
                     const uint8_t* sh_gu_packed, const uint16_t* sh_gu_norms,
                     const uint8_t* sh_dn_packed, const uint16_t* sh_dn_norms,
                     const float* codebook, int64_t E, int64_t H, int64_t F, int64_t topk,
                     int64_t T, const float* router_logits, const uint16_t* X,
                     void* Y, int ydtype, int32_t* topk_ids, float* topk_weights,
                     void* workspace, size_t ws_bytes, unsigned flags, void* stream);

/*
 * Scratch bytes for an operation (0 when none is needed).
 *   HLWQ_OP_GEMM: a = out, b = in, c = M
 *   HLWQ_OP_MOE : a = H,   b = F,  c = T, E = experts, topk
 *   HLWQ_OP_TQ3_GEMM: a = out, b = in, c = M
 */
size_t hlwq_workspace_bytes(int op, int64_t a, int64_t b, int64_t c, int64_t E, int64_t topk);

/* Bytes of library-owned static device memory that hlwq_gemm_noalloc uses as
 * scratch (held by every GPU that loads the library until process exit). */
#define HLWQ_NOALLOC_SCRATCH_BYTES (4u * 1024u * 1024u + 64u * 1024u)

/*
 * hlwq_gemm without a workspace argument, for callers that cannot allocate
 * device memory (for example code that runs where allocation is forbidden, or
 * a plug-in whose host owns every allocation).  No counterpart in the paper:
 * it is the same computation as hlwq_gemm, taking its scratch from a static
 * device array of HLWQ_NOALLOC_SCRATCH_BYTES instead of a caller workspace.
 *   - Allocates nothing (no cudaMalloc / cudaFree, no allocating library call).
 *   - Requests whose smallest tensor-core workspace (about
 *     M * ceil(in / 128) * 256 bytes, see hlwq_gemm) exceeds
 *     HLWQ_NOALLOC_SCRATCH_BYTES return HLWQ_ESCRATCH; shapes that hlwq_gemm
 *     serves without a workspace (M <= 4, in > 8192) use no scratch.
 *   - Invalid arguments return hlwq_gemm's errors before any size is derived.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) and caches it; make that first call before any
 *     stream capture.
 *   - All calls on a device share the array: calls whose executions overlap on
 *     the GPU (other streams, other threads) race on it.
 * Arguments, layouts and the other errors are those of hlwq_gemm.
 */
int hlwq_gemm_noalloc(const uint8_t* packed, const uint16_t* norms, const float* codebook,
                      int64_t out, int64_t in, int64_t M, const uint16_t* X, int64_t ldx,
                      void* Y, int64_t ldy, int ydtype, void* stream);

/*
 * Failure-detection test hook.  No counterpart in the paper.  Only the test
 * build of the library (libhlwq_fault.so, compiled with HLWQ_FAULT_INJECTION)
 * implements it; the product library returns HLWQ_EUNSUPPORTED and its
 * kernels contain none of this.
 *   skip_tma  nonzero: the TMA producers of the GEMV, few-token, fused-MoE and
 *             tensor-core GEMM kernels issue no copies, so every consumer's
 *             bounded wait runs out (no copy is ever in flight); the kernel
 *             then raises HLWQ_DEVERR_TIMEOUT, frees its tensor memory and
 *             returns without writing a result it could not compute.
 *   wait_ns   the limit of every bounded wait (1 .. 2e9 ns; 2e9 is the
 *             product value).
 * Synchronises the current device first.  Errors: HLWQ_EINVAL (wait_ns),
 * HLWQ_ECUDA, HLWQ_EUNSUPPORTED (product build).
 */
int hlwq_fault_inject(unsigned int skip_tma, unsigned long long wait_ns);

/* Reads (after synchronising the current device) and clears the device error word. */
int hlwq_device_error(uint32_t* bits);

/* Static description of a status code. */
const char* hlwq_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int hlwq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HLWQ_H */
