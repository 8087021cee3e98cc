/*
 * sage.h -- C ABI of libsageb200.so: the SageAttention 8-bit attention forward
 * pass on NVIDIA B200 (sm_100a).
 *
 * What is computed (sources are the SageAttention web pages, cited by page
 * title and section):
 *
 *   - K smoothing: K's per-channel mean over the tokens of each
 *     (sequence, head) is subtracted before quantisation
 *     ("SageAttention v1/v2/v2++/v3 overview" (dtcms.com), SageAttention v1,
 *      bullet 1; "SageAttention -- brand new attention" (postsniper.ru),
 *      "SageAttention" bullet 1).
 *   - Per-block INT8 quantisation of Q and smoothed K, 128 tokens x D channels
 *     per block: delta = max|x| / 127, code = round(x / delta)
 *     (postsniper.ru page, quantisation intro steps 1-2; dtcms.com page,
 *      v1 item (1) "per-block").
 *   - INT8 QK^T on the tensor cores, dequantised by deltaQ * deltaK
 *     (postsniper.ru page, step 3), fused with the softmax scale.
 *   - FlashAttention-style tiled online softmax ("Attention机制优化：从
 *     FlashAttention到SageAttention的工程实践", section 3.1) over the 128-key
 *     blocks of the quantised K.
 *   - P.V in 16 bits (postsniper.ru page, "SageAttention" bullet 3), or P and V
 *     in FP8 E4M3 with the FP8 partial product of every 128-key block flushed
 *     into an FP32 accumulator (dtcms.com page, SageAttention 2 bullets 1, 3).
 *     With FP8 P.V, and with bf16 P in 16-bit P.V, p is formed against the
 *     running maximum of whole 128-key blocks; with fp16 P the maximum is
 *     taken per 64-key half-block and moves only when it rises by more than
 *     8 (base 2), which changes only the rounding of P (the rescale factors
 *     cancel in O / l).
 *   - The drop-in attention call shape q, k, v -> out over [B, H, N, D]
 *     ("sageattention in DeepSeek-VL2" (deepseek.csdn.net), step 2), plus a
 *     variable-length packed variant ("SageAttention complete guide"
 *     (jsqmd.com), API list: sageattn_varlen).
 *
 * Conventions for every function below:
 *   - Pointers are DEVICE pointers unless stated otherwise; the caller owns
 *     all memory.  The library allocates nothing.  Buffers must be 16-byte
 *     aligned and densely packed in the stated layout.
 *   - Compute calls are asynchronous on the given stream (cudaStream_t passed
 *     as void*; NULL = legacy default stream).  Argument errors are detected on
 *     the host before anything is launched and returned at once.  Errors found
 *     on the device (a wait that timed out, inconsistent cu_seqlens, K values
 *     outside the exact-mean range) are OR-ed into a status word at the start
 *     of the workspace and reported by sage_sync_status().
 *   - Workspace: every compute call takes (ws, ws_bytes).  Its first 256 bytes
 *     hold the status word and the attention kernel's work-item counters;
 *     sage_workspace_init() must zero them once before first use (each
 *     attention launch leaves the counters at zero again).  Calls on
 *     different streams must use different workspaces.
 *   - Layouts: dense tensors are [B, H, N, D] row-major; varlen tensors are
 *     [T, H, D] row-major with T = cu_seqlens[batch].  D is 64 or 128.
 *   - Causal masking is top-left aligned (query i sees keys j <= i), per
 *     sequence for varlen.
 */
#ifndef SAGE_B200_H
#define SAGE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SAGE_OK = 0,
  SAGE_ERR_INVALID_ARG = 1,   /* bad size, null/misaligned pointer, bad enum   */
  SAGE_ERR_UNSUPPORTED = 2,   /* valid request this library does not implement */
  SAGE_ERR_WORKSPACE = 3,     /* ws_bytes smaller than the size function says  */
  SAGE_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed             */
  SAGE_ERR_TIMEOUT = 5,       /* a device-side wait gave up (status word)      */
  SAGE_ERR_BAD_SEQLENS = 6,   /* cu_seqlens not monotone / not matching T      */
  SAGE_ERR_RANGE = 7          /* a K element is non-finite or |k| >= 65536     */
} sage_status_t;

typedef enum { SAGE_F16 = 0, SAGE_BF16 = 1, SAGE_F32 = 2 /* outputs only */ } sage_dtype_t;

typedef enum {
  SAGE_PV_FP16 = 0, /* P.V with P rounded to V's 16-bit type, fp32 accumulate   */
  SAGE_PV_FP8 = 1   /* P, V in FP8 E4M3, fp32 two-level accumulation: the FP8
                       partial of each 128-key block is flushed into fp32   */
} sage_pv_mode_t;

/* Granularity of the Q and K deltas ("SageAttention v1/v2/v2++/v3 overview",
 * SageAttention v1 item (1): per-block or per-token quantisation of q, k),
 * and Q smoothing (same page, SageAttention2 bullet 2). */
typedef enum {
  SAGE_QK_PER_BLOCK = 0,         /* one delta per 128-token block (and head)     */
  SAGE_QK_PER_TOKEN = 1,         /* one delta per token                           */
  SAGE_QK_PER_BLOCK_SMOOTH_Q = 2 /* per block, each Q block minus its channel
                                    mean before quantisation; the mean's part of
                                    the logit, mean . k~_j, added back per key    */
} sage_qk_gran_t;

/* Token count of one quantisation block and of one attention key/query tile. */
#define SAGE_BLOCK 128

/* ---------------------------------------------------------------- sizes -- */

/* Workspace bytes for sage_attn_fwd on a dense [B,H,N,D] problem (holds the
 * status word, the INT8/FP8 codes and scales, and reduction scratch).
 * Returns 0 for arguments sage_attn_fwd would reject. */
size_t sage_workspace_bytes(int B, int H, int N, int D, int pv_mode);

/* Workspace bytes for sage_attn_fwd_varlen with `batch` sequences packed into
 * total_tokens rows.  Sized for the worst case over all length splits. */
size_t sage_workspace_bytes_varlen(int total_tokens, int batch, int H, int D, int pv_mode);

/* Workspace bytes for sage_quantize / sage_attn_quantized alone (status word
 * plus reduction scratch; the codes live in caller buffers). */
size_t sage_scratch_bytes(int B, int H, int D);

/* Zero the status word of a workspace (stream-ordered).  Call once after
 * allocating a workspace, before its first use. */
sage_status_t sage_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Wait for `stream`, then read and clear the workspace's status word.
 * Returns SAGE_OK or the first device-side error recorded since the last
 * call, in the precedence TIMEOUT > BAD_SEQLENS > RANGE. */
sage_status_t sage_sync_status(void* ws, void* stream);

/* Human-readable name of a status code (static string). */
const char* sage_status_string(sage_status_t s);

/* Message of the last CUDA failure that made a call on this host thread
 * return SAGE_ERR_CUDA (thread-local, static storage; "" if none). */
const char* sage_last_cuda_error(void);

/* ------------------------------------------------------ full forward pass -- */

/*
 * out = SageAttention(q, k, v) for dense [B, H, N, D] tensors.
 *   q, k, v : 16-bit inputs of type in_dt (SAGE_F16 or SAGE_BF16).
 *   out     : [B, H, N, D] of type out_dt (SAGE_F16, SAGE_BF16, or SAGE_F32
 *             for an unrounded fp32 result).
 *   causal  : nonzero for top-left causal masking.
 *   sm_scale: softmax scale; <= 0 selects 1/sqrt(D).
 *   pv_mode : SAGE_PV_FP16 or SAGE_PV_FP8.
 *   ws      : workspace of at least sage_workspace_bytes(B, H, N, D, pv_mode).
 * Runs the quantisation kernels then the fused attention kernel on `stream`.
 * Limits: 1 <= N <= 2^22, D in {64, 128}, B*H <= 65535.
 */
sage_status_t sage_attn_fwd(const void* q, const void* k, const void* v, void* out,
                            int in_dt, int out_dt, int B, int H, int N, int D, int causal,
                            float sm_scale, int pv_mode, void* ws, size_t ws_bytes,
                            void* stream);

/*
 * General dense forward pass: grouped-query heads (Hkv divides H; Hkv = H
 * without grouping, see sage_attn_fwd_gqa) and the Q/K delta granularity
 * qk_gran (sage_qk_gran_t).  With SAGE_QK_PER_TOKEN every query row and key
 * has its own delta = max over its D channels / 127, and the scores are
 * dequantised as y = fp32(S_ij * deltaK_j), arg = fmaf(y, fp32(deltaQ_i *
 * sm_scale * log2 e), -m) (per block: c = fp32(fp32(deltaQ*deltaK) * kappa),
 * arg = fmaf(S, c, -m)).
 * With SAGE_QK_PER_BLOCK_SMOOTH_Q the codes of query block I are those of
 * fp32(q - qmean_I), qmean_I the exact channel mean of the block's rows (the
 * K mean's definition), and the scaled logit is y = fmaf(S, c, b_Ij) with
 * b_Ij = fp32(kappa * qmean_I . fp32(k_j - kmean)), the dot product as fp32
 * fused multiply-adds in channel order (within (D + 2) 2^-24 kappa
 * sum_d |qmean_d k~_jd| of the exact value), then arg = y - m.
 * Its workspace also holds qmean (B*H*NB*D floats) and b for R query blocks
 * at a time (B*H*R*NB*128 floats): the call computes b of query blocks
 * [0, R), attends those query tiles, then the next R, so that the workspace
 * grows with N*R rather than N^2/128.  sage_workspace_bytes_ex gives R = as
 * many blocks as fit 256 MiB (at least 2, at most NB).  A call takes R = the
 * most blocks its ws_bytes holds, an even count unless it is all NB, and
 * fails with SAGE_ERR_WORKSPACE below R = 2.  The output does not depend on
 * R: every term and every query tile is computed as in one pass.
 *   ws : at least sage_workspace_bytes_ex(B, H, Hkv, N, D, pv_mode, qk_gran),
 *        or, with Q smoothing, sage_workspace_bytes_sq(..., R) for a chosen R.
 * sage_attn_fwd(...) = sage_attn_fwd_ex(..., Hkv = H, ..., SAGE_QK_PER_BLOCK).
 */
size_t sage_workspace_bytes_ex(int B, int H, int Hkv, int N, int D, int pv_mode, int qk_gran);
/* Workspace of sage_attn_fwd_ex with SAGE_QK_PER_BLOCK_SMOOTH_Q whose mean term
 * holds q_blocks_per_chunk query blocks (R above; clamped to NB; an even
 * count when below NB).  Returns 0 for invalid arguments. */
size_t sage_workspace_bytes_sq(int B, int H, int Hkv, int N, int D, int pv_mode,
                               int q_blocks_per_chunk);
sage_status_t sage_attn_fwd_ex(const void* q, const void* k, const void* v, void* out,
                               int in_dt, int out_dt, int B, int H, int Hkv, int N, int D,
                               int causal, float sm_scale, int pv_mode, int qk_gran, void* ws,
                               size_t ws_bytes, void* stream);

/*
 * Grouped-query variant: q and out are [B, H, N, D]; k and v are
 * [B, Hkv, N, D] with H a multiple of Hkv, and query head h reads key/value
 * head h / (H / Hkv) of its batch -- the grouping of the "sageattention in
 * DeepSeek-VL2" page's attention code, which repeats each key/value head for
 * H / Hkv consecutive query heads (repeat_kv) before calling attention.  The
 * result equals sage_attn_fwd on the repeated k, v (K means, deltas and V
 * scales are per key/value head, so repeating changes none of them) without
 * materialising the repeat.
 *   ws : at least sage_workspace_bytes_gqa(B, H, Hkv, N, D, pv_mode).
 * Other arguments as sage_attn_fwd; Hkv = H is sage_attn_fwd.  An Hkv that is
 * not a divisor of H returns SAGE_ERR_INVALID_ARG.
 */
size_t sage_workspace_bytes_gqa(int B, int H, int Hkv, int N, int D, int pv_mode);
sage_status_t sage_attn_fwd_gqa(const void* q, const void* k, const void* v, void* out,
                                int in_dt, int out_dt, int B, int H, int Hkv, int N, int D,
                                int causal, float sm_scale, int pv_mode, void* ws,
                                size_t ws_bytes, void* stream);

/*
 * Variable-length packed variant: `batch` sequences, sequence s occupying rows
 * cu_seqlens[s] .. cu_seqlens[s+1]-1 of the [T, H, D] tensors q, k, v, out.
 *   cu_seqlens  : DEVICE int32 [batch + 1], cu_seqlens[0] = 0, non-decreasing,
 *                 cu_seqlens[batch] = total_tokens; every length <= max_seqlen.
 *                 Violations are detected on the device (SAGE_ERR_BAD_SEQLENS
 *                 via sage_sync_status) and leave `out` unspecified.
 *   max_seqlen  : an upper bound on the sequence lengths (used for validation).
 * Every sequence has its own K mean, its own quantisation blocks and (FP8) its
 * own V channel scales.  Other arguments as sage_attn_fwd.
 */
sage_status_t sage_attn_fwd_varlen(const void* q, const void* k, const void* v, void* out,
                                   int in_dt, int out_dt, const int32_t* cu_seqlens, int batch,
                                   int max_seqlen, int total_tokens, int H, int D, int causal,
                                   float sm_scale, int pv_mode, void* ws, size_t ws_bytes,
                                   void* stream);

/*
 * Grouped-query variant of sage_attn_fwd_varlen: q, out are [T, H, D]; k, v
 * are [T, Hkv, D] with Hkv dividing H; query head h reads key/value head
 * h / (H / Hkv) of its sequence (the repeat_kv grouping, see
 * sage_attn_fwd_gqa).  ws: at least sage_workspace_bytes_varlen_gqa(...).
 */
size_t sage_workspace_bytes_varlen_gqa(int total_tokens, int batch, int H, int Hkv, int D,
                                       int pv_mode);
sage_status_t sage_attn_fwd_varlen_gqa(const void* q, const void* k, const void* v, void* out,
                                       int in_dt, int out_dt, const int32_t* cu_seqlens,
                                       int batch, int max_seqlen, int total_tokens, int H,
                                       int Hkv, int D, int causal, float sm_scale, int pv_mode,
                                       void* ws, size_t ws_bytes, void* stream);

/*
 * General variable-length forward pass: grouped-query heads (as
 * sage_attn_fwd_varlen_gqa) and the Q/K delta granularity qk_gran (as
 * sage_attn_fwd_ex; per token, every packed token has its own Q and K delta;
 * with Q smoothing every sequence's Q blocks take their own means and the
 * mean term covers that sequence's keys).
 *   ws : at least sage_workspace_bytes_varlen_ex(...), or for
 *        SAGE_QK_PER_BLOCK_SMOOTH_Q sage_workspace_bytes_varlen_sq(...), whose
 *        size depends on max_seqlen (the mean terms take at most
 *        4 * H * ceil(max_seqlen/128) * (total_tokens + 128*batch) bytes).
 * sage_workspace_bytes_varlen_ex returns 0 for SAGE_QK_PER_BLOCK_SMOOTH_Q.
 */
size_t sage_workspace_bytes_varlen_ex(int total_tokens, int batch, int H, int Hkv, int D,
                                      int pv_mode, int qk_gran);
size_t sage_workspace_bytes_varlen_sq(int total_tokens, int batch, int max_seqlen, int H,
                                      int Hkv, int D, int pv_mode);
sage_status_t sage_attn_fwd_varlen_ex(const void* q, const void* k, const void* v, void* out,
                                      int in_dt, int out_dt, const int32_t* cu_seqlens, int batch,
                                      int max_seqlen, int total_tokens, int H, int Hkv, int D,
                                      int causal, float sm_scale, int pv_mode, int qk_gran,
                                      void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------ the two stages, separately -- */

/*
 * Smoothing and INT8 quantisation of Q and K alone (no V) for a dense
 * [B, H, N, D] problem: K's per-channel mean over the N tokens of each head is
 * subtracted ("SageAttention v1/v2/v2++/v3 overview" (dtcms.com),
 * SageAttention v1 bullet 1), then every 128-token block of Q and of the
 * smoothed K is quantised with delta = max|x| / 127, code = round(x / delta)
 * ("SageAttention -- brand new attention" (postsniper.ru), quantisation intro
 * steps 1-2).  This is the first stage of the qk_int8 entry points in the
 * "SageAttention complete guide" API list.
 *   q, k    : [B, H, N, D] 16-bit of type in_dt (SAGE_F16 or SAGE_BF16).
 *   q_codes, k_codes, q_scale, k_scale, k_mean : as sage_quantize.
 *   ws      : at least sage_scratch_bytes(B, H, D).
 * Equal to sage_quantize with pv_mode SAGE_PV_FP16 (no V outputs); errors as
 * sage_quantize (SAGE_ERR_RANGE through sage_sync_status for a K element
 * outside the exact-mean range).
 */
sage_status_t sage_quant_qk(const void* q, const void* k, int in_dt, int B, int H, int N, int D,
                            int8_t* q_codes, float* q_scale, int8_t* k_codes, float* k_scale,
                            float* k_mean, void* ws, size_t ws_bytes, void* stream);

/*
 * Stage 1 (smoothing + quantisation) of a dense problem into caller buffers:
 *   q_codes, k_codes : int8 [B, H, NP, D], NP = ceil(N/128)*128; padding rows 0.
 *   q_scale, k_scale : fp32 [B, H, NP/128], the per-block deltas (max|x|/127).
 *   k_mean           : fp32 [B, H, D], the per-channel K mean subtracted.
 *   v_codes          : FP8 mode: E4M3 bytes [B, H, N, D]; else may be NULL.
 *   v_scale          : FP8 mode: fp32 [B, H, D], per-channel max|v|/448.
 *   ws               : at least sage_scratch_bytes(B, H, D).
 * Quantiser arithmetic (binary32, round-half-to-even): s = 127/max|x| per
 * block, code = clamp(rint(x*s), -127, 127); a block with max|x| = 0 gets
 * delta 0 and zero codes.  K mean: each k is put on the 2^-24 grid, summed
 * exactly in int64 and divided once in fp64, m = fp32(sum / (N * 2^24)).
 */
sage_status_t sage_quantize(const void* q, const void* k, const void* v, int in_dt, int B, int H,
                            int N, int D, int pv_mode, int8_t* q_codes, float* q_scale,
                            int8_t* k_codes, float* k_scale, float* k_mean, uint8_t* v_codes,
                            float* v_scale, void* ws, size_t ws_bytes, void* stream);

/*
 * Stage 2 (fused INT8 QK^T + online softmax + P.V) of a dense problem from the
 * buffers sage_quantize wrote.  v is the original 16-bit V (FP16 mode; of type
 * v_dt) -- ignored in FP8 mode, where v_codes / v_scale are used instead.
 * ws: at least sage_scratch_bytes(B, H, D).  Other arguments as sage_attn_fwd.
 */
sage_status_t sage_attn_quantized(const int8_t* q_codes, const float* q_scale,
                                  const int8_t* k_codes, const float* k_scale, const void* v,
                                  const uint8_t* v_codes, const float* v_scale, void* out,
                                  int v_dt, int out_dt, int B, int H, int N, int D, int causal,
                                  float sm_scale, int pv_mode, void* ws, size_t ws_bytes,
                                  void* stream);

/*
 * The two stages for grouped-query heads and either delta granularity (see
 * sage_attn_fwd_ex).  Layouts as sage_quantize with H query heads for Q and
 * Hkv key/value heads for K, k_mean and (FP8) V; with SAGE_QK_PER_TOKEN the
 * deltas are fp32 [B, H, NP] (Q) and [B, Hkv, NP] (K), one per code row,
 * padding rows 0.  sage_attn_quantized_ex needs k_scale 16-byte aligned (the
 * kernel copies 128 deltas at a time).  ws: at least sage_scratch_bytes(B, H,
 * D), which covers every Hkv <= H (SAGE_ERR_WORKSPACE when too small).
 * SAGE_QK_PER_BLOCK_SMOOTH_Q has its own two stages (sage_quantize_sq,
 * sage_attn_quantized_sq); these two return SAGE_ERR_INVALID_ARG for it.
 */
sage_status_t sage_quantize_ex(const void* q, const void* k, const void* v, int in_dt, int B,
                               int H, int Hkv, int N, int D, int pv_mode, int qk_gran,
                               int8_t* q_codes, float* q_scale, int8_t* k_codes, float* k_scale,
                               float* k_mean, uint8_t* v_codes, float* v_scale, void* ws,
                               size_t ws_bytes, void* stream);
sage_status_t sage_attn_quantized_ex(const int8_t* q_codes, const float* q_scale,
                                     const int8_t* k_codes, const float* k_scale, const void* v,
                                     const uint8_t* v_codes, const float* v_scale, void* out,
                                     int v_dt, int out_dt, int B, int H, int Hkv, int N, int D,
                                     int causal, float sm_scale, int pv_mode, int qk_gran,
                                     void* ws, size_t ws_bytes, void* stream);

/*
 * The two stages with Q smoothing (SAGE_QK_PER_BLOCK_SMOOTH_Q, dense).
 * sage_quantize_sq writes, besides the outputs of sage_quantize_ex with
 * per-block deltas,
 *   q_mean : fp32 [B, H, NB, D], the block means of Q;
 *   q_bias : fp32 [B, H, NB, NP], q_bias[b,h,I,j] = fp32(kappa * q_mean[b,h,I]
 *            . fp32(k_j - k_mean)) (fp32 FMAs in channel order) for key j of the
 *            key/value head of h, kappa
 *            = fp32(sm_scale * log2 e); keys j >= N give 0; with causal != 0
 *            the blocks I < j/128, which the mask hides, are not written.
 *            16-byte aligned.
 * sm_scale and causal are those the attention stage will use.
 * sage_attn_quantized_sq takes the codes and deltas with q_bias.  ws: as
 * sage_quantize_ex / sage_attn_quantized_ex.
 */
sage_status_t sage_quantize_sq(const void* q, const void* k, const void* v, int in_dt, int B,
                               int H, int Hkv, int N, int D, int pv_mode, int causal,
                               float sm_scale, int8_t* q_codes, float* q_scale, float* q_mean,
                               int8_t* k_codes, float* k_scale, float* k_mean, uint8_t* v_codes,
                               float* v_scale, float* q_bias, void* ws, size_t ws_bytes,
                               void* stream);
sage_status_t sage_attn_quantized_sq(const int8_t* q_codes, const float* q_scale,
                                     const int8_t* k_codes, const float* k_scale,
                                     const float* q_bias, const void* v, const uint8_t* v_codes,
                                     const float* v_scale, void* out, int v_dt, int out_dt, int B,
                                     int H, int Hkv, int N, int D, int causal, float sm_scale,
                                     int pv_mode, void* ws, size_t ws_bytes, void* stream);

/*
 * Stage 1 for a packed varlen batch.  Layouts (TB = number of 128-token blocks
 * over all sequences = sum_s ceil(n_s/128); blocks of sequence s start at
 * block index blk_off[s] = sum_{s'<s} ceil(n_s'/128)):
 *   q_codes, k_codes : int8 [H, TBmax*128, D] with TBmax = total_tokens/128 +
 *                      batch (upper bound of TB); block b of sequence s of head
 *                      h at rows (blk_off[s] + b)*128 ...
 *   q_scale, k_scale : fp32 [H, TBmax].
 *   k_mean           : fp32 [batch, H, D].
 *   v_codes          : FP8 mode: E4M3 [T, H, D]; v_scale fp32 [batch, H, D].
 *   ws               : at least sage_workspace_bytes_varlen(...) (holds the
 *                      per-sequence schedule as well as the scratch).
 */
sage_status_t sage_quantize_varlen(const void* q, const void* k, const void* v, int in_dt,
                                   const int32_t* cu_seqlens, int batch, int max_seqlen,
                                   int total_tokens, int H, int D, int pv_mode, int8_t* q_codes,
                                   float* q_scale, int8_t* k_codes, float* k_scale,
                                   float* k_mean, uint8_t* v_codes, float* v_scale, void* ws,
                                   size_t ws_bytes, void* stream);

/*
 * Stage 1 of a dense problem without a workspace: the same smoothing and
 * quantisation, outputs and layouts as sage_quantize, but its reduction
 * scratch (exact K channel sums, V channel maxima, status word) lives in a
 * fixed SAGE_NOALLOC_SCRATCH_BYTES array of device memory inside the library.
 * The SageAttention pages have no counterpart of this entry point; it exists
 * for callers that may not allocate device memory and cannot pass a
 * workspace (for instance an extension whose host application owns every
 * device allocation, or a path that must not pay cudaMalloc's implicit
 * synchronisation).  It allocates nothing.
 *   status_out : optional DEVICE uint32; cleared by the call, then OR-ed with
 *                4 when a K element is non-finite or |k| >= 65536, and with 1
 *                when a bounded device-side wait gave up (the likeliest sign
 *                of two calls racing on the shared array).  The outputs are
 *                then unspecified.  NULL hides both errors: pass a word unless
 *                the inputs and the call's exclusive use of the array are
 *                known to be fine.
 * Limits and rules:
 *   - B*H*D <= SAGE_NOALLOC_MAX_BHD, else SAGE_ERR_WORKSPACE (nothing runs).
 *   - Every call shares the one array (per device) and it keeps the last
 *     call's contents; calls whose GPU work overlaps in time (other streams,
 *     other host threads) race on it.
 *   - The first call on a device looks the array's address up with that
 *     device current; make that first call before any stream capture.
 *   - Each GPU that loads the library holds the array until the process exits.
 */
#define SAGE_NOALLOC_SCRATCH_BYTES (1 << 20)
#define SAGE_NOALLOC_MAX_BHD 65536
sage_status_t sage_quantize_noalloc(const void* q, const void* k, const void* v, int in_dt, int B,
                                    int H, int N, int D, int pv_mode, int8_t* q_codes,
                                    float* q_scale, int8_t* k_codes, float* k_scale,
                                    float* k_mean, uint8_t* v_codes, float* v_scale,
                                    uint32_t* status_out, void* stream);

/* ------------------------------------------------------------ diagnostics -- */

/*
 * The int32 QK^T scores of the attention kernel itself (postsniper.ru page,
 * "SageAttention" bullet 1: QK^T in INT8).  Runs sage_attn_quantized (same
 * arguments, same output `out`) with the fused attention kernel built to also
 * store every 64-key sub-tile of S it computes, exactly as read from tensor
 * memory before dequantisation, into
 *   s_out : DEVICE int32 [B*H, NP, NP], NP = ceil(N/128)*128,
 *           s_out[bh][i][j] = sum_d q_codes[bh][i][d] * k_codes[bh][j][d]
 *           for query rows i < N and the keys j of every sub-tile the kernel
 *           visits (non-causal: j < ceil(N/64)*64; causal: additionally
 *           j < (i/128 + 1)*128).  Other entries are not written.
 * Diagnostic: fp16 V (SAGE_PV_FP16 with v_dt SAGE_F16) or SAGE_PV_FP8 only,
 * else SAGE_ERR_UNSUPPORTED.
 */
sage_status_t sage_attn_quantized_dump_s(const int8_t* q_codes, const float* q_scale,
                                         const int8_t* k_codes, const float* k_scale,
                                         const void* v, const uint8_t* v_codes,
                                         const float* v_scale, void* out, int v_dt, int out_dt,
                                         int B, int H, int N, int D, int causal, float sm_scale,
                                         int pv_mode, int32_t* s_out, void* ws, size_t ws_bytes,
                                         void* stream);

/*
 * INT8 QK^T tiles by a separate one-tile kernel with the attention kernel's
 * TMA loads and tcgen05 (kind::i8) instructions, as one M128 x N128 product:
 * for each of n_tiles requests tiles[3*t .. 3*t+2] = (bh, I, J) (host int32
 * array), writes S[r][c] = sum_d q_codes[bh][128 I + r][d] *
 * k_codes[bh][128 J + c][d] as int32 into s_out + t*128*128.  q_codes and
 * k_codes are the dense [B*H, NP, D] code arrays of sage_quantize.
 */
sage_status_t sage_qk_int8_tiles(const int8_t* q_codes, const int8_t* k_codes, int BH, int NP,
                                 int D, const int32_t* tiles, int n_tiles, int32_t* s_out,
                                 void* ws, size_t ws_bytes, void* stream);

/*
 * Full-precision attention rows, the reference of the accuracy-driven choice
 * between 16-bit and FP8 P.V ("SageAttention v1/v2/v2++/v3 overview",
 * SageAttention v1: a faster variant serves a layer only where its cosine
 * similarity to full-precision attention exceeds 99.8 %).
 *   q : [B, H, N, D], k, v : [B, Hkv, N, D] (Hkv divides H; query head h
 *       reads key/value head h / (H / Hkv)), 16-bit of type in_dt, DEVICE.
 *   rows : DEVICE int32 [n_rows][3] = (b, h, i) query rows to evaluate.
 *   out  : DEVICE fp32 [n_rows][D], softmax(sm_scale q_i K^T) V in fp32
 *          (causal: keys j <= i); a row outside the input gets NaN.
 * No quantisation: this is the plain definition, for calibration and checks,
 * not a hot path.  sm_scale <= 0 selects 1/sqrt(D).
 */
sage_status_t sage_attn_ref_rows(const void* q, const void* k, const void* v, int in_dt, int B,
                                 int H, int Hkv, int N, int D, int causal, float sm_scale,
                                 const int32_t* rows, int n_rows, float* out, void* stream);

/*
 * Self-test of device-side failure reporting: launches one CTA that waits on
 * a barrier nothing signals, gives up after wait_cycles (1 .. 2^31) SM clock
 * cycles and records SAGE_ERR_TIMEOUT in the workspace's status word, which
 * the next sage_sync_status() returns.  The GPU stays usable.  This is the
 * same bounded-wait path every pipeline wait of the attention kernel takes.
 */
sage_status_t sage_selftest_wait_timeout(long long wait_cycles, void* ws, size_t ws_bytes,
                                         void* stream);

/*
 * Self-test of the fused attention kernel's own failure path: runs
 * sage_attn_quantized (same arguments) with every bounded wait limited to
 * wait_cycles (1 .. 2^31) SM clock cycles, and with skip_k_stage = s > 0 every
 * CTA leaves the K tile of its s-th pipeline stage unloaded, so the barrier
 * of that stage never completes.  The waiting role gives up, records
 * SAGE_ERR_TIMEOUT in the workspace's status word (returned by the next
 * sage_sync_status), and every role of the CTA falls through to the teardown,
 * which waits (bounded) for the CTA's own copies and MMAs and frees its tensor
 * memory: the GPU and the workspace stay usable and `out` is unspecified.
 * skip_k_stage = 0 runs the normal kernel with the shorter limit.
 */
sage_status_t sage_selftest_attn_timeout(const int8_t* q_codes, const float* q_scale,
                                         const int8_t* k_codes, const float* k_scale,
                                         const void* v, const uint8_t* v_codes,
                                         const float* v_scale, void* out, int v_dt, int out_dt,
                                         int B, int H, int N, int D, int causal, float sm_scale,
                                         int pv_mode, long long wait_cycles, int skip_k_stage,
                                         void* ws, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SAGE_B200_H */
