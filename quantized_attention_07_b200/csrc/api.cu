// C ABI of libsageb200.so: argument validation, workspace layout, launches,
// and the device status word.  Nothing here allocates device memory; every
// buffer is the caller's.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>

#include "common.cuh"

namespace sage {

cudaError_t launch_varlen_prep(const int32_t* cu, int batch, int max_seqlen, int total_tokens,
                               int32_t* blk_off, int32_t* pair_off, uint32_t* status,
                               cudaStream_t st, long long* sq_off = nullptr);
cudaError_t launch_quant(const SeqLayout& L, dim3 grid, int D, bool bf16, bool fp8,
                         const void* q, const void* k, const void* v, int8_t* q_codes,
                         float* q_scale, int8_t* k_codes, float* k_scale, float* k_mean,
                         uint8_t* v_codes, float* v_scale, unsigned long long* k_sum,
                         uint32_t* v_amax, uint32_t* status, unsigned int* sync, int parts,
                         int per_token, cudaStream_t st);
cudaError_t launch_quant_q_smooth(const SeqLayout& L, dim3 grid, int D, bool bf16,
                                  const void* q, int8_t* q_codes, float* q_scale, float* q_mean,
                                  uint32_t* status, cudaStream_t st);
cudaError_t launch_q_smooth_bias(const SeqLayout& L, dim3 grid, int H, int Hkv, int D, bool bf16,
                                 int causal, float kappa, const void* k, const float* k_mean,
                                 const float* q_mean, float* bias, long long head_stride,
                                 const long long* sq_off, int qb0, int qrows, cudaStream_t st);
cudaError_t launch_qk_tiles(const int8_t* qc, const int8_t* kc, int BH, int NP, int D,
                            const int32_t* tiles, int n, int32_t* out, uint32_t* status,
                            cudaStream_t st);
}  // namespace sage

#include "attn_launch.cuh"

using namespace sage;

namespace {

thread_local char g_last_error[256] = "";

sage_status_t cuda_fail(cudaError_t e, const char* what) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s", what, cudaGetErrorString(e));
  return SAGE_ERR_CUDA;
}

// Workspace header: the status word at byte 0 and the attention kernel's two
// work-scheduler counters at kSchedOff (zeroed by sage_workspace_init; every
// attention launch leaves them at zero).
constexpr size_t kHeader = 256;
constexpr size_t kSchedOff = 64;
constexpr long long kMaxN = 1LL << 22;

size_t al(size_t x) { return (x + 255) & ~size_t(255); }
bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
bool in_dtype_ok(int dt) { return dt == SAGE_F16 || dt == SAGE_BF16; }
bool out_dtype_ok(int dt) { return dt == SAGE_F16 || dt == SAGE_BF16 || dt == SAGE_F32; }

float kappa_of(float sm_scale, int D) {
  const float s = sm_scale > 0.0f ? sm_scale : (float)(1.0 / std::sqrt((double)D));
  return (float)((double)s * 1.4426950408889634);  // fp32(sm_scale * log2 e)
}

// Workspace layout.  Offsets in bytes from the workspace base.
struct Layout {
  size_t k_sum, v_amax, sync, sync_q, blk_off, pair_off;  // scratch
  size_t q_codes, k_codes, q_scale, k_scale, k_mean;   // quantised operands
  size_t v_codes, v_scale;
  size_t q_mean, q_bias, sq_off;                      // Q smoothing
  int sq_rows;                                        // dense Q smoothing: query blocks per head in q_bias
  long long bias_head_stride;                         // varlen Q smoothing: floats per head
  size_t scratch_end, total;
};

// Dense layout for H query heads and Hkv key/value heads per batch (Hkv = H
// without grouping).  sync: work counter + one completion counter per
// key/value head for the launch that quantises K (and Q when Hkv = H);
// sync_q: the work counter of the separate Q launch when Hkv < H.
// gran: a sage_qk_gran_t (per-token deltas; Q smoothing adds the block means
// and the per-key mean term of sq_rows query blocks per head, by default as
// many as fit kSqTermCap bytes, at least 2 and at most all of them).
constexpr size_t kSqTermCap = size_t(256) << 20;

int sq_rows_default(size_t BH, size_t NB) {
  const size_t row = BH * NB * BLK * 4, fit = (kSqTermCap / row) & ~size_t(1);
  return (int)std::min(NB, std::max<size_t>(2, fit));
}

Layout dense_layout(int B, int H, int N, int D, bool fp8, int Hkv, int gran = SAGE_QK_PER_BLOCK,
                    int sq_rows = 0) {
  const bool per_token = gran == SAGE_QK_PER_TOKEN;
  const size_t BH = (size_t)B * H, BK = (size_t)B * Hkv, NB = ((size_t)N + BLK - 1) / BLK,
               NP = NB * BLK, NS = per_token ? NP : NB;  // deltas per head
  Layout L{};
  size_t o = kHeader;
  L.k_sum = o; o += al(BK * D * 8);
  L.v_amax = o; o += al(BK * D * 4);
  L.sync = o; o += al((BK + 1) * 4);
  L.sync_q = o; o += al(4);
  L.scratch_end = o;
  L.q_codes = o; o += al(BH * NP * D);
  L.k_codes = o; o += al(BK * NP * D);
  L.q_scale = o; o += al(BH * NS * 4);
  L.k_scale = o; o += al(BK * NS * 4);
  L.k_mean = o; o += al(BK * D * 4);
  if (fp8) {
    L.v_codes = o; o += al(BK * (size_t)N * D);
    L.v_scale = o; o += al(BK * D * 4);
  }
  if (gran == SAGE_QK_PER_BLOCK_SMOOTH_Q) {
    L.sq_rows = sq_rows > 0 ? (int)std::min<size_t>(sq_rows, NB) : sq_rows_default(BH, NB);
    L.q_mean = o; o += al(BH * NB * D * 4);
    L.q_bias = o; o += al(BH * (size_t)L.sq_rows * NP * 4);
  }
  L.total = o;
  return L;
}
Layout dense_layout(int B, int H, int N, int D, bool fp8) { return dense_layout(B, H, N, D, fp8, H); }

long long tb_max(long long T, long long batch) { return (T + (BLK - 1) * batch) / BLK; }
long long pair_max(long long T, long long batch) { return (T + (2 * BLK - 1) * batch) / (2 * BLK); }

// Varlen layout for H query heads and Hkv key/value heads (Hkv = H without
// grouping): Q codes / deltas over H heads, everything of K and V over Hkv.
// gran: a sage_qk_gran_t; Q smoothing needs max_seqlen, which bounds the
// per-head size of the mean term: sum_s nb_s^2 <= ceil(max_seqlen/128) * TB.
Layout varlen_layout(int T, int batch, int H, int D, bool fp8, int Hkv = 0,
                     int gran = SAGE_QK_PER_BLOCK, int max_seqlen = 0) {
  if (Hkv <= 0) Hkv = H;
  const bool per_token = gran == SAGE_QK_PER_TOKEN, sq = gran == SAGE_QK_PER_BLOCK_SMOOTH_Q;
  const size_t SH = (size_t)batch * Hkv, TB = (size_t)tb_max(T, batch);
  const size_t NS = per_token ? TB * BLK : TB;  // deltas per head
  Layout L{};
  size_t o = kHeader;
  L.k_sum = o; o += al(SH * D * 8);
  L.v_amax = o; o += al(SH * D * 4);
  L.sync = o; o += al(4);
  L.blk_off = o; o += al(((size_t)batch + 1) * 4);
  L.pair_off = o; o += al(((size_t)batch + 1) * 4);
  if (sq) { L.sq_off = o; o += al(((size_t)batch + 1) * 8); }
  L.scratch_end = o;
  L.q_codes = o; o += al((size_t)H * TB * BLK * D);
  L.k_codes = o; o += al((size_t)Hkv * TB * BLK * D);
  L.q_scale = o; o += al((size_t)H * NS * 4);
  L.k_scale = o; o += al((size_t)Hkv * NS * 4);
  L.k_mean = o; o += al(SH * D * 4);
  if (fp8) {
    L.v_codes = o; o += al((size_t)T * Hkv * D);
    L.v_scale = o; o += al(SH * D * 4);
  }
  if (sq) {
    const size_t MB = ((size_t)max_seqlen + BLK - 1) / BLK;
    L.bias_head_stride = (long long)(MB * TB * BLK);
    L.q_mean = o; o += al((size_t)H * TB * D * 4);
    L.q_bias = o; o += al((size_t)H * MB * TB * BLK * 4);
  }
  L.total = o;
  return L;
}

bool dense_args_ok(int B, int H, int N, int D, int pv_mode) {
  return B >= 1 && H >= 1 && N >= 1 && N <= kMaxN && (D == 64 || D == 128) &&
         (long long)B * H <= 65535 && (pv_mode == SAGE_PV_FP16 || pv_mode == SAGE_PV_FP8);
}

bool gqa_heads_ok(int H, int Hkv) { return Hkv >= 1 && Hkv <= H && H % Hkv == 0; }
bool gran_ok(int g) {
  return g == SAGE_QK_PER_BLOCK || g == SAGE_QK_PER_TOKEN || g == SAGE_QK_PER_BLOCK_SMOOTH_Q;
}
bool gran_varlen_ok(int g) { return g == SAGE_QK_PER_BLOCK || g == SAGE_QK_PER_TOKEN; }
// sage_quantize_ex / sage_attn_quantized_ex: Q smoothing has its own stages
bool gran_split_ok(int g) { return g == SAGE_QK_PER_BLOCK || g == SAGE_QK_PER_TOKEN; }

bool varlen_args_ok(int T, int batch, int max_seqlen, int H, int D, int pv_mode) {
  return T >= 0 && batch >= 1 && max_seqlen >= 0 && max_seqlen <= kMaxN && H >= 1 &&
         H <= 65535 && (D == 64 || D == 128) &&
         (long long)T + 2 * BLK * (long long)batch < (1LL << 31) &&
         (pv_mode == SAGE_PV_FP16 || pv_mode == SAGE_PV_FP8);
}

template <class T> T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

sage_status_t clear_scratch(void* ws, const Layout& L, bool fp8, cudaStream_t st) {
  // K sums, (FP8) V maxima and the dense work/completion counters start at 0
  cudaError_t e = cudaMemsetAsync(at<uint8_t>(ws, L.k_sum), 0, L.v_amax - L.k_sum, st);
  if (e == cudaSuccess && fp8)
    e = cudaMemsetAsync(at<uint8_t>(ws, L.v_amax), 0, L.sync - L.v_amax, st);
  if (e == cudaSuccess) {  // work / completion counters (dense: both launches')
    const size_t sync_end = L.blk_off ? L.blk_off : L.scratch_end;
    e = cudaMemsetAsync(at<uint8_t>(ws, L.sync), 0, sync_end - L.sync, st);
  }
  return e == cudaSuccess ? SAGE_OK : cuda_fail(e, "cudaMemsetAsync");
}

// Dense stage 1 into explicit buffers.
// Hkv < H (grouped-query attention): K (and V) are quantised over the B*Hkv
// key/value heads and Q over the B*H query heads, in two launches.
sage_status_t quantize_dense(const void* q, const void* k, const void* v, int in_dt, int B,
                             int H, int N, int D, int pv_mode, int8_t* q_codes, float* q_scale,
                             int8_t* k_codes, float* k_scale, float* k_mean, uint8_t* v_codes,
                             float* v_scale, void* ws, const Layout& L, cudaStream_t st,
                             int Hkv, int per_token = 0) {
  const bool fp8 = pv_mode == SAGE_PV_FP8;
  sage_status_t r = clear_scratch(ws, L, fp8, st);
  if (r != SAGE_OK) return r;
  SeqLayout S{};
  S.varlen = 0;
  S.N = N;
  S.H = Hkv;
  const unsigned NB = (unsigned)((N + BLK - 1) / BLK);
  const bool grouped = Hkv != H;
  cudaError_t e = launch_quant(S, dim3(NB, (unsigned)(B * Hkv)), D, in_dt == SAGE_BF16, fp8, q,
                               k, v, q_codes, q_scale, k_codes, k_scale, k_mean, v_codes, v_scale,
                               at<unsigned long long>(ws, L.k_sum), at<uint32_t>(ws, L.v_amax),
                               at<uint32_t>(ws, 0), at<unsigned int>(ws, L.sync),
                               grouped ? QUANT_KV : QUANT_Q | QUANT_KV, per_token, st);
  if (e == cudaSuccess && grouped) {
    S.H = H;
    e = launch_quant(S, dim3(NB, (unsigned)(B * H)), D, in_dt == SAGE_BF16, fp8, q, k, v, q_codes,
                     q_scale, k_codes, k_scale, k_mean, v_codes, v_scale,
                     at<unsigned long long>(ws, L.k_sum), at<uint32_t>(ws, L.v_amax),
                     at<uint32_t>(ws, 0), at<unsigned int>(ws, L.sync_q), QUANT_Q, per_token, st);
  }
  if (e == cudaErrorNotSupported) return SAGE_ERR_UNSUPPORTED;
  return e == cudaSuccess ? SAGE_OK : cuda_fail(e, "quantisation launch");
}

// Dense stage 1 with Q smoothing: K (and V) as for per-block deltas over the
// key/value heads, then the smoothed Q blocks and the per-key mean term.
sage_status_t quantize_dense_sq(const void* q, const void* k, const void* v, int in_dt, int B,
                                int H, int N, int D, int pv_mode, int causal, float sm_scale,
                                int8_t* q_codes, float* q_scale, float* q_mean, int8_t* k_codes,
                                float* k_scale, float* k_mean, uint8_t* v_codes, float* v_scale,
                                float* q_bias, void* ws, const Layout& L, cudaStream_t st,
                                int Hkv, bool with_bias = true) {
  const bool fp8 = pv_mode == SAGE_PV_FP8, bf16 = in_dt == SAGE_BF16;
  sage_status_t r = clear_scratch(ws, L, fp8, st);
  if (r != SAGE_OK) return r;
  SeqLayout S{};
  S.varlen = 0;
  S.N = N;
  S.H = Hkv;
  const unsigned NB = (unsigned)((N + BLK - 1) / BLK);
  cudaError_t e = launch_quant(S, dim3(NB, (unsigned)(B * Hkv)), D, bf16, fp8, q, k, v, q_codes,
                               q_scale, k_codes, k_scale, k_mean, v_codes, v_scale,
                               at<unsigned long long>(ws, L.k_sum), at<uint32_t>(ws, L.v_amax),
                               at<uint32_t>(ws, 0), at<unsigned int>(ws, L.sync), QUANT_KV, 0, st);
  S.H = H;
  if (e == cudaSuccess)
    e = launch_quant_q_smooth(S, dim3(NB, (unsigned)(B * H)), D, bf16, q, q_codes, q_scale,
                              q_mean, at<uint32_t>(ws, 0), st);
  if (e == cudaSuccess && with_bias)  // the term of every query block
    e = launch_q_smooth_bias(S, dim3(NB, (unsigned)(B * H)), H, Hkv, D, bf16, causal ? 1 : 0,
                             kappa_of(sm_scale, D), k, k_mean, q_mean, q_bias, 0, nullptr, 0,
                             (int)NB, st);
  if (e == cudaErrorNotSupported) return SAGE_ERR_UNSUPPORTED;
  return e == cudaSuccess ? SAGE_OK : cuda_fail(e, "quantisation launch");
}

sage_status_t attn_dense(const int8_t* q_codes, const float* q_scale, const int8_t* k_codes,
                         const float* k_scale, const void* v, const uint8_t* v_codes,
                         const float* v_scale, void* out, int v_dt, int out_dt, int B, int H,
                         int N, int D, int causal, float sm_scale, int pv_mode, void* ws,
                         cudaStream_t st, int Hkv, int per_token = 0,
                         const float* q_bias = nullptr, int32_t* s_dump = nullptr,
                         long long wait_limit = 0, int fault_skip_k = 0, int pair0 = 0,
                         int npairs = -1, int bias_nb = -1) {
  const bool fp8 = pv_mode == SAGE_PV_FP8;
  AttnLaunch A{};
  A.p.H = H;
  A.p.Hkv = Hkv;
  A.p.per_token = per_token;
  A.p.q_bias = q_bias;
  A.p.N = N;
  A.p.BH = B * H;
  A.p.NB = (N + BLK - 1) / BLK;
  // query tile pairs [pair0, pair0 + npairs) (all by default); q_bias holds
  // bias_nb query blocks per head from block 2*pair0
  A.p.NPAIR = npairs < 0 ? (N + 2 * BLK - 1) / (2 * BLK) : npairs;
  A.p.pair0 = pair0;
  A.p.bias_nb = bias_nb < 0 ? A.p.NB : bias_nb;
  A.p.causal = causal ? 1 : 0;
  A.p.kappa = kappa_of(sm_scale, D);
  A.p.q_scale = q_scale;
  A.p.k_scale = k_scale;
  A.p.v_scale = v_scale;
  A.p.out = out;
  A.p.out_dt = out_dt;
  A.p.varlen = 0;
  A.p.status = at<uint32_t>(ws, 0);
  A.p.sched = at<unsigned int>(ws, kSchedOff);
  A.D = D;
  A.pv8 = fp8;
  A.bf16v = v_dt == SAGE_BF16;
  A.q_codes = q_codes;
  A.k_codes = k_codes;
  A.v = fp8 ? static_cast<const void*>(v_codes) : v;
  A.code_rows = A.p.NB * BLK;
  A.code_z = B * H;
  A.code_z_kv = B * Hkv;
  A.T = 0;
  A.p.items = B * H * A.p.NPAIR;
  A.p.s_dump = s_dump;
  A.p.s_dump_ld = (long long)A.p.NB * BLK;
  A.p.wait_limit = wait_limit;
  A.p.fault_skip_k = fault_skip_k;
  cudaError_t e = launch_attn(A, st);
  if (e == cudaErrorNotSupported) return SAGE_ERR_UNSUPPORTED;
  return e == cudaSuccess ? SAGE_OK : cuda_fail(e, "attention launch");
}

}  // namespace

extern "C" {

size_t sage_workspace_bytes(int B, int H, int N, int D, int pv_mode) {
  if (!dense_args_ok(B, H, N, D, pv_mode)) return 0;
  return dense_layout(B, H, N, D, pv_mode == SAGE_PV_FP8).total;
}

size_t sage_workspace_bytes_varlen(int total_tokens, int batch, int H, int D, int pv_mode) {
  if (!varlen_args_ok(total_tokens, batch, 0, H, D, pv_mode)) return 0;
  return varlen_layout(total_tokens, batch, H, D, pv_mode == SAGE_PV_FP8).total;
}

size_t sage_scratch_bytes(int B, int H, int D) {
  if (B < 1 || H < 1 || (D != 64 && D != 128)) return 0;
  return dense_layout(B, H, 1, D, true).scratch_end;
}

const char* sage_status_string(sage_status_t s) {
  switch (s) {
    case SAGE_OK: return "SAGE_OK";
    case SAGE_ERR_INVALID_ARG: return "SAGE_ERR_INVALID_ARG";
    case SAGE_ERR_UNSUPPORTED: return "SAGE_ERR_UNSUPPORTED";
    case SAGE_ERR_WORKSPACE: return "SAGE_ERR_WORKSPACE";
    case SAGE_ERR_CUDA: return "SAGE_ERR_CUDA";
    case SAGE_ERR_TIMEOUT: return "SAGE_ERR_TIMEOUT";
    case SAGE_ERR_BAD_SEQLENS: return "SAGE_ERR_BAD_SEQLENS";
    case SAGE_ERR_RANGE: return "SAGE_ERR_RANGE";
  }
  return "SAGE_ERR_UNKNOWN";
}

const char* sage_last_cuda_error(void) { return g_last_error; }

sage_status_t sage_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!aligned16(ws) || ws_bytes < kHeader) return SAGE_ERR_INVALID_ARG;
  cudaError_t e = cudaMemsetAsync(ws, 0, kHeader, as_stream(stream));
  return e == cudaSuccess ? SAGE_OK : cuda_fail(e, "cudaMemsetAsync");
}

sage_status_t sage_sync_status(void* ws, void* stream) {
  if (!aligned16(ws)) return SAGE_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  uint32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (word != 0) {
    e = cudaMemsetAsync(ws, 0, sizeof(word), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "status clear");
  }
  if (word & ST_TIMEOUT) return SAGE_ERR_TIMEOUT;
  if (word & ST_BAD_SEQLENS) return SAGE_ERR_BAD_SEQLENS;
  if (word & ST_RANGE) return SAGE_ERR_RANGE;
  return SAGE_OK;
}

sage_status_t sage_quantize_ex(const void* q, const void* k, const void* v, int in_dt, int B,
                               int H, int Hkv, int N, int D, int pv_mode, int qk_gran,
                               int8_t* q_codes, float* q_scale, int8_t* k_codes, float* k_scale,
                               float* k_mean, uint8_t* v_codes, float* v_scale, void* ws,
                               size_t ws_bytes, void* stream) {
  if (!dense_args_ok(B, H, N, D, pv_mode) || !gqa_heads_ok(H, Hkv) || !gran_split_ok(qk_gran) ||
      !in_dtype_ok(in_dt))
    return SAGE_ERR_INVALID_ARG;
  const bool fp8 = pv_mode == SAGE_PV_FP8;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_codes) || !aligned16(k_codes) ||
      !q_scale || !k_scale || !k_mean || !aligned16(ws))
    return SAGE_ERR_INVALID_ARG;
  if (fp8 && (!aligned16(v) || !aligned16(v_codes) || !aligned16(v_scale))) return SAGE_ERR_INVALID_ARG;
  const bool tok = qk_gran == SAGE_QK_PER_TOKEN;
  const Layout L = dense_layout(B, H, N, D, fp8, Hkv, tok);
  if (ws_bytes < L.scratch_end) return SAGE_ERR_WORKSPACE;
  return quantize_dense(q, k, v, in_dt, B, H, N, D, pv_mode, q_codes, q_scale, k_codes, k_scale,
                        k_mean, v_codes, v_scale, ws, L, as_stream(stream), Hkv, tok ? 1 : 0);
}

sage_status_t sage_quantize(const void* q, const void* k, const void* v, int in_dt, int B, int H,
                            int N, int D, int pv_mode, int8_t* q_codes, float* q_scale,
                            int8_t* k_codes, float* k_scale, float* k_mean, uint8_t* v_codes,
                            float* v_scale, void* ws, size_t ws_bytes, void* stream) {
  return sage_quantize_ex(q, k, v, in_dt, B, H, H, N, D, pv_mode, SAGE_QK_PER_BLOCK, q_codes,
                          q_scale, k_codes, k_scale, k_mean, v_codes, v_scale, ws, ws_bytes,
                          stream);
}

sage_status_t sage_quant_qk(const void* q, const void* k, int in_dt, int B, int H, int N, int D,
                            int8_t* q_codes, float* q_scale, int8_t* k_codes, float* k_scale,
                            float* k_mean, void* ws, size_t ws_bytes, void* stream) {
  return sage_quantize_ex(q, k, nullptr, in_dt, B, H, H, N, D, SAGE_PV_FP16, SAGE_QK_PER_BLOCK,
                          q_codes, q_scale, k_codes, k_scale, k_mean, nullptr, nullptr, ws,
                          ws_bytes, stream);
}

sage_status_t sage_attn_quantized_ex(const int8_t* q_codes, const float* q_scale,
                                     const int8_t* k_codes, const float* k_scale, const void* v,
                                     const uint8_t* v_codes, const float* v_scale, void* out,
                                     int v_dt, int out_dt, int B, int H, int Hkv, int N, int D,
                                     int causal, float sm_scale, int pv_mode, int qk_gran,
                                     void* ws, size_t ws_bytes, void* stream) {
  if (!dense_args_ok(B, H, N, D, pv_mode) || !gqa_heads_ok(H, Hkv) || !gran_split_ok(qk_gran) ||
      !out_dtype_ok(out_dt) || !std::isfinite(sm_scale))
    return SAGE_ERR_INVALID_ARG;
  const bool fp8 = pv_mode == SAGE_PV_FP8;
  if (!aligned16(q_codes) || !aligned16(k_codes) || !q_scale || !aligned16(k_scale) ||
      !aligned16(out) || !aligned16(ws))
    return SAGE_ERR_INVALID_ARG;
  if (fp8 ? (!aligned16(v_codes) || !aligned16(v_scale)) : (!aligned16(v) || !in_dtype_ok(v_dt)))
    return SAGE_ERR_INVALID_ARG;
  if (ws_bytes < kHeader) return SAGE_ERR_WORKSPACE;
  return attn_dense(q_codes, q_scale, k_codes, k_scale, v, v_codes, v_scale, out, v_dt, out_dt, B,
                    H, N, D, causal, sm_scale, pv_mode, ws, as_stream(stream), Hkv,
                    qk_gran == SAGE_QK_PER_TOKEN ? 1 : 0);
}

sage_status_t sage_attn_quantized(const int8_t* q_codes, const float* q_scale,
                                  const int8_t* k_codes, const float* k_scale, const void* v,
                                  const uint8_t* v_codes, const float* v_scale, void* out,
                                  int v_dt, int out_dt, int B, int H, int N, int D, int causal,
                                  float sm_scale, int pv_mode, void* ws, size_t ws_bytes,
                                  void* stream) {
  return sage_attn_quantized_ex(q_codes, q_scale, k_codes, k_scale, v, v_codes, v_scale, out,
                                v_dt, out_dt, B, H, H, N, D, causal, sm_scale, pv_mode,
                                SAGE_QK_PER_BLOCK, ws, ws_bytes, stream);
}

sage_status_t sage_quantize_sq(const void* q, const void* k, const void* v, int in_dt, int B,
                               int H, int Hkv, int N, int D, int pv_mode, int causal,
                               float sm_scale, int8_t* q_codes, float* q_scale, float* q_mean,
                               int8_t* k_codes, float* k_scale, float* k_mean, uint8_t* v_codes,
                               float* v_scale, float* q_bias, void* ws, size_t ws_bytes,
                               void* stream) {
  if (!dense_args_ok(B, H, N, D, pv_mode) || !gqa_heads_ok(H, Hkv) || !in_dtype_ok(in_dt) ||
      !std::isfinite(sm_scale))
    return SAGE_ERR_INVALID_ARG;
  const bool fp8 = pv_mode == SAGE_PV_FP8;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_codes) || !aligned16(k_codes) ||
      !q_scale || !aligned16(q_mean) || !k_scale || !aligned16(k_mean) || !aligned16(q_bias) ||
      !aligned16(ws))
    return SAGE_ERR_INVALID_ARG;
  if (fp8 && (!aligned16(v) || !aligned16(v_codes) || !aligned16(v_scale))) return SAGE_ERR_INVALID_ARG;
  const Layout L = dense_layout(B, H, N, D, fp8, Hkv);
  if (ws_bytes < L.scratch_end) return SAGE_ERR_WORKSPACE;
  return quantize_dense_sq(q, k, v, in_dt, B, H, N, D, pv_mode, causal, sm_scale, q_codes,
                           q_scale, q_mean, k_codes, k_scale, k_mean, v_codes, v_scale, q_bias,
                           ws, L, as_stream(stream), Hkv);
}

sage_status_t sage_attn_quantized_sq(const int8_t* q_codes, const float* q_scale,
                                     const int8_t* k_codes, const float* k_scale,
                                     const float* q_bias, const void* v, const uint8_t* v_codes,
                                     const float* v_scale, void* out, int v_dt, int out_dt, int B,
                                     int H, int Hkv, int N, int D, int causal, float sm_scale,
                                     int pv_mode, void* ws, size_t ws_bytes, void* stream) {
  if (!dense_args_ok(B, H, N, D, pv_mode) || !gqa_heads_ok(H, Hkv) || !out_dtype_ok(out_dt) ||
      !std::isfinite(sm_scale))
    return SAGE_ERR_INVALID_ARG;
  const bool fp8 = pv_mode == SAGE_PV_FP8;
  if (!aligned16(q_codes) || !aligned16(k_codes) || !q_scale || !k_scale || !aligned16(q_bias) ||
      !aligned16(out) || !aligned16(ws))
    return SAGE_ERR_INVALID_ARG;
  if (fp8 ? (!aligned16(v_codes) || !aligned16(v_scale)) : (!aligned16(v) || !in_dtype_ok(v_dt)))
    return SAGE_ERR_INVALID_ARG;
  if (ws_bytes < kHeader) return SAGE_ERR_WORKSPACE;
  return attn_dense(q_codes, q_scale, k_codes, k_scale, v, v_codes, v_scale, out, v_dt, out_dt, B,
                    H, N, D, causal, sm_scale, pv_mode, ws, as_stream(stream), Hkv, 2, q_bias);
}

sage_status_t sage_attn_quantized_dump_s(const int8_t* q_codes, const float* q_scale,
                                         const int8_t* k_codes, const float* k_scale,
                                         const void* v, const uint8_t* v_codes,
                                         const float* v_scale, void* out, int v_dt, int out_dt,
                                         int B, int H, int N, int D, int causal, float sm_scale,
                                         int pv_mode, int32_t* s_out, void* ws, size_t ws_bytes,
                                         void* stream) {
  if (!dense_args_ok(B, H, N, D, pv_mode) || !out_dtype_ok(out_dt) || !std::isfinite(sm_scale))
    return SAGE_ERR_INVALID_ARG;
  const bool fp8 = pv_mode == SAGE_PV_FP8;
  if (!aligned16(q_codes) || !aligned16(k_codes) || !q_scale || !aligned16(k_scale) ||
      !aligned16(out) || !aligned16(ws) || !aligned16(s_out))
    return SAGE_ERR_INVALID_ARG;
  if (fp8 ? (!aligned16(v_codes) || !aligned16(v_scale)) : (!aligned16(v) || !in_dtype_ok(v_dt)))
    return SAGE_ERR_INVALID_ARG;
  if (!fp8 && v_dt != SAGE_F16) return SAGE_ERR_UNSUPPORTED;
  if (ws_bytes < kHeader) return SAGE_ERR_WORKSPACE;
  return attn_dense(q_codes, q_scale, k_codes, k_scale, v, v_codes, v_scale, out, v_dt, out_dt, B,
                    H, N, D, causal, sm_scale, pv_mode, ws, as_stream(stream), H, 0, nullptr,
                    s_out);
}

sage_status_t sage_selftest_attn_timeout(const int8_t* q_codes, const float* q_scale,
                                         const int8_t* k_codes, const float* k_scale,
                                         const void* v, const uint8_t* v_codes,
                                         const float* v_scale, void* out, int v_dt, int out_dt,
                                         int B, int H, int N, int D, int causal, float sm_scale,
                                         int pv_mode, long long wait_cycles, int skip_k_stage,
                                         void* ws, size_t ws_bytes, void* stream) {
  if (!dense_args_ok(B, H, N, D, pv_mode) || !out_dtype_ok(out_dt) || !std::isfinite(sm_scale) ||
      wait_cycles < 1 || wait_cycles > (1LL << 31) || skip_k_stage < 0)
    return SAGE_ERR_INVALID_ARG;
  const bool fp8 = pv_mode == SAGE_PV_FP8;
  if (!aligned16(q_codes) || !aligned16(k_codes) || !q_scale || !aligned16(k_scale) ||
      !aligned16(out) || !aligned16(ws))
    return SAGE_ERR_INVALID_ARG;
  if (fp8 ? (!aligned16(v_codes) || !aligned16(v_scale)) : (!aligned16(v) || !in_dtype_ok(v_dt)))
    return SAGE_ERR_INVALID_ARG;
  if (ws_bytes < kHeader) return SAGE_ERR_WORKSPACE;
  return attn_dense(q_codes, q_scale, k_codes, k_scale, v, v_codes, v_scale, out, v_dt, out_dt, B,
                    H, N, D, causal, sm_scale, pv_mode, ws, as_stream(stream), H, 0, nullptr,
                    nullptr, wait_cycles, skip_k_stage);
}

size_t sage_workspace_bytes_ex(int B, int H, int Hkv, int N, int D, int pv_mode, int qk_gran) {
  if (!dense_args_ok(B, H, N, D, pv_mode) || !gqa_heads_ok(H, Hkv) || !gran_ok(qk_gran)) return 0;
  return dense_layout(B, H, N, D, pv_mode == SAGE_PV_FP8, Hkv, qk_gran).total;
}

size_t sage_workspace_bytes_sq(int B, int H, int Hkv, int N, int D, int pv_mode,
                               int q_blocks_per_chunk) {
  if (!dense_args_ok(B, H, N, D, pv_mode) || !gqa_heads_ok(H, Hkv)) return 0;
  const int NB = (N + BLK - 1) / BLK;
  if (q_blocks_per_chunk < 1 || (q_blocks_per_chunk < NB && (q_blocks_per_chunk & 1))) return 0;
  return dense_layout(B, H, N, D, pv_mode == SAGE_PV_FP8, Hkv, SAGE_QK_PER_BLOCK_SMOOTH_Q,
                      q_blocks_per_chunk)
      .total;
}

sage_status_t sage_attn_fwd_ex(const void* q, const void* k, const void* v, void* out, int in_dt,
                               int out_dt, int B, int H, int Hkv, int N, int D, int causal,
                               float sm_scale, int pv_mode, int qk_gran, void* ws,
                               size_t ws_bytes, void* stream) {
  if (!dense_args_ok(B, H, N, D, pv_mode) || !gqa_heads_ok(H, Hkv) || !gran_ok(qk_gran) ||
      !in_dtype_ok(in_dt) || !out_dtype_ok(out_dt) || !std::isfinite(sm_scale))
    return SAGE_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(ws))
    return SAGE_ERR_INVALID_ARG;
  const bool fp8 = pv_mode == SAGE_PV_FP8, tok = qk_gran == SAGE_QK_PER_TOKEN;
  Layout L = dense_layout(B, H, N, D, fp8, Hkv, qk_gran);
  cudaStream_t st = as_stream(stream);
  if (qk_gran == SAGE_QK_PER_BLOCK_SMOOTH_Q) {
    // The mean term of as many query blocks as the workspace holds at a time
    // (an even count unless all fit): each chunk's term, then attention on
    // that chunk's query tiles.  Every value is the one of a single pass.
    const int NB = (N + BLK - 1) / BLK;
    const size_t row = (size_t)B * H * NB * BLK * 4;
    int rows = ws_bytes > L.q_bias ? (int)std::min<size_t>((ws_bytes - L.q_bias) / row, NB) : 0;
    if (rows < NB) rows &= ~1;
    if (rows < 1) return SAGE_ERR_WORKSPACE;
    L = dense_layout(B, H, N, D, fp8, Hkv, qk_gran, rows);
    if (ws_bytes < L.total) return SAGE_ERR_WORKSPACE;
    sage_status_t r = quantize_dense_sq(
        q, k, v, in_dt, B, H, N, D, pv_mode, causal, sm_scale, at<int8_t>(ws, L.q_codes),
        at<float>(ws, L.q_scale), at<float>(ws, L.q_mean), at<int8_t>(ws, L.k_codes),
        at<float>(ws, L.k_scale), at<float>(ws, L.k_mean),
        fp8 ? at<uint8_t>(ws, L.v_codes) : nullptr, fp8 ? at<float>(ws, L.v_scale) : nullptr,
        at<float>(ws, L.q_bias), ws, L, st, Hkv, false);
    SeqLayout S{};
    S.varlen = 0;
    S.N = N;
    S.H = H;
    for (int qb0 = 0; r == SAGE_OK && qb0 < NB; qb0 += rows) {
      const int qr = std::min(rows, NB - qb0);
      // with a causal mask, key tiles past the chunk's last query block add nothing
      const cudaError_t e = launch_q_smooth_bias(
          S, dim3((unsigned)(causal ? qb0 + qr : NB), (unsigned)(B * H)), H, Hkv, D,
          in_dt == SAGE_BF16, causal ? 1 : 0, kappa_of(sm_scale, D), k, at<float>(ws, L.k_mean),
          at<float>(ws, L.q_mean), at<float>(ws, L.q_bias), 0, nullptr, qb0, rows, st);
      if (e != cudaSuccess) return cuda_fail(e, "quantisation launch");
      r = attn_dense(at<int8_t>(ws, L.q_codes), at<float>(ws, L.q_scale),
                     at<int8_t>(ws, L.k_codes), at<float>(ws, L.k_scale), v,
                     fp8 ? at<uint8_t>(ws, L.v_codes) : nullptr,
                     fp8 ? at<float>(ws, L.v_scale) : nullptr, out, in_dt, out_dt, B, H, N, D,
                     causal, sm_scale, pv_mode, ws, st, Hkv, 2, at<float>(ws, L.q_bias), nullptr,
                     0, 0, qb0 / 2, (qr + 1) / 2, rows);
    }
    return r;
  }
  if (ws_bytes < L.total) return SAGE_ERR_WORKSPACE;
  sage_status_t r = quantize_dense(
      q, k, v, in_dt, B, H, N, D, pv_mode, at<int8_t>(ws, L.q_codes), at<float>(ws, L.q_scale),
      at<int8_t>(ws, L.k_codes), at<float>(ws, L.k_scale), at<float>(ws, L.k_mean),
      fp8 ? at<uint8_t>(ws, L.v_codes) : nullptr, fp8 ? at<float>(ws, L.v_scale) : nullptr, ws, L,
      st, Hkv, tok ? 1 : 0);
  if (r != SAGE_OK) return r;
  return attn_dense(at<int8_t>(ws, L.q_codes), at<float>(ws, L.q_scale), at<int8_t>(ws, L.k_codes),
                    at<float>(ws, L.k_scale), v, fp8 ? at<uint8_t>(ws, L.v_codes) : nullptr,
                    fp8 ? at<float>(ws, L.v_scale) : nullptr, out, in_dt, out_dt, B, H, N, D,
                    causal, sm_scale, pv_mode, ws, st, Hkv, tok ? 1 : 0);
}

sage_status_t sage_attn_fwd(const void* q, const void* k, const void* v, void* out, int in_dt,
                            int out_dt, int B, int H, int N, int D, int causal, float sm_scale,
                            int pv_mode, void* ws, size_t ws_bytes, void* stream) {
  return sage_attn_fwd_ex(q, k, v, out, in_dt, out_dt, B, H, H, N, D, causal, sm_scale, pv_mode,
                          SAGE_QK_PER_BLOCK, ws, ws_bytes, stream);
}

size_t sage_workspace_bytes_gqa(int B, int H, int Hkv, int N, int D, int pv_mode) {
  return sage_workspace_bytes_ex(B, H, Hkv, N, D, pv_mode, SAGE_QK_PER_BLOCK);
}

sage_status_t sage_attn_fwd_gqa(const void* q, const void* k, const void* v, void* out, int in_dt,
                                int out_dt, int B, int H, int Hkv, int N, int D, int causal,
                                float sm_scale, int pv_mode, void* ws, size_t ws_bytes,
                                void* stream) {
  return sage_attn_fwd_ex(q, k, v, out, in_dt, out_dt, B, H, Hkv, N, D, causal, sm_scale, pv_mode,
                          SAGE_QK_PER_BLOCK, ws, ws_bytes, stream);
}

static sage_status_t varlen_stage1(const void* q, const void* k, const void* v, int in_dt,
                                   const int32_t* cu, int batch, int max_seqlen, int T, int H,
                                   int D, int pv_mode, int8_t* q_codes, float* q_scale,
                                   int8_t* k_codes, float* k_scale, float* k_mean,
                                   uint8_t* v_codes, float* v_scale, void* ws, const Layout& L,
                                   cudaStream_t st, int Hkv = 0, int per_token = 0,
                                   int causal = 0, float sm_scale = 0.0f) {
  if (Hkv <= 0) Hkv = H;
  const bool fp8 = pv_mode == SAGE_PV_FP8, bf16 = in_dt == SAGE_BF16;
  const bool sq = per_token == 2;  // Q smoothing
  sage_status_t r = clear_scratch(ws, L, fp8, st);
  if (r != SAGE_OK) return r;
  cudaError_t e = launch_varlen_prep(cu, batch, max_seqlen, T, at<int32_t>(ws, L.blk_off),
                                     at<int32_t>(ws, L.pair_off), at<uint32_t>(ws, 0), st,
                                     sq ? at<long long>(ws, L.sq_off) : nullptr);
  if (e != cudaSuccess) return cuda_fail(e, "varlen preparation launch");
  const long long TB = tb_max(T, batch);
  if (TB == 0) return SAGE_OK;
  SeqLayout S{};
  S.varlen = 1;
  S.H = Hkv;
  S.cu = cu;
  S.blk_off = at<int32_t>(ws, L.blk_off);
  S.batch = batch;
  S.TBmax = (int)TB;
  if (sq) {
    // K (, V) per block over the key/value heads; the smoothed Q blocks and
    // the per-key mean term over the query heads
    e = launch_quant(S, dim3((unsigned)TB, Hkv), D, bf16, fp8, q, k, v, q_codes, q_scale, k_codes,
                     k_scale, k_mean, v_codes, v_scale, at<unsigned long long>(ws, L.k_sum),
                     at<uint32_t>(ws, L.v_amax), at<uint32_t>(ws, 0), nullptr, QUANT_KV, 0, st);
    S.H = H;
    if (e == cudaSuccess)
      e = launch_quant_q_smooth(S, dim3((unsigned)TB, H), D, bf16, q, q_codes, q_scale,
                                at<float>(ws, L.q_mean), at<uint32_t>(ws, 0), st);
    if (e == cudaSuccess)
      e = launch_q_smooth_bias(S, dim3((unsigned)TB, H), H, Hkv, D, bf16, causal ? 1 : 0,
                               kappa_of(sm_scale, D), k, k_mean, at<float>(ws, L.q_mean),
                               at<float>(ws, L.q_bias), L.bias_head_stride,
                               at<long long>(ws, L.sq_off), 0, 0, st);
    return e == cudaSuccess ? SAGE_OK : cuda_fail(e, "quantisation launch");
  }
  // grouped-query: K (, V) over the Hkv key/value heads, then Q over the H
  // query heads; otherwise both in one pair of launches
  const bool grouped = Hkv != H;
  e = launch_quant(S, dim3((unsigned)TB, Hkv), D, in_dt == SAGE_BF16, fp8, q, k, v, q_codes,
                   q_scale, k_codes, k_scale, k_mean, v_codes, v_scale,
                   at<unsigned long long>(ws, L.k_sum), at<uint32_t>(ws, L.v_amax),
                   at<uint32_t>(ws, 0), nullptr, grouped ? QUANT_KV : QUANT_Q | QUANT_KV,
                   per_token, st);
  if (e == cudaSuccess && grouped) {
    S.H = H;
    e = launch_quant(S, dim3((unsigned)TB, H), D, in_dt == SAGE_BF16, fp8, q, k, v, q_codes,
                     q_scale, k_codes, k_scale, k_mean, v_codes, v_scale,
                     at<unsigned long long>(ws, L.k_sum), at<uint32_t>(ws, L.v_amax),
                     at<uint32_t>(ws, 0), nullptr, QUANT_Q, per_token, st);
  }
  return e == cudaSuccess ? SAGE_OK : cuda_fail(e, "quantisation launch");
}

sage_status_t sage_quantize_varlen(const void* q, const void* k, const void* v, int in_dt,
                                   const int32_t* cu_seqlens, int batch, int max_seqlen,
                                   int total_tokens, int H, int D, int pv_mode, int8_t* q_codes,
                                   float* q_scale, int8_t* k_codes, float* k_scale,
                                   float* k_mean, uint8_t* v_codes, float* v_scale, void* ws,
                                   size_t ws_bytes, void* stream) {
  if (!varlen_args_ok(total_tokens, batch, max_seqlen, H, D, pv_mode) || !in_dtype_ok(in_dt))
    return SAGE_ERR_INVALID_ARG;
  const bool fp8 = pv_mode == SAGE_PV_FP8;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_codes) || !aligned16(k_codes) ||
      !q_scale || !k_scale || !k_mean || !aligned16(ws) || !cu_seqlens)
    return SAGE_ERR_INVALID_ARG;
  if (fp8 && (!aligned16(v) || !aligned16(v_codes) || !aligned16(v_scale))) return SAGE_ERR_INVALID_ARG;
  const Layout L = varlen_layout(total_tokens, batch, H, D, fp8);
  if (ws_bytes < L.scratch_end) return SAGE_ERR_WORKSPACE;
  if (total_tokens == 0) return SAGE_OK;
  return varlen_stage1(q, k, v, in_dt, cu_seqlens, batch, max_seqlen, total_tokens, H, D, pv_mode,
                       q_codes, q_scale, k_codes, k_scale, k_mean, v_codes, v_scale, ws, L,
                       as_stream(stream));
}

static sage_status_t attn_fwd_varlen_g(const void* q, const void* k, const void* v, void* out,
                                       int in_dt, int out_dt, const int32_t* cu_seqlens,
                                       int batch, int max_seqlen, int total_tokens, int H,
                                       int Hkv, int D, int causal, float sm_scale, int pv_mode,
                                       int qk_gran, void* ws, size_t ws_bytes, void* stream) {
  if (!varlen_args_ok(total_tokens, batch, max_seqlen, H, D, pv_mode) || !gqa_heads_ok(H, Hkv) ||
      !gran_ok(qk_gran) || !in_dtype_ok(in_dt) || !out_dtype_ok(out_dt) ||
      !std::isfinite(sm_scale))
    return SAGE_ERR_INVALID_ARG;
  // 0 per block, 1 per token, 2 per block with Q smoothing
  const int tok = qk_gran == SAGE_QK_PER_TOKEN ? 1 : qk_gran == SAGE_QK_PER_BLOCK_SMOOTH_Q ? 2 : 0;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(ws) ||
      !cu_seqlens)
    return SAGE_ERR_INVALID_ARG;
  const bool fp8 = pv_mode == SAGE_PV_FP8;
  const Layout L = varlen_layout(total_tokens, batch, H, D, fp8, Hkv, qk_gran, max_seqlen);
  if (ws_bytes < L.total) return SAGE_ERR_WORKSPACE;
  if (total_tokens == 0) return SAGE_OK;
  cudaStream_t st = as_stream(stream);
  sage_status_t r = varlen_stage1(
      q, k, v, in_dt, cu_seqlens, batch, max_seqlen, total_tokens, H, D, pv_mode,
      at<int8_t>(ws, L.q_codes), at<float>(ws, L.q_scale), at<int8_t>(ws, L.k_codes),
      at<float>(ws, L.k_scale), at<float>(ws, L.k_mean), fp8 ? at<uint8_t>(ws, L.v_codes) : nullptr,
      fp8 ? at<float>(ws, L.v_scale) : nullptr, ws, L, st, Hkv, tok, causal, sm_scale);
  if (r != SAGE_OK) return r;
  const long long TB = tb_max(total_tokens, batch), PM = pair_max(total_tokens, batch);
  if (PM == 0) return SAGE_OK;
  AttnLaunch A{};
  A.p.H = H;
  A.p.Hkv = Hkv;
  A.p.per_token = tok;
  A.p.causal = causal ? 1 : 0;
  A.p.kappa = kappa_of(sm_scale, D);
  A.p.q_scale = at<float>(ws, L.q_scale);
  A.p.k_scale = at<float>(ws, L.k_scale);
  A.p.v_scale = fp8 ? at<float>(ws, L.v_scale) : nullptr;
  A.p.out = out;
  A.p.out_dt = out_dt;
  A.p.varlen = 1;
  A.p.cu = cu_seqlens;
  A.p.blk_off = at<int32_t>(ws, L.blk_off);
  A.p.pair_off = at<int32_t>(ws, L.pair_off);
  A.p.batch = batch;
  A.p.TBmax = (int)TB;
  A.p.status = at<uint32_t>(ws, 0);
  A.p.sched = at<unsigned int>(ws, kSchedOff);
  if (tok == 2) {
    A.p.q_bias = at<float>(ws, L.q_bias);
    A.p.sq_off = at<long long>(ws, L.sq_off);
    A.p.bias_head_stride = L.bias_head_stride;
  }
  A.D = D;
  A.pv8 = fp8;
  A.bf16v = in_dt == SAGE_BF16;
  A.q_codes = at<int8_t>(ws, L.q_codes);
  A.k_codes = at<int8_t>(ws, L.k_codes);
  A.v = fp8 ? static_cast<const void*>(at<uint8_t>(ws, L.v_codes)) : v;
  A.code_rows = (int)(TB * BLK);
  A.code_z = H;
  A.code_z_kv = Hkv;
  A.T = total_tokens;
  A.p.PM = (int)PM;
  A.p.items = (int)(PM * H);
  cudaError_t e = launch_attn(A, st);
  return e == cudaSuccess ? SAGE_OK : cuda_fail(e, "attention launch");
}

sage_status_t sage_attn_fwd_varlen(const void* q, const void* k, const void* v, void* out,
                                   int in_dt, int out_dt, const int32_t* cu_seqlens, int batch,
                                   int max_seqlen, int total_tokens, int H, int D, int causal,
                                   float sm_scale, int pv_mode, void* ws, size_t ws_bytes,
                                   void* stream) {
  return attn_fwd_varlen_g(q, k, v, out, in_dt, out_dt, cu_seqlens, batch, max_seqlen,
                           total_tokens, H, H, D, causal, sm_scale, pv_mode, SAGE_QK_PER_BLOCK, ws,
                           ws_bytes, stream);
}

size_t sage_workspace_bytes_varlen_ex(int total_tokens, int batch, int H, int Hkv, int D,
                                      int pv_mode, int qk_gran) {
  if (!varlen_args_ok(total_tokens, batch, 0, H, D, pv_mode) || !gqa_heads_ok(H, Hkv) ||
      !gran_varlen_ok(qk_gran))
    return 0;
  return varlen_layout(total_tokens, batch, H, D, pv_mode == SAGE_PV_FP8, Hkv, qk_gran).total;
}

size_t sage_workspace_bytes_varlen_sq(int total_tokens, int batch, int max_seqlen, int H,
                                      int Hkv, int D, int pv_mode) {
  if (!varlen_args_ok(total_tokens, batch, max_seqlen, H, D, pv_mode) || !gqa_heads_ok(H, Hkv))
    return 0;
  return varlen_layout(total_tokens, batch, H, D, pv_mode == SAGE_PV_FP8, Hkv,
                       SAGE_QK_PER_BLOCK_SMOOTH_Q, max_seqlen).total;
}

sage_status_t sage_attn_fwd_varlen_ex(const void* q, const void* k, const void* v, void* out,
                                      int in_dt, int out_dt, const int32_t* cu_seqlens, int batch,
                                      int max_seqlen, int total_tokens, int H, int Hkv, int D,
                                      int causal, float sm_scale, int pv_mode, int qk_gran,
                                      void* ws, size_t ws_bytes, void* stream) {
  return attn_fwd_varlen_g(q, k, v, out, in_dt, out_dt, cu_seqlens, batch, max_seqlen,
                           total_tokens, H, Hkv, D, causal, sm_scale, pv_mode, qk_gran, ws,
                           ws_bytes, stream);
}

size_t sage_workspace_bytes_varlen_gqa(int total_tokens, int batch, int H, int Hkv, int D,
                                       int pv_mode) {
  return sage_workspace_bytes_varlen_ex(total_tokens, batch, H, Hkv, D, pv_mode,
                                        SAGE_QK_PER_BLOCK);
}

sage_status_t sage_attn_fwd_varlen_gqa(const void* q, const void* k, const void* v, void* out,
                                       int in_dt, int out_dt, const int32_t* cu_seqlens,
                                       int batch, int max_seqlen, int total_tokens, int H,
                                       int Hkv, int D, int causal, float sm_scale, int pv_mode,
                                       void* ws, size_t ws_bytes, void* stream) {
  return attn_fwd_varlen_g(q, k, v, out, in_dt, out_dt, cu_seqlens, batch, max_seqlen,
                           total_tokens, H, Hkv, D, causal, sm_scale, pv_mode, SAGE_QK_PER_BLOCK,
                           ws, ws_bytes, stream);
}

sage_status_t sage_qk_int8_tiles(const int8_t* q_codes, const int8_t* k_codes, int BH, int NP,
                                 int D, const int32_t* tiles, int n_tiles, int32_t* s_out,
                                 void* ws, size_t ws_bytes, void* stream) {
  if (BH < 1 || NP < BLK || NP % BLK != 0 || (D != 64 && D != 128) || n_tiles < 1 || !tiles ||
      !aligned16(q_codes) || !aligned16(k_codes) || !aligned16(s_out) || !aligned16(ws))
    return SAGE_ERR_INVALID_ARG;
  for (int t = 0; t < n_tiles; ++t) {
    const int bh = tiles[3 * t], I = tiles[3 * t + 1], J = tiles[3 * t + 2];
    if (bh < 0 || bh >= BH || I < 0 || J < 0 || I >= NP / BLK || J >= NP / BLK)
      return SAGE_ERR_INVALID_ARG;
  }
  const size_t need = kHeader + al((size_t)n_tiles * 3 * 4);
  if (ws_bytes < need) return SAGE_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  int32_t* dtiles = at<int32_t>(ws, kHeader);
  cudaError_t e = cudaMemcpyAsync(dtiles, tiles, (size_t)n_tiles * 3 * 4, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return cuda_fail(e, "tile list copy");
  e = launch_qk_tiles(q_codes, k_codes, BH, NP, D, dtiles, n_tiles, s_out, at<uint32_t>(ws, 0), st);
  return e == cudaSuccess ? SAGE_OK : cuda_fail(e, "QK tile launch");
}

}  // extern "C"
