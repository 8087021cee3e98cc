// Full-precision attention for selected query rows: the reference that the
// accuracy-driven choice between 16-bit and FP8 P.V compares against ("SageAttention
// v1/v2/v2++/v3 overview", SageAttention v1, adaptive quantisation: a faster
// variant is used for a layer only where its cosine similarity to
// full-precision attention exceeds 99.8 %).
//
// One CTA of 8 warps per row, fp32 throughout: warps take keys in turn; the
// 32 lanes of a warp split the D channels (lane, lane+32, ...), so K and V
// rows are read coalesced.  Pass 1 finds the row maximum of the scaled
// scores, pass 2 recomputes each score, weights it by expf(score - max) and
// accumulates the weights and the weighted V rows; the warps' partial sums
// are combined in shared memory.  Grouped-query inputs map query head h to
// key/value head h / (H / Hkv).  Not a hot path.
#include "common.cuh"

namespace sage {
namespace {

constexpr int RR_WARPS = 8;

template <bool BF16>
__device__ __forceinline__ float ld16(const uint16_t* p) {
  const uint16_t u = __ldg(p);
  if constexpr (BF16) return __uint_as_float((uint32_t)u << 16);
  else return __half2float(__ushort_as_half(u));
}

template <int D, bool BF16>
__global__ void __launch_bounds__(32 * RR_WARPS) ref_rows_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
    const uint16_t* __restrict__ v, int B, int H, int Hkv, int N, int causal, float scale,
    const int32_t* __restrict__ rows, int n_rows, float* __restrict__ out) {
  constexpr int C = D / 32;  // channels per lane
  __shared__ float red_m[RR_WARPS], red_l[RR_WARPS];
  __shared__ float red_o[RR_WARPS][D];
  const int r = blockIdx.x;
  if (r >= n_rows) return;
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int b = __ldg(rows + 3 * r), h = __ldg(rows + 3 * r + 1), i = __ldg(rows + 3 * r + 2);
  float* o = out + (long long)r * D;
  if (b < 0 || b >= B || h < 0 || h >= H || i < 0 || i >= N) {  // not a row of the input
    if (threadIdx.x < D) o[threadIdx.x] = __int_as_float(0x7fc00000);
    return;
  }
  const int hk = h / (H / Hkv);
  const uint16_t* qrow = q + (((long long)b * H + h) * N + i) * D;
  const uint16_t* kh = k + ((long long)b * Hkv + hk) * N * D;
  const uint16_t* vh = v + ((long long)b * Hkv + hk) * N * D;
  float qv[C];
#pragma unroll
  for (int c = 0; c < C; ++c) qv[c] = ld16<BF16>(qrow + lane + 32 * c);
  const int limit = causal ? i + 1 : N;

  auto score = [&](int j) {
    const uint16_t* kr = kh + (long long)j * D;
    float s = 0.0f;
#pragma unroll
    for (int c = 0; c < C; ++c) s = fmaf(qv[c], ld16<BF16>(kr + lane + 32 * c), s);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    return s * scale;
  };

  float m = -INFINITY;
  for (int j = warp; j < limit; j += RR_WARPS) m = fmaxf(m, score(j));
  if (lane == 0) red_m[warp] = m;
  __syncthreads();
  m = red_m[0];
#pragma unroll
  for (int w = 1; w < RR_WARPS; ++w) m = fmaxf(m, red_m[w]);

  float l = 0.0f, acc[C];
#pragma unroll
  for (int c = 0; c < C; ++c) acc[c] = 0.0f;
  for (int j = warp; j < limit; j += RR_WARPS) {
    const float p = expf(score(j) - m);
    l += p;
    const uint16_t* vr = vh + (long long)j * D;
#pragma unroll
    for (int c = 0; c < C; ++c) acc[c] = fmaf(p, ld16<BF16>(vr + lane + 32 * c), acc[c]);
  }
  if (lane == 0) red_l[warp] = l;
#pragma unroll
  for (int c = 0; c < C; ++c) red_o[warp][lane + 32 * c] = acc[c];
  __syncthreads();
  if (threadIdx.x < D) {
    float lt = 0.0f, ot = 0.0f;
#pragma unroll
    for (int w = 0; w < RR_WARPS; ++w) {
      lt += red_l[w];
      ot += red_o[w][threadIdx.x];
    }
    o[threadIdx.x] = ot / lt;
  }
}

}  // namespace
}  // namespace sage

extern "C" sage_status_t sage_attn_ref_rows(const void* q, const void* k, const void* v,
                                            int in_dt, int B, int H, int Hkv, int N, int D,
                                            int causal, float sm_scale, const int32_t* rows,
                                            int n_rows, float* out, void* stream) {
  if (B < 1 || H < 1 || Hkv < 1 || Hkv > H || H % Hkv != 0 || N < 1 || (D != 64 && D != 128) ||
      (in_dt != SAGE_F16 && in_dt != SAGE_BF16) || n_rows < 0 || !(sm_scale == sm_scale) ||
      sm_scale > 3.0e38f || sm_scale < -3.0e38f)
    return SAGE_ERR_INVALID_ARG;
  if (n_rows == 0) return SAGE_OK;
  if (!q || !k || !v || !rows || !out) return SAGE_ERR_INVALID_ARG;
  const float scale = sm_scale > 0.0f ? sm_scale : 1.0f / sqrtf((float)D);
  const auto* q16 = static_cast<const uint16_t*>(q);
  const auto* k16 = static_cast<const uint16_t*>(k);
  const auto* v16 = static_cast<const uint16_t*>(v);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const dim3 grid(n_rows), block(32 * sage::RR_WARPS);
  const bool bf16 = in_dt == SAGE_BF16;
#define SAGE_RR(DD, BB)                                                                  \
  sage::ref_rows_kernel<DD, BB><<<grid, block, 0, st>>>(q16, k16, v16, B, H, Hkv, N, causal, \
                                                        scale, rows, n_rows, out)
  if (D == 64) {
    if (bf16) SAGE_RR(64, true);
    else SAGE_RR(64, false);
  } else {
    if (bf16) SAGE_RR(128, true);
    else SAGE_RR(128, false);
  }
#undef SAGE_RR
  return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}
