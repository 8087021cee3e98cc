// Smoothing and quantisation kernels (the two HBM-bound passes before the
// attention kernel).
//
//   pass 1, one CTA per 128-token block of one (sequence, head):
//     - Q: block max|q| -> delta = max/127, s = 127/max, codes = rint(q*s)
//       ("SageAttention -- brand new attention", quantisation intro steps 1-2),
//     - K: exact per-channel sums on the 2^-24 fixed-point grid (int64 atomics,
//       so the mean does not depend on summation order),
//     - V (FP8 P.V only): per-channel max|v| (atomicMax on the float bits).
//   pass 2, same grid:
//     - K: m_d = fp32(sum_d / (n * 2^24)), smoothing k - m_d ("SageAttention
//       v1/v2/v2++/v3 overview", v1 bullet 1), then the block quantiser,
//     - V (FP8 P.V only): codes = e4m3(v * 448/max|v_d|), per channel
//       ("SageAttention v1/v2/v2++/v3 overview", SageAttention 2 bullet 1).
//
// Every arithmetic step is one IEEE binary32 (or binary64 for the mean)
// operation with round-to-nearest-even, written with explicit __f*_rn
// intrinsics so that no multiply-add contraction changes a code.
//
// Thread layout: 256 threads; a 16-byte vector holds 8 channels; thread t owns
// channel group c = t % (D/8) of rows t/(D/8) + i*(256/(D/8)).  Consecutive
// threads read consecutive 16-byte vectors of one row: fully coalesced.
#include "common.cuh"

namespace sage {
namespace {

constexpr int THREADS = 256;

template <int D>
struct Tile {
  static constexpr int CPR = D / 8;            // 16-byte chunks per row
  static constexpr int RS = THREADS / CPR;     // row stride between a thread's rows
  static constexpr int NIT = BLK / RS;         // rows per thread
};

// Where block `blockIdx.x` of head `blockIdx.y` lives.  Returns false when the
// CTA has no block to process (varlen grid slack).
struct BlockPos {
  int seq;        // index into per-sequence arrays (dense: b*H + h)
  int rows;       // valid rows in this block (1..128)
  int n;          // sequence length
  long long row0; // element offset of token 0 of this block in the [rows, D] view / D
  long long row_stride;  // element stride between consecutive tokens / D
  long long code_row0;   // row index of this block's first code row
  long long scale_idx;   // index of this block's delta
  int b;          // block index within the sequence
};

__device__ __forceinline__ bool block_pos(const SeqLayout& L, BlockPos& P) {
  if (!L.varlen) {
    const int bh = blockIdx.y;
    const int NB = (L.N + BLK - 1) / BLK;
    P.b = blockIdx.x;
    P.seq = bh;
    P.n = L.N;
    P.rows = min(BLK, L.N - P.b * BLK);
    P.row0 = (long long)bh * L.N + (long long)P.b * BLK;
    P.row_stride = 1;
    P.code_row0 = ((long long)bh * NB + P.b) * BLK;
    P.scale_idx = (long long)bh * NB + P.b;
    return true;
  }
  const int gb = blockIdx.x, h = blockIdx.y;
  const int total = __ldg(L.blk_off + L.batch);
  if (gb >= total) return false;
  const int s = find_segment(L.blk_off, L.batch + 1, gb);
  const int t0 = __ldg(L.cu + s);
  P.n = __ldg(L.cu + s + 1) - t0;
  P.b = gb - __ldg(L.blk_off + s);
  P.seq = s * L.H + h;
  P.rows = min(BLK, P.n - P.b * BLK);
  P.row0 = ((long long)t0 + (long long)P.b * BLK) * L.H + h;
  P.row_stride = L.H;
  P.code_row0 = ((long long)h * L.TBmax + gb) * BLK;
  P.scale_idx = (long long)h * L.TBmax + gb;
  return true;
}

// Load this thread's rows of a 16-bit [.., D] tensor block as floats (zeros
// past the valid rows).
template <int D, bool BF16>
__device__ __forceinline__ void load_block(const void* base, const BlockPos& P,
                                           float (&x)[Tile<D>::NIT][8]) {
  using T = Tile<D>;
  const int c = threadIdx.x % T::CPR, r0 = threadIdx.x / T::CPR;
  const uint16_t* p16 = static_cast<const uint16_t*>(base);
#pragma unroll
  for (int i = 0; i < T::NIT; ++i) {
    const int r = r0 + i * T::RS;
    uint4 u = make_uint4(0, 0, 0, 0);
    if (r < P.rows) {
      const long long row = P.row0 + (long long)r * P.row_stride;
      u = __ldg(reinterpret_cast<const uint4*>(p16 + row * D) + c);
    }
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 f = In16<BF16>::to_float2(w[e]);
      x[i][2 * e] = f.x;
      x[i][2 * e + 1] = f.y;
    }
  }
}

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x / 32;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int i = 1; i < THREADS / 32; ++i) m = fmaxf(m, red[i]);
  return m;
}

// Quantise this thread's values with the block constant s (amax > 0) and store
// the int8 codes of all 128 rows (padding rows get 0).
template <int D>
__device__ __forceinline__ void store_codes(const float (&x)[Tile<D>::NIT][8], float amax,
                                            int8_t* codes, long long code_row0) {
  using T = Tile<D>;
  const int c = threadIdx.x % T::CPR, r0 = threadIdx.x / T::CPR;
  const float s = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
#pragma unroll
  for (int i = 0; i < T::NIT; ++i) {
    const int r = r0 + i * T::RS;
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      int q = __float2int_rn(__fmul_rn(x[i][e], s));
      q = max(-127, min(127, q));
      packed[e / 4] |= (uint32_t)(q & 0xFF) << (8 * (e % 4));
    }
    *reinterpret_cast<uint2*>(codes + (code_row0 + r) * D + 8 * c) =
        make_uint2(packed[0], packed[1]);
  }
}

// ------------------------------------------------------------------ pass 1 --

template <int D, bool BF16, bool FP8>
__global__ void __launch_bounds__(THREADS) quant_pass1_kernel(
    SeqLayout L, const void* __restrict__ q, const void* __restrict__ k,
    const void* __restrict__ v, int8_t* __restrict__ q_codes, float* __restrict__ q_scale,
    unsigned long long* __restrict__ k_sum, uint32_t* __restrict__ v_amax,
    uint32_t* __restrict__ status) {
  using T = Tile<D>;
  __shared__ float red[THREADS / 32];
  __shared__ long long red64[THREADS / 32][D];
  BlockPos P;
  if (!block_pos(L, P)) return;
  const int c = threadIdx.x % T::CPR;
  const int w = threadIdx.x / 32, lane = threadIdx.x & 31;

  // --- Q: per-block quantiser
  {
    float x[T::NIT][8];
    load_block<D, BF16>(q, P, x);
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < T::NIT; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(x[i][e]));
    const float amax = block_max(a, red);
    store_codes<D>(x, amax, q_codes, P.code_row0);
    if (threadIdx.x == 0) q_scale[P.scale_idx] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
  }

  // --- K: exact fixed-point channel sums
  {
    float x[T::NIT][8];
    load_block<D, BF16>(k, P, x);
    long long acc[8];
    bool bad = false;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0;
#pragma unroll
    for (int i = 0; i < T::NIT; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float xv = x[i][e];
        if (fabsf(xv) < 65536.0f) acc[e] += __float2ll_rn(__fmul_rn(xv, 16777216.0f));
        else bad = true;  // non-finite or out of the exact-mean range
      }
    if (bad) set_status(status, ST_RANGE);
#pragma unroll
    for (int o = T::CPR; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
    if (lane < T::CPR)
#pragma unroll
      for (int e = 0; e < 8; ++e) red64[w][8 * c + e] = acc[e];
    __syncthreads();
    if (threadIdx.x < D) {
      long long s = 0;
#pragma unroll
      for (int i = 0; i < THREADS / 32; ++i) s += red64[i][threadIdx.x];
      atomicAdd(k_sum + (long long)P.seq * D + threadIdx.x, (unsigned long long)s);
    }
  }

  // --- V: per-channel max|v| (FP8 P.V only)
  if constexpr (FP8) {
    float x[T::NIT][8];
    load_block<D, BF16>(v, P, x);
    float m[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) m[e] = 0.0f;
#pragma unroll
    for (int i = 0; i < T::NIT; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], fabsf(x[i][e]));
#pragma unroll
    for (int o = T::CPR; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], __shfl_xor_sync(0xffffffffu, m[e], o));
    __syncthreads();
    float* redf = reinterpret_cast<float*>(&red64[0][0]);
    if (lane < T::CPR)
#pragma unroll
      for (int e = 0; e < 8; ++e) redf[w * D + 8 * c + e] = m[e];
    __syncthreads();
    if (threadIdx.x < D) {
      float s = 0.0f;
#pragma unroll
      for (int i = 0; i < THREADS / 32; ++i) s = fmaxf(s, redf[i * D + threadIdx.x]);
      // non-negative floats order like their bit patterns
      atomicMax(v_amax + (long long)P.seq * D + threadIdx.x, __float_as_uint(s));
    }
  }
}

// ------------------------------------------------------------------ pass 2 --

__device__ __forceinline__ float k_mean_value(unsigned long long sum, int n) {
  const double s = __ll2double_rn((long long)sum);
  const double den = __dmul_rn((double)n, 16777216.0);
  return __double2float_rn(__ddiv_rn(s, den));
}

template <int D, bool BF16, bool FP8>
__global__ void __launch_bounds__(THREADS) quant_pass2_kernel(
    SeqLayout L, const void* __restrict__ k, const void* __restrict__ v,
    const unsigned long long* __restrict__ k_sum, const uint32_t* __restrict__ v_amax,
    int8_t* __restrict__ k_codes, float* __restrict__ k_scale, float* __restrict__ k_mean,
    uint8_t* __restrict__ v_codes, float* __restrict__ v_scale) {
  using T = Tile<D>;
  __shared__ float red[THREADS / 32];
  BlockPos P;
  if (!block_pos(L, P)) return;
  const int c = threadIdx.x % T::CPR, r0 = threadIdx.x / T::CPR;
  const long long chan0 = (long long)P.seq * D;

  if (P.b == 0 && threadIdx.x < D)
    k_mean[chan0 + threadIdx.x] = k_mean_value(__ldg(k_sum + chan0 + threadIdx.x), P.n);

  // --- K: smoothing + per-block quantiser
  {
    float m[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) m[e] = k_mean_value(__ldg(k_sum + chan0 + 8 * c + e), P.n);
    float x[T::NIT][8];
    load_block<D, BF16>(k, P, x);
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < T::NIT; ++i) {
      const bool valid = (r0 + i * T::RS) < P.rows;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        x[i][e] = valid ? __fsub_rn(x[i][e], m[e]) : 0.0f;
        a = fmaxf(a, fabsf(x[i][e]));
      }
    }
    const float amax = block_max(a, red);
    store_codes<D>(x, amax, k_codes, P.code_row0);
    if (threadIdx.x == 0) k_scale[P.scale_idx] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
  }

  // --- V: FP8 E4M3 codes with a per-channel scale
  if constexpr (FP8) {
    float sv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float am = __uint_as_float(__ldg(v_amax + chan0 + 8 * c + e));
      sv[e] = am > 0.0f ? __fdiv_rn(448.0f, am) : 0.0f;
    }
    if (P.b == 0 && threadIdx.x < D) {
      const float am = __uint_as_float(__ldg(v_amax + chan0 + threadIdx.x));
      v_scale[chan0 + threadIdx.x] = am > 0.0f ? __fdiv_rn(am, 448.0f) : 0.0f;
    }
    float x[T::NIT][8];
    load_block<D, BF16>(v, P, x);
#pragma unroll
    for (int i = 0; i < T::NIT; ++i) {
      const int r = r0 + i * T::RS;
      if (r < P.rows) {
        uint32_t w0 = pack_e4m3x4(__fmul_rn(x[i][0], sv[0]), __fmul_rn(x[i][1], sv[1]),
                                  __fmul_rn(x[i][2], sv[2]), __fmul_rn(x[i][3], sv[3]));
        uint32_t w1 = pack_e4m3x4(__fmul_rn(x[i][4], sv[4]), __fmul_rn(x[i][5], sv[5]),
                                  __fmul_rn(x[i][6], sv[6]), __fmul_rn(x[i][7], sv[7]));
        const long long row = P.row0 + (long long)r * P.row_stride;
        *reinterpret_cast<uint2*>(v_codes + row * D + 8 * c) = make_uint2(w0, w1);
      }
    }
  }
}

// -------------------------------------------------------------- varlen prep --

// One thread: validates cu_seqlens and writes the block and pair prefix sums.
// On any inconsistency all prefixes are written as 0, so every later kernel of
// the call finds no work, and the status word records SAGE_ERR_BAD_SEQLENS.
__global__ void varlen_prep_kernel(const int32_t* __restrict__ cu, int batch, int max_seqlen,
                                   int total_tokens, int32_t* blk_off, int32_t* pair_off,
                                   uint32_t* status) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  bool ok = __ldg(cu) == 0 && __ldg(cu + batch) == total_tokens;
  int b = 0, p = 0;
  for (int s = 0; s < batch && ok; ++s) {
    const int n = __ldg(cu + s + 1) - __ldg(cu + s);
    if (n < 0 || n > max_seqlen) { ok = false; break; }
    blk_off[s] = b;
    pair_off[s] = p;
    b += (n + BLK - 1) / BLK;
    p += (n + 2 * BLK - 1) / (2 * BLK);
  }
  if (ok) {
    blk_off[batch] = b;
    pair_off[batch] = p;
  } else {
    for (int s = 0; s <= batch; ++s) blk_off[s] = pair_off[s] = 0;
    set_status(status, ST_BAD_SEQLENS);
  }
}

}  // namespace

// ------------------------------------------------------------------ launch --

cudaError_t launch_varlen_prep(const int32_t* cu, int batch, int max_seqlen, int total_tokens,
                               int32_t* blk_off, int32_t* pair_off, uint32_t* status,
                               cudaStream_t st) {
  varlen_prep_kernel<<<1, 32, 0, st>>>(cu, batch, max_seqlen, total_tokens, blk_off, pair_off,
                                       status);
  return cudaGetLastError();
}

template <int D, bool BF16, bool FP8>
static cudaError_t launch_quant_t(const SeqLayout& L, dim3 grid, const void* q, const void* k,
                                  const void* v, int8_t* q_codes, float* q_scale,
                                  int8_t* k_codes, float* k_scale, float* k_mean,
                                  uint8_t* v_codes, float* v_scale, unsigned long long* k_sum,
                                  uint32_t* v_amax, uint32_t* status, cudaStream_t st) {
  quant_pass1_kernel<D, BF16, FP8>
      <<<grid, THREADS, 0, st>>>(L, q, k, v, q_codes, q_scale, k_sum, v_amax, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  quant_pass2_kernel<D, BF16, FP8><<<grid, THREADS, 0, st>>>(L, k, v, k_sum, v_amax, k_codes,
                                                             k_scale, k_mean, v_codes, v_scale);
  return cudaGetLastError();
}

// Runs both passes.  k_sum / v_amax must be zero on entry (the caller clears
// them on the stream).  grid = (blocks per head or TBmax, B*H or H).
cudaError_t launch_quant(const SeqLayout& L, dim3 grid, int D, bool bf16, bool fp8,
                         const void* q, const void* k, const void* v, int8_t* q_codes,
                         float* q_scale, int8_t* k_codes, float* k_scale, float* k_mean,
                         uint8_t* v_codes, float* v_scale, unsigned long long* k_sum,
                         uint32_t* v_amax, uint32_t* status, cudaStream_t st) {
#define SAGE_Q(DD, BB, FF)                                                                    \
  return launch_quant_t<DD, BB, FF>(L, grid, q, k, v, q_codes, q_scale, k_codes, k_scale,    \
                                    k_mean, v_codes, v_scale, k_sum, v_amax, status, st)
  if (D == 64) {
    if (bf16) { if (fp8) SAGE_Q(64, true, true); else SAGE_Q(64, true, false); }
    else { if (fp8) SAGE_Q(64, false, true); else SAGE_Q(64, false, false); }
  } else {
    if (bf16) { if (fp8) SAGE_Q(128, true, true); else SAGE_Q(128, true, false); }
    else { if (fp8) SAGE_Q(128, false, true); else SAGE_Q(128, false, false); }
  }
#undef SAGE_Q
}

}  // namespace sage
