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
// Dense inputs run both passes in one persistent kernel (one CTA per SM): a
// producer warp streams 128-token slabs into shared memory with bulk copies,
// in the work order  p1(head 0) .. p1(head lag-1), p1(lag), p2(0), p1(lag+1),
// p2(1), ...  so that a head's K (and V) is re-read by pass 2 from L2 shortly
// after pass 1 streamed it; eight consumer warps quantise from shared memory.
// A pass-2 block waits (bounded) until all pass-1 blocks of its head are done.
// Variable-length batches use two separate launches.
//
// Every arithmetic step is one IEEE binary32 (or binary64 for the mean)
// operation with round-to-nearest-even, written with explicit __f*_rn
// intrinsics so that no multiply-add contraction changes a code.
//
// Thread layout: 256 threads; a 16-byte vector holds 8 channels; thread t owns
// channel group c = t % (D/8) of rows t/(D/8) + i*(256/(D/8)).  Consecutive
// threads read consecutive 16-byte vectors of one row: fully coalesced.
#include <type_traits>

#include "common.cuh"
#include "ptx.cuh"

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

__device__ __forceinline__ void dense_block_pos(const SeqLayout& L, int bh, int b, BlockPos& P) {
  const int NB = (L.N + BLK - 1) / BLK;
  P.b = b;
  P.seq = bh;
  P.n = L.N;
  P.rows = min(BLK, L.N - P.b * BLK);
  P.row0 = (long long)bh * L.N + (long long)P.b * BLK;
  P.row_stride = 1;
  P.code_row0 = ((long long)bh * NB + P.b) * BLK;
  P.scale_idx = (long long)bh * NB + P.b;
}

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

// Issue the loads of this thread's rows of a 16-bit [.., D] tensor block
// (zeros past the valid rows).  Callers issue every tensor's loads before they
// use any of them, so a CTA keeps all its 16-byte requests in flight at once.
template <int D>
__device__ __forceinline__ void load_raw(const void* base, const BlockPos& P,
                                         uint4 (&u)[Tile<D>::NIT]) {
  using T = Tile<D>;
  const int c = threadIdx.x % T::CPR, r0 = threadIdx.x / T::CPR;
  const uint16_t* p16 = static_cast<const uint16_t*>(base);
#pragma unroll
  for (int i = 0; i < T::NIT; ++i) {
    const int r = r0 + i * T::RS;
    u[i] = make_uint4(0, 0, 0, 0);
    if (r < P.rows) {
      const long long row = P.row0 + (long long)r * P.row_stride;
      u[i] = __ldg(reinterpret_cast<const uint4*>(p16 + row * D) + c);
    }
  }
}

template <int D, bool BF16>
__device__ __forceinline__ void to_float(const uint4 (&u)[Tile<D>::NIT],
                                         float (&x)[Tile<D>::NIT][8]) {
#pragma unroll
  for (int i = 0; i < Tile<D>::NIT; ++i) {
    const uint32_t w[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = In16<BF16>::to_float2(w[e]);
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

// 1.5 * 2^23: for |y| < 2^22, the fp32 sum y + kMagic is kMagic + rint(y)
// (round to nearest even), and its low mantissa byte is rint(y) mod 256.
constexpr float kMagic = 12582912.0f;

// Low bytes of four floats' bit patterns, packed (a in byte 0).
__device__ __forceinline__ uint32_t low_bytes4(float a, float b, float c, float d) {
  const uint32_t ab = __byte_perm(__float_as_uint(a), __float_as_uint(b), 0x0040);
  const uint32_t cd = __byte_perm(__float_as_uint(c), __float_as_uint(d), 0x0040);
  return __byte_perm(ab, cd, 0x5410);
}

// Per-token quantiser: every row gets its own delta, the max |x - mean| over
// its D channels (held by the D/8 consecutive lanes that own the row, combined
// with shuffles); codes as in the block quantiser.  Padding rows get code 0
// and delta 0.  delta[code_row0 + r] receives the row deltas.
template <int D, bool BF16, bool SUB, bool FULL>
__device__ __forceinline__ void regs_codes_per_row(const uint4 (&u)[Tile<D>::NIT], int rows,
                                                   const float (&mean)[8], int8_t* codes,
                                                   float* delta, long long code_row0) {
  using T = Tile<D>;
  const int c = threadIdx.x % T::CPR, r0 = threadIdx.x / T::CPR;
  float2 nm[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) nm[e] = make_float2(-mean[2 * e], -mean[2 * e + 1]);
#pragma unroll
  for (int i = 0; i < T::NIT; ++i) {
    const int r = r0 + i * T::RS;
    const bool valid = FULL || r < rows;
    const uint32_t w[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
    float2 f[4];
    float a = 0.0f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      f[e] = In16<BF16>::to_float2(w[e]);
      if constexpr (SUB) f[e] = __fadd2_rn(f[e], nm[e]);
      a = fmaxf(a, fmaxf(fabsf(f[e].x), fabsf(f[e].y)));
    }
    if (!valid) a = 0.0f;
#pragma unroll
    for (int o = T::CPR / 2; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    const float s = a > 0.0f ? __fdiv_rn(127.0f, a) : 0.0f;
    float2 y[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      y[e] = make_float2(__fadd_rn(__fmul_rn(f[e].x, s), kMagic),
                         __fadd_rn(__fmul_rn(f[e].y, s), kMagic));
    uint2 out = make_uint2(low_bytes4(y[0].x, y[0].y, y[1].x, y[1].y),
                           low_bytes4(y[2].x, y[2].y, y[3].x, y[3].y));
    if (!valid) out = make_uint2(0u, 0u);
    *reinterpret_cast<uint2*>(codes + (code_row0 + r) * D + 8 * c) = out;
    if (c == 0) delta[code_row0 + r] = a > 0.0f ? __fdiv_rn(a, 127.0f) : 0.0f;
  }
}

// ------------------------------------------------------------------ pass 1 --

template <int D, bool BF16, bool FP8>
__device__ __forceinline__ void pass1_block(
    const BlockPos& P, const void* __restrict__ q, const void* __restrict__ k,
    const void* __restrict__ v, int8_t* __restrict__ q_codes, float* __restrict__ q_scale,
    unsigned long long* __restrict__ k_sum, uint32_t* __restrict__ v_amax,
    uint32_t* __restrict__ status, int parts, int tok) {
  using T = Tile<D>;
  __shared__ float red[THREADS / 32];
  __shared__ long long red64[THREADS / 32][D];
  const int c = threadIdx.x % T::CPR;
  const int w = threadIdx.x / 32, lane = threadIdx.x & 31;
  const bool has_q = (parts & QUANT_Q) != 0, has_kv = (parts & QUANT_KV) != 0;

  uint4 rq[T::NIT], rk[T::NIT], rv[FP8 ? T::NIT : 1];
  if (has_q) load_raw<D>(q, P, rq);
  if (has_kv) load_raw<D>(k, P, rk);
  if constexpr (FP8) {
    if (has_kv) load_raw<D>(v, P, rv);
  }

  // --- Q: per-token quantiser, or per-block below
  if (has_q && tok) {
    const float zero8[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    regs_codes_per_row<D, BF16, false, false>(rq, P.rows, zero8, q_codes, q_scale, P.code_row0);
  } else if (has_q) {
    float x[T::NIT][8];
    to_float<D, BF16>(rq, x);
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
  if (has_kv) {
    float x[T::NIT][8];
    to_float<D, BF16>(rk, x);
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
  if constexpr (FP8) if (has_kv) {
    float x[T::NIT][8];
    to_float<D, BF16>(rv, x);
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

template <int D, bool BF16, bool FP8>
__global__ void __launch_bounds__(THREADS) quant_pass1_kernel(
    SeqLayout L, const void* __restrict__ q, const void* __restrict__ k,
    const void* __restrict__ v, int8_t* __restrict__ q_codes, float* __restrict__ q_scale,
    unsigned long long* __restrict__ k_sum, uint32_t* __restrict__ v_amax,
    uint32_t* __restrict__ status, int parts, int tok) {
  BlockPos P;
  if (!block_pos(L, P)) return;
  pass1_block<D, BF16, FP8>(P, q, k, v, q_codes, q_scale, k_sum, v_amax, status, parts, tok);
}

// ------------------------------------------------------------------ pass 2 --

__device__ __forceinline__ float k_mean_value(unsigned long long sum, int n) {
  const double s = __ll2double_rn((long long)sum);
  const double den = __dmul_rn((double)n, 16777216.0);
  return __double2float_rn(__ddiv_rn(s, den));
}

template <int D, bool BF16, bool FP8>
__device__ __forceinline__ void pass2_block(
    const BlockPos& P, const void* __restrict__ k, const void* __restrict__ v,
    const unsigned long long* k_sum, const uint32_t* v_amax,
    int8_t* __restrict__ k_codes, float* __restrict__ k_scale, float* __restrict__ k_mean,
    uint8_t* __restrict__ v_codes, float* __restrict__ v_scale, int tok) {
  using T = Tile<D>;
  __shared__ float red[THREADS / 32];
  __shared__ float s_chan[2][D];  // K channel means, V scale factors
  const int c = threadIdx.x % T::CPR, r0 = threadIdx.x / T::CPR;
  const long long chan0 = (long long)P.seq * D;

  uint4 rk[T::NIT], rv[FP8 ? T::NIT : 1];
  load_raw<D>(k, P, rk);
  if constexpr (FP8) load_raw<D>(v, P, rv);

  if (threadIdx.x < D) {
    const float mu = k_mean_value(__ldcg(k_sum + chan0 + threadIdx.x), P.n);
    s_chan[0][threadIdx.x] = mu;
    if (P.b == 0) k_mean[chan0 + threadIdx.x] = mu;
    if constexpr (FP8) {
      const float am = __uint_as_float(__ldcg(v_amax + chan0 + threadIdx.x));
      s_chan[1][threadIdx.x] = am > 0.0f ? __fdiv_rn(448.0f, am) : 0.0f;
      if (P.b == 0) v_scale[chan0 + threadIdx.x] = am > 0.0f ? __fdiv_rn(am, 448.0f) : 0.0f;
    }
  }
  __syncthreads();

  // --- K: smoothing + per-token quantiser, or per-block below
  if (tok) {
    float m[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) m[e] = s_chan[0][8 * c + e];
    regs_codes_per_row<D, BF16, true, false>(rk, P.rows, m, k_codes, k_scale, P.code_row0);
  } else {
    float m[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) m[e] = s_chan[0][8 * c + e];
    float x[T::NIT][8];
    to_float<D, BF16>(rk, x);
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
    for (int e = 0; e < 8; ++e) sv[e] = s_chan[1][8 * c + e];
    float x[T::NIT][8];
    to_float<D, BF16>(rv, x);
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

template <int D, bool BF16, bool FP8>
__global__ void __launch_bounds__(THREADS) quant_pass2_kernel(
    SeqLayout L, const void* __restrict__ k, const void* __restrict__ v,
    const unsigned long long* __restrict__ k_sum, const uint32_t* __restrict__ v_amax,
    int8_t* __restrict__ k_codes, float* __restrict__ k_scale, float* __restrict__ k_mean,
    uint8_t* __restrict__ v_codes, float* __restrict__ v_scale, int tok) {
  BlockPos P;
  if (!block_pos(L, P)) return;
  pass2_block<D, BF16, FP8>(P, k, v, k_sum, v_amax, k_codes, k_scale, k_mean, v_codes, v_scale,
                            tok);
}

// ------------------------------------------------------------ Q smoothing --
//
// SageAttention2's smoothing of Q (dtcms.com page, v2 bullet 2): each
// 128-token query block I is quantised after subtracting its own channel mean
// qmean_I, and the part of the logit that the mean carries, qmean_I . k~_j,
// is added back per key by the attention kernel.

// One CTA per (query block, head): the exact block mean (the K mean's
// fixed-point sum, over this block's rows), then per-block codes of
// fp32(q - qmean_I) with one delta, as the K blocks are coded.
// Dense: grid (blocks, B*H), q_mean [B*H][NB][D]; varlen: grid (TBmax, H),
// q_mean [H][TBmax][D] (indexed like the deltas).
template <int D, bool BF16>
__global__ void __launch_bounds__(THREADS) quant_q_smooth_kernel(
    SeqLayout L, const void* __restrict__ q, int8_t* __restrict__ q_codes,
    float* __restrict__ q_scale, float* __restrict__ q_mean, uint32_t* __restrict__ status) {
  using T = Tile<D>;
  __shared__ float red[THREADS / 32];
  __shared__ long long red64[THREADS / 32][D];
  __shared__ float s_mean[D];
  BlockPos P;
  if (!block_pos(L, P)) return;
  const int c = threadIdx.x % T::CPR, r0 = threadIdx.x / T::CPR;
  const int w = threadIdx.x / 32, lane = threadIdx.x & 31;

  uint4 rq[T::NIT];
  load_raw<D>(q, P, rq);
  float x[T::NIT][8];
  to_float<D, BF16>(rq, x);

  // exact channel sums of rint(x * 2^24) (padding rows are zeros)
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
    long long sum = 0;
#pragma unroll
    for (int i = 0; i < THREADS / 32; ++i) sum += red64[i][threadIdx.x];
    const float mu = k_mean_value((unsigned long long)sum, P.rows);
    s_mean[threadIdx.x] = mu;
    q_mean[P.scale_idx * D + threadIdx.x] = mu;
  }
  __syncthreads();

  float m[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) m[e] = s_mean[8 * c + e];
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
  store_codes<D>(x, amax, q_codes, P.code_row0);
  if (threadIdx.x == 0) q_scale[P.scale_idx] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
}

// Where the mean term of one (key tile, query head) CTA lives.
struct BiasPos {
  int n;                 // sequence length
  int nb;                // its query / key blocks
  int qb0, qend;          // query blocks [qb0, qend) written (varlen: all)
  int J;                 // key tile within the sequence
  const uint16_t* k0;    // key token 0 of the sequence, this key/value head
  long long k_stride;    // elements between consecutive tokens of k
  const float* kmean;    // [D] of the key/value head
  const float* qm;       // [nb][D] block means of the query head
  float* out;            // rows of the (sequence, query head), row I - qb0 for block I, nb*128 floats each
};

// Dense: grid (key tiles, B*H), the term of query blocks [qb0, qb0 + qrows)
// into [B*H][qrows][NB*128]; varlen: grid (TBmax, H) over the global key
// blocks, every query block.
__device__ __forceinline__ bool bias_pos(const SeqLayout& L, int Hq, int Hkv, int D,
                                         const void* k, const float* k_mean, const float* q_mean,
                                         float* bias, long long head_stride,
                                         const long long* sq_off, int qb0, int qrows,
                                         BiasPos& P) {
  if (!L.varlen) {
    const int NB = (L.N + BLK - 1) / BLK;
    const int bh = blockIdx.y, b = bh / Hq, h = bh - b * Hq;
    const int bkv = b * Hkv + h / (Hq / Hkv);
    P.n = L.N;
    P.nb = NB;
    P.qb0 = qb0;
    P.qend = min(NB, qb0 + qrows);
    P.J = blockIdx.x;
    P.k0 = static_cast<const uint16_t*>(k) + (long long)bkv * L.N * D;
    P.k_stride = D;
    P.kmean = k_mean + (long long)bkv * D;
    P.qm = q_mean + (long long)bh * NB * D;
    P.out = bias + (long long)bh * qrows * NB * BLK;
    return true;
  }
  const int gb = blockIdx.x, h = blockIdx.y;
  const int total = __ldg(L.blk_off + L.batch);
  if (gb >= total) return false;
  const int s = find_segment(L.blk_off, L.batch + 1, gb);
  const int b0 = __ldg(L.blk_off + s);
  const int t0 = __ldg(L.cu + s);
  const int hk = h / (Hq / Hkv);
  P.n = __ldg(L.cu + s + 1) - t0;
  P.nb = (P.n + BLK - 1) / BLK;
  P.qb0 = 0;
  P.qend = P.nb;
  P.J = gb - b0;
  P.k0 = static_cast<const uint16_t*>(k) + ((long long)t0 * Hkv + hk) * D;
  P.k_stride = (long long)Hkv * D;
  P.kmean = k_mean + ((long long)s * Hkv + hk) * D;
  P.qm = q_mean + ((long long)h * L.TBmax + b0) * D;
  P.out = bias + (long long)h * head_stride + __ldg(sq_off + s) * BLK;
  return true;
}

// The per-key term: bias[I][j] = fp32(acc * kappa), acc the fp32 fused
// multiply-adds of qmean_I[d] and k~_j[d] = fp32(k_j[d] - kmean[d]) in
// channel order, for the key/value head that the query head reads.  The fixed
// order makes the value (and every FP8 code of P that depends on it) the
// oracle's, bit for bit.
// One CTA per (128-key tile J, query head), one thread per key: the thread
// keeps its k~ row in registers and runs over the query blocks, G at a time
// (G independent accumulators, paired into packed FMAs), whose means the CTA
// first stages in shared memory channel-major (every thread then reads the
// same address: a broadcast).  With a causal mask, blocks I < J never see the
// tile and are skipped.  Keys past n get 0.
template <int D, bool BF16>
__global__ void __launch_bounds__(128) q_smooth_bias_kernel(
    SeqLayout L, int H, int Hkv, int causal, float kappa, const void* __restrict__ k,
    const float* __restrict__ k_mean, const float* __restrict__ q_mean,
    float* __restrict__ bias, long long head_stride, const long long* __restrict__ sq_off,
    int qb0, int qrows) {
  constexpr int G = 8;                 // query blocks per pass
  __shared__ __align__(16) float s_qm[D][G];  // means of G blocks, channel-major
  BiasPos P;
  if (!bias_pos(L, H, Hkv, D, k, k_mean, q_mean, bias, head_stride, sq_off, qb0, qrows, P))
    return;
  const int jl = P.J * BLK + threadIdx.x;  // key within the sequence
  float kt[D];
  if (jl < P.n) {
    const uint4* src = reinterpret_cast<const uint4*>(P.k0 + (long long)jl * P.k_stride);
    const float2* km = reinterpret_cast<const float2*>(P.kmean);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      const uint4 u = __ldg(src + c);
      const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = In16<BF16>::to_float2(wv[e]);
        const float2 mu = __ldg(km + 4 * c + e);
        kt[8 * c + 2 * e] = __fsub_rn(f.x, mu.x);
        kt[8 * c + 2 * e + 1] = __fsub_rn(f.y, mu.y);
      }
    }
  } else {
#pragma unroll
    for (int c = 0; c < D; ++c) kt[c] = 0.0f;
  }
  const long long NP = (long long)P.nb * BLK;
  float* out = P.out + jl;
  for (int I0 = max(causal ? P.J : 0, P.qb0); I0 < P.qend; I0 += G) {
    __syncthreads();  // the previous group's means are no longer read
    for (int x = threadIdx.x; x < G * D; x += 128) {
      const int g = x / D, d = x - g * D;
      s_qm[d][g] = I0 + g < P.qend ? __ldg(P.qm + (long long)(I0 + g) * D + d) : 0.0f;
    }
    __syncthreads();
    float2 acc[G / 2];
#pragma unroll
    for (int g2 = 0; g2 < G / 2; ++g2) acc[g2] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int d = 0; d < D; ++d) {
      const float2 kd = make_float2(kt[d], kt[d]);
      const float4* m4 = reinterpret_cast<const float4*>(&s_qm[d][0]);
#pragma unroll
      for (int g4 = 0; g4 < G / 4; ++g4) {
        const float4 m = m4[g4];
        acc[2 * g4] = __ffma2_rn(make_float2(m.x, m.y), kd, acc[2 * g4]);
        acc[2 * g4 + 1] = __ffma2_rn(make_float2(m.z, m.w), kd, acc[2 * g4 + 1]);
      }
    }
#pragma unroll
    for (int g2 = 0; g2 < G / 2; ++g2) {
      const int I = I0 + 2 * g2 - P.qb0;  // row in the output
      if (I0 + 2 * g2 < P.qend) out[(long long)I * NP] = __fmul_rn(acc[g2].x, kappa);
      if (I0 + 2 * g2 + 1 < P.qend) out[(long long)(I + 1) * NP] = __fmul_rn(acc[g2].y, kappa);
    }
  }
}

// ---------------------------------------------------------- streamed, dense --
//
// Dense inputs: one persistent CTA per SM.  Warp 8 claims work items from a
// global counter and streams each item's 128-token slabs (in the dense layout
// a block of one head is one contiguous [rows, D] slab per tensor) into a ring
// of shared-memory slots with cp.async.bulk; warps 0-7 take the slots in the
// same order and write codes, scales and sums.
//
// Work items are (pass, head, block) in groups of NB blocks ordered
//   p1(0) .. p1(lag-1), then p1(u), p2(u-lag) for u = lag .. U-1, then the
//   remaining p2,
// so that pass 2 re-reads a head's K (and V) from L2 shortly after pass 1
// streamed it (pass-1 K and V slabs are loaded with an evict-last L2 policy,
// everything else evict-first).  Before it loads a pass-2 item the producer
// waits (bounded) until every pass-1 block of that head is counted done; those
// were claimed earlier by running CTAs, which finish them without waiting on
// anything claimed later, so the wait ends.

__device__ __forceinline__ void fused_item(int x, int NB, int U, int lag, int& pass, int& u,
                                           int& b) {
  const int g = x / NB;
  b = x - g * NB;
  if (g < lag) { pass = 1; u = g; return; }
  const int k = g - lag;
  if (k < 2 * (U - lag)) {
    u = lag + k / 2;
    if (k & 1) { pass = 2; u -= lag; } else { pass = 1; }
    return;
  }
  pass = 2;
  u = U - lag + (k - 2 * (U - lag));
}

template <int D>
struct Stream {
  static constexpr int CONSUMERS = 256;                   // warps 0-7
  static constexpr int THREADS = CONSUMERS + 32;          // + producer warp 8
  static constexpr int SLOT = BLK * D * 2;                // one [128, D] 16-bit slab
  static constexpr int NS = D == 128 ? 3 : 6;             // ring slots (96 KiB)
  static constexpr size_t SMEM = (size_t)NS * SLOT;
  static constexpr int CTAS_PER_SM = 2;
};

// What a launch quantises: Q, K (with V for FP8 P.V), or both.  Grouped-
// query attention quantises Q over the query heads and K, V over the key /
// value heads in two launches.
enum Parts { PART_Q = 1, PART_KV = 2 };

// Slabs of one work item: pass 1 = (Q,) (K, V), pass 2 = K (, V).
__device__ __forceinline__ int tensors_of(int pass, int parts, bool fp8) {
  const int nkv = fp8 ? 2 : 1;
  if (pass == 2) return nkv;
  return ((parts & PART_Q) ? 1 : 0) + ((parts & PART_KV) ? nkv : 0);
}

// Work item x -> (pass, unit, block).  Without K there is no pass 2 and the
// items are simply the blocks in order.
__device__ __forceinline__ void item_of(int x, int NB, int U, int lag, int parts, int& pass,
                                        int& u, int& b) {
  if (parts & PART_KV) {
    fused_item(x, NB, U, lag, pass, u, b);
  } else {
    pass = 1;
    u = x / NB;
    b = x - u * NB;
  }
}

// Consumer-side helpers.  Thread t owns the 16-byte chunk c = t % (D/8) of
// rows r0 + i*RS of a slab (as in the two-launch path); it copies them from
// shared memory into registers once (zeros past the valid rows), so the slot
// can be handed back to the producer at once.  FULL: all 128 rows valid.

template <int D, bool FULL>
__device__ __forceinline__ void slab_to_regs(const uint4* slab, int rows,
                                             uint4 (&u)[Tile<D>::NIT]) {
  using T = Tile<D>;
  const int c = threadIdx.x % T::CPR, r0 = threadIdx.x / T::CPR;
#pragma unroll
  for (int i = 0; i < T::NIT; ++i) {
    const int r = r0 + i * T::RS;
    u[i] = (FULL || r < rows) ? slab[r * T::CPR + c] : make_uint4(0u, 0u, 0u, 0u);
  }
}

// max |x| over the thread's values (zeros do not change it).  The max of
// 16-bit values is exact; a NaN is ignored as by fmaxf.
template <int D, bool BF16>
__device__ __forceinline__ float regs_absmax(const uint4 (&u)[Tile<D>::NIT]) {
  uint32_t m[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int i = 0; i < Tile<D>::NIT; ++i) {
    m[0] = In16<BF16>::absmax2(m[0], u[i].x);
    m[1] = In16<BF16>::absmax2(m[1], u[i].y);
    m[2] = In16<BF16>::absmax2(m[2], u[i].z);
    m[3] = In16<BF16>::absmax2(m[3], u[i].w);
  }
  float a = 0.0f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = In16<BF16>::to_float2(m[e] & 0x7fff7fffu);
    a = fmaxf(a, fmaxf(f.x, f.y));
  }
  return a;
}

// codes = rint((x - mean) * s) for the valid rows, 0 for padding rows, with
// s = 127/amax.  |x - mean| <= amax bounds |(x - mean) * s| by 127(1 + 2^-23),
// so the codes need no clamp.  Each step is one IEEE fp32 operation
// (x - mean, the product, the rounding), as in the two-launch path.
template <int D, bool BF16, bool SUB, bool FULL>
__device__ __forceinline__ void regs_codes(const uint4 (&u)[Tile<D>::NIT], int rows, float amax,
                                           const float (&mean)[8], int8_t* codes,
                                           long long code_row0) {
  using T = Tile<D>;
  const int c = threadIdx.x % T::CPR, r0 = threadIdx.x / T::CPR;
  const float s = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
  float2 nm[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) nm[e] = make_float2(-mean[2 * e], -mean[2 * e + 1]);
#pragma unroll
  for (int i = 0; i < T::NIT; ++i) {
    const int r = r0 + i * T::RS;
    const uint32_t w[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
    float2 y[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 f = In16<BF16>::to_float2(w[e]);
      if constexpr (SUB) f = __fadd2_rn(f, nm[e]);
      // scalar __fmul_rn / __fadd_rn: documented never to be fused into an
      // fma (which would round x*s and its rint as one step); the packed
      // forms were fused here
      y[e] = make_float2(__fadd_rn(__fmul_rn(f.x, s), kMagic), __fadd_rn(__fmul_rn(f.y, s), kMagic));
    }
    uint2 out = make_uint2(low_bytes4(y[0].x, y[0].y, y[1].x, y[1].y),
                           low_bytes4(y[2].x, y[2].y, y[3].x, y[3].y));
    if (!FULL && r >= rows) out = make_uint2(0u, 0u);
    *reinterpret_cast<uint2*>(codes + (code_row0 + r) * D + 8 * c) = out;
  }
}

// max |x - mean| over the thread's valid rows.
template <int D, bool BF16, bool FULL>
__device__ __forceinline__ float regs_absmax_sub(const uint4 (&u)[Tile<D>::NIT], int rows,
                                                 const float (&mean)[8]) {
  using T = Tile<D>;
  const int r0 = threadIdx.x / T::CPR;
  float2 nm[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) nm[e] = make_float2(-mean[2 * e], -mean[2 * e + 1]);
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < T::NIT; ++i) {
    if (FULL || r0 + i * T::RS < rows) {
      const uint32_t w[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 y = __fadd2_rn(In16<BF16>::to_float2(w[e]), nm[e]);
        a = fmaxf(a, fmaxf(fabsf(y.x), fabsf(y.y)));
      }
    }
  }
  return a;
}

// Exact sums of rint(x * 2^24) over the thread's rows, per channel, as two
// fp32 sums: hi = sum of h = rint(16x), fr = sum of d = 16x - h, so that the
// total is 2^20 (hi + fr).  For |x| < 2^16: |h| <= 2^20 and d is exact with
// |d| <= 1/2 and a multiple of 2^-20 (x is a multiple of 2^-24 for every
// fp16, and for every bf16 of magnitude 2^-17 or more; smaller bf16 values
// take one more rounding of d to that grid, which is rint of x * 2^24).  Over
// the at most 16 rows that meet in one warp, |sum h| <= 2^24 and |sum d| <= 8
// on a 2^-20 grid: neither sum ever rounds.
template <int D, bool BF16>
__device__ __forceinline__ void regs_fixed_sums(const uint4 (&u)[Tile<D>::NIT], float2 (&hi)[4],
                                                float2 (&fr)[4], uint32_t& absbits) {
  const float2 M2 = make_float2(kMagic, kMagic), nM2 = make_float2(-kMagic, -kMagic);
  const float2 k16 = make_float2(16.0f, 16.0f);
  const float2 G2 = make_float2(12.0f, 12.0f), nG2 = make_float2(-12.0f, -12.0f);  // 1.5*2^3
#pragma unroll
  for (int e = 0; e < 4; ++e) hi[e] = fr[e] = make_float2(0.0f, 0.0f);
  absbits = 0u;
#pragma unroll
  for (int i = 0; i < Tile<D>::NIT; ++i) {
    const uint32_t w[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if constexpr (BF16) absbits = __vmaxu2(absbits, w[e] & 0x7fff7fffu);
      const float2 f = In16<BF16>::to_float2(w[e]);
      const float2 h = __fadd2_rn(__ffma2_rn(f, k16, M2), nM2);       // rint(16x)
      float2 d = __ffma2_rn(f, k16, make_float2(-h.x, -h.y));        // 16x - h, exact
      if constexpr (BF16) d = __fadd2_rn(__fadd2_rn(d, G2), nG2);     // onto the 2^-20 grid
      hi[e] = __fadd2_rn(hi[e], h);
      fr[e] = __fadd2_rn(fr[e], d);
    }
  }
}

// Block max over the 256 consumer threads; red is [2][8], used alternately.
__device__ __forceinline__ float consumer_block_max(float v, float* red, int& par) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) red[par * 8 + threadIdx.x / 32] = v;
  ptx::named_sync<256>();
  float m = red[par * 8];
#pragma unroll
  for (int i = 1; i < 8; ++i) m = fmaxf(m, red[par * 8 + i]);
  par ^= 1;
  return m;
}

__device__ __forceinline__ void release_slot(uint64_t* empty) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(empty);
}

// sync[0]: work counter; sync[1 + u]: pass-1 blocks of head u completed.
template <int D, bool BF16, bool FP8>
__global__ void __launch_bounds__(Stream<D>::THREADS, Stream<D>::CTAS_PER_SM) quant_stream_kernel(
    SeqLayout L, int U, int lag, int parts, int tok, const void* __restrict__ q,
    const void* __restrict__ k, const void* __restrict__ v, int8_t* __restrict__ q_codes,
    float* __restrict__ q_scale, int8_t* __restrict__ k_codes, float* __restrict__ k_scale,
    float* __restrict__ k_mean, uint8_t* __restrict__ v_codes, float* __restrict__ v_scale,
    unsigned long long* k_sum, uint32_t* v_amax, uint32_t* status, unsigned int* sync) {
  using S = Stream<D>;
  using T = Tile<D>;
  constexpr int NS = S::NS;
  const bool has_q = (parts & PART_Q) != 0, has_kv = (parts & PART_KV) != 0;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t full[NS], empty[NS];
  __shared__ int info[NS];
  __shared__ float red[16];
  // per slot, written by the producer with a pass-2 slab: the K channel
  // means (K slab) or the V scale factors 448/max|v| (V slab)
  __shared__ float s_side[NS][D];
  // pass 1: the consumer warps' partial channel sums (or V maxima, as float
  // bits) of the block, combined after a barrier
  __shared__ long long red64[8][D];
  __shared__ int s_abort, s_filled, s_consumed;

  const int NB = (L.N + BLK - 1) / BLK;
  const int total = (has_kv ? 2 : 1) * U * NB;
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], 8);
    }
    s_abort = 0;
    s_filled = 0;
    s_consumed = 0;
    ptx::fence_barrier_init();
  }
  __syncthreads();

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    const uint64_t pol_first = ptx::l2_evict_first(), pol_last = ptx::l2_evict_last();
    int fill = 0;
    while (true) {
      int x = 0;
      if (lane == 0) x = (int)atomicAdd(sync, 1u);
      x = __shfl_sync(0xffffffffu, x, 0);
      const bool end = x >= total;
      int pass = 0, u = 0, b = 0;
      if (!end) item_of(x, NB, U, lag, parts, pass, u, b);
      const unsigned target = (unsigned)NB;
      if (!end && pass == 2 && lane == 0) {
        const uint32_t* done = sync + 1 + u;
        if (ptx::ld_acquire_gpu(done) < target) {
          const long long t0 = clock64();
          while (ptx::ld_acquire_gpu(done) < target) {
            if (*reinterpret_cast<volatile uint32_t*>(status) & ST_TIMEOUT) break;
            if (clock64() - t0 > SAGE_WAIT_LIMIT_CYCLES) {
              set_status(status, ST_TIMEOUT);
              break;
            }
            __nanosleep(128);
          }
        }
      }
      __syncwarp();
      const int nt = end ? 1 : tensors_of(pass, parts, FP8);
      const long long row0 = (long long)u * L.N + (long long)b * BLK;
      const int rows = end ? 0 : min(BLK, L.N - b * BLK);
      bool ok = true;
      for (int t = 0; t < nt && ok; ++t) {
        const int slot = fill % NS;
        if (fill >= NS) {  // lane 0 waits; the outcome is the warp's
          if (lane == 0) ok = ptx::mbar_wait(&empty[slot], ((fill / NS) & 1) ^ 1);
          ok = __shfl_sync(0xffffffffu, ok, 0);
        }
        if (!ok) break;
        // tensor t of this item (0 = Q, 1 = K, 2 = V)
        const int which = (pass == 1 && has_q) ? t : t + 1;
        if (lane == 0) {
          info[slot] = end ? -1 : x;
          if (!end) {
            const void* base = which == 0 ? q : which == 1 ? k : v;
            const uint32_t bytes = (uint32_t)rows * D * 2;
            ptx::mbar_expect_tx(&full[slot], bytes);
            ptx::bulk_load(smem + (size_t)slot * S::SLOT,
                           static_cast<const uint16_t*>(base) + row0 * D, bytes, &full[slot],
                           (pass == 1 && which > 0) ? pol_last : pol_first);
          }
        }
        if (!end && pass == 2) {
          // per-channel constants of this head, while the copy is in flight
          // (lane 0's acquire of the completion count, then __syncwarp, orders
          // these reads after every pass-1 block's sums)
          const long long chan0 = (long long)u * D;
#pragma unroll
          for (int j = 0; j < D / 32; ++j) {
            const int ch = lane + 32 * j;
            float val;
            if (which == 1) {
              val = k_mean_value(__ldcg(k_sum + chan0 + ch), L.N);
              if (b == 0) k_mean[chan0 + ch] = val;
            } else {
              const float am = __uint_as_float(__ldcg(v_amax + chan0 + ch));
              val = am > 0.0f ? __fdiv_rn(448.0f, am) : 0.0f;
              if (b == 0) v_scale[chan0 + ch] = am > 0.0f ? __fdiv_rn(am, 448.0f) : 0.0f;
            }
            s_side[slot][ch] = val;
          }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&full[slot]);  // release: info, s_side
        ++fill;
      }
      if (!ok) {
        if (lane == 0) {
          set_status(status, ST_TIMEOUT);
          s_abort = 1;
        }
        break;
      }
      const bool stop = end || *reinterpret_cast<volatile int*>(&s_abort);
      if (__shfl_sync(0xffffffffu, stop, 0)) break;
    }
    if (lane == 0) s_filled = fill;
  } else {
    // ----------------------------------------------------------- consumers
    int cidx = 0, par = 0;
    bool finished = false;  // left the loop at the end-of-work marker
    const int c = threadIdx.x % T::CPR;
    while (true) {
      const int slot0 = cidx % NS;
      bool ok = ptx::mbar_wait(&full[slot0], (cidx / NS) & 1);
      ok = ptx::named_all<256>(ok && !*reinterpret_cast<volatile int*>(&s_abort));
      if (!ok) break;
      const int x = info[slot0];
      if (x < 0) {
        ++cidx;
        finished = true;
        break;
      }
      int pass, u, b;
      item_of(x, NB, U, lag, parts, pass, u, b);
      const int nt = tensors_of(pass, parts, FP8);
      BlockPos P;
      dense_block_pos(L, u, b, P);
      const long long chan0 = (long long)P.seq * D;
      auto slab = [&](int t) {
        return reinterpret_cast<const uint4*>(smem + (size_t)((cidx + t) % NS) * S::SLOT);
      };
      auto empty_of = [&](int t) { return &empty[(cidx + t) % NS]; };
      const float zero8[8] = {0, 0, 0, 0, 0, 0, 0, 0};

      const bool full_blk = P.rows == BLK;
      uint4 rg[T::NIT];
      // slab t of this item -> registers; free the slot.  Slabs after the
      // first are awaited only here, so their copies overlap the work on the
      // earlier ones; a wait that runs out marks the abort, which the next
      // loop's uniform check sees (this item's values are then garbage).
      auto await_slab = [&](int t) {
        if (t > 0 && !ptx::mbar_wait(&full[(cidx + t) % NS], ((cidx + t) / NS) & 1)) {
          set_status(status, ST_TIMEOUT);
          s_abort = 1;
        }
      };
      auto take = [&](int t) {  // (after await_slab(t))
        if (full_blk) slab_to_regs<D, true>(slab(t), P.rows, rg);
        else slab_to_regs<D, false>(slab(t), P.rows, rg);
        release_slot(empty_of(t));
      };
      auto codes = [&](float amax, const float (&mean)[8], int8_t* out, auto sub) {
        constexpr bool SUB = decltype(sub)::value;
        if (full_blk) regs_codes<D, BF16, SUB, true>(rg, P.rows, amax, mean, out, P.code_row0);
        else regs_codes<D, BF16, SUB, false>(rg, P.rows, amax, mean, out, P.code_row0);
      };

      if (pass == 1) {
        const int tk = has_q ? 1 : 0;  // slab index of K (V follows it)
        // Q: per-block (or per-token) quantiser
        if (has_q && tok) {
          take(0);
          if (full_blk)
            regs_codes_per_row<D, BF16, false, true>(rg, P.rows, zero8, q_codes, q_scale,
                                                     P.code_row0);
          else
            regs_codes_per_row<D, BF16, false, false>(rg, P.rows, zero8, q_codes, q_scale,
                                                      P.code_row0);
        } else if (has_q) {
          take(0);
          const float amax = consumer_block_max(regs_absmax<D, BF16>(rg), red, par);
          codes(amax, zero8, q_codes, std::false_type{});
          if (threadIdx.x == 0)
            q_scale[P.scale_idx] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
        }
        // K: exact fixed-point channel sums
        if (has_kv) {
          await_slab(tk);
          take(tk);
          float2 hi[4], fr[4];
          uint32_t absbits;
          regs_fixed_sums<D, BF16>(rg, hi, fr, absbits);
          bool bad;
          if constexpr (BF16) {  // |x| >= 2^16 (bf16 0x4780) or not finite
            bad = (absbits & 0xffffu) >= 0x4780u || (absbits >> 16) >= 0x4780u;
          } else {  // every finite fp16 is below 2^16: only inf / NaN
            bad = false;
#pragma unroll
            for (int e = 0; e < 4; ++e)
              bad |= !(fabsf(hi[e].x) <= 16777216.0f) || !(fabsf(hi[e].y) <= 16777216.0f);
          }
          if (bad) set_status(status, ST_RANGE);
#pragma unroll
          for (int o = T::CPR; o < 32; o <<= 1)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              hi[e].x += __shfl_xor_sync(0xffffffffu, hi[e].x, o);
              hi[e].y += __shfl_xor_sync(0xffffffffu, hi[e].y, o);
              fr[e].x += __shfl_xor_sync(0xffffffffu, fr[e].x, o);
              fr[e].y += __shfl_xor_sync(0xffffffffu, fr[e].y, o);
            }
          if (lane < T::CPR)  // this warp's share of the channel sums
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              red64[warp][8 * c + 2 * e] = (long long)__float2int_rn(hi[e].x) * 1048576LL +
                                           __float2int_rn(fr[e].x * 1048576.0f);
              red64[warp][8 * c + 2 * e + 1] = (long long)__float2int_rn(hi[e].y) * 1048576LL +
                                               __float2int_rn(fr[e].y * 1048576.0f);
            }
          ptx::named_sync<256>();
          if (threadIdx.x < D) {
            long long sum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) sum += red64[i][threadIdx.x];
            atomicAdd(k_sum + chan0 + threadIdx.x, (unsigned long long)sum);
          }
        }
        // V: per-channel max|v| (FP8 P.V only)
        if (FP8 && has_kv) {
          await_slab(tk + 1);
          take(tk + 1);
          uint32_t m2[4] = {0u, 0u, 0u, 0u};
#pragma unroll
          for (int i = 0; i < T::NIT; ++i) {
            m2[0] = In16<BF16>::absmax2(m2[0], rg[i].x);
            m2[1] = In16<BF16>::absmax2(m2[1], rg[i].y);
            m2[2] = In16<BF16>::absmax2(m2[2], rg[i].z);
            m2[3] = In16<BF16>::absmax2(m2[3], rg[i].w);
          }
          float m[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = In16<BF16>::to_float2(m2[e] & 0x7fff7fffu);
            m[2 * e] = f.x;
            m[2 * e + 1] = f.y;
          }
#pragma unroll
          for (int o = T::CPR; o < 32; o <<= 1)
#pragma unroll
            for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], __shfl_xor_sync(0xffffffffu, m[e], o));
          ptx::named_sync<256>();  // red64 is free again
          float* redf = reinterpret_cast<float*>(&red64[0][0]);
          if (lane < T::CPR)
#pragma unroll
            for (int e = 0; e < 8; ++e) redf[warp * D + 8 * c + e] = m[e];
          ptx::named_sync<256>();
          if (threadIdx.x < D) {
            float mx = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) mx = fmaxf(mx, redf[i * D + threadIdx.x]);
            // non-negative floats order like their bit patterns
            atomicMax(v_amax + chan0 + threadIdx.x, __float_as_uint(mx));
          }
        }
        // count this block done once every consumer's atomics are issued
        if (has_kv) {
          ptx::named_sync<256>();
          if (threadIdx.x == 0) ptx::red_release_add_gpu(sync + 1 + u, 1u);
        }
      } else {
        // K: smoothing + per-block quantiser (channel means from the producer)
        {
          float m[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) m[e] = s_side[slot0][8 * c + e];
          take(0);
          if (tok) {  // one delta per token: no block-wide maximum
            if (full_blk)
              regs_codes_per_row<D, BF16, true, true>(rg, P.rows, m, k_codes, k_scale,
                                                      P.code_row0);
            else
              regs_codes_per_row<D, BF16, true, false>(rg, P.rows, m, k_codes, k_scale,
                                                       P.code_row0);
          } else {
          const float a = full_blk ? regs_absmax_sub<D, BF16, true>(rg, P.rows, m)
                                   : regs_absmax_sub<D, BF16, false>(rg, P.rows, m);
          const float amax = consumer_block_max(a, red, par);
          codes(amax, m, k_codes, std::true_type{});
          if (threadIdx.x == 0)
            k_scale[P.scale_idx] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
          }
        }
        // V: FP8 E4M3 codes with a per-channel scale
        if constexpr (FP8) {
          await_slab(1);  // its V scale factors come with the slot
          const float* side = s_side[(cidx + 1) % NS];  // V scale factors
          float2 sv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) sv[e] = make_float2(side[8 * c + 2 * e], side[8 * c + 2 * e + 1]);
          take(1);
          const int r0 = threadIdx.x / T::CPR;
#pragma unroll
          for (int i = 0; i < T::NIT; ++i) {
            const int r = r0 + i * T::RS;
            if (full_blk || r < P.rows) {
              const float2 y0 = __fmul2_rn(In16<BF16>::to_float2(rg[i].x), sv[0]);
              const float2 y1 = __fmul2_rn(In16<BF16>::to_float2(rg[i].y), sv[1]);
              const float2 y2 = __fmul2_rn(In16<BF16>::to_float2(rg[i].z), sv[2]);
              const float2 y3 = __fmul2_rn(In16<BF16>::to_float2(rg[i].w), sv[3]);
              const uint32_t w0 = pack_e4m3x4(y0.x, y0.y, y1.x, y1.y);
              const uint32_t w1 = pack_e4m3x4(y2.x, y2.y, y3.x, y3.y);
              const long long row = P.row0 + (long long)r * P.row_stride;
              *reinterpret_cast<uint2*>(v_codes + row * D + 8 * c) = make_uint2(w0, w1);
            }
          }
        }
      }
      cidx += nt;
    }
    if (threadIdx.x == 0) {
      s_consumed = cidx;
      if (!finished) {  // left the loop on a failed wait
        set_status(status, ST_TIMEOUT);
        s_abort = 1;
      }
    }
  }
  __syncthreads();
  // Teardown: copies issued but not consumed (only after a failed wait) must
  // land before the CTA's shared memory goes away.
  if (warp == 8 && lane == 0) {
    for (int f = s_consumed; f < s_filled; ++f)
      if (!ptx::mbar_wait(&full[f % NS], (f / NS) & 1)) break;
  }
}

// -------------------------------------------------------------- varlen prep --

// One thread: validates cu_seqlens and writes the block and pair prefix sums.
// On any inconsistency all prefixes are written as 0, so every later kernel of
// the call finds no work, and the status word records SAGE_ERR_BAD_SEQLENS.
// sq_off (Q smoothing, may be null): prefix sums of ceil(n_s/128)^2, the
// per-sequence offsets of the mean term in units of 128 floats.
__global__ void varlen_prep_kernel(const int32_t* __restrict__ cu, int batch, int max_seqlen,
                                   int total_tokens, int32_t* blk_off, int32_t* pair_off,
                                   long long* sq_off, uint32_t* status) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  bool ok = __ldg(cu) == 0 && __ldg(cu + batch) == total_tokens;
  int b = 0, p = 0;
  long long q2 = 0;
  for (int s = 0; s < batch && ok; ++s) {
    const int n = __ldg(cu + s + 1) - __ldg(cu + s);
    if (n < 0 || n > max_seqlen) { ok = false; break; }
    blk_off[s] = b;
    pair_off[s] = p;
    if (sq_off) sq_off[s] = q2;
    const int nb = (n + BLK - 1) / BLK;
    b += nb;
    p += (n + 2 * BLK - 1) / (2 * BLK);
    q2 += (long long)nb * nb;
  }
  if (ok) {
    blk_off[batch] = b;
    pair_off[batch] = p;
    if (sq_off) sq_off[batch] = q2;
  } else {
    for (int s = 0; s <= batch; ++s) {
      blk_off[s] = pair_off[s] = 0;
      if (sq_off) sq_off[s] = 0;
    }
    set_status(status, ST_BAD_SEQLENS);
  }
}

}  // namespace

// ------------------------------------------------------------------ launch --

cudaError_t launch_varlen_prep(const int32_t* cu, int batch, int max_seqlen, int total_tokens,
                               int32_t* blk_off, int32_t* pair_off, uint32_t* status,
                               cudaStream_t st, long long* sq_off) {
  varlen_prep_kernel<<<1, 32, 0, st>>>(cu, batch, max_seqlen, total_tokens, blk_off, pair_off,
                                       sq_off, status);
  return cudaGetLastError();
}

template <int D, bool BF16, bool FP8>
static cudaError_t launch_quant_t(const SeqLayout& L, dim3 grid, const void* q, const void* k,
                                  const void* v, int8_t* q_codes, float* q_scale,
                                  int8_t* k_codes, float* k_scale, float* k_mean,
                                  uint8_t* v_codes, float* v_scale, unsigned long long* k_sum,
                                  uint32_t* v_amax, uint32_t* status, unsigned int* sync,
                                  int parts, int tok, cudaStream_t st) {
  const int U = grid.y, NB = grid.x;
  const long long items = ((parts & PART_KV) ? 2LL : 1LL) * U * NB;
  // Dense: one persistent launch in an L2-friendly order (its work counter is
  // 32-bit).  Variable-length batches, and any larger problem: two launches
  // (pass 1 alone for Q only; per-block deltas only).
  if (!L.varlen && items + 4096 < (1LL << 31)) {
    using S = Stream<D>;
    // Per call, on the current device: a function attribute is per device, so
    // a value cached by the first caller would not hold on another device.
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(quant_stream_kernel<D, BF16, FP8>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S::SMEM);
    if (e != cudaSuccess) return e;
    const long long cap = (long long)sms * S::CTAS_PER_SM;
    const int blocks = (int)(items < cap ? items : cap);
    // Items claimed but not yet finished: at most (ring slots + 1) per CTA.
    // A lag of half that many groups of NB, plus one, keeps pass-2 waits rare
    // while the re-read window (about lag heads of Q, K and codes) stays
    // within L2 for long sequences.
    long long lag = ((long long)blocks * (S::NS + 1) + 2LL * NB - 1) / (2LL * NB) + 1;
#ifdef SAGE_QUANT_LAG
    lag = SAGE_QUANT_LAG;
#endif
    if (lag > U) lag = U;
    if (lag < 1) lag = 1;
    quant_stream_kernel<D, BF16, FP8><<<blocks, S::THREADS, S::SMEM, st>>>(
        L, U, (int)lag, parts, tok, q, k, v, q_codes, q_scale, k_codes, k_scale, k_mean, v_codes,
        v_scale, k_sum, v_amax, status, sync);
    return cudaGetLastError();
  }
  quant_pass1_kernel<D, BF16, FP8>
      <<<grid, THREADS, 0, st>>>(L, q, k, v, q_codes, q_scale, k_sum, v_amax, status, parts, tok);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || !(parts & PART_KV)) return e;
  quant_pass2_kernel<D, BF16, FP8><<<grid, THREADS, 0, st>>>(
      L, k, v, k_sum, v_amax, k_codes, k_scale, k_mean, v_codes, v_scale, tok);
  return cudaGetLastError();
}

// Runs both passes.  k_sum / v_amax and (dense) sync[0 .. units] must be zero
// on entry (the caller clears them on the stream).  grid = (blocks per head or
// TBmax, units = B*H or H).  parts: QUANT_Q and/or QUANT_KV (both unless the
// query and key/value heads differ).  per_token: one delta per token (deltas
// indexed like the code rows).
cudaError_t launch_quant(const SeqLayout& L, dim3 grid, int D, bool bf16, bool fp8,
                         const void* q, const void* k, const void* v, int8_t* q_codes,
                         float* q_scale, int8_t* k_codes, float* k_scale, float* k_mean,
                         uint8_t* v_codes, float* v_scale, unsigned long long* k_sum,
                         uint32_t* v_amax, uint32_t* status, unsigned int* sync, int parts,
                         int per_token, cudaStream_t st) {
  static_assert(QUANT_Q == PART_Q && QUANT_KV == PART_KV, "part flags");
#define SAGE_Q(DD, BB, FF)                                                                    \
  return launch_quant_t<DD, BB, FF>(L, grid, q, k, v, q_codes, q_scale, k_codes, k_scale,    \
                                    k_mean, v_codes, v_scale, k_sum, v_amax, status, sync,   \
                                    parts, per_token, st)
  if (D == 64) {
    if (bf16) { if (fp8) SAGE_Q(64, true, true); else SAGE_Q(64, true, false); }
    else { if (fp8) SAGE_Q(64, false, true); else SAGE_Q(64, false, false); }
  } else {
    if (bf16) { if (fp8) SAGE_Q(128, true, true); else SAGE_Q(128, true, false); }
    else { if (fp8) SAGE_Q(128, false, true); else SAGE_Q(128, false, false); }
  }
#undef SAGE_Q
}

// Q smoothing: block means, codes and deltas of the smoothed Q over the
// layout L (dense: grid (blocks, B*H); varlen: grid (TBmax, H)).
cudaError_t launch_quant_q_smooth(const SeqLayout& L, dim3 grid, int D, bool bf16,
                                  const void* q, int8_t* q_codes, float* q_scale, float* q_mean,
                                  uint32_t* status, cudaStream_t st) {
  if (D == 64) {
    if (bf16) quant_q_smooth_kernel<64, true><<<grid, THREADS, 0, st>>>(L, q, q_codes, q_scale, q_mean, status);
    else quant_q_smooth_kernel<64, false><<<grid, THREADS, 0, st>>>(L, q, q_codes, q_scale, q_mean, status);
  } else {
    if (bf16) quant_q_smooth_kernel<128, true><<<grid, THREADS, 0, st>>>(L, q, q_codes, q_scale, q_mean, status);
    else quant_q_smooth_kernel<128, false><<<grid, THREADS, 0, st>>>(L, q, q_codes, q_scale, q_mean, status);
  }
  return cudaGetLastError();
}

// The per-key term of Q smoothing (fp32, kappa applied).  Dense: grid (key
// tiles, B*H), k [B*Hkv, N, D], k_mean [B*Hkv, D], q_mean [B*H, NB, D], the
// term of query blocks [qb0, qb0 + qrows) into bias [B*H][qrows][NB*128].
// Varlen: grid (TBmax, H), k [T, Hkv, D], k_mean [batch, Hkv, D], q_mean
// [H, TBmax, D], bias of sequence s and head h at h*head_stride +
// sq_off[s]*128, [nb_s][nb_s*128] (qb0, qrows unused).
cudaError_t launch_q_smooth_bias(const SeqLayout& L, dim3 grid, int H, int Hkv, int D, bool bf16,
                                 int causal, float kappa, const void* k, const float* k_mean,
                                 const float* q_mean, float* bias, long long head_stride,
                                 const long long* sq_off, int qb0, int qrows, cudaStream_t st) {
#define SAGE_B(DD, BB)                                                                        \
  q_smooth_bias_kernel<DD, BB><<<grid, 128, 0, st>>>(L, H, Hkv, causal, kappa, k, k_mean,    \
                                                     q_mean, bias, head_stride, sq_off, qb0, \
                                                     qrows)
  if (D == 64) {
    if (bf16) SAGE_B(64, true); else SAGE_B(64, false);
  } else {
    if (bf16) SAGE_B(128, true); else SAGE_B(128, false);
  }
#undef SAGE_B
  return cudaGetLastError();
}

}  // namespace sage
