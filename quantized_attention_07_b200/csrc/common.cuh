// Shared device-side definitions of the sm_100a SageAttention kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <cstring>

#include "sage.h"

namespace sage {

constexpr int BLK = SAGE_BLOCK;  // tokens per quantisation block / attention tile

// Bits of the device status word (first word of the workspace).
enum : uint32_t { ST_TIMEOUT = 1u, ST_BAD_SEQLENS = 2u, ST_RANGE = 4u };

// Description of where the tokens of one (sequence, head) live.
//   dense : sequence = b, rows [bh*N, bh*N + N) of a [B*H*N, D] tensor.
//   varlen: sequence s, token t at row (cu[s] + t)*H + h of a [T*H, D] tensor.
struct SeqLayout {
  int varlen;
  int N;                   // dense length
  int H;
  const int32_t* cu;       // varlen: [batch+1]
  const int32_t* blk_off;  // varlen: [batch+1], prefix of ceil(n_s/128)
  int batch;
  int TBmax;               // varlen: row blocks reserved per head in code arrays
};

// Work-layout metadata the varlen preparation kernel writes into the workspace.
struct VarlenMeta {
  int32_t* blk_off;    // [batch+1]
  int32_t* pair_off;   // [batch+1], prefix of ceil(n_s/256)
};

__device__ __forceinline__ void set_status(uint32_t* st, uint32_t bits) { atomicOr(st, bits); }

// Tensors a quantisation launch covers (launch_quant's `parts`).
constexpr int QUANT_Q = 1;
constexpr int QUANT_KV = 2;

// Binary search: the s with off[s] <= x < off[s+1] (off non-decreasing, off[0] = 0).
__device__ __forceinline__ int find_segment(const int32_t* off, int n, int x) {
  int lo = 0, hi = n;  // answer in [lo, hi)
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (__ldg(off + mid) <= x) lo = mid; else hi = mid;
  }
  return lo;
}

template <bool BF16> struct In16;
template <> struct In16<false> {
  using T = __half;
  using T2 = __half2;
  // Lane-wise maximum of two packed pairs (a NaN lane yields the other value).
  __device__ static uint32_t max2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
  }
  // Lane-wise max(|a|, |b|); the sign bit of each lane is garbage (mask it).
  __device__ static uint32_t absmax2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
  }
  // Packed pair (element 0 in the low half) -> two exact floats.
  __device__ static float2 to_float2(uint32_t u) {
    __half2 h;
    memcpy(&h, &u, 4);
    return __half22float2(h);
  }
  __device__ static uint32_t pack(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    uint32_t u;
    memcpy(&u, &h, 4);
    return u;
  }
};
template <> struct In16<true> {
  using T = __nv_bfloat16;
  using T2 = __nv_bfloat162;
  __device__ static uint32_t max2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
  }
  __device__ static uint32_t absmax2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
  }
  // bf16 is the high half of an fp32 bit pattern.
  __device__ static float2 to_float2(uint32_t u) {
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
  }
  __device__ static uint32_t pack(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    uint32_t u;
    memcpy(&u, &h, 4);
    return u;
  }
};

// Four floats -> four E4M3 bytes (round to nearest even, saturate to +-448),
// element 0 in the lowest byte.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return (uint32_t)lo | ((uint32_t)hi << 16);
}

}  // namespace sage
