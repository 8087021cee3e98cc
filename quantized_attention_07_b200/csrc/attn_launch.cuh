// Host/device interface of the fused attention kernel.
#pragma once

#include "common.cuh"

namespace sage {

struct AttnParams {
  int H, N, BH;          // dense: N, BH = B*H (query heads)
  int Hkv;               // dense: key/value heads (H is a multiple; query head h reads h / (H/Hkv))
  int NB;                // dense: key blocks per head = ceil(N/128)
  int NPAIR;             // dense: query tile pairs per head in this launch (all: ceil(N/256))
  int pair0;             // dense: first query tile pair of the launch
  int bias_nb;           // dense per_token 2: query blocks per head in q_bias, from block 2*pair0
  int causal;
  int per_token;         // 1: one delta per token ([BH][NP] / [B*Hkv][NP]), not per block;
                         // 2: per block, Q smoothed (q_bias holds the mean term)
  const float* q_bias;   // per_token 2: dense [BH][bias_nb][NB*128] fp32, kappa applied;
                         // varlen: sequence s, head h at h*bias_head_stride + sq_off[s]*128
  const long long* sq_off;        // varlen per_token 2: [batch+1] prefix of ceil(n_s/128)^2
  long long bias_head_stride;     // varlen per_token 2: floats per query head
  float kappa;           // fp32(sm_scale * log2 e)
  const float* q_scale;  // dense [BH][NB]; varlen [H][TBmax]
  const float* k_scale;
  const float* v_scale;  // FP8: dense [BH][D]; varlen [batch][H][D]
  void* out;
  int out_dt;
  // varlen
  int varlen;
  const int32_t* cu;
  const int32_t* blk_off;
  const int32_t* pair_off;
  int batch;
  int TBmax;
  int PM;                // varlen: work items per head (query tile pairs of the longest layout)
  int items;             // work items of the launch: dense BH*NPAIR, varlen H*PM
  unsigned int* sched;   // [2] in the workspace header: next item, CTAs finished (zero between launches)
  uint32_t* status;
  // diagnostic: when set (dense, per-block deltas, fp16 V or FP8 P.V only),
  // every int32 S sub-tile the kernel computes is also stored here, row-major
  // [BH][s_dump_ld][s_dump_ld] (query row, key), before its dequantisation
  int32_t* s_dump;
  long long s_dump_ld;   // NB * 128
  // bounded waits: cycles before a wait gives up (0: SAGE_WAIT_LIMIT_CYCLES)
  long long wait_limit;
  // self-test of the timeout path: s > 0 leaves the K tile of every CTA's
  // s-th pipeline stage unloaded, so that stage's barrier never completes
  int fault_skip_k;
};

struct AttnLaunch {
  AttnParams p;
  int D, pv8, bf16v;
  const int8_t* q_codes;
  const int8_t* k_codes;
  const void* v;         // 16-bit V (FP16 mode) or E4M3 codes (FP8 mode)
  int code_rows;         // rows per z-slice of the code arrays (NP or TBmax*128)
  int code_z;            // Q^ z-slices: BH (dense) or H (varlen)
  int code_z_kv;         // K^ (and dense V) z-slices: B*Hkv (dense) or H (varlen)
  int T;                 // varlen tokens
};

// Persistent launch: min(p.items, SM count) CTAs, each taking work items
// from the counter p.sched until none is left.
cudaError_t launch_attn(const AttnLaunch& L, cudaStream_t st);

}  // namespace sage
