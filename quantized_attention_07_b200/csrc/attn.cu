// Fused SageAttention forward kernel for sm_100a.
//
// A persistent kernel, one CTA per SM.  A work item is a pair of 128-row
// query tiles of one (sequence, head); the CTA takes items from a counter in
// the workspace and streams each item's keys and values through shared
// memory in 128-key stages; the online softmax works on 64-key sub-tiles.
//
//   control warpgroup (warp 0 of it: TMA producer; warps 1 and 2: MMA
//                issue for query tile 0 / 1, one elected lane each; warp 1
//                also owns TMEM):
//                  S_t[b]  = Q^_t K^_i^T     tcgen05.mma kind::i8 -> int32 TMEM
//                  O_t    += P_t[b] V_i      kind::f16 (16-bit P.V), or
//                  Part_t  = P^_t[b] V^_i    kind::f8f6f4 (FP8 P.V),
//                P read from TMEM (written over S), V from shared memory.
//   softmax warpgroups 0 and 1 (one per query tile, one thread per row):
//                read S from TMEM, dequantise with deltaQ*deltaK*sm_scale*log2 e,
//                mask, online softmax in base 2, write P (fp16/bf16 or e4m3)
//                back over S; 16-bit P.V: rescale O in TMEM when the maximum
//                in use moves; FP8: fold the previous 128-key block's partial
//                into an fp32 register accumulator (two-level accumulation).
//
// Each query tile owns two (D = 128) or three (D = 64) 64-column S buffers,
// so QK^T of the next sub-tiles runs on the tensor core while the softmax
// works on sub-tile i, and the two query tiles keep both softmax warpgroups
// busy.  With FP8 P.V or bf16 P the maximum
// used for p is the plain running maximum over whole 128-key blocks: the first
// half of a block waits for the second half's S as well and takes the maximum
// over both.  With fp16 P it is taken per 64-key sub-tile and moves only when
// a row's sub-tile maximum exceeds it by more than 8, so O rescales are rare.
//
// TMEM columns (512): NBUF S buffers of 64 columns per tile, S_t[b] at
// [64(NBUF t + b), +64), then O_0 at 128 NBUF and O_1 D columns later.  D = 128
// keeps two buffers (O takes 256 columns); D = 64 has room for three, so
// QK^T runs three sub-tiles ahead of the softmax instead of two (with FP8
// P.V the first half of a 128-key block then finds the second half's S
// computed before P.V of the previous block's second half completes).
//
// Method steps (SageAttention pages): INT8 QK^T with the per-block deltas
// ("SageAttention -- brand new attention", quantisation intro step 3 and
// "SageAttention" bullets 1-2), online softmax ("Attention机制优化：从
// FlashAttention到SageAttention的工程实践", section 3.1), P.V in 16 bits
// ("SageAttention" bullet 3) or FP8 with two-level accumulation
// ("SageAttention v1/v2/v2++/v3 overview", SageAttention 2 bullets 1 and 3).
// The template parameter GR picks the Q/K delta granularity (same overview,
// SageAttention v1 item (1)): 0 per block, 1 per token, 2 per block with Q
// smoothing (SageAttention 2 bullet 2), whose per-key mean term joins the
// scaled score before the row maximum.
//
// Every mbarrier wait is bounded.  On a timeout the waiting role records
// ST_TIMEOUT, raises a CTA-wide abort flag that the other roles' waits also
// watch, and everyone falls through to the teardown, which waits (bounded) for
// the CTA's own TMA loads and MMAs and always frees TMEM.
#include <algorithm>

#include "attn_launch.cuh"
#include "ptx.cuh"

namespace sage {

namespace {

constexpr int SUB = 64;  // keys per softmax sub-tile
// fp32(log2 448): FP8 P.V forms p = 448 * 2^(t - m) as 2^(arg + log2 448)
constexpr float kLog2_448 = 8.807354927062988f;

template <int D, bool PV8, int GR>
struct Cfg {
  // warpgroups: 2 softmax, 1 control
  static constexpr int WGS = 3;
  static constexpr int THREADS = WGS * 128;
  static constexpr int WG_CTRL = 2;
  // register split, summing to the launch allocation (384 threads at 168)
  static constexpr int REG_SOFTMAX = 224;
  static constexpr int REG_CTRL = 56;
  static_assert(256 * REG_SOFTMAX + 128 * REG_CTRL <= 384 * 168,
                "register split exceeds the launch allocation");
  // The maximum used for p: with FP8 P.V or bf16 P (a short format whose
  // rounding of p must not depend on where a block is split) it is the plain
  // running maximum over whole 128-key blocks (both 64-key halves of a block
  // share it); with fp16 P it is taken per 64-key sub-tile and moves only when
  // the sub-tile's maximum exceeds it by more than 8 (base 2: p < 2^8, exact
  // in fp16's range), which makes the rescale of O rare.
  static constexpr bool block_max(bool bf16v) { return PV8 || bf16v; }
  static constexpr float tau(bool bf16v) { return block_max(bf16v) ? 0.0f : 8.0f; }

  // S buffers per tile: 2 x NBUF x 64 columns of S and 2 x D of O fit 512.
  // Three at D = 64 (measured +1.0 % on the FP8 video shape, +1.5 % with
  // per-token deltas); with Q smoothing the longer-lived buffer indices cost
  // registers and it measured 0.3 % slower, so two.
  static constexpr int NBUF = (D == 64 && GR != 2) ? 3 : 2;
  static constexpr uint32_t TO = 2 * NBUF * SUB;        // first O column
  static_assert(TO + 2 * D <= 512, "TMEM columns");
  // S buffer of a tile's I-th sub-tile, and the parity of its barrier phase
  // (I >= 0; unsigned, so NBUF = 2 is a mask and a shift)
  static __device__ __forceinline__ int sbuf(int I) { return (int)((unsigned)I % NBUF); }
  static __device__ __forceinline__ uint32_t sphase(int I) { return ((unsigned)I / NBUF) & 1u; }
  static constexpr int QT = BLK * D;                    // bytes of one int8 Q^/K^ tile
  static constexpr int VT = BLK * D * (PV8 ? 1 : 2);    // bytes of one V tile
  // per stage, on the K barrier: the 128 per-token K deltas (GR 1), or the
  // Q-smoothing term of both query tiles for the stage's keys (GR 2)
  static constexpr int KS = GR == 1 ? BLK * 4 : GR == 2 ? 2 * BLK * 4 : 0;
  // barriers (1 KiB), then with FP8 P.V each tile's V scales ([2][D] fp32)
  static constexpr int AUX = 1024 + (PV8 ? 2 * D * 4 : 0);
  static constexpr int SMEM_BUDGET = 227 * 1024 - 1024 - AUX;
  static constexpr int NS_RAW = (SMEM_BUDGET - 2 * QT) / (QT + VT + KS);
  static constexpr int NS = NS_RAW > 8 ? 8 : NS_RAW;    // pipeline stages (128 keys each)
  static constexpr int SMEM = 1024 + 2 * QT + NS * (QT + VT + KS) + AUX;
  // int8 code tiles: rows of D bytes
  static constexpr uint32_t QK_SWZ = (D == 128) ? 2u : 4u;  // 128B : 64B swizzle
  static constexpr uint32_t QK_SBO = 8 * D;                 // 8 rows
  static constexpr uint32_t K_SUB_BYTES = SUB * D;          // 64 keys of K^
  // V tiles, MN-major (D contiguous): 16-bit -> 64-element (128 B) atoms;
  // 8-bit -> one atom of D bytes.
  static constexpr int V_ROW_BYTES = PV8 ? D : 128;
  static constexpr uint32_t V_SWZ = (V_ROW_BYTES == 128) ? 2u : 4u;
  static constexpr uint32_t V_SBO = 8 * V_ROW_BYTES;         // 8 keys
  static constexpr uint32_t V_LBO = BLK * 128;               // next 64-column atom (16-bit)
  static constexpr uint32_t V_SUB_BYTES = (SUB / 8) * V_SBO; // 64 keys
  static constexpr int PV_KSTEP = PV8 ? 32 : 16;             // keys per MMA
  static constexpr uint32_t V_KSTEP_BYTES = (PV_KSTEP / 8) * V_SBO;
  static constexpr int PV_STEPS = SUB / PV_KSTEP;
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static_assert(NS >= 2, "need at least two stages");
  // QK^T of sub-tile i + NBUF reads stage (i + NBUF)/2 before stage i/2 is
  // released: NBUF/2 + 2 stages resident at once
  static_assert(NS >= NBUF / 2 + 2, "stages for the S lookahead");
};

struct Bars {
  uint64_t q_full, done[2];
  uint64_t s_full[2][3];   // [tile][S buffer]: QK^T of a sub-tile landed
  uint64_t p_full[2][3];   // P of a sub-tile written, O rescaled (128 softmax threads)
  uint64_t o_full[2];      // P.V of a sub-tile completed
  uint64_t vs_full[2];     // FP8: a tile's V scales staged for its epilogue (4 softmax warps)
  uint64_t o_done[2];      // the last P.V of a query tile of an item completed
  uint64_t q_empty;        // both MMA warps' last QK^T of the item completed (2 commits)
  uint64_t item_full[2];   // work-item ring: index published by the producer
  uint64_t item_empty[2];  // ... and read by both MMA warps and all 256 softmax threads
  int item[2];
  int sm_loop[8][2];       // per softmax warp: items taken, items with keys (see softmax_wg)
  uint64_t k_full[8], v_full[8], kv_empty[8];
  uint32_t tmem_base;
  volatile int abort;
  long long wait_limit;    // cycles before a bounded wait gives up
};

// Warp-uniform bounded wait: true when the phase completed, false (and the
// abort flag raised) on timeout or when another role aborted.
__device__ __forceinline__ bool wait_bar(Bars* B, uint64_t* bar, uint32_t parity,
                                         uint32_t* status, bool warp_uniform) {
  bool ok = ptx::mbar_try_wait(bar, parity);
  if (!ok) {
    const long long t0 = clock64();
    while (true) {
      if (ptx::mbar_try_wait(bar, parity)) { ok = true; break; }
      if (B->abort) break;
      if (clock64() - t0 > B->wait_limit) {
        set_status(status, ST_TIMEOUT);
        B->abort = 1;
        break;
      }
    }
  }
  if (warp_uniform) ok = __all_sync(0xffffffffu, ok);
  return ok;
}

// Work item of this CTA.
struct Work {
  int valid;
  int n;                 // sequence length (queries = keys)
  int pair;              // query tile pair index within the sequence
  int code_z;            // z coordinate of this query head in the Q^ code map
  int k_z;               // z coordinate of its key/value head in the K^ code map
  int q_y0;              // y coordinate of query tile 0 in the code map
  int k_y0;              // y coordinate of key tile 0 in the code map
  int v_y0, v_z0;        // TMA coordinates of V tile 0 (x = column)
  int v_tok_on_z;        // tokens advance along z (varlen) instead of y (dense)
  long long qs_idx0;     // q_scale index of query tile 0
  long long ks_idx0;     // k_scale index of key block 0
  long long out_row0;    // row (in units of D elements) of token 0 of the output
  long long out_stride;  // rows between consecutive tokens
  long long vs_idx;      // v_scale row index (FP8)
  int nsub0, nsub1;      // 64-key sub-tiles for query tile 0 / 1 (0 = tile absent)
  int nkv;               // 128-key stages to stream
  long long bias_row0;   // Q smoothing: float index of query tile 0's mean-term row
  long long bias_ld;     // floats between the rows of consecutive query blocks
};

// Work item idx of the launch (0 <= idx < p.items).  Dense: idx -> (head,
// query tile pair); varlen: idx = h * PM + item, item over the sequences'
// pairs (items past the last pair are empty).
__device__ __forceinline__ Work decode_work(const AttnParams& p, int idx) {
  Work w{};
  int pair, n;
  if (!p.varlen) {
    int bh;
    if (p.causal) {  // heaviest pairs first
      pair = p.pair0 + p.NPAIR - 1 - idx / p.BH;
      bh = idx % p.BH;
    } else {         // head-major: a head's K^/V stay hot in L2
      bh = idx / p.NPAIR;
      pair = p.pair0 + idx % p.NPAIR;
    }
    n = p.N;
    // grouped-query attention: query head h of batch b reads key/value head
    // h / (H / Hkv) of the same batch (the repeat_kv grouping)
    const int b = bh / p.H, hq = bh - b * p.H;
    const int bkv = b * p.Hkv + hq / (p.H / p.Hkv);
    w.code_z = bh;
    w.k_z = bkv;
    w.q_y0 = pair * 2 * BLK;
    w.k_y0 = 0;
    w.v_y0 = 0;
    w.v_z0 = bkv;
    w.v_tok_on_z = 0;
    w.qs_idx0 = (long long)bh * p.NB + 2 * pair;
    w.ks_idx0 = (long long)bkv * p.NB;
    w.out_row0 = (long long)bh * p.N;
    w.out_stride = 1;
    w.vs_idx = bkv;
    w.bias_ld = (long long)p.NB * BLK;
    w.bias_row0 = ((long long)bh * p.bias_nb + 2 * (pair - p.pair0)) * w.bias_ld;
  } else {
    const int h = idx / p.PM;
    const int item = idx - h * p.PM;
    const int total = __ldg(p.pair_off + p.batch);
    if (item >= total) { w.valid = 0; return w; }
    const int s = find_segment(p.pair_off, p.batch + 1, item);
    const int tok0 = __ldg(p.cu + s);
    n = __ldg(p.cu + s + 1) - tok0;
    const int npairs = __ldg(p.pair_off + s + 1) - __ldg(p.pair_off + s);
    pair = npairs - 1 - (item - __ldg(p.pair_off + s));  // diagonal-heavy pairs first
    const int blk0 = __ldg(p.blk_off + s);
    const int hk = h / (p.H / p.Hkv);  // its key/value head (grouped-query)
    w.code_z = h;
    w.k_z = hk;
    w.q_y0 = (blk0 + 2 * pair) * BLK;
    w.k_y0 = blk0 * BLK;
    w.v_y0 = hk;
    w.v_z0 = tok0;
    w.v_tok_on_z = 1;
    w.qs_idx0 = (long long)h * p.TBmax + blk0 + 2 * pair;
    w.ks_idx0 = (long long)hk * p.TBmax + blk0;
    w.out_row0 = (long long)tok0 * p.H + h;
    w.out_stride = p.H;
    w.vs_idx = (long long)s * p.Hkv + hk;
    if (p.per_token == 2) {  // the sequence's own [nb_s][nb_s*128] block of the term
      w.bias_ld = (long long)((n + BLK - 1) / BLK) * BLK;
      w.bias_row0 = (long long)h * p.bias_head_stride + __ldg(p.sq_off + s) * BLK +
                    2LL * pair * w.bias_ld;
    }
  }
  w.valid = 1;
  w.n = n;
  w.pair = pair;
  const int ns = (n + SUB - 1) / SUB;
  int q0 = 2 * pair, q1 = 2 * pair + 1;
  w.nsub0 = (q0 * BLK >= n) ? 0 : (p.causal ? min(ns, 2 * q0 + 2) : ns);
  w.nsub1 = (q1 * BLK >= n) ? 0 : (p.causal ? min(ns, 2 * q1 + 2) : ns);
  w.nkv = (max(w.nsub0, w.nsub1) + 1) / 2;
  return w;
}

// ------------------------------------------------------- work scheduling --
//
// Work items are handed out dynamically: the producer warp takes the next
// index from a global counter (p.sched[0]) and publishes it to the CTA's other
// roles through a two-slot ring in shared memory; -1 ends the loop.  The
// counter and the count of finished CTAs (p.sched[1]) start at zero; the last
// CTA to finish sets both back to zero for the next launch.

constexpr int ITEM_READERS = 2 + 256;  // item_empty arrivals: 2 MMA warps + 256 softmax threads

// Index of the r-th item taken by this CTA's consumers (false on timeout or
// abort).  The whole warp calls it; `all_lanes` arrive individually
// (softmax) or lane 0 for the warp (MMA warps).
__device__ __forceinline__ bool take_item(Bars* B, int r, uint32_t* status, bool all_lanes,
                                          int& idx) {
  const int s = r & 1;
  if (!wait_bar(B, &B->item_full[s], (r >> 1) & 1, status, true)) return false;
  idx = *reinterpret_cast<volatile int*>(&B->item[s]);
  if (all_lanes) {
    ptx::mbar_arrive(&B->item_empty[s]);
  } else {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(&B->item_empty[s]);
  }
  return true;
}

// --------------------------------------------------------------- producer --

template <int D, bool PV8, int GR>
__device__ void producer(const CUtensorMap* tm_q, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                         const AttnParams& p, Bars* B, uint8_t* sQ, uint8_t* sK, uint8_t* sV,
                         float* sKs) {
  using C = Cfg<D, PV8, GR>;
  [[maybe_unused]] constexpr bool TOK = GR == 1, SMQ = GR == 2;
  // The whole warp runs this loop (uniform control flow); one elected lane
  // issues each TMA instruction.  Stages form one ring across the CTA's work
  // items: G counts the stages loaded so far.
  if (ptx::elect_one()) {
    ptx::prefetch_tmap(tm_q);
    ptx::prefetch_tmap(tm_k);
    ptx::prefetch_tmap(tm_v);
  }
  __syncwarp();
  const int lane = threadIdx.x & 31;
  auto fetch = [&]() -> int {
    int v = 0;
    if (lane == 0) v = (int)atomicAdd(p.sched, 1u);
    v = __shfl_sync(0xffffffffu, v, 0);
    return v < p.items ? v : -1;
  };
  int G = 0, n = 0;
  bool ok = true;
  int next = fetch();
  for (int r = 0; ok; ++r) {
    // publish the r-th item (slot r & 1, free once item r-2 was read)
    const int idx = next;
    const int slot = r & 1;
    if (r >= 2 && !wait_bar(B, &B->item_empty[slot], ((r >> 1) - 1) & 1, p.status, true)) break;
    if (lane == 0) {
      B->item[slot] = idx;
      ptx::mbar_arrive(&B->item_full[slot]);
    }
    __syncwarp();
    if (idx < 0) break;
    const Work w = decode_work(p, idx);
    if (!w.valid) {
      next = fetch();
      continue;
    }
    // the previous item's QK^T must have read both Q^ tiles
    if (n > 0 && !wait_bar(B, &B->q_empty, (n - 1) & 1, p.status, true)) break;
    if (ptx::elect_one()) {
      // both Q^ tiles (an absent second tile reads zero-filled or padding rows)
      ptx::mbar_arrive_expect_tx(&B->q_full, 2 * C::QT);
      ptx::tma_load_3d(sQ, tm_q, &B->q_full, 0, w.q_y0, w.code_z);
      ptx::tma_load_3d(sQ + C::QT, tm_q, &B->q_full, 0, w.q_y0 + BLK, w.code_z);
    }
    __syncwarp();
    ++n;
    for (int j = 0; j < w.nkv; ++j, ++G) {
      const int s = G % C::NS;
      if (G >= C::NS && !wait_bar(B, &B->kv_empty[s], ((G / C::NS) - 1) & 1, p.status, true)) {
        ok = false;
        break;
      }
      if (ptx::elect_one()) {
        if constexpr (SMQ) {
          // Q smoothing: each present query tile's mean term for the stage's
          // 128 keys, on the K barrier (a tile without keys has no bias row)
          const int nt_q = w.nsub1 > 0 ? 2 : 1;
          ptx::mbar_arrive_expect_tx(&B->k_full[s], C::QT + nt_q * BLK * 4);
          for (int tq = 0; tq < nt_q; ++tq)
            ptx::bulk_load_plain(sKs + (s * 2 + tq) * BLK,
                                 p.q_bias + w.bias_row0 + tq * w.bias_ld + (long long)j * BLK,
                                 BLK * 4, &B->k_full[s]);
        } else {
          ptx::mbar_arrive_expect_tx(&B->k_full[s], C::QT + C::KS);
        }
        // (the timeout self-test leaves one K tile unloaded: its barrier then
        // waits for bytes that never come)
        if (p.fault_skip_k == 0 || G != p.fault_skip_k - 1)
          ptx::tma_load_3d(sK + s * C::QT, tm_k, &B->k_full[s], 0, w.k_y0 + j * BLK, w.k_z);
        if constexpr (TOK)  // the stage's 128 per-token K deltas, on the same barrier
          ptx::bulk_load_plain(sKs + s * BLK, p.k_scale + (w.ks_idx0 + j) * BLK, C::KS,
                               &B->k_full[s]);
        ptx::mbar_arrive_expect_tx(&B->v_full[s], C::VT);
        uint8_t* dst = sV + s * C::VT;
        const int y = w.v_tok_on_z ? w.v_y0 : w.v_y0 + j * BLK;
        const int z = w.v_tok_on_z ? w.v_z0 + j * BLK : w.v_z0;
        ptx::tma_load_3d(dst, tm_v, &B->v_full[s], 0, y, z);
        if (!PV8 && D == 128)  // 16-bit V rows are 256 B: second 64-column box
          ptx::tma_load_3d(dst + BLK * 128, tm_v, &B->v_full[s], 64, y, z);
      }
      __syncwarp();
    }
    // The next item is taken only now, when this one's last loads are issued
    // (a few stages before its MMAs end): taking it earlier would bind it to
    // this CTA while another CTA may become free first.
    next = fetch();
  }
  // Teardown: the most recent load of every stage and of Q must have landed
  // before this CTA may exit (the earlier ones were consumed already).
  for (int jj = max(0, G - C::NS); jj < G; ++jj) {
    const int s = jj % C::NS;
    const uint32_t ph = (jj / C::NS) & 1;
    ptx::mbar_wait(&B->k_full[s], ph, B->wait_limit);
    ptx::mbar_wait(&B->v_full[s], ph, B->wait_limit);
  }
  if (n > 0) ptx::mbar_wait(&B->q_full, (n - 1) & 1, B->wait_limit);
}

// ------------------------------------------------------------ MMA issuer --

// One warp per query tile issues that tile's MMAs (the whole warp runs the
// loop; one elected lane issues).  Per 64-key sub-tile i:
//   wait P_t(i) -> O_t (+)= P_t(i) V_i  ->  S_t(i+NBUF) = Q^_t K^_{i+NBUF}^T
// Issue order per thread is execution order, so S_t(i+NBUF) never overwrites
// P_t(i) before P.V has read it.  A 128-key stage is released to the producer
// when both tiles' warps have committed it (kv_empty counts two arrivals).
template <int D, bool PV8, bool BF16V, int GR>
__device__ void mma_issuer(const AttnParams& p, Bars* B, uint32_t tmem, const uint8_t* sQ,
                           const uint8_t* sK, const uint8_t* sV, int t) {
  using C = Cfg<D, PV8, GR>;
  [[maybe_unused]] constexpr bool TOK = GR == 1, SMQ = GR == 2;
  constexpr uint32_t IDESC_QK = ptx::instr_desc(2, 1, 1, 0, 0, 128, SUB);
  constexpr uint32_t IDESC_PV =
      PV8 ? ptx::instr_desc(1, 0, 0, 0, 1, 128, D)
          : ptx::instr_desc(1, BF16V ? 1 : 0, BF16V ? 1 : 0, 0, 1, 128, D);
  uint32_t* status = p.status;
  const uint32_t qa = ptx::smem_u32(sQ + t * C::QT);
  const uint32_t tO = tmem + C::TO + D * t;
  // Counts over the CTA's work items: sub-tiles of this tile (I0: S buffer
  // and barrier phases), stages of the ring (G0), items (n: q_full phase).
  int I0 = 0, G0 = 0, n = 0;
  int nt = 0, released = 0;                   // this item: sub-tiles, stages committed
  int k_ready = -1, v_ready = -1;             // highest ring stage known to be loaded

  auto need_k = [&](int g) -> bool {
    if (k_ready >= g) return true;
    if (!wait_bar(B, &B->k_full[g % C::NS], (g / C::NS) & 1, status, true)) return false;
    k_ready = g;
    return true;
  };
  auto need_v = [&](int g) -> bool {
    if (v_ready >= g) return true;
    if (!wait_bar(B, &B->v_full[g % C::NS], (g / C::NS) & 1, status, true)) return false;
    v_ready = g;
    return true;
  };
  auto issue_qk = [&](int i) {  // i: sub-tile of the item
    const int I = I0 + i, g = G0 + i / 2;
    const uint32_t kb = ptx::smem_u32(sK + (g % C::NS) * C::QT + (i & 1) * C::K_SUB_BYTES);
    const uint32_t dst = tmem + C::NBUF * SUB * t + SUB * C::sbuf(I);
    if (ptx::elect_one()) {
      const uint64_t a0 = ptx::smem_desc(qa, 16, C::QK_SBO, C::QK_SWZ);
      const uint64_t b0 = ptx::smem_desc(kb, 16, C::QK_SBO, C::QK_SWZ);
#pragma unroll
      for (int kk = 0; kk < D / 32; ++kk)  // +32 bytes along K per step: +2 in the address field
        ptx::mma_i8_ss(dst, a0 + 2 * kk, b0 + 2 * kk, IDESC_QK, kk > 0 ? 1u : 0u);
      ptx::mma_commit(&B->s_full[t][C::sbuf(I)]);
      // after the item's last QK^T the Q^ tiles may be reloaded
      if (i == nt - 1) ptx::mma_commit(&B->q_empty);
    }
    __syncwarp();
  };
  auto issue_pv = [&](int i) {
    const int I = I0 + i, g = G0 + i / 2;
    const uint32_t vb = ptx::smem_u32(sV + (g % C::NS) * C::VT + (i & 1) * C::V_SUB_BYTES);
    const uint32_t tP = tmem + C::NBUF * SUB * t + SUB * C::sbuf(I);
    // an item's first P.V starts O; FP8: each block's first half starts a
    // fresh partial, its second half accumulates into it
    const uint32_t acc0 = PV8 ? ((i & 1) ? 1u : 0u) : (i > 0 ? 1u : 0u);
    if (ptx::elect_one()) {
      const uint64_t b0 = ptx::smem_desc(vb, C::V_LBO, C::V_SBO, C::V_SWZ);
#pragma unroll
      for (int kk = 0; kk < C::PV_STEPS; ++kk) {
        const uint64_t bd = b0 + (uint64_t)((kk * C::V_KSTEP_BYTES) >> 4);
        const uint32_t acc = kk > 0 ? 1u : acc0;
        if constexpr (PV8) ptx::mma_f8_ts(tO, tP + 8 * kk, bd, IDESC_PV, acc);
        else ptx::mma_f16_ts(tO, tP + 8 * kk, bd, IDESC_PV, acc);
      }
      ptx::mma_commit(&B->o_full[t]);
      if (i == nt - 1) ptx::mma_commit(&B->o_done[t]);
    }
    __syncwarp();
  };
  // Commit the item's next stage (this warp is done with it).  A stage this
  // tile never reads is first waited for like a used one: then every load
  // this warp releases was seen complete by it, which keeps the parity of
  // the slot's next k_full / v_full phase unambiguous for this warp in a
  // later item, and the producer's refill of the slot (issued only after the
  // previous release) makes the arrival count toward this stage's phase.
  auto release = [&](bool used) -> bool {
    const int g = G0 + released;
    if (!used && !(need_k(g) && need_v(g))) return false;
    if (ptx::elect_one()) ptx::mma_commit(&B->kv_empty[g % C::NS]);
    __syncwarp();
    ++released;
    return true;
  };

  bool ok = true;
  for (int r = 0; ok; ++r) {
    int idx;
    if (!take_item(B, r, status, false, idx) || idx < 0) break;
    const Work w = decode_work(p, idx);
    if (!w.valid) continue;
    nt = t == 0 ? w.nsub0 : w.nsub1;
    released = 0;
    ok = wait_bar(B, &B->q_full, n & 1, status, true);
    if (!ok) break;
    ptx::tc_fence_after();
    if (nt == 0) {  // no key for this tile: its share of q_empty right away
      if (ptx::elect_one()) ptx::mma_commit(&B->q_empty);
      __syncwarp();
    }
    for (int i = 0; ok && i < C::NBUF && i < nt; ++i) {
      ok = need_k(G0 + i / 2);
      if (!ok) break;
      ptx::tc_fence_after();
      issue_qk(i);
    }
    for (int i = 0; ok && i < nt; ++i) {
      ok = need_v(G0 + i / 2) &&
           wait_bar(B, &B->p_full[t][C::sbuf(I0 + i)], C::sphase(I0 + i), status, true);
      if (!ok) break;
      ptx::tc_fence_after();
      issue_pv(i);
      if (i + C::NBUF < nt) {
        ok = need_k(G0 + (i + C::NBUF) / 2);
        if (!ok) break;
        ptx::tc_fence_after();
        issue_qk(i + C::NBUF);
      }
      if ((i & 1) || i == nt - 1) ok = release(true);
    }
    // stages loaded for the other tile only
    while (ok && released < w.nkv && released >= (nt + 1) / 2) ok = release(false);
    if (!ok) break;
    I0 += nt;
    G0 += w.nkv;
    ++n;
  }
  // Drain: every MMA this warp issued completes before TMEM is released.
  if (ptx::elect_one()) ptx::mma_commit(&B->done[t]);
  __syncwarp();
  ptx::mbar_wait(&B->done[t], 0, B->wait_limit);
}

// --------------------------------------------------------------- softmax --

// int32 -> fp32, exact here (|S| <= 127^2 * 128 < 2^24).  On sm_100a the
// conversion instruction measured cheaper than adding and subtracting a
// 1.5 * 2^23 magic constant.
__device__ __forceinline__ float2 s32x2_to_f32x2(uint32_t a, uint32_t b) {
  return make_float2((float)(int)a, (float)(int)b);
}

__device__ __forceinline__ int imax3(int a, int b, int c) { return __vimax3_s32(a, b, c); }

// Row maximum of NC columns of S (all valid).
template <int NC>
__device__ __forceinline__ int row_max(const uint32_t* v, int acc) {
  int m0 = acc, m1 = INT_MIN, m2 = INT_MIN, m3 = INT_MIN;
#pragma unroll
  for (int i = 0; i < NC; i += 8) {
    m0 = imax3(m0, (int)v[i], (int)v[i + 1]);
    m1 = imax3(m1, (int)v[i + 2], (int)v[i + 3]);
    m2 = imax3(m2, (int)v[i + 4], (int)v[i + 5]);
    m3 = imax3(m3, (int)v[i + 6], (int)v[i + 7]);
  }
  return imax3(m0, imax3(m1, m2, m3), INT_MIN);
}

// Row maximum over the columns whose key index first_key + col is below `limit`.
template <int NC>
__device__ __forceinline__ int row_max_masked(const uint32_t* v, int acc, int first_key,
                                              int limit) {
#pragma unroll
  for (int i = 0; i < NC; ++i)
    if (first_key + i < limit) acc = max(acc, (int)v[i]);
  return acc;
}

// Per-token deltas: y_j = fp32(S_j * deltaK_j) in place (as fp32 bits) for NC
// columns, returning max_j y_j over the unmasked keys (-inf if none).
template <int NC, bool MASKED>
__device__ __forceinline__ float row_scale_max(uint32_t* v, const float* dk, int first_key,
                                               int limit) {
  float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
  for (int j = 0; j < NC; j += 4) {
    const float4 d = *reinterpret_cast<const float4*>(dk + j);
    const float dd[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float y = __fmul_rn((float)(int)v[j + e], dd[e]);
      v[j + e] = __float_as_uint(y);
      if (!MASKED || first_key + j + e < limit) {
        if (e & 1) m1 = fmaxf(m1, y);
        else m0 = fmaxf(m0, y);
      }
    }
  }
  return fmaxf(m0, m1);
}

// Q smoothing: y = fma(S, c, bk_j) written back over S (fp32 bit patterns),
// the mean term bk (kappa applied) joining before the maximum; returns max y
// over the unmasked columns (-inf if none).
template <int NC, bool MASKED>
__device__ __forceinline__ float row_bias_max(uint32_t* v, const float* bk, float c, int first_key,
                                              int limit) {
  float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
  for (int j = 0; j < NC; j += 4) {
    const float4 b = *reinterpret_cast<const float4*>(bk + j);
    const float bb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float y = __fmaf_rn((float)(int)v[j + e], c, bb[e]);
      v[j + e] = __float_as_uint(y);
      if (!MASKED || first_key + j + e < limit) {
        if (e & 1) m1 = fmaxf(m1, y);
        else m0 = fmaxf(m0, y);
      }
    }
  }
  return fmaxf(m0, m1);
}

// p for NC columns: p = 2^fma(S, c, -m) (masked columns give 0); returns the
// sum of p.  Results are written to p[].
template <bool MASKED, int NC, bool FIN = false>
__device__ __forceinline__ float row_exp(const uint32_t* v, float c, float neg_m, int first_key,
                                         int limit, float* p) {
  const float2 c2 = make_float2(c, c), n2 = make_float2(neg_m, neg_m);
  float2 s2a = make_float2(0.0f, 0.0f), s2b = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int i = 0; i < NC; i += 2) {
    // FIN: v holds fp32 bit patterns (per-token dequantised scores), else int32 S
    const float2 x = FIN ? make_float2(__uint_as_float(v[i]), __uint_as_float(v[i + 1]))
                         : s32x2_to_f32x2(v[i], v[i + 1]);
    const float2 a = __ffma2_rn(x, c2, n2);
    float p0 = ptx::ex2(a.x), p1 = ptx::ex2(a.y);
    if (MASKED) {
      if (first_key + i >= limit) p0 = 0.0f;
      if (first_key + i + 1 >= limit) p1 = 0.0f;
    }
    p[i] = p0;
    p[i + 1] = p1;
    if ((i & 2) == 0) s2a = __fadd2_rn(s2a, make_float2(p0, p1));
    else s2b = __fadd2_rn(s2b, make_float2(p0, p1));
  }
  const float2 s = __fadd2_rn(s2a, s2b);
  return s.x + s.y;
}

template <int D, bool PV8, bool BF16V, int GR, bool DUMP>
__device__ __forceinline__ bool softmax_item(const AttnParams& p, const Work& w, Bars* B,
                                             uint32_t tmem, int t, const float* sKs, int I0,
                                             int G0, volatile int* loop) {
  using C = Cfg<D, PV8, GR>;
  [[maybe_unused]] constexpr bool TOK = GR == 1, SMQ = GR == 2;
  constexpr bool BM = C::block_max(BF16V);
  constexpr float TAU = C::tau(BF16V);
  // block maximum with 16-bit P: the even half's S stays in registers while
  // the odd half's maximum is taken (FP8 P.V: the fp32 accumulator needs those
  // registers, so S is loaded again)
  // (FP8 at D = 64 with per-token deltas or Q smoothing keeps it as well:
  // there S turns into scaled logits in place, which a reload would redo; the
  // 64-register accumulator leaves room, measured +2 % / +5 %)
  constexpr bool KEEP = BM && (!PV8 || (D == 64 && GR != 0));
  using In = In16<BF16V>;
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int r = quarter * 32 + lane;              // row within the query tile
  const int qt = 2 * w.pair + t;
  const int row = qt * BLK + r;                   // query index in the sequence
  const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
  const uint32_t tS0 = tmem + C::NBUF * SUB * t + lane_off;
  const uint32_t tO = tmem + C::TO + D * t + lane_off;
  const int nsub = t == 0 ? w.nsub0 : w.nsub1;

  // deltaQ of this tile's block, or (per token) of this row
  const float qd = __ldg(p.q_scale + (TOK ? (w.qs_idx0 + t) * BLK + r : w.qs_idx0 + t));
  float m = -INFINITY, l = 0.0f, alpha_prev = 1.0f, c = 0.0f;
  if constexpr (TOK) c = __fmul_rn(qd, p.kappa);  // fp32(deltaQ_i kappa), per row
  float o32[PV8 ? D : 1];
  if constexpr (PV8) {
#pragma unroll
    for (int i = 0; i < D; ++i) o32[i] = 0.0f;
  }
  const int limit = p.causal ? min(w.n, row + 1) : w.n;  // keys >= limit are masked
  // deltaK of the next 128-key block, loaded one block ahead so that its
  // global load is not on the path from S to the exponentials
  float kd_next = 0.0f;
  if (!TOK && nsub > 0) kd_next = __ldg(p.k_scale + w.ks_idx0);

  // sub-tile ii: are all its keys unmasked for every row of the tile?
  auto full_of = [&](int ii) -> bool {
    const int k0 = ii * SUB;
    return (k0 + SUB <= w.n) && (!p.causal || k0 + SUB - 1 <= qt * BLK);
  };
  // wait for QK^T of sub-tile ii and load its 64 columns of S
  auto wait_s = [&](int ii) -> bool {
    const int Ii = I0 + ii;
    if (!wait_bar(B, &B->s_full[t][C::sbuf(Ii)], C::sphase(Ii), p.status, true)) return false;
    ptx::tc_fence_after();
    return true;
  };
  auto load_s = [&](int ii, uint32_t (&sv)[SUB]) {
    const uint32_t tS = tS0 + SUB * C::sbuf(I0 + ii);
#pragma unroll
    for (int cc = 0; cc < SUB / 32; ++cc)
      ptx::tmem_ld32(tS + 32 * cc, *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * cc]));
    ptx::tmem_wait_ld();
  };
  // The scaled maximum of sub-tile ii (-inf when no key of it is unmasked for
  // this row).  Per token, S is first turned into y = fp32(S deltaK_j) in
  // place (with Q smoothing into y = fma(S, c, b_j)); the K deltas or the mean
  // term came with the K tile (wait on its barrier).
  auto tile_max = [&](uint32_t (&sv)[SUB], int ii, float& m_blk) -> bool {
    const int k0 = ii * SUB;
    const bool full = full_of(ii);
    if constexpr (TOK) {
      const int g = G0 + ii / 2;  // ring stage of the sub-tile
      if (!wait_bar(B, &B->k_full[g % C::NS], (g / C::NS) & 1, p.status, true)) return false;
      const float* dk = sKs + (g % C::NS) * BLK + (ii & 1) * SUB;
      const float ym = full ? row_scale_max<SUB, false>(sv, dk, k0, limit)
                            : row_scale_max<SUB, true>(sv, dk, k0, limit);
      m_blk = ym == -INFINITY ? -INFINITY : __fmul_rn(ym, c);
    } else if constexpr (SMQ) {
      const int g = G0 + ii / 2;
      if (!wait_bar(B, &B->k_full[g % C::NS], (g / C::NS) & 1, p.status, true)) return false;
      const float* bk = sKs + ((g % C::NS) * 2 + t) * BLK + (ii & 1) * SUB;
      m_blk = full ? row_bias_max<SUB, false>(sv, bk, c, k0, limit)
                   : row_bias_max<SUB, true>(sv, bk, c, k0, limit);
    } else {
      const int smax = full ? row_max<SUB>(sv, INT_MIN) : row_max_masked<SUB>(sv, INT_MIN, k0, limit);
      m_blk = smax == INT_MIN ? -INFINITY : __fmul_rn((float)smax, c);
    }
    return true;
  };

  for (int i = 0; i < nsub; ++i) {
    const int I = I0 + i;                        // sub-tile count of this tile over the items
    const int b = C::sbuf(I);                    // S buffer
    const uint32_t tS = tS0 + SUB * b;
    if (!TOK && (i & 1) == 0) {  // a new 128-key quantisation block: its delta
      c = __fmul_rn(__fmul_rn(qd, kd_next), p.kappa);
      if (i + 2 < nsub) kd_next = __ldg(p.k_scale + w.ks_idx0 + i / 2 + 1);
    }
    if (!wait_s(i)) return false;
    const int key0 = i * SUB;
    const bool full_tile = full_of(i);
    // `lead`: this sub-tile sets the maximum used for its p -- every sub-tile,
    // or with the block maximum the first half of each 128-key block, whose
    // maximum then covers the second half as well
    const bool lead = !BM || (i & 1) == 0;
    float alpha = 1.0f, rowsum = 0.0f, m_new = m;
    uint32_t sv[SUB];
    load_s(i, sv);
    if constexpr (DUMP) {  // the raw int32 S of this row and sub-tile, as computed
      if (row < w.n) {
        int4* dst = reinterpret_cast<int4*>(
            p.s_dump + ((long long)w.code_z * p.s_dump_ld + row) * p.s_dump_ld + key0);
#pragma unroll
        for (int k = 0; k < SUB / 4; ++k)
          dst[k] = make_int4((int)sv[4 * k], (int)sv[4 * k + 1], (int)sv[4 * k + 2], (int)sv[4 * k + 3]);
      }
    }
    if (lead) {
      float m_blk;
      if (!tile_max(sv, i, m_blk)) return false;
      if (BM && i + 1 < nsub) {
        float m2;
        if (!wait_s(i + 1)) return false;
        if constexpr (KEEP) {
          uint32_t sx[SUB];
          load_s(i + 1, sx);
          if (!tile_max(sx, i + 1, m2)) return false;
        } else {
          load_s(i + 1, sv);
          if (!tile_max(sv, i + 1, m2)) return false;
          load_s(i, sv);
          if constexpr (TOK || SMQ) {
            float unused;
            if (!tile_max(sv, i, unused)) return false;
          }
        }
        m_blk = fmaxf(m_blk, m2);
      }
      // a sub-tile (block) with no unmasked key for this row leaves the maximum unchanged
      m_new = m_blk > __fadd_rn(m, TAU) ? m_blk : m;
      alpha = m_new == m ? 1.0f : ptx::ex2(__fsub_rn(m, m_new));
    } else if constexpr (TOK || SMQ) {
      float unused;  // second half of a block: S to scaled logits in place
      if (!tile_max(sv, i, unused)) return false;
    }

    // multiplier inside the exponent: c, or 1 once S holds the scaled logit
    // (Q smoothing: arg = fp32(y - m))
    const float ce = SMQ ? 1.0f : c;
    if constexpr (!PV8) {
#pragma unroll
      for (int cc = 0; cc < SUB / 32; ++cc) {
        float pv[32];
        rowsum += full_tile ? row_exp<false, 32, TOK || SMQ>(sv + 32 * cc, ce, -m_new, key0 + 32 * cc, limit, pv)
                            : row_exp<true, 32, TOK || SMQ>(sv + 32 * cc, ce, -m_new, key0 + 32 * cc, limit, pv);
        uint32_t packed[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) packed[k] = In::pack(pv[2 * k], pv[2 * k + 1]);
        ptx::tmem_st16(tS + 16 * cc, packed);
      }
      // O <- alpha * O before this sub-tile's P.V accumulates into it (only
      // when some row's maximum moved by more than TAU)
      if (lead && i > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
        if (!wait_bar(B, &B->o_full[t], (I - 1) & 1, p.status, true)) return false;
        ptx::tc_fence_after();
        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t ov[32];
          ptx::tmem_ld32(tO + 32 * cc, ov);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const float2 x = __fmul2_rn(a2, make_float2(__uint_as_float(ov[k]), __uint_as_float(ov[k + 1])));
            ov[k] = __float_as_uint(x.x);
            ov[k + 1] = __float_as_uint(x.y);
          }
          ptx::tmem_st32(tO + 32 * cc, ov);
        }
      }
    } else {
      // P^ = e4m3(p), p formed already scaled by 448 in the exponent
      // (2^(arg + log2 448): no multiply), four per TMEM column, written over S;
      // the row sum l is of the scaled p, so the 448 cancels in the epilogue
      const float sub = __fsub_rn(kLog2_448, m_new);
#pragma unroll
      for (int cc = 0; cc < SUB / 16; ++cc) {
        float pv[16];
        rowsum += full_tile ? row_exp<false, 16, TOK || SMQ>(sv + 16 * cc, ce, sub, key0 + 16 * cc, limit, pv)
                            : row_exp<true, 16, TOK || SMQ>(sv + 16 * cc, ce, sub, key0 + 16 * cc, limit, pv);
        uint32_t packed[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) packed[k] = pack_e4m3x4(pv[4 * k], pv[4 * k + 1], pv[4 * k + 2], pv[4 * k + 3]);
        ptx::tmem_st4(tS + 4 * cc, packed);
      }
      if (lead && i > 0) {
        // two-level accumulation, once per 128-key block: O32 <- alpha_{b-1}
        // O32 + Part_{b-1}, the partial of both halves of the previous block
        // (its P.V completed before this block's QK^T landed)
        if (!wait_bar(B, &B->o_full[t], (I - 1) & 1, p.status, true)) return false;
        ptx::tc_fence_after();
        const float2 a2 = make_float2(alpha_prev, alpha_prev);
#pragma unroll
        for (int cb = 0; cb < D / 32; ++cb) {  // 32 columns per round trip: o32 is live
          uint32_t pv[32];
          ptx::tmem_ld32(tO + 32 * cb, pv);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const float2 x = __ffma2_rn(a2, make_float2(o32[32 * cb + k], o32[32 * cb + k + 1]),
                                        make_float2(__uint_as_float(pv[k]), __uint_as_float(pv[k + 1])));
            o32[32 * cb + k] = x.x;
            o32[32 * cb + k + 1] = x.y;
          }
        }
      }
    }
    l = __fadd_rn(__fmul_rn(alpha, l), rowsum);
    ptx::tmem_wait_st();
    ptx::tc_fence_before();
    ptx::mbar_arrive(&B->p_full[t][b]);
    m = m_new;
    if (lead) alpha_prev = alpha;
  }

  // ------------------------------------------------------------ epilogue --
  // FP8: the tile's V scales, one global load per thread issued before the
  // wait below, staged in shared memory once per item (rather than 8
  // dependent global loads per row)
  [[maybe_unused]] float vsc = 0.0f;
  if constexpr (PV8) {
    if (r < D) vsc = __ldg(p.v_scale + w.vs_idx * D + r);
  }
  // (o_full may lag by two phases here in 16-bit mode; o_done is unambiguous:
  // one phase per item in which this tile has keys)
  if (!wait_bar(B, &B->o_done[t], loop[1] & 1, p.status, true)) return false;
  ptx::tc_fence_after();
  [[maybe_unused]] const float* svs = reinterpret_cast<const float*>(
      reinterpret_cast<const uint8_t*>(B) + 1024) + t * D;
  if constexpr (PV8) {
    // Every warp of the tile is past the previous item's reads of the buffer:
    // this item's last P.V, just waited for, needed all four warps' P, which
    // each stored after its previous epilogue.
    if (r < D) const_cast<float*>(svs)[r] = vsc;
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&B->vs_full[t]);  // release: the lanes' stores
    if (!wait_bar(B, &B->vs_full[t], loop[1] & 1, p.status, true)) return false;
  }
  const bool store = row < w.n;
  const long long orow = (w.out_row0 + (long long)row * w.out_stride) * D;
  const float inv_l = 1.0f / l;
  // 16 (FP8 P.V: its fp32 accumulator is live too) or 32 columns at a time
  constexpr int EC = PV8 ? 16 : 32;
#pragma unroll
  for (int cc = 0; cc < D / EC; ++cc) {
    uint32_t ov[EC];
    if constexpr (EC == 16) ptx::tmem_ld16(tO + EC * cc, ov);
    else ptx::tmem_ld32(tO + EC * cc, ov);
    float vf[PV8 ? EC : 1];
    if constexpr (PV8) {  // the chunk's V scales, from the staged copy
      const float4* vs = reinterpret_cast<const float4*>(svs + EC * cc);
#pragma unroll
      for (int k = 0; k < EC / 4; ++k) {
        const float4 f = vs[k];
        vf[4 * k] = f.x;
        vf[4 * k + 1] = f.y;
        vf[4 * k + 2] = f.z;
        vf[4 * k + 3] = f.w;
      }
    }
    ptx::tmem_wait_ld();
    float o[EC];
#pragma unroll
    for (int k = 0; k < EC; ++k) {
      if constexpr (PV8) {
        const float acc = __fmaf_rn(alpha_prev, o32[EC * cc + k], __uint_as_float(ov[k]));
        o[k] = __fmul_rn(__fmul_rn(acc, vf[k]), inv_l);
      } else {
        o[k] = __fmul_rn(__uint_as_float(ov[k]), inv_l);
      }
    }
    if (!store) continue;
    if (p.out_dt == SAGE_F32) {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow + EC * cc);
#pragma unroll
      for (int k = 0; k < EC / 4; ++k) dst[k] = make_float4(o[4 * k], o[4 * k + 1], o[4 * k + 2], o[4 * k + 3]);
    } else {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + orow + EC * cc);
      const bool ob = p.out_dt == SAGE_BF16;
#pragma unroll
      for (int k = 0; k < EC / 8; ++k) {
        uint32_t u[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a = o[8 * k + 2 * e], bb = o[8 * k + 2 * e + 1];
          u[e] = ob ? In16<true>::pack(a, bb) : In16<false>::pack(a, bb);
        }
        dst[k] = make_uint4(u[0], u[1], u[2], u[3]);
      }
    }
  }
  return true;
}

// One softmax warpgroup per query tile t, over the CTA's work items.  The
// counts carried across items give the S buffer and barrier phases: I0 the
// tile's sub-tiles so far, G0 the ring stages, loop[1] the items with keys
// (o_done phase).  The item counts sit in a per-warp shared-memory slot
// rather than in registers, which the per-sub-tile loop needs.
template <int D, bool PV8, bool BF16V, int GR, bool DUMP>
__device__ void softmax_wg(const AttnParams& p, Bars* B, uint32_t tmem, int t, const float* sKs) {
  volatile int* loop = B->sm_loop[threadIdx.x / 32];  // [0] items taken, [1] items with keys
  loop[0] = 0;
  loop[1] = 0;
  int I0 = 0, G0 = 0;
  while (true) {
    const int r = loop[0];
    int idx;
    if (!take_item(B, r, p.status, true, idx) || idx < 0) return;
    loop[0] = r + 1;
    const Work w = decode_work(p, idx);
    if (!w.valid) continue;
    const int nsub = t == 0 ? w.nsub0 : w.nsub1;
    if (nsub > 0) {
      if (!softmax_item<D, PV8, BF16V, GR, DUMP>(p, w, B, tmem, t, sKs, I0, G0, loop)) return;
      loop[1] = loop[1] + 1;
    }
    I0 += nsub;
    G0 += w.nkv;
  }
}

// ---------------------------------------------------------------- kernel --

template <int D, bool PV8, bool BF16V, int GR, bool DUMP>
__global__ void __launch_bounds__(Cfg<D, PV8, GR>::THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using C = Cfg<D, PV8, GR>;
  [[maybe_unused]] constexpr bool TOK = GR == 1, SMQ = GR == 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + 2 * C::QT;
  uint8_t* sV = sK + C::NS * C::QT;
  float* sKs = reinterpret_cast<float*>(sV + C::NS * C::VT);  // GR 1: [NS][128] K deltas; GR 2: [NS][2][128] mean terms
  Bars* B = reinterpret_cast<Bars*>(sV + C::NS * (C::VT + C::KS));
  static_assert(sizeof(Bars) <= 1024, "aux layout");

  const int warp = threadIdx.x / 32;
  const int wg = warp / 4;
  const int warp_tma = 4 * C::WG_CTRL, warp_mma = 4 * C::WG_CTRL + 1;  // MMA warps: +1, +2

  if (threadIdx.x == 0) {
    ptx::mbar_init(&B->q_full, 1);
    ptx::mbar_init(&B->q_empty, 2);  // one commit per MMA warp
    for (int r = 0; r < 2; ++r) {
      ptx::mbar_init(&B->item_full[r], 1);
      ptx::mbar_init(&B->item_empty[r], ITEM_READERS);
    }
    ptx::mbar_init(&B->done[0], 1);
    ptx::mbar_init(&B->done[1], 1);
    for (int t = 0; t < 2; ++t) {
      ptx::mbar_init(&B->o_full[t], 1);
      ptx::mbar_init(&B->vs_full[t], 4);
      ptx::mbar_init(&B->o_done[t], 1);
      for (int b = 0; b < 3; ++b) {
        ptx::mbar_init(&B->s_full[t][b], 1);
        ptx::mbar_init(&B->p_full[t][b], 128);
      }
    }
    for (int s = 0; s < C::NS; ++s) {
      ptx::mbar_init(&B->k_full[s], 1);
      ptx::mbar_init(&B->v_full[s], 1);
      ptx::mbar_init(&B->kv_empty[s], 2);  // one commit per query tile
    }
    B->abort = 0;
    B->wait_limit = p.wait_limit > 0 ? p.wait_limit : SAGE_WAIT_LIMIT_CYCLES;
    ptx::fence_barrier_init();
  }
  if (warp == warp_mma) {
    ptx::tmem_alloc(&B->tmem_base, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = B->tmem_base;

  if (wg == C::WG_CTRL) {
    ptx::setmaxnreg_dec<C::REG_CTRL>();
    if (warp == warp_tma) {
      producer<D, PV8, GR>(&tm_q, &tm_k, &tm_v, p, B, sQ, sK, sV, sKs);
    } else if (warp == warp_mma || warp == warp_mma + 1) {
      mma_issuer<D, PV8, BF16V, GR>(p, B, tmem, sQ, sK, sV, warp - warp_mma);
    }
  } else {
    ptx::setmaxnreg_inc<C::REG_SOFTMAX>();
    softmax_wg<D, PV8, BF16V, GR, DUMP>(p, B, tmem, wg, sKs);
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == warp_mma) ptx::tmem_dealloc(tmem, 512);
  // Every fetch of this CTA happened before the barrier above: the last CTA
  // to get here resets the scheduler for the next launch.
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.sched + 1, 1u) == gridDim.x - 1) {
      __threadfence();
      atomicExch(p.sched, 0u);
      atomicExch(p.sched + 1, 0u);
    }
  }
}

// ------------------------------------------------ QK^T tile diagnostic --

// One CTA per requested tile (bh, I, J): TMA-load Q^ tile I and K^ tile J,
// the same kind::i8 MMA sequence the attention kernel issues, then 4 warps
// copy the int32 tile out of TMEM.
template <int D>
__global__ void __launch_bounds__(128, 1)
    qk_tile_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const int32_t* __restrict__ tiles, int32_t* __restrict__ s_out,
                   uint32_t* status) {
  constexpr int QT = BLK * D;
  constexpr uint32_t SWZ = (D == 128) ? 2u : 4u;
  constexpr uint32_t IDESC_QK = ptx::instr_desc(2, 1, 1, 0, 0, 128, 128);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + QT;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + 2 * QT);
  uint32_t* tbase = reinterpret_cast<uint32_t*>(bar + 2);
  int* okflag = reinterpret_cast<int*>(tbase + 1);
  const int bh = __ldg(tiles + 3 * blockIdx.x), I = __ldg(tiles + 3 * blockIdx.x + 1),
            J = __ldg(tiles + 3 * blockIdx.x + 2);
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar[0], 1);
    ptx::mbar_init(&bar[1], 1);
    ptx::fence_barrier_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(tbase, 128);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tbase;
  if (threadIdx.x == 0) {
    ptx::mbar_arrive_expect_tx(&bar[0], 2 * QT);
    ptx::tma_load_3d(sA, &tm_q, &bar[0], 0, I * BLK, bh);
    ptx::tma_load_3d(sB, &tm_k, &bar[0], 0, J * BLK, bh);
    bool ok = ptx::mbar_wait(&bar[0], 0);
    if (ok) {
      ptx::tc_fence_after();
      const uint32_t a = ptx::smem_u32(sA), b = ptx::smem_u32(sB);
#pragma unroll
      for (int kk = 0; kk < D / 32; ++kk)
        ptx::mma_i8_ss(tmem, ptx::smem_desc(a + 32 * kk, 16, 8 * D, SWZ),
                       ptx::smem_desc(b + 32 * kk, 16, 8 * D, SWZ), IDESC_QK, kk > 0 ? 1u : 0u);
    }
    ptx::mma_commit(&bar[1]);
    ok = ptx::mbar_wait(&bar[1], 0) && ok;
    if (!ok) set_status(status, ST_TIMEOUT);
    *okflag = ok ? 1 : 0;
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (*okflag) {
    const int r = warp * 32 + lane;
    int32_t* dst = s_out + (long long)blockIdx.x * BLK * BLK + (long long)r * BLK;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t v[32];
      ptx::tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + 32 * cc, v);
      ptx::tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<int4*>(dst + 32 * cc + i) = make_int4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 0) ptx::tmem_dealloc(tmem, 128);
}

}  // namespace

// =================================================================== host ==

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3-D tiled map over a row-major tensor [dim2][dim1][dim0] with element size
// esz; box {b0, b1, b2}.  Returns false when the driver rejects it.
static bool make_map3(CUtensorMap* m, CUtensorMapDataType dt, int esz, const void* base,
                      uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1_bytes, uint64_t s2_bytes,
                      uint32_t b0, uint32_t b1, uint32_t b2, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  (void)esz;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {s1_bytes, s2_bytes};
  const cuuint32_t box[3] = {b0, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static CUtensorMapSwizzle swz_for(int row_bytes) {
  return row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
}

template <int D, bool PV8, bool BF16V, int GR, bool DUMP = false>
static cudaError_t launch_attn_t(const AttnLaunch& L, cudaStream_t st) {
  using C = Cfg<D, PV8, GR>;
  [[maybe_unused]] constexpr bool TOK = GR == 1, SMQ = GR == 2;
  CUtensorMap tq, tk, tv;
  const CUtensorMapSwizzle cs = swz_for(D);
  if (!make_map3(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, L.q_codes, D, L.code_rows, L.code_z, D,
                 (uint64_t)D * L.code_rows, D, BLK, 1, cs) ||
      !make_map3(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, L.k_codes, D, L.code_rows, L.code_z_kv,
                 D, (uint64_t)D * L.code_rows, D, BLK, 1, cs))
    return cudaErrorInvalidValue;
  const int esz = PV8 ? 1 : 2;
  const CUtensorMapDataType vdt = PV8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                      : (BF16V ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                               : CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
  const uint32_t vbox0 = PV8 ? D : 64;  // box inner extent in elements (128 B or 64 B)
  const CUtensorMapSwizzle vs = swz_for(vbox0 * esz);
  bool okv;
  if (!L.p.varlen)
    okv = make_map3(&tv, vdt, esz, L.v, D, L.p.N, L.code_z_kv, (uint64_t)D * esz,
                    (uint64_t)D * esz * L.p.N, vbox0, BLK, 1, vs);
  else
    okv = make_map3(&tv, vdt, esz, L.v, D, L.code_z_kv, L.T, (uint64_t)D * esz,
                    (uint64_t)D * esz * L.code_z_kv, vbox0, 1, BLK, vs);
  if (!okv) return cudaErrorInvalidValue;
  auto kern = attn_fwd_kernel<D, PV8, BF16V, GR, DUMP>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (L.p.items <= 0) return cudaSuccess;
  kern<<<dim3((unsigned)std::min(L.p.items, std::max(sms, 1))), C::THREADS, C::SMEM, st>>>(tq, tk, tv, L.p);
  return cudaGetLastError();
}

template <int GR>
static cudaError_t launch_attn_g(const AttnLaunch& L, cudaStream_t st) {
  if (L.D == 64) {
    if (L.pv8) return launch_attn_t<64, true, false, GR>(L, st);
    return L.bf16v ? launch_attn_t<64, false, true, GR>(L, st)
                   : launch_attn_t<64, false, false, GR>(L, st);
  }
  if (L.pv8) return launch_attn_t<128, true, false, GR>(L, st);
  return L.bf16v ? launch_attn_t<128, false, true, GR>(L, st)
                 : launch_attn_t<128, false, false, GR>(L, st);
}

cudaError_t launch_attn(const AttnLaunch& L, cudaStream_t st) {
  if (L.p.s_dump) {  // diagnostic instances: dense, per-block deltas, fp16 V or FP8 P.V
    if (L.p.varlen || L.p.per_token || (!L.pv8 && L.bf16v)) return cudaErrorNotSupported;
    if (L.D == 64)
      return L.pv8 ? launch_attn_t<64, true, false, 0, true>(L, st)
                   : launch_attn_t<64, false, false, 0, true>(L, st);
    return L.pv8 ? launch_attn_t<128, true, false, 0, true>(L, st)
                 : launch_attn_t<128, false, false, 0, true>(L, st);
  }
  if (L.p.per_token == 2) return launch_attn_g<2>(L, st);
  return L.p.per_token ? launch_attn_g<1>(L, st) : launch_attn_g<0>(L, st);
}

template <int D>
static cudaError_t launch_qk_tiles_t(const int8_t* qc, const int8_t* kc, int BH, int NP,
                                     const int32_t* tiles, int n, int32_t* out, uint32_t* status,
                                     cudaStream_t st) {
  CUtensorMap tq, tk;
  const CUtensorMapSwizzle cs = swz_for(D);
  if (!make_map3(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, qc, D, NP, BH, D, (uint64_t)D * NP, D,
                 BLK, 1, cs) ||
      !make_map3(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kc, D, NP, BH, D, (uint64_t)D * NP, D,
                 BLK, 1, cs))
    return cudaErrorInvalidValue;
  const int smem = 1024 + 2 * BLK * D + 64;
  auto kern = qk_tile_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<n, 128, smem, st>>>(tq, tk, tiles, out, status);
  return cudaGetLastError();
}

cudaError_t launch_qk_tiles(const int8_t* qc, const int8_t* kc, int BH, int NP, int D,
                            const int32_t* tiles, int n, int32_t* out, uint32_t* status,
                            cudaStream_t st) {
  return D == 64 ? launch_qk_tiles_t<64>(qc, kc, BH, NP, tiles, n, out, status, st)
                 : launch_qk_tiles_t<128>(qc, kc, BH, NP, tiles, n, out, status, st);
}

}  // namespace sage
