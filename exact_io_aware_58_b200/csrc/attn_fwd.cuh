// attn_fwd.cuh -- forward kernel: tiled exact attention with online softmax.
//
// Method ("Attention and KV Compression", section "Tiling and online softmax";
// "FlashAttention -- how 100K-token attention fits in memory", sections
// "FlashAttention idea" and "Online softmax intuition"): a block of query rows
// stays on chip while blocks of keys and values stream past it; for each key
// block the scores are formed on chip, a running row max m and row sum l are
// kept, the partial output is rescaled by exp(m_old - m_new) when the max
// grows, and only O and one statistic per row (LSE) are written out.
//
// B200 mapping: a persistent grid of at most one CTA per SM (384 threads).  A
// work item is two 128-row query tiles of one head; items are ordered
// heads-major, heaviest causal blocks first within a head (so that a head's
// K/V stays in L2 while its items run), and dealt out in rounds of one item
// per CTA (every other round in reverse when that balances better).  All
// roles walk the same item sequence and their barrier phases run on across
// items, so the next item's Q load and first QK^T products overlap the
// current item's last softmax and its output stores.
//   warp 9      TMA producer: per item Q0, Q1, then K_j / V_j 128-row tiles
//               into a ring of shared-memory slots (128-byte swizzle) that
//               runs on across items.
//   warp 8      MMA issuer (one thread): S_t = Q_t K_j^T and O_t += P_t V_j as
//               tcgen05.mma with fp32 accumulators in tensor memory (TMEM).
//   warps 10-11 idle: they complete warpgroup 2, whose registers go to the
//               softmax warpgroups (setmaxnreg, see FwdCfg).
//   warps 0-3   softmax for query tile 0, warps 4-7 for tile 1: each thread owns
//               one query row (= one TMEM lane), so the row max and sum need no
//               shuffles.  P is rounded to bf16 and written back into TMEM over
//               the upper half of S, where the PV MMA reads it as its A operand.
//               At the end of an item each thread reads its whole O row out of
//               TMEM in one round trip, releases O_t to the next item's first
//               PV, and writes the normalised row (and LSE) straight to global
//               memory, so that the Q slots are free for the next item as soon
//               as its last QK^T is done.
// The issue order PV_t(j-1), S_t(j) lets the tensor core run one tile's GEMMs
// while the other tile's softmax runs (ping-pong between the two tiles).
//
// Rescaling is lazy but exact: the reference max m_ref used in the exponent is
// only moved when a tile's max exceeds it by more than kRescaleLog2 (2^8); O
// and l always share the same m_ref, so O = acc / l is unchanged, and LSE is
// computed from the same pair.
#pragma once

#include "sm100.cuh"

namespace attn {

constexpr float kRescaleLog2 = 8.0f;
constexpr float kLn2 = 0.6931471805599453f;

struct FwdParams {
  __nv_bfloat16* o;    // [B*H][N][D] output
  float* lse;          // [B*H][N] natural-log LSE
  int n;               // sequence length N
  int n_mblk;          // number of 256-row query blocks per head
  int h;               // query heads per batch
  int h_kv;            // key/value heads per batch (h % h_kv == 0)
  int group;           // h / h_kv query heads share one key/value head
  float scale_log2;    // scale * log2(e)
  const uint8_t* mask; // block-sparse only: [B*H][nt][nt], 1 = query tile attends key tile
  int nt;              // ceil(N / 128)
  float* o32;          // O32 instances only: [B*H][N][D] fp32 copy of the normalised O
  int n_items;         // B*H*n_mblk work items (packed-sequence instances count their own)
  int snake;           // 1: odd rounds of grid-size items are dealt to the CTAs in reverse
  const int* cu_seqlens;   // packed sequences only: [n_seqs + 1] token offsets (device)
  int n_seqs;              // packed sequences only: number of sequences
  int total;               // packed sequences only: total tokens (rows of Q, K, V, O)
};

// The items of round r (items [r*G, r*G + G), G = grid size) go one per CTA;
// with `snake`, odd rounds go in reverse CTA order, which pairs heavy causal
// blocks with light ones (the host picks the order and G that balance best).
__device__ __forceinline__ int fwd_round_item(int r, int G, int snake) {
  const int pos = (snake && (r & 1)) ? G - 1 - int(blockIdx.x) : int(blockIdx.x);
  return r * G + pos;
}

// Key tiles selected for the (up to) two 128-row query tiles of a CTA: bit t of
// flags(j) says query tile t attends key tile j.  Every role scans the same
// bytes, so they all walk the same sequence of tiles.
struct TileSelect {
  const uint8_t* r0;
  const uint8_t* r1;   // null when the second query tile is past N
  __device__ __forceinline__ uint32_t flags(int j) const {
    return (r0[j] ? 1u : 0u) | ((r1 != nullptr && r1[j]) ? 2u : 0u);
  }
  __device__ __forceinline__ int next(int j, int hi) const {   // first selected tile > j, or hi
    for (++j; j < hi; ++j)
      if (flags(j)) return j;
    return hi;
  }
  __device__ __forceinline__ int count(int hi) const {
    int c = 0;
    for (int j = 0; j < hi; ++j) c += flags(j) ? 1 : 0;
    return c;
  }
};

template <int D>
struct FwdCfg {
  static constexpr int kTileBytes = 128 * D * 2;        // one 128 x D bf16 tile
  static constexpr int kBlockBytes = 128 * 128;          // one [128][64] bf16 column block
  static constexpr int kNumBlk = D / 64;
  static constexpr int kSlots = (D == 128) ? 4 : 8;      // K/V ring depth
  // Warps 0-7 softmax (two warpgroups), warpgroup 2 = MMA warp, TMA warp and
  // two idle warps.  Registers are allocated per warpgroup slot, so a block
  // of three warpgroups is launched with 168 per thread (3 * 168 <= 512 per
  // SM sub-partition, which holds one warp of each warpgroup); warpgroup 2
  // then gives registers back (setmaxnreg) and the softmax warpgroups take
  // them: 2 * 176 + 152 = 3 * 168.  The issue warpgroup keeps 152 because its
  // unrolled descriptor code spills below that in the packed-sequence
  // instances; 176 lets the epilogue hold a whole O row without spilling.
  // The host refuses to launch unless the kernel compiled to exactly
  // kRegsLaunch, which the split assumes.
  static constexpr int kThreads = 384;
  static constexpr int kWarpMma = 8;
  static constexpr int kWarpLoad = 9;
  static constexpr uint32_t kRegsLaunch = 168;
  static constexpr uint32_t kRegsIssue = 152;
  static constexpr uint32_t kRegsSoftmax = 176;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128;
  static constexpr uint32_t kColO0 = 256, kColO1 = 256 + D;
  static constexpr uint32_t kColPOff = 64;               // P (bf16 pairs) over S columns 64..127
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = 2 * kTileBytes;
  static constexpr int kOffBar = kOffKV + kSlots * kTileBytes;
  static constexpr int kNumBars = 2 + 2 * kSlots + 2 + 2 + 2 + 2 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;   // + slack for 1024-byte alignment
  static_assert(2 * kRegsSoftmax + kRegsIssue <= 3 * kRegsLaunch, "register split");
};

// Work item -> (query head, first query row, key tiles that may be visible,
// selection, key tiles visited, where its rows live).  Every role evaluates
// the same function on the same increasing item sequence.
struct FwdItem {
  int bh, bkv, m0, kv_hi, nkv;
  int nkv0;             // key tiles query tile 0 visits (causal: one fewer than nkv when the
                        // item's last key tile lies wholly above tile 0's rows)
  int n;                // rows of this item's sequence (N, or the packed sequence's length)
  int head, head_kv;    // query / key-value head (packed sequences)
  int tok0;             // first token of the sequence in the packed tensors (0 otherwise)
  TileSelect sel;
};

// Packed sequences: sequence s holds tokens [cu[s], cu[s+1]); its items are
// its heads times its 256-row blocks, heaviest causal blocks first.  The
// cursor only moves forward, because each role asks for increasing items.
struct SeqCursor {
  int s = 0;       // current sequence
  int base = 0;    // items of the sequences before it
};

// First token and length of sequence s, clamped to [0, total] (offsets past
// the tensors, or decreasing ones, give empty sequences: nothing is read or
// written outside the tensors whatever cu_seqlens holds).
__device__ __forceinline__ int seq_start(const FwdParams& prm, int s) {
  return min(max(prm.cu_seqlens[s], 0), prm.total);
}
__device__ __forceinline__ int seq_len(const FwdParams& prm, int s) {
  return max(min(max(prm.cu_seqlens[s + 1], 0), prm.total) - seq_start(prm, s), 0);
}
__device__ __forceinline__ int seq_blocks(const FwdParams& prm, int s) { return (seq_len(prm, s) + 255) >> 8; }

__device__ __forceinline__ int packed_items(const FwdParams& prm) {
  int total = 0;
  for (int s = 0; s < prm.n_seqs; ++s) total += prm.h * seq_blocks(prm, s);
  return total;
}

template <bool CAUSAL, bool SPARSE, bool VARLEN>
__device__ __forceinline__ FwdItem fwd_item(const FwdParams& prm, int item, SeqCursor& cur) {
  FwdItem w;
  int m_blk, n_mblk;
  if (VARLEN) {
    while (cur.s + 1 < prm.n_seqs && item >= cur.base + prm.h * seq_blocks(prm, cur.s)) {
      cur.base += prm.h * seq_blocks(prm, cur.s);
      ++cur.s;
    }
    n_mblk = max(seq_blocks(prm, cur.s), 1);
    const int local = item - cur.base;
    w.head = local / n_mblk;
    w.head_kv = w.head / prm.group;
    w.tok0 = seq_start(prm, cur.s);
    w.n = seq_len(prm, cur.s);
    w.bh = w.head;
    w.bkv = w.head_kv;
    m_blk = n_mblk - 1 - local % n_mblk;
  } else {
    n_mblk = prm.n_mblk;
    w.bh = item / n_mblk;
    w.bkv = (w.bh / prm.h) * prm.h_kv + (w.bh % prm.h) / prm.group;
    w.head = w.bh;
    w.head_kv = w.bkv;
    w.tok0 = 0;
    w.n = prm.n;
    m_blk = n_mblk - 1 - (item % n_mblk);   // heaviest causal blocks of a head first
  }
  w.m0 = m_blk * 256;
  const int n_kv_total = (w.n + 127) >> 7;
  w.kv_hi = CAUSAL ? min(n_kv_total, (w.m0 >> 7) + 2) : n_kv_total;
  w.sel = TileSelect{nullptr, nullptr};
  if (SPARSE) {
    const int qt0 = w.m0 >> 7;
    w.sel.r0 = prm.mask + (size_t(w.bh) * prm.nt + qt0) * prm.nt;
    w.sel.r1 = (qt0 + 1 < prm.nt) ? w.sel.r0 + prm.nt : nullptr;
  }
  w.nkv = SPARSE ? w.sel.count(w.kv_hi) : w.kv_hi;
  // Causal: key tile 2m+1 (the last one, when N does not cut it off) starts
  // after the last row of query tile 0, so only tile 1 needs it.  (Not in the
  // packed-sequence instances, whose issue warp would spill.)
  w.nkv0 = (CAUSAL && !SPARSE && !VARLEN && w.kv_hi == (w.m0 >> 7) + 2) ? w.nkv - 1 : w.nkv;
  return w;
}

// TMA coordinates of rows [r0, r0 + 128) of a head: BHND tensors are mapped
// as [B*H][N][d] (coordinates x, row, head); packed ones as [total][H][d]
// (coordinates x, head, token).
template <bool VARLEN>
__device__ __forceinline__ void load_rows(const CUtensorMap* map, uint64_t* bar, void* dst, int x, int head,
                                          int tok0, int r0) {
  if (VARLEN)
    tma_load_3d(map, bar, dst, x, head, tok0 + r0);
  else
    tma_load_3d(map, bar, dst, x, r0, head);
}

// O32: also write the normalised rows in fp32 to prm.o32 (a separate
// instance, so the bf16-only instances are compiled without it).
// VARLEN: packed sequences of different lengths ([total][H][d] tensors, one
// causal/non-causal attention per sequence; dense, bf16 output only).
template <int D, bool CAUSAL, bool SPARSE, bool O32 = false, bool VARLEN = false>
__global__ void __launch_bounds__(384, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const FwdParams prm) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;                  // Q0, Q1 of the current item landed
  uint64_t* q_empty = q_full + 1;           // the item's last QK^T products are done: Q slots free
  uint64_t* kv_full = q_empty + 1;
  uint64_t* kv_empty = kv_full + C::kSlots;
  uint64_t* s_full = kv_empty + C::kSlots;  // [2] S_t in TMEM
  uint64_t* p_full = s_full + 2;            // [2] P_t written back (128 arrivals)
  uint64_t* o_full = p_full + 2;            // [2] the item's O_t complete
  uint64_t* o_free = o_full + 2;            // [2] O_t read out by the epilogue (128 arrivals)
  uint64_t* drain = o_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_items = VARLEN ? packed_items(prm) : prm.n_items;
  // d = 64 dense instances give the softmax 192 (the issue warpgroup fits in
  // 120 there); the others use FwdCfg's 176 / 152.
  constexpr uint32_t kRegsSoftmaxI = (D == 64 && !VARLEN) ? 192u : C::kRegsSoftmax;
  constexpr uint32_t kRegsIssueI = 3 * C::kRegsLaunch - 2 * kRegsSoftmaxI;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      mbar_init(&o_full[t], 1);
      mbar_init(&o_free[t], 128);
    }
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == C::kWarpMma) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == C::kWarpLoad && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= C::kWarpMma) {
   // warpgroup 2: one TMA thread, one MMA thread, two idle warps
   regs_dec<kRegsIssueI>();
   if (warp == C::kWarpLoad) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      int issued = 0;    // K/V tiles loaded (ring position)
      int qn = 0;        // items whose Q was loaded
      bool ok = true;
      SeqCursor cur;
      for (int rr = 0, item = fwd_round_item(0, gridDim.x, prm.snake); rr * int(gridDim.x) < n_items && ok;
           item = fwd_round_item(++rr, gridDim.x, prm.snake)) {
        if (item >= n_items) continue;
        const FwdItem w = fwd_item<CAUSAL, SPARSE, VARLEN>(prm, item, cur);
        if (w.nkv == 0) continue;   // block-sparse: nothing selected, nothing loaded
        // the previous item's last QK^T products must be done with the Q slots
        if (qn > 0 && !(ok = mbar_wait(q_empty, (qn - 1) & 1, abort_flag))) break;
        mbar_arrive_expect_tx(q_full, 2 * C::kTileBytes);
        for (int t = 0; t < 2; ++t)
          for (int b = 0; b < C::kNumBlk; ++b)
            load_rows<VARLEN>(&tm_q, q_full, smem + C::kOffQ + t * C::kTileBytes + b * C::kBlockBytes, b * 64,
                              w.bh, w.tok0, w.m0 + 128 * t);
        ++qn;
        int jsel = SPARSE ? w.sel.next(-1, w.kv_hi) : 0;
        for (int kk = 0; kk < 2 * w.nkv; ++kk) {
          const int slot = issued % C::kSlots;
          const int use = issued / C::kSlots;
          if (use > 0 && !(ok = mbar_wait(&kv_empty[slot], (use - 1) & 1, abort_flag))) break;
          const CUtensorMap* tm = (kk & 1) ? &tm_v : &tm_k;
          const int j = SPARSE ? jsel : (kk >> 1);
          if (SPARSE && (kk & 1)) jsel = w.sel.next(jsel, w.kv_hi);
          mbar_arrive_expect_tx(&kv_full[slot], C::kTileBytes);
          for (int b = 0; b < C::kNumBlk; ++b)
            load_rows<VARLEN>(tm, &kv_full[slot], smem + C::kOffKV + slot * C::kTileBytes + b * C::kBlockBytes,
                              b * 64, w.bkv, w.tok0, 128 * j);
          ++issued;
        }
      }
      // No copy may still be landing in shared memory when the CTA leaves.
      if (qn > 0) mbar_wait(q_full, (qn - 1) & 1, abort_flag, false);
      for (int it = max(0, issued - C::kSlots); it < issued; ++it)
        mbar_wait(&kv_full[it % C::kSlots], (it / C::kSlots) & 1, abort_flag, false);
    }
    __syncwarp();
   } else if (warp == C::kWarpMma) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16(128, 128, false, false);
      constexpr uint32_t kIdescPV = idesc_bf16(128, D, false, true);
      const uint32_t sQ = smem_u32(smem + C::kOffQ);
      const uint32_t sKV = smem_u32(smem + C::kOffKV);
      int it = 0;        // K/V tiles consumed (ring position)
      auto wait_kv = [&](int& slot) -> bool {
        slot = it % C::kSlots;
        const bool r = mbar_wait(&kv_full[slot], (it / C::kSlots) & 1, abort_flag);
        ++it;
        return r;
      };
      auto issue_s = [&](int t, int kslot) {
        const uint32_t a0 = sQ + t * C::kTileBytes;
        const uint32_t b0 = sKV + kslot * C::kTileBytes;
        const uint32_t dt = tmem + (t ? C::kColS1 : C::kColS0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kBlockBytes + (kk & 3) * 32;
          mma_ss(dt, smem_desc_sw128(a0 + off, 16, 1024), smem_desc_sw128(b0 + off, 16, 1024), kIdescS,
                 kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int t, int vslot, bool acc) {
        const uint32_t b0 = sKV + vslot * C::kTileBytes;
        const uint32_t dt = tmem + (t ? C::kColO1 : C::kColO0);
        const uint32_t at = tmem + (t ? C::kColS1 : C::kColS0) + C::kColPOff;
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          mma_ts(dt, at + kk * 8, smem_desc_sw128(b0 + kk * 2048, C::kBlockBytes, 1024), kIdescPV,
                 (acc || kk > 0) ? 1u : 0u);
      };

      bool ok = true;
      int qn = 0;        // items processed
      int pc[2] = {0, 0};   // key tiles query tile t processed over all items (S_t/P_t barrier phases)
      SeqCursor cur;
      for (int rr = 0, item = fwd_round_item(0, gridDim.x, prm.snake); rr * int(gridDim.x) < n_items && ok;
           item = fwd_round_item(++rr, gridDim.x, prm.snake)) {
        if (item >= n_items) continue;
        const FwdItem w = fwd_item<CAUSAL, SPARSE, VARLEN>(prm, item, cur);
        const int nkv = w.nkv, nkv0 = w.nkv0;
        if (nkv == 0) continue;
        // PV of key tile jl (of this item) for query tile t; the item's first
        // PV overwrites O_t, which the previous item's epilogue must have read.
        auto pv = [&](int t, int jl, int vslot) -> bool {
          if (!mbar_wait(&p_full[t], (pc[t] + jl) & 1, abort_flag)) return false;
          if (jl == 0 && qn > 0 && !mbar_wait(&o_free[t], (qn - 1) & 1, abort_flag)) return false;
          tc_fence_after();
          issue_pv(t, vslot, jl > 0);
          return true;
        };
        int ks;
        if (!(ok = mbar_wait(q_full, qn & 1, abort_flag))) break;
        if (!(ok = wait_kv(ks))) break;
        tc_fence_after();
        issue_s(0, ks);
        mma_commit(&s_full[0]);
        issue_s(1, ks);
        mma_commit(&s_full[1]);
        mma_commit(&kv_empty[ks]);
        if (nkv == 1) mma_commit(q_empty);
        for (int j = 1; j < nkv && ok; ++j) {
          int vs;
          if (!(ok = wait_kv(vs))) break;
          if (!(ok = wait_kv(ks))) break;
          for (int t = 0; t < 2; ++t) {
            if (!(ok = pv(t, j - 1, vs))) break;
            if (t == 1) mma_commit(&kv_empty[vs]);
            if (t == 0 && j >= nkv0) continue;       // key tile j is wholly masked for tile 0
            issue_s(t, ks);
            mma_commit(&s_full[t]);
          }
          if (!ok) break;
          mma_commit(&kv_empty[ks]);
          if (j == nkv - 1) mma_commit(q_empty);   // the item's last QK^T: Q slots free
        }
        if (!ok) break;
        int vs;
        if (!(ok = wait_kv(vs))) break;
        for (int t = 0; t < 2 && ok; ++t) {
          if (t == 1 || nkv - 1 < nkv0)
            if (!(ok = pv(t, nkv - 1, vs))) break;
          mma_commit(&o_full[t]);               // after the tile's last PV
        }
        if (!ok) break;
        mma_commit(&kv_empty[vs]);
        pc[0] += nkv0;
        pc[1] += nkv;
        ++qn;
      }
      // Every MMA issued so far must finish before tensor memory is released.
      mma_commit(drain);
      mbar_wait(drain, 0, abort_flag, false);
    }
    __syncwarp();
   }
  } else {
    // -------------------------------------------------------------- softmax
    regs_inc<kRegsSoftmaxI>();
    const int t = warp >> 2;
    const int qw = warp & 3;
    const int r = qw * 32 + lane;           // row inside the tile = TMEM lane
    const uint32_t lane_base = uint32_t(qw * 32) << 16;
    const uint32_t tS = tmem + lane_base + (t ? C::kColS1 : C::kColS0);
    const uint32_t tP = tS + C::kColPOff;
    const uint32_t tO = tmem + lane_base + (t ? C::kColO1 : C::kColO0);
    const float c = prm.scale_log2;
    bool ok = true;
    int qn = 0, pc = 0;
    SeqCursor cur;
    for (int rr = 0, item = fwd_round_item(0, gridDim.x, prm.snake); rr * int(gridDim.x) < n_items && ok;
           item = fwd_round_item(++rr, gridDim.x, prm.snake)) {
        if (item >= n_items) continue;
      const FwdItem w = fwd_item<CAUSAL, SPARSE, VARLEN>(prm, item, cur);
      const int m0 = w.m0;
      const int n = VARLEN ? w.n : prm.n;
      const int i = m0 + 128 * t + r;         // query row within its sequence
      // where row i lives: LSE index and (computed where it is used) O element offset
      const size_t l_off = VARLEN ? size_t(w.head) * size_t(prm.total) + size_t(w.tok0 + i)
                                  : size_t(w.bh) * size_t(n) + size_t(i);
      auto o_offset = [&]() -> size_t {
        return VARLEN ? (size_t(w.tok0 + i) * size_t(prm.h) + size_t(w.head)) * D : l_off * D;
      };
      if (w.nkv == 0) {
        // block-sparse: a block that selected nothing: O = 0, LSE = -inf
        if (i < n) {
          const size_t o_off = o_offset();
          uint4* dst = reinterpret_cast<uint4*>(prm.o + o_off);
#pragma unroll
          for (int k = 0; k < D / 8; ++k) dst[k] = make_uint4(0u, 0u, 0u, 0u);
          if (O32) {
            float4* d32 = reinterpret_cast<float4*>(prm.o32 + o_off);
#pragma unroll
            for (int k = 0; k < D / 4; ++k) d32[k] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
          prm.lse[l_off] = -INFINITY;
        }
        continue;
      }
      float m_ref = -INFINITY;
      float l = 0.f;
      int jsel = SPARSE ? w.sel.next(-1, w.kv_hi) : 0;
      const int nkv_t = (t == 0) ? w.nkv0 : w.nkv;   // key tiles this query tile visits
      for (int jj = 0; jj < nkv_t; ++jj) {
        // jj counts visited tiles (barrier phases); j is the key tile itself
        const int j = SPARSE ? jsel : jj;
        const bool tile_on = SPARSE ? ((w.sel.flags(j) >> t) & 1u) != 0 : true;
        if (SPARSE) jsel = w.sel.next(jsel, w.kv_hi);
        if (!(ok = mbar_wait_warp(&s_full[t], (pc + jj) & 1, abort_flag))) break;
        tc_fence_after();
        float s[128];
        {
          uint32_t a[32], b[32], e[32], f[32];
          tmem_ld32(tS + 0, a);
          tmem_ld32(tS + 32, b);
          tmem_ld32(tS + 64, e);
          tmem_ld32(tS + 96, f);
          tmem_ld_wait(a);
          reg_fence32(b);
          reg_fence32(e);
          reg_fence32(f);
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            s[k] = __uint_as_float(a[k]);
            s[32 + k] = __uint_as_float(b[k]);
            s[64 + k] = __uint_as_float(e[k]);
            s[96 + k] = __uint_as_float(f[k]);
          }
        }
        const bool need_mask = !tile_on || (CAUSAL && (128 * j + 127 > m0 + 128 * t)) || (128 * j + 128 > n);
        if (need_mask) {
          int limit = tile_on ? n - 1 - 128 * j : -1;     // a tile this query tile did not select: all masked
          if (CAUSAL) limit = min(limit, i - 128 * j);
#pragma unroll
          for (int k = 0; k < 128; ++k)
            if (k > limit) s[k] = -INFINITY;
        }
        // Row max as 8 independent chains (a single 127-long dependency chain
        // would leave the issue slots idle for its whole latency).
        float mxp[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) mxp[u] = s[u];
#pragma unroll
        for (int k = 8; k < 128; k += 8)
#pragma unroll
          for (int u = 0; u < 8; ++u) mxp[u] = fmaxf(mxp[u], s[k + u]);
        const float mx = fmaxf(fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])),
                               fmaxf(fmaxf(mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7])));
        const float m_tile = mx * c;
        float alpha = 1.f;
        bool rescale = false;
        if (m_tile > m_ref + kRescaleLog2) {
          alpha = ex2(m_ref - m_tile);      // 0 when m_ref is still -inf
          m_ref = m_tile;
          rescale = (jj > 0);
        }
        l *= alpha;
        const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
        // P in 32-key chunks (16 packed columns each): a chunk's registers are
        // free again as soon as it is stored, which keeps the loop spill-free.
        float sump[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float p0 = ex2(fmaf(s[32 * q + 2 * k], c, neg_m));
            const float p1 = ex2(fmaf(s[32 * q + 2 * k + 1], c, neg_m));
            sump[k & 3] += p0 + p1;
            pk[k] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tP + 16 * q, pk);
        }
        l += (sump[0] + sump[1]) + (sump[2] + sump[3]);
        if (__any_sync(0xffffffffu, rescale)) {
          // O_t holds the sum through key tile j-1 (its last PV completed before S_t(j)).
          const float a = rescale ? alpha : 1.f;
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tO + cc * 32, o);
            tmem_ld_wait(o);
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * a);
            tmem_st32(tO + cc * 32, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[t]);
      }
      if (!ok) break;

      // ---------------------------------------------------------- epilogue
      if (!(ok = mbar_wait_warp(&o_full[t], qn & 1, abort_flag))) break;
      tc_fence_after();
      // l == 0 only for rows that see no key at all (block-sparse): O = 0, LSE = -inf.
      const float inv_l = (SPARSE && !(l > 0.f)) ? 0.f : 1.f / l;
      const size_t o_off = o_offset();
      // The whole row in one TMEM round trip (D/32 loads, one wait), so O_t is
      // released to the next item's first PV before any of it is stored.
      uint32_t orow[D / 32][32];
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) tmem_ld32(tO + cc * 32, orow[cc]);
      tmem_ld_wait(orow[0]);
#pragma unroll
      for (int cc = 1; cc < D / 32; ++cc) reg_fence32(orow[cc]);
      tc_fence_before();
      mbar_arrive(&o_free[t]);                // O_t has been read: the next item may overwrite it
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        const uint32_t (&o)[32] = orow[cc];
        if (i < n) {
          uint4* dst = reinterpret_cast<uint4*>(prm.o + o_off + cc * 32);
#pragma unroll
          for (int ch = 0; ch < 4; ++ch)
            dst[ch] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * ch + 0]) * inv_l, __uint_as_float(o[8 * ch + 1]) * inv_l),
                                 pack_bf16x2(__uint_as_float(o[8 * ch + 2]) * inv_l, __uint_as_float(o[8 * ch + 3]) * inv_l),
                                 pack_bf16x2(__uint_as_float(o[8 * ch + 4]) * inv_l, __uint_as_float(o[8 * ch + 5]) * inv_l),
                                 pack_bf16x2(__uint_as_float(o[8 * ch + 6]) * inv_l, __uint_as_float(o[8 * ch + 7]) * inv_l));
          if (O32) {
            // the same normalised row in fp32, before the bf16 rounding
            float4* d32 = reinterpret_cast<float4*>(prm.o32 + o_off + cc * 32);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              d32[k] = make_float4(__uint_as_float(o[4 * k]) * inv_l, __uint_as_float(o[4 * k + 1]) * inv_l,
                                   __uint_as_float(o[4 * k + 2]) * inv_l, __uint_as_float(o[4 * k + 3]) * inv_l);
          }
        }
      }
      if (i < n) prm.lse[l_off] = (SPARSE && !(l > 0.f)) ? -INFINITY : (m_ref + __log2f(l)) * kLn2;
      pc += nkv_t;
      ++qn;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::kWarpMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace attn
