// attn_kvcache.cuh -- forward attention of a few new query rows against a
// key/value cache (decode and chunked-prefill shapes), with split-KV.
//
// Same computation as the square forward ("Attention and KV Compression",
// section "Tiling and online softmax"): key/value tiles stream past query rows
// held on chip, with a running row max and row sum and a rescaled accumulator.
// What changes is the shape regime ("FlashAttention -- how 100K-token attention
// fits in memory", section "Arithmetic intensity"): with Nq << Nk every cached
// key and value is used by only a handful of query rows, so the kernel is bound
// by reading the cache from HBM, not by the tensor cores.
//
// B200 mapping (work item = one 128-row tile of PACKED query rows x one chunk
// of key tiles; a persistent grid of one 192-thread CTA per SM walks the items):
//   * The g = H / H_kv query heads that share a key/value head, and their Nq
//     rows each, are packed into the rows of one MMA tile: packed row r is head
//     kvh*g + r / Nq, position r % Nq.  In a BHND tensor these rows are
//     contiguous, so one TMA box loads them and every cached tile is read once
//     per packed tile instead of once per query head.
//   * Split-KV: the key tiles of a (kv head, row tile) are cut into `splits`
//     contiguous chunks, one work item each, so that a decode batch with few
//     heads still spreads its cache over all SMs.  Each CTA writes an fp32 partial O (normalised by
//     its own row sum) and its partial LSE; attn_kvcache_merge_kernel combines
//     them (O = sum_s exp(LSE_s - LSE) O_s, LSE = log sum_s exp LSE_s).  With
//     one split the item writes the bf16 output directly.
//   * warp 5 TMA producer (each item's Q into one of two buffers, then its
//     K_j / V_j through a ring that runs on across items), warp 4 MMA
//     issuer, warps 0-3 softmax with one query row per thread.  S is double
//     buffered in TMEM, so S(j+1) runs on the tensor core while the softmax of
//     tile j runs; P(j) is written back over the upper half of S(j) and read
//     from TMEM by the PV MMA.  Warps whose 32 rows are all padding only keep
//     the barrier protocol.
//   * Few packed rows (at most 32, e.g. decode with up to 32 query heads per
//     key/value head): the rows are loaded into all four TMEM lane quarters
//     (four copies of the query box), so every lane quarter computes the same
//     scores, and warp w keeps an online softmax over key columns
//     [32w, 32w + 32) of each tile only.  Its P goes to its own 16 packed
//     columns of a dedicated P buffer whose other columns stay zero, so the
//     PV product of lane quarter w sums over its key subset alone: four
//     independent partials per item, merged with the split-KV partials.  The
//     per-warp softmax work per key tile drops fourfold, which is what keeps
//     the cache stream, not the softmax, the limit.
//   * Causal masking is bottom-right aligned: the new rows are the last Nq
//     positions of a sequence of L = kv_lens[b] tokens, so position p sees key
//     j iff j <= p + L - Nq.  Rows that see no key get O = 0 and LSE = -inf.
//   * Cache rows in [L, Nk) are never weighted: their scores are masked, and
//     the V rows of the last partial tile are cleared in shared memory before
//     the PV product, so stale or non-finite cache contents cannot leak in.
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"

namespace attn {

constexpr float kKvcRescaleLog2 = 8.0f;     // lazy rescale threshold (log2 units), as in the square forward
constexpr float kKvcLn2 = 0.6931471805599453f;

struct KvcParams {
  __nv_bfloat16* o;      // single split: [B*H*Nq][D] bf16 output
  float* lse;            // single split: [B*H*Nq] natural-log LSE
  float* part_o;         // split-KV: [splits][B*H*Nq][D] fp32 partial outputs
  float* part_lse;       // split-KV: [splits][B*H*Nq] partial LSE (natural log)
  const int* kv_lens;    // [B] valid cache length per batch entry, or null (= Nk)
  long long total_rows;  // B*H*Nq
  int nq;                // new query rows per head
  int nk;                // cache capacity (rows of K and V per head)
  int h_kv;              // key/value heads per batch entry
  int rows;              // packed query rows per key/value head = (H / H_kv) * Nq
  int n_rt;              // 128-row packed tiles per key/value head
  int splits;            // key chunks per (kv head, row tile)
  int qbox;              // rows of the query TMA box: min(128, rows rounded up to 8)
  int n_items;           // work items = B*H_kv * n_rt * splits
  float scale_log2;      // scale * log2(e)
};

template <int D>
struct KvcCfg {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kBlockBytes = 128 * 128;          // [128][64] bf16 column block
  static constexpr int kNumBlk = D / 64;
  static constexpr int kSlots = (D == 128) ? 6 : 12;     // K/V ring: three key tiles ahead
  static constexpr int kQBufs = 1;                       // query buffers
  static constexpr int kThreads = 192;
  static constexpr int kWarpMma = 4;
  static constexpr int kWarpLoad = 5;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
  static constexpr uint32_t kColPOff = 64;
  static constexpr uint32_t kColP0 = 384, kColP1 = 448;   // replicated mode: P buffers of their own
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = kQBufs * kTileBytes;
  static constexpr int kOffBar = kOffKV + kSlots * kTileBytes;
  // q_full[2], q_empty[2], kv_full[S], kv_empty[S], s_full[2], p_full[2], pv_done, o_full, o_free, drain
  static constexpr int kNumBars = 4 + 2 * kSlots + 4 + 4;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
};

// One work item = (key/value head, 128-row packed query tile, key chunk).
struct KvcItem {
  int bkv;       // b * H_kv + key/value head
  int split;
  int r0;        // first packed row of the tile
  int r_valid;   // packed rows that exist in the tile
  int L;         // valid cache rows of this batch entry
  int j_lo;      // first key tile of the chunk
  int nkv;       // key tiles in the chunk (0: nothing to read)
};

__device__ __forceinline__ KvcItem kvc_item(const KvcParams& prm, int w, bool causal) {
  KvcItem it;
  it.split = w % prm.splits;
  const int rt = (w / prm.splits) % prm.n_rt;
  it.bkv = w / (prm.splits * prm.n_rt);
  const int b = it.bkv / prm.h_kv;
  it.r0 = 128 * rt;
  it.r_valid = min(128, prm.rows - it.r0);
  int L = prm.kv_lens ? prm.kv_lens[b] : prm.nk;
  it.L = min(max(L, 0), prm.nk);
  // Largest key index any row of the tile may see -> key tiles [0, kv_hi).
  int lim_max = it.L - 1;
  if (causal) {
    const int r1 = it.r0 + it.r_valid - 1;
    const int p_max = (it.r0 / prm.nq == r1 / prm.nq) ? (r1 % prm.nq) : (prm.nq - 1);
    lim_max = min(lim_max, p_max + it.L - prm.nq);
  }
  const int kv_hi = lim_max < 0 ? 0 : (lim_max >> 7) + 1;
  const int chunk = (kv_hi + prm.splits - 1) / prm.splits;
  it.j_lo = min(kv_hi, it.split * chunk);
  it.nkv = min(kv_hi, it.j_lo + chunk) - it.j_lo;
  return it;
}

// Persistent: CTA c takes work items c, c + gridDim.x, ...  Every role walks
// the same item sequence and skips the same empty items, and the barrier
// phases run on across items, so the K/V stream never drains between items:
// the next item's Q and first key tiles load while the current item's last
// tiles are still being consumed, and its first S products run while the
// softmax warps write the current item's output.
template <int D, bool CAUSAL, bool SPLIT, bool REPL>
__global__ void __launch_bounds__(192, 1)
attn_kvcache_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const KvcParams prm) {
  using C = KvcCfg<D>;
  static_assert(!REPL || SPLIT, "the replicated mode always writes partials");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* q_empty = q_full + 2;
  uint64_t* kv_full = q_empty + 2;
  uint64_t* kv_empty = kv_full + C::kSlots;
  uint64_t* s_full = kv_empty + C::kSlots;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* o_full = pv_done + 1;
  uint64_t* o_free = o_full + 1;
  uint64_t* drain = o_free + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(&q_full[t], 1);
      mbar_init(&q_empty[t], 1);
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
    }
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(pv_done, 1);
    mbar_init(o_full, 1);
    mbar_init(o_free, 128);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp < 4 && prm.qbox < (REPL ? 32 : 128)) {
    // Query rows past the packed rows are never loaded: clear them (in every
    // query buffer) so the padding rows of the MMA see zeros.
    const int r = threadIdx.x;
    if ((REPL ? (r & 31) : r) >= prm.qbox) {
      for (int qb = 0; qb < C::kQBufs; ++qb)
        for (int blk = 0; blk < C::kNumBlk; ++blk)
          for (int ch = 0; ch < 8; ++ch)
            st_shared_v4(smem_u32(smem + C::kOffQ + qb * C::kTileBytes + blk * C::kBlockBytes) + r * 128 + ch * 16,
                         0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
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
  const int n_items = prm.n_items;
  if (REPL && warp < 4) {
    // Replicated mode: each lane quarter writes P only in its own 16 packed
    // columns of a P buffer; the other columns of its lanes stay zero.
    uint32_t z[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) z[k] = 0u;
    const uint32_t lb = uint32_t(warp * 32) << 16;
    tmem_st32(tmem + lb + C::kColP0, z);
    tmem_st32(tmem + lb + C::kColP0 + 32, z);
    tmem_st32(tmem + lb + C::kColP1, z);
    tmem_st32(tmem + lb + C::kColP1 + 32, z);
    tmem_st_wait();
  }

  if (warp == C::kWarpLoad) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      int qi = 0, it = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
        const KvcItem I = kvc_item(prm, w, CAUSAL);
        if (I.nkv == 0) continue;
        const int qb = qi % C::kQBufs;
        if (qi >= C::kQBufs && !(ok = mbar_wait(&q_empty[qb], uint32_t((qi / C::kQBufs - 1) & 1), abort_flag))) break;
        constexpr int kCopies = REPL ? 4 : 1;   // replicated mode: the rows in every TMEM lane quarter
        mbar_arrive_expect_tx(&q_full[qb], uint32_t(kCopies * prm.qbox * 128 * C::kNumBlk));
        for (int cp = 0; cp < kCopies; ++cp)
          for (int blk = 0; blk < C::kNumBlk; ++blk)
            tma_load_3d(&tm_q, &q_full[qb],
                        smem + C::kOffQ + qb * C::kTileBytes + blk * C::kBlockBytes + cp * 32 * 128, blk * 64,
                        I.bkv * prm.rows + I.r0, 0);
        ++qi;
        for (int t = 0; t < 2 * I.nkv; ++t) {
          const int slot = it % C::kSlots;
          const int use = it / C::kSlots;
          if (use > 0 && !(ok = mbar_wait(&kv_empty[slot], uint32_t((use - 1) & 1), abort_flag))) break;
          mbar_arrive_expect_tx(&kv_full[slot], C::kTileBytes);
          const CUtensorMap* tm = (t & 1) ? &tm_v : &tm_k;
          for (int blk = 0; blk < C::kNumBlk; ++blk)
            tma_load_3d(tm, &kv_full[slot], smem + C::kOffKV + slot * C::kTileBytes + blk * C::kBlockBytes,
                        blk * 64, 128 * (I.j_lo + (t >> 1)), I.bkv);
          ++it;
        }
      }
      // No copy may still be landing in shared memory when the CTA leaves.
      for (int q = max(0, qi - C::kQBufs); q < qi; ++q)
        mbar_wait(&q_full[q % C::kQBufs], uint32_t((q / C::kQBufs) & 1), abort_flag, false);
      for (int k = max(0, it - C::kSlots); k < it; ++k)
        mbar_wait(&kv_full[k % C::kSlots], uint32_t((k / C::kSlots) & 1), abort_flag, false);
    }
    __syncwarp();
  } else if (warp == C::kWarpMma) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16(128, 128, false, false);
      constexpr uint32_t kIdescPV = idesc_bf16(128, D, false, true);
      const uint32_t sKV = smem_u32(smem + C::kOffKV);
      int qi = 0, it = 0, sc = 0, oi = 0;
      bool ok = true;
      bool issued_any = false;
      for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
        const KvcItem I = kvc_item(prm, w, CAUSAL);
        if (I.nkv == 0) continue;
        const int qb = qi % C::kQBufs;
        const uint32_t sQ = smem_u32(smem + C::kOffQ + qb * C::kTileBytes);
        if (!(ok = mbar_wait(&q_full[qb], uint32_t((qi / C::kQBufs) & 1), abort_flag))) break;
        for (int jj = 0; jj <= I.nkv && ok; ++jj) {
          if (jj < I.nkv) {
            // S of this tile overwrites the buffer of the P two tiles back,
            // whose PV was issued before it.
            const int kit = it + 2 * jj;
            if (!(ok = mbar_wait(&kv_full[kit % C::kSlots], uint32_t((kit / C::kSlots) & 1), abort_flag))) break;
            tc_fence_after();
            const uint32_t b0 = sKV + (kit % C::kSlots) * C::kTileBytes;
            const uint32_t dt = tmem + (((sc + jj) & 1) ? C::kColS1 : C::kColS0);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * C::kBlockBytes + (kk & 3) * 32;
              mma_ss(dt, smem_desc_sw128(sQ + off, 16, 1024), smem_desc_sw128(b0 + off, 16, 1024), kIdescS,
                     kk > 0 ? 1u : 0u);
            }
            issued_any = true;
            mma_commit(&s_full[(sc + jj) & 1]);
            mma_commit(&kv_empty[kit % C::kSlots]);
            if (jj == I.nkv - 1) mma_commit(&q_empty[qb]);
          }
          if (jj > 0) {
            const int pj = jj - 1;
            const int ps = sc + pj;
            if (!(ok = mbar_wait(&p_full[ps & 1], uint32_t((ps >> 1) & 1), abort_flag))) break;
            // The first PV of an item overwrites O: the previous item's
            // epilogue must have read it.
            if (pj == 0 && oi > 0 && !(ok = mbar_wait(o_free, uint32_t((oi - 1) & 1), abort_flag))) break;
            const int vit = it + 2 * pj + 1;
            if (!(ok = mbar_wait(&kv_full[vit % C::kSlots], uint32_t((vit / C::kSlots) & 1), abort_flag))) break;
            tc_fence_after();
            const uint32_t b0 = sKV + (vit % C::kSlots) * C::kTileBytes;
            const uint32_t at = REPL ? tmem + ((ps & 1) ? C::kColP1 : C::kColP0)
                                     : tmem + ((ps & 1) ? C::kColS1 : C::kColS0) + C::kColPOff;
#pragma unroll
            for (int kk = 0; kk < 128 / 16; ++kk)
              mma_ts(tmem + C::kColO, at + kk * 8, smem_desc_sw128(b0 + kk * 2048, C::kBlockBytes, 1024), kIdescPV,
                     (pj > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&kv_empty[vit % C::kSlots]);
            mma_commit(pj == I.nkv - 1 ? o_full : pv_done);
          }
        }
        it += 2 * I.nkv;
        sc += I.nkv;
        ++qi;
        ++oi;
      }
      // Every MMA issued so far must finish before tensor memory is released.
      if (issued_any) {
        mma_commit(drain);
        mbar_wait(drain, 0, abort_flag, false);
      }
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------------- softmax
    // Replicated mode: every lane quarter holds the same packed rows (lane =
    // row) and warp w takes key columns [32w, 32w + 32) of each tile: four
    // independent online softmaxes over disjoint key subsets, merged as four
    // partials per key chunk.
    const int r = REPL ? lane : warp * 32 + lane;   // row inside the tile
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const uint32_t tO = tmem + lane_base + C::kColO;
    const float c = prm.scale_log2;
    int it = 0, sc = 0, pvb = 0, oi = 0;
    bool ok = true;

    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const KvcItem I = kvc_item(prm, w, CAUSAL);
      const int rp = I.r0 + r;                // packed row
      const bool row_ok = r < I.r_valid;
      const bool warp_on = REPL || warp * 32 < I.r_valid;
      int lim = I.L - 1;                      // last key this row sees
      if (CAUSAL) lim = min(lim, rp % prm.nq + I.L - prm.nq);
      float m_ref = -INFINITY;
      float l = 0.f;

      for (int jj = 0; jj < I.nkv; ++jj) {
        const int j = I.j_lo + jj;
        const int sb = (sc + jj) & 1;
        const uint32_t tS = tmem + lane_base + (sb ? C::kColS1 : C::kColS0);
        if (!(ok = mbar_wait_warp(&s_full[sb], uint32_t(((sc + jj) >> 1) & 1), abort_flag))) break;
        tc_fence_after();
        // Cache rows past L inside this key tile: clear their V rows (all 128
        // threads, one key row each) so that P = 0 meets V = 0 there.
        if (128 * j + 128 > I.L && I.L < prm.nk) {
          const int vit = it + 2 * jj + 1;
          if (!(ok = mbar_wait_warp(&kv_full[vit % C::kSlots], uint32_t((vit / C::kSlots) & 1), abort_flag))) break;
          const int kr = warp * 32 + lane;     // key row of the V tile cleared by this thread
          if (128 * j + kr >= I.L) {
            uint8_t* vt = smem + C::kOffKV + (vit % C::kSlots) * C::kTileBytes;
            for (int blk = 0; blk < C::kNumBlk; ++blk)
              for (int ch = 0; ch < 8; ++ch)
                st_shared_v4(smem_u32(vt + blk * C::kBlockBytes) + kr * 128 + ch * 16, 0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
        }
        if (REPL) {
          float s[32];
          {
            uint32_t a[32];
            tmem_ld32(tS + 32 * warp, a);
            tmem_ld_wait(a);
#pragma unroll
            for (int k = 0; k < 32; ++k) s[k] = __uint_as_float(a[k]);
          }
          const int limit = row_ok ? lim - 128 * j - 32 * warp : -1;
          if (__any_sync(0xffffffffu, limit < 31)) {
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if (k > limit) s[k] = -INFINITY;
          }
          float mxp[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) mxp[u] = s[u];
#pragma unroll
          for (int k = 4; k < 32; k += 4)
#pragma unroll
            for (int u = 0; u < 4; ++u) mxp[u] = fmaxf(mxp[u], s[k + u]);
          const float m_tile = fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])) * c;
          float alpha = 1.f;
          bool rescale = false;
          if (m_tile > m_ref + kKvcRescaleLog2) {
            alpha = ex2(m_ref - m_tile);
            m_ref = m_tile;
            rescale = (jj > 0);
          }
          l *= alpha;
          const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
          float sump[4] = {0.f, 0.f, 0.f, 0.f};
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float p0 = ex2(fmaf(s[2 * k], c, neg_m));
            const float p1 = ex2(fmaf(s[2 * k + 1], c, neg_m));
            sump[k & 3] += p0 + p1;
            pk[k] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tmem + lane_base + (sb ? C::kColP1 : C::kColP0) + 16 * warp, pk);
          l += (sump[0] + sump[1]) + (sump[2] + sump[3]);
          if (__any_sync(0xffffffffu, rescale)) {
            if (!(ok = mbar_wait_warp(pv_done, uint32_t((pvb + jj - 1) & 1), abort_flag))) break;
            tc_fence_after();
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
        } else if (warp_on) {
          float s[128];
          {
            uint32_t a[32], bb[32], e[32], f[32];
            tmem_ld32(tS + 0, a);
            tmem_ld32(tS + 32, bb);
            tmem_ld32(tS + 64, e);
            tmem_ld32(tS + 96, f);
            tmem_ld_wait(a);
            reg_fence32(bb);
            reg_fence32(e);
            reg_fence32(f);
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              s[k] = __uint_as_float(a[k]);
              s[32 + k] = __uint_as_float(bb[k]);
              s[64 + k] = __uint_as_float(e[k]);
              s[96 + k] = __uint_as_float(f[k]);
            }
          }
          const int limit = row_ok ? lim - 128 * j : -1;     // padding rows: everything masked
          if (__any_sync(0xffffffffu, limit < 127)) {
#pragma unroll
            for (int k = 0; k < 128; ++k)
              if (k > limit) s[k] = -INFINITY;
          }
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
          if (m_tile > m_ref + kKvcRescaleLog2) {
            alpha = ex2(m_ref - m_tile);
            m_ref = m_tile;
            rescale = (jj > 0);
          }
          l *= alpha;
          const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
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
            tmem_st16(tS + C::kColPOff + 16 * q, pk);
          }
          l += (sump[0] + sump[1]) + (sump[2] + sump[3]);
          if (__any_sync(0xffffffffu, rescale)) {
            // O holds this item's sum through tile jj-2 for sure; wait for PV(jj-1).
            if (!(ok = mbar_wait_warp(pv_done, uint32_t((pvb + jj - 1) & 1), abort_flag))) break;
            tc_fence_after();
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
        }
        tc_fence_before();
        mbar_arrive(&p_full[sb]);
      }
      if (!ok) break;

      // ---------------------------------------------------------- epilogue
      if (I.nkv > 0 && warp_on && !(ok = mbar_wait_warp(o_full, uint32_t(oi & 1), abort_flag))) break;
      tc_fence_after();
      const bool has = l > 0.f;                // false: the row saw no key in this chunk
      const float inv_l = has ? 1.f / l : 0.f;
      const long long row = (long long)I.bkv * prm.rows + rp;   // flat B*H*Nq row
      const int part = REPL ? I.split * 4 + warp : I.split;      // partial written by this thread
      if (warp_on) {
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          if (I.nkv > 0) {
            tmem_ld32(tO + cc * 32, o);
            tmem_ld_wait(o);
          } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = 0u;
          }
          if (row_ok) {
            if (SPLIT) {
              float4* dst = reinterpret_cast<float4*>(prm.part_o + ((long long)part * prm.total_rows + row) * D + cc * 32);
#pragma unroll
              for (int k = 0; k < 8; ++k)
                dst[k] = make_float4(__uint_as_float(o[4 * k]) * inv_l, __uint_as_float(o[4 * k + 1]) * inv_l,
                                     __uint_as_float(o[4 * k + 2]) * inv_l, __uint_as_float(o[4 * k + 3]) * inv_l);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(prm.o + row * D + cc * 32);
#pragma unroll
              for (int k = 0; k < 4; ++k)
                dst[k] = make_uint4(
                    pack_bf16x2(__uint_as_float(o[8 * k + 0]) * inv_l, __uint_as_float(o[8 * k + 1]) * inv_l),
                    pack_bf16x2(__uint_as_float(o[8 * k + 2]) * inv_l, __uint_as_float(o[8 * k + 3]) * inv_l),
                    pack_bf16x2(__uint_as_float(o[8 * k + 4]) * inv_l, __uint_as_float(o[8 * k + 5]) * inv_l),
                    pack_bf16x2(__uint_as_float(o[8 * k + 6]) * inv_l, __uint_as_float(o[8 * k + 7]) * inv_l));
            }
          }
        }
        if (row_ok) {
          const float lse = has ? (m_ref + __log2f(l)) * kKvcLn2 : -INFINITY;
          if (SPLIT)
            prm.part_lse[(long long)part * prm.total_rows + row] = lse;
          else
            prm.lse[row] = lse;
        }
      }
      if (I.nkv > 0) {
        // O has been read: the next item's first PV may overwrite it.
        tc_fence_before();
        mbar_arrive(o_free);
        it += 2 * I.nkv;
        sc += I.nkv;
        pvb += I.nkv - 1;
        ++oi;
      }
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

// Combines the split-KV partials of each row: one 256-thread block per row
// (grid-stride).  The partials' LSEs go through shared memory once; each of
// the 8 warps then accumulates every 8th partial (all its loads independent,
// so they are in flight together), and the warps' sums are added in shared
// memory.  Every partial row is written by the main kernel (zeros where a
// chunk saw no key), so no load is conditional.
constexpr int kKvcMaxParts = 1024;

template <int D>
__global__ void __launch_bounds__(256)
attn_kvcache_merge_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                          __nv_bfloat16* __restrict__ o, float* __restrict__ lse, long long total_rows, int parts) {
  constexpr int kPer = D / 32;                 // columns per lane
  __shared__ float s_lse[kKvcMaxParts];
  __shared__ float s_acc[8][D];
  __shared__ float s_red[8];
  __shared__ float s_sum[8];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Launched as a programmatic dependent of the cache kernel: wait until it
  // has completed and its partials are visible (a no-op otherwise).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (long long row = blockIdx.x; row < total_rows; row += gridDim.x) {
    float mx = -INFINITY;
    for (int s = threadIdx.x; s < parts; s += 256) {
      const float v = part_lse[(long long)s * total_rows + row];
      s_lse[s] = v;
      mx = fmaxf(mx, v);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if (lane == 0) s_red[warp] = mx;
    __syncthreads();
    mx = s_red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) mx = fmaxf(mx, s_red[w]);
    float acc[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) acc[k] = 0.f;
    float sum = 0.f;
    if (mx != -INFINITY) {
#pragma unroll 4
      for (int s = warp; s < parts; s += 8) {
        const float ls = s_lse[s];
        const float w = (ls == -INFINITY) ? 0.f : expf(ls - mx);
        sum += w;
        const float* src = part_o + ((long long)s * total_rows + row) * D + lane * kPer;
        if constexpr (kPer == 4) {
          const float4 t = *reinterpret_cast<const float4*>(src);
          acc[0] = fmaf(w, t.x, acc[0]);
          acc[1] = fmaf(w, t.y, acc[1]);
          acc[2] = fmaf(w, t.z, acc[2]);
          acc[3] = fmaf(w, t.w, acc[3]);
        } else {
          const float2 t = *reinterpret_cast<const float2*>(src);
          acc[0] = fmaf(w, t.x, acc[0]);
          acc[1] = fmaf(w, t.y, acc[1]);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kPer; ++k) s_acc[warp][lane * kPer + k] = acc[k];
    if (lane == 0) s_sum[warp] = sum;
    __syncthreads();
    if (warp == 0) {
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) tot += s_sum[w];
      float out[kPer];
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        float a = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) a += s_acc[w][lane * kPer + k];
        out[k] = a;
      }
      const float inv = tot > 0.f ? 1.f / tot : 0.f;
      __nv_bfloat16* dst = o + row * D + lane * kPer;
      if constexpr (kPer == 4) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(out[0] * inv, out[1] * inv),
                                                    pack_bf16x2(out[2] * inv, out[3] * inv));
      } else {
        *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(out[0] * inv, out[1] * inv);
      }
      if (lane == 0) lse[row] = tot > 0.f ? mx + logf(tot) : -INFINITY;
    }
    __syncthreads();   // shared memory is reused by the next row
  }
}

}  // namespace attn
