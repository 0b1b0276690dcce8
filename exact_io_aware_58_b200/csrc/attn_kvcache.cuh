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
// B200 mapping (one CTA = one 128-row tile of PACKED query rows x one chunk of
// key tiles, 192 threads, one CTA per SM):
//   * The g = H / H_kv query heads that share a key/value head, and their Nq
//     rows each, are packed into the rows of one MMA tile: packed row r is head
//     kvh*g + r / Nq, position r % Nq.  In a BHND tensor these rows are
//     contiguous, so one TMA box loads them and every cached tile is read once
//     per packed tile instead of once per query head.
//   * Split-KV: the key tiles of a (kv head, row tile) are cut into `splits`
//     contiguous chunks, one CTA each, so that a decode batch with few heads
//     still covers all SMs.  Each CTA writes an fp32 partial O (normalised by
//     its own row sum) and its partial LSE; attn_kvcache_merge_kernel combines
//     them (O = sum_s exp(LSE_s - LSE) O_s, LSE = log sum_s exp LSE_s).  With
//     one split the CTA writes the bf16 output directly.
//   * warp 5 TMA producer (Q once, then K_j / V_j through a ring), warp 4 MMA
//     issuer, warps 0-3 softmax with one query row per thread.  S is double
//     buffered in TMEM, so S(j+1) runs on the tensor core while the softmax of
//     tile j runs; P(j) is written back over the upper half of S(j) and read
//     from TMEM by the PV MMA.  Warps whose 32 rows are all padding only keep
//     the barrier protocol.
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
  float scale_log2;      // scale * log2(e)
};

template <int D>
struct KvcCfg {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kBlockBytes = 128 * 128;          // [128][64] bf16 column block
  static constexpr int kNumBlk = D / 64;
  static constexpr int kSlots = (D == 128) ? 4 : 8;      // K/V ring: two key tiles ahead
  static constexpr int kThreads = 192;
  static constexpr int kWarpMma = 4;
  static constexpr int kWarpLoad = 5;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
  static constexpr uint32_t kColPOff = 64;
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = kTileBytes;
  static constexpr int kOffBar = kOffKV + kSlots * kTileBytes;
  // q_full, kv_full[S], kv_empty[S], s_full[2], p_full[2], pv_done, o_full, drain
  static constexpr int kNumBars = 1 + 2 * kSlots + 2 + 2 + 3;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
};

template <int D, bool CAUSAL, bool SPLIT>
__global__ void __launch_bounds__(192, 1)
attn_kvcache_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const KvcParams prm) {
  using C = KvcCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = q_full + 1;
  uint64_t* kv_empty = kv_full + C::kSlots;
  uint64_t* s_full = kv_empty + C::kSlots;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* o_full = pv_done + 1;
  uint64_t* drain = o_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.x % prm.splits;
  const int rt = (blockIdx.x / prm.splits) % prm.n_rt;
  const int bkv = blockIdx.x / (prm.splits * prm.n_rt);      // b * H_kv + kv head
  const int b = bkv / prm.h_kv;
  const int r0 = 128 * rt;                                    // first packed row of the tile
  const int r_valid = min(128, prm.rows - r0);                // packed rows that exist
  int L = prm.kv_lens ? prm.kv_lens[b] : prm.nk;
  L = min(max(L, 0), prm.nk);
  const int shift = L - prm.nq;                               // bottom-right causal offset

  // Largest key index any row of this tile may see -> key tiles [0, kv_hi).
  int lim_max = L - 1;
  if (CAUSAL) {
    const int r1 = r0 + r_valid - 1;
    const int p_max = (r0 / prm.nq == r1 / prm.nq) ? (r1 % prm.nq) : (prm.nq - 1);
    lim_max = min(lim_max, p_max + shift);
  }
  const int kv_hi = lim_max < 0 ? 0 : (lim_max >> 7) + 1;
  const int chunk = (kv_hi + prm.splits - 1) / prm.splits;
  const int j_lo = min(kv_hi, split * chunk);
  const int nkv = min(kv_hi, j_lo + chunk) - j_lo;             // key tiles this CTA visits

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
    }
    mbar_init(pv_done, 1);
    mbar_init(o_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp < 4 && prm.qbox < 128) {
    // Query rows past the packed rows are never loaded: clear them so the
    // padding rows of the MMA see zeros rather than stale shared memory.
    const int r = threadIdx.x;
    if (r >= prm.qbox) {
      for (int blk = 0; blk < C::kNumBlk; ++blk)
        for (int ch = 0; ch < 8; ++ch)
          st_shared_v4(smem_u32(smem + C::kOffQ + blk * C::kBlockBytes) + r * 128 + ch * 16, 0u, 0u, 0u, 0u);
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

  if (warp == C::kWarpLoad) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0 && nkv > 0) {
      mbar_arrive_expect_tx(q_full, uint32_t(prm.qbox * 128 * C::kNumBlk));
      for (int blk = 0; blk < C::kNumBlk; ++blk)
        tma_load_3d(&tm_q, q_full, smem + C::kOffQ + blk * C::kBlockBytes, blk * 64,
                    bkv * prm.rows + r0, 0);
      int issued = 0;
      for (int it = 0; it < 2 * nkv; ++it) {
        const int slot = it % C::kSlots;
        const int use = it / C::kSlots;
        if (use > 0 && !mbar_wait(&kv_empty[slot], (use - 1) & 1, abort_flag)) break;
        const CUtensorMap* tm = (it & 1) ? &tm_v : &tm_k;
        mbar_arrive_expect_tx(&kv_full[slot], C::kTileBytes);
        for (int blk = 0; blk < C::kNumBlk; ++blk)
          tma_load_3d(tm, &kv_full[slot], smem + C::kOffKV + slot * C::kTileBytes + blk * C::kBlockBytes,
                      blk * 64, 128 * (j_lo + (it >> 1)), bkv);
        ++issued;
      }
      // No copy may still be landing in shared memory when the CTA leaves.
      mbar_wait(q_full, 0, abort_flag, false);
      for (int it = max(0, issued - C::kSlots); it < issued; ++it)
        mbar_wait(&kv_full[it % C::kSlots], (it / C::kSlots) & 1, abort_flag, false);
    }
    __syncwarp();
  } else if (warp == C::kWarpMma) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0 && nkv > 0) {
      constexpr uint32_t kIdescS = idesc_bf16(128, 128, false, false);
      constexpr uint32_t kIdescPV = idesc_bf16(128, D, false, true);
      const uint32_t sQ = smem_u32(smem + C::kOffQ);
      const uint32_t sKV = smem_u32(smem + C::kOffKV);
      auto slot_of = [](int item) { return item % C::kSlots; };
      auto parity_of = [](int item) { return uint32_t((item / C::kSlots) & 1); };
      auto issue_s = [&](int jj) {           // S(jj) = Q K_jj^T into buffer jj % 2
        const uint32_t b0 = sKV + slot_of(2 * jj) * C::kTileBytes;
        const uint32_t dt = tmem + ((jj & 1) ? C::kColS1 : C::kColS0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kBlockBytes + (kk & 3) * 32;
          mma_ss(dt, smem_desc_sw128(sQ + off, 16, 1024), smem_desc_sw128(b0 + off, 16, 1024), kIdescS,
                 kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int jj) {          // O += P(jj) V_jj
        const uint32_t b0 = sKV + slot_of(2 * jj + 1) * C::kTileBytes;
        const uint32_t at = tmem + ((jj & 1) ? C::kColS1 : C::kColS0) + C::kColPOff;
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          mma_ts(tmem + C::kColO, at + kk * 8, smem_desc_sw128(b0 + kk * 2048, C::kBlockBytes, 1024), kIdescPV,
                 (jj > 0 || kk > 0) ? 1u : 0u);
      };

      bool ok = mbar_wait(q_full, 0, abort_flag);
      for (int jj = 0; jj <= nkv && ok; ++jj) {
        if (jj < nkv) {
          // S(jj) overwrites the buffer of P(jj-2), whose PV was issued before.
          if (!(ok = mbar_wait(&kv_full[slot_of(2 * jj)], parity_of(2 * jj), abort_flag))) break;
          tc_fence_after();
          issue_s(jj);
          mma_commit(&s_full[jj & 1]);
          mma_commit(&kv_empty[slot_of(2 * jj)]);
        }
        if (jj > 0) {
          const int pj = jj - 1;
          if (!(ok = mbar_wait(&p_full[pj & 1], uint32_t((pj >> 1) & 1), abort_flag))) break;
          if (!(ok = mbar_wait(&kv_full[slot_of(2 * pj + 1)], parity_of(2 * pj + 1), abort_flag))) break;
          tc_fence_after();
          issue_pv(pj);
          mma_commit(&kv_empty[slot_of(2 * pj + 1)]);
          mma_commit(pj == nkv - 1 ? o_full : pv_done);
        }
      }
      // Every MMA issued so far must finish before tensor memory is released.
      mma_commit(drain);
      mbar_wait(drain, 0, abort_flag, false);
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------------- softmax
    const int r = warp * 32 + lane;           // row inside the tile = TMEM lane
    const int rp = r0 + r;                    // packed row
    const bool row_ok = r < r_valid;
    const bool warp_on = warp * 32 < r_valid;
    const int p = rp % prm.nq;
    int lim = L - 1;                          // last key this row sees
    if (CAUSAL) lim = min(lim, p + shift);
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const uint32_t tO = tmem + lane_base + C::kColO;
    const float c = prm.scale_log2;
    float m_ref = -INFINITY;
    float l = 0.f;
    bool ok = true;

    for (int jj = 0; jj < nkv; ++jj) {
      const int j = j_lo + jj;
      const uint32_t tS = tmem + lane_base + ((jj & 1) ? C::kColS1 : C::kColS0);
      if (!(ok = mbar_wait_warp(&s_full[jj & 1], uint32_t((jj >> 1) & 1), abort_flag))) break;
      tc_fence_after();
      // Cache rows past L inside this key tile: clear their V rows (all 128
      // threads, one key row each) so that P = 0 meets V = 0 there.
      if (128 * j + 128 > L && L < prm.nk) {
        const int item = 2 * jj + 1;
        if (!(ok = mbar_wait_warp(&kv_full[item % C::kSlots], uint32_t((item / C::kSlots) & 1), abort_flag))) break;
        if (128 * j + r >= L) {
          uint8_t* vt = smem + C::kOffKV + (item % C::kSlots) * C::kTileBytes;
          for (int blk = 0; blk < C::kNumBlk; ++blk)
            for (int ch = 0; ch < 8; ++ch)
              st_shared_v4(smem_u32(vt + blk * C::kBlockBytes) + r * 128 + ch * 16, 0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
      }
      if (warp_on) {
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
          // O holds the sum through tile jj-2 for sure; wait for PV(jj-1).
          if (!(ok = mbar_wait_warp(pv_done, uint32_t((jj - 1) & 1), abort_flag))) break;
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
      mbar_arrive(&p_full[jj & 1]);
    }

    // ------------------------------------------------------------ epilogue
    if (ok && nkv > 0 && warp_on) ok = mbar_wait_warp(o_full, 0, abort_flag);
    if (ok && warp_on) {
      tc_fence_after();
      const bool has = l > 0.f;                // false: the row saw no key in this chunk
      const float inv_l = has ? 1.f / l : 0.f;
      const long long row = (long long)bkv * prm.rows + rp;   // flat B*H*Nq row
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        if (nkv > 0) {
          tmem_ld32(tO + cc * 32, o);
          tmem_ld_wait(o);
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = 0u;
        }
        if (row_ok) {
          if (SPLIT) {
            float4* dst = reinterpret_cast<float4*>(prm.part_o + ((long long)split * prm.total_rows + row) * D + cc * 32);
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
          prm.part_lse[(long long)split * prm.total_rows + row] = lse;
        else
          prm.lse[row] = lse;
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

// Combines the split-KV partials of each row: one warp per row.
template <int D>
__global__ void __launch_bounds__(256)
attn_kvcache_merge_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                          __nv_bfloat16* __restrict__ o, float* __restrict__ lse, long long total_rows, int splits) {
  constexpr int kPer = D / 32;                 // columns per lane
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < total_rows;
       row += warps) {
    float mx = -INFINITY;
    for (int s = lane; s < splits; s += 32) mx = fmaxf(mx, part_lse[(long long)s * total_rows + row]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float acc[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) acc[k] = 0.f;
    float sum = 0.f;
    if (mx != -INFINITY) {
      for (int s = 0; s < splits; ++s) {
        const float ls = part_lse[(long long)s * total_rows + row];
        if (ls == -INFINITY) continue;         // the chunk saw no key for this row
        const float w = expf(ls - mx);
        sum += w;
        const float* src = part_o + ((long long)s * total_rows + row) * D + lane * kPer;
        if constexpr (kPer == 4) {
          const float4 v = *reinterpret_cast<const float4*>(src);
          acc[0] = fmaf(w, v.x, acc[0]);
          acc[1] = fmaf(w, v.y, acc[1]);
          acc[2] = fmaf(w, v.z, acc[2]);
          acc[3] = fmaf(w, v.w, acc[3]);
        } else {
          const float2 v = *reinterpret_cast<const float2*>(src);
          acc[0] = fmaf(w, v.x, acc[0]);
          acc[1] = fmaf(w, v.y, acc[1]);
        }
      }
    }
    const float inv = sum > 0.f ? 1.f / sum : 0.f;
    __nv_bfloat16* dst = o + row * D + lane * kPer;
    if constexpr (kPer == 4) {
      *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv),
                                                  pack_bf16x2(acc[2] * inv, acc[3] * inv));
    } else {
      *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    }
    if (lane == 0) lse[row] = sum > 0.f ? mx + logf(sum) : -INFINITY;
  }
}

}  // namespace attn
