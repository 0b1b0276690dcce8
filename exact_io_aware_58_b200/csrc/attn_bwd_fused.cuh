// attn_bwd_fused.cuh -- backward by recomputation in one pass over the key
// tiles: dK, dV and dQ from the same recomputed score tiles.
//
// Method ("Attention and KV Compression", section "Recomputation in the
// backward pass"; "FlashAttention -- how 100K-token attention fits in memory",
// section "Training backward"): for a key tile j and a query tile i,
//   S^T = K_j Q_i^T,  P^T = exp2(S^T c - LSE2_i),  dP^T = V_j dO_i^T,
//   dS^T = P^T o (dP^T - D_i),
//   dV_j += P^T dO_i,  dK_j += dS^T Q_i,  dQ_i += dS K_j   (scale applied at the end).
// The two-kernel path (attn_bwd.cuh) recomputes S and dP a second time in a
// query-major dQ kernel; here dQ_i's contribution from key tile j is formed in
// the same CTA from the same dS, so a tile pair costs 5 GEMMs instead of 7.
// Different key tiles add into the same dQ rows, so the partials are summed in
// an fp32 accumulator in the caller's workspace with TMA reduce-add (the
// order of those fp32 additions varies from run to run; a small pass then
// scales the sum and rounds it to bf16).
//
// CTA = one 128-key tile of one key/value head, looping over every (query
// head of its group, query tile); 512 threads in four warpgroups:
//   warps 0-7   compute: thread = key row (TMEM lane), group g = query columns
//               [64g, 64g+64).  P^T is written back into TMEM as bf16 (the A
//               operand of dV += P^T dO_i); dS^T is written once to shared
//               memory as a 128B-swizzled [128 keys][128 queries] bf16 tile,
//               the K-major A operand of dK += dS^T Q_i and, read the other
//               way, the MN-major A operand of dQ_i = dS K_j.
//   warp 8      MMA issuer (one thread); per query tile: dV, S^T of the next
//               tile, dQ, dK, dP^T of the next tile.
//   warp 9      TMA producer (resident K_j, V_j; rings of Q_i, dO_i, and the
//               per-row LSE/D vectors).  Warps 8-11 run on fewer registers
//               (setmaxnreg) so that warps 12-15 can have more.
//   warps 12-15 dQ drain: thread = query row (TMEM lane); each reads its row
//               of the dQ_i partial out of TMEM in one go (which frees the
//               columns for the next dP^T), stages it as fp32 in shared
//               memory, and one thread adds the staged boxes into the
//               accumulator with cp.reduce.async.bulk.tensor (this GPU's
//               memory only), while the next tile pair is computed.
// Tensor memory (512 columns): S^T [0,128), dP^T [128,256), dV, dK (D each).
// At D = 128 TMEM is full, so the dQ partial reuses the dP^T columns once the
// compute warps have read dP^T, and the next dP^T waits for the drain; dQ is
// issued before dK so that this read-out overlaps dK.  At D = 64 the dQ
// partial has columns of its own.
#pragma once

#include "attn_bwd.cuh"

namespace attn {

template <int D>
struct FusedCfg {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kBlockBytes = 128 * 128;             // [128][64] bf16 or [128][32] fp32 column block
  static constexpr int kNumBlk = D / 64;
  static constexpr int kVecBytes = 512;                     // 128 fp32
  static constexpr int kThreads = 512;
  static constexpr int kWarpMma = 8;
  static constexpr int kWarpLoad = 9;                       // warps 10, 11 only complete warpgroup 2
  static constexpr int kWarpDrain0 = 12;                    // warps 12..15 (warpgroup 3): lane quarters 0..3
  // Registers per thread: launched with kRegsLaunch for every warp; warpgroup
  // 2 (MMA, TMA, two idle warps) gives back down to kRegsIssue and warpgroup 3
  // (the drain) takes up to kRegsDrain, enough to hold a whole 128-column
  // partial.  2 * 128 + 72 + 184 = 2 * 128 + 80 + 176 = 4 * 128: the
  // per-SM-subpartition register file is used exactly (each holds one warp of
  // every warpgroup).  The split is the smallest drain share without spills
  // at each D (at D = 128 the drain spills with 176, at D = 64 the issue
  // warpgroup spills with 72).
  static constexpr uint32_t kRegsLaunch = 128;
  static constexpr uint32_t kRegsIssue = (D == 128) ? 72 : 80;
  static constexpr uint32_t kRegsDrain = (D == 128) ? 184 : 176;
  static_assert(2 * kRegsLaunch + kRegsIssue + kRegsDrain == 4 * kRegsLaunch, "register split");
  static constexpr uint32_t kTmemCols = 512;
  // Ring depths.  Q_i is read by S^T(i) (issued right after dV(i-1)) and,
  // last, by dK(i); dO_i by dP^T(i) and, last, by dV(i).  dP^T(i+1) is only
  // issued once dK(i), dQ(i) and the drain's TMEM read have happened, long
  // after dV(i) frees the dO slot, so at D = 128 a single dO slot suffices and
  // its 32 KB go to the dQ staging ring.
  static constexpr int kQS = (D == 128) ? 2 : 4;
  static constexpr int kOS = (D == 128) ? 1 : 3;
  static constexpr int kVS = 2;                             // (LSE2, D) vector ring
  static constexpr int kStageBlocks = 2;                    // staging ring of [128][32] fp32 blocks
  // 32-column chunks of each dQ partial added straight from registers with
  // vector reductions instead of through the staging ring (measured: at
  // D = 64 one of the two chunks that way is faster, at D = 128 none).
  static constexpr int kRedChunks = (D == 64) ? 1 : 0;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQ = 2 * kTileBytes;
  static constexpr int kOffDO = kOffQ + kQS * kTileBytes;
  static constexpr int kOffDS = kOffDO + kOS * kTileBytes;  // dS^T, [128 keys][128 queries] bf16
  static constexpr int kDSBytes = 128 * 128 * 2;
  static constexpr int kOffStage = kOffDS + kDSBytes;
  static constexpr int kOffVec = kOffStage + kStageBlocks * kBlockBytes;
  static constexpr int kOffBar = kOffVec + kVS * 2 * kVecBytes;
  static constexpr int kNumBars = 2 * kQS + 2 * kOS + 2 * kVS + 10;
  static constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 16;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  // TMEM columns
  static constexpr uint32_t kColS = 0;
  static constexpr uint32_t kColDP = 128;
  static constexpr uint32_t kColDV = 256;
  static constexpr uint32_t kColDK = 256 + D;
  static constexpr bool kDqInDP = (D == 128);               // dQ partial over the dP^T columns
  static constexpr uint32_t kColDQ = kDqInDP ? kColDP : 256 + 2 * D;
  static_assert(kColDQ + D <= kTmemCols, "tensor memory budget");
};

// Write 32 fp32 values (one row's 32 consecutive columns) into a
// 128B-swizzled [128 rows][32 fp32] staging block (the TMA SWIZZLE_128B layout).
__device__ __forceinline__ void stage_row32(uint32_t block_u32, int r, const uint32_t* v) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    st_shared_v4(block_u32 + sw128_offset(r, c), v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
}

template <int D, bool CAUSAL, bool SPARSE>
__global__ void __launch_bounds__(512, 1)
attn_bwd_fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                      const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                      const __grid_constant__ CUtensorMap tm_dqacc, const BwdParams prm) {
  using C = FusedCfg<D>;
  constexpr int QS = C::kQS, OS = C::kOS, VS = C::kVS;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;                 // [QS]  Q_i landed
  uint64_t* q_empty = q_full + QS;         // [QS]  dK(i) done: slot free
  uint64_t* o_full = q_empty + QS;         // [OS]  dO_i landed
  uint64_t* o_empty = o_full + OS;         // [OS]  dV(i) done: slot free
  uint64_t* v_full = o_empty + OS;         // [VS]  LSE/D vectors of query tile i landed
  uint64_t* v_empty = v_full + VS;         // [VS]  compute warps done reading them
  uint64_t* kv_full = v_empty + VS;
  uint64_t* s_full = kv_full + 1;          // S^T(i) in TMEM
  uint64_t* dp_full = s_full + 1;          // dP^T(i) in TMEM
  uint64_t* p_full = dp_full + 1;          // P^T(i) written back (256 arrivals)
  uint64_t* ds_full = p_full + 1;          // dS^T(i) in shared memory, dP^T(i) read (256 arrivals)
  uint64_t* dq_full = ds_full + 1;         // dQ partial (i) in TMEM
  uint64_t* dq_free = dq_full + 1;         // drain has read it out of TMEM (128 arrivals)
  uint64_t* ds_read = dq_free + 1;         // the dQ(i) MMA is done reading the dS tile
  uint64_t* acc_full = ds_read + 1;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + C::kNumBars) + 1;
  if (smem_u32(smem) & 1023u) {            // the layout needs a 1024-aligned window
    if (threadIdx.x == 0) atomicOr(&g_attn_status, kStatusLayout);
    return;
  }

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nt = prm.n_tiles;
  const int bkv = blockIdx.x / nt;             // key/value head
  const int jt = blockIdx.x % nt;              // key tile; small jt = most work under the causal mask
  const int n0 = jt * 128;
  const int i_start = CAUSAL ? jt : 0;
  const int n_q = nt - i_start;                // query tiles per query head
  const int n_all = prm.group * n_q;           // every (query head sharing this key/value head, query tile)
  const int bq0 = (bkv / prm.h_kv) * prm.h + (bkv % prm.h_kv) * prm.group;   // first such query head
  const uint8_t* mcol = SPARSE ? prm.mask + jt : nullptr;
  auto sel = [&](int L) -> bool {
    return mcol[(size_t(bq0 + L / n_q) * nt + size_t(i_start + L % n_q)) * nt] != 0;
  };
  const int n_it = SPARSE ? sel_count(sel, n_all) : n_all;

  if (threadIdx.x == 0) {
    for (int s = 0; s < QS; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    for (int s = 0; s < OS; ++s) {
      mbar_init(&o_full[s], 1);
      mbar_init(&o_empty[s], 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 256);
    }
    mbar_init(kv_full, 1);
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 256);
    mbar_init(ds_full, 256);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 128);
    mbar_init(ds_read, 1);
    mbar_init(acc_full, 1);
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
    tma_prefetch_desc(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp >= C::kWarpMma && warp < C::kWarpDrain0) {
   // warpgroup 2: one TMA thread, one MMA thread, two idle warps
   regs_dec<C::kRegsIssue>();
   if (warp == C::kWarpLoad) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      if (n_it > 0) {
        mbar_arrive_expect_tx(kv_full, 2 * C::kTileBytes);
        for (int b = 0; b < C::kNumBlk; ++b) {
          tma_load_3d(&tm_k, kv_full, smem + C::kOffK + b * C::kBlockBytes, b * 64, n0, bkv);
          tma_load_3d(&tm_v, kv_full, smem + C::kOffV + b * C::kBlockBytes, b * 64, n0, bkv);
        }
      }
      int q_issued = 0, o_issued = 0, v_issued = 0;
      int Lsel = SPARSE ? sel_next(sel, -1, n_all) : 0;
      for (int it = 0; it < n_it; ++it) {
        const int L = SPARSE ? Lsel : it;
        if (SPARSE) Lsel = sel_next(sel, Lsel, n_all);
        const int qi = i_start + L % n_q;
        const int bq = bq0 + L / n_q;
        {   // LSE*log2(e) and D of query tile i
          const int slot = it % VS, use = it / VS;
          if (use > 0 && !mbar_wait(&v_empty[slot], (use - 1) & 1, abort_flag)) break;
          mbar_arrive_expect_tx(&v_full[slot], 2 * C::kVecBytes);
          const size_t voff = size_t(bq) * size_t(prm.npad) + size_t(qi) * 128;
          uint8_t* vec = smem + C::kOffVec + slot * 2 * C::kVecBytes;
          bulk_load(vec, prm.ws_lse2 + voff, C::kVecBytes, &v_full[slot]);
          bulk_load(vec + C::kVecBytes, prm.ws_d + voff, C::kVecBytes, &v_full[slot]);
          ++v_issued;
        }
        {   // Q_i
          const int slot = it % QS, use = it / QS;
          if (use > 0 && !mbar_wait(&q_empty[slot], (use - 1) & 1, abort_flag)) break;
          mbar_arrive_expect_tx(&q_full[slot], C::kTileBytes);
          for (int b = 0; b < C::kNumBlk; ++b)
            tma_load_3d(&tm_q, &q_full[slot], smem + C::kOffQ + slot * C::kTileBytes + b * C::kBlockBytes, b * 64,
                        qi * 128, bq);
          ++q_issued;
        }
        {   // dO_i
          const int slot = it % OS, use = it / OS;
          if (use > 0 && !mbar_wait(&o_empty[slot], (use - 1) & 1, abort_flag)) break;
          mbar_arrive_expect_tx(&o_full[slot], C::kTileBytes);
          for (int b = 0; b < C::kNumBlk; ++b)
            tma_load_3d(&tm_do, &o_full[slot], smem + C::kOffDO + slot * C::kTileBytes + b * C::kBlockBytes, b * 64,
                        qi * 128, bq);
          ++o_issued;
        }
      }
      // No copy may still be landing in shared memory when the CTA leaves.
      if (n_it > 0) mbar_wait(kv_full, 0, abort_flag, false);
      for (int it = max(0, q_issued - QS); it < q_issued; ++it)
        mbar_wait(&q_full[it % QS], (it / QS) & 1, abort_flag, false);
      for (int it = max(0, o_issued - OS); it < o_issued; ++it)
        mbar_wait(&o_full[it % OS], (it / OS) & 1, abort_flag, false);
      for (int it = max(0, v_issued - VS); it < v_issued; ++it)
        mbar_wait(&v_full[it % VS], (it / VS) & 1, abort_flag, false);
    }
    __syncwarp();
  } else if (warp == C::kWarpMma) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t kIdescT = idesc_bf16(128, 128, false, false);   // S^T, dP^T (both K-major)
      constexpr uint32_t kIdescDV = idesc_bf16(128, D, false, true);     // A = P^T (TMEM), B = dO_i MN-major
      constexpr uint32_t kIdescDK = idesc_bf16(128, D, false, true);     // A = dS^T K-major, B = Q_i MN-major
      constexpr uint32_t kIdescDQ = idesc_bf16(128, D, true, true);      // A = dS MN-major, B = K_j MN-major
      const uint32_t sK = smem_u32(smem + C::kOffK);
      const uint32_t sV = smem_u32(smem + C::kOffV);
      const uint32_t sDS = smem_u32(smem + C::kOffDS);
      auto q_tile = [&](int it) { return smem_u32(smem + C::kOffQ + (it % QS) * C::kTileBytes); };
      auto o_tile = [&](int it) { return smem_u32(smem + C::kOffDO + (it % OS) * C::kTileBytes); };
      auto issue_t = [&](uint32_t dcol, uint32_t a0, uint32_t b0) {   // [128 x 128] = A B^T, K = D
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kBlockBytes + (kk & 3) * 32;
          mma_ss(tmem + dcol, smem_desc_sw128(a0 + off, 16, 1024), smem_desc_sw128(b0 + off, 16, 1024), kIdescT,
                 kk > 0 ? 1u : 0u);
        }
      };
      auto issue_dv = [&](int it) {   // dV += P^T dO_i, K = 128 queries
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + C::kColDV, tmem + C::kColS + 64 * (kk >> 2) + (kk & 3) * 8,
                 smem_desc_sw128(o_tile(it) + kk * 2048, C::kBlockBytes, 1024), kIdescDV, (it > 0 || kk > 0) ? 1u : 0u);
      };
      auto issue_dk = [&](int it) {   // dK += dS^T Q_i, K = 128 queries; A = dS^T K-major from the dS tile
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * C::kBlockBytes + (kk & 3) * 32;
          mma_ss(tmem + C::kColDK, smem_desc_sw128(sDS + off, 16, 1024),
                 smem_desc_sw128(q_tile(it) + kk * 2048, C::kBlockBytes, 1024), kIdescDK, (it > 0 || kk > 0) ? 1u : 0u);
        }
      };
      auto issue_dq = [&]() {         // dQ_i partial = dS K_j, K = 128 keys
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + C::kColDQ, smem_desc_sw128(sDS + kk * 2048, C::kBlockBytes, 1024),
                 smem_desc_sw128(sK + kk * 2048, C::kBlockBytes, 1024), kIdescDQ, kk > 0 ? 1u : 0u);
      };
      auto wait_q = [&](int it) { return mbar_wait(&q_full[it % QS], (it / QS) & 1, abort_flag); };
      auto wait_o = [&](int it) { return mbar_wait(&o_full[it % OS], (it / OS) & 1, abort_flag); };

      bool ok = n_it > 0 && mbar_wait(kv_full, 0, abort_flag) && wait_q(0) && wait_o(0);
      if (ok) {
        tc_fence_after();
        issue_t(C::kColS, sK, q_tile(0));     // S^T = K_j Q_i^T
        mma_commit(s_full);
        issue_t(C::kColDP, sV, o_tile(0));    // dP^T = V_j dO_i^T
        mma_commit(dp_full);
      }
      for (int it = 0; it < n_it && ok; ++it) {
        const bool more = it + 1 < n_it;
        if (!(ok = mbar_wait(p_full, it & 1, abort_flag))) break;
        tc_fence_after();
        issue_dv(it);
        mma_commit(&o_empty[it % OS]);        // dO_i read for the last time
        if (more) {
          if (!(ok = wait_q(it + 1))) break;
          tc_fence_after();
          issue_t(C::kColS, sK, q_tile(it + 1));
          mma_commit(s_full);
        }
        if (!(ok = mbar_wait(ds_full, it & 1, abort_flag))) break;
        // D = 64: the dQ columns are free once the drain has read the previous partial
        if (!C::kDqInDP && it > 0 && !(ok = mbar_wait(dq_free, (it - 1) & 1, abort_flag))) break;
        tc_fence_after();
        // dQ first, so that the drain reads the partial out of TMEM while dK runs
        issue_dq();
        mma_commit(dq_full);
        issue_dk(it);
        mma_commit(&q_empty[it % QS]);        // Q_i read for the last time
        mma_commit(ds_read);                  // the dS tile is no longer read
        if (more) {
          // D = 128: dP^T shares its columns with the dQ partial
          if (C::kDqInDP && !(ok = mbar_wait(dq_free, it & 1, abort_flag))) break;
          if (!(ok = wait_o(it + 1))) break;
          tc_fence_after();
          issue_t(C::kColDP, sV, o_tile(it + 1));
          mma_commit(dp_full);
        }
      }
      if (ok) mma_commit(acc_full);
      mma_commit(drain);
      mbar_wait(drain, 0, abort_flag, false);
    }
    __syncwarp();
   }
  } else if (warp < C::kWarpMma) {
    // -------------------------------------------------------------- compute
    // thread = key row r (TMEM lane), group g = query columns [64g, 64g+64)
    const int g = warp >> 2;
    const int qw = warp & 3;
    const int r = qw * 32 + lane;
    const int key = n0 + r;
    const uint32_t lane_base = uint32_t(qw * 32) << 16;
    const uint32_t tA = tmem + lane_base + C::kColS + 64 * g;
    const uint32_t tB = tmem + lane_base + C::kColDP + 64 * g;
    const uint32_t sDSg = smem_u32(smem + C::kOffDS) + g * C::kBlockBytes;
    const float c = prm.scale_log2;
    bool ok = true;
    int Lsel = SPARSE ? sel_next(sel, -1, n_all) : 0;
    for (int it = 0; it < n_it; ++it) {
      const int L = SPARSE ? Lsel : it;
      if (SPARSE) Lsel = sel_next(sel, Lsel, n_all);
      const int qi = i_start + L % n_q;
      const float* vec = reinterpret_cast<const float*>(smem + C::kOffVec + (it % VS) * 2 * C::kVecBytes);
      if (!(ok = mbar_wait_warp(&v_full[it % VS], (it / VS) & 1, abort_flag))) break;
      if (!(ok = mbar_wait_warp(s_full, it & 1, abort_flag))) break;
      tc_fence_after();
      float p[64];
      tmem_ld64f(tA, p);
      const float4* l4 = reinterpret_cast<const float4*>(vec + 64 * g);
#pragma unroll
      for (int k4 = 0; k4 < 16; ++k4) {
        const float4 lv = l4[k4];
        p[4 * k4 + 0] = ex2(fmaf(p[4 * k4 + 0], c, -lv.x));
        p[4 * k4 + 1] = ex2(fmaf(p[4 * k4 + 1], c, -lv.y));
        p[4 * k4 + 2] = ex2(fmaf(p[4 * k4 + 2], c, -lv.z));
        p[4 * k4 + 3] = ex2(fmaf(p[4 * k4 + 3], c, -lv.w));
      }
      if (CAUSAL && qi == jt) {
        // query (qi*128 + 64g + k) sees this key only if query >= key
        const int lim = key - (qi * 128 + 64 * g);   // mask k < lim
#pragma unroll
        for (int k = 0; k < 64; ++k)
          if (k < lim) p[k] = 0.f;
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) pk[k] = pack_bf16x2(p[2 * k], p[2 * k + 1]);
        tmem_st32(tA, pk);   // P^T over the first 32 of this group's 64 S^T columns
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full);

      if (!(ok = mbar_wait_warp(dp_full, it & 1, abort_flag))) break;
      // the dQ MMA of the previous iteration has read the dS tile
      if (it > 0 && !(ok = mbar_wait_warp(ds_read, (it - 1) & 1, abort_flag))) break;
      tc_fence_after();
      const float4* d4 = reinterpret_cast<const float4*>(vec + 128 + 64 * g);
      // dS^T for 32 query columns at a time into the shared-memory dS tile,
      // the A operand of both dQ (read MN-major) and dK (read K-major).
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t dpr[32];
        tmem_ld32(tB + 32 * h, dpr);
        tmem_ld_wait(dpr);
        uint32_t pk[16];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int k = 32 * h + 8 * ch + 4 * u;            // query column inside the group
            const float4 dv = d4[k >> 2];
            const float s0 = p[k + 0] * (__uint_as_float(dpr[8 * ch + 4 * u + 0]) - dv.x);
            const float s1 = p[k + 1] * (__uint_as_float(dpr[8 * ch + 4 * u + 1]) - dv.y);
            const float s2 = p[k + 2] * (__uint_as_float(dpr[8 * ch + 4 * u + 2]) - dv.z);
            const float s3 = p[k + 3] * (__uint_as_float(dpr[8 * ch + 4 * u + 3]) - dv.w);
            pk[4 * ch + 2 * u] = pack_bf16x2(s0, s1);
            pk[4 * ch + 2 * u + 1] = pack_bf16x2(s2, s3);
          }
          st_shared_v4(sDSg + sw128_offset(r, 4 * h + ch), pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        }
      }
      mbar_arrive(&v_empty[it % VS]);   // this thread is done with the LSE/D vectors
      tc_fence_before();                // dP^T has been read (its columns may be overwritten)
      fence_proxy_async_smem();         // dS^T visible to the tensor core (shared memory)
      mbar_arrive(ds_full);
    }
    // epilogue: group 0 writes dV (staged in the V_j slot), group 1 writes dK (in the K_j slot)
    if (ok && n_it > 0) ok = mbar_wait_warp(acc_full, 0, abort_flag);
    uint8_t* stage = smem + (g == 0 ? C::kOffV : C::kOffK);
    if (ok) {
      tc_fence_after();
      if (n_it > 0)
        tmem_acc_to_smem<D>(tmem + lane_base + (g == 0 ? C::kColDV : C::kColDK), smem_u32(stage), r, 0, D / 32,
                            g == 0 ? 1.f : prm.scale);
      else
        zero_tile_rows<D>(smem_u32(stage), r, 0, D / 32);   // no query tile selected this key tile
    }
    fence_proxy_async_smem();
    named_barrier_sync(1 + g, 128);
    if (qw == 0 && lane == 0 && *abort_flag == 0) {
      const CUtensorMap* tm = (g == 0) ? &tm_dv : &tm_dk;
      for (int b = 0; b < C::kNumBlk; ++b) tma_store_3d(tm, stage + b * C::kBlockBytes, b * 64, n0, bkv);
      bulk_commit_group();
      bulk_wait_group_read0();
    }
  } else {
    // ------------------------------------------------------------ dQ drain
    regs_inc<C::kRegsDrain>();
    // thread = query row r of the partial (TMEM lane); warp w reads lane quarter w % 4.
    // The whole partial is read out of TMEM at once (four loads, one wait), so
    // its columns are released after a single round trip; then each 32-column
    // chunk is staged as a [128][32] fp32 block in a ring of two and added
    // into the accumulator by one TMA reduce.  A block is rewritten only after
    // the reduce that used it two chunks before has read it, so the reduces
    // stream out while the next chunks are staged and while the next tile
    // pair is computed.
    constexpr int NC = D / 32;                // 32-column chunks per partial
    const int qd = warp & 3;
    const int r = qd * 32 + lane;
    const uint32_t tQ = tmem + (uint32_t(qd * 32) << 16) + C::kColDQ;
    const bool leader = (warp == C::kWarpDrain0 && lane == 0);
    uint8_t* stage = smem + C::kOffStage;
    // The four drain warps meet at named barriers inside the loop, so a failed
    // wait must not make one warp leave alone: the first barrier of every
    // iteration ANDs the warps' status and they all stop together.
    int Lsel = SPARSE ? sel_next(sel, -1, n_all) : 0;
    uint32_t pos = 0;                         // chunks staged so far: position in the block ring
    for (int it = 0; it < n_it; ++it) {
      const int L = SPARSE ? Lsel : it;
      if (SPARSE) Lsel = sel_next(sel, Lsel, n_all);
      const int qrow = (i_start + L % n_q) * 128;
      const int bq = bq0 + L / n_q;
      const bool ok = mbar_wait_warp(dq_full, it & 1, abort_flag);
      uint32_t a[NC][32];
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < NC; ++c) tmem_ld32(tQ + 32 * c, a[c]);
        tmem_ld_wait(a[0]);
#pragma unroll
        for (int c = 1; c < NC; ++c) reg_fence32(a[c]);
        tc_fence_before();
        mbar_arrive(dq_free);                 // the partial's TMEM columns are free
      }
      // the last kRed chunks go straight from registers with vector reductions
      constexpr int kRed = C::kRedChunks;
      static_assert(kRed < NC, "at least one chunk goes through the staging ring");
      if (ok && qrow + r < prm.n) {
        float* dst = prm.dq_acc + (size_t(bq) * size_t(prm.npad) + size_t(qrow + r)) * D;
#pragma unroll
        for (int c = NC - kRed; c < NC; ++c)
#pragma unroll
          for (int m = 0; m < 8; ++m)
            red_add_v4(dst + 32 * c + 4 * m, a[c][4 * m], a[c][4 * m + 1], a[c][4 * m + 2], a[c][4 * m + 3]);
      }
      bool go = true;
#pragma unroll
      for (int c = 0; c < NC - kRed; ++c, ++pos) {   // chunk c goes through staging block pos % 2
        // the block was last read by the reduce issued two chunks ago
        if (leader) bulk_wait_group_read1();
        if (c == 0) {
          if (!(go = named_barrier_and(3, 128, ok))) break;
        } else {
          named_barrier_sync(3, 128);
        }
        uint8_t* blk = stage + (pos & 1) * C::kBlockBytes;
        stage_row32(smem_u32(blk), r, a[c]);
        fence_proxy_async_smem();
        named_barrier_sync(3, 128);
        if (leader) {
          tma_reduce_add_3d(&tm_dqacc, blk, 32 * c, qrow, bq);
          bulk_commit_group();
        }
      }
      if (!go) break;
    }
    if (leader) bulk_wait_group0();   // every reduce has completed
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::kWarpMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// dQ = scale * (fp32 accumulator), rounded to bf16; rows i < N of every head.
template <int D>
__global__ void __launch_bounds__(256)
attn_bwd_dq_convert_kernel(const float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dq, int n, int npad,
                           long long rows, float scale) {
  constexpr int kTpr = D / 8;                 // threads per row, 8 elements each
  constexpr int kRowsPerBlock = 256 / kTpr;
  const int sub = threadIdx.x % kTpr;
  const long long stride = (long long)gridDim.x * kRowsPerBlock;
  for (long long row = (long long)blockIdx.x * kRowsPerBlock + threadIdx.x / kTpr; row < rows; row += stride) {
    const long long bh = row / n;
    const int i = int(row - bh * n);
    const float4* src = reinterpret_cast<const float4*>(dq_acc + (size_t(bh) * size_t(npad) + size_t(i)) * D + sub * 8);
    const float4 x = src[0], y = src[1];
    uint4 o;
    o.x = pack_bf16x2(x.x * scale, x.y * scale);
    o.y = pack_bf16x2(x.z * scale, x.w * scale);
    o.z = pack_bf16x2(y.x * scale, y.y * scale);
    o.w = pack_bf16x2(y.z * scale, y.w * scale);
    *reinterpret_cast<uint4*>(dq + size_t(row) * D + sub * 8) = o;
  }
}

}  // namespace attn
