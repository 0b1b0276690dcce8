// attn_bwd.cuh -- backward by recomputation.
//
// Method ("Attention and KV Compression", section "Recomputation in the
// backward pass"; "FlashAttention -- how 100K-token attention fits in memory",
// section "Training backward"): the probabilities are not stored by the
// forward; each score tile is recomputed from Q, K and the saved per-row LSE,
//   P = exp(scale * Q K^T - LSE),  dP = dO V^T,  dS = P o (dP - D),
//   D_i = sum_k dO_ik O_ik,  dV = P^T dO,  dQ = scale dS K,  dK = scale dS^T Q.
//
// Three kernels:
//   bwd_pre   per row: D_i and LSE_i*log2(e) into the workspace (HBM-bound).
//   bwd_dkdv  one CTA per 128-key tile j: Q_i / dO_i tiles stream past a
//             resident K_j, V_j; S^T and dP^T accumulate in TMEM, P^T and dS^T
//             are written back into TMEM (bf16) and used as the A operand of
//             dV += P^T dO_i and dK += dS^T Q_i (4 MMAs per tile pair).
//   bwd_dq    one CTA per 128-query tile i: K_j / V_j tiles stream past a
//             resident Q_i, dO_i; S and dP are recomputed, dS goes back to
//             TMEM and feeds dQ += dS K_j (3 MMAs per tile pair).
// Q_i, dO_i (and K_j) serve both as K-major operands (for S^T, dP^T) and as
// MN-major operands (for dK, dV, dQ): one swizzled shared-memory copy, two
// descriptors.
#pragma once

#include "sm100.cuh"

namespace attn {

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// bwd_pre: D_i = sum_k dO_ik O_ik, lse2_i = LSE_i * log2(e); padding rows
// (i >= N, up to Npad) get D = 0 and lse2 = +inf so that recomputed
// probabilities of padding queries are exactly 0.  ZERO (fused backward
// only): also clears row i < N of the fp32 dQ accumulator [B*H][Npad][D].
// ---------------------------------------------------------------------------
template <int D, bool ZERO = false>
__global__ void __launch_bounds__(256)
attn_bwd_pre_kernel(const __nv_bfloat16* __restrict__ O, const __nv_bfloat16* __restrict__ dO,
                    const float* __restrict__ lse, float* __restrict__ ws_lse2, float* __restrict__ ws_d,
                    int n, int npad, long long rows_pad, float* __restrict__ dq_acc = nullptr) {
  constexpr int kTpr = D / 8;                 // threads per row, 16 bytes each
  constexpr int kRowsPerBlock = 256 / kTpr;
  const int sub = threadIdx.x % kTpr;
  const long long stride = (long long)gridDim.x * kRowsPerBlock;
  for (long long row = (long long)blockIdx.x * kRowsPerBlock + threadIdx.x / kTpr; row < rows_pad; row += stride) {
    const long long bh = row / npad;
    const int i = int(row - bh * npad);
    float acc = 0.f;
    if (i < n) {
      const size_t off = (size_t(bh) * size_t(n) + size_t(i)) * D + sub * 8;
      const uint4 a = *reinterpret_cast<const uint4*>(O + off);
      const uint4 b = *reinterpret_cast<const uint4*>(dO + off);
      const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 fa = __bfloat1622float2(pa[k]);
        const float2 fb = __bfloat1622float2(pb[k]);
        acc = fmaf(fa.x, fb.x, acc);
        acc = fmaf(fa.y, fb.y, acc);
      }
      if (ZERO) {
        float4* z = reinterpret_cast<float4*>(dq_acc + (size_t(bh) * size_t(npad) + size_t(i)) * D + sub * 8);
        z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int o = kTpr / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o, kTpr);
    if (sub == 0) {
      ws_d[row] = (i < n) ? acc : 0.f;
      // padding rows, and rows that see no key (LSE = -inf, block-sparse), get
      // +inf so that every recomputed probability of theirs is exactly 0
      const float lv = (i < n) ? lse[size_t(bh) * size_t(n) + size_t(i)] : -INFINITY;
      ws_lse2[row] = (lv == -INFINITY) ? INFINITY : lv * kLog2e;
    }
  }
}

struct BwdParams {
  const float* ws_lse2;   // [B*H][npad]
  const float* ws_d;      // [B*H][npad]
  int n;
  int npad;
  int n_tiles;            // ceil(N / 128)
  int h;                  // query heads per batch
  int h_kv;               // key/value heads per batch (h % h_kv == 0)
  int group;              // h / h_kv
  float scale;
  float scale_log2;
  const uint8_t* mask;    // block-sparse only: [B*H][nt][nt], 1 = query tile attends key tile
  float* dq_acc;          // fused backward only: [B*H][npad][D] fp32 accumulator of dQ / scale
};

// Selection over a linear range [0, hi): sel(L) != 0 marks the visited items.
// Every role scans the same bytes, so they all walk the same sequence.
template <class F>
__device__ __forceinline__ int sel_next(const F& sel, int L, int hi) {
  for (++L; L < hi; ++L)
    if (sel(L)) return L;
  return hi;
}
template <class F>
__device__ __forceinline__ int sel_count(const F& sel, int hi) {
  int c = 0;
  for (int L = 0; L < hi; ++L) c += sel(L) ? 1 : 0;
  return c;
}

template <int D>
struct BwdCfg {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kBlockBytes = 128 * 128;
  static constexpr int kNumBlk = D / 64;
  static constexpr int kVecBytes = 512;                    // 128 fp32
  static constexpr int kThreads = 320;
  static constexpr int kWarpMma = 8;
  static constexpr int kWarpLoad = 9;
  static constexpr uint32_t kTmemCols = 512;
  // Ring depths.  The operand read last in an iteration (Q_i in dK/dV, K_j in
  // dQ) gets the deeper ring, so its refill has more than one iteration to land.
  static constexpr int kDeep = (D == 128) ? 3 : 4;
  static constexpr int kShallow = (D == 128) ? 2 : 4;
  // dK/dV kernel: resident K_j, V_j; ring of Q_i (+ its LSE/D vectors); ring of dO_i.
  static constexpr int kKV_OffK = 0;
  static constexpr int kKV_OffV = kTileBytes;
  static constexpr int kKV_OffQ = 2 * kTileBytes;
  static constexpr int kKV_OffDO = kKV_OffQ + kDeep * kTileBytes;
  static constexpr int kVecSlots = 2;                                      // ring of (lse2[128], D[128])
  static constexpr int kKV_OffVec = kKV_OffDO + kShallow * kTileBytes;
  static constexpr int kKV_OffBar = kKV_OffVec + kVecSlots * 2 * kVecBytes;
  // dQ kernel: resident Q_i, dO_i, LSE/D vectors; ring of K_j; ring of V_j.
  static constexpr int kQ_OffQ = 0;
  static constexpr int kQ_OffDO = kTileBytes;
  static constexpr int kQ_OffK = 2 * kTileBytes;
  static constexpr int kQ_OffV = kQ_OffK + kDeep * kTileBytes;
  static constexpr int kQ_OffVec = kQ_OffV + kShallow * kTileBytes;
  static constexpr int kQ_OffBar = kQ_OffVec + 2 * kVecBytes;
  static constexpr int kNumBars = 2 * kDeep + 2 * kShallow + 2 * kVecSlots + 8;
  // Every tile offset above is a multiple of 1024 (the 128B-swizzle atom).
  // The dynamic shared memory window starts 1024-byte aligned (checked at run
  // time), so no alignment slack is reserved.
  static constexpr int kKV_SmemBytes = kKV_OffBar + kNumBars * 8 + 16;
  static constexpr int kQ_SmemBytes = kQ_OffBar + kNumBars * 8 + 16;
  static_assert(kKV_SmemBytes <= 232448 && kQ_SmemBytes <= 232448, "shared memory budget");
  // TMEM columns
  static constexpr uint32_t kColA = 0;        // S^T (dkdv) / S (dq)
  static constexpr uint32_t kColB = 128;      // dP^T (dkdv) / dP (dq)
  static constexpr uint32_t kColAcc0 = 256;   // dV (dkdv) / dQ (dq)
  static constexpr uint32_t kColAcc1 = 256 + D;   // dK (dkdv)
};

// Store a [128 x D] fp32 accumulator held in TMEM (this thread's lane = row r,
// columns [c_lo, c_hi) in 32-column chunks) as bf16 into a 128B-swizzled
// shared-memory tile, multiplied by `mul`.
template <int D>
__device__ __forceinline__ void tmem_acc_to_smem(uint32_t t_acc_lane, uint32_t stage_u32, int r, int chunk_lo,
                                                 int chunk_hi, float mul) {
#pragma unroll 1
  for (int cc = chunk_lo; cc < chunk_hi; ++cc) {
    uint32_t o[32];
    tmem_ld32(t_acc_lane + cc * 32, o);
    tmem_ld_wait(o);
    const uint32_t blk = cc >> 1;
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      const uint32_t w0 = pack_bf16x2(__uint_as_float(o[8 * ch + 0]) * mul, __uint_as_float(o[8 * ch + 1]) * mul);
      const uint32_t w1 = pack_bf16x2(__uint_as_float(o[8 * ch + 2]) * mul, __uint_as_float(o[8 * ch + 3]) * mul);
      const uint32_t w2 = pack_bf16x2(__uint_as_float(o[8 * ch + 4]) * mul, __uint_as_float(o[8 * ch + 5]) * mul);
      const uint32_t w3 = pack_bf16x2(__uint_as_float(o[8 * ch + 6]) * mul, __uint_as_float(o[8 * ch + 7]) * mul);
      const uint32_t chunk = (cc & 1) * 4 + ch;
      st_shared_v4(stage_u32 + blk * (128 * 128) + sw128_offset(r, chunk), w0, w1, w2, w3);
    }
  }
}

// Zero row r, 32-column chunks [chunk_lo, chunk_hi), of a 128B-swizzled bf16 tile.
template <int D>
__device__ __forceinline__ void zero_tile_rows(uint32_t stage_u32, int r, int chunk_lo, int chunk_hi) {
  for (int cc = chunk_lo; cc < chunk_hi; ++cc)
#pragma unroll
    for (int ch = 0; ch < 4; ++ch)
      st_shared_v4(stage_u32 + (cc >> 1) * (128 * 128) + sw128_offset(r, (cc & 1) * 4 + ch), 0u, 0u, 0u, 0u);
}

// Load 64 fp32 columns [c0, c0+64) of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld64f(uint32_t taddr, float (&v)[64]) {
  uint32_t a[32], b[32];
  tmem_ld32(taddr, a);
  tmem_ld32(taddr + 32, b);
  tmem_ld_wait(a);
  reg_fence32(b);
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    v[k] = __uint_as_float(a[k]);
    v[32 + k] = __uint_as_float(b[k]);
  }
}

// ---------------------------------------------------------------------------
// dK, dV
// ---------------------------------------------------------------------------
template <int D, bool CAUSAL, bool SPARSE>
__global__ void __launch_bounds__(320, 1)
attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                     const BwdParams prm) {
  using C = BwdCfg<D>;
  constexpr int QS = C::kDeep, OS = C::kShallow, VS = C::kVecSlots;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kKV_OffBar);
  uint64_t* q_full = bars;                 // [QS]  Q_i landed
  uint64_t* q_empty = q_full + QS;         // [QS]  dK(i) done: slot free
  uint64_t* o_full = q_empty + QS;         // [OS]  dO_i landed
  uint64_t* o_empty = o_full + OS;         // [OS]  dV(i) done: slot free
  uint64_t* v_full = o_empty + OS;         // [VS]  LSE/D vectors of Q tile i landed
  uint64_t* v_empty = v_full + VS;         // [VS]  compute warps done reading them
  uint64_t* kv_full = v_empty + VS;
  uint64_t* s_full = kv_full + 1;
  uint64_t* dp_full = s_full + 1;
  uint64_t* p_full = dp_full + 1;
  uint64_t* ds_full = p_full + 1;
  uint64_t* acc_full = ds_full + 1;
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
  // Block-sparse: item L = (query head bq0 + L / n_q, query tile i_start + L % n_q) is visited
  // only if that query tile selected this key tile.
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
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == C::kWarpMma) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::kWarpLoad) {
    if (lane == 0) {
      // A key tile that no query tile selected (block-sparse) loads nothing:
      // its K/V slots are the staging area of the zero dK/dV it writes.
      if (n_it > 0) {
        mbar_arrive_expect_tx(kv_full, 2 * C::kTileBytes);
        for (int b = 0; b < C::kNumBlk; ++b) {
          tma_load_3d(&tm_k, kv_full, smem + C::kKV_OffK + b * C::kBlockBytes, b * 64, n0, bkv);
          tma_load_3d(&tm_v, kv_full, smem + C::kKV_OffV + b * C::kBlockBytes, b * 64, n0, bkv);
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
          uint8_t* vec = smem + C::kKV_OffVec + slot * 2 * C::kVecBytes;
          bulk_load(vec, prm.ws_lse2 + voff, C::kVecBytes, &v_full[slot]);
          bulk_load(vec + C::kVecBytes, prm.ws_d + voff, C::kVecBytes, &v_full[slot]);
          ++v_issued;
        }
        {   // Q_i
          const int slot = it % QS, use = it / QS;
          if (use > 0 && !mbar_wait(&q_empty[slot], (use - 1) & 1, abort_flag)) break;
          mbar_arrive_expect_tx(&q_full[slot], C::kTileBytes);
          for (int b = 0; b < C::kNumBlk; ++b)
            tma_load_3d(&tm_q, &q_full[slot], smem + C::kKV_OffQ + slot * C::kTileBytes + b * C::kBlockBytes, b * 64,
                        qi * 128, bq);
          ++q_issued;
        }
        {   // dO_i
          const int slot = it % OS, use = it / OS;
          if (use > 0 && !mbar_wait(&o_empty[slot], (use - 1) & 1, abort_flag)) break;
          mbar_arrive_expect_tx(&o_full[slot], C::kTileBytes);
          for (int b = 0; b < C::kNumBlk; ++b)
            tma_load_3d(&tm_do, &o_full[slot], smem + C::kKV_OffDO + slot * C::kTileBytes + b * C::kBlockBytes, b * 64,
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
    if (lane == 0) {
      constexpr uint32_t kIdescT = idesc_bf16(128, 128, false, false);   // S^T, dP^T
      constexpr uint32_t kIdescAcc = idesc_bf16(128, D, false, true);    // dV, dK (B MN-major)
      const uint32_t sK = smem_u32(smem + C::kKV_OffK);
      const uint32_t sV = smem_u32(smem + C::kKV_OffV);
      auto q_tile = [&](int it) { return smem_u32(smem + C::kKV_OffQ + (it % QS) * C::kTileBytes); };
      auto o_tile = [&](int it) { return smem_u32(smem + C::kKV_OffDO + (it % OS) * C::kTileBytes); };
      auto issue_kmajor = [&](uint32_t dcol, uint32_t a0, uint32_t b0) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kBlockBytes + (kk & 3) * 32;
          mma_ss(tmem + dcol, smem_desc_sw128(a0 + off, 16, 1024), smem_desc_sw128(b0 + off, 16, 1024), kIdescT,
                 kk > 0 ? 1u : 0u);
        }
      };
      auto issue_acc = [&](uint32_t dcol, uint32_t acol, uint32_t b0, bool acc) {
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          mma_ts(tmem + dcol, tmem + acol + 64 * (kk >> 2) + (kk & 3) * 8,
                 smem_desc_sw128(b0 + kk * 2048, C::kBlockBytes, 1024), kIdescAcc, (acc || kk > 0) ? 1u : 0u);
      };
      auto wait_q = [&](int it) { return mbar_wait(&q_full[it % QS], (it / QS) & 1, abort_flag); };
      auto wait_o = [&](int it) { return mbar_wait(&o_full[it % OS], (it / OS) & 1, abort_flag); };

      bool ok = n_it > 0 && mbar_wait(kv_full, 0, abort_flag) && wait_q(0) && wait_o(0);
      if (ok) {
        tc_fence_after();
        issue_kmajor(C::kColA, sK, q_tile(0));    // S^T = K_j Q_i^T
        mma_commit(s_full);
        issue_kmajor(C::kColB, sV, o_tile(0));    // dP^T = V_j dO_i^T
        mma_commit(dp_full);
      }
      for (int it = 0; it < n_it && ok; ++it) {
        const bool more = it + 1 < n_it;
        if (!(ok = mbar_wait(p_full, it & 1, abort_flag))) break;
        tc_fence_after();
        issue_acc(C::kColAcc0, C::kColA, o_tile(it), it > 0);    // dV += P^T dO_i
        mma_commit(&o_empty[it % OS]);                            // dO_i read for the last time
        if (more) {
          if (!(ok = wait_q(it + 1))) break;
          tc_fence_after();
          issue_kmajor(C::kColA, sK, q_tile(it + 1));
          mma_commit(s_full);
        }
        if (!(ok = mbar_wait(ds_full, it & 1, abort_flag))) break;
        tc_fence_after();
        issue_acc(C::kColAcc1, C::kColB, q_tile(it), it > 0);    // dK += dS^T Q_i
        mma_commit(&q_empty[it % QS]);                            // Q_i read for the last time
        if (more) {
          if (!(ok = wait_o(it + 1))) break;
          tc_fence_after();
          issue_kmajor(C::kColB, sV, o_tile(it + 1));
          mma_commit(dp_full);
        }
      }
      if (ok) mma_commit(acc_full);
      mma_commit(drain);
      mbar_wait(drain, 0, abort_flag, false);
    }
    __syncwarp();
  } else {
    // compute warps: thread = key row r (TMEM lane), group g = query columns [64g, 64g+64)
    const int g = warp >> 2;
    const int qw = warp & 3;
    const int r = qw * 32 + lane;
    const int key = n0 + r;
    const uint32_t lane_base = uint32_t(qw * 32) << 16;
    const uint32_t tA = tmem + lane_base + C::kColA + 64 * g;
    const uint32_t tB = tmem + lane_base + C::kColB + 64 * g;
    const float c = prm.scale_log2;
    bool ok = true;
    int Lsel = SPARSE ? sel_next(sel, -1, n_all) : 0;
    for (int it = 0; it < n_it; ++it) {
      const int L = SPARSE ? Lsel : it;
      if (SPARSE) Lsel = sel_next(sel, Lsel, n_all);
      const int qi = i_start + L % n_q;
      const float* vec = reinterpret_cast<const float*>(smem + C::kKV_OffVec + (it % VS) * 2 * C::kVecBytes);
      // LSE/D vectors of this query tile (released below, after the dS reads).
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
      tc_fence_after();
      {
        float dp[64];
        tmem_ld64f(tB, dp);
        const float4* d4 = reinterpret_cast<const float4*>(vec + 128 + 64 * g);
        uint32_t pk[32];
#pragma unroll
        for (int k4 = 0; k4 < 16; ++k4) {
          const float4 dv = d4[k4];
          const float s0 = p[4 * k4 + 0] * (dp[4 * k4 + 0] - dv.x);
          const float s1 = p[4 * k4 + 1] * (dp[4 * k4 + 1] - dv.y);
          const float s2 = p[4 * k4 + 2] * (dp[4 * k4 + 2] - dv.z);
          const float s3 = p[4 * k4 + 3] * (dp[4 * k4 + 3] - dv.w);
          pk[2 * k4] = pack_bf16x2(s0, s1);
          pk[2 * k4 + 1] = pack_bf16x2(s2, s3);
        }
        tmem_st32(tB, pk);   // dS^T over the first 32 of this group's 64 dP^T columns
      }
      mbar_arrive(&v_empty[it % VS]);   // this thread is done with the LSE/D vectors
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    // epilogue: group 0 writes dV (staged in the V_j slot), group 1 writes dK (in the K_j slot)
    if (ok && n_it > 0) ok = mbar_wait_warp(acc_full, 0, abort_flag);
    uint8_t* stage = smem + (g == 0 ? C::kKV_OffV : C::kKV_OffK);
    if (ok) {
      tc_fence_after();
      if (n_it > 0)
        tmem_acc_to_smem<D>(tmem + lane_base + (g == 0 ? C::kColAcc0 : C::kColAcc1), smem_u32(stage), r, 0, D / 32,
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
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::kWarpMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// dQ
// ---------------------------------------------------------------------------
template <int D, bool CAUSAL, bool SPARSE>
__global__ void __launch_bounds__(320, 1)
attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_dq, const BwdParams prm) {
  using C = BwdCfg<D>;
  constexpr int KS = C::kDeep, VS = C::kShallow;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kQ_OffBar);
  uint64_t* k_full = bars;                 // [KS]
  uint64_t* k_empty = k_full + KS;         // [KS]  dQ(j) done
  uint64_t* v_full = k_empty + KS;         // [VS]
  uint64_t* v_empty = v_full + VS;         // [VS]  dP(j) done
  uint64_t* q_full = v_empty + VS;
  uint64_t* s_full = q_full + 1;
  uint64_t* s_free = s_full + 1;
  uint64_t* dp_full = s_free + 1;
  uint64_t* ds_full = dp_full + 1;
  uint64_t* acc_full = ds_full + 1;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + C::kNumBars) + 1;
  if (smem_u32(smem) & 1023u) {            // the layout needs a 1024-aligned window
    if (threadIdx.x == 0) atomicOr(&g_attn_status, kStatusLayout);
    return;
  }

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n = prm.n;
  const int nt = prm.n_tiles;
  const int bh = blockIdx.x / nt;                                             // query head
  const int bkv = (bh / prm.h) * prm.h_kv + (bh % prm.h) / prm.group;        // its key/value head
  const int it_q = nt - 1 - (blockIdx.x % nt);   // query tile; large = most work under the causal mask
  const int m0 = it_q * 128;
  const int j_hi = CAUSAL ? it_q + 1 : nt;       // key tiles [0, j_hi) may be visible
  const uint8_t* mrow = SPARSE ? prm.mask + (size_t(bh) * nt + it_q) * nt : nullptr;
  auto sel = [&](int j) -> bool { return mrow[j] != 0; };
  const int n_it = SPARSE ? sel_count(sel, j_hi) : j_hi;

  if (threadIdx.x == 0) {
    for (int s = 0; s < KS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(s_full, 1);
    mbar_init(s_free, 256);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, 256);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == C::kWarpMma) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::kWarpLoad) {
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, 2 * C::kTileBytes + 2 * C::kVecBytes);
      for (int b = 0; b < C::kNumBlk; ++b) {
        tma_load_3d(&tm_q, q_full, smem + C::kQ_OffQ + b * C::kBlockBytes, b * 64, m0, bh);
        tma_load_3d(&tm_do, q_full, smem + C::kQ_OffDO + b * C::kBlockBytes, b * 64, m0, bh);
      }
      const size_t voff = size_t(bh) * size_t(prm.npad) + size_t(m0);
      bulk_load(smem + C::kQ_OffVec, prm.ws_lse2 + voff, C::kVecBytes, q_full);
      bulk_load(smem + C::kQ_OffVec + C::kVecBytes, prm.ws_d + voff, C::kVecBytes, q_full);
      int k_issued = 0, v_issued = 0;
      int jsel = SPARSE ? sel_next(sel, -1, j_hi) : 0;
      for (int it = 0; it < n_it; ++it) {
        const int j = SPARSE ? jsel : it;
        if (SPARSE) jsel = sel_next(sel, jsel, j_hi);
        {
          const int slot = it % KS, use = it / KS;
          if (use > 0 && !mbar_wait(&k_empty[slot], (use - 1) & 1, abort_flag)) break;
          mbar_arrive_expect_tx(&k_full[slot], C::kTileBytes);
          for (int b = 0; b < C::kNumBlk; ++b)
            tma_load_3d(&tm_k, &k_full[slot], smem + C::kQ_OffK + slot * C::kTileBytes + b * C::kBlockBytes, b * 64,
                        j * 128, bkv);
          ++k_issued;
        }
        {
          const int slot = it % VS, use = it / VS;
          if (use > 0 && !mbar_wait(&v_empty[slot], (use - 1) & 1, abort_flag)) break;
          mbar_arrive_expect_tx(&v_full[slot], C::kTileBytes);
          for (int b = 0; b < C::kNumBlk; ++b)
            tma_load_3d(&tm_v, &v_full[slot], smem + C::kQ_OffV + slot * C::kTileBytes + b * C::kBlockBytes, b * 64,
                        j * 128, bkv);
          ++v_issued;
        }
      }
      mbar_wait(q_full, 0, abort_flag, false);
      for (int it = max(0, k_issued - KS); it < k_issued; ++it)
        mbar_wait(&k_full[it % KS], (it / KS) & 1, abort_flag, false);
      for (int it = max(0, v_issued - VS); it < v_issued; ++it)
        mbar_wait(&v_full[it % VS], (it / VS) & 1, abort_flag, false);
    }
    __syncwarp();
  } else if (warp == C::kWarpMma) {
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16(128, 128, false, false);
      constexpr uint32_t kIdescAcc = idesc_bf16(128, D, false, true);
      const uint32_t sQ = smem_u32(smem + C::kQ_OffQ);
      const uint32_t sDO = smem_u32(smem + C::kQ_OffDO);
      auto k_tile = [&](int it) { return smem_u32(smem + C::kQ_OffK + (it % KS) * C::kTileBytes); };
      auto v_tile = [&](int it) { return smem_u32(smem + C::kQ_OffV + (it % VS) * C::kTileBytes); };
      auto wait_k = [&](int it) { return mbar_wait(&k_full[it % KS], (it / KS) & 1, abort_flag); };
      auto wait_v = [&](int it) { return mbar_wait(&v_full[it % VS], (it / VS) & 1, abort_flag); };
      auto issue_kmajor = [&](uint32_t dcol, uint32_t a0, uint32_t b0) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kBlockBytes + (kk & 3) * 32;
          mma_ss(tmem + dcol, smem_desc_sw128(a0 + off, 16, 1024), smem_desc_sw128(b0 + off, 16, 1024), kIdescS,
                 kk > 0 ? 1u : 0u);
        }
      };

      bool ok = n_it > 0 && mbar_wait(q_full, 0, abort_flag) && wait_k(0) && wait_v(0);
      if (ok) {
        tc_fence_after();
        issue_kmajor(C::kColA, sQ, k_tile(0));    // S = Q_i K_j^T
        mma_commit(s_full);
        issue_kmajor(C::kColB, sDO, v_tile(0));   // dP = dO_i V_j^T
        mma_commit(dp_full);
        mma_commit(&v_empty[0]);                  // V_j read for the last time
      }
      for (int it = 0; it < n_it && ok; ++it) {
        const bool more = it + 1 < n_it;
        if (more) {
          if (!(ok = wait_k(it + 1))) break;
          if (!(ok = mbar_wait(s_free, it & 1, abort_flag))) break;
          tc_fence_after();
          issue_kmajor(C::kColA, sQ, k_tile(it + 1));
          mma_commit(s_full);
        }
        if (!(ok = mbar_wait(ds_full, it & 1, abort_flag))) break;
        tc_fence_after();
        // dQ += dS K_j: A = dS in TMEM (over dP columns), B = K_j MN-major
        const uint32_t bk = k_tile(it);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          mma_ts(tmem + C::kColAcc0, tmem + C::kColB + 64 * (kk >> 2) + (kk & 3) * 8,
                 smem_desc_sw128(bk + kk * 2048, C::kBlockBytes, 1024), kIdescAcc, (it > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&k_empty[it % KS]);            // K_j read for the last time
        if (more) {
          if (!(ok = wait_v(it + 1))) break;
          tc_fence_after();
          issue_kmajor(C::kColB, sDO, v_tile(it + 1));
          mma_commit(dp_full);
          mma_commit(&v_empty[(it + 1) % VS]);
        }
      }
      if (ok) mma_commit(acc_full);
      mma_commit(drain);
      mbar_wait(drain, 0, abort_flag, false);
    }
    __syncwarp();
  } else {
    // compute warps: thread = query row r, group g = key columns [64g, 64g+64)
    const int g = warp >> 2;
    const int qw = warp & 3;
    const int r = qw * 32 + lane;
    const int row = m0 + r;
    const uint32_t lane_base = uint32_t(qw * 32) << 16;
    const uint32_t tA = tmem + lane_base + C::kColA + 64 * g;
    const uint32_t tB = tmem + lane_base + C::kColB + 64 * g;
    const float c = prm.scale_log2;
    bool ok = mbar_wait_warp(q_full, 0, abort_flag);
    const float* vec = reinterpret_cast<const float*>(smem + C::kQ_OffVec);
    const float neg_lse2 = ok ? -vec[r] : 0.f;
    const float dval = ok ? vec[128 + r] : 0.f;
    int jsel = SPARSE ? sel_next(sel, -1, j_hi) : 0;
    for (int it = 0; it < n_it && ok; ++it) {
      const int j = SPARSE ? jsel : it;               // key tile of this iteration
      if (SPARSE) jsel = sel_next(sel, jsel, j_hi);
      if (!(ok = mbar_wait_warp(s_full, it & 1, abort_flag))) break;
      tc_fence_after();
      float p[64];
      tmem_ld64f(tA, p);
      tc_fence_before();
      mbar_arrive(s_free);
#pragma unroll
      for (int k = 0; k < 64; ++k) p[k] = ex2(fmaf(p[k], c, neg_lse2));
      const int kbase = j * 128 + 64 * g;
      const bool need_mask = (CAUSAL && j == it_q) || (kbase + 64 > n);
      if (need_mask) {
        int lim = n - 1 - kbase;                 // keep k <= lim
        if (CAUSAL) lim = min(lim, row - kbase);
#pragma unroll
        for (int k = 0; k < 64; ++k)
          if (k > lim) p[k] = 0.f;
      }
      if (!(ok = mbar_wait_warp(dp_full, it & 1, abort_flag))) break;
      tc_fence_after();
      {
        float dp[64];
        tmem_ld64f(tB, dp);
        uint32_t pk[32];
#pragma unroll
        for (int k = 0; k < 32; ++k)
          pk[k] = pack_bf16x2(p[2 * k] * (dp[2 * k] - dval), p[2 * k + 1] * (dp[2 * k + 1] - dval));
        tmem_st32(tB, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    if (ok && n_it > 0) ok = mbar_wait_warp(acc_full, 0, abort_flag);
    uint8_t* stage = smem + C::kQ_OffQ;   // Q_i is no longer read
    if (ok) {
      tc_fence_after();
      constexpr int kChunks = D / 32;
      if (n_it > 0)
        tmem_acc_to_smem<D>(tmem + lane_base + C::kColAcc0, smem_u32(stage), r, g * kChunks / 2,
                            (g + 1) * kChunks / 2, prm.scale);
      else
        zero_tile_rows<D>(smem_u32(stage), r, g * kChunks / 2, (g + 1) * kChunks / 2);   // this query tile sees no key
    }
    fence_proxy_async_smem();
    named_barrier_sync(1, 256);
    if (warp == 0 && lane == 0 && *abort_flag == 0) {
      for (int b = 0; b < C::kNumBlk; ++b) tma_store_3d(&tm_dq, stage + b * C::kBlockBytes, b * 64, m0, bh);
      bulk_commit_group();
      bulk_wait_group_read0();
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
