// attn_kvcache_fp8.cuh -- decode against a key/value cache stored in FP8
// (E4M3) with per-tensor dequantisation factors.
//
// The computation is the bf16 cache forward's ("FlashAttention -- how
// 100K-token attention fits in memory", section "Arithmetic intensity": decode
// is bound by reading the cache; "Attention and KV Compression", section "What
// it does and does not change": narrower formats leave the computation
// unchanged) on the dequantised cache K = dk * K8, V = dv * V8.  Halving the
// cache bytes is the point: decode reads every cached byte once per step.
//
// B200 mapping: the persistent, replicated-mode structure of the bf16 cache
// kernel (work item = key/value head x key chunk, up to 32 packed query rows
// replicated over the four TMEM lane quarters, warp w of the softmax owning
// key columns [32w, 32w+32), four partials per item merged by LSE), with one
// change: the cache tiles arrive as E4M3 bytes (TMA, 16 KB per tile) and eight
// dedicated widening warps turn them into one f16 K tile and one f16 V tile
// in shared memory with integer operations only (exactly: every E4M3 value
// times 2^-8 is an f16 value, normal or subnormal; the 2^8 goes into the
// scales).  The MMAs run as kind::f16 with f16 operands: the widening warps
// also convert each work item's query tile from bf16 to f16 in shared memory
// (exact for |q| in [2^-14, 65504]) and the softmax packs P as f16.
// K_{j+1} is widened as soon as S_j has completed, V_j once PV_{j-1} has
// completed, so the widening of one tile overlaps the softmax of the previous
// one.  dk is folded into the exp2 argument and dv into the final 1/l.  Cache
// rows past the valid length are widened as zeros in V.  d = 128.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "attn_kvcache.cuh"

namespace attn {

struct Kvc8Cfg {
  static constexpr int D = 128;
  static constexpr int kTileBytes = 128 * D * 2;       // 16-bit tiles (Q, widened K, widened V)
  static constexpr int kTile8Bytes = 128 * D;          // E4M3 tile: 128 rows x 128 bytes
  static constexpr int kBlockBytes = 128 * 128;
  static constexpr int kNumBlk = D / 64;
  static constexpr int kSlots = 6;                     // E4M3 ring: three key tiles ahead
  static constexpr int kWarpMma = 4;
  static constexpr int kWarpLoad = 5;
  static constexpr int kWarpWiden0 = 6;                // warps 6 .. 6 + kWidenWarps - 1
  static constexpr int kWidenWarps = 8;
  static constexpr int kWidenThreads = 32 * kWidenWarps;
  static constexpr int kThreads = 32 * kWarpWiden0 + kWidenThreads;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
  static constexpr uint32_t kColP0 = 384, kColP1 = 448;
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = kTileBytes;
  static constexpr int kOffKb = kOffRing + kSlots * kTile8Bytes;
  static constexpr int kOffVb = kOffKb + kTileBytes;
  static constexpr int kOffBar = kOffVb + kTileBytes;
  // q_full, q_empty, ring_full[S], ring_empty[S], s_full[2], p_full[2], pv_done, o_full, o_free,
  // kb_full, kb_free, vb_full, vb_free, drain, q_ready
  static constexpr int kNumBars = 2 + 2 * kSlots + 2 + 2 + 3 + 4 + 1 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
};
static_assert(Kvc8Cfg::kSmemBytes <= 227 * 1024, "shared memory");

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// Two E4M3 codes (bytes 0 and 2 of x, bytes 1 and 3 zero) -> one f16x2 word
// holding 2^-8 times their values, with integer operations only.  The code
// s.eeee.mmm placed at f16 bits 15 / 13..10 / 9..7 is the f16 number
// 2^(e-15) * 1.mmm (or 0.mmm * 2^-14 for e = 0), i.e. exactly 2^-8 times the
// E4M3 value 2^(e-7) * 1.mmm (0.mmm * 2^-6).  Shifting the code left by 7
// puts eeee.mmm in place and the sign at bit 14; adding the sign bit once
// more first carries it to bit 15 (a code plus its sign bit is at most 0x17F,
// so nothing crosses into the other half).  The factor 2^8 is folded into the
// dequantisation scales.  (The E4M3 NaN code reads as 2^-8 * 480.)
__device__ __forceinline__ uint32_t e4m3_pair_to_f16x2(uint32_t x) {
  return (x + (x & 0x00800080u)) << 7;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);   // .x (low 16 bits) = lo
  return *reinterpret_cast<uint32_t*>(&v);
}

// Instruction descriptor, kind::f16 with f16 A and B (format code 0), fp32 D.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Widen one 128 x 128 E4M3 tile (128-byte swizzled rows) into an f16 tile
// (two [128][64] column blocks, 128-byte swizzle) with the kWidenThreads
// widening threads: 8 lanes per row (lane c reads bytes 16c..16c+15), 32 rows
// per pass.  Rows >= zero_from are written as zeros.  Lane c's 16 values are
// two 16-byte chunks of column block c / 4; lanes c < 4 store their even
// chunk first and lanes c >= 4 their odd chunk first, so the eight lanes of
// one row hit eight different bank groups in each store.
__device__ __forceinline__ void widen_tile(uint32_t src8, uint32_t dstb, int t, int zero_from) {
  const int c = t & 7;
  const uint32_t blk = dstb + (c >> 2) * Kvc8Cfg::kBlockBytes;
  const uint32_t ch = (c & 3) * 2;
  const bool odd_first = c >= 4;
#pragma unroll 2
  for (int pass = 0; pass < 128 * 8 / Kvc8Cfg::kWidenThreads; ++pass) {
    const int row = pass * (Kvc8Cfg::kWidenThreads / 8) + (t >> 3);
    const uint4 v = ld_shared_v4(src8 + row * 128 + ((c ^ (row & 7)) << 4));
    uint32_t w[8];
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      w[2 * k] = e4m3_pair_to_f16x2(__byte_perm(in[k], 0u, 0x4140));       // codes 4k, 4k+1
      w[2 * k + 1] = e4m3_pair_to_f16x2(__byte_perm(in[k], 0u, 0x4342));   // codes 4k+2, 4k+3
    }
    if (row >= zero_from) {
#pragma unroll
      for (int k = 0; k < 8; ++k) w[k] = 0u;
    }
    const uint32_t a0 = blk + sw128_offset(row, ch);
    const uint32_t a1 = blk + sw128_offset(row, ch + 1);
    if (odd_first) {
      st_shared_v4(a1, w[4], w[5], w[6], w[7]);
      st_shared_v4(a0, w[0], w[1], w[2], w[3]);
    } else {
      st_shared_v4(a0, w[0], w[1], w[2], w[3]);
      st_shared_v4(a1, w[4], w[5], w[6], w[7]);
    }
  }
}

// The query tile (bf16, [128][64] column blocks, 128-byte swizzle) -> f16 in
// place, by the widening threads: 16-byte chunk q = pass * kWidenThreads + t
// is chunk q % 8 of column block (q / 8) % 2 of row q / 16, so the eight lanes
// of a row read and write eight different bank groups.  Rows that are padding
// in every lane quarter are zeros already and are skipped.
__device__ __forceinline__ void convert_q_tile(uint32_t sq, int t, int qbox) {
#pragma unroll 2
  for (int pass = 0; pass < 128 * 16 / Kvc8Cfg::kWidenThreads; ++pass) {
    const int q = pass * Kvc8Cfg::kWidenThreads + t;
    const int row = q >> 4;
    if ((row & 31) >= qbox) continue;
    const uint32_t a = sq + ((q >> 3) & 1) * Kvc8Cfg::kBlockBytes + row * 128 + (q & 7) * 16;
    const uint4 v = ld_shared_v4(a);
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
    uint32_t o4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      o4[k] = pack_f16x2(__uint_as_float(in[k] << 16), __uint_as_float(in[k] & 0xFFFF0000u));
    st_shared_v4(a, o4[0], o4[1], o4[2], o4[3]);
  }
}

template <bool CAUSAL>
__global__ void __launch_bounds__(Kvc8Cfg::kThreads, 1)
attn_kvcache_fp8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k8,
                        const __grid_constant__ CUtensorMap tm_v8, const KvcParams prm, const float v_descale) {
  using C = Kvc8Cfg;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* q_empty = q_full + 1;
  uint64_t* ring_full = q_empty + 1;
  uint64_t* ring_empty = ring_full + C::kSlots;
  uint64_t* s_full = ring_empty + C::kSlots;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* o_full = pv_done + 1;
  uint64_t* o_free = o_full + 1;
  uint64_t* kb_full = o_free + 1;          // the f16 K tile holds the next key tile
  uint64_t* kb_free = kb_full + 1;         // the S product reading it has completed
  uint64_t* vb_full = kb_free + 1;
  uint64_t* vb_free = vb_full + 1;         // the PV product reading it has completed
  uint64_t* drain = vb_free + 1;
  uint64_t* q_ready = drain + 1;           // the query tile has been converted to f16
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(&ring_full[s], 1);
      mbar_init(&ring_empty[s], C::kWidenWarps);   // one arrival per widening warp
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
    }
    mbar_init(pv_done, 1);
    mbar_init(o_full, 1);
    mbar_init(o_free, 128);
    mbar_init(kb_full, C::kWidenWarps);
    mbar_init(kb_free, 1);
    mbar_init(vb_full, C::kWidenWarps);
    mbar_init(vb_free, 1);
    mbar_init(drain, 1);
    mbar_init(q_ready, C::kWidenWarps);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp < 4 && prm.qbox < 32) {
    // Query rows that are padding in every lane quarter are never loaded:
    // zero them once.
    const int r = threadIdx.x;
    if ((r & 31) >= prm.qbox)
      for (int blk = 0; blk < C::kNumBlk; ++blk)
        for (int ch = 0; ch < 8; ++ch)
          st_shared_v4(smem_u32(smem + C::kOffQ + blk * C::kBlockBytes) + r * 128 + ch * 16, 0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  if (warp == C::kWarpMma) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == C::kWarpLoad && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k8);
    tma_prefetch_desc(&tm_v8);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_items = prm.n_items;
  if (warp < 4) {
    // Each lane quarter writes P only in its own 16 packed columns of a P
    // buffer; the other columns of its lanes stay zero.
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
        if (qi >= 1 && !(ok = mbar_wait(q_empty, uint32_t((qi - 1) & 1), abort_flag))) break;
        mbar_arrive_expect_tx(q_full, uint32_t(4 * prm.qbox * 128 * C::kNumBlk));
        for (int cp = 0; cp < 4; ++cp)
          for (int blk = 0; blk < C::kNumBlk; ++blk)
            tma_load_3d(&tm_q, q_full, smem + C::kOffQ + blk * C::kBlockBytes + cp * 32 * 128, blk * 64,
                        I.bkv * prm.rows + I.r0, 0);
        ++qi;
        for (int t = 0; t < 2 * I.nkv; ++t) {
          const int slot = it % C::kSlots;
          const int use = it / C::kSlots;
          if (use > 0 && !(ok = mbar_wait(&ring_empty[slot], uint32_t((use - 1) & 1), abort_flag))) break;
          mbar_arrive_expect_tx(&ring_full[slot], C::kTile8Bytes);
          tma_load_3d((t & 1) ? &tm_v8 : &tm_k8, &ring_full[slot], smem + C::kOffRing + slot * C::kTile8Bytes, 0,
                      128 * (I.j_lo + (t >> 1)), I.bkv);
          ++it;
        }
      }
      for (int q = max(0, qi - 1); q < qi; ++q) mbar_wait(q_full, uint32_t(q & 1), abort_flag, false);
      for (int k = max(0, it - C::kSlots); k < it; ++k)
        mbar_wait(&ring_full[k % C::kSlots], uint32_t((k / C::kSlots) & 1), abort_flag, false);
    }
    __syncwarp();
  } else if (warp == C::kWarpMma) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_f16(128, 128, false, false);
      constexpr uint32_t kIdescPV = idesc_f16(128, D, false, true);
      const uint32_t sQ = smem_u32(smem + C::kOffQ);
      const uint32_t sKb = smem_u32(smem + C::kOffKb);
      const uint32_t sVb = smem_u32(smem + C::kOffVb);
      int qi = 0, sc = 0, oi = 0;
      bool ok = true;
      bool issued_any = false;
      for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
        const KvcItem I = kvc_item(prm, w, CAUSAL);
        if (I.nkv == 0) continue;
        if (!(ok = mbar_wait(q_ready, uint32_t(qi & 1), abort_flag))) break;
        for (int jj = 0; jj <= I.nkv && ok; ++jj) {
          if (jj < I.nkv) {
            // K_jj widened into the f16 K tile (global key tile count sc + jj).
            // S buffer (sc + jj) & 1 was last read by the softmax of tile
            // jj - 2, whose P was waited for before PV_{jj-2} was issued.
            if (!(ok = mbar_wait(kb_full, uint32_t((sc + jj) & 1), abort_flag))) break;
            tc_fence_after();
            const uint32_t dt = tmem + (((sc + jj) & 1) ? C::kColS1 : C::kColS0);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * C::kBlockBytes + (kk & 3) * 32;
              mma_ss(dt, smem_desc_sw128(sQ + off, 16, 1024), smem_desc_sw128(sKb + off, 16, 1024), kIdescS,
                     kk > 0 ? 1u : 0u);
            }
            issued_any = true;
            mma_commit(&s_full[(sc + jj) & 1]);
            mma_commit(kb_free);
            if (jj == I.nkv - 1) mma_commit(q_empty);
          }
          if (jj > 0) {
            const int pj = jj - 1;
            const int ps = sc + pj;
            if (!(ok = mbar_wait(&p_full[ps & 1], uint32_t((ps >> 1) & 1), abort_flag))) break;
            if (pj == 0 && oi > 0 && !(ok = mbar_wait(o_free, uint32_t((oi - 1) & 1), abort_flag))) break;
            if (!(ok = mbar_wait(vb_full, uint32_t(ps & 1), abort_flag))) break;
            tc_fence_after();
            const uint32_t at = tmem + ((ps & 1) ? C::kColP1 : C::kColP0);
#pragma unroll
            for (int kk = 0; kk < 128 / 16; ++kk)
              mma_ts(tmem + C::kColO, at + kk * 8, smem_desc_sw128(sVb + kk * 2048, C::kBlockBytes, 1024), kIdescPV,
                     (pj > 0 || kk > 0) ? 1u : 0u);
            mma_commit(pj == I.nkv - 1 ? o_full : pv_done);
            mma_commit(vb_free);
          }
        }
        sc += I.nkv;
        ++qi;
        ++oi;
      }
      if (issued_any) {
        mma_commit(drain);
        mbar_wait(drain, 0, abort_flag, false);
      }
    }
    __syncwarp();
  } else if (warp >= C::kWarpWiden0) {
    // ------------------------------------------------ widening (8 warps)
    // Per work item: the query tile to f16, then K_0, then K_{jj+1} and V_jj
    // for every key tile jj (K first: S_{jj+1} waits for it, while PV_jj
    // also waits for the softmax of tile jj).  kc / vc count the K / V tiles
    // widened over all items; tile kc may overwrite the K tile once the S
    // product of tile kc - 1 has completed (kb_free), likewise V with PV.
    const int t = threadIdx.x - 32 * C::kWarpWiden0;
    const uint32_t sRing = smem_u32(smem + C::kOffRing);
    const uint32_t sKb = smem_u32(smem + C::kOffKb);
    const uint32_t sVb = smem_u32(smem + C::kOffVb);
    int it = 0, kc = 0, vc = 0, qi = 0;
    bool ok = true;

    // Widen ring item `item` into dst and release its ring slot; then signal
    // `full`.  Every thread fences its own shared-memory writes for the
    // tensor core's (async) proxy before its warp's single arrival.
    auto widen = [&](int item, uint32_t dst, int zero_from, uint64_t* full) -> bool {
      const int slot = item % C::kSlots;
      if (!mbar_wait_warp(&ring_full[slot], uint32_t((item / C::kSlots) & 1), abort_flag)) return false;
      widen_tile(sRing + slot * C::kTile8Bytes, dst, t, zero_from);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&ring_empty[slot]);
        mbar_arrive(full);
      }
      return true;
    };
    auto widen_k = [&](int item) -> bool {
      if (kc > 0 && !mbar_wait_warp(kb_free, uint32_t((kc - 1) & 1), abort_flag)) return false;
      if (!widen(item, sKb, 128, kb_full)) return false;
      ++kc;
      return true;
    };
    auto widen_v = [&](int item, int zero_from) -> bool {
      if (vc > 0 && !mbar_wait_warp(vb_free, uint32_t((vc - 1) & 1), abort_flag)) return false;
      if (!widen(item, sVb, zero_from, vb_full)) return false;
      ++vc;
      return true;
    };

    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const KvcItem I = kvc_item(prm, w, CAUSAL);
      if (I.nkv == 0) continue;
      // The query tile: loaded after the previous item's last S product.
      if (!(ok = mbar_wait_warp(q_full, uint32_t(qi & 1), abort_flag))) break;
      convert_q_tile(smem_u32(smem + C::kOffQ), t, prm.qbox);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
      ++qi;
      if (!(ok = widen_k(it))) break;
      for (int jj = 0; jj < I.nkv && ok; ++jj) {
        if (jj + 1 < I.nkv && !(ok = widen_k(it + 2 * (jj + 1)))) break;
        // rows past the valid length become zeros
        ok = widen_v(it + 2 * jj + 1, I.L - 128 * (I.j_lo + jj));
      }
      it += 2 * I.nkv;
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ softmax (warps 0-3)
    const int r = lane;                       // packed row (replicated in every lane quarter)
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const uint32_t tO = tmem + lane_base + C::kColO;
    const float c = prm.scale_log2;           // includes dk
    int sc = 0, pvb = 0, oi = 0;
    bool ok = true;

    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const KvcItem I = kvc_item(prm, w, CAUSAL);
      const int rp = I.r0 + r;
      const bool row_ok = r < I.r_valid;
      int lim = I.L - 1;
      if (CAUSAL) lim = min(lim, rp % prm.nq + I.L - prm.nq);
      float m_ref = -INFINITY;
      float l = 0.f;

      for (int jj = 0; jj < I.nkv; ++jj) {
        const int j = I.j_lo + jj;
        const int sb = (sc + jj) & 1;
        const uint32_t tS = tmem + lane_base + (sb ? C::kColS1 : C::kColS0);
        if (!(ok = mbar_wait_warp(&s_full[sb], uint32_t(((sc + jj) >> 1) & 1), abort_flag))) break;
        tc_fence_after();

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
          pk[k] = pack_f16x2(p0, p1);
        }
        tmem_st16(tmem + lane_base + (sb ? C::kColP1 : C::kColP0) + 16 * warp, pk);
        l += (sump[0] + sump[1]) + (sump[2] + sump[3]);
        if (__any_sync(0xffffffffu, rescale)) {
          // O may only be rescaled once PV_{jj-1} has completed.  PV_jj needs
          // this tile's P, so pv_done is at most one phase ahead of this wait
          // and the phases skipped when no rescale happens are never misread.
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
        tc_fence_before();
        mbar_arrive(&p_full[sb]);
      }
      if (!ok) break;

      // ---------------------------------------------------------- epilogue
      if (I.nkv > 0 && !(ok = mbar_wait_warp(o_full, uint32_t(oi & 1), abort_flag))) break;
      tc_fence_after();
      const bool has = l > 0.f;
      const float inv_l = has ? v_descale / l : 0.f;
      const long long row = (long long)I.bkv * prm.rows + rp;
      const int part = I.split * 4 + warp;
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
          float4* dst = reinterpret_cast<float4*>(prm.part_o + ((long long)part * prm.total_rows + row) * D + cc * 32);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            dst[k] = make_float4(__uint_as_float(o[4 * k]) * inv_l, __uint_as_float(o[4 * k + 1]) * inv_l,
                                 __uint_as_float(o[4 * k + 2]) * inv_l, __uint_as_float(o[4 * k + 3]) * inv_l);
        }
      }
      if (row_ok) prm.part_lse[(long long)part * prm.total_rows + row] = has ? (m_ref + __log2f(l)) * kKvcLn2 : -INFINITY;
      if (I.nkv > 0) {
        tc_fence_before();
        mbar_arrive(o_free);
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

}  // namespace attn
