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
// change: the cache tiles arrive as E4M3 bytes (TMA, 16 KB per tile) and the
// four softmax warps widen them into one f16 K tile and one f16 V tile in
// shared memory with integer operations only (exactly: every E4M3 value times
// 2^-8 is an f16 value, normal or subnormal; the 2^8 goes into the scales).
// The MMAs run as kind::f16 with f16 operands: the query tile is converted
// from bf16 to f16 in shared memory once per work item (exact for |q| in the
// f16 range, up to 65504) and P is packed as f16.  K_{j+1} is widened as soon as S_j
// has completed (so S_{j+1} runs during the softmax of tile j), V_j once PV_{j-1}
// has completed.  dk is folded into the exp2 argument and dv into the final
// 1/l.  Cache rows past the valid length are widened as zeros in V.  d = 128.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "attn_kvcache.cuh"

namespace attn {

struct Kvc8Cfg {
  static constexpr int D = 128;
  static constexpr int kTileBytes = 128 * D * 2;       // bf16 tiles (Q, widened K, widened V)
  static constexpr int kTile8Bytes = 128 * D;          // E4M3 tile: 128 rows x 128 bytes
  static constexpr int kBlockBytes = 128 * 128;
  static constexpr int kNumBlk = D / 64;
  static constexpr int kSlots = 6;                     // E4M3 ring: three key tiles ahead
  static constexpr int kThreads = 192;
  static constexpr int kWarpMma = 4;
  static constexpr int kWarpLoad = 5;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
  static constexpr uint32_t kColP0 = 384, kColP1 = 448;
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = kTileBytes;
  static constexpr int kOffKb = kOffRing + kSlots * kTile8Bytes;
  static constexpr int kOffVb = kOffKb + kTileBytes;
  static constexpr int kOffBar = kOffVb + kTileBytes;
  // q_full, q_empty, ring_full[S], ring_empty[S], s_full[2], p_full[2], pv_done, o_full, o_free,
  // kb_full, vb_full, drain, q_ready
  static constexpr int kNumBars = 2 + 2 * kSlots + 2 + 2 + 3 + 2 + 1 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
};

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// Two E4M3 codes (bytes 0 and 2 of x, bytes 1 and 3 zero) -> one f16x2 word
// holding 2^-8 times their values, with integer operations only: the code
// s.eeee.mmm placed at f16 bits 15 / 13..10 / 9..7 is the f16 number
// 2^(e-15) * 1.mmm (or 0.mmm * 2^-14 for e = 0), i.e. exactly 2^-8 times the
// E4M3 value 2^(e-7) * 1.mmm (0.mmm * 2^-6).  The factor 2^8 is folded into
// the dequantisation scales.  (The E4M3 NaN code reads as 2^-8 * 480.)
__device__ __forceinline__ uint32_t e4m3_pair_to_f16x2(uint32_t x) {
  return ((x & 0x007F007Fu) << 7) | ((x & 0x00800080u) << 8);
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

// Widen one 128 x 128 E4M3 tile (128-byte swizzled rows) into a bf16 tile
// (two [128][64] column blocks, 128-byte swizzle), all 128 threads: 8 lanes
// per row, 16 rows per pass.  Rows >= zero_from are written as zeros.
__device__ __forceinline__ void widen_tile(uint32_t src8, uint32_t dstb, int tid, int zero_from) {
  const int c = tid & 7;                 // 16-byte chunk of the E4M3 row = elements 16c..16c+15
#pragma unroll 2
  for (int pass = 0; pass < 8; ++pass) {
    const int row = pass * 16 + (tid >> 3);
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
    const uint32_t blk = dstb + (c >> 2) * 16384;
    const uint32_t ch = (c & 3) * 2;
    st_shared_v4(blk + sw128_offset(row, ch), w[0], w[1], w[2], w[3]);
    st_shared_v4(blk + sw128_offset(row, ch + 1), w[4], w[5], w[6], w[7]);
  }
}

template <bool CAUSAL>
__global__ void __launch_bounds__(192, 1)
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
  uint64_t* kb_full = o_free + 1;
  uint64_t* vb_full = kb_full + 1;
  uint64_t* drain = vb_full + 1;
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
      mbar_init(&ring_empty[s], 128);      // released by the widening threads
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
    }
    mbar_init(pv_done, 1);
    mbar_init(o_full, 1);
    mbar_init(o_free, 128);
    mbar_init(kb_full, 128);
    mbar_init(vb_full, 128);
    mbar_init(drain, 1);
    mbar_init(q_ready, 128);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp < 4 && prm.qbox < 32) {
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
            // K_jj widened into the bf16 K tile (global tile count sc + jj)
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
  } else {
    // ------------------------------------------ widening + softmax (warps 0-3)
    const int tid = threadIdx.x;              // 0..127: widening lane
    const int r = lane;                       // packed row (replicated in every lane quarter)
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const uint32_t tO = tmem + lane_base + C::kColO;
    const uint32_t sRing = smem_u32(smem + C::kOffRing);
    const uint32_t sKb = smem_u32(smem + C::kOffKb);
    const uint32_t sVb = smem_u32(smem + C::kOffVb);
    const float c = prm.scale_log2;           // includes dk
    int it = 0, sc = 0, pvb = 0, oi = 0;
    bool ok = true;

    // Widen ring item `item` into dst; the ring slot is then released.
    auto widen = [&](int item, uint32_t dst, int zero_from) -> bool {
      const int slot = item % C::kSlots;
      if (!mbar_wait_warp(&ring_full[slot], uint32_t((item / C::kSlots) & 1), abort_flag)) return false;
      widen_tile(sRing + slot * C::kTile8Bytes, dst, tid, zero_from);
      fence_proxy_async_smem();
      mbar_arrive(&ring_empty[slot]);
      return true;
    };

    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const KvcItem I = kvc_item(prm, w, CAUSAL);
      const int rp = I.r0 + r;
      const bool row_ok = r < I.r_valid;
      int lim = I.L - 1;
      if (CAUSAL) lim = min(lim, rp % prm.nq + I.L - prm.nq);
      float m_ref = -INFINITY;
      float l = 0.f;

      // K_0 of this item: the previous item's S products have all completed
      // (its o_full was waited in its epilogue), so the K tile is free.
      if (I.nkv > 0) {
        // This item's query tile (bf16, four copies) -> f16 in place: thread t
        // converts row t of both column blocks.
        if (!(ok = mbar_wait_warp(q_full, uint32_t(oi & 1), abort_flag))) break;
        if ((tid & 31) < prm.qbox) {
#pragma unroll
          for (int blk = 0; blk < C::kNumBlk; ++blk)
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
              const uint32_t a = smem_u32(smem + C::kOffQ) + blk * C::kBlockBytes + tid * 128 + ch * 16;
              const uint4 v = ld_shared_v4(a);
              const uint32_t in[4] = {v.x, v.y, v.z, v.w};
              uint32_t o4[4];
#pragma unroll
              for (int k = 0; k < 4; ++k)
                o4[k] = pack_f16x2(__uint_as_float(in[k] << 16), __uint_as_float(in[k] & 0xFFFF0000u));
              st_shared_v4(a, o4[0], o4[1], o4[2], o4[3]);
            }
        }
        fence_proxy_async_smem();
        mbar_arrive(q_ready);
        if (!(ok = widen(it, sKb, 128))) break;
        mbar_arrive(kb_full);
      }
      for (int jj = 0; jj < I.nkv; ++jj) {
        const int j = I.j_lo + jj;
        const int sb = (sc + jj) & 1;
        const uint32_t tS = tmem + lane_base + (sb ? C::kColS1 : C::kColS0);
        if (!(ok = mbar_wait_warp(&s_full[sb], uint32_t(((sc + jj) >> 1) & 1), abort_flag))) break;
        tc_fence_after();
        // S_jj has completed: the K tile may take K_{jj+1}.
        if (jj + 1 < I.nkv) {
          if (!(ok = widen(it + 2 * (jj + 1), sKb, 128))) break;
          mbar_arrive(kb_full);
        }
        // V_jj once PV_{jj-1} has completed (the previous item's last PV was
        // waited on through o_full); rows past the valid length become zeros.
        if (jj > 0 && !(ok = mbar_wait_warp(pv_done, uint32_t((pvb + jj - 1) & 1), abort_flag))) break;
        if (!(ok = widen(it + 2 * jj + 1, sVb, I.L - 128 * j))) break;
        mbar_arrive(vb_full);

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
          // PV_{jj-1} has completed (waited above before widening V_jj).
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

}  // namespace attn
