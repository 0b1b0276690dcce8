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
// key columns [32w, 32w+32), four partials per item merged by LSE), with the
// cache tiles arriving as E4M3 bytes (TMA, 16 KB per tile):
//  - S = Q K8^T runs on the E4M3 key tile as it arrived (tcgen05.mma
//    kind::f8f6f4).  The query side is made E4M3 without losing precision:
//    each row is scaled by a power of two 2^k that puts its largest element in
//    [128, 256), and written as the sum of two E4M3 terms, hi = RN(q 2^k) and
//    lo = RN(q 2^k - hi).  Every element of magnitude >= 2^-2 after scaling
//    (>= 2^-10 of the row's largest) is represented exactly -- a bf16 value
//    has 8 significant bits and hi takes 4 of them, the rest fit lo -- and
//    smaller ones to within 2^-10 (the E4M3 subnormal step halved).  So
//    S = (hi K8^T + lo K8^T) / 2^k: two MMAs into one fp32 accumulator.
//  - PV keeps f16 operands: eight widening warps turn each E4M3 value tile
//    into an f16 tile in shared memory with integer operations only (exactly:
//    every E4M3 value times 2^-8 is an f16 value; the 2^8 goes into the
//    scale), and the softmax packs P as f16.
// The widening warps also split each work item's query box (double-buffered,
// loaded ahead); the softmax derives the same per-row power of two from the
// same box.  V_j is widened into one of two V tiles once PV_{j-2} has
// completed.  dk is
// folded into the exp2 argument and dv into the final 1/l.  Cache rows past
// the valid length are widened as zeros in V (their scores are masked).
// d = 128.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "attn_fwd_fp8.cuh"
#include "attn_kvcache.cuh"

namespace attn {

struct Kvc8Cfg {
  static constexpr int D = 128;
  static constexpr int kTileBytes = 128 * D * 2;       // f16 V tile
  static constexpr int kTile8Bytes = 128 * D;          // E4M3 tile: 128 rows x 128 bytes
  static constexpr int kBlockBytes = 128 * 128;
  static constexpr int kStageBlock = 32 * 128;         // bf16 query box: <= 32 rows per 64-column block
  static constexpr int kSlots = 6;                     // E4M3 ring: K in even, V in odd slots
  static constexpr int kVbufs = 2;                     // f16 V tiles
  static constexpr int kWarpMma = 4;
  static constexpr int kWarpLoad = 5;
  static constexpr int kWarpWiden0 = 6;                // warps 6 .. 6 + kWidenWarps - 1
  static constexpr int kWidenWarps = 8;
  static constexpr int kWidenThreads = 32 * kWidenWarps;
  static constexpr int kThreads = 32 * kWarpWiden0 + kWidenThreads;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
  static constexpr uint32_t kColP0 = 384, kColP1 = 448;
  static constexpr int kStageBytes = 2 * kStageBlock;              // one bf16 query box (2 blocks)
  static constexpr int kOffQs = 0;                                 // two query boxes
  static constexpr int kOffQh = kOffQs + 2 * kStageBytes;          // E4M3 hi terms, 4 copies
  static constexpr int kOffQl = kOffQh + kTile8Bytes;              // E4M3 lo terms, 4 copies
  static constexpr int kOffRing = kOffQl + kTile8Bytes;
  static constexpr int kOffVb = kOffRing + kSlots * kTile8Bytes;   // kVbufs f16 V tiles
  static constexpr int kOffBar = kOffVb + kVbufs * kTileBytes;
  // q_full[2], q_free[2], q_empty, ring_full[S], ring_empty[S], s_full[2], p_full[2], pv_done,
  // o_full, o_free, vb_full[kVbufs], vb_free[kVbufs], drain, q_ready
  static constexpr int kNumBars = 5 + 2 * kSlots + 2 + 2 + 3 + 2 * kVbufs + 1 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
};
static_assert(Kvc8Cfg::kSmemBytes <= 227 * 1024, "shared memory");
static_assert(Kvc8Cfg::kSlots % 2 == 0, "key tiles take the even ring slots, value tiles the odd ones");
static_assert(Kvc8Cfg::kOffQh % 1024 == 0 && Kvc8Cfg::kOffRing % 1024 == 0 && Kvc8Cfg::kOffVb % 1024 == 0,
              "128-byte swizzled tiles start on 1024-byte boundaries");

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
// dequantisation scale.  (The E4M3 NaN code reads as 2^-8 * 480.)
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

// The power of two that scales a query row whose largest magnitude is amax
// (finite, >= 0) into [128, 256) -- 2^(134 - E) for amax's biased exponent E
// -- returned as its biased exponent; E is clamped to [8, 254] so that both
// the factor and its inverse are normal floats.
__device__ __forceinline__ uint32_t q_split_exp(float amax) {
  const uint32_t e = min(max((__float_as_uint(amax) >> 23) & 0xFFu, 8u), 254u);
  return 261u - e;                          // biased exponent of 2^(134 - E)
}

// x -> (hi, lo) E4M3 pair terms for two values: hi = RN(x), lo = RN(x - hi).
__device__ __forceinline__ void split_e4m3x2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __nv_fp8x2_storage_t h = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const float2 hf = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(h, __NV_E4M3)));
  const __nv_fp8x2_storage_t l =
      __nv_cvt_float2_to_fp8x2(make_float2(a - hf.x, b - hf.y), __NV_SATFINITE, __NV_E4M3);
  hi = h;
  lo = l;
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

// The bf16 query box (rows < qbox <= 32; two [32][64] column blocks of 128
// swizzled bytes per row) -> E4M3 hi and lo tiles (128 swizzled bytes per
// row), each row written to all four lane-quarter copies (rows r, 32 + r,
// 64 + r, 96 + r).  Thread t handles elements 16c..16c+15 of row t / 8
// (c = t % 8): one 16-byte E4M3 chunk of each tile.  The row's scale comes
// from the maximum over its eight threads.
__device__ __forceinline__ void split_q_tile(uint32_t sqs, uint32_t sqh, uint32_t sql, int t, int qbox) {
  const int row = t >> 3;
  const int c = t & 7;
  const bool live = row < qbox;
  float x[16];
  float amax = 0.f;
  if (live) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int ch = (c & 3) * 2 + h;                       // bf16 chunk within column block c / 4
      const uint4 v = ld_shared_v4(sqs + (c >> 2) * Kvc8Cfg::kStageBlock + row * 128 + ((ch ^ (row & 7)) << 4));
      const uint32_t in[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        x[8 * h + 2 * k] = __uint_as_float(in[k] << 16);
        x[8 * h + 2 * k + 1] = __uint_as_float(in[k] & 0xFFFF0000u);
      }
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(x[k]));
  } else {
#pragma unroll
    for (int k = 0; k < 16; ++k) x[k] = 0.f;
  }
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
  if (!live) return;
  const float sq = __uint_as_float(q_split_exp(amax) << 23);
  uint32_t hw[4], lw[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint32_t h0, l0, h1, l1;
    split_e4m3x2(x[4 * k] * sq, x[4 * k + 1] * sq, h0, l0);
    split_e4m3x2(x[4 * k + 2] * sq, x[4 * k + 3] * sq, h1, l1);
    hw[k] = (h0 & 0xFFFFu) | (h1 << 16);
    lw[k] = (l0 & 0xFFFFu) | (l1 << 16);
  }
  const uint32_t off = row * 128 + ((c ^ (row & 7)) << 4);
#pragma unroll
  for (int cp = 0; cp < 4; ++cp) {
    st_shared_v4(sqh + cp * 32 * 128 + off, hw[0], hw[1], hw[2], hw[3]);
    st_shared_v4(sql + cp * 32 * 128 + off, lw[0], lw[1], lw[2], lw[3]);
  }
}

// The inverse of the same power of two, for the softmax: the largest
// magnitude of row `row` of the staged bf16 query box (128 values).
__device__ __forceinline__ float q_split_inverse(uint32_t sqs, int row) {
  float amax = 0.f;
#pragma unroll 4
  for (int k = 0; k < 16; ++k) {
    const uint4 v = ld_shared_v4(sqs + (k >> 3) * Kvc8Cfg::kStageBlock + row * 128 + (((k & 7) ^ (row & 7)) << 4));
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int u = 0; u < 4; ++u)
      amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(in[u] << 16)), fabsf(__uint_as_float(in[u] & 0xFFFF0000u))));
  }
  return __uint_as_float((254u - q_split_exp(amax)) << 23);   // 2^(E - 134): biased exponent E - 7
}

template <bool CAUSAL>
__global__ void __launch_bounds__(Kvc8Cfg::kThreads, 1)
attn_kvcache_fp8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k8,
                        const __grid_constant__ CUtensorMap tm_v8, const KvcParams prm,
                        const float v_descale) {
  using C = Kvc8Cfg;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;                 // [2]: query box b has landed
  uint64_t* q_free = q_full + 2;           // [2]: query box b has been split and read (may be reloaded)
  uint64_t* q_empty = q_free + 2;          // the last S product of an item has completed
  uint64_t* ring_full = q_empty + 1;
  uint64_t* ring_empty = ring_full + C::kSlots;
  uint64_t* s_full = ring_empty + C::kSlots;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* o_full = pv_done + 1;
  uint64_t* o_free = o_full + 1;
  uint64_t* vb_full = o_free + 1;          // [kVbufs]: f16 V tile b holds the next V tile for it
  uint64_t* vb_free = vb_full + C::kVbufs; // [kVbufs]: the PV product reading V tile b has completed
  uint64_t* drain = vb_free + C::kVbufs;
  uint64_t* q_ready = drain + 1;           // the query tile has been split into E4M3 terms
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&q_full[b], 1);
      mbar_init(&q_free[b], C::kWidenWarps + 4);   // the widening warps and the softmax warps
    }
    mbar_init(q_empty, 1);
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(&ring_full[s], 1);
      // key slots are released by the S product's commit, value slots by
      // the widening warps (one arrival each)
      mbar_init(&ring_empty[s], (s & 1) ? C::kWidenWarps : 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
    }
    mbar_init(pv_done, 1);
    mbar_init(o_full, 1);
    mbar_init(o_free, 128);
    for (int b = 0; b < C::kVbufs; ++b) {
      mbar_init(&vb_full[b], C::kWidenWarps);
      mbar_init(&vb_free[b], 1);
    }
    mbar_init(drain, 1);
    mbar_init(q_ready, C::kWidenWarps);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // The E4M3 query tiles: rows that are padding in every lane quarter are
  // never written again, so zero both tiles once.
  for (int i = threadIdx.x; i < 2 * C::kTile8Bytes / 16; i += C::kThreads)
    st_shared_v4(smem_u32(smem + C::kOffQh) + i * 16, 0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
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
        // the query box, once (the widening warps make the four copies), into
        // box qi & 1 once the box of item qi - 2 has been split
        const int qb = qi & 1;
        if (qi >= 2 && !(ok = mbar_wait(&q_free[qb], uint32_t(((qi >> 1) - 1) & 1), abort_flag))) break;
        mbar_arrive_expect_tx(&q_full[qb], uint32_t(prm.qbox * 128 * 2));
        for (int blk = 0; blk < 2; ++blk)
          tma_load_3d(&tm_q, &q_full[qb], smem + C::kOffQs + qb * C::kStageBytes + blk * C::kStageBlock, blk * 64,
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
      for (int q = max(0, qi - 2); q < qi; ++q) mbar_wait(&q_full[q & 1], uint32_t((q >> 1) & 1), abort_flag, false);
      for (int k = max(0, it - C::kSlots); k < it; ++k)
        mbar_wait(&ring_full[k % C::kSlots], uint32_t((k / C::kSlots) & 1), abort_flag, false);
    }
    __syncwarp();
  } else if (warp == C::kWarpMma) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_e4m3(128, 128, false, false);
      constexpr uint32_t kIdescPV = idesc_f16(128, D, false, true);
      const uint32_t sQh = smem_u32(smem + C::kOffQh);
      const uint32_t sQl = smem_u32(smem + C::kOffQl);
      const uint32_t sRing = smem_u32(smem + C::kOffRing);
      const uint32_t sVb = smem_u32(smem + C::kOffVb);
      int qi = 0, sc = 0, oi = 0, it = 0;
      bool ok = true;
      bool issued_any = false;
      for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
        const KvcItem I = kvc_item(prm, w, CAUSAL);
        if (I.nkv == 0) continue;
        if (!(ok = mbar_wait(q_ready, uint32_t(qi & 1), abort_flag))) break;
        for (int jj = 0; jj <= I.nkv && ok; ++jj) {
          if (jj < I.nkv) {
            // S_jj = (Qhi + Qlo) K8^T on the E4M3 key tile in its ring slot.
            // S buffer (sc + jj) & 1 was last read by the softmax of tile
            // jj - 2, whose P was waited for before PV_{jj-2} was issued.
            const int kit = it + 2 * jj;
            const int slot = kit % C::kSlots;
            if (!(ok = mbar_wait(&ring_full[slot], uint32_t((kit / C::kSlots) & 1), abort_flag))) break;
            tc_fence_after();
            const uint32_t dt = tmem + (((sc + jj) & 1) ? C::kColS1 : C::kColS0);
            const uint32_t sK = sRing + slot * C::kTile8Bytes;
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk)
              mma_ss_f8(dt, smem_desc_sw128(sQh + kk * 32, 16, 1024), smem_desc_sw128(sK + kk * 32, 16, 1024),
                        kIdescS, kk > 0 ? 1u : 0u);
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk)
              mma_ss_f8(dt, smem_desc_sw128(sQl + kk * 32, 16, 1024), smem_desc_sw128(sK + kk * 32, 16, 1024),
                        kIdescS, 1u);
            issued_any = true;
            mma_commit(&s_full[(sc + jj) & 1]);
            mma_commit(&ring_empty[slot]);
            if (jj == I.nkv - 1) mma_commit(q_empty);
          }
          if (jj > 0) {
            const int pj = jj - 1;
            const int ps = sc + pj;
            if (!(ok = mbar_wait(&p_full[ps & 1], uint32_t((ps >> 1) & 1), abort_flag))) break;
            if (pj == 0 && oi > 0 && !(ok = mbar_wait(o_free, uint32_t((oi - 1) & 1), abort_flag))) break;
            const int vb = ps % C::kVbufs;
            if (!(ok = mbar_wait(&vb_full[vb], uint32_t((ps / C::kVbufs) & 1), abort_flag))) break;
            tc_fence_after();
            const uint32_t at = tmem + ((ps & 1) ? C::kColP1 : C::kColP0);
#pragma unroll
            for (int kk = 0; kk < 128 / 16; ++kk)
              mma_ts(tmem + C::kColO, at + kk * 8,
                     smem_desc_sw128(sVb + vb * C::kTileBytes + kk * 2048, C::kBlockBytes, 1024), kIdescPV,
                     (pj > 0 || kk > 0) ? 1u : 0u);
            mma_commit(pj == I.nkv - 1 ? o_full : pv_done);
            mma_commit(&vb_free[vb]);
          }
        }
        it += 2 * I.nkv;
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
    // Per work item: split the query box into the E4M3 hi / lo tiles, then
    // widen V_jj for every key tile jj.  vc counts the V tiles widened over
    // all items; tile vc goes into buffer b = vc % kVbufs once the PV product
    // of the tile before it in that buffer has completed (vb_free[b]).
    const int t = threadIdx.x - 32 * C::kWarpWiden0;
    const uint32_t sRing = smem_u32(smem + C::kOffRing);
    const uint32_t sVb = smem_u32(smem + C::kOffVb);
    int it = 0, vc = 0, qi = 0;
    bool ok = true;

    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const KvcItem I = kvc_item(prm, w, CAUSAL);
      if (I.nkv == 0) continue;
      // The query box (loaded ahead, into box qi & 1); the E4M3 tiles are
      // free once the previous item's last S product has completed.  Every
      // thread fences its own shared-memory writes for the tensor core's
      // (async) proxy before its warp's single arrival.
      const int qb = qi & 1;
      if (!(ok = mbar_wait_warp(&q_full[qb], uint32_t((qi >> 1) & 1), abort_flag))) break;
      if (qi >= 1 && !(ok = mbar_wait_warp(q_empty, uint32_t((qi - 1) & 1), abort_flag))) break;
      split_q_tile(smem_u32(smem + C::kOffQs + qb * C::kStageBytes), smem_u32(smem + C::kOffQh),
                   smem_u32(smem + C::kOffQl), t, prm.qbox);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&q_free[qb]);
        mbar_arrive(q_ready);
      }
      ++qi;
      for (int jj = 0; jj < I.nkv; ++jj) {
        const int item = it + 2 * jj + 1;
        const int slot = item % C::kSlots;
        const int b = vc % C::kVbufs;
        if (vc >= C::kVbufs &&
            !(ok = mbar_wait_warp(&vb_free[b], uint32_t((vc / C::kVbufs - 1) & 1), abort_flag)))
          break;
        if (!(ok = mbar_wait_warp(&ring_full[slot], uint32_t((item / C::kSlots) & 1), abort_flag))) break;
        // rows past the valid length become zeros
        widen_tile(sRing + slot * C::kTile8Bytes, sVb + b * C::kTileBytes, t, I.L - 128 * (I.j_lo + jj));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&ring_empty[slot]);
          mbar_arrive(&vb_full[b]);
        }
        ++vc;
      }
      it += 2 * I.nkv;
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ softmax (warps 0-3)
    const int r = lane;                       // packed row (replicated in every lane quarter)
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const uint32_t tO = tmem + lane_base + C::kColO;
    int sc = 0, pvb = 0, oi = 0, qi = 0;
    bool ok = true;

    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      const KvcItem I = kvc_item(prm, w, CAUSAL);
      const int rp = I.r0 + r;
      const bool row_ok = r < I.r_valid;
      const long long row = (long long)I.bkv * prm.rows + rp;
      int lim = I.L - 1;
      if (CAUSAL) lim = min(lim, rp % prm.nq + I.L - prm.nq);
      float m_ref = -INFINITY;
      float l = 0.f;
      // scale * dk * log2(e), divided by the power of two this row's query
      // terms carry (from the same query box the widening warps split; the
      // box is reloaded only after every warp has read it)
      float c = 0.f;
      if (I.nkv > 0) {
        const int qb = qi & 1;
        if (!(ok = mbar_wait_warp(&q_full[qb], uint32_t((qi >> 1) & 1), abort_flag))) break;
        if (row_ok) c = prm.scale_log2 * q_split_inverse(smem_u32(smem + C::kOffQs + qb * C::kStageBytes), r);
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_free[qb]);
        ++qi;
      }

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
