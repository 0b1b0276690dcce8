// attn_fwd_fp8.cuh -- forward attention on FP8 (E4M3) Q, K, V with per-tensor
// dequantisation factors, fp32 accumulation, bf16 output.
//
// The computation is the square forward's ("Attention and KV Compression",
// sections "Tiling and online softmax" and "What it does and does not change":
// later versions add narrower numeric formats without changing what is
// computed), on the dequantised inputs Q = dq*Q8, K = dk*K8, V = dv*V8:
//   * S = Q8 K8^T by tcgen05.mma kind::f8f6f4 (E4M3 x E4M3 products are exact
//     in the fp32 accumulator); the factor scale*dq*dk is folded into the exp2
//     argument together with log2(e).
//   * The running max, the row sum l and LSE are fp32, from the unrounded p.
//   * P (in [0, 2^8] thanks to the lazy rescale) is rounded to E4M3 for the PV
//     product, O += P8 V8 (kind::f8f6f4, P read from TMEM, V MN-major); the
//     output is dv * O / l in bf16.  The rounding of P is the one step that is
//     not exact: each p changes by at most 2^-4 of itself or 2^-10 absolute.
//
// Layout and roles follow the bf16 forward (two 128-row query tiles per CTA,
// warp 9 TMA, warp 8 MMA, warps 0-3 / 4-7 softmax of tile 0 / 1, warps 10-11
// idle, the same register split, S and O in TMEM), with d = 128 only: one 128-byte swizzled row holds a full 128-wide
// E4M3 row, tiles are 16 KB, and the K/V ring has 8 slots.  The epilogue
// stores each thread's O row straight to global memory.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "sm100.cuh"

namespace attn {

constexpr float kFp8RescaleLog2 = 8.0f;
constexpr float kFp8Ln2 = 0.6931471805599453f;

struct Fp8Params {
  __nv_bfloat16* o;   // [B*H][N][128] bf16
  float* lse;         // [B*H][N]
  int n;
  int n_mblk;         // 256-row query blocks per head
  int h, h_kv, group;
  float c;            // scale * dq * dk * log2(e): exp2 argument per raw score
  float v_descale;    // dv
};

struct Fp8Cfg {
  static constexpr int kTileBytes = 128 * 128;          // 128 rows x 128 E4M3
  static constexpr int kSlots = 8;
  // Warps 0-7 softmax, warpgroup 2 = MMA, TMA and two idle warps; launched
  // with 168 registers per thread (three warpgroup slots), warpgroup 2 gives
  // registers back and the softmax warpgroups take them (setmaxnreg):
  // 2 * kRegsSoftmax + kRegsIssue = 3 * 168.  The host refuses to launch
  // unless the kernel compiled to exactly kRegsLaunch.
  static constexpr int kThreads = 384;
  static constexpr int kWarpMma = 8;
  static constexpr int kWarpLoad = 9;
  static constexpr uint32_t kRegsLaunch = 168;
  static constexpr uint32_t kRegsIssue = 152;
  static constexpr uint32_t kRegsSoftmax = 176;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128;
  static constexpr uint32_t kColO0 = 256, kColO1 = 384;
  static constexpr uint32_t kColPOff = 96;               // P: 128 E4M3 = 32 columns over S 96..127
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = 2 * kTileBytes;
  static constexpr int kOffBar = kOffKV + kSlots * kTileBytes;
  static constexpr int kNumBars = 2 + 2 * kSlots + 2 + 2 + 2 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static_assert(2 * kRegsSoftmax + kRegsIssue <= 3 * kRegsLaunch, "register split");
};

// Instruction descriptor, kind::f8f6f4 with E4M3 A and B (format code 0) and
// fp32 D: same bit positions as the kind::f16 descriptor.
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}\n"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 8 consecutive columns.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

// Four fp32 -> four E4M3 (round to nearest even, saturating to +-448) in one
// 32-bit word, the element with the lowest key index in the lowest byte.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return (lo & 0xFFFFu) | (hi << 16);
}

template <bool CAUSAL>
__global__ void __launch_bounds__(384, 1)
attn_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const Fp8Params prm) {
  using C = Fp8Cfg;
  constexpr int D = 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = q_full + 2;
  uint64_t* kv_empty = kv_full + C::kSlots;
  uint64_t* s_full = kv_empty + C::kSlots;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* drain = o_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n = prm.n;
  const int bh = blockIdx.x / prm.n_mblk;
  const int bkv = (bh / prm.h) * prm.h_kv + (bh % prm.h) / prm.group;
  const int m_blk = prm.n_mblk - 1 - (blockIdx.x % prm.n_mblk);   // heaviest causal blocks first
  const int m0 = m_blk * 256;
  const int n_kv_total = (n + 127) >> 7;
  const int nkv = CAUSAL ? min(n_kv_total, (m0 >> 7) + 2) : n_kv_total;
  // Causal: key tile 2m+1 (the last one, when N does not cut it off) starts
  // after the last row of query tile 0, so only tile 1 visits it.
  const int nkv0 = (CAUSAL && nkv == (m0 >> 7) + 2) ? nkv - 1 : nkv;

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(&q_full[t], 1);
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      mbar_init(&o_full[t], 1);
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
   regs_dec<C::kRegsIssue>();
   if (warp == C::kWarpLoad) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      for (int t = 0; t < 2; ++t) {
        mbar_arrive_expect_tx(&q_full[t], C::kTileBytes);
        tma_load_3d(&tm_q, &q_full[t], smem + C::kOffQ + t * C::kTileBytes, 0, m0 + 128 * t, bh);
      }
      int issued = 0;
      for (int it = 0; it < 2 * nkv; ++it) {
        const int slot = it % C::kSlots;
        const int use = it / C::kSlots;
        if (use > 0 && !mbar_wait(&kv_empty[slot], (use - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(&kv_full[slot], C::kTileBytes);
        tma_load_3d((it & 1) ? &tm_v : &tm_k, &kv_full[slot], smem + C::kOffKV + slot * C::kTileBytes, 0,
                    128 * (it >> 1), bkv);
        ++issued;
      }
      // No copy may still be landing in shared memory when the CTA leaves.
      mbar_wait(&q_full[0], 0, abort_flag, false);
      mbar_wait(&q_full[1], 0, abort_flag, false);
      for (int it = max(0, issued - C::kSlots); it < issued; ++it)
        mbar_wait(&kv_full[it % C::kSlots], (it / C::kSlots) & 1, abort_flag, false);
    }
    __syncwarp();
   } else if (warp == C::kWarpMma) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_e4m3(128, 128, false, false);
      constexpr uint32_t kIdescPV = idesc_e4m3(128, D, false, true);
      const uint32_t sQ = smem_u32(smem + C::kOffQ);
      const uint32_t sKV = smem_u32(smem + C::kOffKV);
      int it = 0;
      auto wait_kv = [&](int& slot) -> bool {
        slot = it % C::kSlots;
        const bool r = mbar_wait(&kv_full[slot], (it / C::kSlots) & 1, abort_flag);
        ++it;
        return r;
      };
      // K-major E4M3 operands: a k-step of 32 elements is 32 bytes inside the
      // 128-byte swizzled row, exactly as a 16-element bf16 step.
      auto issue_s = [&](int t, int kslot) {
        const uint32_t a0 = sQ + t * C::kTileBytes;
        const uint32_t b0 = sKV + kslot * C::kTileBytes;
        const uint32_t dt = tmem + (t ? C::kColS1 : C::kColS0);
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
          mma_ss_f8(dt, smem_desc_sw128(a0 + kk * 32, 16, 1024), smem_desc_sw128(b0 + kk * 32, 16, 1024), kIdescS,
                    kk > 0 ? 1u : 0u);
      };
      // V MN-major: the 128 output columns are one 128-byte swizzle atom; a
      // k-step of 32 keys is 32 rows = 4096 bytes.  P: 32 keys = 8 columns.
      auto issue_pv = [&](int t, int vslot, bool acc) {
        const uint32_t b0 = sKV + vslot * C::kTileBytes;
        const uint32_t dt = tmem + (t ? C::kColO1 : C::kColO0);
        const uint32_t at = tmem + (t ? C::kColS1 : C::kColS0) + C::kColPOff;
#pragma unroll
        for (int kk = 0; kk < 128 / 32; ++kk)
          mma_ts_f8(dt, at + kk * 8, smem_desc_sw128(b0 + kk * 4096, C::kTileBytes, 1024), kIdescPV,
                    (acc || kk > 0) ? 1u : 0u);
      };

      bool ok = mbar_wait(&q_full[0], 0, abort_flag) && mbar_wait(&q_full[1], 0, abort_flag);
      if (ok) {
        int ks;
        ok = wait_kv(ks);
        if (ok) {
          tc_fence_after();
          issue_s(0, ks);
          mma_commit(&s_full[0]);
          issue_s(1, ks);
          mma_commit(&s_full[1]);
          mma_commit(&kv_empty[ks]);
        }
      }
      for (int j = 1; j < nkv && ok; ++j) {
        int vs, ks;
        if (!(ok = wait_kv(vs))) break;
        if (!(ok = wait_kv(ks))) break;
        for (int t = 0; t < 2; ++t) {
          if (!(ok = mbar_wait(&p_full[t], (j - 1) & 1, abort_flag))) break;
          tc_fence_after();
          issue_pv(t, vs, j - 1 > 0);
          if (t == 1) mma_commit(&kv_empty[vs]);
          if (t == 0 && j >= nkv0) continue;     // key tile j is wholly masked for tile 0
          issue_s(t, ks);
          mma_commit(&s_full[t]);
        }
        if (ok) mma_commit(&kv_empty[ks]);
      }
      if (ok) {
        int vs;
        ok = wait_kv(vs);
        for (int t = 0; t < 2 && ok; ++t) {
          if (t == 1 || nkv - 1 < nkv0) {
            if (!(ok = mbar_wait(&p_full[t], (nkv - 1) & 1, abort_flag))) break;
            tc_fence_after();
            issue_pv(t, vs, nkv - 1 > 0);
          }
          mma_commit(&o_full[t]);                 // after the tile's last PV
        }
        if (ok) mma_commit(&kv_empty[vs]);
      }
      mma_commit(drain);
      mbar_wait(drain, 0, abort_flag, false);
    }
    __syncwarp();
   }
  } else {
    // -------------------------------------------------------------- softmax
    regs_inc<C::kRegsSoftmax>();
    const int t = warp >> 2;
    const int qw = warp & 3;
    const int r = qw * 32 + lane;
    const int i = m0 + 128 * t + r;
    const uint32_t lane_base = uint32_t(qw * 32) << 16;
    const uint32_t tS = tmem + lane_base + (t ? C::kColS1 : C::kColS0);
    const uint32_t tP = tS + C::kColPOff;
    const uint32_t tO = tmem + lane_base + (t ? C::kColO1 : C::kColO0);
    const float c = prm.c;
    float m_ref = -INFINITY;
    float l = 0.f;
    bool ok = true;

    const int nkv_t = (t == 0) ? nkv0 : nkv;   // key tiles this query tile visits
    for (int j = 0; j < nkv_t; ++j) {
      if (!(ok = mbar_wait_warp(&s_full[t], j & 1, abort_flag))) break;
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
      const bool need_mask = (CAUSAL && (128 * j + 127 > m0 + 128 * t)) || (128 * j + 128 > n);
      if (need_mask) {
        int limit = n - 1 - 128 * j;
        if (CAUSAL) limit = min(limit, i - 128 * j);
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
      if (m_tile > m_ref + kFp8RescaleLog2) {
        alpha = ex2(m_ref - m_tile);
        m_ref = m_tile;
        rescale = (j > 0);
      }
      l *= alpha;
      const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
      float sump[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q = 0; q < 4; ++q) {            // 32 keys -> 8 columns of four E4M3 each
        uint32_t pk[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float p0 = ex2(fmaf(s[32 * q + 4 * k], c, neg_m));
          const float p1 = ex2(fmaf(s[32 * q + 4 * k + 1], c, neg_m));
          const float p2 = ex2(fmaf(s[32 * q + 4 * k + 2], c, neg_m));
          const float p3 = ex2(fmaf(s[32 * q + 4 * k + 3], c, neg_m));
          sump[k & 3] += (p0 + p1) + (p2 + p3);
          pk[k] = pack_e4m3x4(p0, p1, p2, p3);
        }
        tmem_st8(tP + 8 * q, pk);
      }
      l += (sump[0] + sump[1]) + (sump[2] + sump[3]);
      if (__any_sync(0xffffffffu, rescale)) {
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

    // ------------------------------------------------------------ epilogue
    if (ok) ok = mbar_wait_warp(&o_full[t], 0, abort_flag);
    if (ok) {
      tc_fence_after();
      const float f = prm.v_descale / l;
      uint32_t orow[D / 32][32];              // the whole row: one TMEM round trip
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) tmem_ld32(tO + cc * 32, orow[cc]);
      tmem_ld_wait(orow[0]);
#pragma unroll
      for (int cc = 1; cc < D / 32; ++cc) reg_fence32(orow[cc]);
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        const uint32_t (&o)[32] = orow[cc];
        if (i < n) {
          uint4* dst = reinterpret_cast<uint4*>(prm.o + (size_t(bh) * size_t(n) + size_t(i)) * D + cc * 32);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            dst[k] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * k + 0]) * f, __uint_as_float(o[8 * k + 1]) * f),
                                pack_bf16x2(__uint_as_float(o[8 * k + 2]) * f, __uint_as_float(o[8 * k + 3]) * f),
                                pack_bf16x2(__uint_as_float(o[8 * k + 4]) * f, __uint_as_float(o[8 * k + 5]) * f),
                                pack_bf16x2(__uint_as_float(o[8 * k + 6]) * f, __uint_as_float(o[8 * k + 7]) * f));
        }
      }
      if (i < n) prm.lse[size_t(bh) * size_t(n) + size_t(i)] = (m_ref + __log2f(l)) * kFp8Ln2;
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
