// attn_api.cu -- host side of the C ABI declared in include/attn.h:
// argument checks, TMA tensor maps, kernel selection and launches.
//
// The library allocates no device memory: tensor maps travel as
// __grid_constant__ kernel parameters, the backward's per-row vectors live in
// the caller's workspace, and the only device state is the status word
// g_attn_status (a static __device__ variable).

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdarg>
#include <cstdio>
#include <map>
#include <mutex>
#include <queue>
#include <tuple>
#include <vector>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/attn.h"
#include "attn_bwd.cuh"
#include "attn_bwd_fused.cuh"
#include "attn_fwd.cuh"
#include "attn_fwd_fp8.cuh"
#include "attn_kvcache.cuh"
#include "attn_kvcache_fp8.cuh"

namespace {

// Detail of the most recent failure on this host thread (attn_last_error).
thread_local char g_last_error[256] = "";

__attribute__((format(printf, 2, 3))) int fail(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return status;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D map over a BHND bf16 tensor viewed as [B*H][N][d]; box = 64 columns x
// box_rows rows x 1 head, 128-byte swizzle.  Rows past N read as zeros; stores
// past N are dropped.
bool make_map(CUtensorMap* m, const void* base, int64_t bh, int64_t n, int64_t d, int box_rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    fail(ATTN_ERR_LAUNCH, "driver entry point cuTensorMapEncodeTiled unavailable");
    return false;
  }
  const cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(n), cuuint64_t(bh)};
  const cuuint64_t strides[2] = {cuuint64_t(d * 2), cuuint64_t(n * d * 2)};
  const cuuint32_t box[3] = {64, cuuint32_t(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    fail(ATTN_ERR_LAUNCH, "cuTensorMapEncodeTiled returned CUresult %lld", (long long)r);
    return false;
  }
  return true;
}

// 3-D map over an E4M3 (byte) BHND tensor with d = 128: box = one 128-byte
// row x 128 rows x 1 head, 128-byte swizzle.  Rows past N read as zeros.
bool make_map_u8(CUtensorMap* m, const void* base, int64_t bh, int64_t n, int64_t d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    fail(ATTN_ERR_LAUNCH, "driver entry point cuTensorMapEncodeTiled unavailable");
    return false;
  }
  const cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(n), cuuint64_t(bh)};
  const cuuint64_t strides[2] = {cuuint64_t(d), cuuint64_t(n * d)};
  const cuuint32_t box[3] = {128, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    fail(ATTN_ERR_LAUNCH, "cuTensorMapEncodeTiled returned CUresult %lld", (long long)r);
    return false;
  }
  return true;
}

// 3-D map over the fp32 dQ accumulator [B*H][Npad][d] (rows past N are never
// touched: the map's extent is N, so reduce rows past N are dropped); box = 32
// fp32 columns (128 bytes) x 128 rows x 1 head, 128-byte swizzle.
bool make_map_f32_acc(CUtensorMap* m, const void* base, int64_t bh, int64_t n, int64_t npad, int64_t d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    fail(ATTN_ERR_LAUNCH, "driver entry point cuTensorMapEncodeTiled unavailable");
    return false;
  }
  const cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(n), cuuint64_t(bh)};
  const cuuint64_t strides[2] = {cuuint64_t(d * 4), cuuint64_t(npad * d * 4)};
  const cuuint32_t box[3] = {32, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    fail(ATTN_ERR_LAUNCH, "cuTensorMapEncodeTiled (fp32 accumulator) returned CUresult %lld", (long long)r);
    return false;
  }
  return true;
}

constexpr int64_t kNumSMs = 148;   // B200: sizes the persistent grids and the automatic split count

// 3-D map over a packed [total][H][d] bf16 tensor (coordinates x, head,
// token); box = 64 columns x 1 head x 128 tokens, 128-byte swizzle: the same
// shared-memory tile as make_map's.  Tokens past `total` read as zeros.
bool make_map_packed(CUtensorMap* m, const void* base, int64_t total, int64_t h, int64_t d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    fail(ATTN_ERR_LAUNCH, "driver entry point cuTensorMapEncodeTiled unavailable");
    return false;
  }
  const cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(h), cuuint64_t(total)};
  const cuuint64_t strides[2] = {cuuint64_t(d * 2), cuuint64_t(h * d * 2)};
  const cuuint32_t box[3] = {64, 1, 128};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    fail(ATTN_ERR_LAUNCH, "cuTensorMapEncodeTiled (packed) returned CUresult %lld", (long long)r);
    return false;
  }
  return true;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_sizes(int64_t B, int64_t H, int64_t N, int64_t d) {
  if (B < 1 || H < 1 || N < 1) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (B > INT32_MAX / H || N > INT32_MAX - 256) return ATTN_ERR_INVALID_ARG;
  const int64_t bh = B * H;
  const int64_t nt = (N + 127) / 128;
  if (nt > INT32_MAX / bh) return ATTN_ERR_INVALID_ARG;   // grid size
  return ATTN_OK;
}

int check_heads(int64_t H, int64_t H_kv) {
  if (H_kv < 1 || H_kv > H || H % H_kv != 0) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

int check_scale(float scale) { return (std::isfinite(scale) && scale > 0.f) ? ATTN_OK : ATTN_ERR_INVALID_ARG; }

int launch_status() {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return ATTN_OK;
  return fail(ATTN_ERR_LAUNCH, "kernel launch: %s (%lld)", cudaGetErrorString(e), (long long)e);
}

int set_smem(const void* kern, int bytes) {
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) return ATTN_OK;
  return fail(ATTN_ERR_LAUNCH, "cudaFuncSetAttribute(max dynamic smem): %s (bytes %lld)", cudaGetErrorString(e),
              (long long)bytes);
}

// Kernels that move registers between their warpgroups (setmaxnreg) are only
// correct when every thread was launched with exactly the count the split
// assumes (otherwise a growing warpgroup would wait for registers that never
// come), so each launch checks the compiled count.  It is a property of the
// compiled kernel, queried once per kernel (a failed query is not cached).
template <auto KERN>
int check_launch_regs(int want, const char* what) {
  static std::atomic<int> cached{0};
  int regs = cached.load(std::memory_order_relaxed);
  if (regs == 0) {
    cudaFuncAttributes fa;
    const cudaError_t e = cudaFuncGetAttributes(&fa, KERN);
    if (e != cudaSuccess)
      return fail(ATTN_ERR_LAUNCH, "cudaFuncGetAttributes(%s): %s (%lld)", what, cudaGetErrorString(e), (long long)e);
    regs = fa.numRegs;
    cached.store(regs, std::memory_order_relaxed);
  }
  if (regs != want)
    return fail(ATTN_ERR_LAUNCH, "%s compiled to %d registers per thread, its warpgroup split needs %d", what, regs,
                want);
  return ATTN_OK;
}

template <int D, bool CAUSAL, bool SPARSE, bool O32 = false, bool VARLEN = false>
int launch_fwd(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const attn::FwdParams& prm,
               int grid, cudaStream_t st) {
  using C = attn::FwdCfg<D>;
  auto kern = attn::attn_fwd_kernel<D, CAUSAL, SPARSE, O32, VARLEN>;
  constexpr int smem = C::kSmemBytes;
  if (check_launch_regs<attn::attn_fwd_kernel<D, CAUSAL, SPARSE, O32, VARLEN>>(int(C::kRegsLaunch), "forward") !=
      ATTN_OK)
    return ATTN_ERR_LAUNCH;
  if (set_smem(reinterpret_cast<const void*>(kern), smem) != ATTN_OK) return ATTN_ERR_LAUNCH;
  kern<<<grid, attn::FwdCfg<D>::kThreads, smem, st>>>(q, k, v, prm);
  return launch_status();
}

template <int D, bool CAUSAL, bool SPARSE>
int launch_dkdv(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const CUtensorMap& dO,
                const CUtensorMap& dk, const CUtensorMap& dv, const attn::BwdParams& prm, int grid, cudaStream_t st) {
  using C = attn::BwdCfg<D>;
  auto kern = attn::attn_bwd_dkdv_kernel<D, CAUSAL, SPARSE>;
  if (set_smem(reinterpret_cast<const void*>(kern), C::kKV_SmemBytes) != ATTN_OK) return ATTN_ERR_LAUNCH;
  kern<<<grid, C::kThreads, C::kKV_SmemBytes, st>>>(q, k, v, dO, dk, dv, prm);
  return launch_status();
}

template <int D, bool CAUSAL, bool SPARSE>
int launch_dq(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const CUtensorMap& dO,
              const CUtensorMap& dq, const attn::BwdParams& prm, int grid, cudaStream_t st) {
  using C = attn::BwdCfg<D>;
  auto kern = attn::attn_bwd_dq_kernel<D, CAUSAL, SPARSE>;
  if (set_smem(reinterpret_cast<const void*>(kern), C::kQ_SmemBytes) != ATTN_OK) return ATTN_ERR_LAUNCH;
  kern<<<grid, C::kThreads, C::kQ_SmemBytes, st>>>(q, k, v, dO, dq, prm);
  return launch_status();
}

template <int D>
int launch_bwd_pre(const void* O, const void* dO, const float* lse, float* ws_lse2, float* ws_d, int n, int npad,
                   int64_t rows_pad, cudaStream_t st, float* dq_acc = nullptr) {
  constexpr int rows_per_block = 256 / (D / 8);
  int64_t blocks = (rows_pad + rows_per_block - 1) / rows_per_block;
  if (blocks > 148 * 32) blocks = 148 * 32;
  const __nv_bfloat16* o = static_cast<const __nv_bfloat16*>(O);
  const __nv_bfloat16* d_o = static_cast<const __nv_bfloat16*>(dO);
  if (dq_acc)
    attn::attn_bwd_pre_kernel<D, true><<<int(blocks), 256, 0, st>>>(o, d_o, lse, ws_lse2, ws_d, n, npad,
                                                                    static_cast<long long>(rows_pad), dq_acc);
  else
    attn::attn_bwd_pre_kernel<D, false><<<int(blocks), 256, 0, st>>>(o, d_o, lse, ws_lse2, ws_d, n, npad,
                                                                     static_cast<long long>(rows_pad));
  return launch_status();
}

template <int D, bool CAUSAL, bool SPARSE>
int launch_fused(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const CUtensorMap& dO,
                 const CUtensorMap& dk, const CUtensorMap& dv, const CUtensorMap& dqacc, const attn::BwdParams& prm,
                 int grid, cudaStream_t st) {
  using C = attn::FusedCfg<D>;
  auto kern = attn::attn_bwd_fused_kernel<D, CAUSAL, SPARSE>;
  if (check_launch_regs<attn::attn_bwd_fused_kernel<D, CAUSAL, SPARSE>>(int(C::kRegsLaunch), "fused backward") !=
      ATTN_OK)
    return ATTN_ERR_LAUNCH;
  if (set_smem(reinterpret_cast<const void*>(kern), C::kSmemBytes) != ATTN_OK) return ATTN_ERR_LAUNCH;
  kern<<<grid, C::kThreads, C::kSmemBytes, st>>>(q, k, v, dO, dk, dv, dqacc, prm);
  return launch_status();
}

template <int D>
int launch_dq_convert(const float* dq_acc, void* dQ, int n, int npad, int64_t rows, float scale, cudaStream_t st) {
  constexpr int rows_per_block = 256 / (D / 8);
  int64_t blocks = (rows + rows_per_block - 1) / rows_per_block;
  if (blocks > 148 * 32) blocks = 148 * 32;
  attn::attn_bwd_dq_convert_kernel<D><<<int(blocks), 256, 0, st>>>(dq_acc, static_cast<__nv_bfloat16*>(dQ), n, npad,
                                                                    static_cast<long long>(rows), scale);
  return launch_status();
}

int64_t npad_of(int64_t N) { return (N + 127) / 128 * 128; }

// Selects the kernel instance for head dim, causal mask and block sparsity.
#define ATTN_DISPATCH(FN, ...)                                                                       \
  (d == 128 ? (causal ? (sparse ? FN<128, true, true>(__VA_ARGS__) : FN<128, true, false>(__VA_ARGS__))  \
                      : (sparse ? FN<128, false, true>(__VA_ARGS__) : FN<128, false, false>(__VA_ARGS__))) \
            : (causal ? (sparse ? FN<64, true, true>(__VA_ARGS__) : FN<64, true, false>(__VA_ARGS__))    \
                      : (sparse ? FN<64, false, true>(__VA_ARGS__) : FN<64, false, false>(__VA_ARGS__))))

}  // namespace

#define ATTN_EXPORT __attribute__((visibility("default")))

extern "C" {

}  // extern "C"

namespace {

// Grid size and dealing order of the persistent forward.  A causal item of
// query block m visits min(nt, 2m + 2) key tiles, so items differ in cost; the
// items are dealt in rounds of one per CTA, and the pair (grid size, plain or
// snake order) that gives the smallest predicted makespan -- the largest sum
// of item costs on one CTA, each item also charged a fixed 3 key tiles for its
// set-up and output -- is chosen once per shape and cached, unless one CTA per
// item (scheduled greedily by the hardware) is predicted to finish first.
// Non-causal items all cost the same; block-sparse costs depend on the mask
// (device data), so both use the plain order on every SM.
struct FwdSched {
  int grid;
  int snake;
};

FwdSched fwd_schedule(int64_t bh, int64_t n_mblk, int64_t nt, bool causal, bool sparse) {
  const int64_t items = bh * n_mblk;
  if (items <= kNumSMs) return {int(items), 0};
  if (!causal || sparse) return {int(kNumSMs), 0};
  if (items > 65536) return {int(kNumSMs), 1};
  static std::mutex mu;
  static std::map<std::tuple<int64_t, int64_t, int64_t>, FwdSched> cache;
  const auto key = std::make_tuple(bh, n_mblk, nt);
  {
    std::lock_guard<std::mutex> lock(mu);
    auto f = cache.find(key);
    if (f != cache.end()) return f->second;
  }
  constexpr int64_t kFixed = 3;
  // One CTA per item (grid = items): the hardware hands each SM the next item
  // when it frees up (greedy, in item order), and each item also pays the
  // set-up and drain that the persistent loop overlaps (about one key tile).
  FwdSched best{int(items), 0};
  int64_t best_cost = 0;
  {
    std::priority_queue<int64_t, std::vector<int64_t>, std::greater<int64_t>> sm;
    for (int64_t c = 0; c < kNumSMs; ++c) sm.push(0);
    for (int64_t i = 0; i < items; ++i) {
      const int64_t m = n_mblk - 1 - i % n_mblk;
      const int64_t t = sm.top() + std::min(nt, 2 * m + 2) + kFixed + 1;
      sm.pop();
      sm.push(t);
      best_cost = std::max(best_cost, t);
    }
  }
  std::vector<int64_t> load(size_t(kNumSMs), 0);
  for (int64_t g = kNumSMs; g >= kNumSMs - 28; --g) {
    for (int snake = 0; snake < 2; ++snake) {
      std::fill(load.begin(), load.begin() + g, 0);
      for (int64_t i = 0; i < items; ++i) {
        const int64_t r = i / g;
        int64_t c = i - r * g;
        if (snake && (r & 1)) c = g - 1 - c;
        const int64_t m = n_mblk - 1 - i % n_mblk;
        load[size_t(c)] += std::min(nt, 2 * m + 2) + kFixed;
      }
      const int64_t cost = *std::max_element(load.begin(), load.begin() + g);
      if (cost < best_cost) {
        best_cost = cost;
        best = {int(g), snake};
      }
    }
  }
  std::lock_guard<std::mutex> lock(mu);
  cache[key] = best;
  return best;
}

int fwd_impl(const void* Q, const void* K, const void* V, void* O, float* LSE, const uint8_t* mask, int64_t B,
             int64_t H, int64_t H_kv, int64_t N, int64_t d, int causal, float scale, void* stream,
             float* O32 = nullptr) {
  int s = check_sizes(B, H, N, d);
  if (s != ATTN_OK) return s;
  if ((s = check_heads(H, H_kv)) != ATTN_OK) return s;
  if ((s = check_scale(scale)) != ATTN_OK) return s;
  if (!Q || !K || !V || !O || !LSE) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE) ||
      (O32 && !aligned16(O32)))
    return ATTN_ERR_MISALIGNED;
  const int64_t bh = B * H, bhkv = B * H_kv;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, Q, bh, N, d) || !make_map(&mk, K, bhkv, N, d) || !make_map(&mv, V, bhkv, N, d))
    return ATTN_ERR_LAUNCH;
  attn::FwdParams prm = {};
  prm.o = static_cast<__nv_bfloat16*>(O);
  prm.lse = LSE;
  prm.n = int(N);
  prm.n_mblk = int((N + 255) / 256);
  prm.h = int(H);
  prm.h_kv = int(H_kv);
  prm.group = int(H / H_kv);
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.mask = mask;
  prm.nt = int((N + 127) / 128);
  prm.o32 = O32;
  const bool sparse = mask != nullptr;
  const int64_t items = bh * prm.n_mblk;
  if (items > INT32_MAX) return ATTN_ERR_INVALID_ARG;
  prm.n_items = int(items);
  const FwdSched sched = fwd_schedule(bh, prm.n_mblk, prm.nt, causal != 0, sparse);
  prm.snake = sched.snake;
  const int grid = sched.grid;   // persistent: at most one CTA per SM
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (O32)
    return d == 128 ? (causal ? launch_fwd<128, true, false, true>(mq, mk, mv, prm, grid, st)
                              : launch_fwd<128, false, false, true>(mq, mk, mv, prm, grid, st))
                    : (causal ? launch_fwd<64, true, false, true>(mq, mk, mv, prm, grid, st)
                              : launch_fwd<64, false, false, true>(mq, mk, mv, prm, grid, st));
  return ATTN_DISPATCH(launch_fwd, mq, mk, mv, prm, grid, st);
}

}  // namespace

extern "C" {

ATTN_EXPORT int attn_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int64_t B, int64_t H,
                         int64_t N, int64_t d, int causal, float scale, void* stream) {
  return fwd_impl(Q, K, V, O, LSE, nullptr, B, H, H, N, d, causal, scale, stream);
}

ATTN_EXPORT int attn_fwd_varlen(const void* Q, const void* K, const void* V, void* O, float* LSE,
                                const int32_t* cu_seqlens, int64_t n_seqs, int64_t total, int64_t H, int64_t H_kv,
                                int64_t d, int causal, float scale, void* stream) {
  if (n_seqs < 1 || total < 1 || H < 1) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  int s = check_heads(H, H_kv);
  if (s != ATTN_OK) return s;
  if ((s = check_scale(scale)) != ATTN_OK) return s;
  // item counts (heads x 256-row blocks per sequence) and row indices must fit in 31 bits
  if (n_seqs > INT32_MAX - 1 || total > INT32_MAX - 256 || H * ((total + 255) / 256 + n_seqs) > INT32_MAX)
    return ATTN_ERR_INVALID_ARG;
  if (!Q || !K || !V || !O || !LSE || !cu_seqlens) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE))
    return ATTN_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return ATTN_ERR_MISALIGNED;
  CUtensorMap mq, mk, mv;
  if (!make_map_packed(&mq, Q, total, H, d) || !make_map_packed(&mk, K, total, H_kv, d) ||
      !make_map_packed(&mv, V, total, H_kv, d))
    return ATTN_ERR_LAUNCH;
  attn::FwdParams prm = {};
  prm.o = static_cast<__nv_bfloat16*>(O);
  prm.lse = LSE;
  prm.h = int(H);
  prm.h_kv = int(H_kv);
  prm.group = int(H / H_kv);
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.cu_seqlens = cu_seqlens;
  prm.n_seqs = int(n_seqs);
  prm.total = int(total);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the item count depends on the lengths (device data): a CTA per SM, plain dealing
  const int grid = int(kNumSMs);
  if (d == 128)
    return causal ? launch_fwd<128, true, false, false, true>(mq, mk, mv, prm, grid, st)
                  : launch_fwd<128, false, false, false, true>(mq, mk, mv, prm, grid, st);
  return causal ? launch_fwd<64, true, false, false, true>(mq, mk, mv, prm, grid, st)
                : launch_fwd<64, false, false, false, true>(mq, mk, mv, prm, grid, st);
}

ATTN_EXPORT int attn_fwd_f32out(const void* Q, const void* K, const void* V, void* O, float* O32, float* LSE,
                                int64_t B, int64_t H, int64_t N, int64_t d, int causal, float scale, void* stream) {
  if (!O32) return ATTN_ERR_INVALID_ARG;
  return fwd_impl(Q, K, V, O, LSE, nullptr, B, H, H, N, d, causal, scale, stream, O32);
}

ATTN_EXPORT int attn_fwd_gqa(const void* Q, const void* K, const void* V, void* O, float* LSE, int64_t B, int64_t H,
                             int64_t H_kv, int64_t N, int64_t d, int causal, float scale, void* stream) {
  return fwd_impl(Q, K, V, O, LSE, nullptr, B, H, H_kv, N, d, causal, scale, stream);
}

ATTN_EXPORT int attn_fwd_blocksparse(const void* Q, const void* K, const void* V, void* O, float* LSE,
                                     const uint8_t* block_mask, int64_t B, int64_t H, int64_t H_kv, int64_t N,
                                     int64_t d, int causal, float scale, void* stream) {
  if (!block_mask) return ATTN_ERR_INVALID_ARG;
  return fwd_impl(Q, K, V, O, LSE, block_mask, B, H, H_kv, N, d, causal, scale, stream);
}

ATTN_EXPORT size_t attn_bwd_deterministic_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t d) {
  if (check_sizes(B, H, N, d) != ATTN_OK) return 0;
  return size_t(2) * sizeof(float) * size_t(B * H) * size_t(npad_of(N));
}

ATTN_EXPORT size_t attn_bwd_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t d) {
  if (check_sizes(B, H, N, d) != ATTN_OK) return 0;
  return size_t(B * H) * size_t(npad_of(N)) * sizeof(float) * size_t(2 + d);
}

}  // extern "C"

namespace {

struct BwdSetup {
  int64_t bh = 0, npad = 0;
  float* ws_lse2 = nullptr;
  float* ws_d = nullptr;
};

int bwd_common_checks(int64_t B, int64_t H, int64_t N, int64_t d, const void* workspace, size_t workspace_bytes,
                      BwdSetup* out) {
  int s = check_sizes(B, H, N, d);
  if (s != ATTN_OK) return s;
  if (!workspace) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return ATTN_ERR_MISALIGNED;
  if (workspace_bytes < attn_bwd_deterministic_workspace_bytes(B, H, N, d)) return ATTN_ERR_WORKSPACE;
  out->bh = B * H;
  out->npad = npad_of(N);
  out->ws_lse2 = static_cast<float*>(const_cast<void*>(workspace));
  out->ws_d = out->ws_lse2 + out->bh * out->npad;
  return ATTN_OK;
}

attn::BwdParams bwd_params(const BwdSetup& su, int64_t N, int64_t H, int64_t H_kv, float scale,
                           const uint8_t* mask) {
  attn::BwdParams prm;
  prm.mask = mask;
  prm.dq_acc = nullptr;
  prm.h = int(H);
  prm.h_kv = int(H_kv);
  prm.group = int(H / H_kv);
  prm.ws_lse2 = su.ws_lse2;
  prm.ws_d = su.ws_d;
  prm.n = int(N);
  prm.npad = int(su.npad);
  prm.n_tiles = int(su.npad / 128);
  prm.scale = scale;
  prm.scale_log2 = scale * 1.4426950408889634f;
  return prm;
}

}  // namespace

extern "C" {

ATTN_EXPORT int attn_bwd_preprocess(const void* O, const void* dO, const float* LSE, int64_t B, int64_t H, int64_t N,
                                    int64_t d, void* workspace, size_t workspace_bytes, void* stream) {
  BwdSetup su;
  int s = bwd_common_checks(B, H, N, d, workspace, workspace_bytes, &su);
  if (s != ATTN_OK) return s;
  if (!O || !dO || !LSE) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(O) || !aligned16(dO) || !aligned16(LSE)) return ATTN_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return (d == 128) ? launch_bwd_pre<128>(O, dO, LSE, su.ws_lse2, su.ws_d, int(N), int(su.npad), su.bh * su.npad, st)
                    : launch_bwd_pre<64>(O, dO, LSE, su.ws_lse2, su.ws_d, int(N), int(su.npad), su.bh * su.npad, st);
}

}  // extern "C"

namespace {

int dkdv_impl(const void* Q, const void* K, const void* V, const void* dO, void* dK, void* dV, const uint8_t* mask,
              int64_t B, int64_t H, int64_t H_kv, int64_t N, int64_t d, int causal, float scale, const void* workspace,
              size_t workspace_bytes, void* stream) {
  BwdSetup su;
  int s = bwd_common_checks(B, H, N, d, workspace, workspace_bytes, &su);
  if (s != ATTN_OK) return s;
  if ((s = check_heads(H, H_kv)) != ATTN_OK) return s;
  if ((s = check_scale(scale)) != ATTN_OK) return s;
  if (!Q || !K || !V || !dO || !dK || !dV) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(dO) || !aligned16(dK) || !aligned16(dV))
    return ATTN_ERR_MISALIGNED;
  const int64_t bhkv = B * H_kv;
  CUtensorMap mq, mk, mv, mdo, mdk, mdv;
  if (!make_map(&mq, Q, su.bh, N, d) || !make_map(&mk, K, bhkv, N, d) || !make_map(&mv, V, bhkv, N, d) ||
      !make_map(&mdo, dO, su.bh, N, d) || !make_map(&mdk, dK, bhkv, N, d) || !make_map(&mdv, dV, bhkv, N, d))
    return ATTN_ERR_LAUNCH;
  const attn::BwdParams prm = bwd_params(su, N, H, H_kv, scale, mask);
  const bool sparse = mask != nullptr;
  const int grid = int(bhkv * prm.n_tiles);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return ATTN_DISPATCH(launch_dkdv, mq, mk, mv, mdo, mdk, mdv, prm, grid, st);
}

int dq_impl(const void* Q, const void* K, const void* V, const void* dO, void* dQ, const uint8_t* mask, int64_t B,
            int64_t H, int64_t H_kv, int64_t N, int64_t d, int causal, float scale, const void* workspace,
            size_t workspace_bytes, void* stream) {
  BwdSetup su;
  int s = bwd_common_checks(B, H, N, d, workspace, workspace_bytes, &su);
  if (s != ATTN_OK) return s;
  if ((s = check_heads(H, H_kv)) != ATTN_OK) return s;
  if ((s = check_scale(scale)) != ATTN_OK) return s;
  if (!Q || !K || !V || !dO || !dQ) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(dO) || !aligned16(dQ)) return ATTN_ERR_MISALIGNED;
  const int64_t bhkv = B * H_kv;
  CUtensorMap mq, mk, mv, mdo, mdq;
  if (!make_map(&mq, Q, su.bh, N, d) || !make_map(&mk, K, bhkv, N, d) || !make_map(&mv, V, bhkv, N, d) ||
      !make_map(&mdo, dO, su.bh, N, d) || !make_map(&mdq, dQ, su.bh, N, d))
    return ATTN_ERR_LAUNCH;
  const attn::BwdParams prm = bwd_params(su, N, H, H_kv, scale, mask);
  const bool sparse = mask != nullptr;
  const int grid = int(su.bh * prm.n_tiles);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return ATTN_DISPATCH(launch_dq, mq, mk, mv, mdo, mdq, prm, grid, st);
}

int bwd_impl(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE, void* dQ,
             void* dK, void* dV, const uint8_t* mask, int64_t B, int64_t H, int64_t H_kv, int64_t N, int64_t d,
             int causal, float scale, void* workspace, size_t workspace_bytes, void* stream) {
  int s = check_sizes(B, H, N, d);
  if (s != ATTN_OK) return s;
  if ((s = check_heads(H, H_kv)) != ATTN_OK) return s;
  if ((s = check_scale(scale)) != ATTN_OK) return s;
  if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV || !workspace) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(dO) || !aligned16(LSE) ||
      !aligned16(dQ) || !aligned16(dK) || !aligned16(dV) || !aligned16(workspace))
    return ATTN_ERR_MISALIGNED;
  if (workspace_bytes < attn_bwd_deterministic_workspace_bytes(B, H, N, d)) return ATTN_ERR_WORKSPACE;
  s = attn_bwd_preprocess(O, dO, LSE, B, H, N, d, workspace, workspace_bytes, stream);
  if (s != ATTN_OK) return s;
  s = dkdv_impl(Q, K, V, dO, dK, dV, mask, B, H, H_kv, N, d, causal, scale, workspace, workspace_bytes, stream);
  if (s != ATTN_OK) return s;
  return dq_impl(Q, K, V, dO, dQ, mask, B, H, H_kv, N, d, causal, scale, workspace, workspace_bytes, stream);
}

// The fused backward: bwd_pre (also clearing the fp32 dQ accumulator), one
// pass over the key tiles for dK, dV and the dQ partials, and the dQ
// conversion.  Workspace: [B*H][Npad] LSE*log2(e), [B*H][Npad] D, then the
// accumulator [B*H][Npad][d] fp32.
int fused_setup(int64_t B, int64_t H, int64_t N, int64_t d, void* workspace, size_t workspace_bytes, BwdSetup* su,
                float** dq_acc) {
  int s = check_sizes(B, H, N, d);
  if (s != ATTN_OK) return s;
  if (!workspace) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return ATTN_ERR_MISALIGNED;
  if (workspace_bytes < attn_bwd_workspace_bytes(B, H, N, d)) return ATTN_ERR_WORKSPACE;
  su->bh = B * H;
  su->npad = npad_of(N);
  su->ws_lse2 = static_cast<float*>(workspace);
  su->ws_d = su->ws_lse2 + su->bh * su->npad;
  *dq_acc = su->ws_d + su->bh * su->npad;
  return ATTN_OK;
}

int fused_pre_impl(const void* O, const void* dO, const float* LSE, int64_t B, int64_t H, int64_t N, int64_t d,
                   void* workspace, size_t workspace_bytes, void* stream) {
  BwdSetup su;
  float* dq_acc = nullptr;
  int s = fused_setup(B, H, N, d, workspace, workspace_bytes, &su, &dq_acc);
  if (s != ATTN_OK) return s;
  if (!O || !dO || !LSE) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(O) || !aligned16(dO) || !aligned16(LSE)) return ATTN_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return (d == 128) ? launch_bwd_pre<128>(O, dO, LSE, su.ws_lse2, su.ws_d, int(N), int(su.npad), su.bh * su.npad, st,
                                          dq_acc)
                    : launch_bwd_pre<64>(O, dO, LSE, su.ws_lse2, su.ws_d, int(N), int(su.npad), su.bh * su.npad, st,
                                         dq_acc);
}

int fused_main_impl(const void* Q, const void* K, const void* V, const void* dO, void* dK, void* dV,
                    const uint8_t* mask, int64_t B, int64_t H, int64_t H_kv, int64_t N, int64_t d, int causal,
                    float scale, void* workspace, size_t workspace_bytes, void* stream) {
  BwdSetup su;
  float* dq_acc = nullptr;
  int s = fused_setup(B, H, N, d, workspace, workspace_bytes, &su, &dq_acc);
  if (s != ATTN_OK) return s;
  if ((s = check_heads(H, H_kv)) != ATTN_OK) return s;
  if ((s = check_scale(scale)) != ATTN_OK) return s;
  if (!Q || !K || !V || !dO || !dK || !dV) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(dO) || !aligned16(dK) || !aligned16(dV))
    return ATTN_ERR_MISALIGNED;
  const int64_t bhkv = B * H_kv;
  CUtensorMap mq, mk, mv, mdo, mdk, mdv, macc;
  if (!make_map(&mq, Q, su.bh, N, d) || !make_map(&mk, K, bhkv, N, d) || !make_map(&mv, V, bhkv, N, d) ||
      !make_map(&mdo, dO, su.bh, N, d) || !make_map(&mdk, dK, bhkv, N, d) || !make_map(&mdv, dV, bhkv, N, d) ||
      !make_map_f32_acc(&macc, dq_acc, su.bh, N, su.npad, d))
    return ATTN_ERR_LAUNCH;
  attn::BwdParams prm = bwd_params(su, N, H, H_kv, scale, mask);
  prm.dq_acc = dq_acc;
  const bool sparse = mask != nullptr;
  const int grid = int(bhkv * prm.n_tiles);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return ATTN_DISPATCH(launch_fused, mq, mk, mv, mdo, mdk, mdv, macc, prm, grid, st);
}

int fused_convert_impl(void* dQ, int64_t B, int64_t H, int64_t N, int64_t d, float scale, void* workspace,
                       size_t workspace_bytes, void* stream) {
  BwdSetup su;
  float* dq_acc = nullptr;
  int s = fused_setup(B, H, N, d, workspace, workspace_bytes, &su, &dq_acc);
  if (s != ATTN_OK) return s;
  if ((s = check_scale(scale)) != ATTN_OK) return s;
  if (!dQ) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(dQ)) return ATTN_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return (d == 128) ? launch_dq_convert<128>(dq_acc, dQ, int(N), int(su.npad), su.bh * N, scale, st)
                    : launch_dq_convert<64>(dq_acc, dQ, int(N), int(su.npad), su.bh * N, scale, st);
}

int fused_impl(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
               void* dQ, void* dK, void* dV, const uint8_t* mask, int64_t B, int64_t H, int64_t H_kv, int64_t N,
               int64_t d, int causal, float scale, void* workspace, size_t workspace_bytes, void* stream) {
  // every argument is checked before the first launch
  int s = check_sizes(B, H, N, d);
  if (s != ATTN_OK) return s;
  if ((s = check_heads(H, H_kv)) != ATTN_OK) return s;
  if ((s = check_scale(scale)) != ATTN_OK) return s;
  if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV || !workspace) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(dO) || !aligned16(LSE) ||
      !aligned16(dQ) || !aligned16(dK) || !aligned16(dV) || !aligned16(workspace))
    return ATTN_ERR_MISALIGNED;
  if (workspace_bytes < attn_bwd_workspace_bytes(B, H, N, d)) return ATTN_ERR_WORKSPACE;
  s = fused_pre_impl(O, dO, LSE, B, H, N, d, workspace, workspace_bytes, stream);
  if (s != ATTN_OK) return s;
  s = fused_main_impl(Q, K, V, dO, dK, dV, mask, B, H, H_kv, N, d, causal, scale, workspace, workspace_bytes, stream);
  if (s != ATTN_OK) return s;
  return fused_convert_impl(dQ, B, H, N, d, scale, workspace, workspace_bytes, stream);
}

}  // namespace

extern "C" {

ATTN_EXPORT int attn_bwd_dkdv(const void* Q, const void* K, const void* V, const void* dO, void* dK, void* dV,
                              int64_t B, int64_t H, int64_t N, int64_t d, int causal, float scale,
                              const void* workspace, size_t workspace_bytes, void* stream) {
  return dkdv_impl(Q, K, V, dO, dK, dV, nullptr, B, H, H, N, d, causal, scale, workspace, workspace_bytes, stream);
}

ATTN_EXPORT int attn_bwd_dq(const void* Q, const void* K, const void* V, const void* dO, void* dQ, int64_t B,
                            int64_t H, int64_t N, int64_t d, int causal, float scale, const void* workspace,
                            size_t workspace_bytes, void* stream) {
  return dq_impl(Q, K, V, dO, dQ, nullptr, B, H, H, N, d, causal, scale, workspace, workspace_bytes, stream);
}

ATTN_EXPORT int attn_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
                         void* dQ, void* dK, void* dV, int64_t B, int64_t H, int64_t N, int64_t d, int causal,
                         float scale, void* workspace, size_t workspace_bytes, void* stream) {
  return fused_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, nullptr, B, H, H, N, d, causal, scale, workspace,
                    workspace_bytes, stream);
}

ATTN_EXPORT int attn_bwd_fused_preprocess(const void* O, const void* dO, const float* LSE, int64_t B, int64_t H,
                                          int64_t N, int64_t d, void* workspace, size_t workspace_bytes,
                                          void* stream) {
  return fused_pre_impl(O, dO, LSE, B, H, N, d, workspace, workspace_bytes, stream);
}

ATTN_EXPORT int attn_bwd_fused_dkdvdq(const void* Q, const void* K, const void* V, const void* dO, void* dK,
                                      void* dV, int64_t B, int64_t H, int64_t N, int64_t d, int causal, float scale,
                                      void* workspace, size_t workspace_bytes, void* stream) {
  return fused_main_impl(Q, K, V, dO, dK, dV, nullptr, B, H, H, N, d, causal, scale, workspace, workspace_bytes,
                         stream);
}

ATTN_EXPORT int attn_bwd_fused_dq_convert(void* dQ, int64_t B, int64_t H, int64_t N, int64_t d, float scale,
                                          void* workspace, size_t workspace_bytes, void* stream) {
  return fused_convert_impl(dQ, B, H, N, d, scale, workspace, workspace_bytes, stream);
}

ATTN_EXPORT int attn_bwd_deterministic(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                                       const float* LSE, void* dQ, void* dK, void* dV, int64_t B, int64_t H,
                                       int64_t H_kv, int64_t N, int64_t d, int causal, float scale, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  return bwd_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, nullptr, B, H, H_kv, N, d, causal, scale, workspace,
                  workspace_bytes, stream);
}

ATTN_EXPORT int attn_bwd_gqa(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                             const float* LSE, void* dQ, void* dK, void* dV, int64_t B, int64_t H, int64_t H_kv,
                             int64_t N, int64_t d, int causal, float scale, void* workspace, size_t workspace_bytes,
                             void* stream) {
  return fused_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, nullptr, B, H, H_kv, N, d, causal, scale, workspace,
                    workspace_bytes, stream);
}

ATTN_EXPORT int attn_bwd_blocksparse(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                                     const float* LSE, const uint8_t* block_mask, void* dQ, void* dK, void* dV,
                                     int64_t B, int64_t H, int64_t H_kv, int64_t N, int64_t d, int causal,
                                     float scale, void* workspace, size_t workspace_bytes, void* stream) {
  if (!block_mask) return ATTN_ERR_INVALID_ARG;
  return fused_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, block_mask, B, H, H_kv, N, d, causal, scale, workspace,
                    workspace_bytes, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Forward on FP8 (E4M3) inputs with per-tensor dequantisation factors.
// ---------------------------------------------------------------------------
namespace {

template <bool CAUSAL>
int launch_fp8(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const attn::Fp8Params& prm,
               int grid, cudaStream_t st) {
  using C = attn::Fp8Cfg;
  auto kern = attn::attn_fwd_fp8_kernel<CAUSAL>;
  constexpr int smem = C::kSmemBytes;
  if (check_launch_regs<attn::attn_fwd_fp8_kernel<CAUSAL>>(int(C::kRegsLaunch), "FP8 forward") != ATTN_OK)
    return ATTN_ERR_LAUNCH;
  if (set_smem(reinterpret_cast<const void*>(kern), smem) != ATTN_OK) return ATTN_ERR_LAUNCH;
  kern<<<grid, attn::Fp8Cfg::kThreads, smem, st>>>(q, k, v, prm);
  return launch_status();
}

bool positive_finite(float x) { return std::isfinite(x) && x > 0.f; }

}  // namespace

extern "C" {

ATTN_EXPORT int attn_fwd_fp8(const void* Q8, const void* K8, const void* V8, void* O, float* LSE, int64_t B,
                             int64_t H, int64_t H_kv, int64_t N, int64_t d, int causal, float scale,
                             float q_descale, float k_descale, float v_descale, void* stream) {
  int s = check_sizes(B, H, N, d);
  if (s != ATTN_OK) return s;
  if (d != 128) return fail(ATTN_ERR_UNSUPPORTED, "attn_fwd_fp8 supports d = 128 only (got %lld)", (long long)d);
  if ((s = check_heads(H, H_kv)) != ATTN_OK) return s;
  if ((s = check_scale(scale)) != ATTN_OK) return s;
  if (!positive_finite(q_descale) || !positive_finite(k_descale) || !positive_finite(v_descale))
    return ATTN_ERR_INVALID_ARG;
  if (!Q8 || !K8 || !V8 || !O || !LSE) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(Q8) || !aligned16(K8) || !aligned16(V8) || !aligned16(O) || !aligned16(LSE))
    return ATTN_ERR_MISALIGNED;
  const int64_t bh = B * H, bhkv = B * H_kv;
  CUtensorMap mq, mk, mv;
  if (!make_map_u8(&mq, Q8, bh, N, d) || !make_map_u8(&mk, K8, bhkv, N, d) || !make_map_u8(&mv, V8, bhkv, N, d))
    return ATTN_ERR_LAUNCH;
  attn::Fp8Params prm;
  prm.o = static_cast<__nv_bfloat16*>(O);
  prm.lse = LSE;
  prm.n = int(N);
  prm.n_mblk = int((N + 255) / 256);
  prm.h = int(H);
  prm.h_kv = int(H_kv);
  prm.group = int(H / H_kv);
  prm.c = float(double(scale) * double(q_descale) * double(k_descale) * 1.4426950408889634);
  prm.v_descale = v_descale;
  if (!std::isfinite(prm.c) || !(prm.c > 0.f)) return ATTN_ERR_INVALID_ARG;
  const int64_t grid = bh * prm.n_mblk;
  if (grid > INT32_MAX) return ATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return causal ? launch_fp8<true>(mq, mk, mv, prm, int(grid), st) : launch_fp8<false>(mq, mk, mv, prm, int(grid), st);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Forward against a key/value cache (decode / chunked prefill), split-KV.
// ---------------------------------------------------------------------------
namespace {

constexpr int64_t kMaxSplits = 256;
static_assert(kMaxSplits * 4 <= attn::kKvcMaxParts, "the merge kernel holds every partial's LSE in shared memory");

struct KvcShape {
  int64_t rows = 0;        // packed query rows per key/value head
  int64_t n_rt = 0;        // 128-row tiles of packed rows
  int64_t tiles = 0;       // 128-row key tiles of the cache
  int64_t total_rows = 0;  // B*H*Nq
};

int kvc_check(int64_t B, int64_t H, int64_t H_kv, int64_t Nq, int64_t Nk, int64_t d, KvcShape* sh) {
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  int s = check_heads(H, H_kv);
  if (s != ATTN_OK) return s;
  if (B > INT32_MAX / H || Nq > (INT32_MAX - 128) / (B * H) || Nk > INT32_MAX - 256) return ATTN_ERR_INVALID_ARG;
  sh->rows = (H / H_kv) * Nq;
  sh->n_rt = (sh->rows + 127) / 128;
  sh->tiles = (Nk + 127) / 128;
  sh->total_rows = B * H * Nq;
  return ATTN_OK;
}

// Splits: explicit counts are capped at the number of key tiles; the automatic
// count minimises (work items per SM, rounded up) x (key tiles per item +
// 1/4), the 1/4 standing for an item's fixed cost in the persistent kernel
// (its partial write and the merge traffic).
int64_t kvc_splits(const KvcShape& sh, int64_t B, int64_t H_kv, int64_t num_splits) {
  if (num_splits < 0) return 0;
  const int64_t cap = std::min(sh.tiles, kMaxSplits);
  if (num_splits > 0) return std::min(num_splits, cap);
  const int64_t base = B * H_kv * sh.n_rt;
  int64_t best_s = 1, best_cost = INT64_MAX;
  for (int64_t sp = 1; sp <= cap; ++sp) {
    const int64_t per = (sh.tiles + sp - 1) / sp;
    const int64_t waves = (base * sp + kNumSMs - 1) / kNumSMs;
    const int64_t cost = waves * (4 * per + 1);
    if (cost < best_cost) {
      best_cost = cost;
      best_s = sp;
    }
  }
  return best_s;
}

// With at most 32 packed query rows per key/value head the kernel replicates
// them into all four TMEM lane quarters and splits every key tile four ways,
// so each key chunk yields four partials.
bool kvc_replicated(const KvcShape& sh) { return sh.rows <= 32; }

int64_t kvc_partials(const KvcShape& sh, int64_t splits) { return splits * (kvc_replicated(sh) ? 4 : 1); }

size_t kvc_workspace(const KvcShape& sh, int64_t splits, int64_t d) {
  const int64_t parts = kvc_partials(sh, splits);
  if (parts <= 1) return 0;
  return size_t(parts) * size_t(sh.total_rows) * size_t(d + 1) * sizeof(float);
}

// The split-KV merge, launched as a programmatic dependent of the cache
// kernel just before it on the stream: its grid is set up while the cache
// kernel's last CTAs run, and each block waits (griddepcontrol.wait) until the
// cache kernel has completed and its partials are visible.
template <int D>
int launch_merge(const attn::KvcParams& prm, int parts, cudaStream_t st) {
  int64_t blocks = prm.total_rows;                            // one 256-thread block per row
  if (blocks > kNumSMs * 8) blocks = kNumSMs * 8;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(blocks));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const float* part_o = prm.part_o;
  const float* part_lse = prm.part_lse;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, attn::attn_kvcache_merge_kernel<D>, part_o, part_lse, prm.o,
                                           prm.lse, (long long)prm.total_rows, parts);
  if (e != cudaSuccess)
    return fail(ATTN_ERR_LAUNCH, "split-KV merge launch: %s (%lld)", cudaGetErrorString(e), (long long)e);
  return launch_status();
}

template <int D, bool CAUSAL, bool SPLIT, bool REPL>
int launch_kvc(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const attn::KvcParams& prm,
               int grid, cudaStream_t st) {
  auto kern = attn::attn_kvcache_kernel<D, CAUSAL, SPLIT, REPL>;
  constexpr int smem = attn::KvcCfg<D>::kSmemBytes;
  if (set_smem(reinterpret_cast<const void*>(kern), smem) != ATTN_OK) return ATTN_ERR_LAUNCH;
  kern<<<grid, attn::KvcCfg<D>::kThreads, smem, st>>>(q, k, v, prm);
  int s = launch_status();
  if (s != ATTN_OK || !SPLIT) return s;
  return launch_merge<D>(prm, prm.splits * (REPL ? 4 : 1), st);
}

template <int D, bool CAUSAL>
int dispatch_kvc(bool split, bool repl, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                 const attn::KvcParams& prm, int grid, cudaStream_t st) {
  if (repl) return launch_kvc<D, CAUSAL, true, true>(q, k, v, prm, grid, st);
  return split ? launch_kvc<D, CAUSAL, true, false>(q, k, v, prm, grid, st)
               : launch_kvc<D, CAUSAL, false, false>(q, k, v, prm, grid, st);
}

}  // namespace

extern "C" {

ATTN_EXPORT int64_t attn_fwd_kvcache_splits(int64_t B, int64_t H, int64_t H_kv, int64_t Nq, int64_t Nk, int64_t d,
                                            int64_t num_splits) {
  KvcShape sh;
  if (kvc_check(B, H, H_kv, Nq, Nk, d, &sh) != ATTN_OK) return 0;
  return kvc_splits(sh, B, H_kv, num_splits);
}

ATTN_EXPORT size_t attn_fwd_kvcache_workspace_bytes(int64_t B, int64_t H, int64_t H_kv, int64_t Nq, int64_t Nk,
                                                    int64_t d, int64_t num_splits) {
  KvcShape sh;
  if (kvc_check(B, H, H_kv, Nq, Nk, d, &sh) != ATTN_OK) return 0;
  return kvc_workspace(sh, kvc_splits(sh, B, H_kv, num_splits), d);
}

ATTN_EXPORT int attn_fwd_kvcache(const void* Q, const void* K, const void* V, void* O, float* LSE,
                                 const int32_t* kv_lens, int64_t B, int64_t H, int64_t H_kv, int64_t Nq, int64_t Nk,
                                 int64_t d, int causal, float scale, int64_t num_splits, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  KvcShape sh;
  int s = kvc_check(B, H, H_kv, Nq, Nk, d, &sh);
  if (s != ATTN_OK) return s;
  if ((s = check_scale(scale)) != ATTN_OK) return s;
  const int64_t splits = kvc_splits(sh, B, H_kv, num_splits);
  if (splits < 1) return ATTN_ERR_INVALID_ARG;
  if (!Q || !K || !V || !O || !LSE) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE))
    return ATTN_ERR_MISALIGNED;
  if (kv_lens && (reinterpret_cast<uintptr_t>(kv_lens) & 3u) != 0) return ATTN_ERR_MISALIGNED;
  const bool repl = kvc_replicated(sh);
  const int64_t parts = kvc_partials(sh, splits);
  const bool split = parts > 1;
  if (split) {
    if (!workspace) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return ATTN_ERR_MISALIGNED;
    if (workspace_bytes < kvc_workspace(sh, splits, d)) return ATTN_ERR_WORKSPACE;
  }
  const int64_t n_items = B * H_kv * sh.n_rt * splits;
  if (n_items > INT32_MAX) return ATTN_ERR_INVALID_ARG;
  const int64_t grid = std::min<int64_t>(n_items, kNumSMs);     // persistent: one CTA per SM
  const int qbox = int(std::min<int64_t>(128, (sh.rows + 7) / 8 * 8));
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, Q, 1, sh.total_rows, d, qbox) || !make_map(&mk, K, B * H_kv, Nk, d) ||
      !make_map(&mv, V, B * H_kv, Nk, d))
    return ATTN_ERR_LAUNCH;
  attn::KvcParams prm;
  prm.o = static_cast<__nv_bfloat16*>(O);
  prm.lse = LSE;
  prm.part_o = split ? static_cast<float*>(workspace) : nullptr;
  prm.part_lse = split ? static_cast<float*>(workspace) + size_t(parts) * size_t(sh.total_rows) * size_t(d) : nullptr;
  prm.kv_lens = kv_lens;
  prm.total_rows = sh.total_rows;
  prm.nq = int(Nq);
  prm.nk = int(Nk);
  prm.h_kv = int(H_kv);
  prm.rows = int(sh.rows);
  prm.n_rt = int(sh.n_rt);
  prm.splits = int(splits);
  prm.qbox = qbox;
  prm.n_items = int(n_items);
  prm.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 128)
    return causal ? dispatch_kvc<128, true>(split, repl, mq, mk, mv, prm, int(grid), st)
                  : dispatch_kvc<128, false>(split, repl, mq, mk, mv, prm, int(grid), st);
  return causal ? dispatch_kvc<64, true>(split, repl, mq, mk, mv, prm, int(grid), st)
                : dispatch_kvc<64, false>(split, repl, mq, mk, mv, prm, int(grid), st);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode against an FP8 (E4M3) key/value cache.
// ---------------------------------------------------------------------------
namespace {

template <bool CAUSAL>
int launch_kvc8(const CUtensorMap& q, const CUtensorMap& k8, const CUtensorMap& v8, const attn::KvcParams& prm,
                float v_descale, int grid, cudaStream_t st) {
  auto kern = attn::attn_kvcache_fp8_kernel<CAUSAL>;
  constexpr int smem = attn::Kvc8Cfg::kSmemBytes;
  if (set_smem(reinterpret_cast<const void*>(kern), smem) != ATTN_OK) return ATTN_ERR_LAUNCH;
  kern<<<grid, attn::Kvc8Cfg::kThreads, smem, st>>>(q, k8, v8, prm, v_descale);
  int s = launch_status();
  if (s != ATTN_OK) return s;
  return launch_merge<128>(prm, prm.splits * 4, st);
}

}  // namespace

extern "C" {

ATTN_EXPORT int attn_fwd_kvcache_fp8(const void* Q, const void* K8, const void* V8, void* O, float* LSE,
                                     const int32_t* kv_lens, int64_t B, int64_t H, int64_t H_kv, int64_t Nq,
                                     int64_t Nk, int64_t d, int causal, float scale, float k_descale,
                                     float v_descale, int64_t num_splits, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  KvcShape sh;
  int s = kvc_check(B, H, H_kv, Nq, Nk, d, &sh);
  if (s != ATTN_OK) return s;
  if (d != 128)
    return fail(ATTN_ERR_UNSUPPORTED, "attn_fwd_kvcache_fp8 supports d = 128 only (got %lld)", (long long)d);
  if (!kvc_replicated(sh))
    return fail(ATTN_ERR_UNSUPPORTED,
                "attn_fwd_kvcache_fp8 takes at most 32 query rows per key/value head ((H / H_kv) * Nq = %lld)",
                (long long)sh.rows);
  if ((s = check_scale(scale)) != ATTN_OK) return s;
  if (!(std::isfinite(k_descale) && k_descale > 0.f) || !(std::isfinite(v_descale) && v_descale > 0.f))
    return ATTN_ERR_INVALID_ARG;
  const int64_t splits = kvc_splits(sh, B, H_kv, num_splits);
  if (splits < 1) return ATTN_ERR_INVALID_ARG;
  if (!Q || !K8 || !V8 || !O || !LSE || !workspace) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K8) || !aligned16(V8) || !aligned16(O) || !aligned16(LSE) || !aligned16(workspace))
    return ATTN_ERR_MISALIGNED;
  if (kv_lens && (reinterpret_cast<uintptr_t>(kv_lens) & 3u) != 0) return ATTN_ERR_MISALIGNED;
  if (workspace_bytes < kvc_workspace(sh, splits, d)) return ATTN_ERR_WORKSPACE;
  const int64_t n_items = B * H_kv * sh.n_rt * splits;
  if (n_items > INT32_MAX) return ATTN_ERR_INVALID_ARG;
  const int64_t grid = std::min<int64_t>(n_items, kNumSMs);
  const int qbox = int((sh.rows + 7) / 8 * 8);
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, Q, 1, sh.total_rows, d, qbox) || !make_map_u8(&mk, K8, B * H_kv, Nk, d) ||
      !make_map_u8(&mv, V8, B * H_kv, Nk, d))
    return ATTN_ERR_LAUNCH;
  const int64_t parts = kvc_partials(sh, splits);
  attn::KvcParams prm;
  prm.o = static_cast<__nv_bfloat16*>(O);
  prm.lse = LSE;
  prm.part_o = static_cast<float*>(workspace);
  prm.part_lse = static_cast<float*>(workspace) + size_t(parts) * size_t(sh.total_rows) * size_t(d);
  prm.kv_lens = kv_lens;
  prm.total_rows = sh.total_rows;
  prm.nq = int(Nq);
  prm.nk = int(Nk);
  prm.h_kv = int(H_kv);
  prm.rows = int(sh.rows);
  prm.n_rt = int(sh.n_rt);
  prm.splits = int(splits);
  prm.qbox = qbox;
  prm.n_items = int(n_items);
  // The scores come from the E4M3 key codes themselves (the kernel divides
  // out its per-row query scaling); the widened value tiles hold 2^-8 times
  // the E4M3 values, so that factor goes into the final 1/l.
  prm.scale_log2 = float(double(scale) * double(k_descale) * 1.4426950408889634);
  const float v_scale = float(double(v_descale) * 256.0);
  if (!std::isfinite(prm.scale_log2) || !(prm.scale_log2 > 0.f) || !std::isfinite(v_scale))
    return ATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return causal ? launch_kvc8<true>(mq, mk, mv, prm, v_scale, int(grid), st)
                : launch_kvc8<false>(mq, mk, mv, prm, v_scale, int(grid), st);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Backward with a library-owned, fixed-size workspace.
//
// Some callers cannot allocate device memory at the point where they run the
// backward: code whose memory is owned by another allocator that exposes no
// way to hand out a raw scratch buffer across a C boundary (plugin hosts,
// inference/training runtimes with a "no allocation after start-up" rule),
// and code that runs where cudaMalloc is not allowed or would synchronise the
// device.  For them the workspace lives in this file-scope device array.  It
// exists on every GPU that loads the library, from module load until process
// exit.  It runs the deterministic path (pre, dK/dV, dQ), whose workspace is
// only the two per-row vectors.  The array's device address belongs to the
// module instance of the current context, so it is looked up on every call
// (cudaGetSymbolAddress with the calling thread's current device and context;
// the lookup allocates nothing) rather than cached by device number, which
// would go stale after cudaDeviceReset or under another context.
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) unsigned char g_static_workspace[ATTN_STATIC_WORKSPACE_BYTES];

void* static_workspace_for_current_context() {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_static_workspace);
  if (e != cudaSuccess || p == nullptr) {
    fail(ATTN_ERR_DEVICE, "cudaGetSymbolAddress(static workspace): %s (%lld)", cudaGetErrorString(e), (long long)e);
    return nullptr;
  }
  return p;
}

}  // namespace

extern "C" {

ATTN_EXPORT int attn_bwd_static_workspace(const void* Q, const void* K, const void* V, const void* O,
                                          const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                                          int64_t B, int64_t H, int64_t N, int64_t d, int causal, float scale,
                                          void* stream) {
  const int s = check_sizes(B, H, N, d);
  if (s != ATTN_OK) return s;
  const size_t need = attn_bwd_deterministic_workspace_bytes(B, H, N, d);
  if (need > size_t(ATTN_STATIC_WORKSPACE_BYTES))
    return fail(ATTN_ERR_WORKSPACE,
                "attn_bwd_static_workspace: these sizes need %lld workspace bytes, more than the "
                "ATTN_STATIC_WORKSPACE_BYTES the library holds; use attn_bwd with a caller workspace",
                (long long)need);
  void* ws = static_workspace_for_current_context();
  if (ws == nullptr) return ATTN_ERR_DEVICE;
  return bwd_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, nullptr, B, H, H, N, d, causal, scale, ws,
                  size_t(ATTN_STATIC_WORKSPACE_BYTES), stream);
}

}  // extern "C"

namespace {

// Failure-path self-test: one CTA allocates tensor memory, waits on an
// mbarrier that nothing ever arrives on with a short limit, takes the same
// timeout path as the attention kernels (abort flag + status word), then
// releases its tensor memory and returns.  No fault, trap or endless loop.
__global__ void attn_selftest_timeout_kernel(unsigned long long timeout_ns, int* waited_ok) {
  __shared__ uint64_t bar;
  __shared__ uint32_t tslot;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    attn::mbar_init(&bar, 1);
    abort_flag = 0;
    attn::fence_barrier_init();
  }
  attn::tmem_alloc(&tslot, 32);
  attn::tmem_relinquish();
  attn::tc_fence_before();
  __syncthreads();
  attn::tc_fence_after();
  const uint32_t tmem = tslot;
  bool ok = attn::mbar_wait(&bar, 0, &abort_flag, true, timeout_ns);   // runs out after timeout_ns
  ok = __all_sync(0xffffffffu, ok);
  if (threadIdx.x == 0 && waited_ok) *waited_ok = ok ? 1 : 0;
  attn::tc_fence_before();
  __syncthreads();
  attn::tc_fence_after();
  attn::tmem_dealloc(tmem, 32);
}

}  // namespace

extern "C" {

ATTN_EXPORT int attn_selftest_wait_timeout(void* stream) {
  attn_selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(20ull * 1000 * 1000, nullptr);
  return launch_status();
}

ATTN_EXPORT int attn_check_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_DEVICE;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, attn::g_attn_status, sizeof(v)) != cudaSuccess) return ATTN_ERR_DEVICE;
  if (v != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(attn::g_attn_status, &zero, sizeof(zero)) != cudaSuccess) return ATTN_ERR_DEVICE;
    if (v & attn::kStatusLayout)
      return fail(ATTN_ERR_DEVICE, "a kernel found its shared memory window misaligned and did no work");
    return ATTN_ERR_TIMEOUT;
  }
  return ATTN_OK;
}

ATTN_EXPORT const char* attn_last_error(void) { return g_last_error; }

ATTN_EXPORT const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
    case ATTN_ERR_MISALIGNED: return "ATTN_ERR_MISALIGNED";
    case ATTN_ERR_WORKSPACE: return "ATTN_ERR_WORKSPACE";
    case ATTN_ERR_LAUNCH: return "ATTN_ERR_LAUNCH";
    case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT";
    case ATTN_ERR_DEVICE: return "ATTN_ERR_DEVICE";
    default: return "ATTN_ERR_UNKNOWN";
  }
}

}  // extern "C"
