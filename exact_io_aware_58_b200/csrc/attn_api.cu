// attn_api.cu -- host side of the C ABI declared in include/attn.h:
// argument checks, TMA tensor maps, kernel selection and launches.
//
// The library allocates no device memory: tensor maps travel as
// __grid_constant__ kernel parameters, the backward's per-row vectors live in
// the caller's workspace, and the only device state is the status word
// g_attn_status (a static __device__ variable).

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/attn.h"
#include "attn_bwd.cuh"
#include "attn_fwd.cuh"

namespace {

// Detail of the most recent failure on this host thread (attn_last_error).
thread_local char g_last_error[256] = "";

int fail(int status, const char* fmt, const char* a = "", long long b = 0) {
  std::snprintf(g_last_error, sizeof(g_last_error), fmt, a, b);
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
// 128 rows x 1 head, 128-byte swizzle.  Rows past N read as zeros; stores
// past N are dropped.
bool make_map(CUtensorMap* m, const void* base, int64_t bh, int64_t n, int64_t d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    fail(ATTN_ERR_LAUNCH, "%sdriver entry point cuTensorMapEncodeTiled unavailable%lld", "", 0);
    return false;
  }
  const cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(n), cuuint64_t(bh)};
  const cuuint64_t strides[2] = {cuuint64_t(d * 2), cuuint64_t(n * d * 2)};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    fail(ATTN_ERR_LAUNCH, "%scuTensorMapEncodeTiled returned CUresult %lld", "", (long long)r);
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

template <int D, bool CAUSAL>
int launch_fwd(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const CUtensorMap& o,
               const attn::FwdParams& prm, int grid, cudaStream_t st) {
  auto kern = attn::attn_fwd_kernel<D, CAUSAL>;
  constexpr int smem = attn::FwdCfg<D>::kSmemBytes;
  if (set_smem(reinterpret_cast<const void*>(kern), smem) != ATTN_OK) return ATTN_ERR_LAUNCH;
  kern<<<grid, attn::FwdCfg<D>::kThreads, smem, st>>>(q, k, v, o, prm);
  return launch_status();
}

template <int D, bool CAUSAL>
int launch_dkdv(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const CUtensorMap& dO,
                const CUtensorMap& dk, const CUtensorMap& dv, const attn::BwdParams& prm, int grid, cudaStream_t st) {
  using C = attn::BwdCfg<D>;
  auto kern = attn::attn_bwd_dkdv_kernel<D, CAUSAL>;
  if (set_smem(reinterpret_cast<const void*>(kern), C::kKV_SmemBytes) != ATTN_OK) return ATTN_ERR_LAUNCH;
  kern<<<grid, C::kThreads, C::kKV_SmemBytes, st>>>(q, k, v, dO, dk, dv, prm);
  return launch_status();
}

template <int D, bool CAUSAL>
int launch_dq(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const CUtensorMap& dO,
              const CUtensorMap& dq, const attn::BwdParams& prm, int grid, cudaStream_t st) {
  using C = attn::BwdCfg<D>;
  auto kern = attn::attn_bwd_dq_kernel<D, CAUSAL>;
  if (set_smem(reinterpret_cast<const void*>(kern), C::kQ_SmemBytes) != ATTN_OK) return ATTN_ERR_LAUNCH;
  kern<<<grid, C::kThreads, C::kQ_SmemBytes, st>>>(q, k, v, dO, dq, prm);
  return launch_status();
}

template <int D>
int launch_bwd_pre(const void* O, const void* dO, const float* lse, float* ws_lse2, float* ws_d, int n, int npad,
                   int64_t rows_pad, cudaStream_t st) {
  constexpr int rows_per_block = 256 / (D / 8);
  int64_t blocks = (rows_pad + rows_per_block - 1) / rows_per_block;
  if (blocks > 148 * 32) blocks = 148 * 32;
  attn::attn_bwd_pre_kernel<D><<<int(blocks), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(O), static_cast<const __nv_bfloat16*>(dO), lse, ws_lse2, ws_d, n, npad,
      static_cast<long long>(rows_pad));
  return launch_status();
}

int64_t npad_of(int64_t N) { return (N + 127) / 128 * 128; }

}  // namespace

#define ATTN_EXPORT __attribute__((visibility("default")))

extern "C" {

}  // extern "C"

namespace {

int fwd_impl(const void* Q, const void* K, const void* V, void* O, float* LSE, int64_t B, int64_t H, int64_t H_kv,
             int64_t N, int64_t d, int causal, float scale, void* stream) {
  int s = check_sizes(B, H, N, d);
  if (s != ATTN_OK) return s;
  if ((s = check_heads(H, H_kv)) != ATTN_OK) return s;
  if ((s = check_scale(scale)) != ATTN_OK) return s;
  if (!Q || !K || !V || !O || !LSE) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE))
    return ATTN_ERR_MISALIGNED;
  const int64_t bh = B * H, bhkv = B * H_kv;
  CUtensorMap mq, mk, mv, mo;
  if (!make_map(&mq, Q, bh, N, d) || !make_map(&mk, K, bhkv, N, d) || !make_map(&mv, V, bhkv, N, d) ||
      !make_map(&mo, O, bh, N, d))
    return ATTN_ERR_LAUNCH;
  attn::FwdParams prm;
  prm.lse = LSE;
  prm.n = int(N);
  prm.n_mblk = int((N + 255) / 256);
  prm.h = int(H);
  prm.h_kv = int(H_kv);
  prm.group = int(H / H_kv);
  prm.scale_log2 = scale * 1.4426950408889634f;
  const int64_t grid = bh * prm.n_mblk;
  if (grid > INT32_MAX) return ATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 128)
    return causal ? launch_fwd<128, true>(mq, mk, mv, mo, prm, int(grid), st)
                  : launch_fwd<128, false>(mq, mk, mv, mo, prm, int(grid), st);
  return causal ? launch_fwd<64, true>(mq, mk, mv, mo, prm, int(grid), st)
                : launch_fwd<64, false>(mq, mk, mv, mo, prm, int(grid), st);
}

}  // namespace

extern "C" {

ATTN_EXPORT int attn_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int64_t B, int64_t H,
                         int64_t N, int64_t d, int causal, float scale, void* stream) {
  return fwd_impl(Q, K, V, O, LSE, B, H, H, N, d, causal, scale, stream);
}

ATTN_EXPORT int attn_fwd_gqa(const void* Q, const void* K, const void* V, void* O, float* LSE, int64_t B, int64_t H,
                             int64_t H_kv, int64_t N, int64_t d, int causal, float scale, void* stream) {
  return fwd_impl(Q, K, V, O, LSE, B, H, H_kv, N, d, causal, scale, stream);
}

ATTN_EXPORT size_t attn_bwd_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t d) {
  if (check_sizes(B, H, N, d) != ATTN_OK) return 0;
  return size_t(2) * sizeof(float) * size_t(B * H) * size_t(npad_of(N));
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
  if (workspace_bytes < attn_bwd_workspace_bytes(B, H, N, d)) return ATTN_ERR_WORKSPACE;
  out->bh = B * H;
  out->npad = npad_of(N);
  out->ws_lse2 = static_cast<float*>(const_cast<void*>(workspace));
  out->ws_d = out->ws_lse2 + out->bh * out->npad;
  return ATTN_OK;
}

attn::BwdParams bwd_params(const BwdSetup& su, int64_t N, int64_t H, int64_t H_kv, float scale) {
  attn::BwdParams prm;
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

int dkdv_impl(const void* Q, const void* K, const void* V, const void* dO, void* dK, void* dV, int64_t B, int64_t H,
              int64_t H_kv, int64_t N, int64_t d, int causal, float scale, const void* workspace,
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
  const attn::BwdParams prm = bwd_params(su, N, H, H_kv, scale);
  const int grid = int(bhkv * prm.n_tiles);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 128)
    return causal ? launch_dkdv<128, true>(mq, mk, mv, mdo, mdk, mdv, prm, grid, st)
                  : launch_dkdv<128, false>(mq, mk, mv, mdo, mdk, mdv, prm, grid, st);
  return causal ? launch_dkdv<64, true>(mq, mk, mv, mdo, mdk, mdv, prm, grid, st)
                : launch_dkdv<64, false>(mq, mk, mv, mdo, mdk, mdv, prm, grid, st);
}

int dq_impl(const void* Q, const void* K, const void* V, const void* dO, void* dQ, int64_t B, int64_t H, int64_t H_kv,
            int64_t N, int64_t d, int causal, float scale, const void* workspace, size_t workspace_bytes,
            void* stream) {
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
  const attn::BwdParams prm = bwd_params(su, N, H, H_kv, scale);
  const int grid = int(su.bh * prm.n_tiles);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 128)
    return causal ? launch_dq<128, true>(mq, mk, mv, mdo, mdq, prm, grid, st)
                  : launch_dq<128, false>(mq, mk, mv, mdo, mdq, prm, grid, st);
  return causal ? launch_dq<64, true>(mq, mk, mv, mdo, mdq, prm, grid, st)
                : launch_dq<64, false>(mq, mk, mv, mdo, mdq, prm, grid, st);
}

int bwd_impl(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE, void* dQ,
             void* dK, void* dV, int64_t B, int64_t H, int64_t H_kv, int64_t N, int64_t d, int causal, float scale,
             void* workspace, size_t workspace_bytes, void* stream) {
  int s = check_sizes(B, H, N, d);
  if (s != ATTN_OK) return s;
  if ((s = check_heads(H, H_kv)) != ATTN_OK) return s;
  if ((s = check_scale(scale)) != ATTN_OK) return s;
  if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV || !workspace) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(dO) || !aligned16(LSE) ||
      !aligned16(dQ) || !aligned16(dK) || !aligned16(dV) || !aligned16(workspace))
    return ATTN_ERR_MISALIGNED;
  if (workspace_bytes < attn_bwd_workspace_bytes(B, H, N, d)) return ATTN_ERR_WORKSPACE;
  s = attn_bwd_preprocess(O, dO, LSE, B, H, N, d, workspace, workspace_bytes, stream);
  if (s != ATTN_OK) return s;
  s = dkdv_impl(Q, K, V, dO, dK, dV, B, H, H_kv, N, d, causal, scale, workspace, workspace_bytes, stream);
  if (s != ATTN_OK) return s;
  return dq_impl(Q, K, V, dO, dQ, B, H, H_kv, N, d, causal, scale, workspace, workspace_bytes, stream);
}

}  // namespace

extern "C" {

ATTN_EXPORT int attn_bwd_dkdv(const void* Q, const void* K, const void* V, const void* dO, void* dK, void* dV,
                              int64_t B, int64_t H, int64_t N, int64_t d, int causal, float scale,
                              const void* workspace, size_t workspace_bytes, void* stream) {
  return dkdv_impl(Q, K, V, dO, dK, dV, B, H, H, N, d, causal, scale, workspace, workspace_bytes, stream);
}

ATTN_EXPORT int attn_bwd_dq(const void* Q, const void* K, const void* V, const void* dO, void* dQ, int64_t B,
                            int64_t H, int64_t N, int64_t d, int causal, float scale, const void* workspace,
                            size_t workspace_bytes, void* stream) {
  return dq_impl(Q, K, V, dO, dQ, B, H, H, N, d, causal, scale, workspace, workspace_bytes, stream);
}

ATTN_EXPORT int attn_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
                         void* dQ, void* dK, void* dV, int64_t B, int64_t H, int64_t N, int64_t d, int causal,
                         float scale, void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, H, N, d, causal, scale, workspace, workspace_bytes, stream);
}

ATTN_EXPORT int attn_bwd_gqa(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                             const float* LSE, void* dQ, void* dK, void* dV, int64_t B, int64_t H, int64_t H_kv,
                             int64_t N, int64_t d, int causal, float scale, void* workspace, size_t workspace_bytes,
                             void* stream) {
  return bwd_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, H_kv, N, d, causal, scale, workspace, workspace_bytes,
                  stream);
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
// exit.  Its address is looked up once per device (cudaGetSymbolAddress with
// that device current) and cached.
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) unsigned char g_static_workspace[ATTN_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;

void* static_workspace_for_current_device() {
  static std::mutex mu;
  static void* ptr[kMaxDevices] = {};
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    fail(ATTN_ERR_DEVICE, "cudaGetDevice: %s (%lld)", cudaGetErrorString(e), (long long)dev);
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess || p == nullptr) {
      fail(ATTN_ERR_DEVICE, "cudaGetSymbolAddress(static workspace): %s (%lld)", cudaGetErrorString(e),
           (long long)e);
      return nullptr;
    }
    ptr[dev] = p;
  }
  return ptr[dev];
}

}  // namespace

extern "C" {

ATTN_EXPORT int attn_bwd_static_workspace(const void* Q, const void* K, const void* V, const void* O,
                                          const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                                          int64_t B, int64_t H, int64_t N, int64_t d, int causal, float scale,
                                          void* stream) {
  const int s = check_sizes(B, H, N, d);
  if (s != ATTN_OK) return s;
  const size_t need = attn_bwd_workspace_bytes(B, H, N, d);
  if (need > size_t(ATTN_STATIC_WORKSPACE_BYTES))
    return fail(ATTN_ERR_WORKSPACE,
                "%sattn_bwd_static_workspace: these sizes need %lld workspace bytes, more than the "
                "ATTN_STATIC_WORKSPACE_BYTES the library holds; use attn_bwd with a caller workspace",
                "", (long long)need);
  void* ws = static_workspace_for_current_device();
  if (ws == nullptr) return ATTN_ERR_DEVICE;
  return attn_bwd(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, N, d, causal, scale, ws,
                  size_t(ATTN_STATIC_WORKSPACE_BYTES), stream);
}

ATTN_EXPORT int attn_check_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_DEVICE;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, attn::g_attn_status, sizeof(v)) != cudaSuccess) return ATTN_ERR_DEVICE;
  if (v != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(attn::g_attn_status, &zero, sizeof(zero)) != cudaSuccess) return ATTN_ERR_DEVICE;
    if (v & attn::kStatusLayout)
      return fail(ATTN_ERR_DEVICE, "%sa kernel found its shared memory window misaligned and did no work%lld", "", 0);
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
