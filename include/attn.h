/*
 * attn.h -- C ABI of libattn.so: exact, IO-aware tiled softmax attention on
 * NVIDIA B200 (sm_100a), forward and backward.
 *
 * What is computed (per batch b and head h, rows indexed 0..N-1):
 *
 *   S = scale * Q K^T,  S_ij = -inf for j > i when causal,
 *   P = rowwise softmax(S),  O = P V,  LSE_i = ln sum_j exp(S_ij).
 *
 * The result is the dense softmax attention of the standard four-step
 * computation (score, mask, softmax, weight -- "FlashAttention" flagship
 * module, Beat 01), reached tile by tile: a Q block stays on chip while K/V
 * blocks stream past it, and an online softmax keeps a running row max and
 * row sum and rescales the accumulator when the max grows ("Attention and KV
 * Compression", section "Tiling and online softmax"; "FlashAttention -- how
 * 100K-token attention fits in memory", sections "FlashAttention idea" and
 * "Online softmax intuition").  Only O and one statistic per row (LSE) are
 * written to device memory; no N x N buffer exists at any point.  The
 * backward recomputes score tiles from Q, K, V and LSE instead of storing P
 * ("Attention and KV Compression", section "Recomputation in the backward
 * pass").
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Layout "BHND": contiguous [B][H][N][d] bfloat16 (row stride d elements).
 *    Q, K, V, O, dO, dQ, dK, dV all use it.  LSE is fp32 [B][H][N], natural log.
 *  - d must be 64 or 128 (otherwise ATTN_ERR_UNSUPPORTED).  N >= 1 is any
 *    value; partial tiles are handled.  B, H >= 1.  B*H and N must each fit
 *    in 31 bits.
 *  - scale must be finite and > 0 (otherwise ATTN_ERR_INVALID_ARG).
 *  - Every pointer is a DEVICE pointer owned by the caller; the library keeps
 *    no reference after the call returns and never allocates device memory.
 *    Every pointer must be 16-byte aligned (ATTN_ERR_MISALIGNED otherwise).
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *    enqueued asynchronously on it; the call returns once it is enqueued.
 *  - Argument errors are reported synchronously, before anything is launched.
 *    A launch failure returns ATTN_ERR_LAUNCH.  Device-side waits are bounded:
 *    a wait that runs out sets a device status word that attn_check_status
 *    reports as ATTN_ERR_TIMEOUT (the kernel then releases its tensor memory
 *    and returns; its outputs are undefined).  The library never traps,
 *    aborts or prints.
 */
#ifndef EXACT_ATTN_B200_ATTN_H
#define EXACT_ATTN_B200_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = -1,
  ATTN_ERR_UNSUPPORTED = -2,
  ATTN_ERR_MISALIGNED = -3,
  ATTN_ERR_WORKSPACE = -4,
  ATTN_ERR_LAUNCH = -5,
  ATTN_ERR_TIMEOUT = -6,
  ATTN_ERR_DEVICE = -7
} attn_status_t;

/*
 * Forward pass.  Reads Q, K, V; writes O (bf16, BHND) and LSE (fp32 [B][H][N]).
 * Tiled exact attention with online softmax ("Attention and KV Compression",
 * section "Tiling and online softmax").  O and LSE must not alias the inputs.
 */
int attn_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE,
             int64_t B, int64_t H, int64_t N, int64_t d, int causal, float scale,
             void* stream);

/*
 * attn_fwd that also writes O32: the normalised output rows in fp32 ([B][H][N][d],
 * the same values before their rounding to bf16), for checking the forward
 * against a tolerance finer than the bf16 output's own rounding.  O32 must be
 * non-null (else ATTN_ERR_INVALID_ARG) and 16-byte aligned; it costs one extra
 * write of 4 bytes per output element.  Everything else as attn_fwd.
 */
int attn_fwd_f32out(const void* Q, const void* K, const void* V, void* O, float* O32, float* LSE,
                    int64_t B, int64_t H, int64_t N, int64_t d, int causal, float scale, void* stream);

/*
 * Forward with shared key/value heads (grouped-query / multi-query attention):
 * H query heads, H_kv key/value heads, H % H_kv == 0; query head h of batch b
 * attends with key/value head h / (H / H_kv) of batch b.  Head sharing changes
 * how many key/value heads exist while the kernel still tiles over them
 * ("Attention and KV Compression", section "The composability point").
 * Q, O: [B][H][N][d]; K, V: [B][H_kv][N][d]; LSE: [B][H][N].  attn_fwd is this
 * call with H_kv = H.
 */
int attn_fwd_gqa(const void* Q, const void* K, const void* V, void* O, float* LSE,
                 int64_t B, int64_t H, int64_t H_kv, int64_t N, int64_t d, int causal, float scale,
                 void* stream);

/*
 * Forward over packed sequences of different lengths (prefill of many
 * sequences in one call: "FlashAttention -- how 100K-token attention fits in
 * memory", section "Arithmetic intensity"; the tiling and online softmax are
 * those of attn_fwd).  Sequence s holds tokens [cu_seqlens[s], cu_seqlens[s+1])
 * of the packed tensors and attends only to its own tokens (causal: token i of
 * a sequence sees its tokens 0..i).
 *   Q, O        bf16 [total][H][d]      (token-major, row stride H*d)
 *   K, V        bf16 [total][H_kv][d]   query head h reads key/value head h / (H / H_kv)
 *   LSE         fp32 [H][total]         natural-log row log-sum-exp
 *   cu_seqlens  int32 [n_seqs + 1] DEVICE array, non-decreasing, cu_seqlens[0] = 0,
 *               cu_seqlens[n_seqs] = total (4-byte aligned).  Offsets are clamped
 *               to [0, total] on the device, so nothing outside the tensors is read
 *               or written whatever the array holds; tokens outside every sequence
 *               get no output.  Empty sequences are allowed.
 * d must be 64 or 128 (else ATTN_ERR_UNSUPPORTED); n_seqs, total >= 1.  The
 * result for each sequence equals attn_fwd_gqa on that sequence alone, bit for
 * bit.  Other rules as attn_fwd.
 */
int attn_fwd_varlen(const void* Q, const void* K, const void* V, void* O, float* LSE,
                    const int32_t* cu_seqlens, int64_t n_seqs, int64_t total, int64_t H, int64_t H_kv,
                    int64_t d, int causal, float scale, void* stream);

/*
 * Forward restricted to selected blocks ("Attention and KV Compression",
 * section "The composability point": sparse selection changes which blocks
 * are attended, and the kernel runs on the selected blocks).
 * block_mask: DEVICE pointer to [B*H][nt][nt] bytes, nt = ceil(N/128);
 * block_mask[(b*H + h)*nt*nt + i*nt + j] != 0 means query rows 128i..128i+127
 * of head (b, h) attend key rows 128j..128j+127 (further restricted to j <= i
 * row-wise when causal).  Only selected key tiles are loaded and multiplied.
 * A row that sees no key gets O = 0 and LSE = -inf.  Shared key/value heads
 * as in attn_fwd_gqa (H_kv = H for plain multi-head attention).
 */
int attn_fwd_blocksparse(const void* Q, const void* K, const void* V, void* O, float* LSE,
                         const uint8_t* block_mask,
                         int64_t B, int64_t H, int64_t H_kv, int64_t N, int64_t d, int causal,
                         float scale, void* stream);

/*
 * Forward on FP8 inputs ("Attention and KV Compression", section "What it
 * does and does not change": later versions add narrower numeric formats;
 * the computation is unchanged).
 *   Q8       uint8 [B][H][N][128]   E4M3 codes (OCP FP8 E4M3: bias 7, no inf)
 *   K8, V8   uint8 [B][H_kv][N][128]
 *   O        bf16  [B][H][N][128],  LSE fp32 [B][H][N] (natural log)
 * The attention is that of attn_fwd_gqa on the dequantised tensors
 * Q = q_descale * Q8, K = k_descale * K8, V = v_descale * V8 (each descale
 * finite and > 0).  QK^T and PV run on the E4M3 tensor-core path with fp32
 * accumulation; the products Q8 K8^T are exact, and the row max, row sum and
 * LSE are fp32.  P is rounded to E4M3 for the PV product (each p changes by at
 * most 2^-4 of itself or 2^-10 absolute, p <= 2^8), so per row
 * |O - O_exact| <= v_descale * max|V8| * (2^-4 + n_visible * 2^-10 / l) where
 * l = sum_j exp(S_ij - max_j S_ij), plus the bf16 rounding of O.
 * d must be 128 (else ATTN_ERR_UNSUPPORTED).  Other rules as attn_fwd.
 */
int attn_fwd_fp8(const void* Q8, const void* K8, const void* V8, void* O, float* LSE,
                 int64_t B, int64_t H, int64_t H_kv, int64_t N, int64_t d, int causal, float scale,
                 float q_descale, float k_descale, float v_descale, void* stream);

/*
 * Forward of Nq new query rows against a key/value cache (decode and
 * chunked-prefill shapes: "FlashAttention -- how 100K-token attention fits in
 * memory", section "Arithmetic intensity", where prefill and decode are the
 * same computation in two shape regimes; the tiling and online softmax are
 * those of attn_fwd).
 *   Q, O    bf16 [B][H][Nq][d] row-major (device, 16-byte aligned)
 *   K, V    bf16 [B][H_kv][Nk][d] (the cache; Nk = its capacity in rows)
 *   LSE     fp32 [B][H][Nq] natural-log row log-sum-exp
 *   kv_lens int32 [B] device array, or NULL: batch entry b uses cache rows
 *           [0, L_b), L_b = kv_lens[b] (clamped to [0, Nk]); NULL means L_b = Nk.
 *           Rows [L_b, Nk) are never weighted, whatever they hold.
 * The new rows are the LAST Nq positions of a sequence of L_b tokens: with
 * `causal`, position p (0-based among the Nq rows) sees cache row j iff
 * j <= p + L_b - Nq (bottom-right alignment; Nq = Nk = L_b is attn_fwd's
 * mask).  A row that sees no key (L_b = 0, or p + L_b - Nq < 0) gets O = 0 and
 * LSE = -inf.  Query head h reads key/value head h / (H / H_kv).
 * num_splits: key tiles of each (key/value head, 128 packed query rows) are
 * cut into this many chunks (work items of a persistent grid) and the partial
 * results are merged by their LSE; 0 picks a count that fills the GPU's 148
 * SMs.  When (H / H_kv) * Nq <= 32 the packed rows are replicated into all
 * four TMEM lane quarters and every key tile is split four ways, so each chunk
 * yields four partials.  Whenever there is more than one partial the call
 * needs attn_fwd_kvcache_workspace_bytes() bytes of device workspace
 * (16-byte aligned) for the fp32 partials, else ATTN_ERR_WORKSPACE (or
 * ATTN_ERR_INVALID_ARG for NULL); when that function returns 0, `workspace`
 * may be NULL.  Requires B*H*Nq < 2^31 - 128.
 * Outputs must not alias inputs or the workspace.
 */
int attn_fwd_kvcache(const void* Q, const void* K, const void* V, void* O, float* LSE,
                     const int32_t* kv_lens,
                     int64_t B, int64_t H, int64_t H_kv, int64_t Nq, int64_t Nk, int64_t d,
                     int causal, float scale, int64_t num_splits,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_fwd_kvcache with the cache stored in FP8: K8, V8 are uint8 [B][H_kv][Nk][128]
 * E4M3 codes with per-tensor dequantisation factors k_descale, v_descale (finite,
 * > 0); the result is attn_fwd_kvcache's on K = k_descale * K8, V = v_descale * V8.
 * Reading half the bytes per cached row is the point: decode reads the whole
 * cache every step.  Arithmetic: the scores are formed on the E4M3 key codes
 * directly, with each query row scaled by a power of two (largest element in
 * [128, 256)) and written as the sum of two E4M3 terms -- exact for elements of
 * at least 2^-10 of the row's largest magnitude, within 2^-10 (scaled units)
 * below that -- with fp32 accumulation; the value codes are widened to f16 on
 * chip without rounding and P is rounded to f16.  Statistics are fp32 as in
 * the bf16 path, whose tolerances apply.  Q elements must be finite.  Q, O bf16
 * and LSE, kv_lens, causal alignment, num_splits as in attn_fwd_kvcache.
 * Restrictions: d = 128 and (H / H_kv) * Nq <= 32 (decode
 * shapes), else ATTN_ERR_UNSUPPORTED.  The workspace is always needed, sized by
 * attn_fwd_kvcache_workspace_bytes() with the same arguments.
 */
int attn_fwd_kvcache_fp8(const void* Q, const void* K8, const void* V8, void* O, float* LSE,
                         const int32_t* kv_lens,
                         int64_t B, int64_t H, int64_t H_kv, int64_t Nq, int64_t Nk, int64_t d,
                         int causal, float scale, float k_descale, float v_descale, int64_t num_splits,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * Number of key chunks attn_fwd_kvcache uses for these arguments (num_splits
 * as passed to it, 0 = automatic), and the workspace bytes it then needs:
 * partials * B*H*Nq * (d + 1) * 4 with partials = splits * (4 if
 * (H / H_kv) * Nq <= 32 else 1), or 0 when there is a single partial.  Both
 * return 0 for sizes attn_fwd_kvcache would reject.
 */
int64_t attn_fwd_kvcache_splits(int64_t B, int64_t H, int64_t H_kv, int64_t Nq, int64_t Nk, int64_t d,
                                int64_t num_splits);
size_t attn_fwd_kvcache_workspace_bytes(int64_t B, int64_t H, int64_t H_kv, int64_t Nq, int64_t Nk, int64_t d,
                                        int64_t num_splits);

/*
 * Bytes of caller-provided device workspace that attn_bwd (and attn_bwd_gqa,
 * attn_bwd_blocksparse) need for these sizes: two fp32 per-row vectors per
 * head plus an fp32 dQ accumulator of d values per row, each padded to a
 * multiple of 128 rows: B*H*Npad*(2 + d)*4 bytes, Npad = N rounded up to 128.
 * Returns 0 for sizes that attn_bwd would reject.
 */
size_t attn_bwd_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t d);

/*
 * Bytes of workspace that attn_bwd_deterministic and the three split steps
 * (attn_bwd_preprocess, attn_bwd_dkdv, attn_bwd_dq) need: the two per-row
 * vectors only, B*H*Npad*2*4 bytes.  0 for rejected sizes.
 */
size_t attn_bwd_deterministic_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t d);

/*
 * Backward pass by recomputation ("Attention and KV Compression", section
 * "Recomputation in the backward pass"; "FlashAttention -- how 100K-token
 * attention fits in memory", section "Training backward").
 * Inputs: Q, K, V, the forward's O and LSE, and the output gradient dO.
 * Outputs: dQ, dK, dV (bf16, BHND).  Three kernels run on `stream`:
 *   (1) per row, D_i = sum_k dO_ik O_ik and LSE_i * log2(e) into `workspace`,
 *       and the fp32 dQ accumulator cleared;
 *   (2) per 128-key tile, one pass over the query tiles: the score tiles are
 *       recomputed once and give dK, dV (summed in tensor memory) and, from
 *       the same dS, each query tile's dQ contribution, which is added into
 *       the fp32 accumulator (5 MMAs per tile pair);
 *   (3) dQ = scale * accumulator, rounded to bf16.
 * The additions into the accumulator happen in an order that varies from run
 * to run, so dQ can differ between runs in its last bits (dK and dV do not);
 * attn_bwd_deterministic gives bitwise-reproducible results at a higher cost.
 * `workspace` (device, 16-byte aligned) must hold attn_bwd_workspace_bytes()
 * bytes, else ATTN_ERR_WORKSPACE; its layout after the call is
 * [B*H][Npad] fp32 LSE*log2(e) (padding rows +inf), [B*H][Npad] fp32 D
 * (padding rows 0), then [B*H][Npad][d] fp32 dQ / scale (rows >= N unused).
 * Outputs must not alias inputs or the workspace.
 */
int attn_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
             const float* LSE, void* dQ, void* dK, void* dV,
             int64_t B, int64_t H, int64_t N, int64_t d, int causal, float scale,
             void* workspace, size_t workspace_bytes, void* stream);

/*
 * The three steps of attn_bwd, callable one at a time (same arguments, rules
 * and workspace as attn_bwd; attn_bwd is exactly these three calls in this
 * order on one stream).  Useful to time the steps separately.
 *
 * attn_bwd_fused_preprocess: per row, D_i = sum_k dO_ik O_ik and
 *   LSE_i*log2(e) into `workspace`, and the fp32 dQ accumulator set to zero.
 * attn_bwd_fused_dkdvdq: one CTA per 128-key tile; writes dK and dV and adds
 *   every query tile's dQ contribution (dS K_j, before the scale) into the
 *   accumulator; reads the vectors ("Attention and KV Compression", section
 *   "Recomputation in the backward pass": the score tiles are recomputed once).
 * attn_bwd_fused_dq_convert: dQ = scale * accumulator, rounded to bf16.
 */
int attn_bwd_fused_preprocess(const void* O, const void* dO, const float* LSE,
                              int64_t B, int64_t H, int64_t N, int64_t d,
                              void* workspace, size_t workspace_bytes, void* stream);

int attn_bwd_fused_dkdvdq(const void* Q, const void* K, const void* V, const void* dO,
                          void* dK, void* dV,
                          int64_t B, int64_t H, int64_t N, int64_t d, int causal, float scale,
                          void* workspace, size_t workspace_bytes, void* stream);

int attn_bwd_fused_dq_convert(void* dQ, int64_t B, int64_t H, int64_t N, int64_t d, float scale,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * The same backward with bitwise-reproducible results: (1) the per-row vectors
 * as in attn_bwd, (2) per 128-key tile, dK and dV (score tiles recomputed, 4
 * MMAs per tile pair), (3) per 128-query tile, dQ (score tiles recomputed
 * again, 3 MMAs per tile pair) -- no accumulation across CTAs, so no order
 * dependence, at the price of recomputing S and dP twice.  Shared key/value
 * heads as in attn_bwd_gqa (H_kv = H for multi-head attention).  `workspace`
 * must hold attn_bwd_deterministic_workspace_bytes() bytes (layout: the two
 * per-row vectors of attn_bwd).  It is exactly attn_bwd_preprocess,
 * attn_bwd_dkdv and attn_bwd_dq in this order (for H_kv = H).
 */
int attn_bwd_deterministic(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                           const float* LSE, void* dQ, void* dK, void* dV,
                           int64_t B, int64_t H, int64_t H_kv, int64_t N, int64_t d, int causal, float scale,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward with shared key/value heads (see attn_fwd_gqa for the layout).
 * dQ: [B][H][N][d]; dK, dV: [B][H_kv][N][d], each the sum over the H / H_kv
 * query heads that share the key/value head (the per-key-tile kernel loops
 * over those query heads, so the sum is formed in tensor memory without
 * atomics).  Kernels and workspace as attn_bwd, sized by
 * attn_bwd_workspace_bytes(B, H, N, d) (query heads).  attn_bwd is this call
 * with H_kv = H.
 */
int attn_bwd_gqa(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                 const float* LSE, void* dQ, void* dK, void* dV,
                 int64_t B, int64_t H, int64_t H_kv, int64_t N, int64_t d, int causal, float scale,
                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward of attn_fwd_blocksparse (same block_mask, same layouts and
 * workspace as attn_bwd_gqa).  The per-key-tile kernel visits only the
 * (query head, query tile) pairs that selected its key tile.  Rows with
 * LSE = -inf contribute nothing; key tiles that no query tile selected get
 * dK = dV = 0, and query tiles that selected no key tile get dQ = 0.
 */
int attn_bwd_blocksparse(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                         const float* LSE, const uint8_t* block_mask, void* dQ, void* dK, void* dV,
                         int64_t B, int64_t H, int64_t H_kv, int64_t N, int64_t d, int causal, float scale,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * The three steps of attn_bwd_deterministic, callable one at a time (same
 * arguments and rules; attn_bwd_deterministic with H_kv = H is exactly these
 * three calls in this order on one stream; the workspace is sized by
 * attn_bwd_deterministic_workspace_bytes()).  Useful to time the steps
 * separately or to run dK/dV and dQ on different streams once the preprocess
 * step has completed.
 *
 * attn_bwd_preprocess: per row, D_i = sum_k dO_ik O_ik and LSE_i*log2(e)
 *   into `workspace` (layout as for attn_bwd).  D is the row term of the
 *   softmax gradient dS = P o (dP - D) ("Attention and KV Compression",
 *   section "Recomputation in the backward pass": only the small per-row
 *   statistics are kept from the forward).
 * attn_bwd_dkdv: dK and dV, one CTA per 128-key tile; reads the workspace.
 * attn_bwd_dq: dQ, one CTA per 128-query tile; reads the workspace.
 */
int attn_bwd_preprocess(const void* O, const void* dO, const float* LSE,
                        int64_t B, int64_t H, int64_t N, int64_t d,
                        void* workspace, size_t workspace_bytes, void* stream);

int attn_bwd_dkdv(const void* Q, const void* K, const void* V, const void* dO,
                  void* dK, void* dV,
                  int64_t B, int64_t H, int64_t N, int64_t d, int causal, float scale,
                  const void* workspace, size_t workspace_bytes, void* stream);

int attn_bwd_dq(const void* Q, const void* K, const void* V, const void* dO, void* dQ,
                int64_t B, int64_t H, int64_t N, int64_t d, int causal, float scale,
                const void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward without any caller-provided memory: same computation, arguments
 * and results as attn_bwd_deterministic (H_kv = H), but the workspace is a
 * fixed array that the library owns in device memory.  (The pages have no
 * counterpart: this is a deployment convenience, not part of the method.)
 *
 * Who needs it: callers that cannot allocate device memory where they run
 * the backward -- e.g. code inside a runtime whose memory is owned by another
 * allocator that offers no way to pass a raw scratch buffer across a C
 * boundary, or code under a "no device allocation after start-up" rule (an
 * allocation there can synchronise the device or is forbidden outright).
 *
 * Limits and behaviour:
 *  - The array is ATTN_STATIC_WORKSPACE_BYTES (32 MiB) on every GPU that
 *    loads the library, held from module load until process exit.  Sizes
 *    whose attn_bwd_deterministic_workspace_bytes() exceed it are rejected
 *    with ATTN_ERR_WORKSPACE before anything is launched (attn_last_error()
 *    says how many bytes they need).  32 MiB covers B*H*ceil(N/128)*128 up
 *    to 2^22 rows, e.g. B=8, H=32, N=16384.
 *  - The array belongs to the library's module in the calling thread's
 *    current CUDA context (on its current device); every call looks its
 *    device address up there (cudaGetSymbolAddress, which allocates
 *    nothing).  The first call in a context loads the module there if it
 *    is not loaded yet (work the CUDA runtime does, as for any first kernel
 *    launch from a module).
 *  - It calls no cudaMalloc, cudaFree or other allocating routine.
 *  - Every call in a context shares the one array, and the array keeps the
 *    last call's contents.  Nothing in it needs to start at zero: the
 *    preprocess step writes every workspace element a call reads before the
 *    other kernels read it.  Calls whose GPU work overlaps (e.g. on two
 *    streams, or from two threads) race on the array; serialise them.
 */
#define ATTN_STATIC_WORKSPACE_BYTES (32u * 1024u * 1024u)

int attn_bwd_static_workspace(const void* Q, const void* K, const void* V, const void* O,
                              const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                              int64_t B, int64_t H, int64_t N, int64_t d, int causal, float scale,
                              void* stream);

/*
 * Self-test of the failure path (no counterpart on the pages: it checks the
 * library's bounded waits).  Enqueues one small kernel that allocates tensor
 * memory, waits on a barrier that nothing arrives on, gives up after 20 ms
 * exactly as the attention kernels do when a wait runs out (it raises the
 * device status word, releases its tensor memory and returns), so that the
 * next attn_check_status() reports ATTN_ERR_TIMEOUT and the context stays
 * usable.  Returns ATTN_OK once enqueued.  Nothing faults, traps or hangs.
 */
int attn_selftest_wait_timeout(void* stream);

/*
 * Synchronises `stream`, then reports and clears the device status word:
 * ATTN_OK, ATTN_ERR_TIMEOUT (a bounded device-side wait ran out in some
 * kernel since the last check), or ATTN_ERR_DEVICE (the CUDA context reports
 * an error).
 */
int attn_check_status(void* stream);

/*
 * Detail of the most recent failure reported by an entry point on the calling
 * host thread (which CUDA call failed and its error), or "" if none.  The
 * string is owned by the library and valid until the next call on the thread.
 */
const char* attn_last_error(void);

/* Static, human-readable name of a status code. */
const char* attn_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_ATTN_B200_ATTN_H */
