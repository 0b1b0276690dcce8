"""Plain fp64 CPU oracle for exact softmax attention, forward and backward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may call it.  It shares no code with the CUDA library.

What it computes (the plain definition that the tiled method reaches exactly,
up to floating-point reassociation -- "Attention and KV Compression",
section "What it does and does not change"; "FlashAttention -- how 100K-token
attention fits in memory", section "Why 'exact' matters"):

    S = scale * Q K^T                  (N x N, materialised per head)
    S_ij = -inf  for j > i             (causal mask, if requested)
    P = softmax(S) row-wise            (p_i = e^{s_i} / sum_j e^{s_j}, FlashAttention
                                        page, section "But softmax needs the whole row")
    O = P V
    LSE_i = m_i + ln sum_j exp(S_ij - m_i),   m_i = max_j S_ij

The backward is the explicit chain rule through the same materialised
matrices (the quantities the tiled backward recomputes tile by tile --
"Attention and KV Compression", section "Recomputation in the backward pass"):

    dV = P^T dO
    dP = dO V^T
    D_i = sum_j P_ij dP_ij
    dS = P o (dP - D)
    dQ = scale * dS K
    dK = scale * dS^T Q

All arithmetic is float64 (numpy); matrix products use numpy's matmul as a
library primitive.  Inputs are arrays of shape (BH, N, d) (any float dtype,
upcast to float64 here); heads are processed one at a time so that only one
N x N matrix per head is resident.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(worked online-softmax example, row sums, blockwise-vs-one-shot equality,
closed forms, finite differences, an autograd cross-check).
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "head_scores",
    "row_softmax",
    "attn_fwd",
    "attn_fwd_rows",
    "attn_bwd",
    "expand_kv",
    "attn_fwd_gqa",
    "attn_bwd_gqa",
    "BLOCK",
    "blocksparse_scores",
    "masked_row_softmax",
    "attn_fwd_blocksparse",
    "attn_bwd_blocksparse",
    "attn_fwd_kvcache",
    "e4m3_decode",
    "attn_fwd_fp8",
    "attn_fwd_kvcache_fp8",
    "attn_fwd_varlen",
]


def head_scores(q: np.ndarray, k: np.ndarray, scale: float, causal: bool,
                rows: np.ndarray | None = None) -> np.ndarray:
    """Scaled scores of one head, with the causal mask written in as -inf.

    ``rows`` selects a subset of query rows (their global indices); the mask
    uses those global indices.  The mask form (key j visible to query i iff
    j <= i, queries and keys indexed from the same origin) is the plain
    reading of the "mask" step of standard attention (FlashAttention flagship
    page, Beat 01).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    if rows is None:
        rows = np.arange(q.shape[0])
    else:
        rows = np.asarray(rows, dtype=np.int64)
        q = q[rows]
    s = float(scale) * (q @ k.T)
    if causal:
        cols = np.arange(k.shape[0])
        s[cols[None, :] > rows[:, None]] = -np.inf
    return s


def row_softmax(s: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Row-wise softmax and log-sum-exp of a score matrix.

    p_ij = exp(s_ij - m_i) / sum_j exp(s_ij - m_i) with m_i the row maximum;
    LSE_i = m_i + ln sum_j exp(s_ij - m_i).  Returns (P, LSE).
    """
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    l = np.sum(e, axis=1, keepdims=True)
    p = e / l
    lse = (m + np.log(l))[:, 0]
    return p, lse


def _as3(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    if x.ndim == 2:
        x = x[None]
    if x.ndim != 3:
        raise ValueError("expected (BH, N, d) or (N, d)")
    return x


def attn_fwd(Q, K, V, scale: float, causal: bool, return_probs: bool = False):
    """Forward: O (BH, N, d) and LSE (BH, N); optionally P (BH, N, N)."""
    Q, K, V = _as3(Q), _as3(K), _as3(V)
    bh, n, d = Q.shape
    O = np.empty((bh, n, d), dtype=np.float64)
    LSE = np.empty((bh, n), dtype=np.float64)
    Ps = np.empty((bh, n, n), dtype=np.float64) if return_probs else None
    for h in range(bh):
        s = head_scores(Q[h], K[h], scale, causal)
        p, lse = row_softmax(s)
        del s
        O[h] = p @ V[h]
        LSE[h] = lse
        if return_probs:
            Ps[h] = p
    if return_probs:
        return O, LSE, Ps
    return O, LSE


def attn_fwd_rows(q, k, v, scale: float, causal: bool, rows):
    """Forward for selected query rows of ONE head: O_rows (r, d), LSE_rows (r,).

    Row i of the result depends only on row i of S, so this is the same
    definition evaluated on a subset of rows (used where N is too large to
    materialise the full N x N matrix in host memory).
    """
    v = np.asarray(v, dtype=np.float64)
    s = head_scores(q, k, scale, causal, rows=rows)
    p, lse = row_softmax(s)
    return p @ v, lse


def attn_bwd(Q, K, V, dO, scale: float, causal: bool):
    """Backward: dQ, dK, dV (each (BH, N, d)) from the explicit chain rule."""
    Q, K, V, dO = _as3(Q), _as3(K), _as3(V), _as3(dO)
    bh, n, d = Q.shape
    dQ = np.empty((bh, n, d), dtype=np.float64)
    dK = np.empty((bh, n, d), dtype=np.float64)
    dV = np.empty((bh, n, d), dtype=np.float64)
    for h in range(bh):
        s = head_scores(Q[h], K[h], scale, causal)
        p, _ = row_softmax(s)
        del s
        dV[h] = p.T @ dO[h]
        dp = dO[h] @ V[h].T
        D = np.sum(p * dp, axis=1, keepdims=True)
        ds = p * (dp - D)
        del dp, p
        dQ[h] = float(scale) * (ds @ K[h])
        dK[h] = float(scale) * (ds.T @ Q[h])
    return dQ, dK, dV


# ---------------------------------------------------------------------------
# Shared key/value heads (grouped-query / multi-query attention): H query heads
# and H_kv key/value heads per batch, query head h using key/value head
# h // (H // H_kv) ("Attention and KV Compression", section "The
# composability point": head sharing changes how many key/value heads exist).
# By definition this is multi-head attention on keys/values repeated to H
# heads; the gradient of a shared key/value head is the sum of the gradients
# of its copies (chain rule through the repetition).
# ---------------------------------------------------------------------------

def expand_kv(X, B: int, H: int, H_kv: int):
    """(B*H_kv, N, d) -> (B*H, N, d): row b*H + h is X[b*H_kv + h // (H // H_kv)]."""
    X = _as3(X)
    g = H // H_kv
    idx = np.array([b * H_kv + h // g for b in range(B) for h in range(H)], dtype=np.int64)
    return X[idx]


def attn_fwd_gqa(Q, K, V, scale: float, causal: bool, B: int, H: int, H_kv: int):
    """Forward with shared key/value heads: O, LSE of shape (B*H, N, d), (B*H, N)."""
    return attn_fwd(Q, expand_kv(K, B, H, H_kv), expand_kv(V, B, H, H_kv), scale, causal)


def attn_bwd_gqa(Q, K, V, dO, scale: float, causal: bool, B: int, H: int, H_kv: int):
    """Backward with shared key/value heads: dQ (B*H, N, d); dK, dV (B*H_kv, N, d)."""
    dQ, dKe, dVe = attn_bwd(Q, expand_kv(K, B, H, H_kv), expand_kv(V, B, H, H_kv), dO, scale, causal)
    g = H // H_kv
    n, d = dKe.shape[1:]
    dK = dKe.reshape(B, H_kv, g, n, d).sum(axis=2).reshape(B * H_kv, n, d)
    dV = dVe.reshape(B, H_kv, g, n, d).sum(axis=2).reshape(B * H_kv, n, d)
    return dQ, dK, dV


# ---------------------------------------------------------------------------
# Block-sparse selection ("Attention and KV Compression", section "The
# composability point": sparse selection changes which blocks are attended and
# the kernel runs on the selected blocks).  A block mask M of shape
# (B*H, ceil(N/T), ceil(N/T)), T = 128, marks which key tiles each query tile
# attends; S_ij = -inf unless M[bh, i // T, j // T] (and j <= i when causal).
# Rows left with no visible key have no softmax; their output is taken as
# O = 0, LSE = -inf and they contribute no gradient (the reading used for
# fully masked rows).
# ---------------------------------------------------------------------------

BLOCK = 128


def blocksparse_scores(q, k, scale: float, causal: bool, mask_tiles: np.ndarray) -> np.ndarray:
    """Scores of one head with the block mask (and causal mask) written in as -inf."""
    s = head_scores(q, k, scale, causal)
    n = s.shape[0]
    tiles = np.arange(n) // BLOCK
    keep = np.asarray(mask_tiles, dtype=bool)[tiles[:, None], tiles[None, :]]
    s[~keep] = -np.inf
    return s


def masked_row_softmax(s: np.ndarray):
    """row_softmax, extended to rows with no finite score: P = 0, LSE = -inf."""
    m = np.max(s, axis=1, keepdims=True)
    empty = ~np.isfinite(m[:, 0])
    m_safe = np.where(empty[:, None], 0.0, m)
    e = np.exp(s - m_safe)
    l = np.sum(e, axis=1, keepdims=True)
    p = np.where(empty[:, None], 0.0, e / np.where(empty[:, None], 1.0, l))
    lse = np.where(empty, -np.inf, (m_safe + np.log(np.where(empty[:, None], 1.0, l)))[:, 0])
    return p, lse


def attn_fwd_blocksparse(Q, K, V, scale: float, causal: bool, mask, B: int, H: int, H_kv: int):
    """Forward under a block mask (B*H, nt, nt); K, V have B*H_kv heads."""
    Q = _as3(Q)
    Ke, Ve = expand_kv(K, B, H, H_kv), expand_kv(V, B, H, H_kv)
    bh, n, d = Q.shape
    O = np.empty((bh, n, d))
    LSE = np.empty((bh, n))
    for h in range(bh):
        p, lse = masked_row_softmax(blocksparse_scores(Q[h], Ke[h], scale, causal, mask[h]))
        O[h] = p @ Ve[h]
        LSE[h] = lse
    return O, LSE


def attn_bwd_blocksparse(Q, K, V, dO, scale: float, causal: bool, mask, B: int, H: int, H_kv: int):
    """Backward under a block mask: dQ (B*H, N, d); dK, dV (B*H_kv, N, d)."""
    Q, dO = _as3(Q), _as3(dO)
    Ke, Ve = expand_kv(K, B, H, H_kv), expand_kv(V, B, H, H_kv)
    bh, n, d = Q.shape
    dQ = np.empty((bh, n, d))
    dKe = np.empty((bh, n, d))
    dVe = np.empty((bh, n, d))
    for h in range(bh):
        p, _ = masked_row_softmax(blocksparse_scores(Q[h], Ke[h], scale, causal, mask[h]))
        dVe[h] = p.T @ dO[h]
        dp = dO[h] @ Ve[h].T
        D = np.sum(p * dp, axis=1, keepdims=True)
        ds = p * (dp - D)
        dQ[h] = float(scale) * (ds @ Ke[h])
        dKe[h] = float(scale) * (ds.T @ Q[h])
    g = H // H_kv
    dK = dKe.reshape(B, H_kv, g, n, d).sum(axis=2).reshape(B * H_kv, n, d)
    dV = dVe.reshape(B, H_kv, g, n, d).sum(axis=2).reshape(B * H_kv, n, d)
    return dQ, dK, dV


# ---------------------------------------------------------------------------
# Decode-shaped attention against a key/value cache ("FlashAttention -- how
# 100K-token attention fits in memory", section "Arithmetic intensity": prefill
# and decode are the same computation in different shape regimes).  Nq new
# query rows attend to the first L_b cached keys/values of their batch entry
# (L_b = kv_lens[b], default Nk).  The queries are the LAST Nq positions of that
# length-L_b sequence, so under the causal mask query p (0-based among the new
# rows) sees key j iff j <= p + L_b - Nq (bottom-right alignment; with Nq = Nk
# it is the square mask above).  Rows that see no key follow the fully masked
# row reading: O = 0, LSE = -inf.  Keys past L_b do not exist for that batch
# entry: they are sliced away before any arithmetic.
# ---------------------------------------------------------------------------

def attn_fwd_kvcache(Q, K, V, scale: float, causal: bool, B: int, H: int, H_kv: int, kv_lens=None):
    """Q (B*H, Nq, d); K, V (B*H_kv, Nk, d); kv_lens (B,) or None -> O (B*H, Nq, d), LSE (B*H, Nq)."""
    Q = _as3(Q)
    Ke, Ve = expand_kv(K, B, H, H_kv), expand_kv(V, B, H, H_kv)
    bh, nq, d = Q.shape
    nk = Ke.shape[1]
    lens = [nk] * B if kv_lens is None else [int(x) for x in kv_lens]
    O = np.empty((bh, nq, d))
    LSE = np.empty((bh, nq))
    for h in range(bh):
        L = lens[h // H]
        if not 0 <= L <= nk:
            raise ValueError("kv_lens entries must lie in [0, Nk]")
        k, v = Ke[h, :L], Ve[h, :L]
        s = float(scale) * (Q[h] @ k.T)                      # (Nq, L)
        if causal:
            p = np.arange(nq)[:, None]
            j = np.arange(L)[None, :]
            s[j > p + (L - nq)] = -np.inf
        if L == 0:
            O[h] = 0.0
            LSE[h] = -np.inf
            continue
        pr, lse = masked_row_softmax(s)
        O[h] = pr @ v
        LSE[h] = lse
    return O, LSE


# ---------------------------------------------------------------------------
# Narrower input format: FP8 E4M3 ("Attention and KV Compression", section
# "What it does and does not change": later versions add support for narrower
# numeric formats; the computation itself is unchanged).  Each of Q, K, V is
# given as E4M3 codes plus one per-tensor dequantisation factor; the attention
# is the plain definition above applied to the dequantised values
# X = descale_X * decode(X8).
# ---------------------------------------------------------------------------

def e4m3_decode(codes) -> np.ndarray:
    """E4M3 byte codes -> float64 values, from the format's definition.

    1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; exponent field 0
    holds subnormals m/8 * 2^-6; exponent 15 with mantissa 7 is NaN (the only
    special code: no infinities), so the largest finite magnitude is
    1.75 * 2^8 = 448.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & ((c & 0x7) == 7), np.nan, mag)
    return sign * mag


def attn_fwd_fp8(Q8, K8, V8, q_descale: float, k_descale: float, v_descale: float, scale: float, causal: bool,
                 B: int, H: int, H_kv: int):
    """Forward on E4M3 inputs: Q8 (B*H, N, d), K8, V8 (B*H_kv, N, d) uint8 codes."""
    Q = float(q_descale) * e4m3_decode(Q8)
    K = float(k_descale) * e4m3_decode(K8)
    V = float(v_descale) * e4m3_decode(V8)
    return attn_fwd_gqa(Q, K, V, scale, causal, B, H, H_kv)


def attn_fwd_kvcache_fp8(Q, K8, V8, k_descale: float, v_descale: float, scale: float, causal: bool,
                         B: int, H: int, H_kv: int, kv_lens=None):
    """Decode against an E4M3 cache: attn_fwd_kvcache on K = k_descale * decode(K8), V = v_descale * decode(V8)."""
    K = float(k_descale) * e4m3_decode(K8)
    V = float(v_descale) * e4m3_decode(V8)
    return attn_fwd_kvcache(Q, K, V, scale, causal, B, H, H_kv, kv_lens=kv_lens)


# ---------------------------------------------------------------------------
# Packed variable-length sequences ("FlashAttention -- how 100K-token
# attention fits in memory", section "Arithmetic intensity": prefill of many
# sequences at once).  Sequence s holds tokens [cu[s], cu[s+1]) of the packed
# (total, H, d) tensors and attends only to its own tokens; each sequence is
# the plain attention above.
# ---------------------------------------------------------------------------

def attn_fwd_varlen(Q, K, V, cu_seqlens, scale: float, causal: bool, H: int, H_kv: int):
    """Q (total, H, d), K, V (total, H_kv, d), cu_seqlens (n_seqs + 1,) ->
    O (total, H, d), LSE (H, total).  Query head h reads key/value head
    h // (H // H_kv)."""
    Q, K, V = (np.asarray(x, dtype=np.float64) for x in (Q, K, V))
    total, _, d = Q.shape
    O = np.zeros((total, H, d))
    LSE = np.zeros((H, total))
    cu = [int(c) for c in cu_seqlens]
    for a, b in zip(cu[:-1], cu[1:]):
        if b <= a:
            continue
        q = Q[a:b].transpose(1, 0, 2)                      # (H, len, d)
        k = K[a:b].transpose(1, 0, 2)
        v = V[a:b].transpose(1, 0, 2)
        o, lse = attn_fwd_gqa(q, k, v, scale, causal, 1, H, H_kv)
        O[a:b] = o.transpose(1, 0, 2)
        LSE[:, a:b] = lse
    return O, LSE
