"""Pins for the fp64 oracle: checks against what the pages and mathematics fix.

None of these re-types the oracle's formulas.  Each pin comes from somewhere
else: the worked example printed on the pages, an invariant (rows of P sum to
one, permutation equivariance), an independent blockwise online-softmax
routine written here from the pages' description, closed forms of special
cases, central finite differences, or a library autograd.  Together they are
chosen so that a dropped term, a wrong sign or index, or a transposed operand
anywhere in the oracle fails at least one of them (``test_planted_mistakes``
checks that claim by planting such mistakes).
"""

import math
import os

import numpy as np
import pytest

from oracle import attn_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = (t.strip() for t in line.split("=", 1))
            out[key] = [float(x) for x in val.split()]
    return out


# ---------------------------------------------------------------------------
# Independent blockwise online softmax (test-only), written from the pages'
# description: "Attention and KV Compression", section "Tiling and online
# softmax"; FlashAttention page, sections "FlashAttention idea" and
# "Online softmax intuition".  Plain Python loops, fp64.
# ---------------------------------------------------------------------------

def blockwise_attention(q, k, v, scale, causal, br, bc, trace=None):
    n, d = q.shape
    out = np.zeros((n, d))
    lse = np.zeros(n)
    for i0 in range(0, n, br):
        for r in range(i0, min(i0 + br, n)):
            m_run = -math.inf
            l_run = 0.0
            acc = [0.0] * d
            for j0 in range(0, n, bc):
                cols = range(j0, min(j0 + bc, n))
                s = []
                for c in cols:
                    if causal and c > r:
                        s.append(-math.inf)
                    else:
                        s.append(scale * sum(q[r, t] * k[c, t] for t in range(d)))
                blk_max = max(s)
                m_new = max(m_run, blk_max)
                if m_new == -math.inf:
                    continue
                alpha = 0.0 if m_run == -math.inf else math.exp(m_run - m_new)
                if trace is not None and m_run != -math.inf:
                    trace.append((r, m_run, m_new, alpha))
                l_run *= alpha
                acc = [a * alpha for a in acc]
                for c, sc in zip(cols, s):
                    p = math.exp(sc - m_new)
                    l_run += p
                    for t in range(d):
                        acc[t] += p * v[c, t]
                m_run = m_new
            out[r] = [a / l_run for a in acc]
            lse[r] = m_run + math.log(l_run)
    return out, lse


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------------------
# The worked example printed on the pages
# ---------------------------------------------------------------------------

def test_worked_example_rescale_and_exactness():
    g = _read_golden("online_softmax_worked_example.txt")
    s1, s2 = g["block1_scores"], g["block2_scores"]
    scores = s1 + s2
    n = len(scores)
    # One query whose scores against the keys are exactly the printed ones:
    # q = e_0, k_j = scores[j] e_0, scale 1.  V = identity, so O row 0 = P row 0.
    d = n
    q = np.zeros((n, d)); q[0, 0] = 1.0
    k = np.zeros((n, d)); k[:, 0] = scores
    v = np.eye(n)
    trace = []
    o_blk, lse_blk = blockwise_attention(q, k, v, 1.0, False, br=1, bc=len(s1), trace=trace)
    # The pages: block max 3, then the max moves to 4 and the accumulator is
    # rescaled by e^(3-4) = e^(-1).
    row0 = [t for t in trace if t[0] == 0]
    assert len(row0) == 1
    _, m_old, m_new, alpha = row0[0]
    assert m_old == g["block1_max"][0]
    assert m_new == g["new_max"][0]
    assert alpha == pytest.approx(math.exp(g["rescale_exponent"][0]), rel=0, abs=1e-16)
    # ... and blockwise equals the one-shot global softmax (the oracle).
    O, LSE, P = orc.attn_fwd(q, k, v, 1.0, False, return_probs=True)
    np.testing.assert_allclose(O[0, 0], o_blk[0], rtol=1e-14, atol=1e-16)
    np.testing.assert_allclose(LSE[0, 0], lse_blk[0], rtol=1e-14)
    np.testing.assert_allclose(O[0, 0], P[0, 0], rtol=0, atol=1e-15)
    # Ratios of probabilities are e^(score difference); probabilities sum to 1.
    p = P[0, 0]
    for a in range(n):
        for b in range(n):
            assert p[a] / p[b] == pytest.approx(math.exp(scores[a] - scores[b]), rel=1e-13)
    assert p.sum() == pytest.approx(1.0, abs=1e-15)
    # LSE of the row is ln of the sum of exponentials (math.fsum of math.exp).
    assert LSE[0, 0] == pytest.approx(math.log(math.fsum(math.exp(x) for x in scores)), rel=1e-15)


# ---------------------------------------------------------------------------
# Invariants
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_rows_of_p_sum_to_one(causal):
    q, k, v = _rand((3, 37, 8), 1), _rand((3, 37, 8), 2), _rand((3, 37, 8), 3)
    _, _, P = orc.attn_fwd(q, k, v, 0.7, causal, return_probs=True)
    np.testing.assert_allclose(P.sum(axis=-1), 1.0, rtol=0, atol=1e-14)
    assert (P >= 0).all()
    if causal:
        iu = np.triu_indices(37, 1)
        assert (P[:, iu[0], iu[1]] == 0).all()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,d", [(1, 1), (2, 3), (5, 2), (7, 4), (9, 3)])
def test_blockwise_equals_one_shot_every_split(causal, n, d):
    q, k, v = _rand((n, d), 10 + n), _rand((n, d), 20 + n), _rand((n, d), 30 + n)
    O, LSE = orc.attn_fwd(q, k, v, 0.9, causal)
    for br in range(1, n + 1):
        for bc in range(1, n + 1):
            o_blk, lse_blk = blockwise_attention(q, k, v, 0.9, causal, br, bc)
            np.testing.assert_allclose(o_blk, O[0], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(lse_blk, LSE[0], rtol=1e-12, atol=1e-13)


def test_permutation_equivariance_noncausal():
    rng = np.random.default_rng(5)
    q, k, v = _rand((11, 6), 6), _rand((11, 6), 7), _rand((11, 6), 8)
    O, LSE = orc.attn_fwd(q, k, v, 0.5, False)
    pk = rng.permutation(11)
    O2, LSE2 = orc.attn_fwd(q, k[pk], v[pk], 0.5, False)
    np.testing.assert_allclose(O2, O, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(LSE2, LSE, rtol=1e-13)
    pq = rng.permutation(11)
    O3, LSE3 = orc.attn_fwd(q[pq], k, v, 0.5, False)
    np.testing.assert_allclose(O3[0], O[0][pq], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(LSE3[0], LSE[0][pq], rtol=1e-13)


# ---------------------------------------------------------------------------
# Closed forms
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_equal_scores_give_mean_of_visible_values(causal):
    n, d = 13, 5
    q = _rand((n, d), 40)
    k = np.tile(_rand((1, d), 41), (n, 1))     # every key identical
    v = _rand((n, d), 42)
    O, LSE = orc.attn_fwd(q, k, v, 0.3, causal)
    for i in range(n):
        vis = i + 1 if causal else n
        np.testing.assert_allclose(O[0, i], v[:vis].mean(axis=0), rtol=1e-13, atol=1e-14)
        s = 0.3 * float(q[i] @ k[0])
        assert LSE[0, i] == pytest.approx(s + math.log(vis), rel=1e-13, abs=1e-13)


def test_causal_first_row_is_first_value():
    q, k, v = _rand((9, 4), 50), _rand((9, 4), 51), _rand((9, 4), 52)
    O, LSE = orc.attn_fwd(q, k, v, 0.8, True)
    np.testing.assert_allclose(O[0, 0], v[0], rtol=0, atol=1e-15)
    assert LSE[0, 0] == pytest.approx(0.8 * float(q[0] @ k[0]), rel=1e-14)


def test_single_key_returns_value():
    q, k, v = _rand((1, 7), 53), _rand((1, 7), 54), _rand((1, 7), 55)
    for causal in (False, True):
        O, LSE = orc.attn_fwd(q, k, v, 1.3, causal)
        np.testing.assert_allclose(O[0], v, rtol=0, atol=1e-15)
        assert LSE[0, 0] == pytest.approx(1.3 * float(q[0] @ k[0]), rel=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_scale_is_uniform_average(causal):
    n = 10
    q, k, v = _rand((n, 3), 56), _rand((n, 3), 57), _rand((n, 3), 58)
    O, LSE = orc.attn_fwd(q, k, v, 0.0, causal)
    for i in range(n):
        vis = i + 1 if causal else n
        np.testing.assert_allclose(O[0, i], v[:vis].mean(axis=0), rtol=1e-13, atol=1e-14)
        assert LSE[0, i] == pytest.approx(math.log(vis), rel=1e-14)


def test_constant_values_give_constant_output():
    q, k = _rand((12, 4), 60), _rand((12, 4), 61)
    v = np.tile(np.array([[1.5, -2.0, 0.25, 3.0]]), (12, 1))
    for causal in (False, True):
        O, _ = orc.attn_fwd(q, k, v, 0.6, causal)
        np.testing.assert_allclose(O[0], v, rtol=1e-14, atol=1e-14)


def test_dominant_key_selects_its_value():
    n, d = 6, 3
    q = np.zeros((n, d)); q[:, 0] = 1.0
    k = np.zeros((n, d)); k[4, 0] = 60.0       # score 60 vs 0 elsewhere
    v = _rand((n, d), 62)
    O, LSE = orc.attn_fwd(q, k, v, 1.0, False)
    # weight of key 4 is 1/(1 + 5 e^-60); error < 5 e^-60 * max|v|
    np.testing.assert_allclose(O[0], np.tile(v[4], (n, 1)), rtol=0, atol=1e-24)
    np.testing.assert_allclose(LSE[0], 60.0 + math.log1p(5 * math.exp(-60.0)), rtol=1e-15)


def test_rows_variant_matches_full():
    q, k, v = _rand((40, 8), 63), _rand((40, 8), 64), _rand((40, 8), 65)
    rows = np.array([0, 3, 17, 39, 22])
    for causal in (False, True):
        O, LSE = orc.attn_fwd(q, k, v, 0.35, causal)
        o_r, l_r = orc.attn_fwd_rows(q, k, v, 0.35, causal, rows)
        np.testing.assert_allclose(o_r, O[0][rows], rtol=1e-14, atol=1e-15)
        np.testing.assert_allclose(l_r, LSE[0][rows], rtol=1e-14)


# ---------------------------------------------------------------------------
# Backward: finite differences and a library autograd
# ---------------------------------------------------------------------------

def _loss(q, k, v, g, scale, causal):
    O, _ = orc.attn_fwd(q, k, v, scale, causal)
    return float(np.sum(O[0] * g))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,d", [(1, 2), (2, 3), (3, 4), (5, 2), (8, 3)])
def test_backward_matches_central_differences(causal, n, d):
    scale = 0.45
    q, k, v, g = (_rand((n, d), 70 + i + 10 * n + 100 * d) for i in range(4))
    dQ, dK, dV = orc.attn_bwd(q, k, v, g, scale, causal)
    h = 1e-6
    for name, x, grad in (("q", q, dQ[0]), ("k", k, dK[0]), ("v", v, dV[0])):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}; args_p[name] = xp
            args_m = {"q": q, "k": k, "v": v}; args_m[name] = xm
            fp = _loss(args_p["q"], args_p["k"], args_p["v"], g, scale, causal)
            fm = _loss(args_m["q"], args_m["k"], args_m["v"], g, scale, causal)
            num[idx] = (fp - fm) / (2 * h)
        tol = 1e-7 * max(1.0, float(np.max(np.abs(num))))
        np.testing.assert_allclose(grad, num, rtol=0, atol=tol, err_msg=name)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_torch_autograd_fp64(causal):
    torch = pytest.importorskip("torch")
    bh, n, d, scale = 3, 33, 16, 0.25
    Q, K, V, G = (_rand((bh, n, d), 90 + i) for i in range(4))
    dQ, dK, dV = orc.attn_bwd(Q, K, V, G, scale, causal)
    O, LSE = orc.attn_fwd(Q, K, V, scale, causal)
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (Q, K, V))
    s = scale * tq @ tk.transpose(-1, -2)
    if causal:
        s = s.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), float("-inf"))
    o = torch.softmax(s, dim=-1) @ tv
    o.backward(torch.tensor(G))
    np.testing.assert_allclose(O, o.detach().numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(LSE, torch.logsumexp(s, dim=-1).detach().numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dQ, tq.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dK, tk.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dV, tv.grad.numpy(), rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------------------
# The pins catch plausible mistakes: plant each one in the oracle (on the CPU)
# and check that at least one pin then fails.
# ---------------------------------------------------------------------------

def _pins_hold(mod):
    """Run a compact subset of the pins above against ``mod``; True if all hold."""
    try:
        rng = np.random.default_rng(123)
        n, d = 6, 3
        q, k, v, g = (rng.standard_normal((n, d)) for _ in range(4))
        for causal in (False, True):
            O, LSE = mod.attn_fwd(q, k, v, 0.7, causal)
            for br, bc in ((1, 1), (2, 3), (4, 2)):
                ob, lb = blockwise_attention(q, k, v, 0.7, causal, br, bc)
                if not (np.allclose(ob, O[0], rtol=1e-10, atol=1e-12)
                        and np.allclose(lb, LSE[0], rtol=1e-10, atol=1e-12)):
                    return False
            dQ, dK, dV = mod.attn_bwd(q, k, v, g, 0.7, causal)
            h = 1e-6
            for name, x, grad in (("q", q, dQ[0]), ("k", k, dK[0]), ("v", v, dV[0])):
                for idx in [(0, 0), (n - 1, d - 1), (2, 1)]:
                    a = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
                    b = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
                    a[name][idx] += h
                    b[name][idx] -= h
                    fa = float(np.sum(mod.attn_fwd(a["q"], a["k"], a["v"], 0.7, causal)[0][0] * g))
                    fb = float(np.sum(mod.attn_fwd(b["q"], b["k"], b["v"], 0.7, causal)[0][0] * g))
                    if abs((fa - fb) / (2 * h) - grad[idx]) > 1e-6:
                        return False
        return True
    except Exception:
        return False


def test_pins_hold_for_the_oracle():
    assert _pins_hold(orc)


_MUTANTS = {
    "scores_transposed": lambda m: setattr(
        m, "head_scores", _wrap_scores(lambda s: s.T.copy())),
    "mask_off_by_one": lambda m: setattr(
        m, "head_scores", _shifted_mask_scores),
    "no_normalisation": lambda m: setattr(
        m, "row_softmax", lambda s: (np.exp(s - s.max(1, keepdims=True)), orc.row_softmax(s)[1])),
    "lse_without_max": lambda m: setattr(
        m, "row_softmax", lambda s: (orc.row_softmax(s)[0], np.log(np.sum(np.exp(s - s.max(1, keepdims=True)), 1)))),
    "scale_squared": lambda m: setattr(
        m, "head_scores", lambda q, k, scale, causal, rows=None: orc.head_scores(q, k, scale * scale, causal, rows)),
}


def _wrap_scores(f):
    def hs(q, k, scale, causal, rows=None):
        s = orc.head_scores(q, k, scale, False, rows)
        s = f(s)
        if causal:
            n = s.shape[1]
            r = np.arange(s.shape[0]) if rows is None else np.asarray(rows)
            s[np.arange(n)[None, :] > r[:, None]] = -np.inf
        return s
    return hs


def _shifted_mask_scores(q, k, scale, causal, rows=None):
    s = orc.head_scores(q, k, scale, False, rows)
    if causal:
        n = s.shape[1]
        r = np.arange(s.shape[0]) if rows is None else np.asarray(rows)
        s[np.arange(n)[None, :] >= r[:, None]] = -np.inf
        s[0, 0] = scale * float(np.asarray(q)[0] @ np.asarray(k)[0])
    return s


def _bwd_mutant(kind):
    def bwd(Q, K, V, dO, scale, causal):
        Q, K, V, dO = orc._as3(Q), orc._as3(K), orc._as3(V), orc._as3(dO)
        outs = [np.empty_like(Q) for _ in range(3)]
        for h in range(Q.shape[0]):
            p, _ = orc.row_softmax(orc.head_scores(Q[h], K[h], scale, causal))
            dp = dO[h] @ V[h].T
            D = np.sum(p * dp, axis=1, keepdims=True)
            if kind == "ds_sign":
                ds = p * (dp + D)
            elif kind == "ds_no_D":
                ds = p * dp
            else:
                ds = p * (dp - D)
            dv = p.T @ dO[h] if kind != "dv_untransposed" else p @ dO[h]
            dq = scale * (ds @ K[h]) if kind != "dq_no_scale" else ds @ K[h]
            dk = scale * (ds.T @ Q[h]) if kind != "dk_untransposed" else scale * (ds @ Q[h])
            outs[0][h], outs[1][h], outs[2][h] = dq, dk, dv
        return tuple(outs)
    return bwd


for _k in ("ds_sign", "ds_no_D", "dv_untransposed", "dq_no_scale", "dk_untransposed"):
    _MUTANTS["bwd_" + _k] = (lambda kind: (lambda m: setattr(m, "attn_bwd", _bwd_mutant(kind))))(_k)


@pytest.mark.parametrize("mutant", sorted(_MUTANTS))
def test_planted_mistakes_are_caught(mutant, monkeypatch):
    import importlib
    import types
    mod = types.ModuleType("oracle_mutant")
    src = importlib.import_module("oracle.attn_oracle")
    for name in dir(src):
        setattr(mod, name, getattr(src, name))
    # The mutant's functions look up helpers through ``mod``: rebind the
    # entry points so that they call the (possibly replaced) helpers.
    def attn_fwd(Q, K, V, scale, causal, return_probs=False):
        Q, K, V = orc._as3(Q), orc._as3(K), orc._as3(V)
        O = np.empty_like(Q); L = np.empty(Q.shape[:2])
        for h in range(Q.shape[0]):
            p, lse = mod.row_softmax(mod.head_scores(Q[h], K[h], scale, causal))
            O[h] = p @ V[h]; L[h] = lse
        return O, L
    mod.attn_fwd = attn_fwd
    _MUTANTS[mutant](mod)
    assert not _pins_hold(mod), f"planted mistake {mutant!r} was not caught by any pin"


# ---------------------------------------------------------------------------
# Shared key/value heads
# ---------------------------------------------------------------------------

def test_gqa_with_one_query_head_per_kv_head_is_mha():
    B, H, N, d = 2, 3, 9, 4
    q, k, v, g = (_rand((B * H, N, d), 300 + i) for i in range(4))
    O1, L1 = orc.attn_fwd_gqa(q, k, v, 0.4, True, B, H, H)
    O2, L2 = orc.attn_fwd(q, k, v, 0.4, True)
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(L1, L2)
    a = orc.attn_bwd_gqa(q, k, v, g, 0.4, True, B, H, H)
    b = orc.attn_bwd(q, k, v, g, 0.4, True)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_gqa_heads_read_their_shared_kv_head():
    # query head h of batch b must see exactly key/value head b*H_kv + h // G:
    # give every key/value head a constant, distinct value row and check O.
    B, H, H_kv, N, d = 2, 6, 2, 7, 3
    q, k = _rand((B * H, N, d), 310), _rand((B * H_kv, N, d), 311)
    v = np.zeros((B * H_kv, N, d))
    for j in range(B * H_kv):
        v[j] = float(j + 1)
    O, _ = orc.attn_fwd_gqa(q, k, v, 0.5, False, B, H, H_kv)
    for b in range(B):
        for h in range(H):
            np.testing.assert_allclose(O[b * H + h], b * H_kv + h // (H // H_kv) + 1.0, rtol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_backward_matches_central_differences(causal):
    B, H, H_kv, N, d, scale = 1, 4, 2, 5, 3, 0.45
    q, g = _rand((B * H, N, d), 320), _rand((B * H, N, d), 321)
    k, v = _rand((B * H_kv, N, d), 322), _rand((B * H_kv, N, d), 323)
    dQ, dK, dV = orc.attn_bwd_gqa(q, k, v, g, scale, causal, B, H, H_kv)
    assert dK.shape == k.shape and dV.shape == v.shape and dQ.shape == q.shape

    def loss(q_, k_, v_):
        O, _ = orc.attn_fwd_gqa(q_, k_, v_, scale, causal, B, H, H_kv)
        return float(np.sum(O * g))

    h = 1e-6
    for name, x, grad in (("q", q, dQ), ("k", k, dK), ("v", v, dV)):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}; args_p[name] = xp
            args_m = {"q": q, "k": k, "v": v}; args_m[name] = xm
            num[idx] = (loss(**{kk + "_": vv for kk, vv in args_p.items()})
                        - loss(**{kk + "_": vv for kk, vv in args_m.items()})) / (2 * h)
        np.testing.assert_allclose(grad, num, rtol=0, atol=1e-7 * max(1.0, np.abs(num).max()), err_msg=name)


def test_gqa_matches_torch_autograd_fp64():
    torch = pytest.importorskip("torch")
    B, H, H_kv, N, d, scale = 2, 4, 1, 11, 8, 0.3
    q, g = _rand((B * H, N, d), 330), _rand((B * H, N, d), 331)
    k, v = _rand((B * H_kv, N, d), 332), _rand((B * H_kv, N, d), 333)
    dQ, dK, dV = orc.attn_bwd_gqa(q, k, v, g, scale, True, B, H, H_kv)
    tq = torch.tensor(q.reshape(B, H, N, d), requires_grad=True)
    tk = torch.tensor(k.reshape(B, H_kv, N, d), requires_grad=True)
    tv = torch.tensor(v.reshape(B, H_kv, N, d), requires_grad=True)
    ke = tk.repeat_interleave(H // H_kv, dim=1)
    ve = tv.repeat_interleave(H // H_kv, dim=1)
    s = scale * tq @ ke.transpose(-1, -2)
    s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    o = torch.softmax(s, dim=-1) @ ve
    o.backward(torch.tensor(g.reshape(B, H, N, d)))
    np.testing.assert_allclose(dQ, tq.grad.numpy().reshape(B * H, N, d), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dK, tk.grad.numpy().reshape(B * H_kv, N, d), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dV, tv.grad.numpy().reshape(B * H_kv, N, d), rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------------------
# Block-sparse selection
# ---------------------------------------------------------------------------

def _bs_case(B, H, Hk, N, d, seed):
    return (_rand((B * H, N, d), seed), _rand((B * Hk, N, d), seed + 1), _rand((B * Hk, N, d), seed + 2),
            _rand((B * H, N, d), seed + 3))


@pytest.mark.parametrize("causal", [False, True])
def test_blocksparse_all_selected_is_dense(causal):
    B, H, N, d = 1, 2, 300, 4
    q, k, v, g = _bs_case(B, H, H, N, d, 400)
    nt = -(-N // orc.BLOCK)
    mask = np.ones((B * H, nt, nt), dtype=np.uint8)
    O1, L1 = orc.attn_fwd_blocksparse(q, k, v, 0.3, causal, mask, B, H, H)
    O2, L2 = orc.attn_fwd(q, k, v, 0.3, causal)
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(L1, L2)
    for x, y in zip(orc.attn_bwd_blocksparse(q, k, v, g, 0.3, causal, mask, B, H, H),
                    orc.attn_bwd(q, k, v, g, 0.3, causal)):
        np.testing.assert_allclose(x, y, rtol=1e-13, atol=1e-14)


def test_blocksparse_single_block_is_dense_attention_on_that_block():
    # each query tile selects exactly one key tile: its rows are dense attention
    # over that tile's 128 keys alone (the plain MHA oracle on sliced K, V)
    N, d, T = 384, 3, orc.BLOCK
    q, k, v, _ = _bs_case(1, 1, 1, N, d, 410)
    choice = [2, 0, 1]
    mask = np.zeros((1, 3, 3), dtype=np.uint8)
    for i, j in enumerate(choice):
        mask[0, i, j] = 1
    O, L = orc.attn_fwd_blocksparse(q, k, v, 0.5, False, mask, 1, 1, 1)
    for i, j in enumerate(choice):
        rows = slice(i * T, (i + 1) * T)
        keys = slice(j * T, (j + 1) * T)
        s = 0.5 * (q[0, rows] @ k[0, keys].T)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        np.testing.assert_allclose(O[0, rows], (e / e.sum(1, keepdims=True)) @ v[0, keys], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(L[0, rows], (m + np.log(e.sum(1, keepdims=True)))[:, 0], rtol=1e-13)


def test_blocksparse_empty_rows_give_zero_output_and_no_gradient():
    N, d = 256, 4
    q, k, v, g = _bs_case(1, 1, 1, N, d, 420)
    mask = np.zeros((1, 2, 2), dtype=np.uint8)
    mask[0, 1, 0] = 1                     # query tile 0 selects nothing
    O, L = orc.attn_fwd_blocksparse(q, k, v, 0.5, True, mask, 1, 1, 1)
    assert (O[0, :128] == 0).all() and np.isneginf(L[0, :128]).all()
    assert np.isfinite(O[0, 128:]).all() and np.isfinite(L[0, 128:]).all()
    dQ, dK, dV = orc.attn_bwd_blocksparse(q, k, v, g, 0.5, True, mask, 1, 1, 1)
    assert (dQ[0, :128] == 0).all()
    assert (dK[0, 128:] == 0).all() and (dV[0, 128:] == 0).all()   # key tile 1 is never selected


def test_blocksparse_backward_matches_central_differences():
    B, H, Hk, N, d, scale = 1, 2, 1, 260, 2, 0.7
    q, k, v, g = _bs_case(B, H, Hk, N, d, 430)
    rng = np.random.default_rng(431)
    mask = (rng.random((B * H, 3, 3)) < 0.6).astype(np.uint8)
    mask[0, 1, :] = 0                      # one empty query tile
    dQ, dK, dV = orc.attn_bwd_blocksparse(q, k, v, g, scale, True, mask, B, H, Hk)

    def loss(q_, k_, v_):
        O, _ = orc.attn_fwd_blocksparse(q_, k_, v_, scale, True, mask, B, H, Hk)
        return float(np.sum(O * g))

    h = 1e-6
    pick = [(0, 0, 0), (0, 129, 1), (0, 259, 0), (1, 200, 1), (1, 5, 0)]
    for name, x, grad in (("q", q, dQ), ("k", k, dK), ("v", v, dV)):
        for idx in pick:
            if idx[0] >= x.shape[0]:
                continue
            a = {"q_": q, "k_": k, "v_": v}
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            a[name + "_"] = xp
            fp = loss(**a)
            a[name + "_"] = xm
            fm = loss(**a)
            assert abs((fp - fm) / (2 * h) - grad[idx]) <= 1e-6 * max(1.0, abs(grad[idx])), (name, idx)


# ---------------------------------------------------------------------------
# Key/value cache (decode-shaped) forward
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_kvcache_with_as_many_queries_as_keys_is_plain_attention(causal):
    B, H, N, d = 1, 2, 37, 3
    q, k, v, _ = _bs_case(B, H, H, N, d, 500)
    O1, L1 = orc.attn_fwd_kvcache(q, k, v, 0.4, causal, B, H, H)
    O2, L2 = orc.attn_fwd(q, k, v, 0.4, causal)
    np.testing.assert_allclose(O1, O2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(L1, L2, rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("nq", [1, 3, 16])
def test_kvcache_queries_are_the_last_rows_of_the_sequence(nq):
    # the cache holds all L keys; the new queries are the last nq rows of a
    # length-L causal attention whose earlier query rows are arbitrary
    L, d = 29, 4
    q_full = _rand((1, L, d), 510)
    k, v = _rand((1, L, d), 511), _rand((1, L, d), 512)
    O_full, L_full = orc.attn_fwd(q_full, k, v, 0.6, True)
    O, LSE = orc.attn_fwd_kvcache(q_full[:, L - nq:], k, v, 0.6, True, 1, 1, 1)
    np.testing.assert_allclose(O, O_full[:, L - nq:], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(LSE, L_full[:, L - nq:], rtol=1e-13, atol=1e-14)


def test_kvcache_single_query_brute_force():
    # one query against five cached keys, every sum written out by hand
    q = [0.3, -1.2, 0.7]
    ks = [[1.0, 0.5, -0.2], [-0.4, 0.1, 0.9], [0.0, -1.0, 0.3], [0.8, 0.8, 0.8], [-0.5, 0.2, -0.1]]
    vs = [[1.0, 2.0, 3.0], [-1.0, 0.0, 1.0], [0.5, 0.5, 0.5], [2.0, -2.0, 0.0], [0.0, 1.0, -1.0]]
    scale = 0.9
    for causal in (False, True):
        e = [math.exp(scale * sum(a * b for a, b in zip(q, kj))) for kj in ks]
        tot = sum(e)
        o_ref = [sum(e[j] * vs[j][c] for j in range(5)) / tot for c in range(3)]
        O, LSE = orc.attn_fwd_kvcache(np.array([[q]]), np.array([ks]), np.array([vs]), scale, causal, 1, 1, 1)
        np.testing.assert_allclose(O[0, 0], o_ref, rtol=1e-14)
        assert abs(LSE[0, 0] - math.log(tot)) < 1e-14


def test_kvcache_lengths_truncate_the_cache():
    # entries past kv_lens[b] are never read, even when they hold NaN
    B, H, Hk, nq, nk, d = 3, 4, 2, 5, 40, 3
    q = _rand((B * H, nq, d), 520)
    k, v = _rand((B * Hk, nk, d), 521), _rand((B * Hk, nk, d), 522)
    lens = [40, 17, 6]
    kn, vn = k.copy(), v.copy()
    for b, L in enumerate(lens):
        kn[b * Hk:(b + 1) * Hk, L:] = np.nan
        vn[b * Hk:(b + 1) * Hk, L:] = np.nan
    for causal in (False, True):
        O, LSE = orc.attn_fwd_kvcache(q, kn, vn, 0.5, causal, B, H, Hk, kv_lens=lens)
        for b, L in enumerate(lens):
            qs = slice(b * H, (b + 1) * H)
            ks = slice(b * Hk, (b + 1) * Hk)
            Ob, Lb = orc.attn_fwd_kvcache(q[qs], k[ks, :L], v[ks, :L], 0.5, causal, 1, H, Hk)
            np.testing.assert_array_equal(O[qs], Ob)
            np.testing.assert_array_equal(LSE[qs], Lb)


def test_kvcache_group_heads_read_their_shared_head():
    B, H, Hk, nq, nk, d = 2, 6, 2, 3, 11, 4
    q = _rand((B * H, nq, d), 530)
    k, v = _rand((B * Hk, nk, d), 531), _rand((B * Hk, nk, d), 532)
    O, LSE = orc.attn_fwd_kvcache(q, k, v, 0.5, True, B, H, Hk)
    for b in range(B):
        for h in range(H):
            kv = b * Hk + h // (H // Hk)
            Oh, Lh = orc.attn_fwd_kvcache(q[b * H + h], k[kv], v[kv], 0.5, True, 1, 1, 1)
            np.testing.assert_array_equal(O[b * H + h], Oh[0])
            np.testing.assert_array_equal(LSE[b * H + h], Lh[0])


def test_kvcache_shorter_cache_than_queries_leaves_empty_rows():
    nq, d = 6, 3
    q = _rand((1, nq, d), 540)
    k, v = _rand((1, 10, d), 541), _rand((1, 10, d), 542)
    O, LSE = orc.attn_fwd_kvcache(q, k, v, 0.5, True, 1, 1, 1, kv_lens=[4])
    # rows p < nq - L see no key; row p >= nq - L sees keys 0 .. p - (nq - L)
    assert (O[0, :2] == 0).all() and np.isneginf(LSE[0, :2]).all()
    for p in range(2, nq):
        s = 0.5 * (q[0, p] @ k[0, :p - 1].T)
        e = np.exp(s - s.max())
        np.testing.assert_allclose(O[0, p], e @ v[0, :p - 1] / e.sum(), rtol=1e-13)
    O0, L0 = orc.attn_fwd_kvcache(q, k, v, 0.5, False, 1, 1, 1, kv_lens=[0])
    assert (O0 == 0).all() and np.isneginf(L0).all()


# ---------------------------------------------------------------------------
# FP8 (E4M3) inputs
# ---------------------------------------------------------------------------

def test_e4m3_decode_matches_torch_for_every_code():
    import torch
    codes = np.arange(256, dtype=np.uint8)
    ours = orc.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert (np.isnan(ours) == nan).all() and nan.sum() == 2          # 0x7F and 0xFF
    np.testing.assert_array_equal(ours[~nan], ref[~nan])


def test_e4m3_decode_landmarks():
    d = orc.e4m3_decode
    assert d([0x38])[0] == 1.0                  # exponent field 7 = bias, mantissa 0
    assert d([0x7E])[0] == 448.0                # largest finite
    assert d([0x01])[0] == 2.0 ** -9            # smallest subnormal
    assert d([0x08])[0] == 2.0 ** -6            # smallest normal
    assert d([0xB8])[0] == -1.0
    assert d([0x00])[0] == 0.0 and np.signbit(d([0x80])[0])


def test_fp8_forward_is_attention_on_dequantised_values():
    # codes chosen so the dequantised tensors are known exactly: code 0x38 + k
    # (k < 8) is 1 + k/8, and every descale is a power of two
    rng = np.random.default_rng(600)
    B, H, Hk, N, d = 1, 2, 1, 20, 4
    q8 = (0x38 + rng.integers(0, 8, (B * H, N, d))).astype(np.uint8)
    k8 = (0x30 + rng.integers(0, 8, (B * Hk, N, d))).astype(np.uint8)     # 0x30 + k = (1 + k/8) / 2
    v8 = (0xB8 + rng.integers(0, 8, (B * Hk, N, d))).astype(np.uint8)     # negative values
    Qd = 0.5 * (1 + (q8 - 0x38) / 8.0)
    Kd = 4.0 * 0.5 * (1 + (k8 - 0x30) / 8.0)
    Vd = 0.25 * -(1 + (v8 - 0xB8) / 8.0)
    for causal in (False, True):
        O, L = orc.attn_fwd_fp8(q8, k8, v8, 0.5, 4.0, 0.25, 0.3, causal, B, H, Hk)
        O2, L2 = orc.attn_fwd_gqa(Qd, Kd, Vd, 0.3, causal, B, H, Hk)
        np.testing.assert_allclose(O, O2, rtol=1e-14)
        np.testing.assert_allclose(L, L2, rtol=1e-14)


def test_kvcache_fp8_is_kvcache_on_the_dequantised_cache():
    # codes 0x38 + k (k < 8) decode to 1 + k/8; the descales are powers of two,
    # so the dequantised cache is known exactly without the decoder
    rng = np.random.default_rng(610)
    B, H, Hk, nq, nk, d = 2, 4, 2, 1, 9, 3
    q = _rand((B * H, nq, d), 611)
    k8 = (0x38 + rng.integers(0, 8, (B * Hk, nk, d))).astype(np.uint8)
    v8 = (0xB8 + rng.integers(0, 8, (B * Hk, nk, d))).astype(np.uint8)
    Kd = 0.25 * (1 + (k8 - 0x38) / 8.0)
    Vd = 2.0 * -(1 + (v8 - 0xB8) / 8.0)
    O, L = orc.attn_fwd_kvcache_fp8(q, k8, v8, 0.25, 2.0, 0.7, True, B, H, Hk, kv_lens=[9, 4])
    O2, L2 = orc.attn_fwd_kvcache(q, Kd, Vd, 0.7, True, B, H, Hk, kv_lens=[9, 4])
    np.testing.assert_allclose(O, O2, rtol=1e-14)
    np.testing.assert_allclose(L, L2, rtol=1e-14)


# ---------------------------------------------------------------------------
# Packed variable-length sequences
# ---------------------------------------------------------------------------

def _block_diagonal_reference(Q, K, V, cu, scale, causal, H, H_kv):
    """Brute force over all packed tokens at once: one (total x total) score
    matrix per head, every pair of tokens from different sequences masked
    (and later tokens of the same sequence too, if causal), then a plain
    softmax -- a formulation independent of the per-sequence split."""
    total = Q.shape[0]
    seq = np.zeros(total, dtype=np.int64)
    pos = np.zeros(total, dtype=np.int64)
    for s, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        seq[a:b] = s
        pos[a:b] = np.arange(b - a)
    O = np.zeros_like(Q, dtype=np.float64)
    LSE = np.zeros((H, total))
    for h in range(H):
        kh = h // (H // H_kv)
        S = scale * Q[:, h, :] @ K[:, kh, :].T
        allowed = seq[:, None] == seq[None, :]
        if causal:
            allowed &= pos[None, :] <= pos[:, None]
        S = np.where(allowed, S, -np.inf)
        m = S.max(axis=1, keepdims=True)
        e = np.exp(S - m)
        z = e.sum(axis=1, keepdims=True)
        O[:, h, :] = (e / z) @ V[:, kh, :]
        LSE[h] = (m + np.log(z))[:, 0]
    return O, LSE


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_matches_block_diagonal_brute_force(causal):
    rng = np.random.default_rng(31)
    lens = [3, 1, 0, 7, 5]
    cu = np.concatenate([[0], np.cumsum(lens)])
    total, H, Hk, d = int(cu[-1]), 4, 2, 6
    Q, K, V = (rng.standard_normal((total, h, d)) for h in (H, Hk, Hk))
    O, L = orc.attn_fwd_varlen(Q, K, V, cu, 0.4, causal, H, Hk)
    O_ref, L_ref = _block_diagonal_reference(Q, K, V, cu, 0.4, causal, H, Hk)
    np.testing.assert_allclose(O, O_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(L, L_ref, rtol=1e-12, atol=1e-12)


def test_varlen_sequences_are_independent():
    rng = np.random.default_rng(32)
    cu = np.array([0, 4, 9, 12])
    Q, K, V = (rng.standard_normal((12, 2, 5)) for _ in range(3))
    O, L = orc.attn_fwd_varlen(Q, K, V, cu, 0.3, True, 2, 2)
    K2, V2 = K.copy(), V.copy()
    K2[4:9] += 10.0                      # change only the middle sequence's keys and values
    V2[4:9] *= -3.0
    O2, L2 = orc.attn_fwd_varlen(Q, K2, V2, cu, 0.3, True, 2, 2)
    same = np.r_[0:4, 9:12]
    np.testing.assert_array_equal(O[same], O2[same])
    np.testing.assert_array_equal(L[:, same], L2[:, same])
    assert not np.allclose(O[4:9], O2[4:9])


def test_varlen_single_sequence_is_plain_attention():
    rng = np.random.default_rng(33)
    Q, K, V = (rng.standard_normal((11, 3, 4)) for _ in range(3))
    O, L = orc.attn_fwd_varlen(Q, K, V, [0, 11], 0.5, True, 3, 3)
    O_ref, L_ref = orc.attn_fwd(Q.transpose(1, 0, 2), K.transpose(1, 0, 2), V.transpose(1, 0, 2), 0.5, True)
    np.testing.assert_allclose(O, O_ref.transpose(1, 0, 2), rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(L, L_ref, rtol=1e-13, atol=1e-13)
