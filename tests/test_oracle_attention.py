"""Pins for the oracle's masked ALiBi attention (forward and backward)."""

import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import oracle.genrank_oracle as og


def _tiny(seed, users=((5, 3), (1, 2), (7, 1), (4, 0)), H=2, dh=4, mono=True):
    """Random jagged batch: (n, m) per user, monotone timestamps, shared candidate time."""
    rng = np.random.default_rng(seed)
    offs = [0]
    ts = []
    for n, m in users:
        t = 1_700_000_000 + int(rng.integers(0, 1000))
        for i in range(n):
            if i and rng.random() < 0.6:
                t += int(rng.integers(1, 400))
            ts.append(t)
        t_req = t + int(rng.integers(0, 300))
        ts.extend([t_req] * m)
        offs.append(offs[-1] + n + m)
    T = offs[-1]
    q, k, v = (rng.normal(size=(T, H, dh)) for _ in range(3))
    hl = [n for n, _ in users]
    pos, _, _ = oracle.token_metadata(offs, hl, ts)
    slopes = oracle.alibi_slopes(H) * 4.0  # stronger bias so it matters at tiny sizes
    return dict(q=q, k=k, v=v, offs=offs, hl=hl, ts=np.array(ts, np.int64), pos=pos,
                sp=slopes, st=slopes / 3600.0 * 50.0, scale=1.0 / math.sqrt(dh))


def _call(x, fn=oracle.attention_fwd, **kw):
    a = dict(x)
    a.update(kw)
    return fn(a["q"], a["k"], a["v"], a["offs"], a["hl"], a["pos"], a["ts"], a["sp"], a["st"],
              a["scale"])


def _brute(x):
    """Dense per-user attention from index comparisons written out element by element."""
    q, k, v = x["q"], x["k"], x["v"]
    T, H, dh = q.shape
    O = np.zeros_like(q)
    LSE = np.zeros((H, T))
    for u in range(len(x["hl"])):
        s, e, n = x["offs"][u], x["offs"][u + 1], x["hl"][u]
        L = e - s
        for h in range(H):
            S = np.full((L, L), -np.inf)
            for i in range(L):
                for j in range(L):
                    visible = (j <= i) if i < n else (j < n or j == i)
                    if visible:
                        # position of a token: its 1-based index, or n+1 for any candidate
                        pi = i + 1 if i < n else n + 1
                        pj = j + 1 if j < n else n + 1
                        ti, tj = int(x["ts"][s + i]), int(x["ts"][s + j])
                        S[i, j] = (float(np.dot(q[s + i, h], k[s + j, h])) / math.sqrt(dh)
                                   - x["sp"][h] * abs(pi - pj) - x["st"][h] * abs(ti - tj))
            P = scipy.special.softmax(S, axis=1)
            O[s:e, h] = P @ v[s:e, h]
            LSE[h, s:e] = scipy.special.logsumexp(S, axis=1)
    return O, LSE


def test_matches_brute_force():
    x = _tiny(1)
    O, LSE = _call(x)
    Ob, Lb = _brute(x)
    assert np.max(np.abs(O - Ob)) < 1e-12
    assert np.max(np.abs(LSE - Lb)) < 1e-12


def test_matches_torch_sdpa_with_explicit_bias():
    x = _tiny(2)
    O, _ = _call(x)
    for u in range(len(x["hl"])):
        s, e, n = x["offs"][u], x["offs"][u + 1], x["hl"][u]
        L = e - s
        ii, jj = np.meshgrid(np.arange(L), np.arange(L), indexing="ij")
        vis = np.where(ii < n, jj <= ii, (jj < n) | (jj == ii))
        p = x["pos"][s:e].astype(np.float64)
        t = x["ts"][s:e].astype(np.float64)
        for h in range(x["q"].shape[1]):
            bias = -x["sp"][h] * np.abs(p[:, None] - p[None]) - x["st"][h] * np.abs(t[:, None] - t[None])
            bias = np.where(vis, bias, -np.inf)
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.tensor(x["q"][s:e, h])[None], torch.tensor(x["k"][s:e, h])[None],
                torch.tensor(x["v"][s:e, h])[None], attn_mask=torch.tensor(bias)[None])[0].numpy()
            assert np.max(np.abs(ref - O[s:e, h])) < 1e-12


def test_zero_slopes_no_candidates_is_causal_sdpa():
    x = _tiny(3, users=((9, 0), (6, 0)))
    x["sp"] = np.zeros(2)
    x["st"] = np.zeros(2)
    O, _ = _call(x)
    for u in range(2):
        s, e = x["offs"][u], x["offs"][u + 1]
        for h in range(2):
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.tensor(x["q"][s:e, h])[None], torch.tensor(x["k"][s:e, h])[None],
                torch.tensor(x["v"][s:e, h])[None], is_causal=True)[0].numpy()
            assert np.max(np.abs(ref - O[s:e, h])) < 1e-12


def test_first_token_and_finite_lse():
    x = _tiny(4)
    O, LSE = _call(x)
    for u in range(len(x["hl"])):
        s, n = x["offs"][u], x["hl"][u]
        if n:
            assert np.array_equal(O[s], x["v"][s])  # one visible key: O_1 = v_1 exactly
    assert np.all(np.isfinite(LSE))


def test_lone_candidate_sees_only_itself():
    x = _tiny(5, users=((0, 3),))
    O, _ = _call(x)
    assert np.array_equal(O, x["v"])


def test_separable_bias_identity():
    """On visible pairs p_i >= p_j and t_i >= t_j, so the row part of the bias cancels."""
    x = _tiny(6)
    O, LSE = _call(x)
    for u in range(len(x["hl"])):
        s, e, n = x["offs"][u], x["offs"][u + 1], x["hl"][u]
        L = e - s
        mask = oracle.attention_mask(n, L)
        p = x["pos"][s:e].astype(np.float64)
        t = (x["ts"][s:e] - x["ts"][s]).astype(np.float64)
        ii, jj = np.nonzero(mask)
        assert np.all(p[ii] >= p[jj]) and np.all(t[ii] >= t[jj])
        for h in range(x["q"].shape[1]):
            col = x["sp"][h] * p + x["st"][h] * t
            S = x["q"][s:e, h] @ x["k"][s:e, h].T * x["scale"] + col[None, :]
            S = np.where(mask, S, -np.inf)
            P = scipy.special.softmax(S, axis=1)
            assert np.max(np.abs(P @ x["v"][s:e, h] - O[s:e, h])) < 1e-12
            lse_col = scipy.special.logsumexp(S, axis=1)
            assert np.max(np.abs(lse_col - col - LSE[h, s:e])) < 1e-9


def test_candidates_equal_appending_each_alone():
    x = _tiny(7, users=((6, 4),))
    O, _ = _call(x)
    n = 6
    for c in range(4):
        idx = list(range(n)) + [n + c]
        y = dict(x)
        for key in ("q", "k", "v"):
            y[key] = x[key][idx]
        y["ts"] = x["ts"][idx]
        y["offs"] = [0, n + 1]
        y["hl"] = [n]
        y["pos"] = x["pos"][idx]
        O1, _ = _call(y)
        assert np.max(np.abs(O1[n] - O[n + c])) <= 1e-12


def test_history_rows_ignore_later_tokens_bitwise():
    x = _tiny(8, users=((8, 3),))
    O, LSE = _call(x)
    kk = 5
    y = {key: (val.copy() if isinstance(val, np.ndarray) else val) for key, val in x.items()}
    rng = np.random.default_rng(0)
    for key in ("q", "k", "v"):
        y[key][kk:] = rng.normal(size=y[key][kk:].shape)
    y["ts"][kk:] += 17  # keeps timestamps monotone
    O2, LSE2 = _call(y)
    assert np.array_equal(O[:kk], O2[:kk])
    assert np.array_equal(LSE[:, :kk], LSE2[:, :kk])


def test_candidate_permutation_equivariance():
    x = _tiny(9, users=((5, 4),))
    O, _ = _call(x)
    perm = [5 + c for c in (2, 0, 3, 1)]
    idx = list(range(5)) + perm
    y = dict(x)
    for key in ("q", "k", "v"):
        y[key] = x[key][idx]
    O2, _ = _call(y)
    assert np.max(np.abs(O2 - O[idx])) < 1e-12


def test_backward_matches_finite_differences():
    x = _tiny(10, users=((4, 2), (3, 1)), H=2, dh=3)
    rng = np.random.default_rng(1)
    G = rng.normal(size=x["q"].shape)
    dq, dk, dv = oracle.attention_bwd(x["q"], x["k"], x["v"], G, x["offs"], x["hl"], x["pos"],
                                      x["ts"], x["sp"], x["st"], x["scale"])
    eps = 1e-6

    def loss(y):
        return float(np.sum(_call(y)[0] * G))

    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        for idx in [(0, 0, 0), (2, 1, 2), (5, 0, 1), (7, 1, 0), (9, 1, 1)]:
            yp = dict(x)
            ym = dict(x)
            yp[name] = x[name].copy()
            ym[name] = x[name].copy()
            yp[name][idx] += eps
            ym[name][idx] -= eps
            fd = (loss(yp) - loss(ym)) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-7 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


# ---- planted mistakes: each must make one of the pins above fail ---------------------------

def _planted(monkeypatch, name, fn):
    monkeypatch.setattr(og, name, fn)


def test_planted_mistake_dropped_candidate_self_is_caught(monkeypatch):
    def bad_mask(n, L):
        m = np.zeros((L, L), dtype=bool)
        for i in range(L):
            m[i, :min(i + 1, max(n, 1))] = True
        return m

    _planted(monkeypatch, "attention_mask", bad_mask)
    x = _tiny(11)
    O, _ = _call(x)
    Ob, _ = _brute(x)
    assert np.max(np.abs(O - Ob)) > 1e-6


def test_planted_mistake_time_bias_sign_is_caught(monkeypatch):
    orig = og._user_scores

    def bad(Q, K, p, t, sp, st, scale, n):
        return orig(Q, K, p, t, sp, -st, scale, n)

    _planted(monkeypatch, "_user_scores", bad)
    x = _tiny(12)
    O, _ = _call(x)
    Ob, _ = _brute(x)
    assert np.max(np.abs(O - Ob)) > 1e-6


def test_planted_mistake_transposed_bwd_is_caught():
    x = _tiny(13, users=((4, 2),), H=1, dh=3)
    G = np.random.default_rng(2).normal(size=x["q"].shape)
    dq, dk, dv = oracle.attention_bwd(x["q"], x["k"], x["v"], G, x["offs"], x["hl"], x["pos"],
                                      x["ts"], x["sp"], x["st"], x["scale"])
    # swapping the roles of dq and dk (a transposed dS) must disagree with finite differences
    eps = 1e-6
    yp, ym = dict(x), dict(x)
    yp["q"] = x["q"].copy()
    ym["q"] = x["q"].copy()
    yp["q"][1, 0, 1] += eps
    ym["q"][1, 0, 1] -= eps
    fd = (np.sum(_call(yp)[0] * G) - np.sum(_call(ym)[0] * G)) / (2 * eps)
    assert abs(fd - dq[1, 0, 1]) < 1e-7
    assert abs(fd - dk[1, 0, 1]) > 1e-4


@pytest.mark.parametrize("H", [1, 2, 4, 8, 16])
def test_slopes_are_geometric(H):
    s = oracle.alibi_slopes(H)
    assert s[0] == 2.0 ** (-8.0 / H)
    assert np.allclose(s[1:] / s[:-1], 2.0 ** (-8.0 / H), rtol=0, atol=1e-15)
    assert s[-1] == 2.0 ** -8
