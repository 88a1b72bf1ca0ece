"""Pins for the oracle's candidate scoring from cached history keys and values.

Scoring a request's candidates against a user's cached history must give exactly the
candidate rows of the full batched attention ("GenRank [2025]" chapter notes §1.3.2 on
the KV cache, with fun-rec §7.2.1; §1.4.1 and fun-rec §7.2.1 on what a candidate sees).
"""

import math

import numpy as np

import oracle


def _batch(seed, users=((5, 3), (0, 2), (9, 1), (4, 4)), H=2, dh=4):
    rng = np.random.default_rng(seed)
    offs, ts = [0], []
    for n, m in users:
        t = 1_700_000_000 + int(rng.integers(0, 1000))
        for i in range(n):
            if i and rng.random() < 0.6:
                t += int(rng.integers(1, 400))
            ts.append(t)
        ts.extend([t + int(rng.integers(0, 300))] * m)
        offs.append(offs[-1] + n + m)
    T = offs[-1]
    q, k, v = (rng.normal(size=(T, H, dh)) for _ in range(3))
    hl = [n for n, _ in users]
    pos, _, _ = oracle.token_metadata(offs, hl, ts)
    sp = oracle.alibi_slopes(H) * 4.0
    return dict(q=q, k=k, v=v, offs=offs, hl=hl, ts=np.array(ts, np.int64), pos=pos, sp=sp,
                st=sp / 3600.0 * 50.0, scale=1.0 / math.sqrt(dh))


def _split(x):
    """The batch as a history cache plus candidate arrays."""
    hist_idx, cand_idx, hoffs, coffs = [], [], [0], [0]
    for u, n in enumerate(x["hl"]):
        s, e = x["offs"][u], x["offs"][u + 1]
        hist_idx += list(range(s, s + n))
        cand_idx += list(range(s + n, e))
        hoffs.append(len(hist_idx))
        coffs.append(len(cand_idx))
    return np.array(hist_idx, int), np.array(cand_idx, int), hoffs, coffs


def test_cached_scoring_equals_the_candidate_rows_of_the_full_attention():
    x = _batch(21)
    O, LSE = oracle.attention_fwd(x["q"], x["k"], x["v"], x["offs"], x["hl"], x["pos"], x["ts"],
                                  x["sp"], x["st"], x["scale"])
    hi, ci, hoffs, coffs = _split(x)
    Oc, Lc = oracle.attention_fwd_cached(x["q"][ci], x["k"][ci], x["v"][ci], coffs, x["k"][hi],
                                         x["v"][hi], hoffs, x["pos"][hi], x["ts"][hi], x["ts"][ci],
                                         x["sp"], x["st"], x["scale"])
    assert np.max(np.abs(Oc - O[ci])) < 1e-12
    assert np.max(np.abs(Lc - LSE[:, ci])) < 1e-12


def test_empty_history_gives_each_candidate_its_own_value():
    rng = np.random.default_rng(22)
    q, k, v = (rng.normal(size=(3, 2, 4)) for _ in range(3))
    e = np.zeros((0, 2, 4))
    O, LSE = oracle.attention_fwd_cached(q, k, v, [0, 3], e, e, [0, 0], np.zeros(0, int),
                                         np.zeros(0, int), np.array([5, 5, 5]),
                                         np.array([0.5, 0.25]), np.array([0.1, 0.1]), 0.5)
    assert np.array_equal(O, v)
    for c in range(3):
        for h in range(2):
            assert abs(LSE[h, c] - 0.5 * float(q[c, h] @ k[c, h])) < 1e-15


def test_a_candidate_does_not_see_the_other_candidates():
    """Changing one candidate's key and value leaves every other candidate's row alone."""
    x = _batch(23, users=((6, 4),))
    hi, ci, hoffs, coffs = _split(x)
    args = lambda kc, vc: oracle.attention_fwd_cached(  # noqa: E731
        x["q"][ci], kc, vc, coffs, x["k"][hi], x["v"][hi], hoffs, x["pos"][hi], x["ts"][hi],
        x["ts"][ci], x["sp"], x["st"], x["scale"])
    O1, _ = args(x["k"][ci], x["v"][ci])
    k2, v2 = x["k"][ci].copy(), x["v"][ci].copy()
    k2[1] += 3.0
    v2[1] -= 2.0
    O2, _ = args(k2, v2)
    keep = [0, 2, 3]
    assert np.array_equal(O1[keep], O2[keep])
    assert np.max(np.abs(O1[1] - O2[1])) > 1e-3
