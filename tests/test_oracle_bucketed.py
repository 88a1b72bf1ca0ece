"""Pins for the oracle's bucketed time-bias variant of the masked ALiBi attention.

The variant is the fun-rec "The Overall Generative Ranking Paradigm" §7.2.2 bias
-m_p (p_i - p_j) - m_t bucket(t_i - t_j), with the reading of bucket() and m_t stated
in the oracle: floor(4 log2(delta + 1)) saturating at 62, and m_t = m_h.
"""

import math

import numpy as np
import scipy.special

import oracle

CAP = 62  # the largest gap row of a 64-row pre-request time table


def test_pair_bucket_at_powers_of_two():
    # delta + 1 = 2^k: 4 log2(2^k) = 4k exactly
    for k in range(0, 20):
        assert oracle.pair_time_bucket(2 ** k - 1) == min(CAP, 4 * k)


def test_pair_bucket_same_request_and_saturation():
    assert oracle.pair_time_bucket(0) == 0
    # 4 log2(x) reaches 62 at x = 2^15.5 = 46340.95...: 46340 is below, 46341 above
    assert 4 * math.log2(46340) < 62 < 4 * math.log2(46341)
    assert oracle.pair_time_bucket(46339) == 61
    assert oracle.pair_time_bucket(46340) == 62
    assert oracle.pair_time_bucket(10 ** 9) == CAP


def test_pair_bucket_matches_float_log2_away_from_boundaries():
    rng = np.random.default_rng(3)
    checked = 0
    for d in rng.integers(0, 200_000, size=4000):
        f = 4.0 * math.log2(float(d) + 1.0)
        if abs(f - round(f)) < 1e-6:
            continue
        assert oracle.pair_time_bucket(int(d)) == min(CAP, math.floor(f))
        checked += 1
    assert checked > 3900


def test_pair_bucket_is_monotone():
    """Non-decreasing; from x = delta + 1 = 6 on, 4 log2(x + 1) - 4 log2(x) =
    4 log2(1 + 1/x) <= 1, so the bucket grows by at most one per second."""
    assert [oracle.pair_time_bucket(d) for d in range(6)] == [0, 4, 6, 8, 9, 10]
    prev = oracle.pair_time_bucket(5)
    for d in range(6, 5000):
        b = oracle.pair_time_bucket(d)
        assert prev <= b <= prev + 1
        prev = b


def _tiny(seed, users=((5, 3), (1, 2), (7, 1), (4, 0)), H=2, dh=4):
    """Random jagged batch with monotone timestamps (gaps of seconds to hours)."""
    rng = np.random.default_rng(seed)
    offs, ts = [0], []
    for n, m in users:
        t = 1_700_000_000 + int(rng.integers(0, 1000))
        for i in range(n):
            if i and rng.random() < 0.6:
                t += int(rng.integers(1, 20_000))
            ts.append(t)
        ts.extend([t + int(rng.integers(0, 3000))] * m)
        offs.append(offs[-1] + n + m)
    T = offs[-1]
    q, k, v = (rng.normal(size=(T, H, dh)) for _ in range(3))
    hl = [n for n, _ in users]
    pos, _, _ = oracle.token_metadata(offs, hl, ts)
    slopes = oracle.alibi_slopes(H)
    return dict(q=q, k=k, v=v, offs=offs, hl=hl, ts=np.array(ts, np.int64), pos=pos, sp=slopes,
                stb=slopes, scale=1.0 / math.sqrt(dh))


def _call(x):
    return oracle.attention_fwd_bucketed(x["q"], x["k"], x["v"], x["offs"], x["hl"], x["pos"],
                                         x["ts"], x["sp"], x["stb"], x["scale"])


def test_matches_brute_force_with_float_buckets():
    """Element by element, with the bucket taken from a float log2 (the sample's gaps keep
    4 log2(delta + 1) away from integers) and positions from token indices."""
    x = _tiny(11)
    O, LSE = _call(x)
    q, k, v = x["q"], x["k"], x["v"]
    T, H, dh = q.shape
    for u in range(len(x["hl"])):
        s, e, n = x["offs"][u], x["offs"][u + 1], x["hl"][u]
        L = e - s
        for h in range(H):
            S = np.full((L, L), -np.inf)
            for i in range(L):
                for j in range(L):
                    if (j <= i) if i < n else (j < n or j == i):
                        pi = i + 1 if i < n else n + 1
                        pj = j + 1 if j < n else n + 1
                        dt = int(x["ts"][s + i]) - int(x["ts"][s + j])
                        f = 4.0 * math.log2(dt + 1.0)  # exact when dt + 1 is a power of 2
                        assert abs(f - round(f)) > 1e-9 or (dt + 1) & dt == 0
                        b = min(CAP, math.floor(f))
                        S[i, j] = (float(np.dot(q[s + i, h], k[s + j, h])) * x["scale"]
                                   - x["sp"][h] * (pi - pj) - x["stb"][h] * b)
            P = scipy.special.softmax(S, axis=1)
            assert np.max(np.abs(P @ v[s:e, h] - O[s:e, h])) < 1e-12
            assert np.max(np.abs(scipy.special.logsumexp(S, axis=1) - LSE[h, s:e])) < 1e-12


def test_one_request_reduces_to_the_linear_oracle_without_time_bias():
    """Every timestamp of a user equal: every bucket is 0, so the variant is the linear
    oracle with zero time slopes."""
    x = _tiny(12)
    for u in range(len(x["hl"])):
        s, e = x["offs"][u], x["offs"][u + 1]
        x["ts"][s:e] = x["ts"][s]
    O, LSE = _call(x)
    Or, Lr = oracle.attention_fwd(x["q"], x["k"], x["v"], x["offs"], x["hl"], x["pos"], x["ts"],
                                  x["sp"], np.zeros_like(x["sp"]), x["scale"])
    assert np.max(np.abs(O - Or)) < 1e-12
    assert np.max(np.abs(LSE - Lr)) < 1e-12


def test_worked_example_by_hand():
    """Three history tokens at t = 0, 0, 15 s, positions 1, 2, 3, one head, slope 1/2, zero
    q and k (so only the bias acts) and v = the identity rows.  Row 3 sees keys 1..3 with
    buckets floor(4 log2 16) = 16, 16, 0 and position gaps 2, 1, 0: scores -9, -8.5, 0."""
    q = np.zeros((3, 1, 3))
    k = np.zeros((3, 1, 3))
    v = np.eye(3).reshape(3, 1, 3)
    O, LSE = oracle.attention_fwd_bucketed(q, k, v, [0, 3], [3], np.array([1, 2, 3]),
                                           np.array([0, 0, 15]), np.array([0.5]),
                                           np.array([0.5]), 1.0)
    z = 1.0 + math.exp(-8.5) + math.exp(-9.0)
    assert np.allclose(O[2, 0], [math.exp(-9.0) / z, math.exp(-8.5) / z, 1.0 / z], atol=1e-15)
    assert abs(LSE[0, 2] - math.log(z)) < 1e-14
    # row 2 sees keys 1, 2 in one request: buckets 0, 0 and position gaps 1, 0
    z2 = 1.0 + math.exp(-0.5)
    assert np.allclose(O[1, 0], [math.exp(-0.5) / z2, 1.0 / z2, 0.0], atol=1e-15)


def test_candidates_equal_appending_each_alone():
    x = _tiny(13, users=((6, 4),))
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


def test_planted_mistake_bucket_offset_is_caught(monkeypatch):
    """A bucket that starts at 1 (the embedding's row numbering) instead of 0 shifts every
    pair but a same-request one: the worked example must catch it."""
    real = oracle.genrank_oracle.pair_time_bucket
    monkeypatch.setattr(oracle.genrank_oracle, "pair_time_bucket",
                        lambda d, n_rt=64: real(d, n_rt) + (1 if d > 0 else 0))
    try:
        test_worked_example_by_hand()
    except AssertionError:
        return
    raise AssertionError("the planted mistake was not caught")


def test_backward_matches_finite_differences():
    x = _tiny(14, users=((4, 2), (3, 1)), H=2, dh=3)
    rng = np.random.default_rng(2)
    G = rng.normal(size=x["q"].shape)
    dq, dk, dv = oracle.attention_bwd_bucketed(x["q"], x["k"], x["v"], G, x["offs"], x["hl"],
                                               x["pos"], x["ts"], x["sp"], x["stb"], x["scale"])
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

