"""Pins for the oracle's integer metadata (positions, request index, time bucket)."""

import itertools
import math

import numpy as np
import pytest

import oracle


def _one_user(ts_hist, t_req, m):
    ts = list(ts_hist) + [t_req] * m
    return [0, len(ts)], [len(ts_hist)], ts


def test_shared_candidate_position_worked_example(golden):
    g = golden("position_example.txt")
    n, m = int(g["hist_len"][0]), int(g["num_candidates"][0])
    off, hl, ts = _one_user(range(1000, 1000 + n), 5000, m)
    pos, _, _ = oracle.token_metadata(off, hl, ts, n_ri=128)
    assert list(pos[n:]) == [int(x) for x in g["candidate_positions"]]
    assert pos[n - 1] == int(g["last_history_position"][0])
    assert list(pos[:n]) == list(range(1, n + 1))


def test_alibi_slopes_h8(golden):
    g = golden("alibi_slopes_h8.txt")
    s = oracle.alibi_slopes(int(g["H"][0]))
    assert np.array_equal(1.0 / s, np.array([float(x) for x in g["slope_inverse"]]))


def test_request_index_hand_example(golden):
    g = golden("request_index_example.txt")
    ts = [int(x) for x in g["ts"]]
    off, hl, t = _one_user(ts, int(g["t_req"][0]), 1)
    _, req, rtb = oracle.token_metadata(off, hl, t)
    assert list(req[:-1]) == [int(x) for x in g["req_idx"]]
    assert list(rtb[:-1]) == [int(x) for x in g["rt_bucket"]]
    assert req[-1] == int(g["candidate_req_idx"][0])
    assert rtb[-1] == int(g["candidate_rt_bucket"][0])
    # the gaps line is what the buckets are made of
    for gap, b in zip(g["gaps"], g["rt_bucket"]):
        if gap != "none":
            assert oracle.time_bucket(int(gap)) == int(b)


def test_time_bucket_against_float_log2():
    # exact at powers of two: x = 2^j gives floor(4 log2 x) = 4j
    for j in range(0, 16):
        assert oracle.time_bucket(2 ** j - 1) == 1 + min(62, 4 * j)
    # away from boundaries the float formula agrees
    for delta in range(0, 200000, 7):
        v = 4.0 * math.log2(delta + 1)
        if abs(v - round(v)) < 1e-9:
            continue
        assert oracle.time_bucket(delta) == 1 + min(62, int(math.floor(v)))
    assert oracle.time_bucket(0) == 1
    assert oracle.time_bucket(10 ** 12) == 63
    b = [oracle.time_bucket(x) for x in range(0, 5000)]
    assert all(x <= y for x, y in zip(b, b[1:]))
    with pytest.raises(ValueError):
        oracle.time_bucket(-1)


def _counting_formula(ts_hist, t_req, m, n_ri=128, n_rt=64):
    """An independently written counting form: request starts and group starts."""
    seq = list(ts_hist) + [t_req]
    req, rtb = [], []
    starts = 0
    group_start = 0
    for i, t in enumerate(seq):
        if i == 0 or t != seq[i - 1]:
            if i == 0 or t > seq[i - 1]:
                starts += 1
            group_start = i
        req.append(min(starts, n_ri - 1))
        if group_start == 0:
            rtb.append(0)
        else:
            rtb.append(oracle.time_bucket(t - seq[group_start - 1], n_rt))
    n = len(ts_hist)
    return req[:n] + [req[n]] * m, rtb[:n] + [rtb[n]] * m


def test_metadata_brute_force_small_sequences():
    count = 0
    for L in range(1, 6):
        for ts in itertools.combinations_with_replacement(range(4), L):
            for t_req in range(ts[-1], 5):
                off, hl, t = _one_user(ts, t_req, 2)
                pos, req, rtb = oracle.token_metadata(off, hl, t)
                r2, b2 = _counting_formula(ts, t_req, 2)
                assert list(req) == r2, (ts, t_req)
                assert list(rtb) == b2, (ts, t_req)
                assert list(pos) == list(range(1, L + 1)) + [L + 1, L + 1]
                count += 1
    assert count > 300


def test_request_index_clamp():
    ts = list(range(1000, 1300))  # 300 distinct requests
    off, hl, t = _one_user(ts, 2000, 1)
    _, req, _ = oracle.token_metadata(off, hl, t, n_ri=128)
    assert req.max() == 127
    assert list(req[:127]) == list(range(1, 128))


def test_sequence_length_is_n_plus_m(golden):
    from gen import CONFIGS, make_batch

    g = golden("sequence_length_example.txt")
    n = int(g["n_c"][0])
    assert 2 * n == int(g["interleaved_tokens"][0])
    assert n == int(g["action_oriented_tokens"][0])
    assert (n / (2 * n)) ** 2 == float(g["attention_cost_ratio"][0])
    b = make_batch(CONFIGS["c0"])
    assert b.T == int(sum(b.hist_len) + sum(b.cand_count))
    assert b.T < int(sum(2 * b.hist_len) + sum(b.cand_count))
