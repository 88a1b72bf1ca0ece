"""The seeded input generator: determinism, subsets, structure, and table agreement."""

import numpy as np
import pytest
import torch

from gen import CONFIGS, bf16_round, item_rows, item_table_torch, make_batch, make_model


@pytest.mark.parametrize("name", ["c0", "c1", "c3", "c4_m64"])
def test_structure(name):
    cfg = CONFIGS[name]
    users = list(range(min(cfg.B, 40)))
    b = make_batch(cfg, users=users)
    assert b.seq_offsets[0] == 0 and np.all(np.diff(b.seq_offsets) > 0)
    for u in range(b.B):
        s, e, n = b.seq_offsets[u], b.seq_offsets[u + 1], b.hist_len[u]
        assert e - s == n + cfg.m
        ts = b.ts[s:e]
        assert np.all(np.diff(ts[:n]) >= 0)
        assert np.all(ts[n:] == ts[n]) and ts[n] > ts[n - 1]
        assert np.all(b.action_ids[s + n:e] == 8) and np.all(b.action_ids[s:s + n] < 8)
        kind = cfg.hist[0]
        lo, hi = {"uniform": cfg.hist[1:3], "fixed": (cfg.hist[1],) * 2,
                  "lognormal": cfg.hist[3:5]}[kind]
        assert lo <= n <= hi
    assert b.item_ids.min() >= 0 and b.item_ids.max() < cfg.n_item


def test_subsets_match_full_batch():
    cfg = CONFIGS["c1"].with_(B=12)
    full = make_batch(cfg)
    sub = make_batch(cfg, users=[3, 7])
    for k, u in enumerate([3, 7]):
        s, e = full.seq_offsets[u], full.seq_offsets[u + 1]
        s2, e2 = sub.seq_offsets[k], sub.seq_offsets[k + 1]
        assert np.array_equal(full.item_ids[s:e], sub.item_ids[s2:e2])
        assert np.array_equal(full.ts[s:e], sub.ts[s2:e2])


def test_deterministic():
    a, b = make_batch(CONFIGS["c0"]), make_batch(CONFIGS["c0"])
    assert np.array_equal(a.item_ids, b.item_ids) and np.array_equal(a.ts, b.ts)
    m1, m2 = make_model(CONFIGS["c0"]), make_model(CONFIGS["c0"])
    assert np.array_equal(m1.layers[0]["Wq"], m2.layers[0]["Wq"])


def test_bf16_round_matches_torch():
    x = np.random.default_rng(0).normal(size=100000).astype(np.float32) * 10
    ref = torch.tensor(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(bf16_round(x), ref)


def test_item_table_numpy_vs_torch():
    rows = np.array([0, 1, 77, 4095])
    for dt in ("f32", "bf16"):
        a = item_rows(99, rows, 64, dt)
        t = item_table_torch(99, 4096, 64, dt, "cpu", chunk_rows=1000)
        assert np.array_equal(t[rows].float().numpy(), a)
    x = item_rows(5, np.arange(2000), 64, "f32")
    assert abs(x.std() - 0.02) < 0.001 and abs(x.mean()) < 0.001
