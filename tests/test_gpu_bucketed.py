"""GPU parity of the bucketed time-bias attention (genrank_attn_fwd_bucketed and
genrank_attn_bwd_bucketed) against the oracle.

The bias is -m_p (p_i - p_j) - m_t bucket(t_i - t_j) (fun-rec "The Overall Generative
Ranking Paradigm" §7.2.2), bucket(D) = min(62, floor(4 log2(D + 1))), with the position
slopes as the per-bucket slopes.  Tolerances are those of the linear-bias tests: 2e-2
relative to the max (plus a per-row bound) for bf16 outputs and gradients, 2e-2
absolute for the LSE.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import ref
from gen import CONFIGS, make_batch, make_qkv

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2


@pytest.fixture(scope="module")
def G():
    from generative_ranking_recommendation_b200 import genrank
    from generative_ranking_recommendation_b200.csrc import build

    build.build()
    genrank.lib()
    return genrank


def _dev(x, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to("cuda", dtype=dtype) if dtype is not None else t.to("cuda")


def run(G, cfg, batch, pos, qkv, dO=None, bucketed=True, slope_scale=1.0):
    """Forward (and backward when dO is given) through the C ABI; float64 numpy results."""
    T, H, dh = batch.T, cfg.H, cfg.dh
    d = H * dh
    q = _dev(qkv.reshape(T, 3 * d), torch.bfloat16)
    o = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((H, T), dtype=torch.float32, device="cuda")
    off, hl = _dev(batch.seq_offsets), _dev(batch.hist_len)
    pos_t, ts_t = _dev(pos.astype(np.int32)), _dev(batch.ts)
    msl = int(np.max(np.diff(batch.seq_offsets)))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    sp, st = G.alibi_slopes(H)
    sp = [x * slope_scale for x in sp]
    tb = sp if bucketed else [x * slope_scale for x in st]
    wsf = torch.full((G.attn_workspace_size(batch.B, T, H, dh, msl, False),), 0xFF,
                     dtype=torch.uint8, device="cuda")
    G.attn_fwd(off, hl, msl, q, q[:, d:], q[:, 2 * d:], 3 * d, H, dh, pos_t, ts_t, sp, tb,
               1.0 / math.sqrt(dh), o, d, lse, wsf, err, T=T, bucketed=bucketed)
    out = [o.float().cpu().numpy().astype(np.float64).reshape(T, H, dh),
           lse.cpu().numpy().astype(np.float64)]
    if dO is not None:
        g = _dev(dO.reshape(T, d), torch.bfloat16)
        dq = torch.empty_like(q)
        wsb = torch.full((G.attn_workspace_size(batch.B, T, H, dh, msl, True),), 0xFF,
                         dtype=torch.uint8, device="cuda")
        G.attn_bwd(off, hl, msl, q, q[:, d:], q[:, 2 * d:], 3 * d, H, dh, pos_t, ts_t, sp, tb,
                   1.0 / math.sqrt(dh), o, g, d, lse, dq, dq[:, d:], dq[:, 2 * d:], wsb, err, T=T,
                   bucketed=bucketed)
        gr = dq.float().cpu().numpy().astype(np.float64).reshape(T, 3, H, dh)
        out += [gr[:, 0], gr[:, 1], gr[:, 2]]
    assert G.check_error(err) == 0
    return out


def _rel_rows(a, b, name, noise=None):
    """Relative to the max plus the per-token bound, with the gradients' noise floors
    (see ref.grad_noise_floors)."""
    ref.check_rows(a, b, BF16_TOL, name, noise=noise)


def _noise(batch, pos, qkv, dO, O, H, dh, users=None, slope_scale=1.0):
    sp = oracle.alibi_slopes(H) * slope_scale
    scale = 1.0 / math.sqrt(dh)

    def fwd(q, k, v, offs, hl, p, ts):
        return oracle.attention_fwd_bucketed(q, k, v, offs, hl, p, ts, sp, sp, scale)

    us = range(batch.B) if users is None else users
    return ref.grad_noise_floors(fwd, qkv[:, 0], qkv[:, 1], qkv[:, 2], dO, O, batch, pos, us,
                                 scale)


def _boundary_batch(cfg):
    """Users whose gaps sit on the bucket grid's edges: 46339 s (bucket 61) and 46340 s
    (bucket 62, the cap), gaps far beyond the cap, and several items per request."""
    batch = make_batch(cfg, hist_override=[6, 140, 9, 130, 1],
                       m_override=[3, 130, 1, 2, 4])
    t0 = 1_700_000_000
    gaps = {0: [0, 46339, 46340, 0, 5, 1_000_000], 2: [0, 1, 2, 3, 15, 16, 255, 256, 46340]}
    for u, g in gaps.items():
        s, n = int(batch.seq_offsets[u]), int(batch.hist_len[u])
        ts = t0 + np.cumsum(np.array(g[:n], np.int64))
        batch.ts[s:s + n] = ts
        batch.ts[s + n:int(batch.seq_offsets[u + 1])] = ts[-1] + 46339
    return batch


def _oracle(batch, pos, qkv, H, dh, dO=None, slope_scale=1.0):
    sp = oracle.alibi_slopes(H) * slope_scale
    args = (batch.seq_offsets, batch.hist_len, pos, batch.ts, sp, sp, 1.0 / math.sqrt(dh))
    O, L = oracle.attention_fwd_bucketed(qkv[:, 0], qkv[:, 1], qkv[:, 2], *args)
    if dO is None:
        return O, L
    return (O, L) + tuple(oracle.attention_bwd_bucketed(qkv[:, 0], qkv[:, 1], qkv[:, 2], dO,
                                                        *args))


@pytest.mark.parametrize("slope_scale", [1.0, 8.0])
def test_bucketed_fwd_bwd_parity(G, slope_scale):
    cfg = CONFIGS["c3"].with_(B=5, H=2)
    batch = _boundary_batch(cfg)
    pos, _, _ = ref.meta(batch)
    qkv = make_qkv(cfg, batch.T, seed=61)
    dO = make_qkv(cfg, batch.T, seed=62, n=1)[:, 0]
    got = run(G, cfg, batch, pos, qkv, dO, slope_scale=slope_scale)
    want = _oracle(batch, pos, qkv, cfg.H, cfg.dh, dO, slope_scale=slope_scale)
    _rel_rows(got[0], want[0], "O")
    assert np.max(np.abs(got[1] - want[1])) <= 2e-2
    noise = _noise(batch, pos, qkv, dO, want[0], cfg.H, cfg.dh, slope_scale=slope_scale)
    for k, name in zip(range(2, 5), ("dq", "dk", "dv")):
        _rel_rows(got[k], want[k], name, noise[k - 2])


def test_bucketed_parity_random_users(G):
    cfg = CONFIGS["c1"].with_(B=6, H=4)
    batch = make_batch(cfg, hist_override=[200, 1, 0, 129, 60, 255],
                       m_override=[20, 1, 3, 128, 0, 2])
    pos, _, _ = ref.meta(batch)
    qkv = make_qkv(cfg, batch.T, seed=63)
    dO = make_qkv(cfg, batch.T, seed=64, n=1)[:, 0]
    got = run(G, cfg, batch, pos, qkv, dO)
    want = _oracle(batch, pos, qkv, cfg.H, cfg.dh, dO)
    _rel_rows(got[0], want[0], "O")
    assert np.max(np.abs(got[1] - want[1])) <= 2e-2
    noise = _noise(batch, pos, qkv, dO, want[0], cfg.H, cfg.dh, slope_scale=1.0)
    for k, name in zip(range(2, 5), ("dq", "dk", "dv")):
        _rel_rows(got[k], want[k], name, noise[k - 2])


def test_one_request_per_user_equals_linear_bias_bitwise(G):
    """With every token of a user at one time the time term vanishes for both biases
    (bucket(0) = 0, |0| = 0), and the two kernels must agree bit for bit."""
    cfg = CONFIGS["c1"].with_(B=4)
    batch = make_batch(cfg, hist_override=[300, 17, 128, 0], m_override=[40, 129, 1, 5])
    for u in range(batch.B):
        s, e = int(batch.seq_offsets[u]), int(batch.seq_offsets[u + 1])
        batch.ts[s:e] = batch.ts[s]
    pos, _, _ = ref.meta(batch)
    qkv = make_qkv(cfg, batch.T, seed=65)
    dO = make_qkv(cfg, batch.T, seed=66, n=1)[:, 0]
    a = run(G, cfg, batch, pos, qkv, dO, bucketed=True)
    b = run(G, cfg, batch, pos, qkv, dO, bucketed=False)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_bucketed_full_size_c3_sampled(G):
    """The training workload's shapes in one launch of each kernel; the oracle checks a
    seeded sample of short users (its bucketed attention is an explicit double loop)."""
    cfg = CONFIGS["c3"]
    batch = make_batch(cfg)
    pos = np.zeros(batch.T, np.int64)
    for u in range(batch.B):
        s, e, n = batch.seq_offsets[u], batch.seq_offsets[u + 1], batch.hist_len[u]
        pos[s:s + n] = np.arange(1, n + 1)
        pos[s + n:e] = n + 1
    qkv = make_qkv(cfg, batch.T, seed=67)
    dO = make_qkv(cfg, batch.T, seed=68, n=1)[:, 0]
    got = run(G, cfg, batch, pos, qkv, dO)
    lens = np.diff(batch.seq_offsets)
    short = np.nonzero(lens <= 160)[0]
    users = sorted(np.random.default_rng(7).choice(short, 3, replace=False).tolist())
    sp = oracle.alibi_slopes(cfg.H)
    args = (batch.seq_offsets, batch.hist_len, pos, batch.ts, sp, sp, 1.0 / math.sqrt(cfg.dh))
    O, L = oracle.attention_fwd_bucketed(qkv[:, 0], qkv[:, 1], qkv[:, 2], *args, users=users)
    dq, dk, dv = oracle.attention_bwd_bucketed(qkv[:, 0], qkv[:, 1], qkv[:, 2], dO, *args,
                                               users=users)
    rows = ref.user_rows(batch, users)
    _rel_rows(got[0][rows], O[rows], "O")
    assert np.max(np.abs(got[1][:, rows] - L[:, rows])) <= 2e-2
    noise = _noise(batch, pos, qkv, dO, O, cfg.H, cfg.dh, users=users)
    for k, (name, w) in enumerate((("dq", dq), ("dk", dk), ("dv", dv))):
        _rel_rows(got[2 + k][rows], w[rows], name, noise[k][rows])
