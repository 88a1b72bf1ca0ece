"""GPU parity of candidate scoring from cached history keys and values
(genrank_attn_fwd_cached) against the oracle.

The oracle's ``attention_fwd_cached`` scores each candidate against its user's cached
history and itself ("GenRank [2025]" chapter notes §1.3.2 on the KV cache, §1.4.1 on
what a candidate sees).  Tolerance: 2e-2 relative to the max for O (bf16), with a
per-row bound, and 2e-2 absolute for the natural-log LSE, as for the full forward.
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


def split_cache(batch, qkv):
    """The batch's history rows as a cache ([Th, 2, H, dh] keys and values, positions,
    times) and its candidate rows ([C, 3, H, dh] projections, times)."""
    hist_rows, cand_rows, hoff, coff = [], [], [0], [0]
    for u in range(batch.B):
        s, e, n = int(batch.seq_offsets[u]), int(batch.seq_offsets[u + 1]), int(batch.hist_len[u])
        hist_rows.extend(range(s, s + n))
        cand_rows.extend(range(s + n, e))
        hoff.append(hoff[-1] + n)
        coff.append(coff[-1] + e - s - n)
    hr, cr = np.array(hist_rows, np.int64), np.array(cand_rows, np.int64)
    pos_h = np.concatenate([np.arange(1, int(batch.hist_len[u]) + 1) for u in range(batch.B)])
    return dict(hist_rows=hr, cand_rows=cr, hoff=np.array(hoff, np.int32),
                coff=np.array(coff, np.int32), kv=qkv[hr][:, 1:3], q=qkv[cr],
                pos_h=pos_h.astype(np.int32), ts_h=batch.ts[hr], ts_c=batch.ts[cr])


def run_cached(G, cfg, c, poison=False):
    H, dh = cfg.H, cfg.dh
    d = H * dh
    C, Th = len(c["cand_rows"]), len(c["hist_rows"])
    q = _dev(c["q"].reshape(C, 3 * d), torch.bfloat16)
    kv = _dev(c["kv"].reshape(Th, 2 * d), torch.bfloat16) if Th else None
    o = torch.empty((C, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((H, C), dtype=torch.float32, device="cuda")
    m_max = int(np.max(np.diff(c["coff"]))) if len(c["coff"]) > 1 else 0
    ws = torch.empty(G.attn_cached_workspace_size(len(c["coff"]) - 1, C, Th, H, dh, m_max),
                     dtype=torch.uint8, device="cuda")
    if poison:
        ws.fill_(0xFF)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    sp, st = G.alibi_slopes(H)
    G.attn_fwd_cached(_dev(c["coff"]), m_max, q, q[:, d:], q[:, 2 * d:], 3 * d, _dev(c["hoff"]),
                      kv, kv[:, d:] if Th else None, 2 * d, _dev(c["pos_h"]) if Th else None,
                      _dev(c["ts_h"]) if Th else None, _dev(c["ts_c"]), H, dh, sp, st,
                      1.0 / math.sqrt(dh), o, d, lse, ws, err, C=C, Th=Th)
    code = G.check_error(err)
    return (o.float().cpu().numpy().astype(np.float64).reshape(C, H, dh),
            lse.cpu().numpy().astype(np.float64), code)


def _check(O, L, Or, Lr):
    assert ref.rel_to_max(O, Or) <= BF16_TOL
    den = np.maximum(np.abs(Or).max(axis=(1, 2)), 0.25)
    assert np.max(np.abs(O - Or).max(axis=(1, 2)) / den) <= BF16_TOL
    assert np.max(np.abs(L - Lr)) <= 2e-2


# (history length, candidates) per user: empty history, one candidate, ragged tails around
# 128, several candidate tiles, a user with no candidates
USERS = [(0, 1), (1, 1), (5, 3), (0, 7), (128, 128), (127, 129), (129, 0), (255, 1),
         (300, 200), (2, 130)]


@pytest.mark.parametrize("poison", [False, True])
def test_cached_parity_edge_users(G, poison):
    cfg = CONFIGS["c1"].with_(B=len(USERS), H=2)
    batch = make_batch(cfg, hist_override=[n for n, _ in USERS], m_override=[m for _, m in USERS])
    qkv = make_qkv(cfg, batch.T, seed=51)
    c = split_cache(batch, qkv)
    O, L, code = run_cached(G, cfg, c, poison=poison)
    assert code == 0
    sp, st = ref.slopes(cfg.H)
    Or, Lr = oracle.attention_fwd_cached(c["q"][:, 0], c["q"][:, 1], c["q"][:, 2], c["coff"],
                                         c["kv"][:, 0], c["kv"][:, 1], c["hoff"], c["pos_h"],
                                         c["ts_h"], c["ts_c"], sp, st, 1.0 / math.sqrt(cfg.dh))
    _check(O, L, Or, Lr)


def test_cached_equals_full_forward_candidate_rows(G):
    """The same candidates scored by the full attention over history + candidates."""
    from test_gpu_attention import run_fwd

    cfg = CONFIGS["c1"].with_(B=6)
    batch = make_batch(cfg, hist_override=[480, 33, 0, 200, 129, 1],
                       m_override=[128, 300, 5, 1, 64, 256])
    pos, _, _ = ref.meta(batch)
    qkv = make_qkv(cfg, batch.T, seed=52)
    c = split_cache(batch, qkv)
    O, L, code = run_cached(G, cfg, c)
    assert code == 0
    Of, Lf = run_fwd(G, cfg, batch, pos, qkv)
    assert ref.rel_to_max(O, Of[c["cand_rows"]]) <= 1e-2
    assert np.max(np.abs(L - Lf[:, c["cand_rows"]])) <= 1e-3


def test_cached_full_size_sweep_point_sampled(G):
    """The 1024-candidate sweep point (64 users, 480 cached history rows, 16 heads) in one
    launch; the oracle checks a seeded sample of users (its full attention, whose
    candidate rows the cached oracle equals to 1e-12)."""
    cfg = CONFIGS["c4_m1024"]
    batch = make_batch(cfg)
    qkv = make_qkv(cfg, batch.T, seed=53)
    c = split_cache(batch, qkv)
    O, L, code = run_cached(G, cfg, c)
    assert code == 0
    users = sorted(np.random.default_rng(5).choice(cfg.B, 3, replace=False).tolist())
    pos, _, _ = ref.meta(batch, users=users)
    Or, Lr = ref.attn(qkv[:, 0], qkv[:, 1], qkv[:, 2], batch, pos, users=users)
    rows = ref.cand_rows(batch, users)
    where = {r: k for k, r in enumerate(c["cand_rows"])}
    crow = np.array([where[r] for r in rows])
    _check(O[crow], L[:, crow], Or[rows], Lr[:, rows])


def test_cached_device_error_flags(G):
    cfg = CONFIGS["c1"].with_(B=3, H=2)
    batch = make_batch(cfg, hist_override=[40, 10, 70], m_override=[3, 4, 5])
    qkv = make_qkv(cfg, batch.T, seed=54)
    c = split_cache(batch, qkv)
    bad = dict(c)
    bad["ts_c"] = c["ts_c"].copy()
    bad["ts_c"][0] = c["ts_h"][39] - 1  # a candidate before its user's last history time
    assert run_cached(G, cfg, bad)[2] & G.DERR["TS_ORDER"]
    bad = dict(c)
    bad["pos_h"] = c["pos_h"].copy()
    bad["pos_h"][3] = 500  # beyond n + 1
    assert run_cached(G, cfg, bad)[2] & G.DERR["POS_RANGE"]
    bad = dict(c)
    bad["hoff"] = c["hoff"].copy()
    bad["hoff"][3] = bad["hoff"][3] + 9  # offsets past the cache
    assert run_cached(G, cfg, bad)[2] & G.DERR["LAYOUT"]


def run_candidates(G, cfg, batch, pos, qkv, poison=False):
    """genrank_attn_fwd_candidates on the jagged token array; o and lse start as NaN so
    that rows it must leave alone can be checked."""
    T, H, dh = batch.T, cfg.H, cfg.dh
    d = H * dh
    q = _dev(qkv.reshape(T, 3 * d), torch.bfloat16)
    o = torch.full((T, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((H, T), float("nan"), dtype=torch.float32, device="cuda")
    msl = int(np.max(np.diff(batch.seq_offsets)))
    ws = torch.empty(G.attn_candidates_workspace_size(batch.B, T, H, dh, msl), dtype=torch.uint8,
                     device="cuda")
    if poison:
        ws.fill_(0xFF)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    sp, st = G.alibi_slopes(H)
    G.attn_fwd_candidates(_dev(batch.seq_offsets), _dev(batch.hist_len), msl, q, q[:, d:],
                          q[:, 2 * d:], 3 * d, H, dh, _dev(pos.astype(np.int32)), _dev(batch.ts),
                          sp, st, 1.0 / math.sqrt(dh), o, d, lse, ws, err, T=T)
    code = G.check_error(err)
    return (o.float().cpu().numpy().astype(np.float64).reshape(T, H, dh),
            lse.cpu().numpy().astype(np.float64), code)


@pytest.mark.parametrize("poison", [False, True])
def test_candidates_only_forward_edge_users(G, poison):
    """Candidate rows of the full attention computed alone on the jagged layout (history
    keys and values read in place): against the oracle, and the history rows of o and
    lse left untouched; edge users as for the cached entry."""
    cfg = CONFIGS["c1"].with_(B=len(USERS), H=2)
    batch = make_batch(cfg, hist_override=[n for n, _ in USERS], m_override=[m for _, m in USERS])
    pos, _, _ = ref.meta(batch)
    qkv = make_qkv(cfg, batch.T, seed=54)
    O, L, code = run_candidates(G, cfg, batch, pos, qkv, poison=poison)
    assert code == 0
    rows = ref.cand_rows(batch)
    hist = np.setdiff1d(np.arange(batch.T), rows)
    assert np.all(np.isnan(O[hist])) and np.all(np.isnan(L[:, hist]))
    Or, Lr = ref.attn(qkv[:, 0], qkv[:, 1], qkv[:, 2], batch, pos)
    _check(O[rows], L[:, rows], Or[rows], Lr[:, rows])


def test_candidates_only_equals_full_forward(G):
    """At c2 shapes (16 users, 480 history + 256 candidates, 8 heads) the candidate rows
    agree with the full forward kernel's to within its bf16 rounding."""
    from test_gpu_attention import run_fwd

    cfg = CONFIGS["c2"]
    batch = make_batch(cfg, users=list(range(16)))
    pos, _, _ = ref.meta(batch)
    qkv = make_qkv(cfg, batch.T, seed=55)
    O, L, code = run_candidates(G, cfg, batch, pos, qkv)
    assert code == 0
    Of, Lf = run_fwd(G, cfg, batch, pos, qkv)
    rows = ref.cand_rows(batch)
    assert ref.rel_to_max(O[rows], Of[rows]) <= 1e-2
    assert np.max(np.abs(L[:, rows] - Lf[:, rows])) <= 1e-3
