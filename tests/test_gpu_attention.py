"""GPU parity of the masked ALiBi attention (forward and backward) against the oracle.

Tolerances: max-abs 1e-4 for fp32 workloads, 2e-2 relative-to-max for bf16
workloads.  The bf16 forward runs the tcgen05 kernel (head dim 64); fp32 and
head dim 32 run the CUDA-core kernel.
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
F32_TOL = 1e-4


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


def run_fwd(G, cfg, batch, pos, qkv, need_lse=True, poison=False):
    """qkv: [T, 3, H, dh] host array; returns (O [T,H,dh], LSE [H,T]) as float64 numpy.

    poison: fill the workspace with 0xff bytes (NaN as fp32) before the call."""
    T, H, dh = batch.T, cfg.H, cfg.dh
    d = H * dh
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    q = _dev(qkv.reshape(T, 3 * d), tdt)
    o = torch.empty((T, d), dtype=tdt, device="cuda")
    lse = torch.empty((H, T), dtype=torch.float32, device="cuda") if need_lse else None
    off, hl = _dev(batch.seq_offsets), _dev(batch.hist_len)
    pos_t, ts_t = _dev(pos.astype(np.int32)), _dev(batch.ts)
    msl = int(np.max(np.diff(batch.seq_offsets)))
    ws = torch.empty(G.attn_workspace_size(batch.B, T, H, dh, msl, False), dtype=torch.uint8,
                     device="cuda")
    if poison:
        ws.fill_(0xFF)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    sp, st = G.alibi_slopes(H)
    G.attn_fwd(off, hl, msl, q, q[:, d:], q[:, 2 * d:], 3 * d, H, dh, pos_t, ts_t, sp, st,
               1.0 / math.sqrt(dh), o, d, lse, ws, err, T=T)
    assert G.check_error(err) == 0
    O = o.float().cpu().numpy().astype(np.float64).reshape(T, H, dh)
    L = lse.cpu().numpy().astype(np.float64) if need_lse else None
    return O, L


def _check(cfg, O, L, Or, Lr, rows):
    if cfg.dtype == "f32":
        assert np.max(np.abs(O[rows] - Or[rows])) <= F32_TOL
        assert np.max(np.abs(L[:, rows] - Lr[:, rows])) <= F32_TOL
    else:
        assert ref.rel_to_max(O[rows], Or[rows]) <= BF16_TOL
        # per-row bound as well, so that one wrong row cannot hide behind the max
        den = np.maximum(np.abs(Or[rows]).max(axis=(1, 2)), 0.25)
        assert np.max(np.abs(O[rows] - Or[rows]).max(axis=(1, 2)) / den) <= BF16_TOL
        assert np.max(np.abs(L[:, rows] - Lr[:, rows])) <= 2e-2


@pytest.mark.parametrize("name,B", [("c0", None), ("c1", 24), ("c4_m1024", 4)])
def test_fwd_parity(G, name, B):
    cfg = CONFIGS[name] if B is None else CONFIGS[name].with_(B=B)
    batch = make_batch(cfg)
    pos, _, _ = ref.meta(batch)
    qkv = make_qkv(cfg, batch.T, seed=cfg.seed + 1)
    O, L = run_fwd(G, cfg, batch, pos, qkv)
    Or, Lr = ref.attn(qkv[:, 0], qkv[:, 1], qkv[:, 2], batch, pos)
    _check(cfg, O, L, Or, Lr, np.arange(batch.T))


EDGE_USERS = [(1, 0), (1, 1), (0, 5), (128, 0), (127, 3), (129, 2), (255, 1), (256, 128),
              (257, 7), (480, 1024), (2, 300), (383, 64)]


@pytest.mark.parametrize("dtype,H,dh", [("bf16", 4, 64), ("f32", 2, 32), ("bf16", 2, 32)])
def test_fwd_edge_cases(G, dtype, H, dh):
    cfg = CONFIGS["c1"].with_(B=len(EDGE_USERS), H=H, dh=dh, dtype=dtype)
    batch = make_batch(cfg, hist_override=[n for n, _ in EDGE_USERS],
                       m_override=[m for _, m in EDGE_USERS])
    # one user with every timestamp equal (a single request)
    u = 7
    s, e = batch.seq_offsets[u], batch.seq_offsets[u + 1]
    batch.ts[s:e] = batch.ts[s]
    pos, _, _ = ref.meta(batch)
    qkv = make_qkv(cfg, batch.T, seed=5)
    O, L = run_fwd(G, cfg, batch, pos, qkv)
    Or, Lr = ref.attn(qkv[:, 0], qkv[:, 1], qkv[:, 2], batch, pos)
    _check(cfg, O, L, Or, Lr, np.arange(batch.T))


def test_fwd_workspace_contents_do_not_matter(G):
    """The ragged edge cases with the workspace filled with NaN bit patterns."""
    cfg = CONFIGS["c1"].with_(B=len(EDGE_USERS), H=4, dh=64, dtype="bf16")
    batch = make_batch(cfg, hist_override=[n for n, _ in EDGE_USERS],
                       m_override=[m for _, m in EDGE_USERS])
    pos, _, _ = ref.meta(batch)
    qkv = make_qkv(cfg, batch.T, seed=6)
    O, L = run_fwd(G, cfg, batch, pos, qkv, poison=True)
    Or, Lr = ref.attn(qkv[:, 0], qkv[:, 1], qkv[:, 2], batch, pos)
    _check(cfg, O, L, Or, Lr, np.arange(batch.T))


def test_fwd_full_size_c1_sampled(G):
    """The bench workload's shapes and launch; the oracle checks a seeded user sample."""
    cfg = CONFIGS["c1"]
    batch = make_batch(cfg)
    pos = np.zeros(batch.T, np.int64)
    users = sorted(np.random.default_rng(0).choice(cfg.B, 24, replace=False).tolist())
    pos_s, _, _ = ref.meta(batch, users=users)
    # positions are per user; for the sampled users the oracle's, elsewhere any valid value
    for u in range(batch.B):
        s, e, n = batch.seq_offsets[u], batch.seq_offsets[u + 1], batch.hist_len[u]
        pos[s:s + n] = np.arange(1, n + 1)
        pos[s + n:e] = n + 1
    rows = ref.user_rows(batch, users)
    assert np.array_equal(pos[rows], pos_s[rows])
    qkv = make_qkv(cfg, batch.T, seed=11)
    O, L = run_fwd(G, cfg, batch, pos, qkv)
    Or, Lr = ref.attn(qkv[:, 0], qkv[:, 1], qkv[:, 2], batch, pos, users=users)
    _check(cfg, O, L, Or, Lr, rows)


def test_fwd_candidates_equal_appending_each_alone(G):
    cfg = CONFIGS["c1"].with_(B=3, m=20)
    batch = make_batch(cfg)
    pos, _, _ = ref.meta(batch)
    qkv = make_qkv(cfg, batch.T, seed=3)
    O, _ = run_fwd(G, cfg, batch, pos, qkv)
    for u in range(batch.B):
        s, n = int(batch.seq_offsets[u]), int(batch.hist_len[u])
        for c in (0, 7, 19):
            keep = np.r_[np.arange(s, s + n), s + n + c]
            sub = ref.sub_batch(batch, [u])
            sub.seq_offsets = np.array([0, n + 1], np.int32)
            sub.item_ids, sub.action_ids, sub.ts = (batch.item_ids[keep], batch.action_ids[keep],
                                                    batch.ts[keep])
            O1, _ = run_fwd(G, cfg, sub, pos[keep], qkv[keep])
            assert ref.rel_to_max(O1[n], O[s + n + c]) <= 1e-2


def test_fwd_history_rows_ignore_later_tokens_bitwise(G):
    cfg = CONFIGS["c1"].with_(B=2)
    batch = make_batch(cfg, hist_override=[300, 200], m_override=[64, 16])
    pos, _, _ = ref.meta(batch)
    qkv = make_qkv(cfg, batch.T, seed=8)
    O, L = run_fwd(G, cfg, batch, pos, qkv)
    k = 150  # perturb every token of user 0 from local index 150 on
    qkv2 = qkv.copy()
    s = batch.seq_offsets[0]
    qkv2[s + k:batch.seq_offsets[1]] = make_qkv(cfg, batch.seq_offsets[1] - s - k, seed=9)
    b2 = make_batch(cfg, hist_override=[300, 200], m_override=[64, 16])
    b2.ts[s + k:batch.seq_offsets[1]] += 5
    O2, L2 = run_fwd(G, cfg, b2, pos, qkv2)
    assert np.array_equal(O[s:s + k], O2[s:s + k])
    assert np.array_equal(L[:, s:s + k], L2[:, s:s + k])
    assert np.array_equal(O[batch.seq_offsets[1]:], O2[batch.seq_offsets[1]:])


def test_fwd_device_error_flags(G):
    cfg = CONFIGS["c1"].with_(B=2)
    batch = make_batch(cfg)
    pos, _, _ = ref.meta(batch)
    bad = batch.seq_offsets.copy()
    bad[1] = bad[2] + 5  # the offsets run past T
    T, H, dh = batch.T, cfg.H, cfg.dh
    d = H * dh
    q = torch.zeros((T, 3 * d), dtype=torch.bfloat16, device="cuda")
    o = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(G.attn_workspace_size(2, T, H, dh, 700, False), dtype=torch.uint8,
                     device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    sp, st = G.alibi_slopes(H)
    G.attn_fwd(_dev(bad), _dev(batch.hist_len), 700, q, q[:, d:], q[:, 2 * d:], 3 * d, H, dh,
               _dev(pos.astype(np.int32)), _dev(batch.ts), sp, st, 0.125, o, d, None, ws, err,
               T=T)
    assert G.check_error(err) & G.DERR["LAYOUT"]


# ------------------------------------------------------------------------------------------
# backward
# ------------------------------------------------------------------------------------------
def run_bwd(G, cfg, batch, pos, qkv, dO, poison=False):
    T, H, dh = batch.T, cfg.H, cfg.dh
    d = H * dh
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    q = _dev(qkv.reshape(T, 3 * d), tdt)
    o = torch.empty((T, d), dtype=tdt, device="cuda")
    lse = torch.empty((H, T), dtype=torch.float32, device="cuda")
    off, hl = _dev(batch.seq_offsets), _dev(batch.hist_len)
    pos_t, ts_t = _dev(pos.astype(np.int32)), _dev(batch.ts)
    msl = int(np.max(np.diff(batch.seq_offsets)))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    sp, st = G.alibi_slopes(H)
    wsf = torch.empty(G.attn_workspace_size(batch.B, T, H, dh, msl, False), dtype=torch.uint8,
                      device="cuda")
    if poison:
        wsf.fill_(0xFF)
    G.attn_fwd(off, hl, msl, q, q[:, d:], q[:, 2 * d:], 3 * d, H, dh, pos_t, ts_t, sp, st,
               1.0 / math.sqrt(dh), o, d, lse, wsf, err, T=T)
    g = _dev(dO.reshape(T, d), tdt)
    dq = torch.empty_like(q)
    wsb = torch.empty(G.attn_workspace_size(batch.B, T, H, dh, msl, True), dtype=torch.uint8,
                      device="cuda")
    if poison:
        wsb.fill_(0xFF)
    G.attn_bwd(off, hl, msl, q, q[:, d:], q[:, 2 * d:], 3 * d, H, dh, pos_t, ts_t, sp, st,
               1.0 / math.sqrt(dh), o, g, d, lse, dq, dq[:, d:], dq[:, 2 * d:], wsb, err, T=T)
    assert G.check_error(err) == 0
    out = dq.float().cpu().numpy().astype(np.float64).reshape(T, 3, H, dh)
    return out[:, 0], out[:, 1], out[:, 2]


def _check_grads(cfg, got, want, rows, qkv=None, dO=None, batch=None, pos=None, users=None):
    """fp32: max-abs bound.  bf16: relative to the max, plus a per-token bound over all
    heads (so that one wrong row, a candidate's dk/dv or a short user's dq, cannot hide
    behind the tensor's max): each row within 2e-2 of max(its magnitude, 1/16 of the
    tensor's max) plus the absolute error the bf16 path carries by construction
    (``ref.grad_noise_floors``, from the oracle's probabilities and O)."""
    noise = (None, None, None)
    if cfg.dtype != "f32" and qkv is not None:
        sp, st = ref.slopes(cfg.H)
        scale = 1.0 / math.sqrt(cfg.dh)

        def fwd(q, k, v, offs, hl, p, ts):
            return oracle.attention_fwd(q, k, v, offs, hl, p, ts, sp, st, scale)

        us = range(batch.B) if users is None else users
        O, _ = ref.attn(qkv[:, 0], qkv[:, 1], qkv[:, 2], batch, pos, users=users)
        noise = tuple(x[rows] for x in ref.grad_noise_floors(
            fwd, qkv[:, 0], qkv[:, 1], qkv[:, 2], dO, O, batch, pos, us, scale))
    for name, a, b, nz in zip(("dq", "dk", "dv"), got, want, noise):
        if cfg.dtype == "f32":
            assert np.max(np.abs(a[rows] - b[rows])) <= F32_TOL, name
        else:
            ref.check_rows(a[rows], b[rows], BF16_TOL, name, noise=nz)


@pytest.mark.parametrize("name,B", [("c0", None), ("c3", 6)])
def test_bwd_parity(G, name, B):
    cfg = CONFIGS[name] if B is None else CONFIGS[name].with_(B=B)
    batch = make_batch(cfg)
    pos, _, _ = ref.meta(batch)
    qkv = make_qkv(cfg, batch.T, seed=21)
    dO = make_qkv(cfg, batch.T, seed=22, n=1)[:, 0]
    got = run_bwd(G, cfg, batch, pos, qkv, dO)
    want = ref.attn_bwd(qkv[:, 0], qkv[:, 1], qkv[:, 2], dO, batch, pos)
    _check_grads(cfg, got, want, np.arange(batch.T), qkv, dO, batch, pos)


@pytest.mark.parametrize("name,B", [("c0", None), ("c3", 6)])
def test_bwd_workspace_contents_do_not_matter(G, name, B):
    """Workspaces filled with NaN bit patterns: every scratch value the kernels read must
    be one they wrote (a query tile's per-row terms past the user's end included)."""
    cfg = CONFIGS[name] if B is None else CONFIGS[name].with_(B=B)
    batch = make_batch(cfg)
    pos, _, _ = ref.meta(batch)
    qkv = make_qkv(cfg, batch.T, seed=27)
    dO = make_qkv(cfg, batch.T, seed=28, n=1)[:, 0]
    got = run_bwd(G, cfg, batch, pos, qkv, dO, poison=True)
    want = ref.attn_bwd(qkv[:, 0], qkv[:, 1], qkv[:, 2], dO, batch, pos)
    _check_grads(cfg, got, want, np.arange(batch.T), qkv, dO, batch, pos)


def test_bwd_edge_cases(G):
    cfg = CONFIGS["c3"].with_(B=len(EDGE_USERS), H=2)
    batch = make_batch(cfg, hist_override=[n for n, _ in EDGE_USERS],
                       m_override=[m for _, m in EDGE_USERS])
    pos, _, _ = ref.meta(batch)
    qkv = make_qkv(cfg, batch.T, seed=23)
    dO = make_qkv(cfg, batch.T, seed=24, n=1)[:, 0]
    got = run_bwd(G, cfg, batch, pos, qkv, dO)
    want = ref.attn_bwd(qkv[:, 0], qkv[:, 1], qkv[:, 2], dO, batch, pos)
    _check_grads(cfg, got, want, np.arange(batch.T), qkv, dO, batch, pos)


def test_bwd_full_size_c3_sampled(G):
    cfg = CONFIGS["c3"]
    batch = make_batch(cfg)
    users = sorted(np.random.default_rng(1).choice(cfg.B, 12, replace=False).tolist())
    pos = np.zeros(batch.T, np.int64)
    for u in range(batch.B):
        s, e, n = batch.seq_offsets[u], batch.seq_offsets[u + 1], batch.hist_len[u]
        pos[s:s + n] = np.arange(1, n + 1)
        pos[s + n:e] = n + 1
    pos_s, _, _ = ref.meta(batch, users=users)
    rows = ref.user_rows(batch, users)
    assert np.array_equal(pos[rows], pos_s[rows])
    qkv = make_qkv(cfg, batch.T, seed=25)
    dO = make_qkv(cfg, batch.T, seed=26, n=1)[:, 0]
    got = run_bwd(G, cfg, batch, pos, qkv, dO)
    want = ref.attn_bwd(qkv[:, 0], qkv[:, 1], qkv[:, 2], dO, batch, pos, users=users)
    _check_grads(cfg, got, want, rows, qkv, dO, batch, pos, users=users)


def test_bwd_c2_shapes(G):
    """The four-layer inference workload's attention shapes (8 heads, 480 history tokens,
    256 candidates per user) through the backward: the candidate path with m >= 128."""
    cfg = CONFIGS["c2"].with_(B=12)
    batch = make_batch(cfg)
    pos, _, _ = ref.meta(batch)
    qkv = make_qkv(cfg, batch.T, seed=41)
    dO = make_qkv(cfg, batch.T, seed=42, n=1)[:, 0]
    got = run_bwd(G, cfg, batch, pos, qkv, dO)
    want = ref.attn_bwd(qkv[:, 0], qkv[:, 1], qkv[:, 2], dO, batch, pos)
    _check_grads(cfg, got, want, np.arange(batch.T), qkv, dO, batch, pos)


def test_fwd_year_long_histories(G):
    """Histories stretched to about a year: with the linear time slope the column terms
    reach thousands of log2 units, and they enter the scores through the MMA as three
    bf16 parts of c / (scale log2 e) summed in fp32 next to q.k.  The softmax of each
    row still matches the oracle."""
    cfg = CONFIGS["c1"].with_(B=6)
    batch = make_batch(cfg, hist_override=[300, 20, 500, 129, 1, 64])
    for u in range(batch.B):
        s, e = batch.seq_offsets[u], batch.seq_offsets[u + 1]
        t = batch.ts[s:e]
        span = max(int(t[-1] - t[0]), 1)
        batch.ts[s:e] = t[0] + (t - t[0]) * (31_536_000 // span)  # order kept
    pos, _, _ = ref.meta(batch)
    qkv = make_qkv(cfg, batch.T, seed=41)
    O, L = run_fwd(G, cfg, batch, pos, qkv)
    Or, Lr = ref.attn(qkv[:, 0], qkv[:, 1], qkv[:, 2], batch, pos)
    assert np.all(np.isfinite(O)) and np.all(np.isfinite(L))
    _check(cfg, O, L, Or, Lr, np.arange(batch.T))


def test_fwd_older_keys_dominating_take_the_exact_path(G):
    """Keys are visited most recent first; when much older keys score far higher
    (beyond 2^100 in a row sum), the tile is recomputed with an exact offset."""
    cfg = CONFIGS["c1"].with_(B=3)
    batch = make_batch(cfg, hist_override=[400, 300, 130], m_override=[20, 7, 140])
    pos, _, _ = ref.meta(batch)
    qkv = make_qkv(cfg, batch.T, seed=31, std=0.5)
    for u in range(batch.B):
        s = batch.seq_offsets[u]
        qkv[s:s + 100, 1] = 3.0  # oldest keys: large positive scores against ...
        qkv[s + 100:batch.seq_offsets[u + 1], 0] = 3.0  # ... queries pointing the same way
    O, L = run_fwd(G, cfg, batch, pos, qkv)
    Or, Lr = ref.attn(qkv[:, 0], qkv[:, 1], qkv[:, 2], batch, pos)
    assert np.all(np.isfinite(O)) and np.all(np.isfinite(L))
    _check(cfg, O, L, Or, Lr, np.arange(batch.T))
