"""GPU parity of the metadata + embedding assembly (forward and backward)."""

import numpy as np
import pytest
import torch

import oracle
import ref
from gen import CONFIGS, make_batch, make_model

pytestmark = pytest.mark.gpu


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


def _tables(cfg, model, item_tab=None):
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    if item_tab is None:
        from gen import item_table_torch

        item_tab = item_table_torch(cfg.seed, cfg.n_item, cfg.d, cfg.dtype, "cuda")
    return (item_tab, _dev(model.action_tab, tdt), _dev(model.pos_tab, tdt),
            _dev(model.ri_tab, tdt), _dev(model.rt_tab, tdt))


def run_embed(G, cfg, batch, tabs):
    T, d = batch.T, cfg.d
    tdt = tabs[0].dtype
    E = torch.empty((T, d), dtype=tdt, device="cuda")
    meta = [torch.empty(T, dtype=torch.int32, device="cuda") for _ in range(3)]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.embed_assemble(_dev(batch.seq_offsets), _dev(batch.hist_len), _dev(batch.item_ids),
                     _dev(batch.action_ids), _dev(batch.ts), *tabs, E, *meta, err)
    code = G.check_error(err)
    return E, meta, code


def _compare(cfg, batch, model, E, meta, users=None):
    Er, mr = ref.embed(batch, model, users)
    rows = np.arange(batch.T) if users is None else ref.user_rows(batch, users)
    for got, want in zip(meta, mr):
        assert np.array_equal(got.cpu().numpy()[rows], want[rows])
    Eg = E.float().cpu().numpy().astype(np.float64)
    if cfg.dtype == "f32":
        assert np.max(np.abs(Eg[rows] - Er[rows])) <= 1e-4
    else:
        assert ref.rel_to_max(Eg[rows], Er[rows]) <= 2e-2
        # one rounding of the fp32 sum: within half a bf16 ulp (plus fp32 slack) everywhere
        assert np.all(np.abs(Eg[rows] - Er[rows]) <= np.abs(Er[rows]) * 2.0 ** -8 + 1e-6)


@pytest.mark.parametrize("name", ["c0", "c1"])
def test_embed_parity_full(G, name):
    cfg = CONFIGS[name]
    batch = make_batch(cfg)
    model = make_model(cfg)
    E, meta, code = run_embed(G, cfg, batch, _tables(cfg, model))
    assert code == 0
    _compare(cfg, batch, model, E, meta)


@pytest.mark.parametrize("name", ["c2", "c4_m1024"])
def test_embed_parity_full_size_sampled(G, name):
    cfg = CONFIGS[name]
    batch = make_batch(cfg)
    model = make_model(cfg)
    E, meta, code = run_embed(G, cfg, batch, _tables(cfg, model))
    assert code == 0
    users = sorted(np.random.default_rng(2).choice(cfg.B, 16, replace=False).tolist())
    _compare(cfg, batch, model, E, meta, users)


def test_embed_edge_cases(G):
    users = [(1, 0), (1, 1), (0, 5), (480, 3), (300, 0), (2, 1), (129, 128)]
    cfg = CONFIGS["c1"].with_(B=len(users), n_item=5000)
    batch = make_batch(cfg, hist_override=[n for n, _ in users], m_override=[m for _, m in users])
    s, e = batch.seq_offsets[3], batch.seq_offsets[4]
    batch.ts[s:e] = batch.ts[s]  # every timestamp equal: one request, no earlier request
    s, e = batch.seq_offsets[5], batch.seq_offsets[6]
    batch.ts[s + 2:e] = batch.ts[s + 1]  # candidate in the same request as the last history item
    batch.item_ids[0] = 0
    batch.item_ids[-1] = cfg.n_item - 1  # table bounds
    model = make_model(cfg)
    E, meta, code = run_embed(G, cfg, batch, _tables(cfg, model))
    assert code == 0
    _compare(cfg, batch, model, E, meta)


def test_embed_long_history_chunks_and_clamps(G):
    """History longer than one scan chunk and more requests than request-index rows."""
    cfg = CONFIGS["c1"].with_(B=2, n_item=5000, n_pos=1400, group_mean=1.2)
    batch = make_batch(cfg, hist_override=[1300, 700], m_override=[3, 2])
    model = make_model(cfg)
    E, meta, code = run_embed(G, cfg, batch, _tables(cfg, model))
    assert code == 0
    _compare(cfg, batch, model, E, meta)
    assert meta[1].max().item() == cfg.n_ri - 1


def test_embed_device_error_flags(G):
    cfg = CONFIGS["c1"].with_(B=3, n_item=5000)
    model = make_model(cfg)
    tabs = _tables(cfg, model)
    b = make_batch(cfg)
    b.item_ids[5] = cfg.n_item + 3
    _, _, code = run_embed(G, cfg, b, tabs)
    assert code & G.DERR["ITEM_ID"]
    b = make_batch(cfg)
    b.action_ids[2] = 8  # a history token may not use the mask action
    _, _, code = run_embed(G, cfg, b, tabs)
    assert code & G.DERR["ACTION_ID"]
    b = make_batch(cfg)
    s = b.seq_offsets[1]
    b.ts[s + 3] = b.ts[s + 2] - 100
    _, _, code = run_embed(G, cfg, b, tabs)
    assert code & G.DERR["TS_ORDER"]
    b = make_batch(cfg)
    b.hist_len[1] = 10_000  # more history than tokens
    _, _, code = run_embed(G, cfg, b, tabs)
    assert code & G.DERR["LAYOUT"]


# ------------------------------------------------------------------------------------------
# backward
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["c0", "c3"])
def test_embed_bwd_parity(G, name):
    """c3 runs on its full 4M-row item table, so the Zipf(1.05)-hot rows meet the
    contention they meet in training; rows no token reads must stay exactly zero."""
    cfg = CONFIGS[name]
    batch = make_batch(cfg)
    mr = ref.meta(batch)
    T, d = batch.T, cfg.d
    rng = np.random.default_rng(4)
    dE = rng.normal(size=(T, d)).astype(np.float32)
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    dE_t = _dev(dE, tdt)
    dE_used = dE_t.float().cpu().numpy().astype(np.float64)
    f32 = dict(dtype=torch.float32, device="cuda")
    g = [torch.zeros((cfg.n_item, d), **f32), torch.zeros((9, d), **f32),
         torch.zeros((cfg.n_pos, d), **f32), torch.zeros((cfg.n_ri, d), **f32),
         torch.zeros((cfg.n_rt, d), **f32)]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.embed_assemble_bwd(_dev(batch.seq_offsets), _dev(batch.hist_len), _dev(batch.item_ids),
                         _dev(batch.action_ids), *[_dev(m.astype(np.int32)) for m in mr], dE_t,
                         *g, err)
    assert G.check_error(err) == 0
    uniq, inv = np.unique(batch.item_ids, return_inverse=True)
    want = oracle.embed_assemble_bwd(dE_used, batch.seq_offsets, batch.hist_len, inv,
                                     batch.action_ids, mr, len(uniq), 9, cfg.n_pos, cfg.n_ri,
                                     cfg.n_rt)
    touched = torch.zeros(cfg.n_item, dtype=torch.bool, device="cuda")
    touched[_dev(uniq.astype(np.int64))] = True
    assert float(g[0][~touched].abs().max()) == 0.0  # on the device: the table is 8 GB at c3
    got_item = g[0][_dev(uniq.astype(np.int64))].cpu().numpy().astype(np.float64)
    pairs = [(got_item, want["item"])] + [
        (t.cpu().numpy().astype(np.float64), want[k])
        for t, k in zip(g[1:], ("action", "pos", "ri", "rt"))]
    for got, w in pairs:
        # fp32 accumulation of O(T) terms of size O(1): allow a few ulps of the row sums
        assert np.max(np.abs(got - w)) <= 1e-4 * max(1.0, np.max(np.abs(w))), np.max(np.abs(got - w))


def _run_fused(G, cfg, batch, tabs, eps=1e-6):
    T, d = batch.T, cfg.d
    x = torch.full((T, d), float("nan"), device="cuda")
    a = torch.full((T, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    meta = [torch.empty(T, dtype=torch.int32, device="cuda") for _ in range(3)]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.embed_assemble_rmsnorm(_dev(batch.seq_offsets), _dev(batch.hist_len), _dev(batch.item_ids),
                             _dev(batch.action_ids), _dev(batch.ts), *tabs, x, a, *meta, err,
                             eps=eps)
    return x, a, meta, G.check_error(err)


@pytest.mark.parametrize("users", [16, None])
def test_embed_rmsnorm_equals_gather_sum_then_rmsnorm(G, users):
    """The fused entry gives, bit for bit, the residual rows and normalised rows of the
    gather-sum followed by the RMSNorm pass (the first block's input at c2 shapes)."""
    cfg = CONFIGS["c2"]
    batch = make_batch(cfg, users=list(range(users)) if users else None)
    tabs = _tables(cfg, make_model(cfg))
    E, meta, code = run_embed(G, cfg, batch, tabs)
    assert code == 0
    x2 = torch.empty((batch.T, cfg.d), device="cuda")
    a2 = torch.empty((batch.T, cfg.d), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.rmsnorm(E, a2, err, x_out=x2, eps=1e-6)
    assert G.check_error(err) == 0
    x, a, meta_f, code_f = _run_fused(G, cfg, batch, tabs)
    assert code_f == 0
    assert torch.equal(x, x2)
    assert torch.equal(a, a2)
    for m1, m2 in zip(meta_f, meta):
        assert torch.equal(m1, m2)


def test_embed_rmsnorm_against_oracle(G):
    """x_out is E (the five rows' sum, rounded once to bf16) and a_out its RMSNorm,
    checked against the float64 oracle on a seeded sample of c2 users."""
    cfg = CONFIGS["c2"]
    batch = make_batch(cfg, users=list(range(8)))
    model = make_model(cfg)
    x, a, meta, code = _run_fused(G, cfg, batch, _tables(cfg, model))
    assert code == 0
    _compare(cfg, batch, model, x, meta)
    Er, _ = ref.embed(batch, model, None)
    want = Er / np.sqrt((Er * Er).mean(axis=1, keepdims=True) + 1e-6)
    got = a.double().cpu().numpy()
    assert ref.rel_to_max(got, want) <= 2e-2
    err_r = np.abs(got - want).max(axis=1) / np.abs(want).max(axis=1)
    assert np.max(err_r) <= 2e-2


def test_embed_rmsnorm_rejects_other_widths(G):
    cfg = CONFIGS["c1"]  # d = 256
    batch = make_batch(cfg, users=list(range(2)))
    with pytest.raises(G.GenRankError):
        _run_fused(G, cfg, batch, _tables(cfg, make_model(cfg)))
