"""Pins for the oracle's embedding assembly, the blocks around attention and the backward."""

import numpy as np
import pytest

import oracle
from gen import CONFIGS, make_batch, make_model


def _compact_items(batch, model):
    """Gather the item rows a batch uses; remap ids into the compact table."""
    uniq, inv = np.unique(batch.item_ids, return_inverse=True)
    return model.item_rows(uniq), inv.astype(np.int64)


def _small(cfg_name="c0", B=3, layers=None, dtype="f32", d=None):
    cfg = CONFIGS[cfg_name].with_(B=B, dtype=dtype)
    if layers is not None:
        cfg = cfg.with_(layers=layers)
    b = make_batch(cfg)
    mdl = make_model(cfg)
    return cfg, b, mdl


def _embed(b, mdl, tabs=None):
    item, ids = _compact_items(b, mdl)
    meta = oracle.token_metadata(b.seq_offsets, b.hist_len, b.ts)
    t = dict(item=item, action=mdl.action_tab, pos=mdl.pos_tab, ri=mdl.ri_tab, rt=mdl.rt_tab)
    if tabs:
        t.update(tabs)
    E = oracle.embed_assemble(b.seq_offsets, b.hist_len, ids, b.action_ids, meta, t["item"],
                              t["action"], t["pos"], t["ri"], t["rt"])
    return E, meta, ids, t


def test_embed_single_table_closed_form():
    cfg, b, mdl = _small()
    E, meta, ids, t = _embed(b, mdl)
    zeros = {k: np.zeros_like(v) for k, v in t.items()}
    for name in t:
        only = dict(zeros)
        only[name] = t[name]
        E1, _, _, _ = _embed(b, mdl, only)
        if name == "item":
            ref = t["item"][ids]
        elif name == "action":
            a = b.action_ids.astype(np.int64).copy()
            for u in range(b.B):
                a[b.seq_offsets[u] + b.hist_len[u]:b.seq_offsets[u + 1]] = 8
            ref = t["action"][a]
        else:
            ref = t[name][{"pos": meta[0], "ri": meta[1], "rt": meta[2]}[name]]
        assert np.array_equal(E1, ref.astype(np.float64)), name


def test_candidates_use_mask_action_row():
    cfg, b, mdl = _small()
    scrambled = b.action_ids.copy()
    for u in range(b.B):
        scrambled[b.seq_offsets[u] + b.hist_len[u]:b.seq_offsets[u + 1]] = 3
    E, meta, ids, t = _embed(b, mdl)
    E2 = oracle.embed_assemble(b.seq_offsets, b.hist_len, ids, scrambled, meta, t["item"],
                               t["action"], t["pos"], t["ri"], t["rt"])
    assert np.array_equal(E, E2)


def test_embed_backward_is_the_adjoint():
    cfg, b, mdl = _small()
    E, meta, ids, t = _embed(b, mdl)
    dE = np.random.default_rng(0).normal(size=E.shape)
    g = oracle.embed_assemble_bwd(dE, b.seq_offsets, b.hist_len, ids, b.action_ids, meta,
                                  t["item"].shape[0], 9, t["pos"].shape[0], t["ri"].shape[0],
                                  t["rt"].shape[0])
    # E is linear in the tables: <E(tables), dE> = sum over tables <table, grad>
    lhs = float(np.sum(E * dE))
    rhs = sum(float(np.sum(np.asarray(t[k], np.float64) * g[k])) for k in t)
    assert abs(lhs - rhs) < 1e-12 * max(1.0, abs(lhs))
    for k in g:
        assert np.allclose(g[k].sum(axis=0), dE.sum(axis=0), atol=1e-10)


def _forward(cfg, b, mdl, E=None):
    if E is None:
        E, meta, _, _ = _embed(b, mdl)
    else:
        meta = oracle.token_metadata(b.seq_offsets, b.hist_len, b.ts)
    z, cache = oracle.block_forward(E, mdl.layers, mdl.w_head, b.seq_offsets, b.hist_len,
                                    meta[0], b.ts, cfg.H, cfg.ffn)
    return z, cache, E, meta


@pytest.mark.parametrize("ffn", [False, True])
def test_model_candidates_equal_appending_each_alone(ffn):
    cfg = CONFIGS["c0"].with_(B=2, ffn=ffn, layers=2 if ffn else 1, m=4)
    b = make_batch(cfg)
    mdl = make_model(cfg)
    z, _, _, _ = _forward(cfg, b, mdl)
    k = 0
    for u in range(b.B):
        n = int(b.hist_len[u])
        for c in range(int(b.cand_count[u])):
            b1 = make_batch(cfg, users=[u], m_override=[1])
            s = int(b.seq_offsets[u])
            keep = list(range(s, s + n)) + [s + n + c]
            b1.item_ids = b.item_ids[keep]
            b1.action_ids = b.action_ids[keep]
            b1.ts = b.ts[keep]
            z1, _, _, _ = _forward(cfg, b1, mdl)
            assert abs(z1[0] - z[k]) <= 1e-12 * max(1.0, abs(z[k]))
            k += 1


def test_model_history_rows_ignore_later_tokens_bitwise():
    cfg = CONFIGS["c0"].with_(B=1, ffn=True, layers=2)
    b = make_batch(cfg)
    mdl = make_model(cfg)
    _, cache, _, _ = _forward(cfg, b, mdl)
    kk = int(b.hist_len[0]) // 2
    b2 = make_batch(cfg)
    b2.item_ids[kk:] = (b2.item_ids[kk:] + 7) % cfg.n_item
    b2.action_ids[kk:int(b2.hist_len[0])] = (b2.action_ids[kk:int(b2.hist_len[0])] + 1) % 8
    b2.ts[kk:] += 11
    _, cache2, _, _ = _forward(cfg, b2, mdl)
    assert np.array_equal(cache["x_out"][:kk], cache2["x_out"][:kk])
    assert not np.array_equal(cache["x_out"][kk:], cache2["x_out"][kk:])


@pytest.mark.parametrize("ffn", [False, True])
def test_model_backward_matches_finite_differences(ffn):
    cfg = CONFIGS["c0"].with_(B=2, ffn=ffn, layers=2 if ffn else 1, m=3, training=True,
                              hist=("uniform", 5, 9))
    b = make_batch(cfg)
    mdl = make_model(cfg)
    z, cache, E, meta = _forward(cfg, b, mdl)
    y = b.labels
    dE = oracle.block_backward(z, y, cache, mdl.layers, mdl.w_head, b.seq_offsets, b.hist_len,
                               meta[0], b.ts, cfg.H, cfg.ffn)
    eps = 1e-6
    rng = np.random.default_rng(3)
    for _ in range(8):
        i, j = int(rng.integers(0, E.shape[0])), int(rng.integers(0, E.shape[1]))
        Ep, Em = E.copy(), E.copy()
        Ep[i, j] += eps
        Em[i, j] -= eps
        fp = oracle.bce_loss(_forward(cfg, b, mdl, Ep)[0], y)
        fm = oracle.bce_loss(_forward(cfg, b, mdl, Em)[0], y)
        fd = (fp - fm) / (2 * eps)
        assert abs(fd - dE[i, j]) <= 1e-7 * max(1e-3, abs(fd)) + 1e-10, (i, j, fd, dE[i, j])
