"""End-to-end parity of the scoring and training steps (library kernels + torch
blocks) against the float64 oracle on the same seeded inputs."""

import numpy as np
import pytest
import torch

import oracle
import ref
from gen import CONFIGS, make_batch, make_model

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    from generative_ranking_recommendation_b200 import model as M
    from generative_ranking_recommendation_b200.csrc import build

    build.build()
    return M


@pytest.mark.parametrize("name,users", [("c0", None), ("c1", 32), ("c2", 6), ("c4_m256", 6)])
def test_logits_parity(M, name, users):
    cfg = CONFIGS[name]
    batch = make_batch(cfg)
    model = make_model(cfg)
    gm = M.GenRankModel(cfg, model, "cuda")
    db = M.DeviceBatch.from_batch(batch, "cuda")
    z = gm.forward(db).cpu().numpy().astype(np.float64)
    from generative_ranking_recommendation_b200 import genrank as G

    assert G.check_error(gm.err) == 0
    sel = list(range(batch.B)) if users is None else sorted(
        np.random.default_rng(3).choice(cfg.B, users, replace=False).tolist())
    zr = ref.model_logits(batch, model, sel)
    cr_all = ref.cand_rows(batch)
    where = {r: k for k, r in enumerate(cr_all)}
    zg = z[[where[r] for r in ref.cand_rows(batch, sel)]]
    if cfg.dtype == "f32":
        assert np.max(np.abs(zg - zr)) <= 1e-4
    else:
        assert ref.rel_to_max(zg, zr) <= 2e-2


def test_train_step_parity(M):
    cfg = CONFIGS["c3"].with_(B=6, n_item=100_000)
    batch = make_batch(cfg)
    model = make_model(cfg)
    gm = M.GenRankModel(cfg, model, "cuda")
    db = M.DeviceBatch.from_batch(batch, "cuda")
    loss, z, grads = gm.train_step(db)
    from generative_ranking_recommendation_b200 import genrank as G

    assert G.check_error(gm.err) == 0
    # oracle: forward, BCE, analytic backward, scatter into the tables
    item, ids = ref.compact_items(batch, model)
    mr = ref.meta(batch)
    E = oracle.embed_assemble(batch.seq_offsets, batch.hist_len, ids, batch.action_ids, mr, item,
                              model.action_tab, model.pos_tab, model.ri_tab, model.rt_tab)
    zr, cache = oracle.block_forward(E, model.layers, model.w_head, batch.seq_offsets,
                                     batch.hist_len, mr[0], batch.ts, cfg.H, cfg.ffn)
    assert ref.rel_to_max(z.cpu().numpy(), zr) <= 2e-2
    lr = oracle.bce_loss(zr, batch.labels)
    assert abs(float(loss) - lr) <= 2e-2 * abs(lr)
    dE = oracle.block_backward(zr, batch.labels, cache, model.layers, model.w_head,
                               batch.seq_offsets, batch.hist_len, mr[0], batch.ts, cfg.H, cfg.ffn)
    uniq = np.unique(batch.item_ids)
    gr = oracle.embed_assemble_bwd(dE, batch.seq_offsets, batch.hist_len, ids, batch.action_ids,
                                   mr, len(uniq), 9, cfg.n_pos, cfg.n_ri, cfg.n_rt)
    got = {k: v.cpu().numpy().astype(np.float64) for k, v in grads.items()}
    assert ref.rel_to_max(got["item"][uniq], gr["item"]) <= 2e-2
    for k in ("action", "pos", "ri", "rt"):
        assert ref.rel_to_max(got[k], gr[k]) <= 2e-2, k


@pytest.mark.parametrize("name", ["c0", "c2"])
def test_captured_step_matches_forward(M, name):
    """The graph-captured step gives the eager forward's logits bit for bit, and
    scores new inputs loaded into the captured batch."""
    cfg = CONFIGS[name]
    batch = make_batch(cfg, users=list(range(4)))
    gm = M.GenRankModel(cfg, make_model(cfg), "cuda")
    db = M.DeviceBatch.from_batch(batch, "cuda")
    step = M.CapturedStep(gm, db)
    z0 = step.run().clone()
    assert torch.equal(z0, gm.forward(M.DeviceBatch.from_batch(batch, "cuda")))
    # same shapes, other items: load into the captured buffers and replay
    b2 = make_batch(cfg, users=list(range(4)))
    b2.item_ids[:] = np.random.default_rng(5).integers(0, cfg.n_item, b2.item_ids.shape)
    step.load([torch.from_numpy(np.ascontiguousarray(a)) for a in M.DeviceBatch.host_arrays(b2)])
    z1 = step.run().clone()
    assert torch.equal(z1, gm.forward(M.DeviceBatch.from_batch(b2, "cuda")))
    assert not torch.equal(z0, z1)
    from generative_ranking_recommendation_b200 import genrank as G

    assert G.check_error(gm.err) == 0


@pytest.mark.parametrize("name", ["c2", "c1"])
def test_fused_blocks_match_torch_blocks(M, name):
    """The scoring step on the library's fused linear layers and the same step with the
    blocks as torch ops give the same logits within the bf16 tolerance."""
    cfg = CONFIGS[name]
    batch = make_batch(cfg, users=list(range(16)))
    gm = M.GenRankModel(cfg, make_model(cfg), "cuda")
    gm.fused_qkv = True  # the library's QKV projection in the one-block step as well
    assert gm.fused_blocks == (name == "c2")
    db = M.DeviceBatch.from_batch(batch, "cuda")
    z_fused = gm.forward(db).double().cpu().numpy()
    z_torch = gm.forward(db, blocks="torch").double().cpu().numpy()
    assert ref.rel_to_max(z_fused, z_torch) <= 2e-2
    from generative_ranking_recommendation_b200 import genrank as G

    assert G.check_error(gm.err) == 0


def test_train_step_gradient_tables_start_clean(M):
    """The gradient tables are reused across steps, the previous step's item rows zeroed:
    a second step's tables equal those of a model that ran only that step, and item rows
    only the first batch touched are exactly zero."""
    cfg = CONFIGS["c3"].with_(B=4, n_item=50_000)
    model = make_model(cfg)
    b1, b2 = make_batch(cfg, seed=101), make_batch(cfg, seed=202)
    gm = M.GenRankModel(cfg, model, "cuda")
    gm.train_step(M.DeviceBatch.from_batch(b1, "cuda"))
    _, _, g2 = gm.train_step(M.DeviceBatch.from_batch(b2, "cuda"))
    g2 = {k: v.cpu().numpy().astype(np.float64) for k, v in g2.items()}
    fresh = M.GenRankModel(cfg, model, "cuda")
    _, _, gf = fresh.train_step(M.DeviceBatch.from_batch(b2, "cuda"))
    gf = {k: v.cpu().numpy().astype(np.float64) for k, v in gf.items()}
    from generative_ranking_recommendation_b200 import genrank as G

    assert G.check_error(gm.err) == 0 and G.check_error(fresh.err) == 0
    for k in g2:  # equal up to the order of the atomic additions
        assert ref.rel_to_max(g2[k], gf[k]) <= 1e-4, k
    only1 = np.setdiff1d(np.unique(b1.item_ids), np.unique(b2.item_ids))
    assert only1.size > 0 and not g2["item"][only1].any()
