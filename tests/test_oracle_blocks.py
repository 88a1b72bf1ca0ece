"""Pins for the oracle's blocks around the attention (norms, FFN, residuals, head) and
its loss, independent of the oracle's own code.

* hand-worked examples (``tests/golden/block_hand_example.txt``, every step worked
  out by hand from the definitions cited there);
* closed forms: RMSNorm of a constant vector, SiLU(0) = 0 and SiLU(x) -> x, the
  loss at z = 0 equal to ln 2;
* an independent float64 torch composition (``F.rms_norm``, ``F.silu``,
  ``F.scaled_dot_product_attention`` with an explicit additive bias and mask,
  ``F.binary_cross_entropy_with_logits``), library routines rather than the oracle;
* "history rows carry no loss" ("GenRank [2025]" chapter notes, §1.3.1): with the
  attention's projections zeroed, the only route from a history row to the loss is
  closed, so its gradient is exactly zero while a candidate row's is dz * w_head;
* planted mistakes: mutated copies of the oracle's source (sum for mean in the RMS,
  eps outside the root, a dropped residual or final norm, sigmoid for SiLU, sum for
  mean in the loss) each fail one of the pins above.
"""

import inspect
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import oracle.genrank_oracle as og
from gen import CONFIGS, make_batch, make_model

TS0 = 1_700_000_000


def _g(golden, key):
    return [float(x) for x in golden("block_hand_example.txt")[key]]


# ------------------------------------------------------------------------------------------
# hand-worked examples
# ------------------------------------------------------------------------------------------
def _example_a(block=None):
    block = block or oracle.block_forward
    E = np.array([[1.0, 0.0], [0.0, 1.0]])
    eye = np.eye(2)
    layers = [{"Wq": eye, "Wk": eye, "Wv": eye, "Wo": eye}]
    z, _ = block(E, layers, np.array([1.0, 0.0]), np.array([0, 2]), np.array([1]),
                 np.array([1, 2]), np.array([TS0, TS0 + 3600]), 1, False)
    return z


def _example_b(block=None):
    block = block or oracle.block_forward
    E = np.array([[1.0, 1.0], [1.0, -1.0]])
    W1 = np.zeros((2, 8))
    W1[0, 0] = 1.0
    W2 = np.zeros((8, 2))
    W2[0, 0] = 1.0
    layers = [{"Wq": np.zeros((2, 2)), "Wk": np.zeros((2, 2)), "Wv": np.eye(2), "Wo": np.eye(2),
               "W1": W1, "W2": W2}]
    z, cache = block(E, layers, np.array([1.0, 0.0]), np.array([0, 2]), np.array([1]),
                     np.array([1, 2]), np.array([TS0, TS0]), 1, True)
    return z, cache


def test_one_layer_scorer_hand_example(golden):
    z = _example_a()
    assert z.shape == (1,)
    assert abs(z[0] - _g(golden, "A_z")[0]) <= 1e-15


def test_ffn_block_hand_example(golden):
    z, cache = _example_b()
    c = cache["layers"][0]
    r = _g(golden, "B_r")[0]
    assert np.allclose(c["r_in"][:, 0], r, rtol=0, atol=1e-15)
    assert np.allclose(c["x_mid"][1], _g(golden, "B_x1"), rtol=0, atol=1e-14)
    assert abs(c["U"][1, 0] - _g(golden, "B_silu")[0]) <= 1e-14
    assert np.all(c["U"][:, 1:] == 0.0)  # SiLU(0) = 0 in the seven zero hidden units
    assert abs(z[0] - _g(golden, "B_z")[0]) <= 1e-14


def test_bce_hand_values(golden):
    z, y = _g(golden, "bce_z"), _g(golden, "bce_y")
    assert abs(oracle.bce_loss(z, y) - _g(golden, "bce_value")[0]) <= 1e-15
    ln2 = _g(golden, "bce_at_zero")[0]
    for lab in (0.0, 1.0):
        assert abs(oracle.bce_loss([0.0, 0.0, 0.0], [lab, lab, 1.0 - lab]) - ln2) <= 1e-15


# ------------------------------------------------------------------------------------------
# closed forms of the pieces
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("c,d", [(1.0, 2), (-3.5, 7), (1e-2, 512), (0.0, 4)])
def test_rms_norm_of_a_constant_vector(c, d):
    # mean square c^2, so every entry becomes c / sqrt(c^2 + eps)
    y, r = og._rms(np.full((1, d), c))
    assert np.allclose(y, c / math.sqrt(c * c + 1e-6), rtol=1e-15, atol=0)
    assert abs(r[0, 0] - 1.0 / math.sqrt(c * c + 1e-6)) <= 1e-12 / math.sqrt(c * c + 1e-6)


def test_rms_norm_345():
    # [3, 4]: mean square (9 + 16) / 2 = 12.5
    y, _ = og._rms(np.array([[3.0, 4.0]]))
    assert np.allclose(y, np.array([[3.0, 4.0]]) / math.sqrt(12.5 + 1e-6), rtol=1e-15, atol=0)


def test_silu_limits():
    x = np.array([0.0, 40.0, -40.0, 1.0])
    s = x * og._sigmoid(x)
    assert s[0] == 0.0
    assert abs(s[1] - 40.0) <= 1e-12  # SiLU(x) -> x
    assert abs(s[2]) <= 1e-15  # SiLU(x) -> 0 from below
    assert abs(s[3] - 1.0 / (1.0 + math.exp(-1.0))) <= 1e-16


# ------------------------------------------------------------------------------------------
# an independent torch float64 composition of the same blocks
# ------------------------------------------------------------------------------------------
def _torch_logits(E, layers, w_head, offs, hl, pos, ts, H, ffn):
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))  # noqa: E731
    x = t(E)
    T, d = x.shape
    dh = d // H
    slopes = 2.0 ** (-8.0 * (np.arange(H) + 1) / H)
    # per-user additive bias + mask as a dense [T, T] float matrix per head (-inf across
    # users and on masked pairs)
    bias = torch.full((H, T, T), float("-inf"), dtype=torch.float64)
    for u in range(len(hl)):
        s, e, n = int(offs[u]), int(offs[u + 1]), int(hl[u])
        for i in range(s, e):
            for j in range(s, e):
                li, lj = i - s, j - s
                if (li < n and lj <= li) or (li >= n and (lj < n or lj == li)):
                    dp, dt = abs(int(pos[i]) - int(pos[j])), abs(int(ts[i]) - int(ts[j]))
                    bias[:, i, j] = torch.from_numpy(-slopes * dp - slopes / 3600.0 * dt)
    norm = (lambda v: F.rms_norm(v, (d,), eps=1e-6)) if ffn else (lambda v: v)
    for L in layers:
        a = norm(x)
        q, k, v = ((a @ t(L[w])).reshape(T, H, dh).transpose(0, 1) for w in ("Wq", "Wk", "Wv"))
        o = F.scaled_dot_product_attention(q[None], k[None], v[None], attn_mask=bias[None])[0]
        x = x + o.transpose(0, 1).reshape(T, d) @ t(L["Wo"])
        if ffn:
            x = x + F.silu(norm(x) @ t(L["W1"])) @ t(L["W2"])
    x = norm(x)
    rows = [i for u in range(len(hl)) for i in range(int(offs[u]) + int(hl[u]), int(offs[u + 1]))]
    return (x[rows] @ t(w_head)).numpy()


def _random_model(ffn, layers, seed=0):
    cfg = CONFIGS["c0"].with_(B=3, ffn=ffn, layers=layers, m=3, hist=("uniform", 4, 9),
                              training=True)
    b = make_batch(cfg, seed=seed)
    mdl = make_model(cfg, seed=seed)
    rng = np.random.default_rng(seed)
    # unit-scale weights so the softmax, norms and SiLU are far from their linear ranges
    for L in mdl.layers:
        for k in L:
            L[k] = rng.normal(0.0, 1.0 / math.sqrt(L[k].shape[0]), size=L[k].shape)
    E = rng.normal(size=(b.T, cfg.d))
    pos, _, _ = oracle.token_metadata(b.seq_offsets, b.hist_len, b.ts)
    return cfg, b, mdl, E, pos


@pytest.mark.parametrize("ffn,layers", [(False, 1), (True, 1), (True, 2)])
def test_blocks_match_torch_composition(ffn, layers):
    cfg, b, mdl, E, pos = _random_model(ffn, layers)
    z, _ = oracle.block_forward(E, mdl.layers, mdl.w_head, b.seq_offsets, b.hist_len, pos, b.ts,
                                cfg.H, ffn)
    zt = _torch_logits(E, mdl.layers, mdl.w_head, b.seq_offsets, b.hist_len, pos, b.ts, cfg.H, ffn)
    assert np.max(np.abs(z - zt)) <= 1e-12 * max(1.0, np.max(np.abs(zt)))


def test_bce_matches_torch():
    rng = np.random.default_rng(4)
    z = rng.normal(0, 3, size=37)
    y = (rng.random(37) < 0.3).astype(np.float64)
    want = F.binary_cross_entropy_with_logits(torch.from_numpy(z), torch.from_numpy(y)).item()
    assert abs(oracle.bce_loss(z, y) - want) <= 1e-15 * max(1.0, abs(want))


# ------------------------------------------------------------------------------------------
# history rows carry no loss
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("ffn,layers", [(False, 1), (True, 2)])
def test_history_rows_carry_no_loss(ffn, layers):
    """With W_q = W_k = W_v = 0 no row reads another, so a history row reaches the loss
    only if the loss itself sits there: its gradient must be exactly 0.  For the
    one-layer scorer a candidate row's gradient is then exactly dz * w_head."""
    cfg, b, mdl, E, pos = _random_model(ffn, layers, seed=5)
    for L in mdl.layers:
        for k in ("Wq", "Wk", "Wv"):
            L[k] = np.zeros_like(L[k])
    z, cache = oracle.block_forward(E, mdl.layers, mdl.w_head, b.seq_offsets, b.hist_len, pos,
                                    b.ts, cfg.H, ffn)
    dE = oracle.block_backward(z, b.labels, cache, mdl.layers, mdl.w_head, b.seq_offsets,
                               b.hist_len, pos, b.ts, cfg.H, ffn)
    rows = cache["rows"]
    hist = np.setdiff1d(np.arange(b.T), rows)
    assert np.all(dE[hist] == 0.0)
    assert np.all(np.any(dE[rows] != 0.0, axis=1))
    if not ffn:
        dz = (1.0 / (1.0 + np.exp(-z)) - b.labels) / len(z)
        assert np.allclose(dE[rows], dz[:, None] * mdl.w_head[None, :], rtol=1e-14, atol=0)


def test_zero_head_gives_ln2_and_no_gradient():
    cfg, b, mdl, E, pos = _random_model(True, 2, seed=6)
    w0 = np.zeros_like(mdl.w_head)
    z, cache = oracle.block_forward(E, mdl.layers, w0, b.seq_offsets, b.hist_len, pos, b.ts,
                                    cfg.H, True)
    assert np.all(z == 0.0)
    assert oracle.bce_loss(z, b.labels) == math.log(2.0)
    dE = oracle.block_backward(z, b.labels, cache, mdl.layers, w0, b.seq_offsets, b.hist_len,
                               pos, b.ts, cfg.H, True)
    assert np.all(dE == 0.0)


# ------------------------------------------------------------------------------------------
# planted mistakes: mutated copies of the oracle's own source must fail the pins
# ------------------------------------------------------------------------------------------
def _mutant(edits):
    """Copies of the oracle's _rms, block_forward and bce_loss with ``edits``
    ((old, new) source replacements, each of which must apply) in a private namespace."""
    ns = dict(vars(og))
    for fn in (og._rms, og.block_forward, og.bce_loss):
        src = inspect.getsource(fn)
        for old, new in edits:
            src = src.replace(old, new)
        exec(compile(src, f"<mutant {fn.__name__}>", "exec"), ns)
    applied = all(any(old in inspect.getsource(f) for f in (og._rms, og.block_forward,
                                                          og.bce_loss)) for old, _ in edits)
    assert applied, "a planted edit no longer matches the oracle source"
    return ns


MUTANTS = {
    "rms sum for mean": [("(x * x).mean(axis=-1", "(x * x).sum(axis=-1")],
    "eps outside the root": [("np.sqrt((x * x).mean(axis=-1, keepdims=True) + RMS_EPS)",
                              "(np.sqrt((x * x).mean(axis=-1, keepdims=True)) + RMS_EPS)")],
    "dropped final norm": [("xf, rf = _rms(x)", "xf, rf = x, None")],
    "dropped attention residual": [('x = x + O.reshape(T, d) @ f(L["Wo"])',
                                    'x = O.reshape(T, d) @ f(L["Wo"])')],
    "dropped FFN residual": [('x = x + U @ f(L["W2"])', 'x = U @ f(L["W2"])')],
    "sigmoid for SiLU": [("U = G * _sigmoid(G)", "U = _sigmoid(G)")],
    "FFN without its pre-norm": [("fa, r2 = _rms(x)", "fa, r2 = x, 1.0")],
}


def _pins_hold(ns, golden):
    zb, _ = _example_b(ns["block_forward"])
    za = _example_a(ns["block_forward"])
    ok = abs(zb[0] - _g(golden, "B_z")[0]) <= 1e-14 and abs(za[0] - _g(golden, "A_z")[0]) <= 1e-15
    cfg, b, mdl, E, pos = _random_model(True, 2)
    z, _ = ns["block_forward"](E, mdl.layers, mdl.w_head, b.seq_offsets, b.hist_len, pos, b.ts,
                               cfg.H, True)
    zt = _torch_logits(E, mdl.layers, mdl.w_head, b.seq_offsets, b.hist_len, pos, b.ts, cfg.H, True)
    return ok and np.max(np.abs(z - zt)) <= 1e-12 * max(1.0, np.max(np.abs(zt)))


def test_unmutated_copy_passes(golden):
    assert _pins_hold(_mutant([]), golden)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_block_mistake_is_caught(golden, name):
    assert not _pins_hold(_mutant(MUTANTS[name]), golden)


@pytest.mark.parametrize("edit", [("np.mean(np.logaddexp", "np.sum(np.logaddexp"),
                                  ("- y * z", "+ y * z")])
def test_planted_loss_mistake_is_caught(golden, edit):
    bad = _mutant([edit])["bce_loss"]
    z, y = _g(golden, "bce_z"), _g(golden, "bce_y")
    assert abs(bad(z, y) - _g(golden, "bce_value")[0]) > 1e-6
