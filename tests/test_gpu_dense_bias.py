"""GPU parity of the comparison path: attention with a dense per-user N x N bias on the
interleaved layout (genrank_attn_fwd_dense_bias) against the oracle's
``attention_fwd_dense_bias`` (fun-rec "The Overall Generative Ranking Paradigm" §7.2.0
and §7.2.2).  Tolerances as for the ALiBi forward: 2e-2 relative to the max with a
per-row bound for O (bf16), 2e-2 absolute for the LSE."""

import math

import numpy as np
import pytest
import torch

import oracle
import ref
from gen import CONFIGS, dense_bias_torch, interleave_batch, make_batch, make_qkv

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


def run_dense(G, cfg, batch, qkv, bias, poison=True):
    T, H, dh = batch.T, cfg.H, cfg.dh
    d = H * dh
    q = _dev(qkv.reshape(T, 3 * d), torch.bfloat16)
    o = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((H, T), dtype=torch.float32, device="cuda")
    msl = int(np.max(np.diff(batch.seq_offsets)))
    ws = torch.empty(G.attn_workspace_size(batch.B, T, H, dh, msl, False), dtype=torch.uint8,
                     device="cuda")
    if poison:
        ws.fill_(0xFF)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.attn_fwd_dense_bias(_dev(batch.seq_offsets), _dev(batch.hist_len), msl, q, q[:, d:],
                          q[:, 2 * d:], 3 * d, H, dh, bias, 1.0 / math.sqrt(dh), o, d, lse, ws,
                          err, T=T)
    assert G.check_error(err) == 0
    return (o.float().cpu().numpy().astype(np.float64).reshape(T, H, dh),
            lse.cpu().numpy().astype(np.float64))


def _check(O, L, Or, Lr):
    assert ref.rel_to_max(O, Or) <= BF16_TOL
    den = np.maximum(np.abs(Or).max(axis=(1, 2)), 0.25)
    assert np.max(np.abs(O - Or).max(axis=(1, 2)) / den) <= BF16_TOL
    assert np.max(np.abs(L - Lr)) <= 2e-2


@pytest.mark.parametrize("std", [0.5, 4.0])
def test_dense_bias_parity_interleaved(G, std):
    """HSTU-shaped inputs: history interactions as token pairs, ragged users, a dense
    bias (std 4 exercises the offset redo path)."""
    cfg = CONFIGS["c1"].with_(B=7, H=2)
    base = make_batch(cfg, hist_override=[100, 0, 64, 1, 190, 63, 5],
                      m_override=[20, 3, 0, 129, 1, 2, 128])
    batch = interleave_batch(base)
    Lpad = 512
    assert int(np.max(np.diff(batch.seq_offsets))) <= Lpad
    bias = dense_bias_torch(71, batch.B, Lpad, "cuda", std=std)
    qkv = make_qkv(cfg, batch.T, seed=72)
    O, L = run_dense(G, cfg, batch, qkv, bias)
    Or, Lr = oracle.attention_fwd_dense_bias(qkv[:, 0], qkv[:, 1], qkv[:, 2], batch.seq_offsets,
                                             batch.hist_len, bias.float().cpu().numpy(),
                                             1.0 / math.sqrt(cfg.dh))
    _check(O, L, Or, Lr)


def test_dense_bias_holding_alibi_matches_the_alibi_kernel(G):
    """One head, the dense bias filled with that head's ALiBi values (rounded to bf16):
    the dense-bias kernel and the ALiBi kernel agree within the bf16 bias rounding."""
    from test_gpu_attention import run_fwd

    cfg = CONFIGS["c1"].with_(B=3, H=1)
    batch = make_batch(cfg, hist_override=[200, 17, 129], m_override=[40, 3, 130])
    pos, _, _ = ref.meta(batch)
    qkv = make_qkv(cfg, batch.T, seed=73)
    sp, st = ref.slopes(1)
    Lpad = 384
    b = np.zeros((batch.B, Lpad, Lpad), np.float32)
    for u in range(batch.B):
        s, e = int(batch.seq_offsets[u]), int(batch.seq_offsets[u + 1])
        p, t = pos[s:e].astype(np.float64), batch.ts[s:e].astype(np.float64)
        b[u, :e - s, :e - s] = -sp[0] * np.abs(p[:, None] - p[None]) - st[0] * np.abs(
            t[:, None] - t[None])
    bias = torch.from_numpy(b).to("cuda", torch.bfloat16)
    O, L = run_dense(G, cfg, batch, qkv, bias)
    Of, Lf = run_fwd(G, cfg, batch, pos, qkv)
    assert ref.rel_to_max(O, Of) <= BF16_TOL
    Or, Lr = oracle.attention_fwd_dense_bias(qkv[:, 0], qkv[:, 1], qkv[:, 2], batch.seq_offsets,
                                             batch.hist_len, bias.float().cpu().numpy(),
                                             1.0 / math.sqrt(cfg.dh))
    _check(O, L, Or, Lr)
