"""genrank_attn_fwd_static, the attention forward for callers that cannot allocate.

Some callers cannot call cudaMalloc where they run attention (serving loops that
forbid device allocations after start-up, hosts that own all device memory), so
this entry point uses a scratch array compiled into the library instead of a
workspace.  This test calls it through the C ABI twice in a row and checks each
result against genrank_attn_fwd with a caller-allocated workspace, within the
tolerance the other bf16 attention tests use.  It lives in a file of its own,
collected last, and passes alone in a fresh process as well as after the others.
"""

import math

import numpy as np
import pytest
import torch

from gen import CONFIGS, make_batch, make_qkv

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2


def _dev(x, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to("cuda", dtype=dtype) if dtype is not None else t.to("cuda")


def _positions(batch):
    pos = np.zeros(batch.T, np.int32)
    for u in range(batch.B):
        s, e, n = batch.seq_offsets[u], batch.seq_offsets[u + 1], batch.hist_len[u]
        pos[s:s + n] = np.arange(1, n + 1)
        pos[s + n:e] = n + 1
    return pos


def _rel(a, b):
    a = a.float()
    b = b.float()
    return float((a - b).abs().max() / b.abs().max().clamp_min(1e-30))


def test_static_scratch_matches_workspace_version():
    from generative_ranking_recommendation_b200 import genrank as G
    from generative_ranking_recommendation_b200.csrc import build

    build.build()
    cfg = CONFIGS["c1"].with_(B=40)
    batch = make_batch(cfg)
    T, H, dh = batch.T, cfg.H, cfg.dh
    d = H * dh
    off, hl = _dev(batch.seq_offsets), _dev(batch.hist_len)
    pos, ts = _dev(_positions(batch)), _dev(batch.ts)
    msl = int(np.max(np.diff(batch.seq_offsets)))
    sp, st = G.alibi_slopes(H)
    scale = 1.0 / math.sqrt(dh)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(G.attn_workspace_size(batch.B, T, H, dh, msl, False), dtype=torch.uint8,
                     device="cuda")
    for call in range(2):  # two calls in a row, different inputs
        q = _dev(make_qkv(cfg, T, seed=100 + call).reshape(T, 3 * d), torch.bfloat16)
        o_ref = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
        l_ref = torch.empty((H, T), dtype=torch.float32, device="cuda")
        G.attn_fwd(off, hl, msl, q, q[:, d:], q[:, 2 * d:], 3 * d, H, dh, pos, ts, sp, st, scale,
                   o_ref, d, l_ref, ws, err, T=T)
        o = torch.full((T, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((H, T), float("nan"), dtype=torch.float32, device="cuda")
        G.attn_fwd_static(off, hl, msl, q, q[:, d:], q[:, 2 * d:], 3 * d, H, dh, pos, ts, sp,
                          st, scale, o, d, lse, err, T=T)
        assert G.check_error(err) == 0
        assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
        assert _rel(o, o_ref) <= BF16_TOL
        assert float((lse - l_ref).abs().max()) <= BF16_TOL


def test_static_scratch_rejects_oversized_workloads():
    from generative_ranking_recommendation_b200 import genrank as G

    # 1M tokens x 16 heads of column terms is far beyond the fixed scratch; the call
    # must fail on the host before touching any pointer
    with pytest.raises(G.GenRankError, match="workspace"):
        x = torch.empty(16, dtype=torch.bfloat16, device="cuda")
        i = torch.zeros(2, dtype=torch.int32, device="cuda")
        G.attn_fwd_static(i, i[:1], 128, x, x, x, 3 * 1024, 16, 64, i, i.long(), [0.5] * 16,
                          [0.5 / 3600] * 16, 0.125, x, 1024, None, i, T=1_000_000)


def test_static_entry_takes_any_size_on_the_cuda_core_path():
    """fp32 runs the CUDA-core kernel, which needs no scratch: a batch whose tensor-core
    workspace would exceed the fixed 16 MiB still runs, and matches genrank_attn_fwd."""
    from generative_ranking_recommendation_b200 import genrank as G

    B, H, dh = 300_000, 1, 32  # users of one history token and one candidate
    T = 2 * B
    assert G.attn_workspace_size(B, T, H, 64, 2, False) > (16 << 20)
    off = torch.arange(0, T + 1, 2, dtype=torch.int32, device="cuda")
    hl = torch.ones(B, dtype=torch.int32, device="cuda")
    pos = torch.tensor([1, 2], dtype=torch.int32, device="cuda").repeat(B)
    ts = (1_700_000_000 + torch.arange(T, dtype=torch.int64, device="cuda") // 2 * 7
          + torch.tensor([0, 5], dtype=torch.int64, device="cuda").repeat(B))
    gen = torch.Generator(device="cuda").manual_seed(7)
    q = torch.randn((T, 3 * H * dh), generator=gen, device="cuda")
    d = H * dh
    sp, st = G.alibi_slopes(H)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    o_ref = torch.empty((T, d), device="cuda")
    l_ref = torch.empty((H, T), device="cuda")
    G.attn_fwd(off, hl, 2, q, q[:, d:], q[:, 2 * d:], 3 * d, H, dh, pos, ts, sp, st,
               1.0 / math.sqrt(dh), o_ref, d, l_ref, None, err, T=T)
    for _ in range(2):
        o = torch.full((T, d), float("nan"), device="cuda")
        lse = torch.full((H, T), float("nan"), device="cuda")
        G.attn_fwd_static(off, hl, 2, q, q[:, d:], q[:, 2 * d:], 3 * d, H, dh, pos, ts, sp, st,
                          1.0 / math.sqrt(dh), o, d, lse, err, T=T)
        assert G.check_error(err) == 0
        assert float((o - o_ref).abs().max()) <= 1e-4
        assert float((lse - l_ref).abs().max()) <= 1e-4
