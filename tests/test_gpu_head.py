"""Candidate-side calls: the fused candidate head (genrank_candidate_logits) against a
float64 host sum of the same inputs, and the candidate-row gather (genrank_gather_rows)
against host indexing, bit for bit; with their argument and index checks."""

import numpy as np
import pytest
import torch

from generative_ranking_recommendation_b200 import genrank as G

pytestmark = pytest.mark.gpu


def _case(T, d, M, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, d, generator=g).to(dtype).cuda()
    o = torch.randn(T, d, generator=g).to(dtype).cuda()
    w = torch.randn(d, generator=g).cuda()
    u = torch.randn(d, generator=g).cuda()
    rows = torch.randint(0, T, (M,), generator=g, dtype=torch.int64).cuda()
    return rows, x, o, w, u


@pytest.mark.parametrize("dtype,d,M", [(torch.bfloat16, 256, 1000), (torch.bfloat16, 1024, 77),
                                       (torch.float32, 64, 513), (torch.bfloat16, 8, 5)])
def test_logits_match_host_sum(dtype, d, M):
    T = 3000
    rows, x, o, w, u = _case(T, d, M, dtype, 7 + d)
    z = torch.empty(M, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.candidate_logits(rows, x, o, w, u, z, err)
    assert G.check_error(err) == 0
    r = rows.cpu().numpy()
    ref = (x.double().cpu().numpy()[r] @ w.double().cpu().numpy()
           + o.double().cpu().numpy()[r] @ u.double().cpu().numpy())
    got = z.cpu().numpy()
    # fp32 accumulation of 2 d products of magnitude ~1
    assert np.max(np.abs(got - ref)) <= 1e-4 * (2 * d) ** 0.5 + 1e-5


def test_empty_and_bad_rows():
    T, d = 100, 64
    rows, x, o, w, u = _case(T, d, 4, torch.bfloat16, 1)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    z = torch.empty(4, dtype=torch.float32, device="cuda")
    G.candidate_logits(rows[:0], x, o, w, u, z, err)  # M = 0 launches nothing
    bad = torch.tensor([0, T, -1, 5], dtype=torch.int64, device="cuda")
    G.candidate_logits(bad, x, o, w, u, z, err)
    assert G.check_error(err) & G.DERR["INDEX"]
    zz = z.cpu().numpy()
    assert zz[1] == 0 and zz[2] == 0 and np.isfinite(zz).all()


def test_rejects_misaligned_width():
    T = 16
    rows, x, o, w, u = _case(T, 64, 3, torch.bfloat16, 2)
    z = torch.empty(3, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(G.GenRankError):
        G.candidate_logits(rows, x[:, :60], o[:, :60], w[:60], u[:60], z, err)


@pytest.mark.parametrize("dtype,d,M,T", [(torch.bfloat16, 512, 262_144, 753_664),
                                         (torch.float32, 512, 1000, 3000),
                                         (torch.bfloat16, 8, 33, 40)])
def test_gather_rows_bitwise(dtype, d, M, T):
    """The last block's candidate rows (the first case: the four-layer workload's
    1024 users x 256 candidates out of its 753 664 tokens), every row sampled at random
    with repeats."""
    g = torch.Generator(device="cuda").manual_seed(d + M)
    src = torch.randn((T, d), generator=g, device="cuda").to(dtype)
    rows = torch.randint(0, T, (M,), generator=g, device="cuda", dtype=torch.int64)
    dst = torch.full((M, d), float("nan"), dtype=dtype, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.gather_rows(rows, src, dst, err)
    assert G.check_error(err) == 0
    want = src.cpu().numpy()[rows.cpu().numpy()] if dtype == torch.float32 else None
    if want is None:  # compare bf16 bit patterns
        a = dst.view(torch.int16).cpu().numpy()
        b = src.view(torch.int16).cpu().numpy()[rows.cpu().numpy()]
        assert np.array_equal(a, b)
    else:
        assert np.array_equal(dst.cpu().numpy(), want)


def test_gather_rows_strided_and_bad_rows():
    """Rows of a wider matrix (a column slice with its row stride), an empty gather, and
    indices outside [0, T): flagged, their rows zeroed, the others copied."""
    T, d = 50, 64
    big = torch.randn((T, 3 * d), device="cuda").to(torch.bfloat16)
    src = big[:, d:2 * d]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dst = torch.full((4, d), 1.0, dtype=torch.bfloat16, device="cuda")
    G.gather_rows(torch.empty(0, dtype=torch.int64, device="cuda"), src, dst[:0], err)
    assert G.check_error(err) == 0
    bad = torch.tensor([3, T, -1, 7], dtype=torch.int64, device="cuda")
    G.gather_rows(bad, src, dst, err)
    assert G.check_error(err) & G.DERR["INDEX"]
    got = dst.float().cpu().numpy()
    ref = src.float().cpu().numpy()
    assert np.array_equal(got[0], ref[3]) and np.array_equal(got[3], ref[7])
    assert not got[1].any() and not got[2].any()
