"""GPU parity of the tensor-core linear layers with fused epilogues (genrank_linear,
genrank_linear_residual_rmsnorm, genrank_rmsnorm) against float64 host references
of the same operations (bf16 inputs upcast exactly; the four-layer workload's block:
pre-RMSNorm with eps 1e-6 and unit gain, 4d SiLU FFN, fp32 residual stream).

Tolerances: bf16 outputs 2e-2 relative to the max with a per-row bound (one bf16
rounding of an fp32 sum), fp32 residual rows 1e-3 relative to the max (fp32
accumulation of K bf16 products), logits 2e-2 relative to the max.
"""

import numpy as np
import pytest
import torch

import ref

pytestmark = pytest.mark.gpu

EPS = 1e-6


@pytest.fixture(scope="module")
def G():
    from generative_ranking_recommendation_b200 import genrank
    from generative_ranking_recommendation_b200.csrc import build

    build.build()
    genrank.lib()
    return genrank


def _bf(shape, seed, std=1.0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return (torch.randn(shape, generator=g, device="cuda") * std).to(torch.bfloat16)


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


def _rms(x):
    return x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + EPS)


def _rows_ok(got, want, tol=2e-2):
    assert ref.rel_to_max(got, want) <= tol
    err = np.abs(got - want).max(axis=1)
    den = np.maximum(np.abs(want).max(axis=1), np.abs(want).max() / 16.0)
    assert np.max(err / den) <= tol, int(np.argmax(err / den))


@pytest.mark.parametrize("M,N,K,epi", [(1000, 1536, 512, 0), (129, 256, 64, 0),
                                       (4097, 2048, 512, 1), (1, 512, 2048, 1),
                                       (255, 512, 128, 0), (257, 256, 192, 1)])
def test_linear_parity(G, M, N, K, epi):
    A = _bf((M, K), 1, 1.0)
    Wt = _bf((N, K), 2, 1.0 / np.sqrt(K))
    C = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.linear(A, Wt, C, err, epilogue=epi)
    assert G.check_error(err) == 0
    want = _np(A) @ _np(Wt).T
    if epi == 1:
        want = want / (1.0 + np.exp(-want))
    _rows_ok(_np(C), want)


@pytest.mark.parametrize("M,K,head", [(1000, 512, False), (300, 2048, True), (128, 512, True)])
def test_linear_residual_rmsnorm_parity(G, M, K, head):
    d = 512
    A = _bf((M, K), 3, 1.0)
    Wt = _bf((d, K), 4, 1.0 / np.sqrt(K))
    x = torch.randn((M, d), generator=torch.Generator(device="cuda").manual_seed(5),
                    device="cuda")
    x_np = x.double().cpu().numpy()
    a_out = torch.full((M, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    w = torch.randn(d, generator=torch.Generator(device="cuda").manual_seed(6), device="cuda")
    z = torch.full((M,), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.linear_residual_rmsnorm(A, Wt, x, x, a_out, err, w_head=w if head else None,
                              z=z if head else None)  # in place: x_out aliases x_in
    assert G.check_error(err) == 0
    xo = x_np + _np(A) @ _np(Wt).T
    assert ref.rel_to_max(x.double().cpu().numpy(), xo) <= 1e-3
    _rows_ok(_np(a_out), _rms(xo))
    if head:
        assert ref.rel_to_max(z.double().cpu().numpy(), _rms(xo) @ w.double().cpu().numpy()) <= 2e-2


@pytest.mark.parametrize("M,N,epi", [(20001, 1536, 0), (12345, 2048, 1)])
def test_linear_many_tiles(G, M, N, epi):
    """More 256-row tiles than SM pairs, so every pair runs several tiles through both
    accumulator buffers and the operand ring wraps many times; ragged last tile."""
    K = 512
    A = _bf((M, K), 5, 1.0)
    Wt = _bf((N, K), 6, 1.0 / np.sqrt(K))
    C = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.linear(A, Wt, C, err, epilogue=epi)
    assert G.check_error(err) == 0
    want = _np(A) @ _np(Wt).T
    if epi == 1:
        want = want / (1.0 + np.exp(-want))
    _rows_ok(_np(C), want)


@pytest.mark.parametrize("M,K", [(50_000, 512), (40_001, 2048)])
def test_linear_residual_rmsnorm_many_tiles(G, M, K):
    """Several row tiles per CTA (each CTA of the persistent grid loads its next tile's
    residual rows while finishing the current one), out of place, with the head; the
    float64 reference runs on the device."""
    d = 512
    A = _bf((M, K), 7, 1.0)
    Wt = _bf((d, K), 8, 1.0 / np.sqrt(K))
    x = torch.randn((M, d), generator=torch.Generator(device="cuda").manual_seed(9),
                    device="cuda")
    x0 = x.clone()
    xo = torch.full_like(x, float("nan"))
    a_out = torch.full((M, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    w = torch.randn(d, generator=torch.Generator(device="cuda").manual_seed(10), device="cuda")
    z = torch.full((M,), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.linear_residual_rmsnorm(A, Wt, x, xo, a_out, err, w_head=w, z=z)
    assert G.check_error(err) == 0
    assert torch.equal(x, x0)
    want = x.double() + A.double() @ Wt.double().T
    got = xo.double()
    assert float((got - want).abs().max() / want.abs().max()) <= 1e-3
    nrm = want / torch.sqrt((want * want).mean(dim=1, keepdim=True) + EPS)
    an = a_out.double()
    err_r = (an - nrm).abs().max(dim=1).values
    den = torch.clamp(nrm.abs().max(dim=1).values, min=float(nrm.abs().max()) / 16.0)
    assert float((err_r / den).max()) <= 2e-2
    zw = nrm @ w.double()
    assert float((z.double() - zw).abs().max() / zw.abs().max()) <= 2e-2


def test_linear_residual_rmsnorm_head_only(G):
    """The last block's form: no normalised rows written, only the head's logits."""
    M, K, d = 333, 2048, 512
    A = _bf((M, K), 11, 1.0)
    Wt = _bf((d, K), 12, 1.0 / np.sqrt(K))
    x = torch.randn((M, d), generator=torch.Generator(device="cuda").manual_seed(13),
                    device="cuda")
    x_np = x.double().cpu().numpy()
    xo = torch.empty_like(x)
    w = torch.randn(d, generator=torch.Generator(device="cuda").manual_seed(14), device="cuda")
    z = torch.full((M,), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.linear_residual_rmsnorm(A, Wt, x, xo, None, err, w_head=w, z=z)
    assert G.check_error(err) == 0
    want = x_np + _np(A) @ _np(Wt).T
    assert ref.rel_to_max(xo.double().cpu().numpy(), want) <= 1e-3
    zw = _rms(want) @ w.double().cpu().numpy()
    assert ref.rel_to_max(z.double().cpu().numpy(), zw) <= 2e-2


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_rmsnorm_parity(G, dtype):
    M, d = 777, 512
    x = torch.randn((M, d), generator=torch.Generator(device="cuda").manual_seed(7),
                    device="cuda").to(dtype)
    a = torch.empty((M, d), dtype=torch.bfloat16, device="cuda")
    xo = torch.empty((M, d), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.rmsnorm(x, a, err, x_out=xo)
    assert G.check_error(err) == 0
    xn = x.double().cpu().numpy()
    assert np.array_equal(xo.double().cpu().numpy(), xn)
    _rows_ok(_np(a), _rms(xn))
