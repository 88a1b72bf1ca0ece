"""The C ABI library without a GPU: it loads, exports every declared entry point,
and its host-only calls and host-side argument checks behave as documented."""

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "genrank.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(genrank_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    from generative_ranking_recommendation_b200 import genrank as G
    from generative_ranking_recommendation_b200.csrc import build

    build.build()
    return G.lib()


def test_every_declared_symbol_is_exported(L):
    from generative_ranking_recommendation_b200 import genrank as G

    names = _declared()
    assert len(names) >= 9
    assert sorted(G.EXPORTS) == names
    out = subprocess.run(["nm", "-D", "--defined-only", G.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (genrank_\w+)", out))
    for n in names:
        assert n in exported, n
        assert hasattr(L, n)


def test_alibi_slopes_host_call(L):
    from generative_ranking_recommendation_b200 import genrank as G

    sp, st = G.alibi_slopes(8)
    assert [1.0 / x for x in sp] == [2, 4, 8, 16, 32, 64, 128, 256]
    assert np.allclose(np.array(st) * 3600.0, sp, rtol=1e-6)


def test_status_strings(L):
    from generative_ranking_recommendation_b200 import genrank as G

    assert G.status_string(0) == "ok"
    assert "invalid" in G.status_string(1)
    assert "workspace" in G.status_string(3)
    assert G.device_error_string(0) == "clean"
    assert "timed out" in G.device_error_string(G.DERR["TIMEOUT"])


def test_workspace_size_host_call(L):
    from generative_ranking_recommendation_b200 import genrank as G

    n = G.attn_workspace_size(256, 100000, 4, 64, 608, False)
    assert n >= 256 * 5 * 4
    nb = G.attn_workspace_size(256, 100000, 4, 64, 608, True)
    assert nb >= 100000 * 4 * 4
    assert G.attn_workspace_size(0, 10, 4, 64, 10, False) == 0


def test_host_side_argument_checks_return_before_launch(L):
    """Invalid arguments are rejected on the host, without touching a GPU."""
    P = ctypes.c_void_p
    fake = P(0x10000)  # never dereferenced: every call below fails its host checks
    sp = (ctypes.c_float * 4)(0.5, 0.25, 0.125, 0.0625)
    st = (ctypes.c_float * 4)(*(x / 3600 for x in sp))
    base = dict(B=1, T=10, off=fake, hl=fake, msl=10, q=fake, k=fake, v=fake, stride=768, H=4,
                dh=64, pos=fake, ts=fake, scale=0.125, dtype=1, o=fake, ostride=256, lse=None,
                ws=fake, wsb=1 << 20, err=fake)

    def call(**kw):
        a = dict(base)
        a.update(kw)
        return L.genrank_attn_fwd(a["B"], a["T"], a["off"], a["hl"], a["msl"], a["q"], a["k"],
                                  a["v"], a["stride"], a["H"], a["dh"], a["pos"], a["ts"],
                                  ctypes.cast(sp, P), ctypes.cast(st, P), a["scale"], a["dtype"],
                                  a["o"], a["ostride"], a["lse"], a["ws"], a["wsb"], a["err"], None)

    assert call(B=0) == 1
    assert call(off=None) == 1
    assert call(scale=0.0) == 1
    assert call(stride=100) == 1  # not a multiple of 16 bytes / smaller than H*dh
    assert call(q=P(0x10008)) == 1  # misaligned base
    assert call(dtype=7) == 1
    assert call(dh=48, stride=192, ostride=192) == 2  # bf16 head dim 48: unsupported
    assert call(ws=None) == 3
    assert call(wsb=16) == 3
    # embedding: bad table sizes and misaligned rows
    r = L.genrank_embed_assemble(1, 10, fake, fake, fake, fake, fake, fake, 100, fake, 8, fake,
                                 600, fake, 128, fake, 64, 12, 1, fake, fake, fake, fake, fake,
                                 None)
    assert r == 1  # 12 bf16 = 24 bytes per row: not a multiple of 16
    r = L.genrank_embed_assemble(1, 10, fake, fake, fake, fake, fake, fake, 100, fake, 8, fake,
                                 600, fake, 128, fake, 80, 64, 1, fake, fake, fake, fake, fake,
                                 None)
    assert r == 2  # 80 time buckets: beyond what the integer bucket supports


def test_gather_rows_host_checks(L):
    """The candidate-row gather rejects bad sizes and alignment on the host."""
    P = ctypes.c_void_p
    fake = P(0x10000)  # never dereferenced: every call below fails its host checks

    def call(M=4, rows=fake, T=10, rb=1024, src=fake, ss=1024, dst=fake, ds=1024, err=fake):
        return L.genrank_gather_rows(M, rows, T, rb, src, ss, dst, ds, err, None)

    assert call(M=-1) == 1
    assert call(rb=0) == 1
    assert call(rb=24, ss=32, ds=32) == 1  # not a multiple of 16 bytes
    assert call(ss=512) == 1  # src stride shorter than a row
    assert call(ds=1040 + 8) == 1  # dst stride not a multiple of 16
    assert call(src=P(0x10008)) == 1  # misaligned
    assert call(rows=None) == 1
    assert call(err=None) == 1
    assert call(M=0, rows=None, src=None, dst=None) == 0  # nothing to do


def test_backward_workspace_covers_its_regions(L):
    """The backward scratch holds the fp32 dQ accumulator [T, H, 64], three fp32 per-row
    arrays [H, T] (column term, log2 LSE, D) and an 8-byte record per token."""
    from generative_ranking_recommendation_b200 import genrank as G

    B, T, H, dh, msl = 256, 100000, 4, 64, 608
    nb = G.attn_workspace_size(B, T, H, dh, msl, True)
    assert nb >= T * H * dh * 4 + 3 * H * T * 4 + T * 8
    # grows with every token by at least those bytes
    nb2 = G.attn_workspace_size(B, T + 1000, H, dh, msl, True)
    assert nb2 - nb >= 1000 * (H * dh * 4 + 3 * H * 4 + 8)


def test_backward_host_side_argument_checks(L):
    """Invalid backward arguments are rejected on the host, without touching a GPU."""
    P = ctypes.c_void_p
    fake = P(0x10000)  # never dereferenced: every call below fails its host checks
    sp = (ctypes.c_float * 4)(0.5, 0.25, 0.125, 0.0625)
    st = (ctypes.c_float * 4)(*(x / 3600 for x in sp))
    base = dict(B=1, T=10, off=fake, hl=fake, msl=10, q=fake, k=fake, v=fake, stride=768, H=4,
                dh=64, pos=fake, ts=fake, scale=0.125, dtype=1, o=fake, dO=fake, ostride=256,
                lse=fake, dq=fake, dk=fake, dv=fake, ws=fake, wsb=1 << 20, err=fake)

    def call(**kw):
        a = dict(base)
        a.update(kw)
        return L.genrank_attn_bwd(a["B"], a["T"], a["off"], a["hl"], a["msl"], a["q"], a["k"],
                                  a["v"], a["stride"], a["H"], a["dh"], a["pos"], a["ts"],
                                  ctypes.cast(sp, P), ctypes.cast(st, P), a["scale"], a["dtype"],
                                  a["o"], a["dO"], a["ostride"], a["lse"], a["dq"], a["dk"],
                                  a["dv"], a["ws"], a["wsb"], a["err"], None)

    assert call(B=0) == 1
    assert call(dO=None) == 1
    assert call(lse=None) == 1  # the backward needs the forward's LSE
    assert call(dq=P(0x10008)) == 1  # misaligned output
    assert call(dtype=7) == 1
    assert call(dh=48, stride=192, ostride=192) == 2
    assert call(ws=None) == 3
    assert call(wsb=16) == 3



def test_candidates_and_fused_embedding_host_checks(L):
    """The candidate-only attention and the gather-sum with the first RMSNorm reject bad
    arguments on the host; the candidate workspace covers the cached form's."""
    P = ctypes.c_void_p
    fake = P(0x10000)
    sp = (ctypes.c_float * 4)(0.5, 0.25, 0.125, 0.0625)
    st = (ctypes.c_float * 4)(*(x / 3600 for x in sp))

    def cand(**kw):
        a = dict(B=1, T=10, off=fake, hl=fake, msl=10, q=fake, k=fake, v=fake, stride=768, H=4,
                 dh=64, pos=fake, ts=fake, scale=0.125, dtype=1, o=fake, ostride=256, lse=None,
                 ws=fake, wsb=1 << 20, err=fake)
        a.update(kw)
        return L.genrank_attn_fwd_candidates(
            a["B"], a["T"], a["off"], a["hl"], a["msl"], a["q"], a["k"], a["v"], a["stride"],
            a["H"], a["dh"], a["pos"], a["ts"], ctypes.cast(sp, P), ctypes.cast(st, P),
            a["scale"], a["dtype"], a["o"], a["ostride"], a["lse"], a["ws"], a["wsb"], a["err"],
            None)

    assert cand(B=0) == 1
    assert cand(hl=None) == 1
    assert cand(o=P(0x10008)) == 1
    assert cand(dtype=0, stride=768, ostride=256) == 2  # fp32: the tensor-core kernel only
    assert cand(ws=None) == 3
    assert cand(wsb=16) == 3
    n = L.genrank_attn_candidates_workspace_size(64, 100000, 16, 64, 1504)
    assert n == L.genrank_attn_cached_workspace_size(64, 100000, 100000, 16, 64, 1504) > 0
    assert L.genrank_attn_candidates_workspace_size(0, 10, 4, 64, 10) == 0

    def emb(d=512, eps=1e-6, x=fake, a=fake, n_rt=64):
        return L.genrank_embed_assemble_rmsnorm(1, 10, fake, fake, fake, fake, fake, fake, 100,
                                                fake, 8, fake, 600, fake, 128, fake, n_rt, d, x,
                                                a, eps, fake, fake, fake, fake, None)

    assert emb(d=256) == 2  # the fused form takes d = 512 only
    assert emb(eps=-1.0) == 1
    assert emb(x=None) == 1
    assert emb(a=P(0x10008)) == 1
    assert emb(n_rt=80) == 2
