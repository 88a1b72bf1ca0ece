"""Pins for the oracle's comparison path: the interleaved layout (two tokens per history
interaction) and attention with a dense per-user N x N bias (fun-rec "The Overall
Generative Ranking Paradigm" §7.2.0 and §7.2.2; "GenRank [2025]" §1.4.2)."""

import math

import numpy as np
import torch
import torch.nn.functional as F

import oracle


def _case(seed=0, users=((5, 3), (1, 2), (7, 1), (4, 0), (0, 2)), H=2, dh=4, Lpad=16):
    rng = np.random.default_rng(seed)
    offs = np.zeros(len(users) + 1, np.int64)
    offs[1:] = np.cumsum([n + m for n, m in users])
    T = int(offs[-1])
    q, k, v = (rng.normal(size=(T, H, dh)) for _ in range(3))
    bias = rng.normal(0, 0.7, size=(len(users), Lpad, Lpad))
    return dict(q=q, k=k, v=v, offs=offs, hl=np.array([n for n, _ in users]), bias=bias,
                scale=1.0 / math.sqrt(dh))


def test_interleaved_layout_lengths(golden):
    # the pages' worked example: 800 history interactions take 1600 tokens interleaved
    g = golden("sequence_length_example.txt")
    n_c = int(g["n_c"][0])
    off, hl = oracle.interleaved_layout(np.array([0, n_c]), np.array([n_c]))
    assert int(hl[0]) == int(g["interleaved_tokens"][0]) and int(off[-1]) == 2 * n_c
    # (n, m) = (5, 3), (1, 2), (0, 0): 2n + m = 13, 4, 0 tokens
    off, hl = oracle.interleaved_layout(np.array([0, 8, 11, 11]), np.array([5, 1, 0]))
    assert off.tolist() == [0, 13, 17, 17] and hl.tolist() == [10, 2, 0]


def test_dense_bias_matches_torch_sdpa():
    x = _case()
    O, L = oracle.attention_fwd_dense_bias(x["q"], x["k"], x["v"], x["offs"], x["hl"], x["bias"],
                                           x["scale"])
    for u in range(len(x["hl"])):
        s, e, n = int(x["offs"][u]), int(x["offs"][u + 1]), int(x["hl"][u])
        if e == s:
            continue
        mask = oracle.attention_mask(n, e - s)
        add = torch.from_numpy(np.where(mask, x["bias"][u][:e - s, :e - s], -np.inf))
        tq, tk, tv = (torch.from_numpy(x[c][s:e]).transpose(0, 1)[None] for c in "qkv")
        o = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=add, scale=x["scale"])
        assert np.max(np.abs(o[0].transpose(0, 1).numpy() - O[s:e])) <= 1e-12
        S = np.einsum("ihd,jhd->hij", x["q"][s:e], x["k"][s:e]) * x["scale"] + np.where(
            mask, x["bias"][u][:e - s, :e - s], -np.inf)[None]
        lse = np.log(np.exp(S - S.max(-1, keepdims=True)).sum(-1)) + S.max(-1)
        assert np.max(np.abs(lse - L[:, s:e])) <= 1e-12


def test_dense_bias_equal_to_alibi_reduces_to_attention_fwd():
    """A dense bias that holds the ALiBi values of one head gives that head's
    attention_fwd exactly (up to rounding)."""
    rng = np.random.default_rng(3)
    users = ((6, 2), (3, 3), (1, 1))
    offs = np.zeros(len(users) + 1, np.int64)
    offs[1:] = np.cumsum([n + m for n, m in users])
    hl = np.array([n for n, _ in users])
    T = int(offs[-1])
    ts = []
    for n, m in users:
        t = 1_700_000_000 + int(rng.integers(0, 100))
        row = []
        for i in range(n):
            t += int(rng.integers(0, 500)) if i else 0
            row.append(t)
        ts += row + [t + 77] * m
    ts = np.array(ts, np.int64)
    pos, _, _ = oracle.token_metadata(offs, hl, ts)
    q, k, v = (rng.normal(size=(T, 1, 8)) for _ in range(3))
    sp = np.array([0.3])
    st = np.array([0.002])
    Lpad = 12
    bias = np.zeros((len(users), Lpad, Lpad))
    for u in range(len(users)):
        s, e = int(offs[u]), int(offs[u + 1])
        p, t = pos[s:e].astype(np.float64), ts[s:e].astype(np.float64)
        bias[u, :e - s, :e - s] = -sp[0] * np.abs(p[:, None] - p[None]) - st[0] * np.abs(
            t[:, None] - t[None])
    O1, L1 = oracle.attention_fwd_dense_bias(q, k, v, offs, hl, bias, 1 / math.sqrt(8))
    O2, L2 = oracle.attention_fwd(q, k, v, offs, hl, pos, ts, sp, st, 1 / math.sqrt(8))
    assert np.max(np.abs(O1 - O2)) <= 1e-12 and np.max(np.abs(L1 - L2)) <= 1e-12


def test_dense_bias_reads_only_the_users_own_block():
    """Entries outside a user's L x L block (and masked entries inside it) do not matter."""
    x = _case(seed=5)
    O, L = oracle.attention_fwd_dense_bias(x["q"], x["k"], x["v"], x["offs"], x["hl"], x["bias"],
                                           x["scale"])
    b2 = x["bias"].copy()
    for u in range(len(x["hl"])):
        Lu = int(x["offs"][u + 1] - x["offs"][u])
        b2[u, Lu:, :] = 1e9
        b2[u, :, Lu:] = -1e9
        mask = oracle.attention_mask(int(x["hl"][u]), Lu)
        blk = b2[u, :Lu, :Lu]
        blk[~mask] = 123.0
    O2, L2 = oracle.attention_fwd_dense_bias(x["q"], x["k"], x["v"], x["offs"], x["hl"], b2,
                                             x["scale"])
    assert np.array_equal(O, O2) and np.array_equal(L, L2)


def test_planted_transposed_bias_is_caught():
    """Reading bias[u][j][i] instead of bias[u][i][j] must fail the SDPA pin."""
    x = _case(seed=9)
    bt = np.transpose(x["bias"], (0, 2, 1))
    O, _ = oracle.attention_fwd_dense_bias(x["q"], x["k"], x["v"], x["offs"], x["hl"], bt,
                                           x["scale"])
    O_ok, _ = oracle.attention_fwd_dense_bias(x["q"], x["k"], x["v"], x["offs"], x["hl"],
                                              x["bias"], x["scale"])
    assert np.max(np.abs(O - O_ok)) > 1e-3


def test_generator_interleaving_matches_the_oracle_layout():
    from gen import CONFIGS, interleave_batch, make_batch

    b = make_batch(CONFIGS["c1"].with_(B=5), hist_override=[3, 0, 7, 1, 2],
                   m_override=[2, 4, 0, 1, 3])
    hb = interleave_batch(b)
    off, hl = oracle.interleaved_layout(b.seq_offsets, b.hist_len)
    assert hb.seq_offsets.tolist() == off.tolist() and hb.hist_len.tolist() == hl.tolist()
    # history interactions occupy token pairs at one time; candidates keep theirs
    for u in range(b.B):
        s, n = int(hb.seq_offsets[u]), int(hb.hist_len[u])
        s0, n0 = int(b.seq_offsets[u]), int(b.hist_len[u])
        assert np.array_equal(hb.ts[s:s + n:2], b.ts[s0:s0 + n0])
        assert np.array_equal(hb.ts[s + 1:s + n:2], b.ts[s0:s0 + n0])
        assert np.array_equal(hb.item_ids[s:s + n:2], b.item_ids[s0:s0 + n0])
        assert np.array_equal(hb.ts[s + n:int(hb.seq_offsets[u + 1])],
                              b.ts[s0 + n0:int(b.seq_offsets[u + 1])])
