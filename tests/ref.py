"""Oracle-side helpers for the GPU parity tests (host, float64; no GPU code)."""

import math

import numpy as np

import oracle


def compact_items(batch, model, users=None):
    """Item rows used by ``users`` and the batch's ids remapped into them."""
    ids = batch.item_ids
    if users is not None:
        sel = np.concatenate([np.arange(batch.seq_offsets[u], batch.seq_offsets[u + 1])
                              for u in users])
        uniq = np.unique(ids[sel])
    else:
        uniq = np.unique(ids)
    remap = np.full(batch.item_ids.shape, 0, np.int64)
    pos = np.searchsorted(uniq, ids)
    ok = (pos < len(uniq)) & (uniq[np.minimum(pos, len(uniq) - 1)] == ids)
    remap[ok] = pos[ok]
    return model.item_rows(uniq), remap


def meta(batch, users=None, cfg=None):
    c = batch.cfg if cfg is None else cfg
    return oracle.token_metadata(batch.seq_offsets, batch.hist_len, batch.ts, c.n_ri, c.n_rt,
                                 users=users)


def embed(batch, model, users=None):
    item, ids = compact_items(batch, model, users)
    m = meta(batch, users)
    E = oracle.embed_assemble(batch.seq_offsets, batch.hist_len, ids, batch.action_ids, m, item,
                              model.action_tab, model.pos_tab, model.ri_tab, model.rt_tab,
                              users=users)
    return E, m


def slopes(H):
    s = oracle.alibi_slopes(H)
    return s, s / 3600.0


def user_rows(batch, users):
    return np.concatenate([np.arange(batch.seq_offsets[u], batch.seq_offsets[u + 1])
                           for u in users])


def cand_rows(batch, users=None):
    users = range(batch.B) if users is None else users
    return np.concatenate([np.arange(batch.seq_offsets[u] + batch.hist_len[u],
                                     batch.seq_offsets[u + 1]) for u in users])


def rel_to_max(x, ref):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.max(np.abs(x - ref)) / max(np.max(np.abs(ref)), 1e-30))


def model_logits(batch, model, users):
    """Oracle logits at the candidates of ``users`` (the users are independent)."""
    cfg = batch.cfg
    sub = _sub_batch(batch, users)
    E, m = embed(sub, model)
    z, _ = oracle.block_forward(E, model.layers, model.w_head, sub.seq_offsets, sub.hist_len,
                                m[0], sub.ts, cfg.H, cfg.ffn)
    return z


def _sub_batch(batch, users):
    from gen.synth import Batch

    rows = user_rows(batch, users)
    lens = np.array([batch.seq_offsets[u + 1] - batch.seq_offsets[u] for u in users])
    off = np.zeros(len(users) + 1, np.int32)
    off[1:] = np.cumsum(lens)
    labels = None
    if batch.labels is not None:
        cr_all = cand_rows(batch)
        where = {r: k for k, r in enumerate(cr_all)}
        labels = batch.labels[[where[r] for r in cand_rows(batch, users)]]
    return Batch(batch.cfg, [batch.users[u] for u in users], off,
                 batch.hist_len[list(users)].copy(), batch.item_ids[rows].copy(),
                 batch.action_ids[rows].copy(), batch.ts[rows].copy(), labels)


def sub_batch(batch, users):
    return _sub_batch(batch, users)


def attn(q, k, v, batch, pos, users=None, scale=None):
    H, dh = q.shape[1], q.shape[2]
    sp, st = slopes(H)
    return oracle.attention_fwd(q, k, v, batch.seq_offsets, batch.hist_len, pos, batch.ts, sp,
                                st, 1.0 / math.sqrt(dh) if scale is None else scale, users=users)


def attn_bwd(q, k, v, dO, batch, pos, users=None):
    H, dh = q.shape[1], q.shape[2]
    sp, st = slopes(H)
    return oracle.attention_bwd(q, k, v, dO, batch.seq_offsets, batch.hist_len, pos, batch.ts,
                                sp, st, 1.0 / math.sqrt(dh), users=users)


def dq_noise_floor(k, dO, O, seq_offsets, scale):
    """Per (token, head) absolute error of dq that the bf16 path carries by construction.

    dq_i = scale sum_j P_ij (dP_ij - D_i) k_j with D_i = rowsum(dO_i * O_i) taken from O
    as stored in bf16: O's rounding (relative 2^-9 per element) moves D_i by up to
    2^-9 sum_e |dO_ie O_ie|, and that shift reaches dq_i as scale * dD_i * sum_j P_ij k_j,
    at most scale * |dD_i| * max_j |k_j| (the P_ij sum to 1).  Rows whose dP_ij - D_i
    nearly cancel (one dominant key, e.g. a user's first tokens) have dq far below that
    size, so a per-row relative bound alone cannot hold there.  Returned with a factor 4
    of slack (2^-7) for the other bf16 roundings on the path."""
    k = np.asarray(k, np.float64)
    T, H, _ = k.shape
    out = np.zeros((T, H))
    dd = (np.abs(np.asarray(dO, np.float64)) * np.abs(np.asarray(O, np.float64))).sum(-1)
    for u in range(len(seq_offsets) - 1):
        s, e = int(seq_offsets[u]), int(seq_offsets[u + 1])
        if e > s:
            kmax = np.abs(k[s:e]).max(axis=(0, 2))  # per head
            out[s:e] = scale * 2.0 ** -7 * dd[s:e] * kmax[None, :]
    return out


def check_rows(got, want, tol, name, floor=None, noise=None):
    """Relative-to-max bound, and a per-token bound over all heads: each row's error
    within tol of max(its own magnitude, the tensor's max / 16), plus an optional
    absolute per (token, head) noise allowance ``noise``."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert rel_to_max(got, want) <= tol, name
    err = np.abs(got - want).max(axis=-1)  # [rows, H]
    mag = np.abs(want).max(axis=-1)
    gmax = np.abs(want).max()
    allow = tol * np.maximum(mag.max(axis=1, keepdims=True), gmax / 16.0 if floor is None else floor)
    if noise is not None:
        allow = allow + noise
    bad = err > allow
    if bad.any():
        r, h = np.argwhere(bad)[0]
        raise AssertionError((name, int(r), int(h), float(err[r, h]), float(allow[r, h])))
