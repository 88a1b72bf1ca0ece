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


def attention_probs(fwd, q, k, batch, pos, u):
    """The oracle's attention probabilities P[i, h, j] of user u, read off its forward
    with one-hot values (v_j = e_j gives O_i = sum_j P_ij e_j = P_i).  ``fwd(q, k, v,
    seq_offsets, hist_len, pos, ts)`` is an oracle forward (linear or bucketed bias)."""
    sub = sub_batch(batch, [u])
    rows = user_rows(batch, [u])
    L, H, dh = len(rows), q.shape[1], q.shape[2]
    P = np.zeros((L, H, L))
    for c0 in range(0, L, dh):  # dh one-hot value columns per call
        c1 = min(L, c0 + dh)
        v = np.zeros((L, H, dh))
        for h in range(H):
            v[c0:c1, h, :c1 - c0] = np.eye(c1 - c0)
        O, _ = fwd(q[rows], k[rows], v, sub.seq_offsets, sub.hist_len, np.asarray(pos)[rows],
                   sub.ts)
        P[:, :, c0:c1] = O[:, :, :c1 - c0]
    return P


def grad_noise_floors(fwd, q, k, v, dO, O, batch, pos, users, scale):
    """Per (token, head) absolute errors that the bf16 backward carries by construction,
    for dq, dk and dv.

    With P from the oracle, dP = dO V^T and D_i = rowsum(dO_i * O_i):
      * D_i is formed from O as the forward wrote it: P rounded to bf16 before P V and O
        rounded to bf16, each element off by up to 2^-9 (|O_ie| + sum_j P_ij |v_je|), which
        moves D_i by up to 2^-9 sum_e |dO_ie| (|O_ie| + (P |V|)_ie);
      * dS_ij = P_ij (dP_ij - D_i) is rounded to bf16 once (2^-9 of |dS_ij|);
      * P is rounded to bf16 for dV = P^T dO.
    So |ddq_i| <= scale max|k| sum_j E_ij, |ddk_j| <= scale max|q| sum_i E_ij with
    E_ij = P_ij 2^-9 (sum_e |dO_ie| (|O_ie| + (P |V|)_ie) + |dP_ij - D_i|), and |ddv_j| <= 2^-9
    max|dO| sum_i P_ij.  Rows whose terms nearly cancel (a user's first tokens; keys
    seen by few queries) have gradients far below these sums, where a per-row relative
    bound alone cannot hold.  Returned with a factor 4 of slack (2^-7 for 2^-9)."""
    q, k, v, dO, O = (np.asarray(x, np.float64) for x in (q, k, v, dO, O))
    T, H, _ = q.shape
    nq, nk, nv = np.zeros((T, H)), np.zeros((T, H)), np.zeros((T, H))
    for u in users:
        rows = user_rows(batch, [u])
        if len(rows) == 0:
            continue
        P = attention_probs(fwd, q, k, batch, pos, u)
        for h in range(H):
            Ph = P[:, h, :]
            g, vv, oo = dO[rows, h], v[rows, h], O[rows, h]
            dP = g @ vv.T
            D = (g * oo).sum(-1)
            A = (np.abs(g) * (np.abs(oo) + Ph @ np.abs(vv))).sum(-1)
            E = Ph * (A[:, None] + np.abs(dP - D[:, None])) * 2.0 ** -7
            nq[rows, h] = scale * np.abs(k[rows, h]).max() * E.sum(axis=1)
            nk[rows, h] = scale * np.abs(q[rows, h]).max() * E.sum(axis=0)
            nv[rows, h] = 2.0 ** -7 * np.abs(g).max() * Ph.sum(axis=0)
    return nq, nk, nv


def check_rows(got, want, tol, name, floor_frac=1.0 / 16.0, noise=None):
    """Relative-to-max bound, and a per-token bound over all heads: each row's error
    within tol of max(its own magnitude, floor_frac * the tensor's max), plus an
    optional absolute per (token, head) noise allowance ``noise``."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert rel_to_max(got, want) <= tol, name
    err = np.abs(got - want).max(axis=-1)  # [rows, H]
    mag = np.abs(want).max(axis=-1)
    gmax = np.abs(want).max()
    allow = tol * np.maximum(mag.max(axis=1, keepdims=True), floor_frac * gmax)
    allow = np.broadcast_to(allow + (0.0 if noise is None else noise), err.shape)
    bad = err > allow
    if bad.any():
        r, h = np.argwhere(bad)[0]
        raise AssertionError((name, int(r), int(h), float(err[r, h]), float(allow[r, h])))
