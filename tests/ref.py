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
