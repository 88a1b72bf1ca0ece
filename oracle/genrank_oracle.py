"""Plain, slow float64 oracle of the GenRank data-parallel hot path.

TEST INFRASTRUCTURE ONLY: used by ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / reference leg of ``bench.py``.  The product never
imports it, and it shares no code, table or helper with the CUDA library.

Sources (web pages about "Towards Large-scale Generative Ranking", GenRank):

* [HXZ] huaxiaozhuan.com chapter notes "GenRank [2025]":
  §1.4.1 Item-Action Organization (token sums, mask action, candidate mask),
  §1.4.2 Position & Time Biases (position / request-index / pre-request time
  embeddings, the five-way input sum, the ALiBi score and slope formulas).
* [WLN] wln20.github.io "生成式排序 —— 小红书 GenRank 精读笔记": the candidate
  mask and its equivalence to appending each candidate alone.
* [FUN-EN] fun-rec mdbook "The Overall Generative Ranking Paradigm",
  §7.2.1 (history causal, candidates see all history, masked from each other)
  and §7.2.2 (the three embeddings; ALiBi extended to position and time).

Readings taken where the pages are silent or disagree (all listed in the
design notes): scale 1/sqrt(d_head); slopes 2^(-8(h+1)/H) for h = 0..H-1;
position bias on the shared positions p (all candidates at n+1); time bias
linear, slope_h/3600 per second of |t_i - t_j|; a candidate sees itself;
positions 1-based; request index clamped to n_ri - 1; bucket(delta) =
1 + min(n_rt - 2, floor(4 log2(delta + 1))) with 0 for "no earlier request".
The bucketed time-bias variant uses min(n_rt - 2, floor(4 log2(delta + 1))) per pair
and the position slopes as its per-bucket slopes.

Every function loops over users (and heads) and writes the definitions out
with explicit masks; no blocking, fusion or reordering beyond a library
matmul as one step.
"""

from __future__ import annotations

import math

import numpy as np

RMS_EPS = 1e-6


# ----------------------------------------------------------------------------------------
# step a1: per-token integer metadata
# ----------------------------------------------------------------------------------------

def alibi_slopes(H: int) -> np.ndarray:
    """m_h = 2^(-8(h+1)/H), h = 0..H-1 ([HXZ] §1.4.2, slope formula and its H=8 example)."""
    return np.array([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)], dtype=np.float64)


def time_bucket(delta: int, n_rt: int = 64) -> int:
    """Row of the pre-request time table for a gap of ``delta`` >= 0 seconds.

    [HXZ] §1.4.2 (Pre-Request Time Embeddings) applies an unspecified bucket()
    to t_i - max_{t_j < t_i} t_j.  Reading: quarter-octave log spacing,
    1 + floor(4 * log2(delta + 1)), saturating at row n_rt - 1.  Row 0 is kept
    for tokens with no earlier request.  floor(4 log2 x) is the largest k with
    2^k <= x^4, i.e. bit_length(x^4) - 1, exact in Python integers.
    """
    if delta < 0:
        raise ValueError("negative gap")
    k = ((int(delta) + 1) ** 4).bit_length() - 1
    return 1 + min(n_rt - 2, k)


def token_metadata(seq_offsets, hist_len, ts, n_ri: int = 128, n_rt: int = 64, users=None):
    """pos, req_idx, rt_bucket for every token (int64 arrays [T]).

    [HXZ] §1.4.2: E_pe uses the item's index in the sequence and every
    candidate of the current request shares one position (n = 100 history
    items give position 101 to each candidate); E_ri uses |{t_1..t_i}|, the
    number of distinct timestamps so far; E_rt uses bucket(t_i - max_{t_j<t_i} t_j).
    A candidate's values are those of the token obtained by appending the
    candidate alone (time t_req) to the history ([WLN], candidate mask).
    Written with a Python set and max over each prefix, not a running counter.
    """
    seq_offsets = np.asarray(seq_offsets, dtype=np.int64)
    ts = np.asarray(ts, dtype=np.int64)
    T = int(seq_offsets[-1])
    pos = np.zeros(T, np.int64)
    req = np.zeros(T, np.int64)
    rtb = np.zeros(T, np.int64)
    for u in (range(len(hist_len)) if users is None else users):
        s, e, n = int(seq_offsets[u]), int(seq_offsets[u + 1]), int(hist_len[u])
        hist = [int(t) for t in ts[s:s + n]]
        for i in range(e - s):
            if i < n:
                prefix = hist[:i + 1]
                p = i + 1
            else:
                prefix = hist + [int(ts[s + i])]
                p = n + 1
            t_i = prefix[-1]
            earlier = [t for t in prefix if t < t_i]
            pos[s + i] = p
            req[s + i] = min(len(set(prefix)), n_ri - 1)
            rtb[s + i] = 0 if not earlier else time_bucket(t_i - max(earlier), n_rt)
    return pos, req, rtb


# ----------------------------------------------------------------------------------------
# step a2: five-way embedding sum
# ----------------------------------------------------------------------------------------

def embed_assemble(seq_offsets, hist_len, item_ids, action_ids, meta, item_tab, action_tab,
                   pos_tab, ri_tab, rt_tab, users=None):
    """E_i = psi(x_i) + phi(a_i) + E_pe + E_ri + E_rt in float64 ([HXZ] §1.4.2, input sum).

    History tokens use their action row ([HXZ] §1.4.1: e_i = psi(x_i) + phi(a_i));
    candidate tokens use the mask-action row M, the last row of ``action_tab``
    ([HXZ] §1.4.1: e_j = psi(x_j) + m).
    """
    pos, req, rtb = meta
    T = int(seq_offsets[-1])
    d = item_tab.shape[1]
    M = action_tab.shape[0] - 1
    E = np.zeros((T, d), np.float64)
    f = lambda a: np.asarray(a, np.float64)  # noqa: E731
    for u in (range(len(hist_len)) if users is None else users):
        s, e, n = int(seq_offsets[u]), int(seq_offsets[u + 1]), int(hist_len[u])
        for i in range(s, e):
            a = int(action_ids[i]) if i - s < n else M
            E[i] = (f(item_tab[item_ids[i]]) + f(action_tab[a]) + f(pos_tab[pos[i]])
                    + f(ri_tab[req[i]]) + f(rt_tab[rtb[i]]))
    return E


def embed_assemble_bwd(dE, seq_offsets, hist_len, item_ids, action_ids, meta, n_item, n_action_rows,
                       n_pos, n_ri, n_rt):
    """Gradients of the five tables: each token's dE_i added to the five rows it read."""
    pos, req, rtb = meta
    dE = np.asarray(dE, np.float64)
    d = dE.shape[1]
    g = {k: np.zeros((r, d)) for k, r in (("item", n_item), ("action", n_action_rows),
                                          ("pos", n_pos), ("ri", n_ri), ("rt", n_rt))}
    M = n_action_rows - 1
    for u in range(len(hist_len)):
        s, e, n = int(seq_offsets[u]), int(seq_offsets[u + 1]), int(hist_len[u])
        for i in range(s, e):
            a = int(action_ids[i]) if i - s < n else M
            g["item"][item_ids[i]] += dE[i]
            g["action"][a] += dE[i]
            g["pos"][pos[i]] += dE[i]
            g["ri"][req[i]] += dE[i]
            g["rt"][rtb[i]] += dE[i]
    return g


# ----------------------------------------------------------------------------------------
# step a3/a4: masked multi-head attention with ALiBi position and time biases
# ----------------------------------------------------------------------------------------

def attention_mask(n: int, L: int) -> np.ndarray:
    """Boolean [L, L] visibility for one user with n history tokens and L - n candidates.

    History rows are causal ([HXZ] §1.3.1; [FUN-EN] §7.2.1).  A candidate row
    sees every history token and itself, never another candidate ([WLN];
    [FUN-EN] §7.2.1 and the mask figure caption of §7.2.2).
    """
    mask = np.zeros((L, L), dtype=bool)
    for i in range(L):
        if i < n:
            mask[i, :i + 1] = True
        else:
            mask[i, :n] = True
            mask[i, i] = True
    return mask


def _user_scores(Q, K, p, t, slope_pos, slope_time, scale, n):
    """score_ij = q_i.k_j * scale - m|p_i - p_j| - m_t|t_i - t_j| ([HXZ] §1.4.2 ALiBi score)."""
    S = (Q @ K.T) * scale
    dp = np.abs(p[:, None] - p[None, :]).astype(np.float64)
    dt = np.abs(t[:, None] - t[None, :]).astype(np.float64)
    S = S - slope_pos * dp - slope_time * dt
    mask = attention_mask(n, len(p))
    return np.where(mask, S, -np.inf), mask


def attention_fwd(q, k, v, seq_offsets, hist_len, pos, ts, slope_pos, slope_time, scale,
                  users=None):
    """O [T,H,dh] and natural-log LSE [H,T] of the masked ALiBi attention, per user and head."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    T, H, dh = q.shape
    O = np.zeros((T, H, dh))
    LSE = np.full((H, T), np.nan)
    users = range(len(hist_len)) if users is None else users
    for u in users:
        s, e, n = int(seq_offsets[u]), int(seq_offsets[u + 1]), int(hist_len[u])
        p = np.asarray(pos[s:e], np.int64)
        t = np.asarray(ts[s:e], np.int64)
        for h in range(H):
            S, _ = _user_scores(q[s:e, h], k[s:e, h], p, t, slope_pos[h], slope_time[h], scale, n)
            mx = S.max(axis=1, keepdims=True)
            P = np.exp(S - mx)
            l = P.sum(axis=1, keepdims=True)
            O[s:e, h] = (P / l) @ v[s:e, h]
            LSE[h, s:e] = (mx + np.log(l))[:, 0]
    return O, LSE


def attention_bwd(q, k, v, dO, seq_offsets, hist_len, pos, ts, slope_pos, slope_time, scale,
                  users=None):
    """dQ, dK, dV of the attention above; the biases carry no parameters, so no bias grad.

    With P = softmax(S) row-wise and O = P V:  dV = P^T dO,  dP = dO V^T,
    dS = P * (dP - rowsum(P * dP)),  dQ = scale * dS K,  dK = scale * dS^T Q.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    dO = np.asarray(dO, np.float64)
    T, H, dh = q.shape
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    users = range(len(hist_len)) if users is None else users
    for u in users:
        s, e, n = int(seq_offsets[u]), int(seq_offsets[u + 1]), int(hist_len[u])
        p = np.asarray(pos[s:e], np.int64)
        t = np.asarray(ts[s:e], np.int64)
        for h in range(H):
            Q, K, V, G = q[s:e, h], k[s:e, h], v[s:e, h], dO[s:e, h]
            S, _ = _user_scores(Q, K, p, t, slope_pos[h], slope_time[h], scale, n)
            P = np.exp(S - S.max(axis=1, keepdims=True))
            P /= P.sum(axis=1, keepdims=True)
            dP = G @ V.T
            dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
            dq[s:e, h] = scale * dS @ K
            dk[s:e, h] = scale * dS.T @ Q
            dv[s:e, h] = P.T @ G
    return dq, dk, dv


# ----------------------------------------------------------------------------------------
# variant: bucketed time bias (a NEXT row of the scope table)
# ----------------------------------------------------------------------------------------

def pair_time_bucket(delta: int, n_rt: int = 64) -> int:
    """bucket(t_i - t_j) of the bucketed time bias, for a gap of ``delta`` >= 0 seconds.

    [FUN-EN] §7.2.2 (and its zh twin) writes the time term of the ALiBi bias as
    -m_t bucket(t_i - t_j) without defining bucket().  Reading: the quarter-octave grid
    of the pre-request time embedding, floor(4 log2(delta + 1)), saturating at
    n_rt - 2 (that table's largest gap row) and without its "no earlier request" row,
    so that two items of one request (delta = 0) are in bucket 0.  As for the
    embedding, floor(4 log2 x) = bit_length(x^4) - 1 in Python integers.
    """
    if delta < 0:
        raise ValueError("negative gap")
    k = ((int(delta) + 1) ** 4).bit_length() - 1
    return min(n_rt - 2, k)


def _user_scores_bucketed(Q, K, p, t, slope_pos, slope_tb, scale, n, n_rt):
    """score_ij = q_i.k_j * scale - m_p (p_i - p_j) - m_t bucket(t_i - t_j) on visible
    pairs ([FUN-EN] §7.2.2 bias formula; p_i >= p_j and t_i >= t_j there)."""
    L = len(p)
    S = (Q @ K.T) * scale
    mask = attention_mask(n, L)
    B = np.zeros((L, L))
    for i in range(L):
        for j in range(L):
            if mask[i, j]:
                B[i, j] = (slope_pos * float(int(p[i]) - int(p[j]))
                           + slope_tb * float(pair_time_bucket(int(t[i]) - int(t[j]), n_rt)))
    return np.where(mask, S - B, -np.inf)


def attention_fwd_bucketed(q, k, v, seq_offsets, hist_len, pos, ts, slope_pos, slope_tb, scale,
                           n_rt: int = 64, users=None):
    """O [T,H,dh] and natural-log LSE [H,T] of the masked attention with the bucketed time
    bias; the mask and position term are those of ``attention_fwd``."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    T, H, dh = q.shape
    O = np.zeros((T, H, dh))
    LSE = np.full((H, T), np.nan)
    users = range(len(hist_len)) if users is None else users
    for u in users:
        s, e, n = int(seq_offsets[u]), int(seq_offsets[u + 1]), int(hist_len[u])
        p = np.asarray(pos[s:e], np.int64)
        t = np.asarray(ts[s:e], np.int64)
        for h in range(H):
            S = _user_scores_bucketed(q[s:e, h], k[s:e, h], p, t, slope_pos[h], slope_tb[h],
                                      scale, n, n_rt)
            mx = S.max(axis=1, keepdims=True)
            P = np.exp(S - mx)
            l = P.sum(axis=1, keepdims=True)
            O[s:e, h] = (P / l) @ v[s:e, h]
            LSE[h, s:e] = (mx + np.log(l))[:, 0]
    return O, LSE


def attention_bwd_bucketed(q, k, v, dO, seq_offsets, hist_len, pos, ts, slope_pos, slope_tb,
                           scale, n_rt: int = 64, users=None):
    """dQ, dK, dV of ``attention_fwd_bucketed``.  The bucketed bias has no parameters
    either, so the gradients are those of ``attention_bwd`` with these scores:
    dV = P^T dO, dS = P * (dP - rowsum(P * dP)), dQ = scale dS K, dK = scale dS^T Q."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    dO = np.asarray(dO, np.float64)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    users = range(len(hist_len)) if users is None else users
    for u in users:
        s, e, n = int(seq_offsets[u]), int(seq_offsets[u + 1]), int(hist_len[u])
        p = np.asarray(pos[s:e], np.int64)
        t = np.asarray(ts[s:e], np.int64)
        for h in range(q.shape[1]):
            Q, K, V, G = q[s:e, h], k[s:e, h], v[s:e, h], dO[s:e, h]
            S = _user_scores_bucketed(Q, K, p, t, slope_pos[h], slope_tb[h], scale, n, n_rt)
            P = np.exp(S - S.max(axis=1, keepdims=True))
            P /= P.sum(axis=1, keepdims=True)
            dP = G @ V.T
            dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
            dq[s:e, h] = scale * dS @ K
            dk[s:e, h] = scale * dS.T @ Q
            dv[s:e, h] = P.T @ G
    return dq, dk, dv


# ----------------------------------------------------------------------------------------
# variant: scoring candidates against cached history keys and values (a NEXT row)
# ----------------------------------------------------------------------------------------

def attention_fwd_cached(q_c, k_c, v_c, cand_offsets, k_hist, v_hist, hist_offsets, pos_hist,
                         ts_hist, ts_cand, slope_pos, slope_time, scale):
    """O [C,H,dh] and natural-log LSE [H,C] of the candidate rows only, from a cache of the
    users' history keys and values.

    [HXZ] §1.3.2 (its feature-engineering paragraph) credits the KV cache with keeping
    generative ranking efficient as the candidate set grows, and [FUN-EN] §7.2.1 counts
    the halved KV cache among the action-oriented layout's gains.  [HXZ] §1.4.1 and
    [FUN-EN] §7.2.1 fix what a candidate sees: the whole history of its user and itself.  User u's history rows are
    k_hist/v_hist[hist_offsets[u]:hist_offsets[u+1]] with positions pos_hist and times
    ts_hist; its candidates are rows cand_offsets[u]:cand_offsets[u+1] of q_c, k_c, v_c,
    all at position n_u + 1 and time ts_cand.  The score of candidate c against history
    key j is q_c.k_j * scale - m |p_c - p_j| - m_t |t_c - t_j|; against itself it is
    q_c.k_c * scale (no distance).
    """
    q_c = np.asarray(q_c, np.float64)
    k_c = np.asarray(k_c, np.float64)
    v_c = np.asarray(v_c, np.float64)
    k_hist = np.asarray(k_hist, np.float64)
    v_hist = np.asarray(v_hist, np.float64)
    C, H, dh = q_c.shape
    O = np.zeros((C, H, dh))
    LSE = np.full((H, C), np.nan)
    for u in range(len(cand_offsets) - 1):
        hs, he = int(hist_offsets[u]), int(hist_offsets[u + 1])
        n = he - hs
        p_c = n + 1
        for c in range(int(cand_offsets[u]), int(cand_offsets[u + 1])):
            t_c = int(ts_cand[c])
            for h in range(H):
                scores = []
                values = []
                for j in range(hs, he):
                    sj = (float(q_c[c, h] @ k_hist[j, h]) * scale
                          - slope_pos[h] * abs(p_c - int(pos_hist[j]))
                          - slope_time[h] * abs(t_c - int(ts_hist[j])))
                    scores.append(sj)
                    values.append(v_hist[j, h])
                scores.append(float(q_c[c, h] @ k_c[c, h]) * scale)
                values.append(v_c[c, h])
                sc = np.array(scores)
                mx = sc.max()
                w = np.exp(sc - mx)
                O[c, h] = (w / w.sum()) @ np.array(values)
                LSE[h, c] = mx + math.log(w.sum())
    return O, LSE


# ----------------------------------------------------------------------------------------
# comparison: the interleaved layout with a dense N x N relative bias (a NEXT row)
# ----------------------------------------------------------------------------------------

def interleaved_layout(seq_offsets, hist_len):
    """Token layout of the interleaved organisation for the same users: each history
    interaction spends two tokens (its item, then its action), so a user with n history
    interactions and m candidates has 2n + m tokens ([FUN-EN] §7.2.0, the interleaving
    [Phi_0, a_0, Phi_1, a_1, ...] and its length 2 n_c + m; [HXZ] §1.4.1).  Returns the
    new offsets [B+1] and history lengths [B] (= 2n)."""
    n = np.asarray(hist_len, np.int64)
    m = np.diff(np.asarray(seq_offsets, np.int64)) - n
    off = np.zeros(len(n) + 1, np.int64)
    off[1:] = np.cumsum(2 * n + m)
    return off, 2 * n


def attention_fwd_dense_bias(q, k, v, seq_offsets, hist_len, bias, scale, users=None):
    """O [T,H,dh] and natural-log LSE [H,T] with a dense per-user bias read for every pair.

    [FUN-EN] §7.2.2 writes the relative attention bias of the interleaved model as
    score_ij = q_i.k_j / sqrt(d) + rab(i, j), an N x N matrix per sequence that the
    forward reads in full; [HXZ] §1.4.2 notes that its I/O grows with the square of the
    length.  Here bias[u] is user u's [Lpad, Lpad] matrix (shared by the heads), local
    indices; the mask is the one of ``attention_fwd`` (history causal, a candidate sees
    the history and itself).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    T, H, dh = q.shape
    O = np.zeros((T, H, dh))
    LSE = np.full((H, T), np.nan)
    users = range(len(hist_len)) if users is None else users
    for u in users:
        s, e, n = int(seq_offsets[u]), int(seq_offsets[u + 1]), int(hist_len[u])
        L = e - s
        Bu = np.asarray(bias[u][:L, :L], np.float64)
        mask = attention_mask(n, L)
        for h in range(H):
            S = np.where(mask, (q[s:e, h] @ k[s:e, h].T) * scale + Bu, -np.inf)
            mx = S.max(axis=1, keepdims=True)
            P = np.exp(S - mx)
            l = P.sum(axis=1, keepdims=True)
            O[s:e, h] = (P / l) @ v[s:e, h]
            LSE[h, s:e] = (mx + np.log(l))[:, 0]
    return O, LSE


# ----------------------------------------------------------------------------------------
# the model blocks around the hot path (projections, norms, FFN, head, loss)
# ----------------------------------------------------------------------------------------

def _rms(x):
    r = 1.0 / np.sqrt((x * x).mean(axis=-1, keepdims=True) + RMS_EPS)
    return x * r, r


def _rms_bwd(x, r, dy):
    d = x.shape[-1]
    return r * dy - (r ** 3 / d) * x * (x * dy).sum(axis=-1, keepdims=True)


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def _cand_rows(seq_offsets, hist_len):
    rows = []
    for u in range(len(hist_len)):
        rows.extend(range(int(seq_offsets[u]) + int(hist_len[u]), int(seq_offsets[u + 1])))
    return np.array(rows, dtype=np.int64)


def block_forward(E, layers, w_head, seq_offsets, hist_len, pos, ts, H, ffn: bool):
    """Logits at candidate rows; returns (logits, cache for ``block_backward``).

    One-layer configs: h = E + Attn(E Wq, E Wk, E Wv) Wo.  Four-layer configs:
    pre-RMSNorm (eps 1e-6, unit gain) attention and 4d SiLU FFN residual
    blocks, then a final RMSNorm.  The head is a dot with w_head at candidate
    rows only: loss lives only at candidate positions ([HXZ] §1.3.1).
    """
    E = np.asarray(E, np.float64)
    T, d = E.shape
    dh = d // H
    slopes = alibi_slopes(H)
    scale = 1.0 / math.sqrt(dh)
    f = lambda a: np.asarray(a, np.float64)  # noqa: E731
    x = E
    cache = []
    for L in layers:
        c = {"x_in": x}
        if ffn:
            a, r = _rms(x)
            c["r_in"] = r
        else:
            a = x
        c["a"] = a
        Q, K, V = (a @ f(L["Wq"])).reshape(T, H, dh), (a @ f(L["Wk"])).reshape(T, H, dh), \
            (a @ f(L["Wv"])).reshape(T, H, dh)
        O, _ = attention_fwd(Q, K, V, seq_offsets, hist_len, pos, ts, slopes, slopes / 3600.0, scale)
        c.update(Q=Q, K=K, V=V, O=O)
        x = x + O.reshape(T, d) @ f(L["Wo"])
        if ffn:
            c["x_mid"] = x
            fa, r2 = _rms(x)
            G = fa @ f(L["W1"])
            U = G * _sigmoid(G)
            c.update(r_mid=r2, fa=fa, G=G, U=U)
            x = x + U @ f(L["W2"])
        cache.append(c)
    rows = _cand_rows(seq_offsets, hist_len)
    if ffn:
        xf, rf = _rms(x)
    else:
        xf, rf = x, None
    z = xf[rows] @ f(w_head)
    return z, {"layers": cache, "x_out": x, "r_out": rf, "xf": xf, "rows": rows}


def bce_loss(z, y):
    """Mean binary cross-entropy with logits over all candidates of the batch."""
    z = np.asarray(z, np.float64)
    y = np.asarray(y, np.float64)
    return float(np.mean(np.logaddexp(0.0, z) - y * z))


def block_backward(z, y, cache, layers, w_head, seq_offsets, hist_len, pos, ts, H, ffn: bool):
    """dL/dE for the mean BCE loss (history rows carry no loss); analytic, float64."""
    f = lambda a: np.asarray(a, np.float64)  # noqa: E731
    y = np.asarray(y, np.float64)
    dz = (_sigmoid(z) - y) / len(z)
    rows = cache["rows"]
    x = cache["x_out"]
    T, d = x.shape
    dh = d // H
    slopes = alibi_slopes(H)
    scale = 1.0 / math.sqrt(dh)
    dxf = np.zeros((T, d))
    dxf[rows] = dz[:, None] * f(w_head)[None, :]
    dx = _rms_bwd(x, cache["r_out"], dxf) if ffn else dxf
    for L, c in zip(reversed(layers), reversed(cache["layers"])):
        if ffn:
            dU = dx @ f(L["W2"]).T
            sg = _sigmoid(c["G"])
            dG = dU * sg * (1.0 + c["G"] * (1.0 - sg))
            dfa = dG @ f(L["W1"]).T
            dx = dx + _rms_bwd(c["x_mid"], c["r_mid"], dfa)
        dO = (dx @ f(L["Wo"]).T).reshape(T, H, dh)
        dq, dk, dv = attention_bwd(c["Q"], c["K"], c["V"], dO, seq_offsets, hist_len, pos, ts,
                                   slopes, slopes / 3600.0, scale)
        da = (dq.reshape(T, d) @ f(L["Wq"]).T + dk.reshape(T, d) @ f(L["Wk"]).T
              + dv.reshape(T, d) @ f(L["Wv"]).T)
        dx = dx + (_rms_bwd(c["x_in"], c["r_in"], da) if ffn else da)
    return dx
