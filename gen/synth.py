"""Seeded synthetic workloads shaped like the GenRank pages' ranking traffic.

The proprietary Explore Feed exposure logs ("Towards Large-scale Generative
Ranking", Problem Setup section) are not available, so every input here is
synthetic.  The recipe:

* history lengths per config (uniform, fixed, or lognormal clipped);
* request groups: sizes ~ Geometric(1/mean) on {1,2,...}, the last group
  truncated so the history holds exactly n tokens; every item in a group
  shares one integer timestamp (seconds);
* gaps between requests: ceil(Exp(mean)) >= 1 s, or a weighted mixture of
  exponentials; the first request of a user starts at 1.7e9 s plus a
  uniform offset within a day; the current request time t_req (shared by
  all candidates) is one more gap after the last history request;
* item ids: bounded Zipf(s) over ranks 1..V by inverse CDF, mapped through
  a seeded permutation of [0, V) so that hot rows are scattered;
* history action ids: categorical with p(k) proportional to 1/(k+1),
  k = 0..7; candidate slots carry the mask-action row index 8;
* click labels (training config): Bernoulli(0.1) per candidate;
* tables and weights: N(0, 0.02), rounded to bf16 for bf16 configs.

Each user draws from its own numpy PCG64 stream keyed by (seed, user), so
any subset of users can be regenerated without generating the others.  The
item table, which reaches 4M x 512, is defined element-wise by a
counter-based generator (the splitmix64 finaliser of Steele, Lea & Flood,
OOPSLA 2014, feeding a Box-Muller transform), so a few rows can be produced
on the host while the full table is produced on the device by the same
definition.  Nothing in this module computes any part of the ranking method.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from functools import lru_cache

import numpy as np

TS_BASE = 1_700_000_000  # seconds; the start of every synthetic history
N_ACTION = 8  # real actions; row 8 of the action table is the mask action M


@dataclass(frozen=True)
class Config:
    """One workload shape.  ``d = H * dh``; tables per the pages' design."""

    name: str
    seed: int
    B: int
    hist: tuple  # ("uniform", lo, hi) | ("fixed", n) | ("lognormal", median, sigma, lo, hi)
    m: int
    H: int
    dh: int
    layers: int
    dtype: str  # "f32" | "bf16"
    n_item: int
    zipf_s: float
    gaps: tuple  # ((weight, mean_seconds), ...)
    group_mean: float
    training: bool = False
    ffn: bool = False  # pre-RMSNorm + 4d SiLU FFN blocks (the 4-layer configs)
    n_pos: int = 600
    n_ri: int = 128
    n_rt: int = 64
    label_p: float = 0.1

    @property
    def d(self) -> int:
        return self.H * self.dh

    @property
    def n_action_rows(self) -> int:
        return N_ACTION + 1

    def with_(self, **kw) -> "Config":
        return replace(self, **kw)


_C0 = Config("c0", 20250500, 4, ("uniform", 16, 64), 8, 2, 32, 1, "f32", 10_000, 1.1,
             ((1.0, 30.0),), 3.0)
_C1 = Config("c1", 20250501, 256, ("uniform", 32, 480), 128, 4, 64, 1, "bf16", 1_000_000,
             1.1, ((1.0, 30.0),), 3.0)
_C2 = Config("c2", 20250502, 1024, ("fixed", 480), 256, 8, 64, 4, "bf16", 4_000_000, 1.05,
             ((1.0, 30.0),), 3.0, ffn=True)
_C3 = Config("c3", 20250503, 512, ("lognormal", 240.0, 0.5, 16, 480), 16, 8, 64, 4, "bf16",
             4_000_000, 1.05, ((1.0, 30.0),), 3.0, training=True, ffn=True)


def _c4(m: int, k: int) -> Config:
    return Config(f"c4_m{m}", 20250504 + 100 * k, 64, ("fixed", 480), m, 16, 64, 1, "bf16",
                  1_000_000, 1.1, ((0.5, 5.0), (0.5, 3600.0)), 6.0)


CONFIGS = {c.name: c for c in (_C0, _C1, _C2, _C3, _c4(64, 0), _c4(256, 1), _c4(1024, 2))}


def config_by_name(name: str) -> Config:
    return CONFIGS[name]


# ----------------------------------------------------------------------------------------
# bf16 rounding (round to nearest even) of float32 data, kept as float32 arrays
# ----------------------------------------------------------------------------------------

def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 value (ties to even); finite inputs only."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32)


def _cast(x: np.ndarray, dtype: str) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32)
    return bf16_round(x) if dtype == "bf16" else x


# ----------------------------------------------------------------------------------------
# counter-based item table: value(row, col) depends only on (seed, row*d + col)
# ----------------------------------------------------------------------------------------

_GOLDEN = 0x9E3779B97F4A7C15
_MIX1 = 0xBF58476D1CE4E5B9
_MIX2 = 0x94D049BB133111EB
_M64 = (1 << 64) - 1


def _to_i64(c: int) -> int:
    return c - (1 << 64) if c >= (1 << 63) else c


def _table_key(seed: int) -> int:
    z = (seed * _GOLDEN + 0x5EED) & _M64
    z = ((z ^ (z >> 30)) * _MIX1) & _M64
    z = ((z ^ (z >> 27)) * _MIX2) & _M64
    return z ^ (z >> 31)


def _mix_np(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(_MIX1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(_MIX2)
    return z ^ (z >> np.uint64(31))


def item_rows(seed: int, rows, d: int, dtype: str, std: float = 0.02) -> np.ndarray:
    """Rows ``rows`` of the item table (float32, bf16-valued for bf16 configs)."""
    rows = np.asarray(rows, dtype=np.uint64).reshape(-1)
    key = np.uint64(_table_key(seed))
    e = rows[:, None] * np.uint64(d) + np.arange(d, dtype=np.uint64)[None, :]
    with np.errstate(over="ignore"):
        x0 = _mix_np(key + (np.uint64(2) * e + np.uint64(1)) * np.uint64(_GOLDEN))
        x1 = _mix_np(key + (np.uint64(2) * e + np.uint64(2)) * np.uint64(_GOLDEN))
    u1 = ((x0 >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53
    u2 = (x1 >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
    z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)
    return _cast((std * z).astype(np.float32), dtype)


def item_table_torch(seed: int, n_rows: int, d: int, dtype: str, device, std: float = 0.02,
                     chunk_rows: int = 1 << 16):
    """The whole item table as a torch tensor on ``device`` (same values as ``item_rows``).

    Integer hashing is exact in two's-complement int64; logical right shifts are
    emulated by masking.  The float tail (log/cos in float64) may differ from
    numpy's by an ulp of float64, which survives the cast to float32/bf16 only
    at rounding ties; the tests measure that rate.
    """
    import torch

    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = torch.empty((n_rows, d), dtype=tdt, device=device)
    key = _to_i64(_table_key(seed))
    g, m1, m2 = _to_i64(_GOLDEN), _to_i64(_MIX1), _to_i64(_MIX2)

    def lsr(x, k):
        return (x >> k) & ((1 << (64 - k)) - 1)

    def mix(z):
        z = (z ^ lsr(z, 30)) * m1
        z = (z ^ lsr(z, 27)) * m2
        return z ^ lsr(z, 31)

    cols = torch.arange(d, dtype=torch.int64, device=device)
    for r0 in range(0, n_rows, chunk_rows):
        r1 = min(n_rows, r0 + chunk_rows)
        rows = torch.arange(r0, r1, dtype=torch.int64, device=device)
        e = rows[:, None] * d + cols[None, :]
        x0 = mix(key + (2 * e + 1) * g)
        x1 = mix(key + (2 * e + 2) * g)
        u1 = (lsr(x0, 11).to(torch.float64) + 1.0) * 2.0 ** -53
        u2 = lsr(x1, 11).to(torch.float64) * 2.0 ** -53
        z = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(2.0 * math.pi * u2)
        out[r0:r1] = (std * z).to(torch.float32).to(tdt)
    return out


# ----------------------------------------------------------------------------------------
# Zipf ids
# ----------------------------------------------------------------------------------------

@lru_cache(maxsize=8)
def _zipf_cdf(V: int, s: float) -> np.ndarray:
    w = np.arange(1, V + 1, dtype=np.float64) ** (-s)
    c = np.cumsum(w)
    return c / c[-1]


@lru_cache(maxsize=8)
def _id_perm(seed: int, V: int) -> np.ndarray:
    return np.random.default_rng([seed, 2]).permutation(V).astype(np.int32)


def _zipf_ids(rng, n: int, V: int, s: float, seed: int) -> np.ndarray:
    ranks = np.searchsorted(_zipf_cdf(V, s), rng.random(n), side="right")
    ranks = np.minimum(ranks, V - 1)
    return _id_perm(seed, V)[ranks]


# ----------------------------------------------------------------------------------------
# per-user sequences
# ----------------------------------------------------------------------------------------

_ACTION_P = np.array([1.0 / (k + 1) for k in range(N_ACTION)])
_ACTION_P /= _ACTION_P.sum()


def _hist_len(rng, hist) -> int:
    kind = hist[0]
    if kind == "uniform":
        return int(rng.integers(hist[1], hist[2] + 1))
    if kind == "fixed":
        return int(hist[1])
    if kind == "lognormal":
        med, sigma, lo, hi = hist[1:]
        return int(np.clip(round(float(np.exp(rng.normal(math.log(med), sigma)))), lo, hi))
    raise ValueError(kind)


def _gap(rng, gaps) -> int:
    w = np.array([g[0] for g in gaps])
    k = int(rng.choice(len(gaps), p=w / w.sum())) if len(gaps) > 1 else 0
    return max(1, int(math.ceil(rng.exponential(gaps[k][1]))))


@dataclass
class UserSeq:
    n: int
    m: int
    item_ids: np.ndarray  # int32 [n+m]
    action_ids: np.ndarray  # int32 [n+m]; candidates carry N_ACTION
    ts: np.ndarray  # int64 [n+m]; candidates carry t_req
    labels: np.ndarray | None  # float32 [m]


def make_user(cfg: Config, u: int, seed: int | None = None, n: int | None = None,
              m: int | None = None) -> UserSeq:
    seed = cfg.seed if seed is None else seed
    rng = np.random.default_rng([seed, 10, u])
    n = _hist_len(rng, cfg.hist) if n is None else n
    m = cfg.m if m is None else m
    ts_h = np.empty(n, dtype=np.int64)
    t = TS_BASE + int(rng.integers(0, 86400))
    i = 0
    first = True
    while i < n:
        if not first:
            t += _gap(rng, cfg.gaps)
        first = False
        g = int(rng.geometric(1.0 / cfg.group_mean))
        ts_h[i:i + g] = t
        i += g
    t_req = t + _gap(rng, cfg.gaps)
    items = _zipf_ids(rng, n + m, cfg.n_item, cfg.zipf_s, seed)
    acts = np.full(n + m, N_ACTION, dtype=np.int32)
    acts[:n] = rng.choice(N_ACTION, size=n, p=_ACTION_P)
    ts = np.concatenate([ts_h, np.full(m, t_req, dtype=np.int64)])
    labels = (rng.random(m) < cfg.label_p).astype(np.float32) if cfg.training else None
    return UserSeq(n, m, items.astype(np.int32), acts, ts, labels)


@dataclass
class Batch:
    cfg: Config
    users: list  # global user indices held by this batch
    seq_offsets: np.ndarray  # int32 [B+1]
    hist_len: np.ndarray  # int32 [B]
    item_ids: np.ndarray  # int32 [T]
    action_ids: np.ndarray  # int32 [T]
    ts: np.ndarray  # int64 [T]
    labels: np.ndarray | None  # float32 [sum m]

    @property
    def B(self) -> int:
        return len(self.hist_len)

    @property
    def T(self) -> int:
        return int(self.seq_offsets[-1])

    @property
    def cand_count(self) -> np.ndarray:
        return np.diff(self.seq_offsets).astype(np.int64) - self.hist_len


def make_batch(cfg: Config, users=None, seed: int | None = None, hist_override=None,
               m_override=None) -> Batch:
    """Batch of users (all ``cfg.B`` by default) laid out history-then-candidates."""
    users = list(range(cfg.B)) if users is None else list(users)
    seqs = []
    for k, u in enumerate(users):
        n = None if hist_override is None else int(hist_override[k])
        m = None if m_override is None else int(m_override[k])
        seqs.append(make_user(cfg, u, seed, n, m))
    lens = np.array([s.n + s.m for s in seqs], dtype=np.int64)
    off = np.zeros(len(seqs) + 1, dtype=np.int64)
    off[1:] = np.cumsum(lens)
    cat = (lambda xs, dt: np.concatenate(xs).astype(dt) if xs else np.zeros(0, dt))
    labels = None
    if cfg.training:
        labels = cat([s.labels for s in seqs], np.float32)
    return Batch(cfg, users, off.astype(np.int32), np.array([s.n for s in seqs], np.int32),
                 cat([s.item_ids for s in seqs], np.int32),
                 cat([s.action_ids for s in seqs], np.int32),
                 cat([s.ts for s in seqs], np.int64), labels)


# ----------------------------------------------------------------------------------------
# tables and weights
# ----------------------------------------------------------------------------------------

@dataclass
class Model:
    cfg: Config
    action_tab: np.ndarray  # [9, d]; row 8 = mask action M
    pos_tab: np.ndarray  # [n_pos, d]
    ri_tab: np.ndarray  # [n_ri, d]
    rt_tab: np.ndarray  # [n_rt, d]
    layers: list = field(default_factory=list)  # dicts of Wq, Wk, Wv, Wo (+ W1, W2)
    w_head: np.ndarray | None = None  # [d]

    def item_rows(self, rows) -> np.ndarray:
        c = self.cfg
        return item_rows(c.seed, rows, c.d, c.dtype)


def make_model(cfg: Config, seed: int | None = None) -> Model:
    seed = cfg.seed if seed is None else seed
    d, dt = cfg.d, cfg.dtype
    rt = np.random.default_rng([seed, 20])
    tab = lambda r: _cast(rt.normal(0.0, 0.02, size=(r, d)), dt)  # noqa: E731
    action, pos, ri, rtt = tab(cfg.n_action_rows), tab(cfg.n_pos), tab(cfg.n_ri), tab(cfg.n_rt)
    rw = np.random.default_rng([seed, 30])
    w = lambda *s: _cast(rw.normal(0.0, 0.02, size=s), dt)  # noqa: E731
    layers = []
    for _ in range(cfg.layers):
        L = {"Wq": w(d, d), "Wk": w(d, d), "Wv": w(d, d), "Wo": w(d, d)}
        if cfg.ffn:
            L["W1"] = w(d, 4 * d)
            L["W2"] = w(4 * d, d)
        layers.append(L)
    return Model(cfg, action, pos, ri, rtt, layers, w(d))


def make_qkv(cfg: Config, T: int, seed: int, std: float = 1.0, n: int = 3) -> np.ndarray:
    """Standalone attention operands: ``n`` arrays [T, H, dh] stacked as [T, n, H, dh]."""
    rng = np.random.default_rng([seed, 40])
    return _cast(rng.normal(0.0, std, size=(T, n, cfg.H, cfg.dh)), cfg.dtype)


# ----------------------------------------------------------------------------------------
# comparison inputs: the interleaved layout and a dense per-user bias
# ----------------------------------------------------------------------------------------

def interleave_batch(batch: Batch) -> Batch:
    """The same users laid out as the interleaved organisation does: each history
    interaction becomes two tokens (the item, then its action; both at the interaction's
    time), followed by the candidates.  Item ids of action tokens are the action index;
    only the layout matters to the attention that consumes it."""
    offs, hl, items, acts, ts = [0], [], [], [], []
    for u in range(batch.B):
        s, e, n = int(batch.seq_offsets[u]), int(batch.seq_offsets[u + 1]), int(batch.hist_len[u])
        it2 = np.empty(2 * n, np.int32)
        it2[0::2] = batch.item_ids[s:s + n]
        it2[1::2] = batch.action_ids[s:s + n]
        ac2 = np.empty(2 * n, np.int32)
        ac2[0::2] = batch.action_ids[s:s + n]
        ac2[1::2] = batch.action_ids[s:s + n]
        items += [it2, batch.item_ids[s + n:e]]
        acts += [ac2, batch.action_ids[s + n:e]]
        ts += [np.repeat(batch.ts[s:s + n], 2), batch.ts[s + n:e]]
        hl.append(2 * n)
        offs.append(offs[-1] + 2 * n + (e - s - n))
    cat = (lambda xs, dt: np.concatenate(xs).astype(dt) if xs else np.zeros(0, dt))
    return Batch(batch.cfg, list(batch.users), np.array(offs, np.int32), np.array(hl, np.int32),
                 cat(items, np.int32), cat(acts, np.int32), cat(ts, np.int64), batch.labels)


def dense_bias_torch(seed: int, B: int, Lpad: int, device, std: float = 0.5):
    """A bf16 [B, Lpad, Lpad] tensor of N(0, std) values (a stand-in for a learned
    relative bias), drawn on ``device`` by a seeded torch generator."""
    import torch

    g = torch.Generator(device=device).manual_seed(int(seed))
    return (torch.randn((B, Lpad, Lpad), generator=g, device=device) * std).to(torch.bfloat16)
