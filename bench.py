#!/usr/bin/env python
"""Benchmark of the GenRank hot path on B200.

Default workload (c2): inference scoring, 1024 users, every history at the
480-token maximum, 256 candidates each, d = 512 (8 heads x 64), 4 stacked
layers (pre-RMSNorm attention + 4d SiLU FFN), bf16 with fp32 accumulation,
item table 4M rows with Zipf(1.05) ids, synthetic seeded data.  One step =
embedding assembly (metadata + five-way gather-sum) -> 4 x [RMSNorm -> fused
QKV projection -> candidate-masked ALiBi attention -> output projection and
residual -> RMSNorm -> FFN] -> final RMSNorm -> candidate head.  Metric:
candidates scored per second (whole job), with the attention kernel's
algorithmic TFLOP/s against the bf16 peak in ``roofline``.  The line also
carries the embedding gather-sum's algorithmic GB/s against HBM bandwidth and
two more kernel rooflines: the forward on the 1024-candidate sweep point and the
backward on the training workload's shapes.

    python bench.py [--gpus N --steps K --warmup W] [--config c2|c1|c3|c4_m64|...]
                    [--impl reference] [--no-cpu-baseline]

``--config c3`` times the training step (forward, mean BCE over candidates,
backward through the blocks, the attention and the embedding assembly) and
reports the attention backward's roofline.

Multi-GPU: one process per GPU (torchrun), each rank takes its own shard of
users (weak scaling, no collective on the data path); the step time is the max
over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "candidates scored/sec and attention TFLOP/s (% of B200 bf16 tensor peak)"
UNIT = "candidates/s"
DEFAULT_CONFIG = "c2"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_fwd_tc_traffic.json")
CSRC = os.path.join(ROOT, "generative_ranking_recommendation_b200", "csrc")
L2_FLUSH_BYTES = 256 << 20  # larger than the 126 MB L2


# ------------------------------------------------------------------------------------------
# workload arithmetic
# ------------------------------------------------------------------------------------------
def attn_pairs(seq_offsets, hist_len) -> int:
    """Visible (query, key) pairs: n(n+1)/2 causal history + m n candidates x history + m self."""
    n = np.asarray(hist_len, np.int64)
    m = np.diff(np.asarray(seq_offsets, np.int64)) - n
    return int(np.sum(n * (n + 1) // 2 + m * n + m))


def attn_flops(seq_offsets, hist_len, d, backward=False) -> float:
    """4 d flops per visible pair forward (Q K^T and P V), 10 d backward."""
    return (10.0 if backward else 4.0) * d * attn_pairs(seq_offsets, hist_len)


def embed_bytes(T, d, elem) -> float:
    """Item row read + E row written + ids/ts read + 3 int32 metadata written, per token."""
    return float(T) * (2 * d * elem + 4 + 4 + 8 + 12)


def embed_bwd_bytes(T, d, elem) -> float:
    """dE row read + the fp32 item-row reduction + ids and metadata, per token."""
    return float(T) * (d * elem + 4 * d + 28)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(src="attn_tc.cu") -> str:
    with open(os.path.join(CSRC, src), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def measured_traffic(workload: str):
    """DRAM bytes per launch of the attention kernel from an ncu capture, if it was
    taken on the current kernel source; else None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("source_sha256_16") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


# ------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k] == "Active"})
        loaded = [x for x in sm if x > 0.5 * (max(mx) if mx else 1)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------------------------------------
# CPU baseline: the float64 oracle on the host cores (process pool over users)
# ------------------------------------------------------------------------------------------
_ORACLE_MODELS = {}


def _oracle_user(args):
    """One user's step in the float64 oracle (users are independent): metadata, embedding
    sum, the blocks and the head; for a training workload also the mean-BCE backward
    through the blocks and the table gradients.  Returns the user's candidate count."""
    name, u = args
    import oracle
    from gen import CONFIGS, make_batch, make_model

    cfg = CONFIGS[name]
    mdl = _ORACLE_MODELS.get(name)
    if mdl is None:  # weights are drawn once per worker, outside the per-user work
        mdl = _ORACLE_MODELS[name] = make_model(cfg)
    b = make_batch(cfg, users=[u])
    uniq, ids = np.unique(b.item_ids, return_inverse=True)
    meta = oracle.token_metadata(b.seq_offsets, b.hist_len, b.ts, cfg.n_ri, cfg.n_rt)
    E = oracle.embed_assemble(b.seq_offsets, b.hist_len, ids, b.action_ids, meta,
                              mdl.item_rows(uniq), mdl.action_tab, mdl.pos_tab, mdl.ri_tab,
                              mdl.rt_tab)
    z, cache = oracle.block_forward(E, mdl.layers, mdl.w_head, b.seq_offsets, b.hist_len,
                                    meta[0], b.ts, cfg.H, cfg.ffn)
    if cfg.training:
        oracle.bce_loss(z, b.labels)
        dE = oracle.block_backward(z, b.labels, cache, mdl.layers, mdl.w_head, b.seq_offsets,
                                   b.hist_len, meta[0], b.ts, cfg.H, cfg.ffn)
        oracle.embed_assemble_bwd(dE, b.seq_offsets, b.hist_len, ids, b.action_ids, meta,
                                  len(uniq), cfg.n_action_rows, cfg.n_pos, cfg.n_ri, cfg.n_rt)
    return len(z)


def _pool(cores):
    """Spawned workers, one BLAS thread each (one user per task)."""
    import multiprocessing as mp

    for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[k] = "1"
    return mp.get_context("spawn").Pool(cores)


def _user_pairs(cfg, users):
    """Visible attention pairs of each of ``users`` (their lengths only)."""
    from gen import make_batch

    b = make_batch(cfg, users=list(users))
    return np.array([attn_pairs(b.seq_offsets[k:k + 2] - b.seq_offsets[k], b.hist_len[k:k + 1])
                     for k in range(len(users))], np.float64)


def cpu_baseline(name: str, B: int, target_s: float = 10.0):
    """The oracle timed on one core and on all cores, each on a bounded seeded sample of
    the workload's users, extrapolated to the whole batch by visible attention pairs
    (the oracle's cost is dominated by its per-user attention and projections, which
    scale with the pairs and the tokens alike)."""
    from gen import CONFIGS

    cfg = CONFIGS[name]
    cores = max(1, len(os.sched_getaffinity(0)))
    rng = np.random.default_rng(12345)
    order = rng.permutation(B).tolist()
    all_pairs = float(np.sum(_user_pairs(cfg, range(B))))
    total_cands = B * cfg.m

    def leg(n_workers, users):
        with _pool(n_workers) as pool:
            pool.map(_oracle_user, [(name, users[0])] * n_workers)  # imports and weights
            t0 = time.perf_counter()
            cands = sum(pool.map(_oracle_user, [(name, u) for u in users], chunksize=1))
            dt = time.perf_counter() - t0
        sp = float(np.sum(_user_pairs(cfg, users)))
        est = dt * all_pairs / sp  # seconds for the whole batch
        return {"value": total_cands / est, "seconds": dt, "users": len(users),
                "candidates": int(cands), "extrapolated_batch_seconds": est}

    # one core: as many users as fit the target time (at least 2)
    with _pool(1) as pool:
        pool.map(_oracle_user, [(name, order[0])])
        t0 = time.perf_counter()
        pool.map(_oracle_user, [(name, order[1])])
        per_user = time.perf_counter() - t0
    n1 = int(min(B, max(2, round(target_s / max(per_user, 1e-3)))))
    one = leg(1, order[:n1])
    # all cores: at least 64 users (or the whole batch), about target_s of wall time
    nn = int(min(B, max(64, cores * round(target_s / max(per_user, 1e-3)))))
    many = leg(cores, order[:nn])
    what = "training step (forward, loss, backward)" if cfg.training else "scoring pass"
    return {"value": many["value"], "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"float64 numpy oracle, one {what} per user; {many['users']} seeded-random "
                      f"users of the {B} ({many['candidates']} candidates) in a {cores}-process "
                      f"pool, {many['seconds']:.1f} s, extrapolated to the whole batch by "
                      f"visible attention pairs",
            "seconds": many["seconds"],
            "one_core": {"value": one["value"], "unit": UNIT, "cores": 1,
                         "sample": f"{one['users']} seeded-random users ({one['candidates']} "
                                   f"candidates) in one process, {one['seconds']:.1f} s, "
                                   f"extrapolated by visible attention pairs",
                         "seconds": one["seconds"]}}


# ------------------------------------------------------------------------------------------
# arms
# ------------------------------------------------------------------------------------------
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_users(B_per_rank: int, rank: int):
    """The users rank `rank` scores: its own block of B_per_rank (weak scaling; users
    are independent, so no data crosses ranks)."""
    return list(range(rank * B_per_rank, (rank + 1) * B_per_rank))


def max_over_ranks(values, world: int, device):
    """Element-wise max over ranks of a list of floats (the slowest rank's times)."""
    if world == 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def history_label(hist) -> str:
    kind = hist[0]
    if kind == "uniform":
        return f"history lengths U[{hist[1]},{hist[2]}]"
    if kind == "fixed":
        return f"every history at {hist[1]} tokens"
    if kind == "lognormal":
        med, sigma, lo, hi = hist[1:]
        return f"history lengths lognormal(median {med:g}, sigma {sigma:g}) clipped to [{lo},{hi}]"
    raise ValueError(f"unknown history kind {kind!r}")


def workload_label(cfg) -> str:
    mode = ("training step (forward, mean BCE over candidates, backward)" if cfg.training
            else "inference scoring (forward only)")
    blocks = (f"{cfg.layers} layers (pre-RMSNorm attention + 4d SiLU FFN, final RMSNorm)"
              if cfg.ffn else f"{cfg.layers} layer (h = E + Attn(E) W_o)")
    return (f"{mode}, {cfg.name}: {cfg.B} users/GPU, {history_label(cfg.hist)}, {cfg.m} "
            f"candidates each, d={cfg.d} ({cfg.H}x{cfg.dh}), {blocks}, {cfg.dtype}, item table "
            f"{cfg.n_item} rows, Zipf({cfg.zipf_s:g}) ids")


def config_block(cfg, world, extra=None):
    c = {"workload": workload_label(cfg), "config": cfg.name,
         "global_batch_users": cfg.B * world, "candidates_per_step": cfg.B * cfg.m * world,
         "parallelism": f"users sharded over {world} GPU(s), no collective on the data path",
         "l2": "flushed (256 MB write) before every device-timed step and kernel launch; the "
               "pipelined e2e loop is not flushed (a step's working set, with the item table, "
               "is several times the 126 MB L2)"}
    if extra:
        c.update(extra)
    return c


def run_reference(args, cfg, world, rank):
    """The oracle as the reference arm: each step runs a bounded sample of users."""
    if rank != 0:
        return
    cores = max(1, len(os.sched_getaffinity(0)))
    users_per_step = cores
    with _pool(cores) as pool:
        times = []
        cands = 0
        for k in range(args.warmup + args.steps):
            batch_users = [(cfg.name, (k * users_per_step + j) % cfg.B) for j in range(users_per_step)]
            t0 = time.perf_counter()
            c = sum(pool.map(_oracle_user, batch_users, chunksize=1))
            dt = time.perf_counter() - t0
            if k >= args.warmup:
                times.append(dt)
                cands += c
    total = sum(times)
    value = cands / total
    what = "training step" if cfg.training else "scoring pass"
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded generator shaped like the pages' workloads)",
           "config": config_block(cfg, 1, {"reference_sample": f"{users_per_step} users per step"}),
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                            "sample": f"{users_per_step} users of the workload per step, one "
                                      f"float64 oracle {what} per user, {cores}-process pool"},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


class Timer:
    """Device time of a callable captured once as a CUDA graph and replayed, with L2
    flushed before each replay; events bracket the replay only, on the current stream."""

    def __init__(self, torch, flush):
        self.torch = torch
        self.flush = flush

    def graph(self, fn, warmup=2):
        torch = self.torch
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(max(1, warmup)):
                fn()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        g.replay()
        torch.cuda.synchronize()
        return g

    def time(self, run, n, name="timed"):
        torch = self.torch
        ev = []
        for k in range(n):
            self.flush.zero_()
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.nvtx.range_push(name)
            s.record()
            run(k)
            e.record()
            torch.cuda.nvtx.range_pop()
            ev.append((s, e))
        torch.cuda.synchronize()
        return [s.elapsed_time(e) for s, e in ev]


def _attention_kernel_line(torch, G, timer, cfg, steps, backward, peak, peak_src, dev):
    """Roofline line of the attention forward or backward alone on ``cfg``'s batch shapes,
    with unit-scale random bf16 operands resident in HBM."""
    from gen import make_batch

    batch = make_batch(cfg)
    T, H, dh, d = batch.T, cfg.H, cfg.dh, cfg.d
    off = torch.from_numpy(batch.seq_offsets).to(dev)
    hl = torch.from_numpy(batch.hist_len).to(dev)
    ts = torch.from_numpy(batch.ts).to(dev)
    pos = np.zeros(T, np.int32)
    for u in range(batch.B):
        s, e, n = batch.seq_offsets[u], batch.seq_offsets[u + 1], batch.hist_len[u]
        pos[s:s + n] = np.arange(1, n + 1)
        pos[s + n:e] = n + 1
    pos = torch.from_numpy(pos).to(dev)
    msl = int(np.max(np.diff(batch.seq_offsets)))
    gen = torch.Generator(device=dev).manual_seed(cfg.seed)
    qkv = torch.randn((T, 3 * d), device=dev, generator=gen).to(torch.bfloat16)
    o = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((H, T), dtype=torch.float32, device=dev)
    ws = torch.empty(G.attn_workspace_size(batch.B, T, H, dh, msl, backward), dtype=torch.uint8,
                     device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    sp, st = G.alibi_slopes(H)
    scale = 1.0 / math.sqrt(dh)

    def fwd():
        G.attn_fwd(off, hl, msl, qkv, qkv[:, d:], qkv[:, 2 * d:], 3 * d, H, dh, pos, ts, sp, st,
                   scale, o, d, lse, ws if not backward else wsf, err, T=T)

    if backward:
        wsf = torch.empty(G.attn_workspace_size(batch.B, T, H, dh, msl, False),
                          dtype=torch.uint8, device=dev)
        fwd()
        do = torch.randn((T, d), device=dev, generator=gen).to(torch.bfloat16)
        dqkv = torch.empty_like(qkv)

        def fn():
            G.attn_bwd(off, hl, msl, qkv, qkv[:, d:], qkv[:, 2 * d:], 3 * d, H, dh, pos, ts, sp,
                       st, scale, o, do, d, lse, dqkv, dqkv[:, d:], dqkv[:, 2 * d:], ws, err, T=T)
        kernel = "k_attn_bwd_tc (+ prologue, per-row, candidate and finishing passes)"
    else:
        fn = fwd
        kernel = "k_attn_fwd_tc (+ prologue)"
    g = timer.graph(fn)
    ms = float(np.mean(timer.time(lambda k: g.replay(), steps, name="timed_kernel")))
    assert G.check_error(err) == 0, "device error flags raised in a kernel timing"
    flops = attn_flops(batch.seq_offsets, batch.hist_len, d, backward)
    ach = flops / (ms / 1e3) / 1e12
    return {"kernel": kernel, "workload": f"{cfg.name} shapes ({batch.B} users, T={T}, "
                                          f"{H}x{dh}), random unit-scale bf16 operands",
            "bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
            "frac": ach / peak, "peak_source": peak_src, "avg_launch_ms": ms,
            "algorithmic_flops_per_launch": flops}


def _linear_kernel_lines(torch, G, timer, cfg, steps, peak, peak_src, hbm, hbm_src, dev):
    """Roofline lines of the four-layer block's linear layers (library tensor-core GEMMs
    with fused epilogues) at the workload's token count, on random bf16 operands: 2 M N K
    algorithmic flops each, and for the residual + RMSNorm layers also their algorithmic
    HBM bytes (A in, the fp32 residual in and out, the bf16 normalised row out)."""
    from gen import make_batch

    T = make_batch(cfg).T
    d = cfg.d
    gen = torch.Generator(device=dev).manual_seed(7)
    bf = torch.bfloat16
    a = torch.randn((T, d), device=dev, generator=gen).to(bf)
    u = torch.randn((T, 4 * d), device=dev, generator=gen).to(bf)
    x = torch.randn((T, d), device=dev, generator=gen)
    ws = {"qkv": (torch.randn((3 * d, d), device=dev, generator=gen) / d ** 0.5).to(bf),
          "w1": (torch.randn((4 * d, d), device=dev, generator=gen) / d ** 0.5).to(bf),
          "wo": (torch.randn((d, d), device=dev, generator=gen) / d ** 0.5).to(bf),
          "w2": (torch.randn((d, 4 * d), device=dev, generator=gen) / (4 * d) ** 0.5).to(bf)}
    out3 = torch.empty((T, 3 * d), dtype=bf, device=dev)
    out4 = torch.empty((T, 4 * d), dtype=bf, device=dev)
    a2 = torch.empty((T, d), dtype=bf, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    cases = [("QKV projection (store)", 3 * d, d, None,
              lambda: G.linear(a, ws["qkv"], out3, err)),
             ("W1 (SiLU epilogue)", 4 * d, d, None,
              lambda: G.linear(a, ws["w1"], out4, err, epilogue=G.EPI_SILU)),
             ("W_o (residual + RMSNorm epilogue)", d, d, T * (2 * d + 8 * d + 2 * d),
              lambda: G.linear_residual_rmsnorm(a, ws["wo"], x, x, a2, err)),
             ("W2 (residual + RMSNorm epilogue)", d, 4 * d, T * (8 * d + 8 * d + 2 * d),
              lambda: G.linear_residual_rmsnorm(u, ws["w2"], x, x, a2, err))]
    lines = []
    for name, N, K, nbytes, fn in cases:
        g = timer.graph(fn)
        ms = float(np.mean(timer.time(lambda k: g.replay(), steps, name="timed_kernel")))
        fl = 2.0 * T * N * K
        line = {"kernel": f"k_gemm_tc: {name}", "workload": f"{cfg.name} token count "
                f"(M={T}, N={N}, K={K}), random bf16 operands", "bound": "tensor",
                "achieved": fl / (ms / 1e3) / 1e12, "peak": peak, "unit": "TFLOP/s",
                "frac": fl / (ms / 1e3) / 1e12 / peak, "peak_source": peak_src,
                "avg_launch_ms": ms, "algorithmic_flops_per_launch": fl}
        if nbytes:
            gbs = nbytes / (ms / 1e3) / 1e9
            line["hbm"] = {"achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                           "peak_source": hbm_src, "algorithmic_bytes_per_launch": nbytes}
        lines.append(line)
    assert G.check_error(err) == 0, "device error flags raised in a kernel timing"
    return lines


def run_native(args, cfg, world, rank, local):
    import torch
    import torch.distributed as dist

    from gen import CONFIGS, make_batch, make_model
    from generative_ranking_recommendation_b200 import genrank as G
    from generative_ranking_recommendation_b200.model import CapturedStep, DeviceBatch, GenRankModel

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev)

    users = rank_users(cfg.B, rank)
    batches = [make_batch(cfg, users=users, seed=cfg.seed + 1000 * k) for k in range(2)]
    mdl = make_model(cfg)
    gm = GenRankModel(cfg, mdl, dev)
    dbs = [DeviceBatch.from_batch(b, dev) for b in batches]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    timer = Timer(torch, flush)
    peaks, src = load_peaks()
    es = 2 if cfg.dtype == "bf16" else 4

    def sync_all():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    training = cfg.training
    if training:
        # one training step per batch, run eagerly (torch autograd drives the blocks around
        # the library's attention and embedding backward calls)
        def step(k):
            loss, _, grads = gm.train_step(dbs[k % 2])
            return loss
        for k in range(args.warmup):
            step(k)
        torch.cuda.synchronize()
        assert G.check_error(gm.err) == 0, "device error flags raised during warm-up"
        run_step = step
    else:
        for k in range(args.warmup):
            gm.forward(dbs[k % 2])
        torch.cuda.synchronize()
        assert G.check_error(gm.err) == 0, "device error flags raised during warm-up"
        # each batch's step as a CUDA graph (no host launch work inside the step)
        steps = [CapturedStep(gm, db) for db in dbs]
        for k in range(args.warmup):
            steps[k % 2].run()
        torch.cuda.synchronize()
        run_step = lambda k: steps[k % 2].run()  # noqa: E731

    # ---- device-resident inputs, one step per timed iteration
    sampler = ClockSampler(local)
    sync_all()
    sampler.start()
    step_ms = timer.time(run_step, args.steps, name="timed_step")
    clocks = sampler.stop()
    total_ms = sum(step_ms)

    # ---- the dominant kernels alone (their own graphs), for the rooflines
    if not training:
        attn = [CapturedStep(gm, db, part="attention") for db in dbs]
        attn_ms = timer.time(lambda k: attn[k % 2].run(), args.steps, name="timed_attention")
        embed = [CapturedStep(gm, db, part="embed") for db in dbs]
        embed_ms = timer.time(lambda k: embed[k % 2].run(), args.steps, name="timed_embed")
        del attn, embed

    # ---- end to end through the public API: pinned host inputs -> device -> result -> host
    host = [DeviceBatch.host_arrays(b) for b in batches]
    pinned = [[torch.from_numpy(np.ascontiguousarray(a)).pin_memory() for a in h] for h in host]
    h2d = sum(p.numel() * p.element_size() for p in pinned[0])
    comp = torch.cuda.current_stream()
    if training:
        # each step uploads its batch (labels included), trains on it and reads the loss back
        loss_host = torch.empty(1, dtype=torch.float32).pin_memory()
        d2h = 4

        def e2e_loop(n):
            for k in range(n):
                i = k % 2
                for d_, s_ in zip([dbs[i].seq_offsets, dbs[i].hist_len, dbs[i].item_ids,
                                   dbs[i].action_ids, dbs[i].ts, dbs[i].cand_rows,
                                   dbs[i].labels], pinned[i]):
                    d_.copy_(s_, non_blocking=True)
                loss, _, _ = gm.train_step(dbs[i])
                loss_host.copy_(loss.reshape(1), non_blocking=True)
    else:
        n_cand = [int(b.cand_count.sum()) for b in batches]
        out_host = [torch.empty(n, dtype=torch.float32).pin_memory() for n in n_cand]
        d2h = out_host[0].numel() * out_host[0].element_size()
        # Pipelined as a serving loop runs it: step k+1's inputs cross PCIe on a copy
        # stream while step k computes (each captured step owns its device buffers, so a
        # buffer is reloaded only after the step two back has finished with it); every
        # step still uploads its inputs and reads its logits back inside the timed span.
        copy = torch.cuda.Stream(device=dev)
        loaded = [torch.cuda.Event() for _ in range(2)]
        done = [torch.cuda.Event() for _ in range(2)]

        def e2e_loop(n):
            for k in range(n):
                i = k % 2
                with torch.cuda.stream(copy):
                    if k >= 2:
                        copy.wait_event(done[i])
                    steps[i].load(pinned[i])
                    loaded[i].record(copy)
                comp.wait_event(loaded[i])
                out_host[i].copy_(steps[i].run(), non_blocking=True)
                done[i].record(comp)

    e2e_loop(2)
    sync_all()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(comp)
    if not training:
        copy.wait_stream(comp)
    e2e_loop(args.steps)
    if not training:
        comp.wait_stream(copy)
    e.record(comp)
    sync_all()
    e2e_ms = s.elapsed_time(e)
    assert G.check_error(gm.err) == 0, "device error flags raised during the timed region"
    if not training:
        del steps

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], world, dev)

    # ---- extra kernel lines (rank 0 only, after the timed and collective parts)
    peak_burst = float(peaks["bf16_tflops"])
    hbm = float(peaks["hbm_gbs"])
    burst_src = f"{src} bf16 (burst, cuBLAS GEMM)"
    kernels = []
    if rank == 0 and training:  # the training step's roofline is the attention backward
        kernels.append(_attention_kernel_line(torch, G, timer, cfg, args.steps, True,
                                              peak_burst, burst_src, dev))
    if rank == 0 and not args.no_extra_kernels:
        if training:
            kernels.append(_attention_kernel_line(torch, G, timer, cfg, args.steps, False,
                                                  peak_burst, burst_src, dev))
        else:
            for extra_cfg, bwd in ((CONFIGS["c4_m1024"], False), (CONFIGS["c3"], True)):
                if extra_cfg.name != cfg.name:
                    kernels.append(_attention_kernel_line(torch, G, timer, extra_cfg,
                                                          args.steps, bwd, peak_burst,
                                                          burst_src, dev))
            if gm.fused_blocks:
                kernels += _linear_kernel_lines(torch, G, timer, cfg, args.steps, peak_burst,
                                                burst_src, hbm, f"{src} HBM copy bandwidth",
                                                dev)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return

    cands_per_step = cfg.B * cfg.m * world
    value = cands_per_step / (total_ms / args.steps / 1e3)
    T_avg = float(np.mean([b.T for b in batches]))
    if training:
        bwd = kernels[0]
        roofline = {"bound": "tensor", "kernel": "k_attn_bwd_tc (attention backward call)",
                    "achieved": bwd["achieved"], "peak": bwd["peak"], "unit": "TFLOP/s",
                    "frac": bwd["frac"], "peak_source": bwd["peak_source"], "traffic": None,
                    "algorithmic_flops_per_launch": bwd["algorithmic_flops_per_launch"],
                    "avg_launch_ms": bwd["avg_launch_ms"],
                    "note": "timed alone on the step's shapes, one layer's call"}
        embed_line = None
    else:
        flops = float(np.mean([attn_flops(b.seq_offsets, b.hist_len, cfg.d) for b in batches]))
        attn_avg_ms = float(np.mean(attn_ms))
        achieved = flops / (attn_avg_ms / 1e3) / 1e12
        roofline = {"bound": "tensor", "kernel": "k_attn_fwd_tc", "achieved": achieved,
                    "peak": peak_burst, "unit": "TFLOP/s", "frac": achieved / peak_burst,
                    "peak_source": burst_src, "traffic": measured_traffic(cfg.name),
                    "algorithmic_flops_per_launch": flops, "avg_launch_ms": attn_avg_ms,
                    "note": "one layer's attention call (prologue + kernel) timed alone on its "
                            "own graph; avg_launch_ms includes the prologue.  On the fused "
                            "four-layer step the W2 linear layer's kernel has about the same "
                            "share of device time (its line is in kernels)"}
        emb_ms = float(np.mean(embed_ms))
        gbs = embed_bytes(T_avg, cfg.d, es) / (emb_ms / 1e3) / 1e9
        embed_line = {"kernel": "k_token_meta + k_embed_fwd (genrank_embed_assemble)",
                      "bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                      "frac": gbs / hbm, "peak_source": f"{src} HBM copy bandwidth",
                      "avg_launch_ms": emb_ms,
                      "algorithmic_bytes_per_launch": embed_bytes(T_avg, cfg.d, es)}
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if cfg.dtype == "bf16" else "f32",
        "data": "synthetic (seeded generator shaped like the pages' workloads; random-init "
                "tables and weights)",
        "config": config_block(cfg, world),
        "attention_tflops": roofline["achieved"],
        "attention_pct_of_bf16_peak": 100.0 * roofline["frac"],
        "roofline": roofline,
        "e2e": {"value": cands_per_step / (e2e_ms / args.steps / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)},
        # per step: metadata scan + gather-sum (with the first RMSNorm on the fused
        # blocks), attention prologue + kernel per layer, on the fused blocks the four
        # linear layers per layer (QKV, W_o, W1, W2) and the last layer's two candidate-row
        # gathers, and for training the backward's five
        # kernels per layer plus the embedding backward; a one-block model without FFN
        # adds the fused candidate head
        "gpu_launches": args.steps * (2 + 2 * cfg.layers + (5 * cfg.layers + 1 if training else 0)
                                      + (4 * cfg.layers + 2 if (gm.fused_blocks and not training)
                                         else 0)
                                      + (0 if (cfg.ffn or cfg.layers > 1 or training) else 1)),
        "clocks": clocks,
    }
    if embed_line is not None:
        out["embedding"] = embed_line
    if kernels:
        out["kernels"] = kernels
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(cfg.name, cfg.B)
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra-kernels", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from gen import CONFIGS

    cfg = CONFIGS[args.config]
    world, rank, local = dist_setup()
    if args.impl == "reference":
        run_reference(args, cfg, world, rank)
    else:
        run_native(args, cfg, world, rank, local)


if __name__ == "__main__":
    main()
