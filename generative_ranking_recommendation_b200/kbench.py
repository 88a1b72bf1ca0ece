"""Per-kernel benchmark of the hot path on one workload configuration.

    python -m generative_ranking_recommendation_b200.kbench --config c2 \
        [--kernels embed_fwd,attn_fwd,attn_bwd,embed_bwd,linear,bucketed,cached,hstu]
        [--iters 20] [--warmup 3] [--users B]

Times each library call with CUDA events around a replay of the call captured as
a CUDA graph (inputs resident in HBM, L2 flushed before every timed replay) and prints one JSON line per kernel with its
algorithmic throughput: GB/s for the embedding kernels, TFLOP/s for attention
(4 d flops per visible pair forward, 10 d backward; masked pairs and padding
not counted).  Attention operands are unit-scale random bf16 values.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from gen import CONFIGS, item_table_torch, make_batch, make_model  # noqa: E402

from . import genrank as G  # noqa: E402


def visible_pairs(off, hl):
    n = np.asarray(hl, np.int64)
    m = np.diff(np.asarray(off, np.int64)) - n
    return int(np.sum(n * (n + 1) // 2 + m * n + m))


def positions(batch):
    pos = np.zeros(batch.T, np.int32)
    for u in range(batch.B):
        s, e, n = batch.seq_offsets[u], batch.seq_offsets[u + 1], batch.hist_len[u]
        pos[s:s + n] = np.arange(1, n + 1)
        pos[s + n:e] = n + 1
    return pos


def timed(fn, iters, warmup, flush):
    """Median device time of one call of fn.  The call is captured once as a CUDA
    graph and replayed, so host work inside it (argument marshalling, tensor-map
    encoding) cannot idle the GPU inside the timed span; L2 is flushed before each
    replay."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(max(1, warmup)):
            fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fn()
    graph.replay()
    torch.cuda.synchronize()
    ts = []
    for _ in range(iters):
        flush.zero_()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        graph.replay()
        e.record()
        ts.append((s, e))
    torch.cuda.synchronize()
    return float(np.median([s.elapsed_time(e) for s, e in ts]))


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="c1")
    ap.add_argument("--kernels", default="embed_fwd,attn_fwd,attn_bwd,embed_bwd")
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--users", type=int, default=None, help="batch size (default: the config's)")
    args = ap.parse_args(argv)
    cfg = CONFIGS[args.config]
    if args.users:
        cfg = cfg.with_(B=args.users)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    batch = make_batch(cfg)
    T, H, dh, d = batch.T, cfg.H, cfg.dh, cfg.d
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    es = 2 if cfg.dtype == "bf16" else 4
    off = torch.from_numpy(batch.seq_offsets).to(dev)
    hl = torch.from_numpy(batch.hist_len).to(dev)
    ids = torch.from_numpy(batch.item_ids).to(dev)
    acts = torch.from_numpy(batch.action_ids).to(dev)
    ts = torch.from_numpy(batch.ts).to(dev)
    pos = torch.from_numpy(positions(batch)).to(dev)
    msl = int(np.max(np.diff(batch.seq_offsets)))
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    sp, st = G.alibi_slopes(H)
    scale = 1.0 / math.sqrt(dh)
    kernels = args.kernels.split(",")
    base = {"config": cfg.name, "T": T, "B": batch.B, "H": H, "dh": dh}
    pairs = visible_pairs(batch.seq_offsets, batch.hist_len)

    if "embed_fwd" in kernels or "embed_bwd" in kernels:
        mdl = make_model(cfg)
        item = item_table_torch(cfg.seed, cfg.n_item, d, cfg.dtype, dev)
        tabs = [item] + [torch.from_numpy(x).to(dev, tdt)
                         for x in (mdl.action_tab, mdl.pos_tab, mdl.ri_tab, mdl.rt_tab)]
        E = torch.empty((T, d), dtype=tdt, device=dev)
        meta = [torch.empty(T, dtype=torch.int32, device=dev) for _ in range(3)]

        def fe():
            G.embed_assemble(off, hl, ids, acts, ts, *tabs, E, *meta, err)

        if "embed_fwd" in kernels:
            ms = timed(fe, args.iters, args.warmup, flush)
            nbytes = T * (2 * d * es + 28)
            print(json.dumps({**base, "kernel": "embed_fwd", "ms": ms,
                              "GB_per_s": nbytes / ms / 1e6, "algorithmic_bytes": nbytes}),
                  flush=True)
        if "embed_bwd" in kernels:
            fe()
            dE = torch.randn((T, d), device=dev).to(tdt)
            f32 = dict(dtype=torch.float32, device=dev)
            grads = [torch.zeros(t.shape, **f32) for t in tabs]

            def fb():
                G.embed_assemble_bwd(off, hl, ids, acts, *meta, dE, *grads, err)

            ms = timed(fb, args.iters, args.warmup, flush)
            nbytes = T * (d * es + 4 * d + 28)  # dE read, item-row reduction, ids and metadata
            print(json.dumps({**base, "kernel": "embed_bwd", "ms": ms,
                              "GB_per_s": nbytes / ms / 1e6, "algorithmic_bytes": nbytes}),
                  flush=True)

    if "attn_fwd" in kernels or "attn_bwd" in kernels:
        g = torch.Generator(device=dev)
        g.manual_seed(cfg.seed)
        qkv = torch.randn((T, 3 * d), device=dev, generator=g).to(tdt)
        o = torch.empty((T, d), dtype=tdt, device=dev)
        lse = torch.empty((H, T), dtype=torch.float32, device=dev)
        ws = torch.empty(max(G.attn_workspace_size(batch.B, T, H, dh, msl, False),
                             G.attn_workspace_size(batch.B, T, H, dh, msl, True)),
                         dtype=torch.uint8, device=dev)

        def fa():
            G.attn_fwd(off, hl, msl, qkv, qkv[:, d:], qkv[:, 2 * d:], 3 * d, H, dh, pos, ts, sp,
                       st, scale, o, d, lse, ws, err, T=T)

        if "attn_fwd" in kernels:
            ms = timed(fa, args.iters, args.warmup, flush)
            fl = 4.0 * d * pairs
            print(json.dumps({**base, "kernel": "attn_fwd", "ms": ms, "TFLOP_per_s": fl / ms / 1e9,
                              "algorithmic_flops": fl, "visible_pairs": pairs}), flush=True)
        if "attn_bwd" in kernels:
            fa()
            do = torch.randn((T, d), device=dev, generator=g).to(tdt)
            dqkv = torch.empty_like(qkv)

            def fb():
                G.attn_bwd(off, hl, msl, qkv, qkv[:, d:], qkv[:, 2 * d:], 3 * d, H, dh, pos, ts,
                           sp, st, scale, o, do, d, lse, dqkv, dqkv[:, d:], dqkv[:, 2 * d:], ws,
                           err, T=T)

            ms = timed(fb, args.iters, args.warmup, flush)
            fl = 10.0 * d * pairs
            print(json.dumps({**base, "kernel": "attn_bwd", "ms": ms, "TFLOP_per_s": fl / ms / 1e9,
                              "algorithmic_flops": fl, "visible_pairs": pairs}), flush=True)
    if "bucketed" in kernels:
        # the bucketed time bias against the linear one on the same operands
        g = torch.Generator(device=dev)
        g.manual_seed(cfg.seed)
        qkv = torch.randn((T, 3 * d), device=dev, generator=g).to(tdt)
        do = torch.randn((T, d), device=dev, generator=g).to(tdt)
        o = torch.empty((T, d), dtype=tdt, device=dev)
        lse = torch.empty((H, T), dtype=torch.float32, device=dev)
        dqkv = torch.empty_like(qkv)
        wsf = torch.empty(G.attn_workspace_size(batch.B, T, H, dh, msl, False), dtype=torch.uint8,
                          device=dev)
        wsb = torch.empty(G.attn_workspace_size(batch.B, T, H, dh, msl, True), dtype=torch.uint8,
                          device=dev)
        for bucketed in (False, True):
            slope_t = sp if bucketed else st

            def ff():
                G.attn_fwd(off, hl, msl, qkv, qkv[:, d:], qkv[:, 2 * d:], 3 * d, H, dh, pos, ts,
                           sp, slope_t, scale, o, d, lse, wsf, err, T=T, bucketed=bucketed)

            def fb():
                G.attn_bwd(off, hl, msl, qkv, qkv[:, d:], qkv[:, 2 * d:], 3 * d, H, dh, pos, ts,
                           sp, slope_t, scale, o, do, d, lse, dqkv, dqkv[:, d:], dqkv[:, 2 * d:],
                           wsb, err, T=T, bucketed=bucketed)

            ms_f = timed(ff, args.iters, args.warmup, flush)
            ff()
            ms_b = timed(fb, args.iters, args.warmup, flush)
            tag = "bucketed" if bucketed else "linear"
            print(json.dumps({**base, "kernel": f"attn_{tag}", "fwd_ms": ms_f,
                              "fwd_TFLOP_per_s": 4.0 * d * pairs / ms_f / 1e9, "bwd_ms": ms_b,
                              "bwd_TFLOP_per_s": 10.0 * d * pairs / ms_b / 1e9}), flush=True)

    if "cached" in kernels:
        # candidates scored against a history K/V cache, against the full attention over
        # history + candidates (whose candidate rows it equals)
        g = torch.Generator(device=dev)
        g.manual_seed(cfg.seed)
        qkv = torch.randn((T, 3 * d), device=dev, generator=g).to(tdt)
        n_u = batch.hist_len.astype(np.int64)
        hist_rows = np.concatenate([np.arange(batch.seq_offsets[u], batch.seq_offsets[u] + n_u[u])
                                    for u in range(batch.B)])
        cand_rows = np.concatenate([np.arange(batch.seq_offsets[u] + n_u[u], batch.seq_offsets[u + 1])
                                    for u in range(batch.B)])
        hr = torch.from_numpy(hist_rows).to(dev)
        cr = torch.from_numpy(cand_rows).to(dev)
        kv = qkv[:, d:].index_select(0, hr).contiguous()  # [Th, 2d]
        qc = qkv.index_select(0, cr).contiguous()          # [C, 3d]
        C, Th = int(cr.numel()), int(hr.numel())
        hoff = torch.from_numpy(np.concatenate([[0], np.cumsum(n_u)]).astype(np.int32)).to(dev)
        m_u = np.diff(batch.seq_offsets).astype(np.int64) - n_u
        coff = torch.from_numpy(np.concatenate([[0], np.cumsum(m_u)]).astype(np.int32)).to(dev)
        pos_h = pos.index_select(0, hr).contiguous()
        ts_h, ts_c = ts.index_select(0, hr).contiguous(), ts.index_select(0, cr).contiguous()
        oc = torch.empty((C, d), dtype=tdt, device=dev)
        of = torch.empty((T, d), dtype=tdt, device=dev)
        m_max = int(m_u.max())
        wsc = torch.empty(G.attn_cached_workspace_size(batch.B, C, Th, H, dh, m_max),
                          dtype=torch.uint8, device=dev)
        wsf = torch.empty(G.attn_workspace_size(batch.B, T, H, dh, msl, False), dtype=torch.uint8,
                          device=dev)

        def fc():
            G.attn_fwd_cached(coff, m_max, qc, qc[:, d:], qc[:, 2 * d:], 3 * d, hoff, kv,
                              kv[:, d:], 2 * d, pos_h, ts_h, ts_c, H, dh, sp, st, scale, oc, d,
                              None, wsc, err, C=C, Th=Th)

        def ffull():
            G.attn_fwd(off, hl, msl, qkv, qkv[:, d:], qkv[:, 2 * d:], 3 * d, H, dh, pos, ts, sp,
                       st, scale, of, d, None, wsf, err, T=T)

        cand_pairs = int(np.sum(m_u * n_u + m_u))
        ms_c = timed(fc, args.iters, args.warmup, flush)
        ms_f = timed(ffull, args.iters, args.warmup, flush)
        print(json.dumps({**base, "kernel": "attn_cached", "ms": ms_c, "full_ms": ms_f,
                          "candidates": C, "candidates_per_s": C / ms_c * 1e3,
                          "TFLOP_per_s": 4.0 * d * cand_pairs / ms_c / 1e9,
                          "speedup_vs_full": ms_f / ms_c}), flush=True)

    if "hstu" in kernels:
        # the interleaved layout (2n + m tokens) with a dense N x N bias read from HBM,
        # against the action-oriented layout (n + m tokens) with the ALiBi terms computed
        # on the fly, both on the same tensor-core attention kernel
        from gen import dense_bias_torch, interleave_batch

        ib = interleave_batch(batch)
        Ti = ib.T
        msl_i = int(np.max(np.diff(ib.seq_offsets)))
        Lpad = (msl_i + 127) // 128 * 128
        bias = dense_bias_torch(cfg.seed, ib.B, Lpad, dev)
        g = torch.Generator(device=dev)
        g.manual_seed(cfg.seed)
        qkv_i = torch.randn((Ti, 3 * d), device=dev, generator=g).to(tdt)
        qkv = torch.randn((T, 3 * d), device=dev, generator=g).to(tdt)
        o_i = torch.empty((Ti, d), dtype=tdt, device=dev)
        o = torch.empty((T, d), dtype=tdt, device=dev)
        off_i = torch.from_numpy(ib.seq_offsets).to(dev)
        hl_i = torch.from_numpy(ib.hist_len).to(dev)
        ws_i = torch.empty(G.attn_workspace_size(ib.B, Ti, H, dh, msl_i, False),
                           dtype=torch.uint8, device=dev)
        ws = torch.empty(G.attn_workspace_size(batch.B, T, H, dh, msl, False), dtype=torch.uint8,
                         device=dev)

        def fh():
            G.attn_fwd_dense_bias(off_i, hl_i, msl_i, qkv_i, qkv_i[:, d:], qkv_i[:, 2 * d:],
                                  3 * d, H, dh, bias, scale, o_i, d, None, ws_i, err, T=Ti)

        def fg():
            G.attn_fwd(off, hl, msl, qkv, qkv[:, d:], qkv[:, 2 * d:], 3 * d, H, dh, pos, ts, sp,
                       st, scale, o, d, None, ws, err, T=T)

        ms_h = timed(fh, args.iters, args.warmup, flush)
        ms_g = timed(fg, args.iters, args.warmup, flush)
        pairs_i = visible_pairs(ib.seq_offsets, ib.hist_len)
        print(json.dumps({**base, "kernel": "attn_hstu_shaped", "interleaved_ms": ms_h,
                          "interleaved_tokens": Ti, "interleaved_pairs": pairs_i,
                          "bias_bytes": int(bias.numel() * 2), "action_oriented_ms": ms_g,
                          "action_oriented_tokens": T, "action_oriented_pairs": pairs,
                          "time_ratio": ms_g / ms_h, "pair_ratio": pairs / pairs_i}), flush=True)

    if "linear" in kernels:
        # the four-layer block's linear layers at this workload's token count, on the
        # library's fused tensor-core kernels and, for comparison, as torch ops (cuBLAS
        # GEMM + elementwise kernels); 2 M N K flops per GEMM
        gg = torch.Generator(device=dev)
        gg.manual_seed(7)
        bf = torch.bfloat16
        a = torch.randn((T, d), device=dev, generator=gg).to(bf)
        wqkv = (torch.randn((3 * d, d), device=dev, generator=gg) / math.sqrt(d)).to(bf)
        wo = (torch.randn((d, d), device=dev, generator=gg) / math.sqrt(d)).to(bf)
        w1 = (torch.randn((4 * d, d), device=dev, generator=gg) / math.sqrt(d)).to(bf)
        w2 = (torch.randn((d, 4 * d), device=dev, generator=gg) / math.sqrt(4 * d)).to(bf)
        x = torch.randn((T, d), device=dev, generator=gg)
        u = torch.randn((T, 4 * d), device=dev, generator=gg).to(bf)
        out3 = torch.empty((T, 3 * d), dtype=bf, device=dev)
        out4 = torch.empty((T, 4 * d), dtype=bf, device=dev)
        a2 = torch.empty((T, d), dtype=bf, device=dev)

        def rms(v):
            return v * torch.rsqrt((v * v).mean(dim=-1, keepdim=True) + 1e-6)

        cases = [
            ("qkv", 3 * d, d, lambda: G.linear(a, wqkv, out3, err),
             lambda: a @ wqkv.t()),
            ("w1_silu", 4 * d, d, lambda: G.linear(a, w1, out4, err, epilogue=G.EPI_SILU),
             lambda: torch.nn.functional.silu(a @ w1.t())),
            ("wo_res_rms", d, d, lambda: G.linear_residual_rmsnorm(a, wo, x, x, a2, err),
             lambda: rms(x + (a @ wo.t()).float()).to(bf)),
            ("w2_res_rms", d, 4 * d, lambda: G.linear_residual_rmsnorm(u, w2, x, x, a2, err),
             lambda: rms(x + (u @ w2.t()).float()).to(bf)),
        ]
        for name, N, K, ours, theirs in cases:
            if d != 512 and name.endswith("res_rms"):
                continue
            fl = 2.0 * T * N * K
            ms = timed(ours, args.iters, args.warmup, flush)
            ms_t = timed(theirs, args.iters, args.warmup, flush)
            print(json.dumps({**base, "kernel": f"linear_{name}", "ms": ms,
                              "TFLOP_per_s": fl / ms / 1e9, "torch_ms": ms_t,
                              "torch_TFLOP_per_s": fl / ms_t / 1e9, "M": T, "N": N, "K": K}),
                  flush=True)
    code = G.check_error(err)
    if code:
        raise SystemExit(f"device error flags: {code}")


if __name__ == "__main__":
    main()
