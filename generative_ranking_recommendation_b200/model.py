"""The GenRank scoring and training step built on libgenrank.

The hot path (metadata + embedding assembly, masked ALiBi attention forward
and backward, embedding backward) runs in the library's kernels.  The blocks
around it are torch ops: the fused QKV projection, the output projection and
residual, pre-RMSNorm (eps 1e-6, unit gain) and the 4d SiLU FFN of the 4-layer
workloads, the final RMSNorm and the candidate head (a dot with w_head at
candidate rows only, as the loss lives only at candidate positions:
"GenRank [2025]" chapter notes §1.3.1; for one block without FFN it is the
library's fused candidate-logits kernel).  The residual stream is kept in fp32;
projections run in the storage dtype with fp32 accumulation.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

from . import genrank as G

RMS_EPS = 1e-6


@dataclass
class DeviceBatch:
    B: int
    T: int
    max_seqlen: int
    seq_offsets: torch.Tensor  # int32 [B+1]
    hist_len: torch.Tensor  # int32 [B]
    item_ids: torch.Tensor  # int32 [T]
    action_ids: torch.Tensor  # int32 [T]
    ts: torch.Tensor  # int64 [T]
    cand_rows: torch.Tensor  # int64 [sum m]
    labels: torch.Tensor | None  # float32 [sum m]

    @staticmethod
    def host_arrays(batch):
        """The per-step input arrays of a generated batch, in upload order."""
        cand = np.concatenate([np.arange(batch.seq_offsets[u] + batch.hist_len[u],
                                         batch.seq_offsets[u + 1]) for u in range(batch.B)])
        arrs = [batch.seq_offsets, batch.hist_len, batch.item_ids, batch.action_ids, batch.ts,
                cand.astype(np.int64)]
        if batch.labels is not None:
            arrs.append(batch.labels)
        return arrs

    @classmethod
    def from_tensors(cls, batch, tensors):
        t = list(tensors)
        labels = t[6] if len(t) > 6 else None
        return cls(batch.B, batch.T, int(np.max(np.diff(batch.seq_offsets))) if batch.B else 0,
                   t[0], t[1], t[2], t[3], t[4], t[5], labels)

    @classmethod
    def from_batch(cls, batch, device):
        arrs = cls.host_arrays(batch)
        return cls.from_tensors(batch, [torch.from_numpy(np.ascontiguousarray(a)).to(device)
                                        for a in arrs])


def _tt(x, dtype, device):
    return torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dtype)


class GenRankModel:
    """Device-resident tables and weights of one workload configuration."""

    def __init__(self, cfg, model, device="cuda", item_tab: torch.Tensor | None = None):
        self.cfg = cfg
        self.device = torch.device(device)
        self.dtype = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
        dt, dev = self.dtype, self.device
        if item_tab is None:
            from gen import item_table_torch  # seeded input generator (data only)
            item_tab = item_table_torch(cfg.seed, cfg.n_item, cfg.d, cfg.dtype, dev)
        self.item_tab = item_tab
        self.action_tab = _tt(model.action_tab, dt, dev)
        self.pos_tab = _tt(model.pos_tab, dt, dev)
        self.ri_tab = _tt(model.ri_tab, dt, dev)
        self.rt_tab = _tt(model.rt_tab, dt, dev)
        self.layers = []
        for L in model.layers:
            W = {"Wqkv": _tt(np.concatenate([L["Wq"], L["Wk"], L["Wv"]], axis=1), dt, dev),
                 "Wo": _tt(L["Wo"], dt, dev)}
            if cfg.ffn:
                W["W1"] = _tt(L["W1"], dt, dev)
                W["W2"] = _tt(L["W2"], dt, dev)
            # the library's linear layers take each weight transposed ([N][K], K-major)
            for k in list(W):
                W[k + "T"] = W[k].t().contiguous()
            self.layers.append(W)
        self.w_head = _tt(model.w_head, torch.float32, dev)
        self.H, self.dh, self.d = cfg.H, cfg.dh, cfg.d
        self.slope_pos, self.slope_time = G.alibi_slopes(cfg.H)
        self.scale = 1.0 / math.sqrt(cfg.dh)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self._ws = {}
        self._head_u = None
        # the fp32 gradient tables of the training step, kept across steps: a step zeroes
        # only the item rows the previous one accumulated into (and the small tables)
        self._grads = None
        self._grad_rows = None
        # the scoring step runs its projections on the library's tensor-core linear
        # layers (bf16; widths the tiles divide), the four-layer block with the fused
        # residual + RMSNorm epilogues (d = 512); otherwise the blocks are torch ops
        d = cfg.d
        self.fused_blocks = (cfg.dtype == "bf16" and cfg.ffn and d == 512)
        # a lone QKV projection (the one-block workloads) stays on cuBLAS, which is
        # faster than the library's plain-store GEMM at these shapes; set True to use
        # the library's linear layer for it too
        self.fused_qkv = False

    # -------------------------------------------------------------------------------------
    def workspace(self, db: DeviceBatch, bwd, cand_only=False) -> torch.Tensor:
        if cand_only:
            n = G.attn_candidates_workspace_size(db.B, db.T, self.H, self.dh, db.max_seqlen)
            key = "cand"
        else:
            n = G.attn_workspace_size(db.B, db.T, self.H, self.dh, db.max_seqlen, bwd)
            key = bool(bwd)
        w = self._ws.get(key)
        if w is None or w.numel() < n:
            w = torch.empty(max(n, 256), dtype=torch.uint8, device=self.device)
            self._ws[key] = w
        return w

    def embed(self, db: DeviceBatch):
        T, dev = db.T, self.device
        E = torch.empty((T, self.d), dtype=self.dtype, device=dev)
        pos = torch.empty(T, dtype=torch.int32, device=dev)
        req = torch.empty(T, dtype=torch.int32, device=dev)
        rtb = torch.empty(T, dtype=torch.int32, device=dev)
        G.embed_assemble(db.seq_offsets, db.hist_len, db.item_ids, db.action_ids, db.ts,
                         self.item_tab, self.action_tab, self.pos_tab, self.ri_tab, self.rt_tab,
                         E, pos, req, rtb, self.err)
        return E, (pos, req, rtb)

    def attention(self, db: DeviceBatch, qkv: torch.Tensor, pos: torch.Tensor, need_lse=False,
                  cand_only=False):
        """O (and the LSE) of every token, or with ``cand_only`` of the candidate rows only
        (the other rows of O are left unwritten)."""
        d = self.d
        o = torch.empty((db.T, d), dtype=qkv.dtype, device=self.device)
        lse = torch.empty((self.H, db.T), dtype=torch.float32, device=self.device) if need_lse else None
        fn = G.attn_fwd_candidates if cand_only else G.attn_fwd
        fn(db.seq_offsets, db.hist_len, db.max_seqlen, qkv, qkv[:, d:], qkv[:, 2 * d:], 3 * d,
           self.H, self.dh, pos, db.ts, self.slope_pos, self.slope_time, self.scale, o, d, lse,
           self.workspace(db, False, cand_only), self.err, T=db.T)
        return o, lse

    def attention_bwd(self, db, qkv, pos, o, lse, do):
        d = self.d
        dqkv = torch.empty_like(qkv)
        G.attn_bwd(db.seq_offsets, db.hist_len, db.max_seqlen, qkv, qkv[:, d:], qkv[:, 2 * d:],
                   3 * d, self.H, self.dh, pos, db.ts, self.slope_pos, self.slope_time,
                   self.scale, o, do.contiguous(), d, lse, dqkv, dqkv[:, d:], dqkv[:, 2 * d:],
                   self.workspace(db, True), self.err, T=db.T)
        return dqkv

    def head_u(self, W) -> torch.Tensor:
        """u = W_o w_head (fp32 [d]) for the fused candidate head, recomputed when W_o
        changes in place."""
        key = (W["Wo"].data_ptr(), W["Wo"]._version)
        if self._head_u is None or self._head_u[0] != key:
            self._head_u = (key, (W["Wo"].float() @ self.w_head).contiguous())
        return self._head_u[1]

    @staticmethod
    def rms(x):
        # x / sqrt(mean(x^2) + eps), unit gain, as one torch kernel
        return torch.nn.functional.rms_norm(x, (x.shape[-1],), eps=RMS_EPS)

    # -------------------------------------------------------------------------------------
    def _event(self, attn_events):
        if attn_events is None:
            return None
        ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        ev[0].record()
        attn_events.append(ev)
        return ev

    def _linear(self, a, Wt, epilogue=G.EPI_STORE):
        out = torch.empty((a.shape[0], Wt.shape[0]), dtype=self.dtype, device=self.device)
        G.linear(a, Wt, out, self.err, epilogue=epilogue)
        return out

    @torch.no_grad()
    def forward(self, db: DeviceBatch, attn_events=None, blocks: str = "auto") -> torch.Tensor:
        """Candidate logits (fp32 [sum m]) for one batch.

        ``blocks``: "auto" runs the projections, norms and FFN on the library's fused
        tensor-core linear layers where the shapes allow (``fused_blocks`` /
        ``fused_qkv``), "torch" runs them as torch ops (cuBLAS + elementwise kernels).
        """
        if blocks == "auto" and self.fused_blocks:
            return self._forward_fused(db, attn_events)
        return self._forward_torch(db, attn_events, fused_qkv=blocks == "auto" and self.fused_qkv)

    def _forward_fused(self, db: DeviceBatch, attn_events=None) -> torch.Tensor:
        """The four-layer scoring step on the library's kernels end to end: embedding
        assembly with the first RMSNorm, per layer the QKV projection, the attention, W_o with the
        residual update and the next RMSNorm in its epilogue, W1 with SiLU in its
        epilogue and W2 with the residual update and the next RMSNorm; the last layer's
        W_o and FFN run on candidate rows only and its W2 epilogue applies the final
        RMSNorm and the head."""
        T, d, dev = db.T, self.d, self.device
        # the gather-sum writes the fp32 residual rows and their RMSNorm directly
        x = torch.empty((T, d), dtype=torch.float32, device=dev)
        a = torch.empty((T, d), dtype=self.dtype, device=dev)
        pos = torch.empty(T, dtype=torch.int32, device=dev)
        req = torch.empty(T, dtype=torch.int32, device=dev)
        rtb = torch.empty(T, dtype=torch.int32, device=dev)
        G.embed_assemble_rmsnorm(db.seq_offsets, db.hist_len, db.item_ids, db.action_ids, db.ts,
                                 self.item_tab, self.action_tab, self.pos_tab, self.ri_tab,
                                 self.rt_tab, x, a, pos, req, rtb, self.err, eps=RMS_EPS)
        nl = len(self.layers)
        for li, W in enumerate(self.layers):
            qkv = self._linear(a, W["WqkvT"])
            ev = self._event(attn_events)
            # after the last attention only candidate rows reach the head
            o, _ = self.attention(db, qkv, pos, cand_only=li == nl - 1)
            if ev is not None:
                ev[1].record()
            if li == nl - 1:  # only candidate rows reach the head
                rows = db.cand_rows
                oc = torch.empty((rows.numel(), d), dtype=o.dtype, device=dev)
                xc = torch.empty((rows.numel(), d), dtype=x.dtype, device=dev)
                G.gather_rows(rows, o, oc, self.err)
                G.gather_rows(rows, x, xc, self.err)
                o, x = oc, xc
            a2 = torch.empty_like(o)
            G.linear_residual_rmsnorm(o, W["WoT"], x, x, a2, self.err, eps=RMS_EPS)
            u = self._linear(a2, W["W1T"], G.EPI_SILU)
            if li == nl - 1:
                z = torch.empty(x.shape[0], dtype=torch.float32, device=dev)
                G.linear_residual_rmsnorm(u, W["W2T"], x, x, None, self.err, w_head=self.w_head,
                                          z=z, eps=RMS_EPS)
                return z
            G.linear_residual_rmsnorm(u, W["W2T"], x, x, a, self.err, eps=RMS_EPS)
        raise ValueError("a model needs at least one layer")

    def _forward_torch(self, db: DeviceBatch, attn_events=None, fused_qkv=False) -> torch.Tensor:
        """Candidate logits with the blocks as torch ops (the QKV projection optionally on
        the library's linear layer).

        Every layer's attention but the last runs over all tokens (history rows feed
        the next layer's keys and values); only candidate rows reach the head, so the
        last attention (bf16, head dim 64) computes candidate rows alone, and the last
        output projection, residual, FFN and final norm run on candidate rows alone; with one block and no FFN the head is one fused
        kernel, z = E . w_head + o . (W_o w_head) at candidate rows (the same sum
        regrouped).  ``attn_events``: optional list; a (start, end)
        pair of CUDA events recorded on the current stream around each attention
        launch is appended to it.
        """
        E, (pos, _, _) = self.embed(db)
        ffn = self.cfg.ffn
        nl = len(self.layers)
        x = E.float() if (ffn or nl > 1) else None  # fp32 residual stream where needed
        for li, W in enumerate(self.layers):
            if ffn:
                a = self.rms(x).to(self.dtype)
            else:
                a = E if li == 0 else x.to(self.dtype)
            qkv = self._linear(a, W["WqkvT"]) if fused_qkv else a @ W["Wqkv"]
            ev = self._event(attn_events)
            # the last attention is needed at candidate rows only (the candidate-only
            # kernel takes bf16 with head dim 64; other forms run the full attention)
            cand_only = li == nl - 1 and self.dtype == torch.bfloat16 and self.dh == 64
            o, _ = self.attention(db, qkv, pos, cand_only=cand_only)
            if ev is not None:
                ev[1].record()
            if li == nl - 1 and x is None:
                # one block, no FFN: z = E . w_head + o . (W_o w_head) at candidate rows,
                # one fused gather-dot kernel
                z = torch.empty(db.cand_rows.numel(), dtype=torch.float32, device=self.device)
                G.candidate_logits(db.cand_rows, E, o, self.w_head, self.head_u(W), z, self.err)
                return z
            if li == nl - 1:
                rows = db.cand_rows
                base = x.index_select(0, rows)
                h = base + (o.index_select(0, rows) @ W["Wo"])
                if ffn:
                    f = self.rms(h).to(self.dtype)
                    h = h + (torch.nn.functional.silu(f @ W["W1"]) @ W["W2"])
                    h = self.rms(h)
                return h @ self.w_head
            x = x + (o @ W["Wo"])  # the add promotes the bf16 product to fp32 exactly
            if ffn:
                f = self.rms(x).to(self.dtype)
                x = x + (torch.nn.functional.silu(f @ W["W1"]) @ W["W2"])
        raise ValueError("a model needs at least one layer")

    # -------------------------------------------------------------------------------------
    def train_step(self, db: DeviceBatch):
        """Mean BCE over candidates, and the five fp32 table gradients.

        The attention backward and the embedding backward run in the library;
        torch autograd carries the gradient through the blocks around them.  The
        gradient tables are the model's own, valid until the next call: instead of
        zeroing the whole item table (4M rows at the training workload) every step, a
        step zeroes the rows the previous step wrote.
        """
        E, (pos, req, rtb) = self.embed(db)
        Eg = E.detach().requires_grad_(True)
        model = self

        class _Attn(torch.autograd.Function):
            @staticmethod
            def forward(ctx, qkv):
                o, lse = model.attention(db, qkv, pos, need_lse=True)
                ctx.save_for_backward(qkv, o, lse)
                return o

            @staticmethod
            def backward(ctx, do):
                qkv, o, lse = ctx.saved_tensors
                return model.attention_bwd(db, qkv, pos, o, lse, do)

        ffn = self.cfg.ffn
        nl = len(self.layers)
        x = Eg.float()
        z = None
        for li, W in enumerate(self.layers):
            a = (self.rms(x) if ffn else x).to(self.dtype)
            qkv = a @ W["Wqkv"]
            o = _Attn.apply(qkv)
            if li == nl - 1:  # only candidate rows reach the loss
                rows = db.cand_rows
                h = x.index_select(0, rows) + (o.index_select(0, rows) @ W["Wo"])
                if ffn:
                    f = self.rms(h).to(self.dtype)
                    h = h + (torch.nn.functional.silu(f @ W["W1"]) @ W["W2"])
                    h = self.rms(h)
                z = h @ self.w_head
                break
            x = x + (o @ W["Wo"])  # the add promotes the bf16 product to fp32 exactly
            if ffn:
                f = self.rms(x).to(self.dtype)
                x = x + (torch.nn.functional.silu(f @ W["W1"]) @ W["W2"])
        loss = torch.nn.functional.binary_cross_entropy_with_logits(z, db.labels)
        loss.backward()
        dE = Eg.grad.to(self.dtype).contiguous()
        f32 = dict(dtype=torch.float32, device=self.device)
        if self._grads is None:
            self._grads = {"item": torch.zeros(self.item_tab.shape, **f32),
                           "action": torch.zeros(self.action_tab.shape, **f32),
                           "pos": torch.zeros(self.pos_tab.shape, **f32),
                           "ri": torch.zeros(self.ri_tab.shape, **f32),
                           "rt": torch.zeros(self.rt_tab.shape, **f32)}
        else:
            self._grads["item"].index_fill_(0, self._grad_rows, 0.0)
            for k in ("action", "pos", "ri", "rt"):
                self._grads[k].zero_()
        grads = self._grads
        # ids outside the table are skipped by the kernel (and flagged); clamped here, they
        # only make the next step zero a row that is zero already
        self._grad_rows = db.item_ids.long().clamp_(0, self.item_tab.shape[0] - 1)
        G.embed_assemble_bwd(db.seq_offsets, db.hist_len, db.item_ids, db.action_ids, pos, req,
                             rtb, dE, grads["item"], grads["action"], grads["pos"], grads["ri"],
                             grads["rt"], self.err)
        return loss.detach(), z.detach(), grads


class CapturedStep:
    """One batch's scoring step captured as a CUDA graph.

    The library calls and the torch ops of ``model.forward(db)`` are recorded once
    and replayed without host launch work (argument marshalling, tensor-map
    encoding, dispatch), which otherwise leaves the GPU idle between the short
    kernels of a step.  The graph reads the batch's device tensors: to score new
    inputs of the same shapes, copy them into ``db``'s tensors (``load``) and
    ``run()``.  The logits tensor returned by ``run()`` is overwritten by the next
    replay.  The captured workspace stays referenced by this object, so later
    captures of other shapes cannot free it.
    """

    def __init__(self, model: GenRankModel, db: DeviceBatch, part: str = "forward"):
        self.model, self.db = model, db
        stream = torch.cuda.Stream(device=model.device)
        stream.wait_stream(torch.cuda.current_stream(model.device))
        with torch.cuda.stream(stream):
            if part == "attention":  # the first layer's attention alone
                E, (pos, _, _) = model.embed(db)
                W = model.layers[0]
                a = model.rms(E.float()).to(model.dtype) if model.cfg.ffn else E
                self._qkv, self._pos = a @ W["Wqkv"], pos
                fn = lambda: model.attention(db, self._qkv, self._pos)[0]  # noqa: E731
            elif part == "embed":  # metadata + gather-sum alone
                fn = lambda: model.embed(db)[0]  # noqa: E731
            elif part == "forward":
                fn = lambda: model.forward(db)  # noqa: E731
            else:
                raise ValueError(f"unknown part {part!r}")
            fn()  # warm-up: function attributes, workspace
        torch.cuda.current_stream(model.device).wait_stream(stream)
        torch.cuda.synchronize(model.device)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.out = fn()
        self._ws = dict(model._ws)  # keep the captured workspaces alive

    def load(self, tensors):
        """Copy new per-step inputs (host or device tensors, upload order of
        ``DeviceBatch.host_arrays``) into the captured batch."""
        dst = [self.db.seq_offsets, self.db.hist_len, self.db.item_ids, self.db.action_ids,
               self.db.ts, self.db.cand_rows] + ([self.db.labels] if self.db.labels is not None
                                                  else [])
        for d, s in zip(dst, tensors):
            d.copy_(s, non_blocking=True)

    def run(self) -> torch.Tensor:
        self.graph.replay()
        return self.out
