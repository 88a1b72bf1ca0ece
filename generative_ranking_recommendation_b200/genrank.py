"""Thin Python binding of libgenrank (include/genrank.h), by the same names.

Argument marshalling only: torch tensors supply device pointers and the
current CUDA stream; every step of the computation runs in the library's
kernels.  There is no fallback: if the shared library is missing or the call
fails, an exception is raised.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgenrank.so")

F32, BF16 = 0, 1
DERR = {
    "LAYOUT": 1 << 0, "ITEM_ID": 1 << 1, "ACTION_ID": 1 << 2, "TS_ORDER": 1 << 3,
    "POS_RANGE": 1 << 4, "INDEX": 1 << 5, "TIMEOUT": 1 << 6,
}

# every entry point declared in include/genrank.h
EXPORTS = (
    "genrank_status_string", "genrank_device_error_string", "genrank_check_error",
    "genrank_alibi_slopes", "genrank_embed_assemble", "genrank_embed_assemble_rmsnorm",
    "genrank_embed_assemble_bwd",
    "genrank_attn_fwd", "genrank_attn_bwd", "genrank_attn_workspace_size",
    "genrank_attn_fwd_candidates", "genrank_attn_candidates_workspace_size",
    "genrank_attn_fwd_static", "genrank_candidate_logits", "genrank_attn_fwd_cached",
    "genrank_attn_cached_workspace_size", "genrank_attn_fwd_bucketed",
    "genrank_attn_bwd_bucketed", "genrank_attn_fwd_dense_bias", "genrank_linear",
    "genrank_linear_residual_rmsnorm", "genrank_rmsnorm", "genrank_gather_rows",
)
EPI_STORE, EPI_SILU = 0, 1


class GenRankError(RuntimeError):
    pass


_lib = None
_P, _I, _L, _F, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t


def lib():
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise GenRankError(
                f"{LIB_PATH} is missing; build it with "
                "`python -m generative_ranking_recommendation_b200.csrc.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.genrank_status_string.restype = ctypes.c_char_p
        L.genrank_status_string.argtypes = [_I]
        L.genrank_device_error_string.restype = ctypes.c_char_p
        L.genrank_device_error_string.argtypes = [_I]
        L.genrank_check_error.restype = _I
        L.genrank_check_error.argtypes = [_P, _P]
        L.genrank_alibi_slopes.restype = _I
        L.genrank_alibi_slopes.argtypes = [_I, _P, _P]
        L.genrank_embed_assemble.restype = _I
        L.genrank_embed_assemble.argtypes = [
            _I, _L, _P, _P, _P, _P, _P, _P, _L, _P, _I, _P, _I, _P, _I, _P, _I, _I, _I,
            _P, _P, _P, _P, _P, _P]
        L.genrank_embed_assemble_rmsnorm.restype = _I
        L.genrank_embed_assemble_rmsnorm.argtypes = [
            _I, _L, _P, _P, _P, _P, _P, _P, _L, _P, _I, _P, _I, _P, _I, _P, _I, _I, _P, _P, _F,
            _P, _P, _P, _P, _P]
        L.genrank_embed_assemble_bwd.restype = _I
        L.genrank_embed_assemble_bwd.argtypes = [
            _I, _L, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _P, _L, _P, _I, _P, _I, _P, _I,
            _P, _I, _P, _P]
        L.genrank_attn_fwd.restype = _I
        L.genrank_attn_fwd.argtypes = [
            _I, _L, _P, _P, _I, _P, _P, _P, _L, _I, _I, _P, _P, _P, _P, _F, _I, _P, _L, _P,
            _P, _Z, _P, _P]
        L.genrank_attn_fwd_candidates.restype = _I
        L.genrank_attn_fwd_candidates.argtypes = L.genrank_attn_fwd.argtypes
        L.genrank_attn_candidates_workspace_size.restype = _Z
        L.genrank_attn_candidates_workspace_size.argtypes = [_I, _L, _I, _I, _I]
        L.genrank_attn_fwd_bucketed.restype = _I
        L.genrank_attn_fwd_bucketed.argtypes = L.genrank_attn_fwd.argtypes
        L.genrank_attn_bwd.restype = _I
        L.genrank_attn_bwd.argtypes = [
            _I, _L, _P, _P, _I, _P, _P, _P, _L, _I, _I, _P, _P, _P, _P, _F, _I, _P, _P, _L,
            _P, _P, _P, _P, _P, _Z, _P, _P]
        L.genrank_attn_fwd_dense_bias.restype = _I
        L.genrank_attn_fwd_dense_bias.argtypes = [
            _I, _L, _P, _P, _I, _P, _P, _P, _L, _I, _I, _P, _L, _F, _I, _P, _L, _P, _P, _Z, _P,
            _P]
        L.genrank_linear.restype = _I
        L.genrank_linear.argtypes = [_I, _I, _I, _P, _L, _P, _L, _I, _P, _L, _P, _P]
        L.genrank_linear_residual_rmsnorm.restype = _I
        L.genrank_linear_residual_rmsnorm.argtypes = [
            _I, _I, _I, _P, _L, _P, _L, _P, _P, _L, _P, _L, _P, _P, _F, _P, _P]
        L.genrank_rmsnorm.restype = _I
        L.genrank_rmsnorm.argtypes = [_L, _I, _P, _L, _I, _P, _L, _P, _L, _F, _P, _P]
        L.genrank_attn_bwd_bucketed.restype = _I
        L.genrank_attn_bwd_bucketed.argtypes = L.genrank_attn_bwd.argtypes
        L.genrank_attn_fwd_static.restype = _I
        L.genrank_attn_fwd_static.argtypes = [
            _I, _L, _P, _P, _I, _P, _P, _P, _L, _I, _I, _P, _P, _P, _P, _F, _I, _P, _L, _P,
            _P, _P]
        L.genrank_candidate_logits.restype = _I
        L.genrank_candidate_logits.argtypes = [
            _I, _P, _L, _I, _P, _L, _P, _L, _I, _P, _P, _P, _P, _P]
        L.genrank_gather_rows.restype = _I
        L.genrank_gather_rows.argtypes = [_L, _P, _L, _L, _P, _L, _P, _L, _P, _P]
        L.genrank_attn_fwd_cached.restype = _I
        L.genrank_attn_fwd_cached.argtypes = [
            _I, _L, _P, _I, _P, _P, _P, _L, _L, _P, _P, _P, _L, _P, _P, _P, _I, _I, _P, _P, _F,
            _I, _P, _L, _P, _P, _Z, _P, _P]
        L.genrank_attn_cached_workspace_size.restype = _Z
        L.genrank_attn_cached_workspace_size.argtypes = [_I, _L, _L, _I, _I, _I]
        L.genrank_attn_workspace_size.restype = _Z
        L.genrank_attn_workspace_size.argtypes = [_I, _L, _I, _I, _I, _I]
        _lib = L
    return _lib


def _check(rc: int, what: str):
    if rc != 0:
        msg = lib().genrank_status_string(rc).decode()
        raise GenRankError(f"{what}: {msg} (code {rc})")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise GenRankError(f"unsupported dtype {t.dtype}")


def status_string(code: int) -> str:
    return lib().genrank_status_string(int(code)).decode()


def device_error_string(bit: int) -> str:
    return lib().genrank_device_error_string(int(bit)).decode()


def alibi_slopes(H: int):
    """(slope_pos, slope_time) as Python float lists, from the library."""
    sp = (ctypes.c_float * H)()
    st = (ctypes.c_float * H)()
    _check(lib().genrank_alibi_slopes(H, ctypes.cast(sp, _P), ctypes.cast(st, _P)),
           "genrank_alibi_slopes")
    return list(sp), list(st)


def check_error(dev_err: torch.Tensor, stream=None) -> int:
    """Synchronises the stream and returns the device error word (0 = clean)."""
    rc = lib().genrank_check_error(_ptr(dev_err), _stream(stream))
    if rc < 0:
        _check(-rc, "genrank_check_error")
    return rc


def embed_assemble(seq_offsets, hist_len, item_ids, action_ids, ts, item_tab, action_tab,
                   pos_tab, ri_tab, rt_tab, E, pos, req_idx, rt_bucket, dev_err, stream=None):
    """genrank_embed_assemble on torch tensors (all on one CUDA device)."""
    B = hist_len.numel()
    T = item_ids.numel()
    d = item_tab.shape[1]
    rc = lib().genrank_embed_assemble(
        B, T, _ptr(seq_offsets), _ptr(hist_len), _ptr(item_ids), _ptr(action_ids), _ptr(ts),
        _ptr(item_tab), item_tab.shape[0], _ptr(action_tab), action_tab.shape[0] - 1,
        _ptr(pos_tab), pos_tab.shape[0], _ptr(ri_tab), ri_tab.shape[0], _ptr(rt_tab),
        rt_tab.shape[0], d, _dtype_code(item_tab), _ptr(E), _ptr(pos), _ptr(req_idx),
        _ptr(rt_bucket), _ptr(dev_err), _stream(stream))
    _check(rc, "genrank_embed_assemble")


def embed_assemble_rmsnorm(seq_offsets, hist_len, item_ids, action_ids, ts, item_tab, action_tab,
                           pos_tab, ri_tab, rt_tab, x_out, a_out, pos, req_idx, rt_bucket, dev_err,
                           eps=1e-6, stream=None):
    """genrank_embed_assemble_rmsnorm: the gather-sum written as the fp32 residual rows
    (x_out) and their RMSNorm in bf16 (a_out) instead of E."""
    B = hist_len.numel()
    T = item_ids.numel()
    d = item_tab.shape[1]
    rc = lib().genrank_embed_assemble_rmsnorm(
        B, T, _ptr(seq_offsets), _ptr(hist_len), _ptr(item_ids), _ptr(action_ids), _ptr(ts),
        _ptr(item_tab), item_tab.shape[0], _ptr(action_tab), action_tab.shape[0] - 1,
        _ptr(pos_tab), pos_tab.shape[0], _ptr(ri_tab), ri_tab.shape[0], _ptr(rt_tab),
        rt_tab.shape[0], d, _ptr(x_out), _ptr(a_out), float(eps), _ptr(pos), _ptr(req_idx),
        _ptr(rt_bucket), _ptr(dev_err), _stream(stream))
    _check(rc, "genrank_embed_assemble_rmsnorm")


def embed_assemble_bwd(seq_offsets, hist_len, item_ids, action_ids, pos, req_idx, rt_bucket, dE,
                       d_item, d_action, d_pos, d_ri, d_rt, dev_err, stream=None):
    """genrank_embed_assemble_bwd: accumulates into the fp32 gradient tables."""
    B = hist_len.numel()
    T = item_ids.numel()
    rc = lib().genrank_embed_assemble_bwd(
        B, T, _ptr(seq_offsets), _ptr(hist_len), _ptr(item_ids), _ptr(action_ids), _ptr(pos),
        _ptr(req_idx), _ptr(rt_bucket), _ptr(dE), dE.shape[1], _dtype_code(dE), _ptr(d_item),
        d_item.shape[0], _ptr(d_action), d_action.shape[0] - 1, _ptr(d_pos), d_pos.shape[0],
        _ptr(d_ri), d_ri.shape[0], _ptr(d_rt), d_rt.shape[0], _ptr(dev_err), _stream(stream))
    _check(rc, "genrank_embed_assemble_bwd")


def attn_workspace_size(B, T, H, dh, max_seqlen, is_bwd=False) -> int:
    return int(lib().genrank_attn_workspace_size(B, T, H, dh, max_seqlen, int(bool(is_bwd))))


def _host_floats(xs):
    arr = (ctypes.c_float * len(xs))(*[float(x) for x in xs])
    return arr


def attn_fwd(seq_offsets, hist_len, max_seqlen, q, k, v, tok_stride, H, dh, pos, ts, slope_pos,
             slope_time, scale, o, o_stride, lse, ws, dev_err, T=None, stream=None,
             bucketed=False):
    """genrank_attn_fwd (genrank_attn_fwd_bucketed with ``bucketed``, slope_time then
    being the slope per time bucket).  q/k/v are tensors whose data_ptr is the first
    element of head 0 of token 0 (views into a fused QKV buffer are fine); slopes are
    host lists."""
    B = hist_len.numel()
    T = o.shape[0] if T is None else T
    sp, st = _host_floats(slope_pos), _host_floats(slope_time)
    fn = lib().genrank_attn_fwd_bucketed if bucketed else lib().genrank_attn_fwd
    rc = fn(
        B, T, _ptr(seq_offsets), _ptr(hist_len), int(max_seqlen), _ptr(q), _ptr(k), _ptr(v),
        int(tok_stride), H, dh, _ptr(pos), _ptr(ts), ctypes.cast(sp, _P), ctypes.cast(st, _P),
        float(scale), _dtype_code(q), _ptr(o), int(o_stride), _ptr(lse), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _ptr(dev_err), _stream(stream))
    _check(rc, "genrank_attn_fwd_bucketed" if bucketed else "genrank_attn_fwd")


def attn_fwd_candidates(seq_offsets, hist_len, max_seqlen, q, k, v, tok_stride, H, dh, pos, ts,
                        slope_pos, slope_time, scale, o, o_stride, lse, ws, dev_err, T=None,
                        stream=None):
    """genrank_attn_fwd_candidates: genrank_attn_fwd's candidate rows only (history rows of
    o and lse are left as they are); the same arguments."""
    B = hist_len.numel()
    T = o.shape[0] if T is None else T
    sp, st = _host_floats(slope_pos), _host_floats(slope_time)
    rc = lib().genrank_attn_fwd_candidates(
        B, T, _ptr(seq_offsets), _ptr(hist_len), int(max_seqlen), _ptr(q), _ptr(k), _ptr(v),
        int(tok_stride), H, dh, _ptr(pos), _ptr(ts), ctypes.cast(sp, _P), ctypes.cast(st, _P),
        float(scale), _dtype_code(q), _ptr(o), int(o_stride), _ptr(lse), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _ptr(dev_err), _stream(stream))
    _check(rc, "genrank_attn_fwd_candidates")


def attn_candidates_workspace_size(B, T, H, dh, max_seqlen) -> int:
    return int(lib().genrank_attn_candidates_workspace_size(B, T, H, dh, max_seqlen))


def attn_bwd(seq_offsets, hist_len, max_seqlen, q, k, v, tok_stride, H, dh, pos, ts, slope_pos,
             slope_time, scale, o, dO, o_stride, lse, dq, dk, dv, ws, dev_err, T=None,
             stream=None, bucketed=False):
    """genrank_attn_bwd (genrank_attn_bwd_bucketed with ``bucketed``); dq/dk/dv share
    the layout (tok_stride) of q/k/v."""
    B = hist_len.numel()
    T = o.shape[0] if T is None else T
    sp, st = _host_floats(slope_pos), _host_floats(slope_time)
    fn = lib().genrank_attn_bwd_bucketed if bucketed else lib().genrank_attn_bwd
    rc = fn(
        B, T, _ptr(seq_offsets), _ptr(hist_len), int(max_seqlen), _ptr(q), _ptr(k), _ptr(v),
        int(tok_stride), H, dh, _ptr(pos), _ptr(ts), ctypes.cast(sp, _P), ctypes.cast(st, _P),
        float(scale), _dtype_code(q), _ptr(o), _ptr(dO), int(o_stride), _ptr(lse), _ptr(dq),
        _ptr(dk), _ptr(dv), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
        _ptr(dev_err), _stream(stream))
    _check(rc, "genrank_attn_bwd_bucketed" if bucketed else "genrank_attn_bwd")


def attn_fwd_static(seq_offsets, hist_len, max_seqlen, q, k, v, tok_stride, H, dh, pos, ts,
                    slope_pos, slope_time, scale, o, o_stride, lse, dev_err, T=None, stream=None):
    """genrank_attn_fwd_static: the forward without a caller workspace (the library's
    fixed 16 MiB scratch is used; see include/genrank.h for the rules)."""
    B = hist_len.numel()
    T = o.shape[0] if T is None else T
    sp, st = _host_floats(slope_pos), _host_floats(slope_time)
    rc = lib().genrank_attn_fwd_static(
        B, T, _ptr(seq_offsets), _ptr(hist_len), int(max_seqlen), _ptr(q), _ptr(k), _ptr(v),
        int(tok_stride), H, dh, _ptr(pos), _ptr(ts), ctypes.cast(sp, _P), ctypes.cast(st, _P),
        float(scale), _dtype_code(q), _ptr(o), int(o_stride), _ptr(lse), _ptr(dev_err),
        _stream(stream))
    _check(rc, "genrank_attn_fwd_static")


def candidate_logits(rows, x, o, w, u, z, dev_err, stream=None):
    """genrank_candidate_logits: z[c] = x[rows[c]] . w + o[rows[c]] . u (fp32)."""
    if o.dtype != x.dtype:
        raise GenRankError("candidate_logits: x and o must share a dtype")
    rc = lib().genrank_candidate_logits(
        int(rows.numel()), _ptr(rows), int(x.shape[0]), int(x.shape[1]), _ptr(x),
        int(x.stride(0)), _ptr(o), int(o.stride(0)), _dtype_code(x), _ptr(w), _ptr(u), _ptr(z),
        _ptr(dev_err), _stream(stream))
    _check(rc, "genrank_candidate_logits")


def gather_rows(rows, src, dst, dev_err, stream=None):
    """genrank_gather_rows: dst[k] = src[rows[k]] for 2-D tensors of one element type
    whose rows are contiguous; dst has rows.numel() rows."""
    if src.dtype != dst.dtype or src.dim() != 2 or dst.dim() != 2 or src.shape[1] != dst.shape[1]:
        raise GenRankError("gather_rows: src and dst must be 2-D of one dtype and width")
    if src.stride(1) != 1 or dst.stride(1) != 1 or dst.shape[0] != rows.numel():
        raise GenRankError("gather_rows: contiguous rows, one dst row per index")
    es = src.element_size()
    rc = lib().genrank_gather_rows(
        int(rows.numel()), _ptr(rows), int(src.shape[0]), int(src.shape[1]) * es, _ptr(src),
        int(src.stride(0)) * es, _ptr(dst), int(dst.stride(0)) * es, _ptr(dev_err),
        _stream(stream))
    _check(rc, "genrank_gather_rows")


def attn_cached_workspace_size(B, C, Th, H, dh, max_cand) -> int:
    return int(lib().genrank_attn_cached_workspace_size(B, C, Th, H, dh, max_cand))


def attn_fwd_cached(cand_offsets, max_cand, q_c, k_c, v_c, cand_stride, hist_offsets, k_hist,
                    v_hist, hist_stride, pos_hist, ts_hist, ts_cand, H, dh, slope_pos,
                    slope_time, scale, o, o_stride, lse, ws, dev_err, C=None, Th=None,
                    stream=None):
    """genrank_attn_fwd_cached: candidate rows scored against a history K/V cache.  The
    candidate and cache tensors are views whose data_ptr is head 0 of row 0; C and Th
    default to the row counts of o and pos_hist."""
    B = cand_offsets.numel() - 1
    C = o.shape[0] if C is None else C
    Th = (pos_hist.numel() if pos_hist is not None else 0) if Th is None else Th
    sp, st = _host_floats(slope_pos), _host_floats(slope_time)
    rc = lib().genrank_attn_fwd_cached(
        B, int(C), _ptr(cand_offsets), int(max_cand), _ptr(q_c), _ptr(k_c), _ptr(v_c),
        int(cand_stride), int(Th), _ptr(hist_offsets), _ptr(k_hist), _ptr(v_hist),
        int(hist_stride), _ptr(pos_hist), _ptr(ts_hist), _ptr(ts_cand), H, dh,
        ctypes.cast(sp, _P), ctypes.cast(st, _P), float(scale), _dtype_code(q_c), _ptr(o),
        int(o_stride), _ptr(lse), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
        _ptr(dev_err), _stream(stream))
    _check(rc, "genrank_attn_fwd_cached")


def attn_fwd_dense_bias(seq_offsets, hist_len, max_seqlen, q, k, v, tok_stride, H, dh, bias,
                        scale, o, o_stride, lse, ws, dev_err, T=None, stream=None):
    """genrank_attn_fwd_dense_bias: bias is a bf16 [B, Lpad, Lpad] tensor."""
    B = hist_len.numel()
    T = o.shape[0] if T is None else T
    rc = lib().genrank_attn_fwd_dense_bias(
        B, int(T), _ptr(seq_offsets), _ptr(hist_len), int(max_seqlen), _ptr(q), _ptr(k),
        _ptr(v), int(tok_stride), H, dh, _ptr(bias), int(bias.shape[-1]), float(scale),
        _dtype_code(q), _ptr(o), int(o_stride), _ptr(lse), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _ptr(dev_err), _stream(stream))
    _check(rc, "genrank_attn_fwd_dense_bias")


def linear(A, Wt, C, dev_err, epilogue=EPI_STORE, stream=None):
    """genrank_linear: C = bf16(A Wt^T), or bf16(SiLU(A Wt^T)) with EPI_SILU.  A [M, K],
    Wt [N, K] (the transposed weight), C [M, N]; bf16, row strides from the tensors."""
    M, K = A.shape
    N = Wt.shape[0]
    rc = lib().genrank_linear(int(M), int(N), int(K), _ptr(A), int(A.stride(0)), _ptr(Wt),
                              int(Wt.stride(0)), int(epilogue), _ptr(C), int(C.stride(0)),
                              _ptr(dev_err), _stream(stream))
    _check(rc, "genrank_linear")


def linear_residual_rmsnorm(A, Wt, x_in, x_out, a_out, dev_err, w_head=None, z=None,
                            eps=1e-6, stream=None):
    """genrank_linear_residual_rmsnorm: x_out = x_in + A Wt^T (fp32), a_out = bf16 rms of
    it (or None), z = rms(x_out) . w_head when w_head is given."""
    M, K = A.shape
    d = Wt.shape[0]
    rc = lib().genrank_linear_residual_rmsnorm(
        int(M), int(d), int(K), _ptr(A), int(A.stride(0)), _ptr(Wt), int(Wt.stride(0)),
        _ptr(x_in), _ptr(x_out), int(x_out.stride(0)), _ptr(a_out),
        int(a_out.stride(0)) if a_out is not None else 0, _ptr(w_head), _ptr(z), float(eps),
        _ptr(dev_err), _stream(stream))
    _check(rc, "genrank_linear_residual_rmsnorm")


def rmsnorm(x, a_out, dev_err, x_out=None, eps=1e-6, stream=None):
    """genrank_rmsnorm: a_out = bf16 rms(x); x_out = fp32 copy of x when given."""
    M, d = x.shape
    rc = lib().genrank_rmsnorm(int(M), int(d), _ptr(x), int(x.stride(0)), _dtype_code(x),
                               _ptr(x_out), int(x_out.stride(0)) if x_out is not None else 0,
                               _ptr(a_out), int(a_out.stride(0)), float(eps), _ptr(dev_err),
                               _stream(stream))
    _check(rc, "genrank_rmsnorm")
