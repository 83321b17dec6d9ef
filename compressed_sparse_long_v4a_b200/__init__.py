"""Python binding of libv4a.so, the B200 compressed-attention library.

The functions here carry the C ABI's names (``include/v4a.h``) and only
marshal arguments: they read pointers, sizes and strides off torch tensors,
pass the current CUDA stream, and raise ``V4AError`` with the library's
one-line reason when a call returns a non-OK status.  Every step of the
computation runs in the library's CUDA kernels; there is no other path.  If
the shared library has not been built, importing this package fails.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "V4AError", "F32", "BF16", "FP8E4M3", "MXFP4", "lib", "library_path",
    "v4a_compress", "v4a_compress_dual", "v4a_quantize_mxfp4", "v4a_index_scores", "v4a_index_scores_mxfp4",
    "v4a_topk", "v4a_topk_mxfp4", "v4a_topk_noalloc", "v4a_csa_attend", "v4a_hca_attend",
    "v4a_ring_append", "v4a_compress_paged", "v4a_topk_paged", "v4a_topk_mxfp4_paged", "v4a_csa_attend_paged",
    "v4a_hca_attend_paged",
    "v4a_workspace_size", "v4a_status_string", "v4a_version", "n_entries", "window_rows",
]

F32, BF16, FP8E4M3, MXFP4 = 0, 1, 2, 3
_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libv4a.so")


class V4AError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"v4a status {status}: {message}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("n_q", ctypes.c_int), ("heads", ctypes.c_int), ("d", ctypes.c_int),
                ("m", ctypes.c_int), ("k", ctypes.c_int), ("window", ctypes.c_int), ("ctx_len", ctypes.c_longlong)]


class CompressIO(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("gate", ctypes.c_void_p), ("out", ctypes.c_void_p),
                ("out_scale", ctypes.c_void_p), ("channels", ctypes.c_int), ("in_dtype", ctypes.c_int),
                ("out_dtype", ctypes.c_int), ("x_batch_stride", ctypes.c_longlong),
                ("gate_batch_stride", ctypes.c_longlong), ("out_batch_stride", ctypes.c_longlong),
                ("scale_batch_stride", ctypes.c_longlong), ("out_exp", ctypes.c_void_p),
                ("exp_batch_stride", ctypes.c_longlong)]


class SeriesB(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("gate", ctypes.c_void_p), ("prev_x", ctypes.c_void_p),
                ("prev_gate", ctypes.c_void_p), ("x_batch_stride", ctypes.c_longlong),
                ("gate_batch_stride", ctypes.c_longlong), ("prev_batch_stride", ctypes.c_longlong)]


class AttendExt(ctypes.Structure):
    _fields_ = [("sink", ctypes.c_void_p), ("rope_dims", ctypes.c_int), ("rope_base", ctypes.c_float)]


class Paged(ctypes.Structure):
    _fields_ = [("block_table", ctypes.c_void_p), ("bt_stride", ctypes.c_int), ("block_tokens", ctypes.c_int),
                ("n_blocks", ctypes.c_longlong), ("ring_rows", ctypes.c_int)]


class RingIO(ctypes.Structure):
    _fields_ = [("src", ctypes.c_void_p), ("ring", ctypes.c_void_p), ("channels", ctypes.c_int),
                ("ring_rows", ctypes.c_int), ("dtype", ctypes.c_int), ("src_batch_stride", ctypes.c_longlong)]


def library_path() -> str:
    return _LIB_PATH


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"libv4a.so is not built at {_LIB_PATH}; run __graft_entry__.build() "
                          "(python -c 'import __graft_entry__ as g; g.build()')")
    L = ctypes.CDLL(_LIB_PATH)
    vp, i32, ll, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t
    P = ctypes.POINTER
    L.v4a_compress.restype = i32
    L.v4a_compress.argtypes = [P(CompressIO), P(CompressIO), i32, ll, i32, vp]
    L.v4a_csa_attend_ex.restype = i32
    L.v4a_csa_attend_ex.argtypes = [vp, vp, vp, vp, ll, ll, vp, i32, vp, sz, vp, P(AttendExt), P(Shape), vp]
    L.v4a_hca_attend_ex.restype = i32
    L.v4a_hca_attend_ex.argtypes = [vp, vp, vp, ll, ll, vp, i32, vp, sz, P(AttendExt), P(Shape), vp]
    L.v4a_compress_dual.restype = i32
    L.v4a_compress_dual.argtypes = [P(CompressIO), P(SeriesB), i32, ll, i32, vp]
    L.v4a_index_scores.restype = i32
    L.v4a_index_scores.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, P(Shape), vp]
    L.v4a_topk.restype = i32
    L.v4a_topk.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, sz, P(Shape), vp]
    L.v4a_quantize_mxfp4.restype = i32
    L.v4a_quantize_mxfp4.argtypes = [vp, i32, ll, i32, vp, vp, vp]
    L.v4a_index_scores_mxfp4.restype = i32
    L.v4a_index_scores_mxfp4.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, P(Shape), vp]
    L.v4a_topk_mxfp4.restype = i32
    L.v4a_topk_mxfp4.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, vp, sz, P(Shape), vp]
    L.v4a_ring_append.restype = i32
    L.v4a_ring_append.argtypes = [P(RingIO), i32, i32, ll, vp]
    L.v4a_compress_paged.restype = i32
    L.v4a_compress_paged.argtypes = [P(CompressIO), P(CompressIO), i32, ll, i32, ll, P(Paged), vp]
    L.v4a_topk_paged.restype = i32
    L.v4a_topk_paged.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, sz, vp, P(Paged), P(Shape), vp]
    L.v4a_topk_mxfp4_paged.restype = i32
    L.v4a_topk_mxfp4_paged.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, vp, sz, vp, P(Paged), P(Shape), vp]
    L.v4a_csa_attend_paged.restype = i32
    L.v4a_csa_attend_paged.argtypes = [vp, vp, vp, vp, vp, i32, vp, sz, vp, P(AttendExt), P(Paged), P(Shape), vp]
    L.v4a_hca_attend_paged.restype = i32
    L.v4a_hca_attend_paged.argtypes = [vp, vp, vp, vp, i32, vp, sz, vp, P(AttendExt), P(Paged), P(Shape), vp]
    L.v4a_topk_noalloc.restype = i32
    L.v4a_topk_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, P(Shape), vp]
    L.v4a_csa_attend.restype = i32
    L.v4a_csa_attend.argtypes = [vp, vp, vp, vp, ll, ll, vp, i32, vp, sz, vp, P(Shape), vp]
    L.v4a_hca_attend.restype = i32
    L.v4a_hca_attend.argtypes = [vp, vp, vp, ll, ll, vp, i32, vp, sz, P(Shape), vp]
    L.v4a_workspace_size.restype = sz
    L.v4a_workspace_size.argtypes = [ctypes.c_char_p, P(Shape), i32, i32]
    L.v4a_status_string.restype = ctypes.c_char_p
    L.v4a_status_string.argtypes = [i32]
    L.v4a_last_error.restype = ctypes.c_char_p
    L.v4a_last_error.argtypes = []
    L.v4a_version.restype = i32
    L.v4a_version.argtypes = []
    return L


lib = _load()


def _check(status: int) -> None:
    if status != 0:
        raise V4AError(status, lib.v4a_last_error().decode() or lib.v4a_status_string(status).decode())


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return FP8E4M3
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libv4a takes CUDA tensors")
    return t.data_ptr()


def _contig(t: torch.Tensor, name: str) -> None:
    if t is not None and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def n_entries(ctx_len: int, m: int) -> int:
    return ctx_len // m


def window_rows(ctx_len: int, n_q: int, window: int):
    """(tok_pos0, l_tok): the token rows that every query's window needs."""
    p0 = max(0, ctx_len - n_q - window + 1)
    return p0, ctx_len - p0


def _shape(batch=0, n_q=1, heads=0, d=0, m=1, k=0, window=0, ctx_len=1) -> Shape:
    return Shape(int(batch), int(n_q), int(heads), int(d), int(m), int(k), int(window), int(ctx_len))


def v4a_workspace_size(op: str, *, batch, n_q=1, heads=0, d=0, m=1, k=0, window=0, ctx_len=1, heads_i=0,
                       d_i=0) -> int:
    s = _shape(batch, n_q, heads, d, m, k, window, ctx_len)
    return int(lib.v4a_workspace_size(op.encode(), ctypes.byref(s), int(heads_i), int(d_i)))


def v4a_status_string(status: int) -> str:
    return lib.v4a_status_string(int(status)).decode()


def v4a_version() -> int:
    return int(lib.v4a_version())


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def _io(x, gate, out, out_scale, out_exp=None) -> CompressIO:
    """One compress stream.  out_exp given: MXFP4 output, out holding [batch][entries][channels/2]
    code bytes and out_exp [batch][entries][channels/32] block exponents."""
    for t, name in ((x, "x"), (gate, "gate"), (out, "out")):
        if t.dim() != 3 or t.stride(2) != 1 or t.stride(1) != t.shape[2]:
            raise ValueError(f"{name} must be [batch][rows][channels] with dense rows")
    sc_stride = 0
    if out_scale is not None:
        if out_scale.dim() != 2 or out_scale.stride(1) != 1:
            raise ValueError("out_scale must be [batch][entries] with dense rows")
        sc_stride = out_scale.stride(0)
    if out_exp is None:
        return CompressIO(_ptr(x), _ptr(gate), _ptr(out), _ptr(out_scale), int(x.shape[2]), _dtype(x), _dtype(out),
                          x.stride(0), gate.stride(0), out.stride(0), sc_stride, None, 0)
    if out.dtype != torch.uint8 or out.shape[2] * 2 != x.shape[2]:
        raise ValueError("MXFP4 out must be uint8 [batch][entries][channels/2]")
    if out_exp.dtype != torch.uint8 or out_exp.dim() != 3 or out_exp.stride(2) != 1 or \
            out_exp.stride(1) != out_exp.shape[2] or out_exp.shape[2] * 32 != x.shape[2]:
        raise ValueError("out_exp must be uint8 [batch][entries][channels/32] with dense rows")
    return CompressIO(_ptr(x), _ptr(gate), _ptr(out), None, int(x.shape[2]), _dtype(x), MXFP4, x.stride(0),
                      gate.stride(0), 2 * out.stride(0), 0, _ptr(out_exp), out_exp.stride(0))


def v4a_compress(x, gate, out, *, m: int, n_tok: int | None = None, out_scale=None, xi=None, gate_i=None,
                 out_i=None, out_i_scale=None, out_i_exp=None, stream=None) -> None:
    """Compress complete m-token chunks of x (gated by `gate`) into `out`;
    optionally the indexer-key stream (xi, gate_i -> out_i [, out_i_scale]) in
    the same launch; out_i_exp given: the indexer keys are written as MXFP4
    (codes in out_i, block exponents in out_i_exp).  Tensors are
    [batch][rows][channels] (views into larger buffers are fine: the batch
    stride is read off the tensor)."""
    n = x.shape[1] if n_tok is None else int(n_tok)
    kv = _io(x, gate, out, out_scale)
    idx = None
    if xi is not None:
        idx = _io(xi, gate_i, out_i, out_i_scale, out_i_exp)
    _check(lib.v4a_compress(ctypes.byref(kv), ctypes.byref(idx) if idx is not None else None, int(x.shape[0]), n,
                            int(m), _stream(stream)))


def v4a_compress_dual(x_a, gate_a, x_b, gate_b, out, *, m: int, prev_x_b=None, prev_gate_b=None, out_scale=None,
                      n_tok: int | None = None, stream=None) -> None:
    """Dual-series compression: entry s of the range mixes series a over block s and series b over
    block s-1 (prev_x_b / prev_gate_b [batch][m][channels] for block -1, or None at the start of a
    sequence) under one per-channel softmax.  Tensors are [batch][rows][channels]."""
    n = x_a.shape[1] if n_tok is None else int(n_tok)
    a = _io(x_a, gate_a, out, out_scale)
    for t, name in ((x_b, "x_b"), (gate_b, "gate_b"), (prev_x_b, "prev_x_b"), (prev_gate_b, "prev_gate_b")):
        if t is not None and (t.dim() != 3 or t.stride(2) != 1 or t.stride(1) != t.shape[2]):
            raise ValueError(f"{name} must be [batch][rows][channels] with dense rows")
    prev_bs = prev_x_b.stride(0) if prev_x_b is not None else 0
    if prev_x_b is not None and prev_gate_b is not None and prev_gate_b.stride(0) != prev_bs:
        raise ValueError("prev_x_b and prev_gate_b must have the same batch stride")
    b = SeriesB(_ptr(x_b), _ptr(gate_b), _ptr(prev_x_b), _ptr(prev_gate_b), x_b.stride(0), gate_b.stride(0), prev_bs)
    _check(lib.v4a_compress_dual(ctypes.byref(a), ctypes.byref(b), int(x_a.shape[0]), n, int(m), _stream(stream)))


def v4a_quantize_mxfp4(x, codes, exps, stream=None) -> None:
    """MXFP4 quantisation of x [..][cols] (fp32 or bf16, cols a multiple of 32) into codes
    [..][cols/2] and exps [..][cols/32] (uint8)."""
    for t, n in ((x, "x"), (codes, "codes"), (exps, "exps")):
        _contig(t, n)
    cols = int(x.shape[-1])
    rows = x.numel() // cols if cols else 0
    if codes.dtype != torch.uint8 or exps.dtype != torch.uint8 or codes.numel() * 2 != x.numel() or \
            exps.numel() * 32 != x.numel():
        raise ValueError("codes / exps must be uint8 with numel x/2 and x/32")
    _check(lib.v4a_quantize_mxfp4(_ptr(x), _dtype(x), rows, cols, _ptr(codes), _ptr(exps), _stream(stream)))


def v4a_index_scores_mxfp4(q_i, w, k_codes, k_exp, scores, *, m: int, ctx_len: int, stream=None) -> None:
    """Indexer scores with MXFP4 keys (k_codes [B][N][d_i/2], k_exp [B][N][d_i/32]) and the query
    quantised to MXFP4 per head inside the call."""
    for t, n in ((q_i, "q_i"), (w, "w"), (k_codes, "k_codes"), (k_exp, "k_exp"), (scores, "scores")):
        _contig(t, n)
    B, T, HI, DI = q_i.shape
    s = _shape(batch=B, n_q=T, m=m, ctx_len=ctx_len)
    _check(lib.v4a_index_scores_mxfp4(_ptr(q_i), _ptr(w), _ptr(k_codes), _ptr(k_exp), _ptr(scores), HI, DI,
                                      _dtype(q_i), ctypes.byref(s), _stream(stream)))


def v4a_topk_mxfp4(q_i, w, k_codes, k_exp, idx_out, score_out=None, *, m: int, k: int, ctx_len: int,
                   workspace=None, stream=None) -> None:
    """Indexer + top-k with MXFP4 keys and FP4 dot products (see v4a_index_scores_mxfp4)."""
    for t, n in ((q_i, "q_i"), (w, "w"), (k_codes, "k_codes"), (k_exp, "k_exp"), (idx_out, "idx_out"),
                 (score_out, "score_out")):
        _contig(t, n)
    B, T, HI, DI = q_i.shape
    s = _shape(batch=B, n_q=T, m=m, k=k, ctx_len=ctx_len)
    if workspace is None:
        workspace = _workspace(lib.v4a_workspace_size(b"topk", ctypes.byref(s), HI, DI), q_i.device)
    _check(lib.v4a_topk_mxfp4(_ptr(q_i), _ptr(w), _ptr(k_codes), _ptr(k_exp), _ptr(idx_out), _ptr(score_out), HI, DI,
                              _dtype(q_i), _ptr(workspace), workspace.numel() * workspace.element_size(),
                              ctypes.byref(s), _stream(stream)))


def v4a_index_scores(q_i, w, k_i, k_scale, scores, *, m: int, ctx_len: int, stream=None) -> None:
    for t, n in ((q_i, "q_i"), (w, "w"), (k_i, "k_i"), (k_scale, "k_scale"), (scores, "scores")):
        _contig(t, n)
    B, T, HI, DI = q_i.shape
    s = _shape(batch=B, n_q=T, m=m, ctx_len=ctx_len)
    _check(lib.v4a_index_scores(_ptr(q_i), _ptr(w), _ptr(k_i), _ptr(k_scale), _ptr(scores), HI, DI, _dtype(q_i),
                                _dtype(k_i), ctypes.byref(s), _stream(stream)))


def v4a_topk(q_i, w, k_i, k_scale, idx_out, score_out=None, *, m: int, k: int, ctx_len: int, workspace=None,
             stream=None) -> None:
    for t, n in ((q_i, "q_i"), (w, "w"), (k_i, "k_i"), (k_scale, "k_scale"), (idx_out, "idx_out"),
                 (score_out, "score_out")):
        _contig(t, n)
    B, T, HI, DI = q_i.shape
    s = _shape(batch=B, n_q=T, m=m, k=k, ctx_len=ctx_len)
    if workspace is None:
        workspace = _workspace(lib.v4a_workspace_size(b"topk", ctypes.byref(s), HI, DI), q_i.device)
    _check(lib.v4a_topk(_ptr(q_i), _ptr(w), _ptr(k_i), _ptr(k_scale), _ptr(idx_out), _ptr(score_out), HI, DI,
                        _dtype(q_i), _dtype(k_i), _ptr(workspace), workspace.numel() * workspace.element_size(),
                        ctypes.byref(s), _stream(stream)))


def v4a_topk_noalloc(q_i, w, k_i, k_scale, idx_out, score_out=None, *, m: int, k: int, ctx_len: int,
                     stream=None) -> None:
    """v4a_topk with the library's built-in scratch: no workspace argument and
    no device allocation (see include/v4a.h for the size limit)."""
    for t, n in ((q_i, "q_i"), (w, "w"), (k_i, "k_i"), (k_scale, "k_scale"), (idx_out, "idx_out"),
                 (score_out, "score_out")):
        _contig(t, n)
    B, T, HI, DI = q_i.shape
    s = _shape(batch=B, n_q=T, m=m, k=k, ctx_len=ctx_len)
    _check(lib.v4a_topk_noalloc(_ptr(q_i), _ptr(w), _ptr(k_i), _ptr(k_scale), _ptr(idx_out), _ptr(score_out), HI,
                                DI, _dtype(q_i), _dtype(k_i), ctypes.byref(s), _stream(stream)))


def _ext(sink, rope_dims: int, rope_base: float):
    """The _ex options, or None when neither the sink nor the output RoPE is asked for."""
    if sink is None and not rope_dims:
        return None
    if sink is not None:
        _contig(sink, "sink")
        if sink.dtype != torch.float32 or sink.dim() != 1:
            raise ValueError("sink must be a float32 vector [heads]")
    return AttendExt(_ptr(sink), int(rope_dims), float(rope_base))


def v4a_csa_attend(q, entries, idx, token_kv, tok_pos0: int, out, *, m: int, window: int, ctx_len: int,
                   workspace=None, dev_status=None, sink=None, rope_dims: int = 0, rope_base: float = 10000.0,
                   stream=None) -> None:
    """CSA attention; sink ([heads] fp32 logits) and rope_dims / rope_base select the attention sink
    and the output RoPE at minus the query position (v4a_csa_attend_ex)."""
    for t, n in ((q, "q"), (entries, "entries"), (idx, "idx"), (token_kv, "token_kv"), (out, "out")):
        _contig(t, n)
    B, T, H, d = q.shape
    s = _shape(batch=B, n_q=T, heads=H, d=d, m=m, k=idx.shape[-1], window=window, ctx_len=ctx_len)
    if workspace is None:
        workspace = _workspace(lib.v4a_workspace_size(b"csa_attend", ctypes.byref(s), 0, 0), q.device)
    args = (_ptr(q), _ptr(entries), _ptr(idx), _ptr(token_kv), int(tok_pos0), int(token_kv.shape[1]), _ptr(out),
            _dtype(q), _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_status))
    ext = _ext(sink, rope_dims, rope_base)
    if ext is None:
        _check(lib.v4a_csa_attend(*args, ctypes.byref(s), _stream(stream)))
    else:
        _check(lib.v4a_csa_attend_ex(*args, ctypes.byref(ext), ctypes.byref(s), _stream(stream)))


def v4a_hca_attend(q, entries, token_kv, tok_pos0: int, out, *, m: int, window: int, ctx_len: int, workspace=None,
                   sink=None, rope_dims: int = 0, rope_base: float = 10000.0, stream=None) -> None:
    """HCA attention; sink and rope_dims / rope_base as for v4a_csa_attend (v4a_hca_attend_ex)."""
    for t, n in ((q, "q"), (entries, "entries"), (token_kv, "token_kv"), (out, "out")):
        _contig(t, n)
    B, T, H, d = q.shape
    s = _shape(batch=B, n_q=T, heads=H, d=d, m=m, window=window, ctx_len=ctx_len)
    if workspace is None:
        workspace = _workspace(lib.v4a_workspace_size(b"hca_attend", ctypes.byref(s), 0, 0), q.device)
    args = (_ptr(q), _ptr(entries), _ptr(token_kv), int(tok_pos0), int(token_kv.shape[1]), _ptr(out), _dtype(q),
            _ptr(workspace), workspace.numel() * workspace.element_size())
    ext = _ext(sink, rope_dims, rope_base)
    if ext is None:
        _check(lib.v4a_hca_attend(*args, ctypes.byref(s), _stream(stream)))
    else:
        _check(lib.v4a_hca_attend_ex(*args, ctypes.byref(ext), ctypes.byref(s), _stream(stream)))


# ----------------------------------------------------------------------
# heterogeneous KV cache: paged classical cache + token rings
# ----------------------------------------------------------------------

def _paged(block_table, block_tokens: int, n_blocks: int, ring_rows: int = 0) -> Paged:
    _contig(block_table, "block_table")
    if block_table.dtype != torch.int32 or block_table.dim() != 2:
        raise ValueError("block_table must be int32 [batch][blocks]")
    return Paged(_ptr(block_table), int(block_table.shape[1]), int(block_tokens), int(n_blocks), int(ring_rows))


def v4a_ring_append(pairs, pos: int, stream=None) -> None:
    """Append the token at position `pos`: for each (src [batch][channels], ring [batch][ring_rows][channels])
    pair, src row b goes to ring row pos % ring_rows of sequence b (one launch for up to 8 pairs)."""
    ios = (RingIO * max(1, len(pairs)))()
    batch = None
    for i, (src, ring) in enumerate(pairs):
        if src.dim() != 2 or src.stride(1) != 1 or ring.dim() != 3 or not ring.is_contiguous():
            raise ValueError("src must be [batch][channels] with dense rows, ring [batch][rows][channels] contiguous")
        if src.dtype != ring.dtype or src.shape[1] != ring.shape[2] or src.shape[0] != ring.shape[0]:
            raise ValueError("src and ring disagree")
        batch = int(src.shape[0]) if batch is None else batch
        ios[i] = RingIO(_ptr(src), _ptr(ring), int(ring.shape[2]), int(ring.shape[1]), _dtype(src), src.stride(0))
    _check(lib.v4a_ring_append(ios, len(pairs), batch or 0, int(pos), _stream(stream)))


def _pool_io(x, gate, out, out_scale=None, out_exp=None) -> CompressIO:
    """A compress stream whose output is a pool of rows [pool_rows][channels] (codes [pool_rows][channels/2]
    with exps [pool_rows][channels/32] for MXFP4)."""
    for t, name in ((x, "x"), (gate, "gate")):
        if t.dim() != 3 or t.stride(2) != 1 or t.stride(1) != t.shape[2]:
            raise ValueError(f"{name} must be [batch][rows][channels] with dense rows")
    _contig(out, "out")
    C = int(x.shape[2])
    if out_exp is not None:
        _contig(out_exp, "out_exp")
        return CompressIO(_ptr(x), _ptr(gate), _ptr(out), None, C, _dtype(x), MXFP4, x.stride(0), gate.stride(0), 0, 0,
                          _ptr(out_exp), 0)
    if out_scale is not None:
        _contig(out_scale, "out_scale")
    return CompressIO(_ptr(x), _ptr(gate), _ptr(out), _ptr(out_scale), C, _dtype(x), _dtype(out), x.stride(0),
                      gate.stride(0), 0, 0, None, 0)


def v4a_compress_paged(x, gate, out_pool, *, m: int, first_entry: int, block_table, block_tokens: int,
                       n_tok: int | None = None, out_scale=None, xi=None, gate_i=None, out_i=None, out_i_scale=None,
                       out_i_exp=None, stream=None) -> None:
    """Compress complete chunks of x (e.g. a slice of the token rings) into pool rows through the block
    table: entry first_entry + s of sequence b -> row block_table[b][e // epb] * epb + e % epb (epb =
    block_tokens // m).  The indexer-key stream (xi, gate_i -> out_i pools) rides in the same launch."""
    n = x.shape[1] if n_tok is None else int(n_tok)
    epb = block_tokens // m
    kv = _pool_io(x, gate, out_pool, out_scale)
    idx = _pool_io(xi, gate_i, out_i, out_i_scale, out_i_exp) if xi is not None else None
    pg = _paged(block_table, block_tokens, out_pool.shape[0] // epb)
    _check(lib.v4a_compress_paged(ctypes.byref(kv), ctypes.byref(idx) if idx is not None else None, int(x.shape[0]),
                                  n, int(m), int(first_entry), ctypes.byref(pg), _stream(stream)))


def v4a_topk_paged(q_i, w, k_pool, k_scale_pool, idx_out, score_out=None, *, m: int, k: int, ctx_len: int,
                   block_table, block_tokens: int, workspace=None, dev_status=None, stream=None) -> None:
    """v4a_topk over key pools [pool_rows][d_i] (+ scales [pool_rows]) addressed through the block table."""
    for t, n in ((q_i, "q_i"), (w, "w"), (k_pool, "k_pool"), (k_scale_pool, "k_scale_pool"), (idx_out, "idx_out"),
                 (score_out, "score_out")):
        _contig(t, n)
    B, T, HI, DI = q_i.shape
    s = _shape(batch=B, n_q=T, m=m, k=k, ctx_len=ctx_len)
    pg = _paged(block_table, block_tokens, k_pool.shape[0] // (block_tokens // m))
    if workspace is None:
        workspace = _workspace(lib.v4a_workspace_size(b"topk", ctypes.byref(s), HI, DI), q_i.device)
    _check(lib.v4a_topk_paged(_ptr(q_i), _ptr(w), _ptr(k_pool), _ptr(k_scale_pool), _ptr(idx_out), _ptr(score_out),
                              HI, DI, _dtype(q_i), _dtype(k_pool), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _ptr(dev_status), ctypes.byref(pg),
                              ctypes.byref(s), _stream(stream)))


def v4a_topk_mxfp4_paged(q_i, w, k_codes_pool, k_exp_pool, idx_out, score_out=None, *, m: int, k: int, ctx_len: int,
                         block_table, block_tokens: int, workspace=None, dev_status=None, stream=None) -> None:
    """v4a_topk_mxfp4 over MXFP4 key pools (codes [pool_rows][d_i/2], exps [pool_rows][d_i/32])."""
    for t, n in ((q_i, "q_i"), (w, "w"), (k_codes_pool, "k_codes_pool"), (k_exp_pool, "k_exp_pool"),
                 (idx_out, "idx_out"), (score_out, "score_out")):
        _contig(t, n)
    B, T, HI, DI = q_i.shape
    s = _shape(batch=B, n_q=T, m=m, k=k, ctx_len=ctx_len)
    pg = _paged(block_table, block_tokens, k_codes_pool.shape[0] // (block_tokens // m))
    if workspace is None:
        workspace = _workspace(lib.v4a_workspace_size(b"topk", ctypes.byref(s), HI, DI), q_i.device)
    _check(lib.v4a_topk_mxfp4_paged(_ptr(q_i), _ptr(w), _ptr(k_codes_pool), _ptr(k_exp_pool), _ptr(idx_out),
                                    _ptr(score_out), HI, DI, _dtype(q_i), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _ptr(dev_status), ctypes.byref(pg),
                                    ctypes.byref(s), _stream(stream)))


def v4a_csa_attend_paged(q, ent_pool, idx, ring, out, *, m: int, window: int, ctx_len: int, block_table,
                         block_tokens: int, workspace=None, dev_status=None, sink=None, rope_dims: int = 0,
                         rope_base: float = 10000.0, stream=None) -> None:
    """CSA attention over an entry pool [pool_rows][d] (block table) and the K=V ring [batch][ring_rows][d]."""
    for t, n in ((q, "q"), (ent_pool, "ent_pool"), (idx, "idx"), (ring, "ring"), (out, "out")):
        _contig(t, n)
    B, T, H, d = q.shape
    s = _shape(batch=B, n_q=T, heads=H, d=d, m=m, k=idx.shape[-1], window=window, ctx_len=ctx_len)
    pg = _paged(block_table, block_tokens, ent_pool.shape[0] // (block_tokens // m), ring.shape[1])
    if workspace is None:
        workspace = _workspace(lib.v4a_workspace_size(b"csa_attend", ctypes.byref(s), 0, 0), q.device)
    ext = _ext(sink, rope_dims, rope_base)
    _check(lib.v4a_csa_attend_paged(_ptr(q), _ptr(ent_pool), _ptr(idx), _ptr(ring), _ptr(out), _dtype(q),
                                    _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_status),
                                    ctypes.byref(ext) if ext is not None else None, ctypes.byref(pg), ctypes.byref(s),
                                    _stream(stream)))


def v4a_hca_attend_paged(q, ent_pool, ring, out, *, m: int, window: int, ctx_len: int, block_table,
                         block_tokens: int, workspace=None, dev_status=None, sink=None, rope_dims: int = 0,
                         rope_base: float = 10000.0, stream=None) -> None:
    """HCA attention over an entry pool [pool_rows][d] (block table) and the K=V ring."""
    for t, n in ((q, "q"), (ent_pool, "ent_pool"), (ring, "ring"), (out, "out")):
        _contig(t, n)
    B, T, H, d = q.shape
    s = _shape(batch=B, n_q=T, heads=H, d=d, m=m, window=window, ctx_len=ctx_len)
    pg = _paged(block_table, block_tokens, ent_pool.shape[0] // (block_tokens // m), ring.shape[1])
    if workspace is None:
        workspace = _workspace(lib.v4a_workspace_size(b"hca_attend", ctypes.byref(s), 0, 0), q.device)
    ext = _ext(sink, rope_dims, rope_base)
    _check(lib.v4a_hca_attend_paged(_ptr(q), _ptr(ent_pool), _ptr(ring), _ptr(out), _dtype(q), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _ptr(dev_status),
                                    ctypes.byref(ext) if ext is not None else None, ctypes.byref(pg), ctypes.byref(s),
                                    _stream(stream)))
