"""CPU oracle for the hybrid compressed-attention step (test infrastructure).

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference legs of ``bench.py`` may import this package.  It wraps the plain C
implementation in ``v4a_oracle.c`` (binary64 accumulation, storage formats
decoded from their definitions) through ctypes and numpy; it never touches the
CUDA library and the CUDA library never touches it.

Every function returns numpy arrays.  Inputs are numpy arrays (or anything
``numpy.ascontiguousarray`` accepts) holding the *stored* bytes: float32,
bfloat16 as uint16 bit patterns, e4m3 as uint8 codes, binary64 values as
float64 (the decoded operands of the MXFP4 indexer).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

F32, BF16, E4M3, F64 = 0, 1, 2, 3  # storage-format codes of the oracle's own C API

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "v4a_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile v4a_oracle.c into liboracle.so beside it (gcc, -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-shared", "-fPIC", "-o", _LIB, _SRC,
                               "-lm", "-lpthread"])
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    ll, i32, dbl, vp = ctypes.c_longlong, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
    lib.v4ao_bf16_decode.restype = dbl
    lib.v4ao_bf16_decode.argtypes = [ctypes.c_uint16]
    lib.v4ao_bf16_encode.restype = ctypes.c_uint16
    lib.v4ao_bf16_encode.argtypes = [dbl]
    lib.v4ao_e4m3_decode.restype = dbl
    lib.v4ao_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.v4ao_e4m3_encode.restype = ctypes.c_uint8
    lib.v4ao_e4m3_encode.argtypes = [dbl]
    lib.v4ao_e2m1_decode.restype = dbl
    lib.v4ao_e2m1_decode.argtypes = [ctypes.c_uint8]
    lib.v4ao_e2m1_encode.restype = ctypes.c_uint8
    lib.v4ao_e2m1_encode.argtypes = [dbl]
    lib.v4ao_quantize_mxfp4.restype = i32
    lib.v4ao_quantize_mxfp4.argtypes = [vp, ll, ll, vp, vp]
    lib.v4ao_decode_mxfp4.restype = i32
    lib.v4ao_decode_mxfp4.argtypes = [vp, vp, ll, ll, vp]
    lib.v4ao_set_threads.argtypes = [i32]
    lib.v4ao_get_threads.restype = i32
    lib.v4ao_n_visible.restype = ll
    lib.v4ao_n_visible.argtypes = [ll, ll]
    lib.v4ao_compress.restype = i32
    lib.v4ao_compress.argtypes = [vp, vp, i32, ll, ll, ll, ll, vp]
    lib.v4ao_attend_ex.restype = i32
    lib.v4ao_attend_ex.argtypes = [vp, vp, vp, ll, vp, ll, ll, i32, ll, ll, ll, ll, ll, ll, ll, vp, ll,
                                   ctypes.c_double, vp]
    lib.v4ao_rope.restype = i32
    lib.v4ao_rope.argtypes = [vp, ll, ll, vp, ll, ctypes.c_double]
    lib.v4ao_compress_dual.restype = i32
    lib.v4ao_compress_dual.argtypes = [vp, vp, vp, vp, vp, vp, i32, ll, ll, ll, ll, vp]
    lib.v4ao_quantize_e4m3_rows.restype = i32
    lib.v4ao_quantize_e4m3_rows.argtypes = [vp, ll, ll, vp, vp]
    lib.v4ao_index_scores.restype = i32
    lib.v4ao_index_scores.argtypes = [vp, i32, vp, vp, i32, vp, ll, ll, ll, ll, ll, ll, vp]
    lib.v4ao_select_row.restype = i32
    lib.v4ao_select_row.argtypes = [vp, ll, ll, vp, vp, vp]
    lib.v4ao_topk.restype = i32
    lib.v4ao_topk.argtypes = [vp, i32, vp, vp, i32, vp, ll, ll, ll, ll, ll, ll, ll, vp, vp, vp, vp]
    lib.v4ao_attend.restype = i32
    lib.v4ao_attend.argtypes = [vp, vp, vp, ll, vp, ll, ll, i32, ll, ll, ll, ll, ll, ll, ll, vp]
    lib.v4ao_attend_weights.restype = ll
    lib.v4ao_attend_weights.argtypes = [vp, vp, vp, ll, vp, ll, ll, i32, ll, ll, ll, ll, ll, ll, ll, ll, ll, vp]
    _lib = lib
    return lib


def _c(a, dtype=None):
    a = np.ascontiguousarray(a if dtype is None else np.asarray(a, dtype=dtype))
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def fmt_of(a: np.ndarray) -> int:
    """Storage-format code of a numpy array of stored bytes."""
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.uint8:
        return E4M3
    if a.dtype == np.float64:
        return F64
    raise TypeError(f"unsupported storage dtype {a.dtype}")


def set_threads(n: int) -> None:
    _load().v4ao_set_threads(int(n))


def get_threads() -> int:
    return int(_load().v4ao_get_threads())


def bf16_decode(codes) -> np.ndarray:
    lib = _load()
    c = np.asarray(codes, dtype=np.uint16)
    return np.array([lib.v4ao_bf16_decode(int(v)) for v in c.ravel()]).reshape(c.shape)


def bf16_encode(values) -> np.ndarray:
    lib = _load()
    v = np.asarray(values, dtype=np.float64)
    return np.array([lib.v4ao_bf16_encode(float(x)) for x in v.ravel()], dtype=np.uint16).reshape(v.shape)


def e4m3_decode(codes) -> np.ndarray:
    lib = _load()
    c = np.asarray(codes, dtype=np.uint8)
    return np.array([lib.v4ao_e4m3_decode(int(v)) for v in c.ravel()]).reshape(c.shape)


def e4m3_encode(values) -> np.ndarray:
    lib = _load()
    v = np.asarray(values, dtype=np.float64)
    return np.array([lib.v4ao_e4m3_encode(float(x)) for x in v.ravel()], dtype=np.uint8).reshape(v.shape)


_tables: dict = {}


def decode(a: np.ndarray) -> np.ndarray:
    """Stored bytes -> binary64 values, by the oracle's own decoders."""
    f = fmt_of(a)
    if f in (F32, F64):
        return a.astype(np.float64)
    if f not in _tables:
        fn = _load().v4ao_bf16_decode if f == BF16 else _load().v4ao_e4m3_decode
        _tables[f] = np.array([fn(i) for i in range(65536 if f == BF16 else 256)])
    return _tables[f][a]


def n_visible(t: int, m: int) -> int:
    """Entries visible to query position t: those s with m*(s+1) <= t+1."""
    return int(_load().v4ao_n_visible(int(t), int(m)))


def compress(x, gate, m: int) -> np.ndarray:
    """x, gate: [B][n_tok][C] stored bytes -> entries [B][n_tok//m][C] float64."""
    x, gate = _c(x), _c(gate)
    assert x.shape == gate.shape and x.dtype == gate.dtype and x.ndim == 3
    B, n_tok, C = x.shape
    out = np.zeros((B, n_tok // m, C), dtype=np.float64)
    st = _load().v4ao_compress(_ptr(x), _ptr(gate), fmt_of(x), B, n_tok, C, m, _ptr(out))
    if st:
        raise ValueError(f"oracle compress: status {st}")
    return out


def compress_dual(xa, za, xb, zb, m: int, prev_xb=None, prev_zb=None) -> np.ndarray:
    """Dual-series compression: xa, za, xb, zb [B][n_tok][C] stored bytes over the same token range
    (starting at a block boundary); prev_xb, prev_zb [B][m][C] series b over the block before the
    range, or None when the range starts the sequence -> entries [B][n_tok//m][C] float64."""
    xa, za, xb, zb = _c(xa), _c(za), _c(xb), _c(zb)
    assert xa.shape == za.shape == xb.shape == zb.shape and xa.ndim == 3
    assert xa.dtype == za.dtype == xb.dtype == zb.dtype
    B, n_tok, C = xa.shape
    if prev_xb is not None:
        prev_xb, prev_zb = _c(prev_xb), _c(prev_zb)
        assert prev_xb.shape == prev_zb.shape == (B, m, C) and prev_xb.dtype == xa.dtype
    out = np.zeros((B, n_tok // m, C), dtype=np.float64)
    st = _load().v4ao_compress_dual(_ptr(xa), _ptr(za), _ptr(xb), _ptr(zb), _ptr(prev_xb), _ptr(prev_zb), fmt_of(xa),
                                    B, n_tok, C, m, _ptr(out))
    if st:
        raise ValueError(f"oracle compress_dual: status {st}")
    return out


def quantize_e4m3_rows(values) -> tuple[np.ndarray, np.ndarray]:
    """Per-row e4m3 quantisation (scale = amax/448): returns (codes uint8, scales float64)."""
    v = _c(values, np.float64)
    rows = int(np.prod(v.shape[:-1]))
    codes = np.zeros(v.shape, dtype=np.uint8)
    scales = np.zeros(v.shape[:-1], dtype=np.float64)
    st = _load().v4ao_quantize_e4m3_rows(_ptr(v), rows, v.shape[-1], _ptr(codes), _ptr(scales))
    if st:
        raise ValueError(f"oracle quantize: status {st}")
    return codes, scales


def e2m1_decode(codes) -> np.ndarray:
    lib = _load()
    c = np.asarray(codes, dtype=np.uint8)
    return np.array([lib.v4ao_e2m1_decode(int(v)) for v in c.ravel()]).reshape(c.shape)


def e2m1_encode(values) -> np.ndarray:
    lib = _load()
    v = np.asarray(values, dtype=np.float64)
    return np.array([lib.v4ao_e2m1_encode(float(x)) for x in v.ravel()], dtype=np.uint8).reshape(v.shape)


def quantize_mxfp4(values) -> tuple[np.ndarray, np.ndarray]:
    """MXFP4 (OCP MX) quantisation along the last axis (a multiple of 32) of binary64 values:
    returns (codes uint8 [..][cols/2], two e2m1 codes per byte with the even element in the low
    nibble; exps uint8 [..][cols/32], the E8M0 block exponents X + 127)."""
    v = _c(values, np.float64)
    cols = v.shape[-1]
    rows = int(np.prod(v.shape[:-1]))
    codes = np.zeros(v.shape[:-1] + (cols // 2,), dtype=np.uint8)
    exps = np.zeros(v.shape[:-1] + (cols // 32,), dtype=np.uint8)
    st = _load().v4ao_quantize_mxfp4(_ptr(v), rows, cols, _ptr(codes), _ptr(exps))
    if st:
        raise ValueError(f"oracle quantize_mxfp4: status {st}")
    return codes, exps


def decode_mxfp4(codes, exps) -> np.ndarray:
    """MXFP4 codes [..][cols/2] and block exponents [..][cols/32] -> binary64 values [..][cols]."""
    c, x = _c(codes, np.uint8), _c(exps, np.uint8)
    cols = c.shape[-1] * 2
    assert x.shape == c.shape[:-1] + (cols // 32,)
    rows = int(np.prod(c.shape[:-1]))
    out = np.zeros(c.shape[:-1] + (cols,), dtype=np.float64)
    st = _load().v4ao_decode_mxfp4(_ptr(c), _ptr(x), rows, cols, _ptr(out))
    if st:
        raise ValueError(f"oracle decode_mxfp4: status {st}")
    return out


def mxfp4_query(q_i) -> np.ndarray:
    """The indexer query as the FP4 dot product sees it: every head's d_I values (stored bytes)
    quantised to MXFP4 and decoded back, as binary64."""
    return decode_mxfp4(*quantize_mxfp4(decode(_c(q_i))))


def index_scores_mxfp4(q_i, w, k_codes, k_exps, ctx_len: int, m: int) -> np.ndarray:
    """Indexer scores with MXFP4 keys (codes [B][N][d_I/2], exps [B][N][d_I/32]) and the query
    quantised to MXFP4 per head: the score definition on the decoded values of both operands."""
    return index_scores(mxfp4_query(q_i), w, decode_mxfp4(k_codes, k_exps), None, ctx_len, m)


def topk_mxfp4(q_i, w, k_codes, k_exps, ctx_len: int, m: int, k: int, want_scores: bool = False):
    """Indexer + top-k with MXFP4 keys and queries (see index_scores_mxfp4)."""
    return topk(mxfp4_query(q_i), w, decode_mxfp4(k_codes, k_exps), None, ctx_len, m, k, want_scores)


def index_scores(q_i, w, k_i, k_scale, ctx_len: int, m: int) -> np.ndarray:
    """q_i [B][T][H_I][d_I], w [B][T][H_I] f32, k_i [B][N][d_I], k_scale [B][N] f32 or None
    -> scores [B][T][N] float64 (-inf for entries not visible to the query)."""
    q_i, k_i = _c(q_i), _c(k_i)
    w = _c(w, np.float32)
    ks = None if k_scale is None else _c(k_scale, np.float32)
    B, T, HI, DI = q_i.shape
    N = ctx_len // m
    assert k_i.shape == (B, N, DI), (k_i.shape, (B, N, DI))
    out = np.zeros((B, T, N), dtype=np.float64)
    st = _load().v4ao_index_scores(_ptr(q_i), fmt_of(q_i), _ptr(w), _ptr(k_i), fmt_of(k_i), _ptr(ks), B, T,
                                   ctx_len, m, HI, DI, _ptr(out))
    if st:
        raise ValueError(f"oracle index_scores: status {st}")
    return out


def select_row(scores, nvis: int, k: int):
    """Top-k of one score row over its first nvis entries -> (idx int32 [k], sel [k], kth)."""
    s = _c(scores, np.float64)
    idx = np.zeros(k, dtype=np.int32)
    sel = np.zeros(k, dtype=np.float64)
    kth = ctypes.c_double(0.0)
    st = _load().v4ao_select_row(_ptr(s), nvis, k, _ptr(idx), _ptr(sel), ctypes.byref(kth))
    if st:
        raise ValueError(f"oracle select_row: status {st}")
    return idx, sel, kth.value


def topk(q_i, w, k_i, k_scale, ctx_len: int, m: int, k: int, want_scores: bool = False):
    """Indexer + top-k: returns dict(idx [B][T][k] int32 ascending, -1 padded; sel [B][T][k];
    kth [B][T]; scores [B][T][N] if want_scores)."""
    q_i, k_i = _c(q_i), _c(k_i)
    w = _c(w, np.float32)
    ks = None if k_scale is None else _c(k_scale, np.float32)
    B, T, HI, DI = q_i.shape
    N = ctx_len // m
    idx = np.zeros((B, T, k), dtype=np.int32)
    sel = np.zeros((B, T, k), dtype=np.float64)
    kth = np.zeros((B, T), dtype=np.float64)
    sc = np.zeros((B, T, N), dtype=np.float64) if want_scores else None
    st = _load().v4ao_topk(_ptr(q_i), fmt_of(q_i), _ptr(w), _ptr(k_i), fmt_of(k_i), _ptr(ks), B, T, ctx_len, m,
                           HI, DI, k, _ptr(idx), _ptr(sel), _ptr(kth), _ptr(sc))
    if st:
        raise ValueError(f"oracle topk: status {st}")
    r = dict(idx=idx, sel=sel, kth=kth)
    if want_scores:
        r["scores"] = sc
    return r


def attend(q, entries, idx, token_kv, tok_pos0: int, ctx_len: int, m: int, window: int,
           allow_bad_index: bool = False, sink=None, rope_dims: int = 0, rope_base: float = 10000.0) -> np.ndarray:
    """Joint-softmax attention over selected (idx given: CSA) or all visible
    (idx None: HCA) compressed entries plus the window tokens.
    q [B][T][H][d], entries [B][N][d], idx [B][T][k] int32 or None,
    token_kv [B][L_tok][d] (row r = position tok_pos0 + r) -> out [B][T][H][d] float64.
    sink: per-head sink logits [H] (joining each head's softmax denominator as e^sink), or None;
    rope_dims > 0: the output's last rope_dims dims rotated by RoPE at minus the query position."""
    q, entries, token_kv = _c(q), _c(entries), _c(token_kv)
    assert q.dtype == entries.dtype == token_kv.dtype
    B, T, H, d = q.shape
    ix = None if idx is None else _c(idx, np.int32)
    ksel = 0 if ix is None else ix.shape[-1]
    sk = None if sink is None else _c(sink, np.float64)
    assert sk is None or sk.shape == (H,)
    out = np.zeros((B, T, H, d), dtype=np.float64)
    st = _load().v4ao_attend_ex(_ptr(q), _ptr(entries), _ptr(ix), ksel, _ptr(token_kv), tok_pos0, token_kv.shape[1],
                                fmt_of(q), B, T, H, d, m, window, ctx_len, _ptr(sk), int(rope_dims), float(rope_base),
                                _ptr(out))
    if st and not (allow_bad_index and st == 4):
        raise ValueError(f"oracle attend: status {st}")
    return out


def rope(x, pos, rope_dims: int, base: float = 10000.0) -> np.ndarray:
    """RoPE on the last rope_dims dims of rows x [..][d] (float64 copy), row i at position pos[i]
    (pos broadcast over the leading dims)."""
    x = np.array(x, dtype=np.float64, copy=True)
    d = x.shape[-1]
    rows = x.reshape(-1, d)
    p = np.ascontiguousarray(np.broadcast_to(np.asarray(pos, dtype=np.float64), x.shape[:-1]).reshape(-1))
    st = _load().v4ao_rope(_ptr(rows), rows.shape[0], d, _ptr(p), int(rope_dims), float(base))
    if st:
        raise ValueError(f"oracle rope: status {st}")
    return rows.reshape(x.shape)


def attend_weights(q, entries, idx, token_kv, tok_pos0: int, ctx_len: int, m: int, window: int,
                   b: int, j: int, h: int) -> np.ndarray:
    """Softmax weights of one (sequence, query, head) over its candidate list."""
    q, entries, token_kv = _c(q), _c(entries), _c(token_kv)
    B, T, H, d = q.shape
    ix = None if idx is None else _c(idx, np.int32)
    ksel = 0 if ix is None else ix.shape[-1]
    cap = (ksel if ix is not None else ctx_len // m) + window + 1
    w = np.zeros(cap, dtype=np.float64)
    n = _load().v4ao_attend_weights(_ptr(q), _ptr(entries), _ptr(ix), ksel, _ptr(token_kv), tok_pos0,
                                    token_kv.shape[1], fmt_of(q), T, H, d, m, window, ctx_len, b, j, h, _ptr(w))
    if n < 0:
        raise ValueError("oracle attend_weights: bad argument")
    return w[:n]
