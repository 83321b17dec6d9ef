"""Seeded synthetic inputs for the compressed-attention workloads.

This module only draws random numbers and stores them in the formats the
workloads name (float32, bfloat16, float8 e4m3 with one float32 scale per
row).  It holds none of the method's arithmetic; the CUDA library and the CPU
oracle both consume exactly the bytes it returns.

Every builder takes a seed and returns a dict of contiguous CPU tensors plus
the integer parameters of the case.  The named workloads (``CONFIGS``) are the
five published shapes:

* ``fp32_l4096``: CSA + HCA decode, one query, 4,096-token context, fp32,
  d = 128, 16 heads, indexer 4 x 64, top-64, HCA 32 entries, window 128.
* ``csa_l64k``: CSA decode, batch 8, 65,536-token context, bf16, d = 512,
  64 heads, indexer 16 x 128 (bf16 keys), top-512.
* ``hca_l1m``: HCA decode, batch 32, 1,048,576-token context, bf16, 8,192
  entries of d = 512, 64 heads.
* ``csa_l1m_fp8``: CSA decode, batch 4, 1,048,576-token context, 262,144
  entries, bf16 K=V, FP8-e4m3 indexer keys with a per-entry fp32 scale,
  top-1024.
* ``prefill_c4096``: a 4,096-token causal prefill chunk at positions
  126,976 ... 131,071 of a 131,072-token bf16 sequence, top-512.
"""
from __future__ import annotations

import math

import torch

FP8_MAX = 448.0  # largest finite float8 e4m3 magnitude


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(int(seed))
    return g


def normal(g: torch.Generator, shape, std: float = 1.0) -> torch.Tensor:
    t = torch.randn(shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t


def uniform(g: torch.Generator, shape) -> torch.Tensor:
    return torch.rand(shape, generator=g, dtype=torch.float32)


def store(t32: torch.Tensor, fmt: str) -> torch.Tensor:
    """fp32 master -> stored tensor ('f32' or 'bf16', round-to-nearest-even)."""
    if fmt == "f32":
        return t32.contiguous()
    if fmt == "bf16":
        return t32.to(torch.bfloat16).contiguous()
    raise ValueError(fmt)


def store_e4m3_rows(t32: torch.Tensor):
    """fp32 master [..., C] -> (uint8 e4m3 codes [..., C], fp32 scale [...]) with
    scale = amax/448 per row (1 for an all-zero row); the cast is torch's."""
    amax = t32.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / FP8_MAX, torch.ones_like(amax)).to(torch.float32)
    codes = (t32 / scale.unsqueeze(-1)).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.contiguous()


def _normal_stored(g, shape, fmt, std=1.0, chunk_dim0=False):
    """Draw N(0, std^2) and store it; large tensors are drawn slice by slice
    along dim 0 to bound the fp32 master's footprint."""
    if not chunk_dim0 or shape[0] == 1:
        return store(normal(g, shape, std), fmt)
    out = torch.empty(shape, dtype=torch.float32 if fmt == "f32" else torch.bfloat16)
    for i in range(shape[0]):
        out[i] = store(normal(g, shape[1:], std), fmt)
    return out


def window_rows(ctx_len: int, n_q: int, window: int):
    """(tok_pos0, l_tok): the token rows every query's window needs."""
    p0 = max(0, ctx_len - n_q - window + 1)
    return p0, ctx_len - p0


# ----------------------------------------------------------------------
# generic builders
# ----------------------------------------------------------------------

def compress_case(batch: int, n_tok: int, channels: int, fmt: str, seed: int, gate_std: float = 1.0):
    g = _gen(seed)
    x = store(normal(g, (batch, n_tok, channels)), fmt)
    z = store(normal(g, (batch, n_tok, channels), gate_std), fmt)
    return dict(x=x, gate=z)


def index_case(batch, n_q, ctx_len, m, heads_i, d_i, q_fmt, key_fmt, seed, n_ent=None):
    """Indexer inputs: q_i, w, k_i (+ k_scale for e4m3 keys)."""
    g = _gen(seed)
    N = ctx_len // m if n_ent is None else n_ent
    q_i = store(normal(g, (batch, n_q, heads_i, d_i)), q_fmt)
    w = uniform(g, (batch, n_q, heads_i))
    if key_fmt == "e4m3":
        k32 = normal(g, (batch, N, d_i))
        k_i, k_scale = store_e4m3_rows(k32)
        del k32
    else:
        k_i, k_scale = _normal_stored(g, (batch, N, d_i), key_fmt, chunk_dim0=True), None
    return dict(q_i=q_i, w=w, k_i=k_i, k_scale=k_scale)


def attend_case(batch, n_q, ctx_len, m, heads, d, window, fmt, seed, q_std=1.0, entry_std=1.0):
    """Attention inputs: q, entries (all ctx_len//m of them), window token rows."""
    g = _gen(seed)
    N = ctx_len // m
    tok_pos0, l_tok = window_rows(ctx_len, n_q, window)
    q = store(normal(g, (batch, n_q, heads, d), q_std), fmt)
    entries = _normal_stored(g, (batch, N, d), fmt, entry_std, chunk_dim0=True)
    token_kv = store(normal(g, (batch, l_tok, d), entry_std), fmt)
    return dict(q=q, entries=entries, token_kv=token_kv, tok_pos0=tok_pos0)


def random_topk_idx(batch, n_q, ctx_len, m, k, seed, pad_fraction=0.0):
    """Random valid selections (ascending, distinct, visible, -1 padded) for
    exercising the attention kernels on their own."""
    g = _gen(seed)
    idx = torch.full((batch, n_q, k), -1, dtype=torch.int32)
    for b in range(batch):
        for j in range(n_q):
            t = ctx_len - n_q + j
            nvis = (t + 1) // m
            take = min(k, nvis)
            if pad_fraction > 0 and take > 1:
                take = max(1, int(take * (1.0 - pad_fraction)))
            if take > 0:
                sel = torch.randperm(nvis, generator=g)[:take].sort().values
                idx[b, j, :take] = sel.to(torch.int32)
    return idx


# ----------------------------------------------------------------------
# the named workloads
# ----------------------------------------------------------------------

CONFIGS = {
    "fp32_l4096": dict(kind="csa+hca", batch=1, ctx_len=4096, heads=16, d=128, m=4, m_hca=128, heads_i=4, d_i=64,
                       k=64, window=128, fmt="f32", key_fmt="f32", q_std=1.0 / math.sqrt(128), seed=1234),
    "csa_l64k": dict(kind="csa", batch=8, ctx_len=65536, heads=64, d=512, m=4, heads_i=16, d_i=128, k=512,
                     window=128, fmt="bf16", key_fmt="bf16", q_std=1.0, seed=1235),
    "hca_l1m": dict(kind="hca", batch=32, ctx_len=1048576, heads=64, d=512, m=128, window=128, fmt="bf16",
                    q_std=1.0, seed=1236),
    "csa_l1m_fp8": dict(kind="csa", batch=4, ctx_len=1048576, heads=64, d=512, m=4, heads_i=16, d_i=128, k=1024,
                        window=128, fmt="bf16", key_fmt="e4m3", q_std=1.0, seed=1237),
    "prefill_c4096": dict(kind="prefill", batch=1, ctx_len=131072, n_q=4096, heads=64, d=512, m=4, heads_i=16,
                          d_i=128, k=512, window=128, fmt="bf16", key_fmt="bf16", q_std=1.0, seed=1238),
}


def fp32_l4096(seed: int | None = None):
    """Token KV x, two sets of gate logits (CSA, HCA layers), queries and the
    indexer's keys; the compressed entries are the path's own output."""
    c = CONFIGS["fp32_l4096"]
    g = _gen(c["seed"] if seed is None else seed)
    L, d = c["ctx_len"], c["d"]
    x = normal(g, (1, L, d))
    z_csa = normal(g, (1, L, d))
    z_hca = normal(g, (1, L, d))
    q = normal(g, (1, 1, c["heads"], d), c["q_std"])
    k_i = normal(g, (1, L // c["m"], c["d_i"]))
    q_i = normal(g, (1, 1, c["heads_i"], c["d_i"]))
    w = uniform(g, (1, 1, c["heads_i"]))
    return dict(cfg=c, x=x, z_csa=z_csa, z_hca=z_hca, q=q, q_i=q_i, w=w, k_i=k_i, k_scale=None,
                token_kv=x, tok_pos0=0)


def csa_decode(name: str, seed: int | None = None, with_tail: bool = True, key_fmt: str | None = None):
    """CSA decode at the last position t = L-1 of each sequence.  History
    entries and indexer keys for s < N-1 are drawn; with_tail additionally
    draws the raw inputs of the chunk that completes at t (its token rows are
    the last m window rows, plus gate logits and the indexer's token keys and
    gates), whose entry N-1 the path compresses itself.  key_fmt overrides the
    stored format of the indexer keys (e.g. 'bf16' masters that a caller then
    quantises to MXFP4); the draws are the same N(0,1) values either way."""
    c = dict(CONFIGS[name])
    if key_fmt is not None:
        c["key_fmt"] = key_fmt
    g = _gen(c["seed"] if seed is None else seed)
    B, L, H, d, m = c["batch"], c["ctx_len"], c["heads"], c["d"], c["m"]
    N = L // m
    tok_pos0, l_tok = window_rows(L, 1, c["window"])
    q = store(normal(g, (B, 1, H, d), c["q_std"]), c["fmt"])
    token_kv = store(normal(g, (B, l_tok, d)), c["fmt"])
    entries = _normal_stored(g, (B, N, d), c["fmt"], chunk_dim0=True)
    q_i = store(normal(g, (B, 1, c["heads_i"], c["d_i"])), c["fmt"])
    w = uniform(g, (B, 1, c["heads_i"]))
    if c["key_fmt"] == "e4m3":
        k_i = torch.empty((B, N, c["d_i"]), dtype=torch.uint8)
        k_scale = torch.empty((B, N), dtype=torch.float32)
        for b in range(B):
            k_i[b], k_scale[b] = store_e4m3_rows(normal(g, (N, c["d_i"])))
    else:
        k_i, k_scale = _normal_stored(g, (B, N, c["d_i"]), c["key_fmt"], chunk_dim0=True), None
    out = dict(cfg=c, q=q, token_kv=token_kv, tok_pos0=tok_pos0, entries=entries, q_i=q_i, w=w, k_i=k_i,
               k_scale=k_scale)
    if with_tail:
        out["gate_tail"] = store(normal(g, (B, m, d)), c["fmt"])
        out["xi_tail"] = store(normal(g, (B, m, c["d_i"])), c["fmt"])
        out["gate_i_tail"] = store(normal(g, (B, m, c["d_i"])), c["fmt"])
    return out


def hca_decode(name: str = "hca_l1m", seed: int | None = None, with_tail: bool = True):
    """HCA decode at t = L-1; entries s < N-1 drawn, the completing chunk's
    gate logits drawn (its tokens are the m' = 128 window rows)."""
    c = CONFIGS[name]
    g = _gen(c["seed"] if seed is None else seed)
    B, L, H, d, m = c["batch"], c["ctx_len"], c["heads"], c["d"], c["m"]
    N = L // m
    tok_pos0, l_tok = window_rows(L, 1, c["window"])
    q = store(normal(g, (B, 1, H, d), c["q_std"]), c["fmt"])
    token_kv = store(normal(g, (B, l_tok, d)), c["fmt"])
    entries = _normal_stored(g, (B, N, d), c["fmt"], chunk_dim0=True)
    out = dict(cfg=c, q=q, token_kv=token_kv, tok_pos0=tok_pos0, entries=entries)
    if with_tail:
        out["gate_tail"] = store(normal(g, (B, m, d)), c["fmt"])
    return out


def prefill_chunk(name: str = "prefill_c4096", seed: int | None = None):
    """Prefill chunk: history entries/keys for the 31,744 entries before the
    chunk, the chunk's token rows X and gate logits (KV and indexer streams),
    127 earlier token rows so the first queries' windows are complete, and
    per-query q, q_i, w."""
    c = CONFIGS[name]
    g = _gen(c["seed"] if seed is None else seed)
    B, L, T, H, d, m = c["batch"], c["ctx_len"], c["n_q"], c["heads"], c["d"], c["m"]
    N = L // m
    start = L - T
    n_hist = start // m
    hist_entries = store(normal(g, (B, n_hist, d)), c["fmt"])
    hist_keys = store(normal(g, (B, n_hist, c["d_i"])), c["key_fmt"])
    x = store(normal(g, (B, T, d)), c["fmt"])
    z = store(normal(g, (B, T, d)), c["fmt"])
    xi = store(normal(g, (B, T, c["d_i"])), c["fmt"])
    zi = store(normal(g, (B, T, c["d_i"])), c["fmt"])
    tok_pos0 = start - (c["window"] - 1)
    pre = store(normal(g, (B, c["window"] - 1, d)), c["fmt"])
    token_kv = torch.cat([pre, x], dim=1).contiguous()
    q = store(normal(g, (B, T, H, d), c["q_std"]), c["fmt"])
    q_i = store(normal(g, (B, T, c["heads_i"], c["d_i"])), c["fmt"])
    w = uniform(g, (B, T, c["heads_i"]))
    return dict(cfg=c, N=N, n_hist=n_hist, hist_entries=hist_entries, hist_keys=hist_keys, x=x, gate=z, xi=xi,
                gate_i=zi, token_kv=token_kv, tok_pos0=tok_pos0, q=q, q_i=q_i, w=w)


def stored_numpy(t: torch.Tensor):
    """The stored bytes of a tensor as the numpy array the oracle takes
    (float32, bfloat16 as uint16, e4m3 as uint8)."""
    if t.dtype == torch.bfloat16:
        return t.contiguous().view(torch.int16).numpy().view("uint16")
    if t.dtype == torch.float8_e4m3fn:
        return t.contiguous().view(torch.uint8).numpy()
    return t.contiguous().numpy()
