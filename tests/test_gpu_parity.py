"""GPU parity: every entry point of libv4a.so, called through the C ABI (via
the thin binding), against the CPU oracle on the same seeded inputs.

Small cases span several tiles and a ragged tail and cover the edge cases
(padding, ties, empty windows, contexts shorter than a chunk, bad indices);
the full-size workloads are checked on sampled sequences / query rows that the
oracle computes one by one.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workload as wl
from parity_utils import ATOL_F32, check_attention, check_scores, check_topk, dev, host

pytestmark = pytest.mark.gpu

cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


@pytest.fixture(scope="module")
def v4a():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import compressed_sparse_long_v4a_b200 as v
    return v


def _sync():
    torch.cuda.synchronize()


# ----------------------------------------------------------------------
# compress
# ----------------------------------------------------------------------

@pytest.mark.parametrize("fmt,m,n_tok,C", [("f32", 4, 4 * 37 + 3, 128), ("f32", 1, 29, 64), ("f32", 128, 128 * 5 + 17, 128),
                                         ("bf16", 4, 4 * 300 + 1, 512), ("bf16", 128, 128 * 3, 512),
                                         # long chunks with a partial channel tile and a chunk not a multiple of 32
                                         ("bf16", 40, 40 * 7 + 3, 72), ("f32", 64, 64 * 4, 264)])
def test_compress_matches_oracle(v4a, fmt, m, n_tok, C):
    case = wl.compress_case(2, n_tok, C, fmt, seed=100 + m + C)
    x, z = dev(case["x"]), dev(case["gate"])
    n_ent = n_tok // m
    out = torch.empty((2, n_ent, C), dtype=x.dtype, device="cuda")
    v4a.v4a_compress(x, z, out, m=m)
    _sync()
    ref = oracle.compress(host(case["x"]), host(case["gate"]), m)
    g = out.double().cpu().numpy()
    if fmt == "f32":
        assert np.abs(g - ref).max() <= 2e-6 * max(1.0, np.abs(ref).max())
    else:  # bf16 output: within one bf16 rounding of the fp64 value (+ fp32 slack)
        assert (np.abs(g - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6).all()


def test_compress_fused_streams_fp8_keys_and_strided_cache(v4a):
    """K=V stream (bf16 -> bf16) and indexer stream (bf16 -> fp8 + scale) in one
    launch, writing into the middle of larger cache buffers."""
    B, m, n_tok, d, di = 3, 4, 4 * 50, 512, 128
    kv = wl.compress_case(B, n_tok, d, "bf16", seed=7)
    ik = wl.compress_case(B, n_tok, di, "bf16", seed=8, gate_std=2.0)
    cap, s0 = 80, 17
    ent = torch.zeros((B, cap, d), dtype=torch.bfloat16, device="cuda")
    keys = torch.zeros((B, cap, di), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((B, cap), dtype=torch.float32, device="cuda")
    n_ent = n_tok // m
    v4a.v4a_compress(dev(kv["x"]), dev(kv["gate"]), ent[:, s0:s0 + n_ent], m=m,
                     xi=dev(ik["x"]), gate_i=dev(ik["gate"]), out_i=keys[:, s0:s0 + n_ent],
                     out_i_scale=scales[:, s0:s0 + n_ent])
    _sync()
    ref_kv = oracle.compress(host(kv["x"]), host(kv["gate"]), m)
    g = ent[:, s0:s0 + n_ent].double().cpu().numpy()
    assert (np.abs(g - ref_kv) <= np.abs(ref_kv) * 2.0 ** -8 + 1e-6).all()
    assert (ent[:, :s0] == 0).all() and (ent[:, s0 + n_ent:] == 0).all()  # nothing outside the slice
    ref_k = oracle.compress(host(ik["x"]), host(ik["gate"]), m)
    codes = keys[:, s0:s0 + n_ent].cpu().numpy()
    sc = scales[:, s0:s0 + n_ent].double().cpu().numpy()
    _, ref_sc = oracle.quantize_e4m3_rows(ref_k)
    assert np.allclose(sc, ref_sc, rtol=1e-5)
    deq = oracle.e4m3_decode(codes) * sc[..., None]
    # each stored value is the nearest e4m3 grid point of value/scale, up to the fp32 arithmetic of the
    # compressed value (a code may sit one step away only when the value lies on a rounding midpoint)
    v = ref_k / ref_sc[..., None]
    step = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -6))) - 3), 2.0 ** -9)
    err = np.abs(deq / sc[..., None] - v)
    assert (err <= 0.5 * step * (1 + 1e-4) + 1e-5 * np.abs(v)).all()
    assert (scales[:, :s0] == 0).all() and (keys[:, s0 + n_ent:] == 0).all()


@pytest.mark.parametrize("fmt,m,n_tok,C,with_prev", [("f32", 4, 4 * 37 + 3, 128, False), ("f32", 4, 4 * 20, 64, True),
                                                   ("bf16", 4, 4 * 300 + 1, 512, True), ("bf16", 1, 33, 128, False),
                                                   ("bf16", 16, 16 * 9, 512, True), ("f32", 128, 128 * 3 + 5, 128, True)])
def test_compress_dual_matches_oracle(v4a, fmt, m, n_tok, C, with_prev):
    """Dual-series compression of a token range: series a over each block, series b over the block
    before it (the range's previous block, or prev_* for the first entry when given)."""
    B = 2
    ca = wl.compress_case(B, n_tok, C, fmt, seed=200 + m)
    cb = wl.compress_case(B, n_tok, C, fmt, seed=300 + m, gate_std=2.0)
    pr = wl.compress_case(B, m, C, fmt, seed=400 + m) if with_prev else None
    n_ent = n_tok // m
    out = torch.empty((B, n_ent, C), dtype=dev(ca["x"]).dtype, device="cuda")
    v4a.v4a_compress_dual(dev(ca["x"]), dev(ca["gate"]), dev(cb["x"]), dev(cb["gate"]), out, m=m,
                          prev_x_b=dev(pr["x"]) if pr else None, prev_gate_b=dev(pr["gate"]) if pr else None)
    _sync()
    ref = oracle.compress_dual(host(ca["x"]), host(ca["gate"]), host(cb["x"]), host(cb["gate"]), m,
                               prev_xb=host(pr["x"]) if pr else None, prev_zb=host(pr["gate"]) if pr else None)
    g = out.double().cpu().numpy()
    if fmt == "f32":
        assert np.abs(g - ref).max() <= 2e-6 * max(1.0, np.abs(ref).max())
    else:  # bf16 output: within one bf16 rounding of the fp64 value (+ fp32 slack)
        assert (np.abs(g - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6).all()


def test_compress_dual_fp8_output_into_cache_slice(v4a):
    """bf16 series -> FP8 entries + scales written into the middle of a larger cache, the block before
    the range given."""
    B, m, n_tok, C = 3, 4, 4 * 40, 128
    ca = wl.compress_case(B, n_tok + m, C, "bf16", seed=501)
    cb = wl.compress_case(B, n_tok + m, C, "bf16", seed=502, gate_std=2.0)
    cap, s0, n_ent = 60, 9, n_tok // m
    keys = torch.zeros((B, cap, C), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((B, cap), dtype=torch.float32, device="cuda")
    xa, za, xb, zb = (dev(t) for t in (ca["x"], ca["gate"], cb["x"], cb["gate"]))
    v4a.v4a_compress_dual(xa[:, m:], za[:, m:], xb[:, m:], zb[:, m:], keys[:, s0:s0 + n_ent], m=m,
                          prev_x_b=xb[:, :m], prev_gate_b=zb[:, :m], out_scale=scales[:, s0:s0 + n_ent])
    _sync()
    full = oracle.compress_dual(host(ca["x"]), host(ca["gate"]), host(cb["x"]), host(cb["gate"]), m)
    ref = full[:, 1:]
    _, ref_sc = oracle.quantize_e4m3_rows(ref)
    sc = scales[:, s0:s0 + n_ent].double().cpu().numpy()
    assert np.allclose(sc, ref_sc, rtol=1e-5)
    deq = oracle.e4m3_decode(keys[:, s0:s0 + n_ent].cpu().numpy()) * sc[..., None]
    # each code is the nearest e4m3 grid point of value/scale (half a grid step), up to the fp32 arithmetic
    # of the compressed value, as for the single-series FP8 output
    v = ref / ref_sc[..., None]
    step = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -6))) - 3), 2.0 ** -9)
    err = np.abs(deq / sc[..., None] - v)
    assert (err <= 0.5 * step * (1 + 1e-4) + 1e-5 * np.abs(v)).all()
    assert (keys[:, :s0] == 0).all() and (keys[:, s0 + n_ent:] == 0).all()


def test_compress_empty_and_short(v4a):
    x = torch.randn((2, 3, 64), device="cuda")
    out = torch.full((2, 1, 64), 7.0, device="cuda")
    v4a.v4a_compress(x, x, out, m=4)  # no complete chunk: nothing written
    _sync()
    assert (out == 7.0).all()
    v4a.v4a_compress(x[:0], x[:0], out[:0], m=1)  # empty batch


# ----------------------------------------------------------------------
# indexer scores and top-k
# ----------------------------------------------------------------------

@pytest.mark.parametrize("qf,kf,HI,DI,T,L,m", [("f32", "f32", 4, 64, 1, 4096, 4), ("bf16", "bf16", 16, 128, 3, 2050, 4),
                                              ("bf16", "e4m3", 16, 128, 5, 4099, 4), ("f32", "bf16", 1, 32, 2, 300, 8),
                                              ("bf16", "e4m3", 32, 128, 2, 4096 + 12, 4),
                                              ("bf16", "e4m3", 5, 128, 1, 1000, 4),
                                              ("bf16", "bf16", 24, 128, 2, 3000, 4)])
def test_index_scores_match_oracle(v4a, qf, kf, HI, DI, T, L, m):
    c = wl.index_case(2, T, L, m, HI, DI, qf, kf, seed=11 + HI)
    N = L // m
    scores = torch.empty((2, T, N), dtype=torch.float32, device="cuda")
    v4a.v4a_index_scores(dev(c["q_i"]), dev(c["w"]), dev(c["k_i"]), dev(c["k_scale"]), scores, m=m, ctx_len=L)
    _sync()
    ref = oracle.index_scores(host(c["q_i"]), host(c["w"]), host(c["k_i"]),
                              None if c["k_scale"] is None else host(c["k_scale"]), L, m)
    check_scores(scores, ref, f"{qf}/{kf}")


def test_index_scores_fp8_keys_tiny_query_elements(v4a):
    """Query elements far below their head's largest one (down to 1e-9 of it)
    must still count: the FP8-key path splits q into e4m3 pieces per magnitude
    class, and its scores must stay within f32 rounding of the oracle."""
    c = wl.index_case(2, 2, 4096, 4, 16, 128, "bf16", "e4m3", seed=91)
    q = c["q_i"].float()
    g = torch.Generator().manual_seed(92)
    factors = torch.tensor([1.0, 1e-3, 1e-5, 1e-7, 1e-9])[torch.randint(0, 5, q.shape, generator=g)]
    c["q_i"] = (q * factors).to(torch.bfloat16)
    N = 4096 // 4
    scores = torch.empty((2, 2, N), dtype=torch.float32, device="cuda")
    v4a.v4a_index_scores(dev(c["q_i"]), dev(c["w"]), dev(c["k_i"]), dev(c["k_scale"]), scores, m=4, ctx_len=4096)
    _sync()
    ref = oracle.index_scores(host(c["q_i"]), host(c["w"]), host(c["k_i"]), host(c["k_scale"]), 4096, 4)
    check_scores(scores, ref, "bf16/e4m3 tiny q elements")


@pytest.mark.parametrize("qf,kf,HI,DI,T,L,m,k", [("f32", "f32", 4, 64, 1, 4096, 4, 64),
                                                ("bf16", "bf16", 16, 128, 2, 8192 + 7, 4, 512),
                                                ("bf16", "e4m3", 16, 128, 3, 16384 + 2, 4, 1024),
                                                ("bf16", "e4m3", 32, 128, 2, 8192 + 300, 4, 256),
                                                ("bf16", "bf16", 8, 64, 4, 40, 4, 16),   # N_vis < k: padding
                                                ("f32", "f32", 2, 32, 1, 257, 4, 1)])
def test_topk_matches_oracle(v4a, qf, kf, HI, DI, T, L, m, k):
    c = wl.index_case(2, T, L, m, HI, DI, qf, kf, seed=21 + k)
    idx = torch.empty((2, T, k), dtype=torch.int32, device="cuda")
    sco = torch.empty((2, T, k), dtype=torch.float32, device="cuda")
    v4a.v4a_topk(dev(c["q_i"]), dev(c["w"]), dev(c["k_i"]), dev(c["k_scale"]), idx, sco, m=m, k=k, ctx_len=L)
    _sync()
    ref = oracle.topk(host(c["q_i"]), host(c["w"]), host(c["k_i"]),
                      None if c["k_scale"] is None else host(c["k_scale"]), L, m, k, want_scores=True)
    check_topk(idx, ref, L, m, k, gpu_scores=sco)


def test_topk_exact_ties_take_lower_index(v4a):
    """Keys repeated many times give exactly equal scores; the select must take
    the lowest entries among equals (and agree with the oracle bit for bit)."""
    L, m, k, HI, DI = 4 * 3000, 4, 300, 4, 64
    c = wl.index_case(1, 2, L, m, HI, DI, "f32", "f32", seed=5)
    base = c["k_i"][:, :7].clone()
    c["k_i"] = base.repeat(1, (L // m) // 7 + 1, 1)[:, :L // m].contiguous()  # 7 distinct keys, repeated
    idx = torch.empty((1, 2, k), dtype=torch.int32, device="cuda")
    v4a.v4a_topk(dev(c["q_i"]), dev(c["w"]), dev(c["k_i"]), None, idx, m=m, k=k, ctx_len=L)
    _sync()
    ref = oracle.topk(host(c["q_i"]), host(c["w"]), host(c["k_i"]), None, L, m, k, want_scores=True)
    assert np.array_equal(idx.cpu().numpy(), ref["idx"])


def test_topk_zero_entries(v4a):
    """Context shorter than one chunk: nothing to select, all padding."""
    c = wl.index_case(2, 2, 3, 4, 4, 64, "bf16", "bf16", seed=3, n_ent=0)
    idx = torch.zeros((2, 2, 8), dtype=torch.int32, device="cuda")
    v4a.v4a_topk(dev(c["q_i"]), dev(c["w"]), torch.empty((2, 0, 64), dtype=torch.bfloat16, device="cuda"), None,
                 idx, m=4, k=8, ctx_len=3)
    _sync()
    assert (idx == -1).all()


# ----------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------

def _attend_inputs(B, T, L, m, H, d, W, fmt, seed, k=None, pad=0.0, dup=False):
    a = wl.attend_case(B, T, L, m, H, d, W, fmt, seed, q_std=1.0 / math.sqrt(d) if fmt == "f32" else 1.0)
    if k is not None:
        idx = wl.random_topk_idx(B, T, L, m, k, seed + 1, pad_fraction=pad)
        if dup:  # repeat a selected entry: it must count twice
            idx[:, :, 1] = idx[:, :, 0]
        a["idx"] = idx
    return a


@pytest.mark.parametrize("fmt,B,T,L,m,H,d,W,k", [
    ("f32", 1, 1, 4096, 4, 16, 128, 128, 64),
    ("f32", 2, 3, 1000, 4, 8, 64, 128, 37),
    ("bf16", 2, 1, 65536 // 8, 4, 64, 512, 128, 512),
    ("bf16", 3, 2, 5000, 4, 64, 512, 128, 300),
    ("bf16", 1, 4, 100, 4, 16, 256, 128, 64),      # short context: window clipped at 0, k > N_vis
    ("bf16", 2, 1, 2048, 4, 32, 512, 0, 128),      # no window
    ("bf16", 2, 1, 4 * 3000, 4, 64, 512, 128, 2500),  # k > 2048: the 48-row-tile kernel
])
def test_csa_attend_matches_oracle(v4a, fmt, B, T, L, m, H, d, W, k):
    a = _attend_inputs(B, T, L, m, H, d, W, fmt, seed=L + k, k=k, pad=0.1)
    out = torch.empty((B, T, H, d), dtype=torch.float32, device="cuda")
    st = torch.full((1,), 9, dtype=torch.int32, device="cuda")
    v4a.v4a_csa_attend(dev(a["q"]), dev(a["entries"]), dev(a["idx"]), dev(a["token_kv"]), a["tok_pos0"], out,
                       m=m, window=W, ctx_len=L, dev_status=st)
    _sync()
    assert int(st.item()) == 0
    ref = oracle.attend(host(a["q"]), host(a["entries"]), host(a["idx"]), host(a["token_kv"]), a["tok_pos0"], L, m, W)
    check_attention(out, ref, fmt == "f32", f"csa {fmt} L={L}")


def test_csa_attend_duplicates_and_bad_indices(v4a):
    B, T, L, m, H, d, W, k = 2, 2, 3000, 4, 16, 128, 128, 40
    a = _attend_inputs(B, T, L, m, H, d, W, "f32", seed=77, k=k, dup=True)
    out = torch.empty((B, T, H, d), dtype=torch.float32, device="cuda")
    st = torch.zeros((1,), dtype=torch.int32, device="cuda")
    v4a.v4a_csa_attend(dev(a["q"]), dev(a["entries"]), dev(a["idx"]), dev(a["token_kv"]), a["tok_pos0"], out,
                       m=m, window=W, ctx_len=L, dev_status=st)
    _sync()
    assert int(st.item()) == 0
    ref = oracle.attend(host(a["q"]), host(a["entries"]), host(a["idx"]), host(a["token_kv"]), a["tok_pos0"], L, m, W)
    check_attention(out, ref, True, "duplicates")
    # out-of-range slots (not visible / negative) are skipped and reported
    bad = a["idx"].clone()
    bad[0, 0, 3] = (L - T) // m + 5
    bad[1, 1, 5] = -7
    v4a.v4a_csa_attend(dev(a["q"]), dev(a["entries"]), dev(bad), dev(a["token_kv"]), a["tok_pos0"], out,
                       m=m, window=W, ctx_len=L, dev_status=st)
    _sync()
    assert int(st.item()) == 4
    ref = oracle.attend(host(a["q"]), host(a["entries"]), host(bad), host(a["token_kv"]), a["tok_pos0"], L, m, W,
                        allow_bad_index=True)
    check_attention(out, ref, True, "bad indices skipped")


@pytest.mark.parametrize("fmt,B,T,L,H,d,W", [
    ("f32", 1, 1, 4096, 16, 128, 128),
    ("bf16", 2, 1, 128 * 300, 64, 512, 128),
    ("bf16", 3, 3, 128 * 77 + 64, 64, 512, 128),
    ("f32", 2, 2, 100, 8, 64, 128),      # shorter than one chunk: pure sliding window
    ("bf16", 1, 1, 127, 64, 512, 128),
    ("bf16", 2, 1, 128 * 40, 32, 256, 0),  # no window
    ("bf16", 1, 1, 128 * 2100 + 77, 64, 512, 128),  # more than 2,048 entries: the 48-row-tile kernel
])
def test_hca_attend_matches_oracle(v4a, fmt, B, T, L, H, d, W):
    m = 128
    a = _attend_inputs(B, T, L, m, H, d, W, fmt, seed=L + H)
    out = torch.empty((B, T, H, d), dtype=torch.float32, device="cuda")
    v4a.v4a_hca_attend(dev(a["q"]), dev(a["entries"]) if a["entries"].shape[1] else None, dev(a["token_kv"]),
                       a["tok_pos0"], out, m=m, window=W, ctx_len=L)
    _sync()
    ref = oracle.attend(host(a["q"]), host(a["entries"]), None, host(a["token_kv"]), a["tok_pos0"], L, m, W)
    check_attention(out, ref, fmt == "f32", f"hca {fmt} L={L}")


@pytest.mark.parametrize("kind,fmt,B,T,L,H,d,W", [
    ("hca", "bf16", 2, 1, 128 * 40 + 77, 64, 512, 128),  # tensor cores, queries split between CTAs
    ("hca", "bf16", 3, 1, 100, 64, 512, 64),             # tensor cores, one tile per query (written whole)
    ("csa", "bf16", 2, 2, 4 * 2000 + 3, 64, 512, 128),   # tensor cores, CSA
    ("hca", "f32", 2, 1, 128 * 30 + 5, 16, 128, 128),    # CUDA cores, several splits
    ("csa", "f32", 1, 3, 4 * 200, 16, 128, 128),         # CUDA cores
])
def test_attend_sink_and_output_rope_match_oracle(v4a, kind, fmt, B, T, L, H, d, W):
    """The attention sink (per-head logit in the softmax denominator) and the output RoPE at minus the
    query position on the last 64 dims ("1M Context != Lossless Long Memory", sections 7 and 8)."""
    m, k = (128, 0) if kind == "hca" else (4, 200)
    a = _attend_inputs(B, T, L, m, H, d, W, fmt, seed=L + 7 * H, k=k if k else None, pad=0.1)
    g = torch.Generator().manual_seed(L)
    sink = (2.0 * torch.randn(H, generator=g)).float()
    out = torch.empty((B, T, H, d), dtype=torch.float32, device="cuda")
    ent = dev(a["entries"]) if a["entries"].shape[1] else None
    if kind == "hca":
        v4a.v4a_hca_attend(dev(a["q"]), ent, dev(a["token_kv"]), a["tok_pos0"], out, m=m, window=W, ctx_len=L,
                           sink=sink.cuda(), rope_dims=64, rope_base=10000.0)
    else:
        v4a.v4a_csa_attend(dev(a["q"]), ent, dev(a["idx"]), dev(a["token_kv"]), a["tok_pos0"], out, m=m, window=W,
                           ctx_len=L, sink=sink.cuda(), rope_dims=64, rope_base=10000.0)
    _sync()
    ref = oracle.attend(host(a["q"]), host(a["entries"]), host(a["idx"]) if kind == "csa" else None,
                        host(a["token_kv"]), a["tok_pos0"], L, m, W, sink=sink.double().numpy(), rope_dims=64)
    check_attention(out, ref, fmt == "f32", f"{kind} {fmt} L={L} with sink and output RoPE")


def test_csa_with_every_entry_selected_equals_hca(v4a):
    B, T, L, m, H, d, W = 2, 1, 4 * 200, 4, 64, 512, 128
    a = _attend_inputs(B, T, L, m, H, d, W, "bf16", seed=9)
    N = L // m
    idx = torch.arange(N, dtype=torch.int32).repeat(B, T, 1).contiguous()
    o1 = torch.empty((B, T, H, d), dtype=torch.float32, device="cuda")
    o2 = torch.empty_like(o1)
    v4a.v4a_csa_attend(dev(a["q"]), dev(a["entries"]), dev(idx), dev(a["token_kv"]), a["tok_pos0"], o1, m=m,
                       window=W, ctx_len=L)
    v4a.v4a_hca_attend(dev(a["q"]), dev(a["entries"]), dev(a["token_kv"]), a["tok_pos0"], o2, m=m, window=W,
                       ctx_len=L)
    _sync()
    assert (o1 - o2).abs().max().item() <= 1e-3


# ----------------------------------------------------------------------
# the fp32 workload end to end: compress -> top-k -> CSA; compress -> HCA
# ----------------------------------------------------------------------

def test_fp32_workload_end_to_end(v4a):
    w = wl.fp32_l4096()
    c = w["cfg"]
    L, d, H, m, mh, k, W = c["ctx_len"], c["d"], c["heads"], c["m"], c["m_hca"], c["k"], c["window"]
    x = dev(w["x"])
    ent = torch.empty((1, L // m, d), device="cuda")
    ent_h = torch.empty((1, L // mh, d), device="cuda")
    v4a.v4a_compress(x, dev(w["z_csa"]), ent, m=m)
    v4a.v4a_compress(x, dev(w["z_hca"]), ent_h, m=mh)
    idx = torch.empty((1, 1, k), dtype=torch.int32, device="cuda")
    v4a.v4a_topk(dev(w["q_i"]), dev(w["w"]), dev(w["k_i"]), None, idx, m=m, k=k, ctx_len=L)
    out_c = torch.empty((1, 1, H, d), device="cuda")
    out_h = torch.empty((1, 1, H, d), device="cuda")
    v4a.v4a_csa_attend(dev(w["q"]), ent, idx, x, 0, out_c, m=m, window=W, ctx_len=L)
    v4a.v4a_hca_attend(dev(w["q"]), ent_h, x, 0, out_h, m=mh, window=W, ctx_len=L)
    _sync()
    xs = host(w["x"])
    r_ent = oracle.compress(xs, host(w["z_csa"]), m).astype(np.float32)
    r_enth = oracle.compress(xs, host(w["z_hca"]), mh).astype(np.float32)
    assert np.abs(ent.cpu().numpy() - r_ent).max() < 1e-5
    r_top = oracle.topk(host(w["q_i"]), host(w["w"]), host(w["k_i"]), None, L, m, k, want_scores=True)
    check_topk(idx, r_top, L, m, k)
    r_c = oracle.attend(host(w["q"]), r_ent, r_top["idx"], xs, 0, L, m, W)
    r_h = oracle.attend(host(w["q"]), r_enth, None, xs, 0, L, mh, W)
    check_attention(out_c, r_c, True, "fp32 CSA chain")
    check_attention(out_h, r_h, True, "fp32 HCA chain")


# ----------------------------------------------------------------------
# full-size workloads, sampled
# ----------------------------------------------------------------------

def _sub(t, bs):
    return t[bs].contiguous() if t is not None else None


def test_csa_l64k_full_size_sampled(v4a):
    w = wl.csa_decode("csa_l64k", with_tail=False)
    c = w["cfg"]
    B, L, m, k, H, d, W = c["batch"], c["ctx_len"], c["m"], c["k"], c["heads"], c["d"], c["window"]
    idx = torch.empty((B, 1, k), dtype=torch.int32, device="cuda")
    v4a.v4a_topk(dev(w["q_i"]), dev(w["w"]), dev(w["k_i"]), None, idx, m=m, k=k, ctx_len=L)
    out = torch.empty((B, 1, H, d), device="cuda")
    v4a.v4a_csa_attend(dev(w["q"]), dev(w["entries"]), idx, dev(w["token_kv"]), w["tok_pos0"], out, m=m, window=W,
                       ctx_len=L)
    _sync()
    bs = [0, B - 1]
    r_top = oracle.topk(host(_sub(w["q_i"], bs)), host(_sub(w["w"], bs)), host(_sub(w["k_i"], bs)), None, L, m, k,
                        want_scores=True)
    check_topk(idx[bs], r_top, L, m, k)
    r = oracle.attend(host(_sub(w["q"], bs)), host(_sub(w["entries"], bs)), r_top["idx"],
                      host(_sub(w["token_kv"], bs)), w["tok_pos0"], L, m, W)
    check_attention(out[bs], r, False, "csa_l64k")


def test_hca_l1m_full_size_sampled(v4a):
    w = wl.hca_decode("hca_l1m", with_tail=False)
    c = w["cfg"]
    B, L, m, H, d, W = c["batch"], c["ctx_len"], c["m"], c["heads"], c["d"], c["window"]
    out = torch.empty((B, 1, H, d), device="cuda")
    v4a.v4a_hca_attend(dev(w["q"]), dev(w["entries"]), dev(w["token_kv"]), w["tok_pos0"], out, m=m, window=W,
                       ctx_len=L)
    _sync()
    bs = [0, 13, B - 1]
    r = oracle.attend(host(_sub(w["q"], bs)), host(_sub(w["entries"], bs)), None, host(_sub(w["token_kv"], bs)),
                      w["tok_pos0"], L, m, W)
    check_attention(out[bs], r, False, "hca_l1m")


def test_csa_l1m_fp8_full_size_sampled(v4a):
    w = wl.csa_decode("csa_l1m_fp8", with_tail=False)
    c = w["cfg"]
    B, L, m, k, H, d, W = c["batch"], c["ctx_len"], c["m"], c["k"], c["heads"], c["d"], c["window"]
    idx = torch.empty((B, 1, k), dtype=torch.int32, device="cuda")
    v4a.v4a_topk(dev(w["q_i"]), dev(w["w"]), dev(w["k_i"]), dev(w["k_scale"]), idx, m=m, k=k, ctx_len=L)
    out = torch.empty((B, 1, H, d), device="cuda")
    v4a.v4a_csa_attend(dev(w["q"]), dev(w["entries"]), idx, dev(w["token_kv"]), w["tok_pos0"], out, m=m, window=W,
                       ctx_len=L)
    _sync()
    bs = [1, B - 1]
    r_top = oracle.topk(host(_sub(w["q_i"], bs)), host(_sub(w["w"], bs)), host(_sub(w["k_i"], bs)),
                        host(_sub(w["k_scale"], bs)), L, m, k, want_scores=True)
    rep = check_topk(idx[bs], r_top, L, m, k)
    r = oracle.attend(host(_sub(w["q"], bs)), host(_sub(w["entries"], bs)), r_top["idx"],
                      host(_sub(w["token_kv"], bs)), w["tok_pos0"], L, m, W)
    check_attention(out[bs], r, False, "csa_l1m_fp8")
    print("tie band entries:", rep["tie_band_entries"])


# ----------------------------------------------------------------------
# paths of the tensor-core kernel (bf16, d = 512, 64 heads)
# ----------------------------------------------------------------------

def test_attend_rescale_path_increasing_logits(v4a):
    """Logits that grow by more than 2^8 per 64-row tile force the running
    maximum (and the accumulated output) to be rescaled tile after tile."""
    B, T, m, H, d, W = 2, 1, 128, 64, 512, 128
    L = m * 192 + 5
    g = wl._gen(31)
    q = torch.ones((B, T, H, d), dtype=torch.bfloat16)
    N = L // m
    ramp = (torch.arange(N, dtype=torch.float32) * 0.005)[None, :, None]
    ent = (ramp + 0.05 * wl.normal(g, (B, N, d))).to(torch.bfloat16)
    p0, lt = wl.window_rows(L, T, W)
    tok = (0.05 * wl.normal(g, (B, lt, d))).to(torch.bfloat16)
    out = torch.empty((B, T, H, d), device="cuda")
    v4a.v4a_hca_attend(dev(q), dev(ent), dev(tok), p0, out, m=m, window=W, ctx_len=L)
    _sync()
    ref = oracle.attend(host(q), host(ent), None, host(tok), p0, L, m, W)
    check_attention(out, ref, False, "rescale path")


def test_csa_many_queries_split_rows(v4a):
    """Many queries (multi-query CSA): each CTA runs several queries and some
    queries are split between CTAs and merged afterwards."""
    B, T, L, m, H, d, W, k = 2, 200, 4 * 3000, 4, 64, 512, 128, 128
    a = _attend_inputs(B, T, L, m, H, d, W, "bf16", seed=55, k=k, pad=0.05)
    out = torch.empty((B, T, H, d), dtype=torch.float32, device="cuda")
    st = torch.zeros((1,), dtype=torch.int32, device="cuda")
    v4a.v4a_csa_attend(dev(a["q"]), dev(a["entries"]), dev(a["idx"]), dev(a["token_kv"]), a["tok_pos0"], out,
                       m=m, window=W, ctx_len=L, dev_status=st)
    _sync()
    assert int(st.item()) == 0
    ref = oracle.attend(host(a["q"]), host(a["entries"]), host(a["idx"]), host(a["token_kv"]), a["tok_pos0"], L, m, W)
    check_attention(out, ref, False, "csa multi-query")


def test_hca_single_long_query_split_over_many_ctas(v4a):
    """One 1M-context HCA query: its 130 tiles land on 130 CTAs and the
    combine merges 130 pieces."""
    B, T, L, m, H, d, W = 1, 1, 1 << 20, 128, 64, 512, 128
    a = _attend_inputs(B, T, L, m, H, d, W, "bf16", seed=61)
    out = torch.empty((B, T, H, d), device="cuda")
    v4a.v4a_hca_attend(dev(a["q"]), dev(a["entries"]), dev(a["token_kv"]), a["tok_pos0"], out, m=m, window=W,
                       ctx_len=L)
    _sync()
    ref = oracle.attend(host(a["q"]), host(a["entries"]), None, host(a["token_kv"]), a["tok_pos0"], L, m, W)
    check_attention(out, ref, False, "hca one long query")


def test_topk_many_rows_matches_oracle(v4a):
    """More query rows than the few-rows select serves (2 x 150 = 300 > 256) take the per-row
    histogram select; the rows see different numbers of entries and include exact ties."""
    B, T, L, m, k, HI, DI = 2, 150, 4 * 3000 + 5, 4, 200, 16, 128
    c = wl.index_case(B, T, L, m, HI, DI, "bf16", "bf16", seed=81)
    c["k_i"][:, 100:400] = c["k_i"][:, 100:101].clone()  # 300 copies of one key: equal scores in every row
    idx = torch.empty((B, T, k), dtype=torch.int32, device="cuda")
    sco = torch.empty((B, T, k), dtype=torch.float32, device="cuda")
    v4a.v4a_topk(dev(c["q_i"]), dev(c["w"]), dev(c["k_i"]), None, idx, sco, m=m, k=k, ctx_len=L)
    _sync()
    ref = oracle.topk(host(c["q_i"]), host(c["w"]), host(c["k_i"]), None, L, m, k, want_scores=True)
    check_topk(idx, ref, L, m, k, gpu_scores=sco)


def test_topk_many_rows_all_equal_takes_lowest_entries(v4a):
    """Many rows whose scores are all equal: the threshold bin holds every entry, more than the
    per-row select keeps in shared memory, and the exact radix select takes the lowest entries."""
    B, T, L, m, k, HI, DI = 1, 300, 4 * 10000, 4, 333, 16, 128
    c = wl.index_case(B, T, L, m, HI, DI, "bf16", "bf16", seed=82)
    c["k_i"] = c["k_i"][:, :1].expand(B, L // m, DI).contiguous()
    idx = torch.empty((B, T, k), dtype=torch.int32, device="cuda")
    v4a.v4a_topk(dev(c["q_i"]), dev(c["w"]), dev(c["k_i"]), None, idx, m=m, k=k, ctx_len=L)
    _sync()
    want = np.broadcast_to(np.arange(k, dtype=np.int32), (B, T, k))
    assert np.array_equal(idx.cpu().numpy(), want)


def test_topk_all_scores_equal_takes_lowest_entries(v4a):
    """Every entry scores the same: the candidate set exceeds what the fast
    select holds in shared memory and the full radix select takes over; ties
    go to the lowest entries."""
    B, L, m, k, HI, DI = 2, 4 * 40000, 4, 777, 16, 128
    c = wl.index_case(B, 1, L, m, HI, DI, "bf16", "bf16", seed=71)
    c["k_i"] = c["k_i"][:, :1].expand(B, L // m, DI).contiguous()  # one key repeated everywhere
    idx = torch.empty((B, 1, k), dtype=torch.int32, device="cuda")
    sco = torch.empty((B, 1, k), dtype=torch.float32, device="cuda")
    v4a.v4a_topk(dev(c["q_i"]), dev(c["w"]), dev(c["k_i"]), None, idx, sco, m=m, k=k, ctx_len=L)
    _sync()
    want = np.broadcast_to(np.arange(k, dtype=np.int32), (B, 1, k))
    assert np.array_equal(idx.cpu().numpy(), want)
    s = sco.cpu().numpy()
    assert (s == s[:, :, :1]).all()
