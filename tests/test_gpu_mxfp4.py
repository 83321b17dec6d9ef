"""GPU parity of the FP4 indexer path (MXFP4 keys and queries) against the oracle.

The keys are MXFP4 (OCP MX: e2m1 codes, 32-element blocks with an E8M0
exponent).  The quantiser must agree with the oracle's bit for bit; the
compress kernel's MXFP4 output may differ from the oracle's only where the
fp32 value it quantises sits on a rounding boundary within fp32 slack; scores
and top-k sets follow the same bars as the other key formats.
"""
import numpy as np
import pytest
import torch

import oracle
import workload as wl
from parity_utils import check_scores, check_topk, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def v4a():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import compressed_sparse_long_v4a_b200 as v
    return v


def _sync():
    torch.cuda.synchronize()


def _gpu_quantize(v4a, x):
    codes = torch.empty(x.shape[:-1] + (x.shape[-1] // 2,), dtype=torch.uint8, device="cuda")
    exps = torch.empty(x.shape[:-1] + (x.shape[-1] // 32,), dtype=torch.uint8, device="cuda")
    v4a.v4a_quantize_mxfp4(dev(x), codes, exps)
    _sync()
    return codes, exps


def _boundary_values(rng, rows):
    """Blocks whose values sit exactly on e2m1 rounding ties and grid points at their block scale,
    plus saturating, all-zero, subnormal-range and huge blocks."""
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    ties = (grid[:-1] + grid[1:]) / 2
    out = np.zeros((rows, 128), dtype=np.float32)
    for r in range(rows):
        X = int(rng.integers(-20, 20))
        vals = rng.choice(np.concatenate([grid, ties, [6.5, 7.9]]), size=128) * rng.choice([-1.0, 1.0], size=128)
        vals[::32] = 4.0  # fixes the block exponent at X: amax in [4, 8) * 2^X
        out[r] = np.ldexp(vals, X)
    out[0, 32:64] = 0.0
    out[1, :32] = np.float32(1e-41) * rng.integers(-5, 6, size=32)  # subnormal block
    out[2, 64:96] = rng.normal(size=32).astype(np.float32) * np.float32(1e37)
    return out


@pytest.mark.parametrize("fmt,rows,cols", [("f32", 37, 96), ("bf16", 1000, 128), ("f32", 5000, 128),
                                           ("boundary", 64, 128)])
def test_quantize_mxfp4_matches_oracle(v4a, fmt, rows, cols):
    rng = np.random.default_rng(300 + rows)
    if fmt == "boundary":
        x = torch.from_numpy(_boundary_values(rng, rows))
    else:
        x32 = torch.from_numpy((rng.normal(size=(rows, cols)) * np.exp2(rng.integers(-8, 8, size=(rows, 1))))
                               .astype(np.float32))
        x = x32 if fmt == "f32" else x32.to(torch.bfloat16)
    codes, exps = _gpu_quantize(v4a, x)
    rc, rx = oracle.quantize_mxfp4(oracle.decode(host(x)))
    assert np.array_equal(exps.cpu().numpy(), rx)
    assert np.array_equal(codes.cpu().numpy(), rc)


def test_compress_writes_mxfp4_indexer_keys(v4a):
    """K=V stream (bf16) and indexer stream (bf16 -> MXFP4) in one launch, into a strided cache."""
    B, m, n_tok, d, di = 3, 4, 4 * 70 + 2, 512, 128
    ck = wl.compress_case(B, n_tok, d, "bf16", seed=310)
    ci = wl.compress_case(B, n_tok, di, "bf16", seed=311)
    n_ent = n_tok // m
    cap = n_ent + 9
    ent = torch.empty((B, cap, d), dtype=torch.bfloat16, device="cuda")
    kc = torch.full((B, cap, di // 2), 0xAB, dtype=torch.uint8, device="cuda")
    ke = torch.full((B, cap, di // 32), 0xCD, dtype=torch.uint8, device="cuda")
    v4a.v4a_compress(dev(ck["x"]), dev(ck["gate"]), ent[:, 3:3 + n_ent], m=m, xi=dev(ci["x"]),
                     gate_i=dev(ci["gate"]), out_i=kc[:, 3:3 + n_ent], out_i_exp=ke[:, 3:3 + n_ent])
    _sync()
    # untouched cache rows
    assert (kc[:, :3] == 0xAB).all() and (kc[:, 3 + n_ent:] == 0xAB).all()
    assert (ke[:, :3] == 0xCD).all() and (ke[:, 3 + n_ent:] == 0xCD).all()
    ref = oracle.compress(host(ci["x"]), host(ci["gate"]), m)  # fp64 values
    rc, rx = oracle.quantize_mxfp4(ref)
    gc = kc[:, 3:3 + n_ent].cpu().numpy()
    gx = ke[:, 3:3 + n_ent].cpu().numpy()
    # the GPU quantises its fp32 result: a decision may differ only on a boundary within fp32 slack
    slack = 1e-5
    blocks = np.abs(ref).reshape(B, n_ent, di // 32, 32).max(axis=-1)
    diff_x = gx != rx
    if diff_x.any():
        lg = np.log2(blocks[diff_x])
        assert np.all(np.abs(lg - np.round(lg)) < slack), "block exponent differs away from a power of two"
    X = (rx.astype(np.int64) - 127).repeat(32, axis=-1)
    scaled = np.abs(np.ldexp(ref, -X))
    nib_g = np.stack([gc & 0xF, gc >> 4], axis=-1).reshape(ref.shape)
    nib_r = np.stack([rc & 0xF, rc >> 4], axis=-1).reshape(ref.shape)
    same_block = ~diff_x.repeat(32, axis=-1)
    bad = (nib_g != nib_r) & same_block
    if bad.any():
        ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
        dist = np.abs(scaled[bad][:, None] - ties[None, :]).min(axis=1)
        zero_sign = ((nib_g[bad] ^ nib_r[bad]) == 0x8) & ((nib_r[bad] & 0x7) == 0)
        assert np.all((dist < slack * 8) | zero_sign), "an element code differs away from a rounding tie"
    assert bad.mean() < 1e-3 and diff_x.mean() < 1e-2
    # and the K=V stream is still the plain bf16 compression
    ref_e = oracle.compress(host(ck["x"]), host(ck["gate"]), m)
    g = ent[:, 3:3 + n_ent].double().cpu().numpy()
    assert (np.abs(g - ref_e) <= np.abs(ref_e) * 2.0 ** -8 + 1e-6).all()


def _fp4_keys(c):
    """Oracle-quantised MXFP4 keys of the case's key masters (host arrays and device tensors)."""
    kc, kx = oracle.quantize_mxfp4(oracle.decode(host(c["k_i"])))
    return kc, kx, torch.from_numpy(kc).cuda(), torch.from_numpy(kx).cuda()


# tensor-core path: bf16 q, d_I = 128, <= 32 heads; CUDA-core path otherwise
@pytest.mark.parametrize("qf,HI,DI,T,L,m", [("bf16", 16, 128, 1, 4096 * 4 + 44, 4), ("bf16", 16, 128, 3, 2050, 4),
                                           ("bf16", 32, 128, 2, 4096 + 12, 4), ("bf16", 5, 128, 1, 1000, 4),
                                           ("f32", 4, 64, 1, 4096, 4), ("bf16", 48, 128, 2, 3000, 4),
                                           ("f32", 16, 128, 1, 2000, 8)])
def test_index_scores_mxfp4_match_oracle(v4a, qf, HI, DI, T, L, m):
    c = wl.index_case(2, T, L, m, HI, DI, qf, "bf16", seed=320 + HI + T)
    kc, kx, dkc, dkx = _fp4_keys(c)
    N = L // m
    scores = torch.empty((2, T, N), dtype=torch.float32, device="cuda")
    v4a.v4a_index_scores_mxfp4(dev(c["q_i"]), dev(c["w"]), dkc, dkx, scores, m=m, ctx_len=L)
    _sync()
    ref = oracle.index_scores_mxfp4(host(c["q_i"]), host(c["w"]), kc, kx, L, m)
    check_scores(scores, ref, f"mxfp4 {qf} HI={HI}")


def test_index_scores_mxfp4_wide_block_scales(v4a):
    """Key and query blocks whose scales span many binades (2^-40 .. 2^40 across the blocks of one
    row): the per-block powers of two must be applied exactly."""
    c = wl.index_case(2, 2, 4096, 4, 16, 128, "bf16", "bf16", seed=330)
    g = torch.Generator().manual_seed(331)
    kf = c["k_i"].float() * torch.exp2(torch.randint(-40, 40, (2, 1024, 4, 1), generator=g).float()).repeat_interleave(
        32, dim=-1).view(2, 1024, 128)
    qf = c["q_i"].float() * torch.exp2(torch.randint(-20, 20, (2, 2, 16, 4, 1), generator=g).float()).repeat_interleave(
        32, dim=-1).view(2, 2, 16, 128)
    c["k_i"] = kf.to(torch.bfloat16)
    c["q_i"] = qf.to(torch.bfloat16)
    kc, kx, dkc, dkx = _fp4_keys(c)
    scores = torch.empty((2, 2, 1024), dtype=torch.float32, device="cuda")
    v4a.v4a_index_scores_mxfp4(dev(c["q_i"]), dev(c["w"]), dkc, dkx, scores, m=4, ctx_len=4096)
    _sync()
    ref = oracle.index_scores_mxfp4(host(c["q_i"]), host(c["w"]), kc, kx, 4096, 4)
    check_scores(scores, ref, "mxfp4 wide block scales")


@pytest.mark.parametrize("qf,HI,DI,T,L,m,k", [("bf16", 16, 128, 1, 16384 * 4 + 8, 4, 1024),
                                             ("bf16", 16, 128, 3, 8192 + 7, 4, 512),
                                             ("bf16", 32, 128, 2, 8192 + 300, 4, 256),
                                             ("bf16", 16, 128, 4, 40, 4, 16),   # N_vis < k: padding
                                             ("f32", 4, 64, 1, 4096, 4, 64),
                                             ("bf16", 16, 128, 300, 4096, 4, 64)])  # many rows: one block per row
def test_topk_mxfp4_matches_oracle(v4a, qf, HI, DI, T, L, m, k):
    c = wl.index_case(2, T, L, m, HI, DI, qf, "bf16", seed=340 + k + T)
    kc, kx, dkc, dkx = _fp4_keys(c)
    idx = torch.empty((2, T, k), dtype=torch.int32, device="cuda")
    sco = torch.empty((2, T, k), dtype=torch.float32, device="cuda")
    v4a.v4a_topk_mxfp4(dev(c["q_i"]), dev(c["w"]), dkc, dkx, idx, sco, m=m, k=k, ctx_len=L)
    _sync()
    ref = oracle.topk_mxfp4(host(c["q_i"]), host(c["w"]), kc, kx, L, m, k, want_scores=True)
    check_topk(idx, ref, L, m, k, gpu_scores=sco)


def test_csa_l1m_mxfp4_keys_full_size_sampled(v4a):
    """The 1M-context CSA decode (4 sequences, 262,144 entries, top-1024) with its indexer keys in
    MXFP4: the GPU quantises the N(0,1) keys of all 4 sequences, the oracle those of two sampled
    ones (bit-identical), then top-k of the sampled rows against the oracle."""
    w = wl.csa_decode("csa_l1m_fp8", with_tail=False, key_fmt="bf16")
    c = w["cfg"]
    B, L, m, k = c["batch"], c["ctx_len"], c["m"], c["k"]
    dkc, dkx = _gpu_quantize(v4a, w["k_i"])
    idx = torch.empty((B, 1, k), dtype=torch.int32, device="cuda")
    v4a.v4a_topk_mxfp4(dev(w["q_i"]), dev(w["w"]), dkc, dkx, idx, m=m, k=k, ctx_len=L)
    _sync()
    bs = [1, B - 1]
    kc, kx = oracle.quantize_mxfp4(oracle.decode(host(w["k_i"][bs])))
    assert np.array_equal(dkc[bs].cpu().numpy(), kc) and np.array_equal(dkx[bs].cpu().numpy(), kx)
    ref = oracle.topk_mxfp4(host(w["q_i"][bs]), host(w["w"][bs]), kc, kx, L, m, k, want_scores=True)
    rep = check_topk(idx[bs], ref, L, m, k)
    print("tie band entries:", rep["tie_band_entries"])
