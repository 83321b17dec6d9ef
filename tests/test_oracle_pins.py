"""Pins of the CPU oracle to what the pages and the mathematics fix.

None of these tests re-types the oracle's formulas: each checks a printed
worked example, a closed form, an invariant, a special case that reduces to a
library routine (torch / numpy), or brute force over tiny inputs, chosen so a
dropped term, a wrong sign or index or a transposed operand fails one of them.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden
from workload import stored_numpy

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ----------------------------------------------------------------------
# storage formats
# ----------------------------------------------------------------------

def test_e4m3_decode_all_codes_match_library():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2  # S.1111.111 for both signs
    assert np.array_equal(ours[~nan], lib[~nan])
    assert ours[~nan].max() == 448.0 and ours[~nan].min() == -448.0
    assert oracle.e4m3_decode([0x01])[0] == 2.0 ** -9  # smallest subnormal


def test_e4m3_encode_roundtrip_and_rounding():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    assert np.array_equal(oracle.e4m3_encode(oracle.e4m3_decode(codes)), codes)
    rng = np.random.default_rng(0)
    vals = np.concatenate([rng.normal(0, 50, 3000), rng.normal(0, 0.01, 1000)]).astype(np.float32)
    # midpoints between neighbouring codes exercise ties-to-even
    pos = np.sort(oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8)))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    vals = np.concatenate([vals, mids, -mids]).astype(np.float32)
    vals = vals[np.abs(vals) <= 448]
    lib = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = oracle.e4m3_encode(vals.astype(np.float64))
    assert np.array_equal(ours, lib)
    assert oracle.e4m3_encode([1e6])[0] == 0x7E and oracle.e4m3_encode([-1e6])[0] == 0xFE


def test_bf16_decode_all_codes_match_library():
    codes = np.arange(65536, dtype=np.uint16)
    ours = oracle.decode(codes)
    lib = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], lib[~nan])


def test_bf16_encode_matches_library_rne():
    rng = np.random.default_rng(1)
    vals = np.concatenate([rng.normal(0, 1, 4000), rng.normal(0, 1e-30, 200), rng.normal(0, 1e30, 200)])
    vals = vals.astype(np.float32)  # exactly representable: no double rounding on the library side
    lib = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.bf16_encode(vals.astype(np.float64)), lib)


# ----------------------------------------------------------------------
# compressor
# ----------------------------------------------------------------------

def test_compress_worked_example(golden_dir):
    g = read_golden(os.path.join(golden_dir, "compress_worked_example.txt"))
    C = np.array([g[f"C{i}"] for i in range(4)], dtype=np.float32)
    S = np.array([g[f"S{i}"] for i in range(4)], dtype=np.float64)
    assert np.allclose(S.sum(axis=0), 1.0)
    Z = np.log(S).astype(np.float32)
    out = oracle.compress(C[None], Z[None], m=4)
    assert out.shape == (1, 1, 3)
    assert np.allclose(out[0, 0], g["EXPECTED"], atol=1e-6)


def test_compress_m1_is_identity():
    rng = np.random.default_rng(2)
    x = rng.normal(size=(2, 37, 24)).astype(np.float32)
    z = rng.normal(size=(2, 37, 24)).astype(np.float32)
    assert np.array_equal(oracle.compress(x, z, m=1), x.astype(np.float64))


def test_compress_equal_logits_give_chunk_mean():
    rng = np.random.default_rng(3)
    x = rng.normal(size=(1, 4 * 9, 16)).astype(np.float32)
    z = np.full_like(x, 0.37)
    out = oracle.compress(x, z, m=4)
    mean = x.astype(np.float64).reshape(1, 9, 4, 16).mean(axis=2)
    assert np.allclose(out, mean, atol=1e-12)
    # the tail (tokens of an incomplete chunk) is not compressed
    out2 = oracle.compress(x[:, :35], z[:, :35], m=4)
    assert out2.shape == (1, 8, 16) and np.allclose(out2, mean[:, :8], atol=1e-12)


def test_compress_dominant_gate_selects_that_token_per_channel():
    """A gate logit far above the others in one channel makes the entry equal
    to that token's value in that channel: pins the token/chunk/channel
    indexing and that the softmax runs over tokens, not channels."""
    rng = np.random.default_rng(4)
    B, n_ent, m, C = 2, 6, 8, 5
    x = rng.normal(size=(B, n_ent * m, C)).astype(np.float32)
    z = rng.normal(size=(B, n_ent * m, C)).astype(np.float32)
    pick = rng.integers(0, m, size=(B, n_ent, C))
    for b, s, c in itertools.product(range(B), range(n_ent), range(C)):
        z[b, s * m + pick[b, s, c], c] = 200.0
    out = oracle.compress(x, z, m=m)
    for b, s, c in itertools.product(range(B), range(n_ent), range(C)):
        assert out[b, s, c] == pytest.approx(float(x[b, s * m + pick[b, s, c], c]), abs=1e-12)


def test_compress_shift_invariance_and_bf16_input():
    rng = np.random.default_rng(5)
    x = rng.normal(size=(1, 128, 8)).astype(np.float32)
    z = rng.normal(size=(1, 128, 8)).astype(np.float32)
    a = oracle.compress(x, z, m=128)
    b = oracle.compress(x, (z + 3.0).astype(np.float32), m=128)
    assert np.allclose(a, b, atol=1e-6)
    # two-token closed form: weight of token 0 is sigmoid(z0 - z1)
    x2 = np.array([[[2.0], [-1.0]]], dtype=np.float32)
    z2 = np.array([[[0.25], [-0.5]]], dtype=np.float32)
    s = 1.0 / (1.0 + math.exp(-(0.25 + 0.5)))
    assert oracle.compress(x2, z2, m=2)[0, 0, 0] == pytest.approx(s * 2.0 + (1 - s) * -1.0, abs=1e-12)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    zb = torch.from_numpy(z).to(torch.bfloat16)
    ob = oracle.compress(stored_numpy(xb), stored_numpy(zb), m=128)
    of = oracle.compress(xb.float().numpy(), zb.float().numpy(), m=128)
    assert np.allclose(ob, of, atol=1e-12)


# ----------------------------------------------------------------------
# dual-series compressor ("DeepSeek-V4: Million-Token Context via Hybrid Compressed Attention",
# CSA, "Dual-series KV compression"): entry i mixes series a over block i and series b over
# block i-1 under one softmax of their 2m gate logits
# ----------------------------------------------------------------------

def test_compress_dual_without_series_b_is_single_series():
    """Gate logits of series b at -inf take it out of every softmax: the single-series result of a."""
    rng = np.random.default_rng(31)
    xa, za, xb = (rng.normal(size=(2, 40, 16)).astype(np.float32) for _ in range(3))
    zb = np.full_like(za, -np.inf)
    got = oracle.compress_dual(xa, za, xb, zb, 4)
    assert np.allclose(got, oracle.compress(xa, za, 4), rtol=1e-13, atol=1e-13)


def test_compress_dual_same_series_is_a_sliding_2m_window():
    """With both series equal, entry i (i >= 1) is the single-series entry over the 2m tokens
    [m(i-1), m(i+1)); entry 0 of a sequence has only its own block."""
    rng = np.random.default_rng(32)
    m = 4
    x = rng.normal(size=(3, 44, 8)).astype(np.float32)
    z = (2.0 * rng.normal(size=(3, 44, 8))).astype(np.float32)
    got = oracle.compress_dual(x, z, x, z, m)
    for i in range(1, 44 // m):
        win = slice(m * (i - 1), m * (i + 1))
        ref = oracle.compress(x[:, win], z[:, win], 2 * m)[:, 0]
        assert np.allclose(got[:, i], ref, rtol=1e-13, atol=1e-13), i
    assert np.allclose(got[:, 0], oracle.compress(x[:, :m], z[:, :m], m)[:, 0], rtol=1e-13, atol=1e-13)


def test_compress_dual_previous_block_continues_the_sequence():
    """Compressing a range with the previous block's series b given equals compressing the longer
    range that includes that block, minus its first entry."""
    rng = np.random.default_rng(33)
    m = 4
    xa, za, xb, zb = (rng.normal(size=(2, 48, 12)).astype(np.float32) for _ in range(4))
    full = oracle.compress_dual(xa, za, xb, zb, m)
    part = oracle.compress_dual(xa[:, m:], za[:, m:], xb[:, m:], zb[:, m:], m, prev_xb=xb[:, :m], prev_zb=zb[:, :m])
    assert np.allclose(part, full[:, 1:], rtol=1e-13, atol=1e-13)


def test_compress_dual_weights_sum_to_one_and_bf16_input():
    """Constant content gives that constant whatever the logits; bf16 codes decode before use."""
    rng = np.random.default_rng(34)
    za, zb = (rng.normal(size=(1, 32, 8)) * 5 for _ in range(2))
    ones = np.ones((1, 32, 8), dtype=np.float32)
    got = oracle.compress_dual(ones, za.astype(np.float32), ones, zb.astype(np.float32), 4)
    assert np.allclose(got, 1.0, rtol=0, atol=1e-14)
    xa = rng.normal(size=(1, 32, 8))
    codes = [oracle.bf16_encode(v) for v in (xa, za, xa, zb)]
    values = [oracle.bf16_decode(c).astype(np.float32) for c in codes]
    assert np.array_equal(oracle.compress_dual(*codes, 4), oracle.compress_dual(*values, 4))


def test_quantize_rows_bounds():
    rng = np.random.default_rng(6)
    v = rng.normal(size=(50, 128))
    v[3] = 0.0
    codes, scales = oracle.quantize_e4m3_rows(v)
    assert scales[3] == 1.0 and np.all(codes[3] == 0)
    deq = oracle.e4m3_decode(codes) * scales[:, None]
    amax = np.abs(v).max(axis=1)
    assert np.allclose(np.abs(deq).max(axis=1), amax, rtol=1e-12)  # the row max maps to exactly 448
    # nearest-code error: at most half a step of the e4m3 grid (relative 2^-4 for normals)
    rel = np.abs(deq - v) / np.maximum(np.abs(v), 2.0 ** -6 * scales[:, None])
    assert rel.max() <= 2.0 ** -4 + 1e-12


# ----------------------------------------------------------------------
# MXFP4 (OCP MX: e2m1 elements, blocks of 32 sharing an E8M0 power of two)
# ----------------------------------------------------------------------

def _lib_e2m1_codes(vals):
    import ml_dtypes
    return np.asarray(vals, dtype=np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF


def test_e2m1_decode_all_codes_match_library():
    import ml_dtypes
    codes = np.arange(16, dtype=np.uint8)
    lib = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    ours = oracle.e2m1_decode(codes)
    assert np.array_equal(ours, lib) and np.array_equal(np.signbit(ours), np.signbit(lib))
    assert sorted(set(np.abs(ours))) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_encode_matches_library_rne_and_saturates():
    grid = oracle.e2m1_decode(np.arange(8, dtype=np.uint8))
    mids = (grid[:-1] + grid[1:]) / 2  # ties: 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5
    rng = np.random.default_rng(40)
    vals = np.concatenate([grid, mids, mids * (1 + 2.0 ** -20), mids * (1 - 2.0 ** -20),
                           rng.uniform(-7, 7, 4000), [6.5, 7.99, 8.0, 100.0, 1e30, 1e-9, 0.0]])
    vals = np.concatenate([vals, -vals]).astype(np.float32)
    assert np.array_equal(oracle.e2m1_encode(vals.astype(np.float64)), _lib_e2m1_codes(vals))
    assert oracle.e2m1_encode([-1e-9])[0] == 0x8  # the sign survives a round to zero


def test_mxfp4_block_exponent_rule():
    rng = np.random.default_rng(41)
    v = rng.normal(size=(64, 128)) * np.exp2(rng.integers(-20, 20, size=(64, 1)))
    v[5, 32:64] = 0.0                       # an all-zero block
    v[6, :32] = rng.normal(size=32) * 2.0 ** -140  # below the smallest scale
    codes, exps = oracle.quantize_mxfp4(v)
    assert codes.shape == (64, 64) and exps.shape == (64, 4)
    X = exps.astype(np.int64) - 127
    amax = np.abs(v).reshape(64, 4, 32).max(axis=2)
    normal = (amax > 0) & (X > -127)
    # the block maximum lands in [4, 8) times the block scale: 2^(X+2) <= amax < 2^(X+3)
    assert np.all(np.exp2(X[normal] + 2.0) <= amax[normal]) and np.all(amax[normal] < np.exp2(X[normal] + 3.0))
    assert exps[5, 1] == 0 and np.all(codes[5, 16:32] == 0)
    assert exps[6, 0] == 0  # clamped at X = -127


def test_mxfp4_codes_are_the_library_cast_at_the_block_scale():
    rng = np.random.default_rng(42)
    v = rng.normal(size=(40, 64)) * np.exp2(rng.integers(-6, 6, size=(40, 1)))
    codes, exps = oracle.quantize_mxfp4(v)
    X = (exps.astype(np.int64) - 127).repeat(32, axis=1)
    scaled = np.ldexp(v, -X)                 # exact: a power of two
    nib = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(v.shape)
    assert np.array_equal(nib, _lib_e2m1_codes(scaled.astype(np.float32)))
    deq = oracle.decode_mxfp4(codes, exps)
    # nearest-code error: at most half the widest step (2 between 4 and 6), i.e. 2^X, below
    # saturation; above 6 * 2^X the value clamps to 6 * 2^X
    sat = np.abs(v) > 6 * np.exp2(X)
    assert np.all(np.abs(deq - v)[~sat] <= np.exp2(X)[~sat])
    assert np.array_equal(np.abs(deq[sat]), 6 * np.exp2(X[sat]))


def test_mxfp4_roundtrip_on_the_grid():
    rng = np.random.default_rng(43)
    codes = rng.integers(0, 256, size=(16, 64), dtype=np.uint8)
    # each block needs a code of magnitude 4 or 6 so that its own exponent is reproduced
    codes[:, ::16] = (codes[:, ::16] & 0xF0) | rng.choice(np.array([0x6, 0x7, 0xE, 0xF], dtype=np.uint8), size=(16, 4))
    exps = rng.integers(100, 150, size=(16, 4), dtype=np.uint8)
    v = oracle.decode_mxfp4(codes, exps)
    c2, x2 = oracle.quantize_mxfp4(v)
    assert np.array_equal(x2, exps)
    # equal values: only a signed zero may come back with the other sign
    assert np.array_equal(oracle.decode_mxfp4(c2, x2), v)
    same = (c2 == codes) | (((c2 ^ codes) & 0x77) == 0)
    assert same.all()


def _on_grid(rng, shape):
    """Values on the MXFP4 grid: each 32-block holds e2m1 values times 2^X with a 4 or 6 in it."""
    rows = int(np.prod(shape[:-1]))
    codes = rng.integers(0, 256, size=(rows, shape[-1] // 2), dtype=np.uint8)
    codes[:, ::16] = (codes[:, ::16] & 0xF0) | 0x7
    exps = rng.integers(120, 130, size=(rows, shape[-1] // 32), dtype=np.uint8)
    return oracle.decode_mxfp4(codes, exps).reshape(shape), codes.reshape(shape[:-1] + (-1,)), \
        exps.reshape(shape[:-1] + (-1,))


def test_mxfp4_scores_on_the_grid_equal_the_f32_scores():
    """Quantising values that are already on the MXFP4 grid changes nothing, so the FP4 score of
    such operands is the (pinned) f32 score of the same values."""
    rng = np.random.default_rng(44)
    B, T, L, m, HI, DI = 2, 3, 256, 4, 4, 64
    q, _, _ = _on_grid(rng, (B, T, HI, DI))
    k, kc, kx = _on_grid(rng, (B, L // m, DI))
    w = rng.uniform(size=(B, T, HI)).astype(np.float32)
    s4 = oracle.index_scores_mxfp4(q.astype(np.float32), w, kc, kx, ctx_len=L, m=m)
    s32 = oracle.index_scores(q.astype(np.float32), w, k.astype(np.float32), None, ctx_len=L, m=m)
    assert np.array_equal(s4, s32)


def test_mxfp4_scores_scale_with_powers_of_two_and_quantise_q_per_head():
    rng = np.random.default_rng(45)
    B, T, L, m, HI, DI = 1, 2, 512, 4, 3, 64
    q = rng.normal(size=(B, T, HI, DI)).astype(np.float32)
    w = rng.uniform(size=(B, T, HI)).astype(np.float32)
    kc, kx = oracle.quantize_mxfp4(rng.normal(size=(B, L // m, DI)))
    s = oracle.index_scores_mxfp4(q, w, kc, kx, ctx_len=L, m=m)
    # keys times 2^5: every block exponent + 5, every score times 32, exactly
    assert np.array_equal(oracle.index_scores_mxfp4(q, w, kc, kx + 5, ctx_len=L, m=m), 32 * s)
    # the query quantiser commutes with powers of two
    assert np.array_equal(oracle.index_scores_mxfp4(q * np.float32(0.125), w, kc, kx, ctx_len=L, m=m), s / 8)
    # each head's query is quantised on its own: a large value in head 2 leaves heads 0 and 1 alone
    q2 = q.copy()
    q2[:, :, 2, 0] = 1e6
    w01 = w.copy()
    w01[:, :, 2] = 0
    assert np.array_equal(oracle.index_scores_mxfp4(q2, w01, kc, kx, ctx_len=L, m=m),
                          oracle.index_scores_mxfp4(q, w01, kc, kx, ctx_len=L, m=m))
    # ... while the dequantised query of that head shows the block scale of its own block only
    qd = oracle.mxfp4_query(q2)
    assert np.array_equal(qd[:, :, 2, 32:], oracle.mxfp4_query(q)[:, :, 2, 32:])


# ----------------------------------------------------------------------
# visibility and counts
# ----------------------------------------------------------------------

def test_page_counts(golden_dir):
    g = read_golden(os.path.join(golden_dir, "page_counts.txt"))
    L, m, n = g["HCA"]
    assert oracle.n_visible(int(L) - 1, int(m)) == int(n)
    L, m, n = g["CSA"]
    assert oracle.n_visible(int(L) - 1, int(m)) == int(n)
    k, n, pct = g["TOPK_FRACTION_PERCENT"]
    assert round(100.0 * k / n, 2) == pct
    w, mh = g["WINDOW_EQUALS_HCA_RATE"]
    assert w == mh
    # the workloads' own counts
    assert oracle.n_visible(4095, 4) == 1024 and oracle.n_visible(4095, 128) == 32
    assert oracle.n_visible(1048575, 4) == 262144 and oracle.n_visible(1048575, 128) == 8192
    assert oracle.n_visible(126976 - 1, 4) == 31744 and oracle.n_visible(131071, 4) == 32768


def test_visibility_coverage_invariant():
    """With n_win = m' = 128, every token 0..t lies in a visible HCA entry or
    in the window, and no visible entry reaches past t."""
    m, W = 128, 128
    for t in list(range(0, 600)) + [1048575, 1048574, 1048448, 1048447]:
        nvis = oracle.n_visible(t, m)
        covered_hi = nvis * m  # entries cover [0, covered_hi)
        assert covered_hi <= t + 1
        win_lo = max(0, t - W + 1)
        assert win_lo <= covered_hi  # no gap between entries and window
    # a block ending exactly at t is visible; one ending at t+1 is not
    assert oracle.n_visible(3, 4) == 1 and oracle.n_visible(2, 4) == 0


# ----------------------------------------------------------------------
# Lightning indexer
# ----------------------------------------------------------------------

def _idx_case(rng, B, T, L, m, HI, DI):
    q = rng.normal(size=(B, T, HI, DI)).astype(np.float32)
    w = rng.uniform(size=(B, T, HI)).astype(np.float32)
    k = rng.normal(size=(B, L // m, DI)).astype(np.float32)
    return q, w, k


def test_index_single_head_unit_weight_is_relu_dot():
    rng = np.random.default_rng(7)
    q, _, k = _idx_case(rng, 1, 1, 64, 4, 1, 32)
    w = np.ones((1, 1, 1), dtype=np.float32)
    s = oracle.index_scores(q, w, k, None, ctx_len=64, m=4)
    dots = k[0].astype(np.float64) @ q[0, 0, 0].astype(np.float64)
    assert np.allclose(s[0, 0], np.maximum(dots, 0.0), atol=1e-12)
    # ReLU closed form: score(q) + score(-q) = |q.k|
    s_neg = oracle.index_scores(-q, w, k, None, ctx_len=64, m=4)
    assert np.allclose(s[0, 0] + s_neg[0, 0], np.abs(dots), atol=1e-12)


def test_index_heads_add_and_contribute_nonnegatively():
    rng = np.random.default_rng(8)
    q, w, k = _idx_case(rng, 2, 1, 256, 4, 4, 16)
    full = oracle.index_scores(q, w, k, None, ctx_len=256, m=4)
    parts = [oracle.index_scores(q[:, :, h:h + 1], w[:, :, h:h + 1], k, None, ctx_len=256, m=4) for h in range(4)]
    assert np.allclose(full, sum(parts), atol=1e-10)
    assert all((p >= 0).all() for p in parts)  # w >= 0: a head can only add relevance
    # raising one head's query along a key that it already matches cannot lower the score
    q2 = q.copy()
    q2[0, 0, 1] += 0.5 * k[0, 5]
    s2 = oracle.index_scores(q2, w, k, None, ctx_len=256, m=4)
    assert s2[0, 0, 5] >= full[0, 0, 5]
    # w scales linearly
    s3 = oracle.index_scores(q, (2 * w).astype(np.float32), k, None, ctx_len=256, m=4)
    assert np.allclose(s3, 2 * full, atol=1e-10)


def test_index_scale_and_fp8_keys():
    rng = np.random.default_rng(9)
    q, w, k = _idx_case(rng, 1, 1, 128, 4, 3, 16)
    codes, scales = oracle.quantize_e4m3_rows(k[0].astype(np.float64))
    sc32 = scales.astype(np.float32)[None]
    s8 = oracle.index_scores(q, w, codes[None], sc32, ctx_len=128, m=4)
    s8_unit = oracle.index_scores(q, w, codes[None], np.ones_like(sc32), ctx_len=128, m=4)
    # the per-entry scale multiplies that entry's score
    assert np.allclose(s8, s8_unit * sc32.astype(np.float64)[:, None, :], rtol=1e-14, atol=0)
    # e4m3 values are exact in float32: coded keys score like their decoded values
    dec32 = oracle.e4m3_decode(codes).astype(np.float32)[None]
    assert np.array_equal(s8_unit, oracle.index_scores(q, w, dec32, None, ctx_len=128, m=4))
    # a NULL scale means 1
    assert np.array_equal(s8_unit, oracle.index_scores(q, w, codes[None], None, ctx_len=128, m=4))


def test_index_visibility_boundary():
    rng = np.random.default_rng(10)
    L, m, T = 40, 4, 7
    q, w, k = _idx_case(rng, 1, T, L, m, 2, 8)
    s = oracle.index_scores(q, w, k, None, ctx_len=L, m=m)
    for j in range(T):
        t = L - T + j
        nvis = (t + 1) // m
        assert np.all(np.isfinite(s[0, j, :nvis]))
        assert np.all(np.isneginf(s[0, j, nvis:]))


# ----------------------------------------------------------------------
# top-k
# ----------------------------------------------------------------------

def _better(a, b):
    """(score, index) a ranks before b: higher score, then lower index."""
    return a[0] > b[0] or (a[0] == b[0] and a[1] < b[1])


@pytest.mark.parametrize("n", [1, 5, 9])
def test_topk_brute_force_over_subsets(n):
    rng = np.random.default_rng(11 + n)
    for trial in range(6):
        # few distinct values -> many exact ties
        scores = rng.integers(0, 4, size=n).astype(np.float64) if trial % 2 else rng.normal(size=n)
        for k in range(1, n + 2):
            idx, sel, kth = oracle.select_row(scores, n, k)
            take = min(k, n)
            want = None
            for comb in itertools.combinations(range(n), take):
                inside = [(scores[i], i) for i in comb]
                outside = [(scores[i], i) for i in range(n) if i not in comb]
                if all(_better(a, b) for a in inside for b in outside):
                    assert want is None  # the defining property has one solution
                    want = list(comb)
            assert list(idx[:take]) == want
            assert list(idx[take:]) == [-1] * (k - take)
            assert np.all(np.diff(idx[:take]) > 0)  # ascending index order
            assert kth == (min(scores[i] for i in want) if take == k else -math.inf)
            assert np.array_equal(sel[:take], scores[idx[:take]])


def test_topk_ties_prefer_lower_index_and_pad():
    scores = np.array([5, 7, 7, 7, 1, 7, 0], dtype=np.float64)
    idx, _, kth = oracle.select_row(scores, 7, 3)
    assert list(idx) == [1, 2, 3] and kth == 7
    idx, _, _ = oracle.select_row(scores, 4, 6)  # only 4 visible
    assert list(idx) == [0, 1, 2, 3, -1, -1]


def test_topk_end_to_end_matches_library_sort():
    rng = np.random.default_rng(12)
    B, T, L, m, HI, DI, k = 2, 3, 200, 4, 2, 8, 11
    q, w, kk = _idx_case(rng, B, T, L, m, HI, DI)
    r = oracle.topk(q, w, kk, None, ctx_len=L, m=m, k=k, want_scores=True)
    sc = r["scores"]
    for b, j in itertools.product(range(B), range(T)):
        t = L - T + j
        nvis = (t + 1) // m
        order = sorted(range(nvis), key=lambda s: (-sc[b, j, s], s))[:k]  # library sort
        assert list(r["idx"][b, j]) == sorted(order) + [-1] * (k - len(order))


# ----------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------

def _att_case(rng, B, T, L, m, H, d, W, fmt="f32"):
    q = rng.normal(size=(B, T, H, d)) / math.sqrt(d)
    ent = rng.normal(size=(B, L // m, d))
    p0 = max(0, L - T - W + 1)
    tok = rng.normal(size=(B, L - p0, d))
    cast = (lambda a: a.astype(np.float32)) if fmt == "f32" else \
        (lambda a: stored_numpy(torch.from_numpy(a).to(torch.bfloat16)))
    return cast(q), cast(ent), cast(tok), p0


def test_short_context_hca_is_textbook_window_attention():
    """Context shorter than one HCA chunk: no visible entry, so HCA is plain
    softmax attention over the window rows (library SDPA in fp64)."""
    rng = np.random.default_rng(13)
    for L, W in [(100, 128), (127, 128), (90, 32)]:
        B, T, H, d = 2, 3, 4, 16
        q, ent, tok, p0 = _att_case(rng, B, T, max(L, 128), 128, H, d, W)
        ent = ent[:, : L // 128]
        tok = rng.normal(size=(B, L - max(0, L - T - W + 1), d)).astype(np.float32)
        p0 = max(0, L - T - W + 1)
        out = oracle.attend(q, ent if ent.shape[1] else np.zeros((B, 0, d), np.float32), None, tok, p0, L, 128, W)
        for j in range(T):
            t = L - T + j
            lo = max(0, t - W + 1)
            rows = torch.from_numpy(tok[:, lo - p0: t - p0 + 1].astype(np.float64))  # [B][n][d]
            qq = torch.from_numpy(q[:, j].astype(np.float64))[:, :, None, :]  # [B][H][1][d]
            kv = rows[:, None].expand(B, H, -1, d)
            ref = torch.nn.functional.scaled_dot_product_attention(qq, kv, kv)[:, :, 0]
            assert np.allclose(out[:, j], ref.numpy(), atol=1e-12)


def test_topk_covering_all_entries_equals_dense():
    rng = np.random.default_rng(14)
    B, T, L, m, H, d, W = 2, 5, 64, 4, 3, 8, 8
    q, ent, tok, p0 = _att_case(rng, B, T, L, m, H, d, W)
    N = L // m
    idx = np.full((B, T, N + 3), -1, dtype=np.int32)
    for j in range(T):
        nvis = (L - T + j + 1) // m
        for b in range(B):
            idx[b, j, :nvis] = rng.permutation(nvis)  # order must not matter
    sparse = oracle.attend(q, ent, idx, tok, p0, L, m, W)
    dense = oracle.attend(q, ent, None, tok, p0, L, m, W)
    assert np.allclose(sparse, dense, atol=1e-12)


def test_attention_weights_sum_to_one_and_two_candidate_closed_form():
    rng = np.random.default_rng(15)
    B, T, L, m, H, d, W = 1, 2, 48, 4, 2, 8, 4
    q, ent, tok, p0 = _att_case(rng, B, T, L, m, H, d, W)
    for j, h in itertools.product(range(T), range(H)):
        wts = oracle.attend_weights(q, ent, None, tok, p0, L, m, W, 0, j, h)
        assert wts.shape[0] == (L - T + j + 1) // m + W
        assert abs(wts.sum() - 1.0) < 1e-12 and (wts > 0).all()
    # exactly two candidates (context 2, window 2, no entry visible with m = 4):
    # weight of token 0 = sigmoid((q.x0 - q.x1)/sqrt(d))
    q2 = rng.normal(size=(1, 1, 1, 8)).astype(np.float32)
    tok2 = rng.normal(size=(1, 2, 8)).astype(np.float32)
    ent2 = np.zeros((1, 0, 8), np.float32)
    wts = oracle.attend_weights(q2, ent2, None, tok2, 0, 2, 4, 2, 0, 0, 0)
    z = float(np.dot(q2[0, 0, 0].astype(np.float64), tok2[0, 0].astype(np.float64) - tok2[0, 1].astype(np.float64))) / math.sqrt(8)
    assert wts[0] == pytest.approx(1.0 / (1.0 + math.exp(-z)), abs=1e-14)
    out = oracle.attend(q2, ent2, None, tok2, 0, 2, 4, 2)
    assert np.allclose(out[0, 0, 0], wts[0] * tok2[0, 0] + wts[1] * tok2[0, 1], atol=1e-12)


def test_single_candidate_returns_that_row_and_duplicates_count_twice():
    rng = np.random.default_rng(16)
    d = 16
    q = rng.normal(size=(1, 1, 2, d)).astype(np.float32)
    tok = rng.normal(size=(1, 1, d)).astype(np.float32)
    ent = np.zeros((1, 0, d), np.float32)
    out = oracle.attend(q, ent, None, tok, 0, 1, 4, 1)  # context of one token, window 1
    assert np.allclose(out[0, 0], np.broadcast_to(tok[0, 0], (2, d)), atol=1e-15)
    # a candidate listed twice gets twice the weight: with e = entry 0 listed
    # twice and the window token once, weight(e) = 2a/(2a+b)
    ent1 = rng.normal(size=(1, 1, d)).astype(np.float32)
    tok1 = rng.normal(size=(1, 4, d)).astype(np.float32)
    idx = np.array([[[0, 0]]], dtype=np.int32)
    o = oracle.attend(q[:, :, :1], ent1, idx, tok1, 0, 4, 4, 1)
    a = math.exp(float(np.dot(q[0, 0, 0].astype(np.float64), ent1[0, 0].astype(np.float64))) / math.sqrt(d))
    bb = math.exp(float(np.dot(q[0, 0, 0].astype(np.float64), tok1[0, 3].astype(np.float64))) / math.sqrt(d))
    we = 2 * a / (2 * a + bb)
    assert np.allclose(o[0, 0, 0], we * ent1[0, 0] + (1 - we) * tok1[0, 3], atol=1e-12)


def test_visibility_boundary_in_attention():
    """An entry whose block ends exactly at the query position is attended;
    the next one (block not yet complete) is not."""
    d, m = 8, 4
    q = np.zeros((1, 1, 1, d), np.float32)
    q[0, 0, 0, 0] = 60.0
    ent = np.zeros((1, 3, d), np.float32)
    ent[0, 1, 0] = 10.0  # block [4, 8): visible to t = 7, not to t = 6
    ent[0, 2, 0] = 20.0  # block [8, 12)
    tok = np.zeros((1, 12, d), np.float32)
    o7 = oracle.attend(q, ent, None, tok[:, :8], 0, 8, m, 1)
    assert o7[0, 0, 0, 0] == pytest.approx(10.0, rel=1e-9)
    o6 = oracle.attend(q, ent[:, :1], None, tok[:, :7], 0, 7, m, 1)
    assert o6[0, 0, 0, 0] == pytest.approx(0.0, abs=1e-9)
    idx = np.array([[[1, 2]]], dtype=np.int32)
    with pytest.raises(ValueError):
        oracle.attend(q, ent[:, :2], idx, tok[:, :8], 0, 8, m, 1)  # entry 2 is not visible at t = 7


def test_bf16_attention_matches_fp32_of_same_values():
    rng = np.random.default_rng(17)
    q, ent, tok, p0 = _att_case(rng, 1, 2, 256, 4, 4, 32, 16, fmt="bf16")
    o_b = oracle.attend(q, ent, None, tok, p0, 256, 4, 16)
    f = lambda a: oracle.decode(a).astype(np.float32)
    o_f = oracle.attend(f(q), f(ent), None, f(tok), p0, 256, 4, 16)
    assert np.allclose(o_b, o_f, atol=1e-12)


# ----------------------------------------------------------------------
# attention sink and output RoPE ("1M Context != Lossless Long Memory", sections 7 and 8)
# ----------------------------------------------------------------------

def test_rope_is_the_textbook_rotation():
    """Pair k of the last R dims turns by pos * 10000^(-2k/R): pair 0 by pos radians; position 0
    is the identity; rotations compose and keep norms; the first d - R dims are untouched."""
    d, R = 12, 8
    e = np.zeros((1, d))
    e[0, d - R] = 1.0
    got = oracle.rope(e, [0.7], R)
    assert np.allclose(got[0, d - R:d - R + 2], [np.cos(0.7), np.sin(0.7)], rtol=0, atol=1e-15)
    e2 = np.zeros((1, d))
    e2[0, d - 2] = 1.0  # last pair: frequency 10000^(-(R-2)/R)
    f = 10000.0 ** (-(R - 2) / R)
    assert np.allclose(oracle.rope(e2, [3.0], R)[0, d - 2:], [np.cos(3 * f), np.sin(3 * f)], rtol=0, atol=1e-15)
    rng = np.random.default_rng(41)
    x = rng.normal(size=(5, d))
    assert np.array_equal(oracle.rope(x, np.zeros(5), R), x)
    a = oracle.rope(oracle.rope(x, [1, 2, 3, 4, 5], R), [10, 20, 30, 40, 50], R)
    assert np.allclose(a, oracle.rope(x, [11, 22, 33, 44, 55], R), rtol=0, atol=1e-12)
    assert np.allclose(np.linalg.norm(a, axis=1), np.linalg.norm(x, axis=1), rtol=1e-14)
    assert np.array_equal(a[:, :d - R], x[:, :d - R])


def _window_case(seed, L, H=4, d=16, W=8):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(1, 1, H, d)).astype(np.float32)
    tok = rng.normal(size=(1, L, d)).astype(np.float32)
    ent = np.zeros((1, max(L // 128, 1), d), dtype=np.float32)
    return q, ent, tok


def test_sink_at_minus_infinity_changes_nothing_and_single_row_closed_form():
    L, W, H, d = 50, 8, 4, 16
    q, ent, tok = _window_case(42, L, H, d, W)
    plain = oracle.attend(q, ent, None, tok, 0, L, 128, W)
    assert np.array_equal(oracle.attend(q, ent, None, tok, 0, L, 128, W, sink=np.full(H, -np.inf)), plain)
    # one candidate row v (window 1, no entries): out = v * e^l / (e^l + e^z) with l = q.v / sqrt(d)
    z = np.array([-1.0, 0.0, 0.5, 3.0])
    got = oracle.attend(q, ent, None, tok, 0, L, 128, 1, sink=z)
    v = tok[0, L - 1].astype(np.float64)
    for h in range(H):
        ell = float(q[0, 0, h].astype(np.float64) @ v) / np.sqrt(d)
        assert np.allclose(got[0, 0, h], v / (1.0 + np.exp(z[h] - ell)), rtol=1e-13, atol=1e-15)


def test_output_rope_is_undone_by_rope_at_the_query_position():
    L, W, H, d, R = 70, 16, 4, 32, 8
    q, ent, tok = _window_case(43, L, H, d, W)
    plain = oracle.attend(q, ent, None, tok, 0, L, 128, W)
    rot = oracle.attend(q, ent, None, tok, 0, L, 128, W, rope_dims=R)
    assert np.array_equal(rot[..., :d - R], plain[..., :d - R])
    assert np.allclose(oracle.rope(rot, L - 1, R), plain, rtol=0, atol=1e-12)


def test_output_rope_turns_absolute_positions_into_distances():
    """With RoPE at each row's own position on the last R dims of the query and of the K=V rows, the
    rotated output depends only on distances: shifting every position by the same amount (same
    content) leaves it unchanged ("1M Context != ...", section 8)."""
    H, d, R, W = 4, 32, 8, 12
    rng = np.random.default_rng(44)
    q0 = rng.normal(size=(1, 1, H, d))
    rows0 = rng.normal(size=(W, d))
    outs = []
    for L in (40, 40 + 37, 40 + 1000):  # query at t = L-1, window rows at positions L-W .. L-1
        t = L - 1
        pos = np.arange(L - W, L)
        q = oracle.rope(q0, t, R).astype(np.float32)
        tok = np.zeros((1, L, d), dtype=np.float32)
        tok[0, L - W:] = oracle.rope(rows0, pos, R).astype(np.float32)
        ent = np.zeros((1, 1, d), dtype=np.float32)
        # m larger than every context here: no compressed entry is visible, only the window
        # (the fp32 inputs round differently at each shift: compare with float32-level tolerance)
        outs.append(oracle.attend(q, ent, None, tok, 0, L, 1 << 20, W, rope_dims=R))
    for o in outs[1:]:
        assert np.allclose(o, outs[0], rtol=1e-5, atol=1e-5)
