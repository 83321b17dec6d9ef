"""The prefill-chunk workload at full size: 4,096 causal query tokens at
positions 126,976 .. 131,071 of a 131,072-token bf16 sequence, m = 4, 16
indexer heads x 128, top-512, 64 heads x 512, window 128.

The GPU compresses the chunk (both streams) and runs top-k and sparse
attention for all 4,096 queries; the oracle checks every compressed entry and
key, and the top-k sets and attention outputs of sampled query rows (first,
last and some in between) one by one.  Top-k and attention read the same
bytes on both sides: the history entries and keys from the input generator,
followed by the chunk's entries and keys as the oracle compresses them.
"""
import numpy as np
import pytest
import torch

import oracle
import workload as wl
from parity_utils import check_attention, check_topk, dev, host

pytestmark = pytest.mark.gpu

SAMPLE_ROWS = [0, 1, 127, 1024, 2047, 3001, 4094, 4095]


@pytest.fixture(scope="module")
def v4a():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import compressed_sparse_long_v4a_b200 as v
    return v


def _bf16(values: np.ndarray) -> torch.Tensor:
    codes = oracle.bf16_encode(values)
    return torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16)


def test_prefill_c4096_full_size_sampled(v4a):
    w = wl.prefill_chunk()
    c = w["cfg"]
    B, L, T, H, d, m, k, W = c["batch"], c["ctx_len"], c["n_q"], c["heads"], c["d"], c["m"], c["k"], c["window"]
    n_hist, N = w["n_hist"], w["N"]
    n_new = T // m
    assert n_hist + n_new == N

    # 1. the chunk's compression, both streams, every entry
    ent_new = torch.empty((B, n_new, d), dtype=torch.bfloat16, device="cuda")
    key_new = torch.empty((B, n_new, c["d_i"]), dtype=torch.bfloat16, device="cuda")
    v4a.v4a_compress(dev(w["x"]), dev(w["gate"]), ent_new, m=m, xi=dev(w["xi"]), gate_i=dev(w["gate_i"]),
                     out_i=key_new)
    torch.cuda.synchronize()
    ref_e = oracle.compress(host(w["x"]), host(w["gate"]), m)
    ref_k = oracle.compress(host(w["xi"]), host(w["gate_i"]), m)
    for got, ref, what in ((ent_new, ref_e, "entries"), (key_new, ref_k, "indexer keys")):
        g = got.float().cpu().numpy()
        # one bf16 rounding of an f32 result: within 2^-8 of the value (plus f32 accumulation slack)
        assert np.all(np.abs(g - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6), f"compressed {what}"

    # 2. history followed by the oracle-compressed chunk, the same bytes for both sides
    entries = torch.cat([w["hist_entries"], _bf16(ref_e)], dim=1).contiguous()
    keys = torch.cat([w["hist_keys"], _bf16(ref_k)], dim=1).contiguous()

    # 3. top-k and sparse attention for all 4,096 queries
    idx = torch.empty((B, T, k), dtype=torch.int32, device="cuda")
    v4a.v4a_topk(dev(w["q_i"]), dev(w["w"]), dev(keys), None, idx, m=m, k=k, ctx_len=L)
    out = torch.empty((B, T, H, d), dtype=torch.float32, device="cuda")
    v4a.v4a_csa_attend(dev(w["q"]), dev(entries), idx, dev(w["token_kv"]), w["tok_pos0"], out, m=m, window=W,
                       ctx_len=L)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()

    # 4. sampled query rows against the oracle, each as its own one-query problem at t = L - T + j
    ent_h, key_h, tok_h = host(entries), host(keys), host(w["token_kv"])
    for j in SAMPLE_ROWS:
        Lj = L - T + j + 1
        ref = oracle.topk(host(w["q_i"][:, j:j + 1]), host(w["w"][:, j:j + 1]), key_h, None, Lj, m, k,
                          want_scores=True)
        check_topk(idx[:, j:j + 1], ref, Lj, m, k)
        r_out = oracle.attend(host(w["q"][:, j:j + 1]), ent_h, ref["idx"], tok_h, w["tok_pos0"], Lj, m, W)
        check_attention(out[:, j:j + 1], r_out, False, f"prefill row {j}")
