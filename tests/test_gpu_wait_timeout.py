"""The tensor-core attention's bounded waits, made to run out on purpose.

Every wait on an mbarrier in the attention kernel gives up after a bounded
number of polls; the kernel then records V4A_ERR_DEVICE_FAULT, writes NaN to
every output it contributes to, frees its tensor memory and returns.  The test
hook v4a_test_attend_fault makes each CTA withhold one stage -- it issues no
copy and no arrival for it, so nothing is in flight while the CTA winds down --
and shortens the waits, so the give-up path runs in milliseconds.  Nothing
traps and nothing is left waiting: the next normal call on the same stream
must match the oracle.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
import workload as wl
from parity_utils import check_attention, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def v4a():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import compressed_sparse_long_v4a_b200 as v
    return v


def _csa_inputs(B, L, m, H, d, W, k, seed):
    a = wl.attend_case(B, 1, L, m, H, d, W, "bf16", seed)
    a["idx"] = wl.random_topk_idx(B, 1, L, m, k, seed + 1)
    return a


def _call(v4a, a, out, st, L, m, W):
    v4a.v4a_csa_attend(dev(a["q"]), dev(a["entries"]), dev(a["idx"]), dev(a["token_kv"]), a["tok_pos0"], out,
                       m=m, window=W, ctx_len=L, dev_status=st)


@pytest.mark.parametrize("withhold", [0, 1])
def test_withheld_stage_times_out_then_the_next_call_is_exact(v4a, withhold):
    # the tensor-core shape (bf16, d = 512, 64 heads); k = 256 + a 128-row window = 6 tiles per query, so
    # 40 queries are 240 tiles over 148 CTAs: every CTA has a tile 0, 92 of them a tile 1
    B, L, m, H, d, W, k = 40, 4096, 4, 64, 512, 128, 256
    a = _csa_inputs(B, L, m, H, d, W, k, seed=900 + withhold)
    out = torch.zeros((B, 1, H, d), dtype=torch.float32, device="cuda")
    st = torch.zeros((1,), dtype=torch.int32, device="cuda")
    v4a.lib.v4a_test_attend_fault(ctypes.c_int(withhold), ctypes.c_int(64))
    try:
        _call(v4a, a, out, st, L, m, W)
        torch.cuda.synchronize()
    finally:
        v4a.lib.v4a_test_attend_fault(ctypes.c_int(-1), ctypes.c_int(0))
    assert int(st.item()) == 4  # V4A_ERR_DEVICE_FAULT
    o = out.cpu().numpy()
    assert np.isnan(o).any(), "a timed-out CTA poisons its outputs"
    if withhold == 0:  # every CTA withheld its first tile: every query's output is poisoned
        for b in range(B):
            assert np.isnan(o[b]).any()
    # the same stream, a normal call: no kernel was left waiting, the context is intact, results exact
    st.zero_()
    out2 = torch.empty((B, 1, H, d), dtype=torch.float32, device="cuda")
    _call(v4a, a, out2, st, L, m, W)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = oracle.attend(host(a["q"]), host(a["entries"]), host(a["idx"]), host(a["token_kv"]), a["tok_pos0"], L, m,
                        W)
    check_attention(out2, ref, False, "after a timed-out call")
