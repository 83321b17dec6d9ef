"""v4a_topk_noalloc: the top-k entry point for callers that cannot allocate
device memory (a plug-in whose host framework owns every allocation, a serving
loop where allocating is not allowed).  It must give exactly what v4a_topk
gives with a caller-provided workspace, call after call, although every call
reuses the same built-in scratch array; and it must refuse shapes whose
scratch would not fit, saying so.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import workload as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def v4a():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import compressed_sparse_long_v4a_b200 as v
    return v


def _case(seed):
    # the 1M-context CSA decode shape: 4 sequences x 262,144 entries, fp8 keys, top-1024
    c = wl.index_case(4, 1, 1 << 20, 4, 16, 128, "bf16", "e4m3", seed=seed)
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in c.items()}


def _with_workspace(v4a, c, k):
    idx = torch.empty((4, 1, k), dtype=torch.int32, device="cuda")
    sco = torch.empty((4, 1, k), dtype=torch.float32, device="cuda")
    v4a.v4a_topk(c["q_i"], c["w"], c["k_i"], c["k_scale"], idx, sco, m=4, k=k, ctx_len=1 << 20)
    return idx, sco


def _no_alloc(v4a, c, k):
    idx = torch.full((4, 1, k), -7, dtype=torch.int32, device="cuda")
    sco = torch.full((4, 1, k), 7.0, dtype=torch.float32, device="cuda")
    v4a.v4a_topk_noalloc(c["q_i"], c["w"], c["k_i"], c["k_scale"], idx, sco, m=4, k=k, ctx_len=1 << 20)
    return idx, sco


def test_no_alloc_topk_matches_workspace_topk_twice(v4a):
    k = 1024
    first, second = _case(seed=41), _case(seed=42)
    for c in (first, second):  # two calls in a row, each after the other left the scratch dirty
        ref_idx, ref_sco = _with_workspace(v4a, c, k)
        idx, sco = _no_alloc(v4a, c, k)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx)
        assert (idx >= 0).all()
        np.testing.assert_allclose(sco.cpu().numpy(), ref_sco.cpu().numpy(), rtol=0, atol=0)
    # and the same inputs again right after: identical
    idx2, sco2 = _no_alloc(v4a, second, k)
    torch.cuda.synchronize()
    assert torch.equal(idx2, idx) and torch.equal(sco2, sco)


def test_no_alloc_topk_refuses_shapes_beyond_its_scratch(v4a):
    q_i = torch.zeros((1, 1, 16, 128), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((1, 1, 16), dtype=torch.float32, device="cuda")
    k_i = torch.zeros((1, 1, 128), dtype=torch.uint8, device="cuda")
    k_s = torch.ones((1, 1), dtype=torch.float32, device="cuda")
    idx = torch.full((1, 1, 8), -7, dtype=torch.int32, device="cuda")
    # a context whose top-k scratch needs more than the built-in 64 MiB (4 bytes per score)
    too_long = 4 * (20 << 20)
    assert v4a.v4a_workspace_size("topk", batch=1, m=4, k=8, ctx_len=too_long, heads_i=16, d_i=128) > (64 << 20)
    with pytest.raises(v4a.V4AError) as e:
        v4a.v4a_topk_noalloc(q_i, w, k_i, k_s, idx, m=4, k=8, ctx_len=too_long)
    assert e.value.status == 1 and "v4a_topk_noalloc" in str(e.value) and str(64 << 20) in str(e.value)
    torch.cuda.synchronize()
    assert (idx == -7).all()  # nothing was launched


def test_no_alloc_topk_many_rows_matches_workspace_topk(v4a):
    # more query rows than the few-rows select takes (a prefill-like block of 512 queries): the per-row
    # select path also works out of the built-in scratch, bit-equal to the workspace call
    c = wl.index_case(1, 512, 4096, 4, 16, 128, "bf16", "bf16", seed=43)
    c = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in c.items()}
    k = 64
    ref_idx = torch.empty((1, 512, k), dtype=torch.int32, device="cuda")
    ref_sco = torch.empty((1, 512, k), dtype=torch.float32, device="cuda")
    v4a.v4a_topk(c["q_i"], c["w"], c["k_i"], c["k_scale"], ref_idx, ref_sco, m=4, k=k, ctx_len=4096)
    for _ in range(2):
        idx = torch.full((1, 512, k), -7, dtype=torch.int32, device="cuda")
        sco = torch.full((1, 512, k), 7.0, dtype=torch.float32, device="cuda")
        v4a.v4a_topk_noalloc(c["q_i"], c["w"], c["k_i"], c["k_scale"], idx, sco, m=4, k=k, ctx_len=4096)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx)
        assert torch.equal(sco, ref_sco)


def test_no_alloc_topk_reports_bad_shapes_as_argument_errors(v4a):
    q_i = torch.zeros((1, 1, 16, 128), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((1, 1, 16), dtype=torch.float32, device="cuda")
    k_i = torch.zeros((1, 1, 128), dtype=torch.uint8, device="cuda")
    k_s = torch.ones((1, 1), dtype=torch.float32, device="cuda")
    idx = torch.full((1, 1, 8), -7, dtype=torch.int32, device="cuda")
    with pytest.raises(v4a.V4AError) as e:
        v4a.v4a_topk_noalloc(q_i, w, k_i, k_s, idx, m=4, k=8, ctx_len=-5)
    assert e.value.status == 1 and "scratch" not in str(e.value)
    torch.cuda.synchronize()
    assert (idx == -7).all()
