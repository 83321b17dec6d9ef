"""The heterogeneous KV cache on the GPU: incremental decode through token rings (the state cache) and
a paged classical cache of 128-token blocks (lcm(4, 128)), with block ids handed out in shuffled order.

* fp32 (d = 128, CUDA-core attention): token by token from an empty cache; at checkpoints the pools
  (read back through the block table), the top-k sets and both attention outputs are checked against
  the oracle run on the whole sequence.
* bf16 / FP8 / MXFP4 at the tensor-core shapes (d = 512, 64 heads, 16 x 128 indexer): the paged path
  must give bit for bit what the contiguous path (already pinned to the oracle) gives on the same
  tokens: same kernels, same arithmetic, other addressing.
"""
import numpy as np
import pytest
import torch

import oracle
import workload as wl
from parity_utils import check_attention, check_topk, host

pytestmark = pytest.mark.gpu

BLOCK = 128  # lcm(m, m') tokens per block


@pytest.fixture(scope="module")
def v4a():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import compressed_sparse_long_v4a_b200 as v
    return v


class Layers:
    """A CSA layer (m = 4, indexer keys) and an HCA layer (m' = 128) decoding B sequences in lockstep."""

    def __init__(self, v4a, B, T, d, di, fmt, key_fmt, ring_rows, seed):
        g = wl._gen(seed)
        st = lambda shape: wl.store(wl.normal(g, shape), fmt).cuda()
        self.v, self.B, self.T, self.d, self.di, self.R = v4a, B, T, d, di, ring_rows
        self.kv, self.gc, self.xi, self.gi = st((B, T, d)), st((B, T, d)), st((B, T, di)), st((B, T, di))
        self.kvh, self.gh = st((B, T, d)), st((B, T, d))
        dt = self.kv.dtype
        R = ring_rows
        self.r_kv, self.r_gc = torch.zeros((B, R, d), dtype=dt, device="cuda"), torch.zeros((B, R, d), dtype=dt,
                                                                                              device="cuda")
        self.r_xi, self.r_gi = torch.zeros((B, R, di), dtype=dt, device="cuda"), torch.zeros((B, R, di), dtype=dt,
                                                                                               device="cuda")
        self.r_kvh, self.r_gh = torch.zeros((B, R, d), dtype=dt, device="cuda"), torch.zeros((B, R, d), dtype=dt,
                                                                                               device="cuda")
        nb_seq = (T + BLOCK - 1) // BLOCK
        self.n_blocks = B * nb_seq + 3
        rng = np.random.default_rng(seed)
        self.free = list(rng.permutation(self.n_blocks))
        self.bt_host = np.full((B, nb_seq), -1, dtype=np.int32)
        self.bt = torch.full((B, nb_seq), -1, dtype=torch.int32, device="cuda")
        P = self.n_blocks
        self.ent = torch.zeros((P * 32, d), dtype=dt, device="cuda")
        self.key_fmt = key_fmt
        if key_fmt == "e4m3":
            self.key = torch.zeros((P * 32, di), dtype=torch.uint8, device="cuda")
            self.kscale = torch.zeros((P * 32,), dtype=torch.float32, device="cuda")
            self.kexp = None
        elif key_fmt == "mxfp4":
            self.key = torch.zeros((P * 32, di // 2), dtype=torch.uint8, device="cuda")
            self.kexp = torch.zeros((P * 32, di // 32), dtype=torch.uint8, device="cuda")
            self.kscale = None
        else:
            self.key = torch.zeros((P * 32, di), dtype=dt, device="cuda")
            self.kscale = self.kexp = None
        self.hent = torch.zeros((P, d), dtype=dt, device="cuda")

    def step(self, t):
        v, R = self.v, self.R
        if t % BLOCK == 0:  # a new block for every sequence
            for b in range(self.B):
                self.bt_host[b, t // BLOCK] = self.free.pop()
            self.bt.copy_(torch.from_numpy(self.bt_host))
        v.v4a_ring_append([(self.kv[:, t], self.r_kv), (self.gc[:, t], self.r_gc), (self.xi[:, t], self.r_xi),
                           (self.gi[:, t], self.r_gi), (self.kvh[:, t], self.r_kvh), (self.gh[:, t], self.r_gh)], t)
        if (t + 1) % 4 == 0:
            r0 = (t - 3) % R
            kw = dict(out_i=self.key, out_i_scale=self.kscale, out_i_exp=self.kexp)
            v.v4a_compress_paged(self.r_kv[:, r0:r0 + 4], self.r_gc[:, r0:r0 + 4], self.ent, m=4,
                                 first_entry=(t + 1) // 4 - 1, block_table=self.bt, block_tokens=BLOCK,
                                 xi=self.r_xi[:, r0:r0 + 4], gate_i=self.r_gi[:, r0:r0 + 4], **kw)
        if (t + 1) % 128 == 0:
            r0 = (t - 127) % R
            v.v4a_compress_paged(self.r_kvh[:, r0:r0 + 128], self.r_gh[:, r0:r0 + 128], self.hent, m=128,
                                 first_entry=(t + 1) // 128 - 1, block_table=self.bt, block_tokens=BLOCK)

    def pool_rows(self, m, n):
        """Pool row of entries 0 .. n-1 of every sequence."""
        epb = BLOCK // m
        s = np.arange(n)
        return self.bt_host[:, s // epb].astype(np.int64) * epb + s % epb


def _queries(B, H, d, HI, DI, fmt, seed, q_std=1.0):
    g = wl._gen(seed)
    q = wl.store(wl.normal(g, (B, 1, H, d), q_std), fmt).cuda()
    qi = wl.store(wl.normal(g, (B, 1, HI, DI)), fmt).cuda()
    w = wl.uniform(g, (B, 1, HI)).cuda()
    return q, qi, w


def test_incremental_decode_fp32_matches_oracle(v4a):
    B, T, d, di, H, HI, k, W, R = 2, 1300, 128, 64, 16, 4, 64, 128, 256
    L = Layers(v4a, B, T, d, di, "f32", "f32", R, seed=400)
    checkpoints = {128, 129, 512, 1028, 1100, 1300}
    kv64, kvh64 = host(L.kv).astype(np.float64), host(L.kvh).astype(np.float64)
    for t in range(T):
        L.step(t)
        ctx = t + 1
        if ctx not in checkpoints:
            continue
        q, qi, w = _queries(B, H, d, HI, di, "f32", seed=410 + ctx, q_std=1.0 / np.sqrt(d))
        idx = torch.empty((B, 1, k), dtype=torch.int32, device="cuda")
        out = torch.empty((B, 1, H, d), device="cuda")
        outh = torch.empty((B, 1, H, d), device="cuda")
        st = torch.zeros((1,), dtype=torch.int32, device="cuda")
        v4a.v4a_topk_paged(qi, w, L.key, None, idx, m=4, k=k, ctx_len=ctx, block_table=L.bt, block_tokens=BLOCK,
                           dev_status=st)
        v4a.v4a_csa_attend_paged(q, L.ent, idx, L.r_kv, out, m=4, window=W, ctx_len=ctx, block_table=L.bt,
                                 block_tokens=BLOCK, dev_status=st)
        v4a.v4a_hca_attend_paged(q, L.hent, L.r_kvh, outh, m=128, window=W, ctx_len=ctx, block_table=L.bt,
                                 block_tokens=BLOCK, dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        N, Nh = ctx // 4, ctx // 128
        ref_e = oracle.compress(host(L.kv[:, :ctx]), host(L.gc[:, :ctx]), 4)
        ref_k = oracle.compress(host(L.xi[:, :ctx]), host(L.gi[:, :ctx]), 4)
        ref_h = oracle.compress(host(L.kvh[:, :ctx]), host(L.gh[:, :ctx]), 128)
        # the pools, read back through the block table
        for pool, ref, m in ((L.ent, ref_e, 4), (L.key, ref_k, 4), (L.hent, ref_h, 128)):
            if ref.shape[1] == 0:
                continue
            got = pool.double().cpu().numpy()[L.pool_rows(m, ref.shape[1])]
            assert np.abs(got - ref).max() <= 2e-6 * max(1.0, np.abs(ref).max()), f"pool m={m} at ctx {ctx}"
        ref_t = oracle.topk(host(qi), host(w), ref_k, None, ctx, 4, k, want_scores=True)
        check_topk(idx, ref_t, ctx, 4, k)
        q64 = host(q).astype(np.float64)
        r_out = oracle.attend(q64, ref_e, ref_t["idx"], kv64[:, :ctx], 0, ctx, 4, W)
        check_attention(out, r_out, True, f"paged csa ctx {ctx}")
        r_outh = oracle.attend(q64, ref_h if Nh else np.zeros((B, 0, d)), None, kvh64[:, :ctx], 0, ctx, 128, W)
        check_attention(outh, r_outh, True, f"paged hca ctx {ctx}")


@pytest.mark.parametrize("key_fmt", ["e4m3", "mxfp4"])
def test_paged_tensor_core_path_equals_contiguous(v4a, key_fmt):
    """bf16 d=512 x 64 heads, 16 x 128 indexer: decode through rings and shuffled blocks, then the same
    tokens through the contiguous calls; idx, scores and outputs must be identical."""
    B, T, d, di, H, HI, k, W, R = 2, 900, 512, 128, 64, 16, 64, 128, 256
    L = Layers(v4a, B, T, d, di, "bf16", key_fmt, R, seed=420)
    checkpoints = {640, 900}
    for t in range(T):
        L.step(t)
        ctx = t + 1
        if ctx not in checkpoints:
            continue
        q, qi, w = _queries(B, H, d, HI, di, "bf16", seed=430 + ctx)
        N, Nh = ctx // 4, ctx // 128
        # paged
        idx_p = torch.empty((B, 1, k), dtype=torch.int32, device="cuda")
        sc_p = torch.empty((B, 1, k), device="cuda")
        out_p = torch.empty((B, 1, H, d), device="cuda")
        outh_p = torch.empty((B, 1, H, d), device="cuda")
        st = torch.zeros((1,), dtype=torch.int32, device="cuda")
        kw = dict(m=4, k=k, ctx_len=ctx, block_table=L.bt, block_tokens=BLOCK, dev_status=st)
        if key_fmt == "mxfp4":
            v4a.v4a_topk_mxfp4_paged(qi, w, L.key, L.kexp, idx_p, sc_p, **kw)
        else:
            v4a.v4a_topk_paged(qi, w, L.key, L.kscale, idx_p, sc_p, **kw)
        v4a.v4a_csa_attend_paged(q, L.ent, idx_p, L.r_kv, out_p, m=4, window=W, ctx_len=ctx, block_table=L.bt,
                                 block_tokens=BLOCK, dev_status=st)
        v4a.v4a_hca_attend_paged(q, L.hent, L.r_kvh, outh_p, m=128, window=W, ctx_len=ctx, block_table=L.bt,
                                 block_tokens=BLOCK, dev_status=st)
        # contiguous: compress the whole prefix, then the plain calls
        ent = torch.empty((B, N, d), dtype=torch.bfloat16, device="cuda")
        hent = torch.empty((B, max(Nh, 1), d), dtype=torch.bfloat16, device="cuda")
        if key_fmt == "mxfp4":
            key = torch.empty((B, N, di // 2), dtype=torch.uint8, device="cuda")
            kexp = torch.empty((B, N, di // 32), dtype=torch.uint8, device="cuda")
            v4a.v4a_compress(L.kv[:, :ctx], L.gc[:, :ctx], ent, m=4, xi=L.xi[:, :ctx], gate_i=L.gi[:, :ctx],
                             out_i=key, out_i_exp=kexp)
        else:
            key = torch.empty((B, N, di), dtype=torch.uint8, device="cuda")
            ksc = torch.empty((B, N), dtype=torch.float32, device="cuda")
            v4a.v4a_compress(L.kv[:, :ctx], L.gc[:, :ctx], ent, m=4, xi=L.xi[:, :ctx], gate_i=L.gi[:, :ctx],
                             out_i=key, out_i_scale=ksc)
        v4a.v4a_compress(L.kvh[:, :ctx], L.gh[:, :ctx], hent[:, :Nh], m=128)
        idx_c = torch.empty_like(idx_p)
        sc_c = torch.empty_like(sc_p)
        if key_fmt == "mxfp4":
            v4a.v4a_topk_mxfp4(qi, w, key, kexp, idx_c, sc_c, m=4, k=k, ctx_len=ctx)
        else:
            v4a.v4a_topk(qi, w, key, ksc, idx_c, sc_c, m=4, k=k, ctx_len=ctx)
        p0 = ctx - W
        tok = L.kv[:, p0:ctx].contiguous()
        tokh = L.kvh[:, p0:ctx].contiguous()
        out_c = torch.empty_like(out_p)
        outh_c = torch.empty_like(outh_p)
        v4a.v4a_csa_attend(q, ent, idx_c, tok, p0, out_c, m=4, window=W, ctx_len=ctx)
        v4a.v4a_hca_attend(q, hent[:, :Nh].contiguous(), tokh, p0, outh_c, m=128, window=W, ctx_len=ctx)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        # the pools hold exactly the contiguous entries
        assert torch.equal(L.ent[torch.from_numpy(L.pool_rows(4, N)).cuda()], ent)
        assert torch.equal(L.hent[torch.from_numpy(L.pool_rows(128, Nh)).cuda()], hent[:, :Nh])
        assert torch.equal(idx_p, idx_c) and torch.equal(sc_p, sc_c), f"top-k at ctx {ctx}"
        assert torch.equal(out_p, out_c), f"csa at ctx {ctx}"
        assert torch.equal(outh_p, outh_c), f"hca at ctx {ctx}"
        if ctx == 900:
            # and straight against the oracle on the bytes the cache holds: top-k (tie band), CSA and HCA
            # attention (bf16 tolerance), not only transitively through the contiguous calls
            if key_fmt == "mxfp4":
                r_top = oracle.topk_mxfp4(host(qi), host(w), host(key), host(kexp), ctx, 4, k, want_scores=True)
            else:
                r_top = oracle.topk(host(qi), host(w), host(key), host(ksc), ctx, 4, k, want_scores=True)
            check_topk(idx_p, r_top, ctx, 4, k)
            r_c = oracle.attend(host(q), host(ent), r_top["idx"], host(tok), p0, ctx, 4, W)
            check_attention(out_p, r_c, False, f"paged csa vs oracle at ctx {ctx}")
            r_h = oracle.attend(host(q), host(hent[:, :Nh].contiguous()), None, host(tokh), p0, ctx, 128, W)
            check_attention(outh_p, r_h, False, f"paged hca vs oracle at ctx {ctx}")


def test_paged_bad_block_id_is_skipped_and_reported(v4a):
    """A block id outside the pool: attention skips the entries and reports V4A_ERR_DEVICE_FAULT; the
    indexer reads them as zero keys and reports it too; nothing reads outside the pools."""
    B, d, H, HI, di, W, R = 1, 512, 64, 16, 128, 128, 256
    ctx = 4 * 128 * 3
    n_blocks = 3
    g = wl._gen(440)
    ent = wl.store(wl.normal(g, (n_blocks * 32, d)), "bf16").cuda()
    hent = wl.store(wl.normal(g, (n_blocks, d)), "bf16").cuda()
    key = wl.store(wl.normal(g, (n_blocks * 32, di)), "bf16").cuda()
    ring = wl.store(wl.normal(g, (B, R, d)), "bf16").cuda()
    bt = torch.tensor([[0, n_blocks + 7, 1, 2] + [0] * 8], dtype=torch.int32, device="cuda")  # block 1 is bad
    q, qi, w = _queries(B, H, d, HI, di, "bf16", seed=441)
    idx = torch.empty((B, 1, 64), dtype=torch.int32, device="cuda")
    out = torch.empty((B, 1, H, d), device="cuda")
    for fn in ("topk", "csa", "hca"):
        st = torch.zeros((1,), dtype=torch.int32, device="cuda")
        if fn == "topk":
            v4a.v4a_topk_paged(qi, w, key, None, idx, m=4, k=64, ctx_len=512, block_table=bt, block_tokens=BLOCK,
                               dev_status=st)
        elif fn == "csa":
            sel = torch.arange(64, dtype=torch.int32, device="cuda").view(1, 1, 64) * 2  # entries 0..126: some in block 1
            v4a.v4a_csa_attend_paged(q, ent, sel, ring, out, m=4, window=W, ctx_len=512, block_table=bt,
                                     block_tokens=BLOCK, dev_status=st)
        else:
            v4a.v4a_hca_attend_paged(q, hent, ring, out, m=128, window=W, ctx_len=ctx, block_table=bt,
                                     block_tokens=BLOCK, dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 4, fn
        if fn != "topk":
            assert torch.isfinite(out).all()
