"""Comparison helpers shared by the GPU parity tests.

Tolerances (spec bar): fp32 inputs -> max-abs <= 1e-4 on the attention
output; bf16/fp8 inputs -> max-abs <= 2e-2 AND relative-L2 <= 1e-2.  Top-k
index sets must be identical except for entries whose oracle (fp64) score lies
within 1e-6 relative of the oracle's k-th score (the tie band).
"""
from __future__ import annotations

import numpy as np
import torch

from workload import stored_numpy

ATOL_F32 = 1e-4
ATOL_BF16 = 2e-2
RL2_BF16 = 1e-2
TIE_BAND = 1e-6


def dev(t: torch.Tensor | None) -> torch.Tensor | None:
    return None if t is None else t.cuda()


def host(t):
    return stored_numpy(t.cpu()) if isinstance(t, torch.Tensor) else t


def check_attention(gpu: torch.Tensor, ref: np.ndarray, fp32: bool, what: str = "") -> dict:
    g = gpu.detach().cpu().double().numpy()
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - ref)
    max_abs = float(err.max()) if err.size else 0.0
    rl2 = float(np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-30)) if err.size else 0.0
    if fp32:
        assert max_abs <= ATOL_F32, f"{what}: max-abs {max_abs:.3e} > {ATOL_F32}"
    else:
        assert max_abs <= ATOL_BF16, f"{what}: max-abs {max_abs:.3e} > {ATOL_BF16}"
        assert rl2 <= RL2_BF16, f"{what}: rel-L2 {rl2:.3e} > {RL2_BF16}"
    return dict(max_abs=max_abs, rel_l2=rl2)


def check_topk(gpu_idx: torch.Tensor, ref: dict, ctx_len: int, m: int, k: int, gpu_scores=None,
               rows=None) -> dict:
    """gpu_idx [B][T][k] vs the oracle's topk() dict (needs 'scores').  Returns
    the tie-band report: how many rows differed and every differing entry."""
    g = gpu_idx.cpu().numpy()
    B, T, _ = g.shape
    band_hits = []
    rows = rows if rows is not None else [(b, j) for b in range(B) for j in range(T)]
    for (b, j) in rows:
        t = ctx_len - T + j
        nvis = min((t + 1) // m, ref["scores"].shape[-1])
        take = min(k, nvis)
        row = g[b, j]
        sel = row[:take]
        assert (row[take:] == -1).all(), f"row {(b, j)}: padding"
        assert ((sel >= 0) & (sel < nvis)).all(), f"row {(b, j)}: index out of range"
        assert (np.diff(sel) > 0).all(), f"row {(b, j)}: not strictly ascending"
        want = ref["idx"][b, j, :take]
        if np.array_equal(sel, want):
            continue
        kth = ref["kth"][b, j]
        sc = ref["scores"][b, j]
        diff = np.setxor1d(sel, want)
        for s in diff:
            rel = abs(sc[s] - kth) / max(abs(kth), 1e-300)
            assert rel < TIE_BAND, (f"row {(b, j)}: entry {s} score {sc[s]!r} vs k-th {kth!r} "
                                    f"(rel {rel:.2e}) differs outside the tie band")
            band_hits.append((b, j, int(s), float(sc[s]), float(kth)))
    if gpu_scores is not None:
        gs = gpu_scores.cpu().double().numpy()
        for (b, j) in rows:
            t = ctx_len - T + j
            nvis = min((t + 1) // m, ref["scores"].shape[-1])
            take = min(k, nvis)
            sel = g[b, j, :take]
            exp = ref["scores"][b, j][sel]
            assert np.allclose(gs[b, j, :take], exp, rtol=2e-5, atol=1e-5 * max(1.0, np.abs(exp).max(initial=0))), \
                f"row {(b, j)}: selected scores"
            assert np.isneginf(gs[b, j, take:]).all()
    return dict(tie_band_entries=band_hits)


def check_scores(gpu: torch.Tensor, ref: np.ndarray, what: str = "") -> None:
    g = gpu.cpu().double().numpy()
    vis = np.isfinite(ref)
    assert np.array_equal(np.isneginf(g), ~vis), f"{what}: visibility mask"
    scale = max(1.0, float(np.abs(ref[vis]).max(initial=0.0)))
    err = float(np.abs(g[vis] - ref[vis]).max(initial=0.0))
    assert err <= 2e-5 * scale, f"{what}: score error {err:.3e} (scale {scale:.3e})"
