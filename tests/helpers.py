"""Parity helpers shared by the GPU tests (comparison rules only; no arithmetic of the method)."""
import numpy as np
import torch

# Tolerances of the acceptance rules: compressed entries max |err| <= 2e-2; attention output
# max |err| <= 2e-2 and mean |err| <= 2e-3 against fp64; top-k sets exact except near-ties whose
# score gap is below 1e-6 relative to the k-th score (floor 1e-6 * mean |I| for exact-zero ties).
C_MAX_ABS = 2e-2
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
TIE_REL = 1e-6


def to_np(t):
    return t.detach().float().cpu().double().numpy() if isinstance(t, torch.Tensor) else np.asarray(t)


def check_close(got, ref, max_abs, mean_abs=None, what=""):
    got, ref = to_np(got), np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    err = np.abs(got - ref)
    assert err.max() <= max_abs, f"{what}: max abs err {err.max():.3e} > {max_abs}"
    if mean_abs is not None:
        assert err.mean() <= mean_abs, f"{what}: mean abs err {err.mean():.3e} > {mean_abs}"
    return float(err.max()), float(err.mean())


def check_topk_sets(gpu_idx, ref_idx, ref_scores, vis, k):
    """Compare selected sets row by row. Returns the list of (row, symmetric difference) near-tie
    exceptions; raises on any other difference or on an invalid GPU row."""
    g = to_np(gpu_idx).astype(np.int64)
    o = np.asarray(ref_idx, np.int64)
    exceptions = []
    for i in range(g.shape[0]):
        n = int(vis[i])
        gs = g[i][g[i] >= 0]
        assert len(gs) == min(k, n), f"row {i}: {len(gs)} selected, expected {min(k, n)}"
        assert len(set(gs.tolist())) == len(gs), f"row {i}: duplicate indices"
        assert (gs < n).all(), f"row {i}: index not visible"
        assert (g[i][len(gs):] == -1).all() and (g[i][:len(gs)] >= 0).all(), f"row {i}: -1 padding not at the end"
        G, O = set(gs.tolist()), set(o[i][o[i] >= 0].tolist())
        diff = G ^ O
        if not diff:
            continue
        sc = np.asarray(ref_scores[i][:n], np.float64)
        kth = np.sort(sc)[::-1][min(k, n) - 1]
        tol = TIE_REL * abs(kth) + TIE_REL * float(np.abs(sc).mean())
        bad = [s for s in diff if abs(sc[s] - kth) > tol]
        assert not bad, f"row {i}: selection differs beyond the near-tie band: {sorted(bad)[:8]} (kth={kth})"
        exceptions.append((i, sorted(diff)))
    return exceptions
