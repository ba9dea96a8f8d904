"""Comparison rules shared by the GPU parity tests.

Tolerances (from the stated targets; written here once):
  * floating point outputs stored in bf16: max |gpu - oracle| <= 2e-2 (absolute, the stated
    bound) AND max |gpu - oracle| <= 1e-2 * max |oracle| (norm-wise). The second bound keeps
    the check meaningful where the outputs themselves are far below 2e-2 (long candidate
    lists of small rows average to |O| ~ 1e-3): a zeroed or wrongly gathered output fails it.
    bf16 storage of O contributes 2^-9 relative, the bf16 softmax weights about as much;
  * fp32 outputs: max |gpu - oracle| <= 1e-4 * max |oracle| (norm-wise relative);
  * LSE: the same rule as the output of that dtype;
  * integer / byte outputs (FP4 codes, scale bytes, top-k indices, counts): bit-exact,
    except top-k members whose fp64 scores lie within a 1e-6 * max(1, |I_(k)|) gap of
    the k-th score (ties). The selected set is listed in ascending entry order.
"""
from __future__ import annotations

import numpy as np
import torch

BF16_ABS = 2e-2
BF16_REL = 1e-2
F32_REL = 1e-4
TIE_REL = 1e-6


def assert_close(gpu, ref, dtype: str, what: str, verbose: bool = False):
    """Compare under the rule of `dtype` ("bf16" or "f32"); returns max |diff|. With verbose,
    prints the observed error, the reference scale and the relative error."""
    g = gpu.detach().to("cpu").to(torch.float64).numpy() if isinstance(gpu, torch.Tensor) else np.asarray(gpu, np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    mask = ~np.isnan(r)
    assert np.isfinite(g[mask]).all(), f"{what}: non-finite GPU values"
    err = np.abs(g[mask] - r[mask]).max() if mask.any() else 0.0
    rmax = np.abs(r[mask]).max() if mask.any() else 0.0
    if verbose:
        print(f"[parity] {what}: max|diff| {err:.3e}, max|ref| {rmax:.3e}, "
              f"rel {err / max(rmax, 1e-30):.3e}")
    if dtype == "bf16":
        bound = min(BF16_ABS, BF16_REL * max(rmax, 1e-30))
    else:
        bound = F32_REL * max(rmax, 1e-30)
    assert err <= bound, f"{what}: max |diff| {err:.3e} > {bound:.3e} (max |ref| {rmax:.3e})"
    return err


def topk_ref_from_scores(scores: np.ndarray, k: int) -> list:
    """Brute-force TopK of a score vector (used on GPU fp32 scores): the k largest, ties to the
    lower index, as a set listed in ascending entry order."""
    order = sorted(range(len(scores)), key=lambda j: (-float(scores[j]), j))
    return sorted(order[:min(k, len(scores))])


def check_topk_query(gpu_idx_row, gpu_count, oracle_scores: np.ndarray, k: int,
                     gpu_scores_row=None, score_bound=None, what=""):
    """Check one query's TopK against the fp64 scores (see module docstring)."""
    E = len(oracle_scores)
    keff = min(k, E)
    assert int(gpu_count) == keff, f"{what}: count {gpu_count} != {keff}"
    row = np.asarray(gpu_idx_row)
    assert (row[keff:] == -1).all(), f"{what}: padding is not -1"
    sel = row[:keff].astype(np.int64)
    assert len(set(sel.tolist())) == keff, f"{what}: duplicate indices"
    assert ((sel >= 0) & (sel < E)).all(), f"{what}: index out of range"
    if gpu_scores_row is not None:
        gs = np.asarray(gpu_scores_row[:E], dtype=np.float32)
        # (i) the GPU's own selection is exact w.r.t. its fp32 scores (ascending entry order)
        assert sel.tolist() == topk_ref_from_scores(gs, k), f"{what}: selection vs own scores"
        if score_bound is not None:
            err = np.abs(gs.astype(np.float64) - oracle_scores)
            assert (err <= score_bound).all(), f"{what}: score error {err.max():.3e}"
    if keff == 0 or keff == E:
        return 0
    # (ii) the set equals the fp64 TopK except for ties within the stated gap
    ref = np.lexsort((np.arange(E), -oracle_scores))[:keff]
    kth = oracle_scores[ref[-1]]
    gap = TIE_REL * max(1.0, abs(kth))
    diff = set(sel.tolist()) ^ set(ref.tolist())
    for j in diff:
        assert abs(oracle_scores[j] - kth) <= gap, \
            f"{what}: entry {j} score {oracle_scores[j]!r} vs k-th {kth!r} is not a tie"
    return len(diff)


def sample_positions(n: int, m: int, extra=(), count: int = 24, seed: int = 0) -> list:
    """Query positions to compare at full size: both ends, block boundaries, ramps, random."""
    rng = np.random.default_rng(seed)
    pos = {0, 1, m - 2, m - 1, m, n - 1, n - 2, n // 2}
    pos |= {int(p) for p in extra}
    pos |= {int(p) for p in rng.integers(0, n, size=count)}
    return sorted(p for p in pos if 0 <= p < n)
