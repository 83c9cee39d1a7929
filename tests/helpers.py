"""Comparison helpers shared by the GPU parity tests (no method arithmetic)."""

import numpy as np
import torch

# Tolerances for floating-point outputs (bf16 compute, fp32 accumulation):
# max-abs 2e-2 and relative L2 1e-2 for bf16 KV, 5e-2 relative L2 for FP8 KV.
MAX_ABS = 2e-2
REL_L2_BF16 = 1e-2
REL_L2_FP8 = 5e-2


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def rel_l2(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((got - ref).ravel())
    return float(num / den) if den > 0 else float(num)


def assert_close(got, ref, rel=REL_L2_BF16, max_abs=MAX_ABS, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin), f"{what}: inf/nan pattern differs"
    d = np.abs(got[fin] - ref[fin])
    ma = float(d.max()) if d.size else 0.0
    rl = rel_l2(got[fin], ref[fin])
    assert ma <= max_abs and rl <= rel, f"{what}: max-abs {ma:.3e} rel-L2 {rl:.3e}"
    return ma, rl


def assert_close_scaled(got, ref, rel=REL_L2_BF16, max_rel_abs=MAX_ABS, what=""):
    """Max-abs relative to the largest |ref| (only for outputs that grow far
    beyond O(1) on purpose, where one bf16 ulp exceeds the absolute bound)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    fin = np.isfinite(ref)
    scale = max(1.0, float(np.abs(ref[fin]).max())) if fin.any() else 1.0
    return assert_close(got / scale, ref / scale, rel, max_rel_abs, what)


def sample_rows(L: int, n: int, seed: int) -> np.ndarray:
    """First rows, last rows and a seeded spread in between, sorted, unique."""
    rng = np.random.default_rng(seed)
    k = max(1, n // 4)
    rows = np.concatenate([np.arange(min(k, L)), np.arange(max(0, L - k), L),
                           rng.integers(0, L, max(0, n - 2 * k))])
    return np.unique(rows)


def check_selection(got_idx, ref_idx, ref_scores, n_vis: int, k: int, tol: float = MAX_ABS):
    """Compares a GPU selection row with the oracle's row built from the
    oracle's own scores. Returns True when they are identical. When they
    differ, every entry in the symmetric difference must be a near-tie: its
    oracle score lies within `tol` (the score tolerance) of the oracle's k-th
    largest visible score, so a rounding difference inside the tolerance can
    move it across the threshold; anything else fails."""
    got_idx = np.asarray(got_idx)
    ref_idx = np.asarray(ref_idx)
    if np.array_equal(got_idx, ref_idx):
        return True
    s = np.asarray(ref_scores, dtype=np.float64)[:n_vis]
    kk = min(k, n_vis)
    kth = np.sort(s)[::-1][kk - 1]
    diff = np.setxor1d(got_idx[got_idx >= 0], ref_idx[ref_idx >= 0])
    assert (got_idx >= 0).sum() == kk, "valid slot count differs from min(k, n_vis)"
    far = diff[np.abs(s[diff] - kth) > tol]
    assert far.size == 0, f"selection differs beyond near-ties: entries {far[:8]} (k-th score {kth})"
    return False


def max_differing(n_rows: int) -> int:
    """Rows whose selection may differ from the oracle's (each a verified
    near-tie): 1 % of the rows, at least one."""
    return max(1, n_rows // 100)
