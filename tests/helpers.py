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
    """Scores are O(10-100): max-abs is taken relative to the largest |ref|."""
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
