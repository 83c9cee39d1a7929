"""GPU parity of the compressor front end (hidden states -> the 4 W
projections -> window compression in one tcgen05 kernel) against the oracle's
float64 projections and compression, through the C ABI."""

import numpy as np
import pytest
import torch

import oracle as O
from compressed_sparse_long_compress_b200 import workloads as W
from tests.helpers import assert_close, f64, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def C(cuda_device):
    from compressed_sparse_long_compress_b200 import cslc
    return cslc


def _inputs(B, L, dm, m, overlap, seed):
    h = W.randn_bf16((B, L, dm), seed)
    Wt = W.randn_bf16((4 if overlap else 2, 128, dm), seed + 1, std=dm ** -0.5)
    bias = W.randn_bf16((2 * m if overlap else m, 128), seed + 2, std=0.1)
    return h, Wt, bias


@pytest.mark.parametrize("B,L,dm,m,overlap", [
    (2, 600, 256, 4, True),      # several tiles of 31 entries, a ragged last tile
    (1, 300, 128, 2, True),
    (1, 3, 64, 4, True),         # shorter than one window: no entry
    (2, 700, 192, 128, False),   # HCA: 5 entries, a ragged tail
])
def test_front_end_matches_oracle(C, B, L, dm, m, overlap):
    h, Wt, bias = _inputs(B, L, dm, m, overlap, 800 + dm)
    got = C.compress_front_end(h.cuda(), Wt.cuda(), bias.cuda(), m, overlap)
    torch.cuda.synchronize()
    assert got.shape == (B, L // m, 128)
    if L // m == 0:
        return
    ref = O.compressor_front_end(f64(h), f64(Wt), f64(bias), m, overlap)
    assert_close(f64(got), ref, what="front end entries")
    assert np.mean(f64(got) == ref) > 0.95   # all but rounding-boundary cases bit-exact


def test_front_end_full_size_sampled(C):
    """The 65,536-token CSA workload with d_model = 7168, as bench.py times it;
    sampled entries against the oracle on their own window's tokens."""
    L, dm, m = 65536, 7168, 4
    h = W.randn_bf16((1, L, dm), 811, device="cuda")
    Wt = W.randn_bf16((4, 128, dm), 812, device="cuda", std=dm ** -0.5)
    bias = W.randn_bf16((2 * m, 128), 813, device="cuda", std=0.1)
    got = C.compress_front_end(h, Wt, bias, m, True)
    torch.cuda.synchronize()
    Wf = f64(Wt)
    bf = f64(bias)
    for i in sample_rows(L // m, 24, seed=814):
        i = int(i)
        t0 = max(0, (i - 1) * m)
        toks = f64(h[:, t0:(i + 1) * m])
        ref = O.compressor_front_end(toks, Wf, bf, m, True)[:, -1]   # the slice's last entry is entry i
        assert_close(f64(got[:, i]), ref, what=f"entry {i}")
