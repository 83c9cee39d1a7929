"""The allocation-free decode top-k (cslc_decode_topk_noalloc).

It serves callers that cannot call cudaMalloc (memory planned at start-up,
paths where an allocation would synchronise the device, C callers without an
allocator): its scratch is a static device array inside the library. This
file checks, through the C ABI, that two calls in a row give exactly the same
indices as the workspace-based cslc_decode_topk, and that an oversized call
is rejected. It runs last so a failure here never hides the other tests.
"""

import ctypes

import numpy as np
import pytest
import torch

from compressed_sparse_long_compress_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def C(cuda_device):
    from compressed_sparse_long_compress_b200 import cslc
    return cslc


def _case(B, n_max, n_list, seed, ties):
    s = W.rand_f32((B, n_max), seed=seed, device="cuda")
    if ties:
        s = torch.round(s * 4) / 4
    return s, torch.tensor(n_list, dtype=torch.int32, device="cuda")


def test_noalloc_matches_workspace_version_twice(C):
    cases = [
        (_case(8, 200000, [200000, 150000, 1024, 900, 0, 5, 199999, 131072], 1201, False), 1024),
        (_case(3, 50000, [50000, 40000, 17], 1202, True), 2048),
    ]
    for (scores, n), topk in cases:     # two calls in a row, different shapes and contents
        ref = C.decode_topk(scores, n, topk)
        got = C.decode_topk_noalloc(scores, n, topk)
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
    # and the same call again after a different one reused the scratch
    (scores, n), topk = cases[0]
    again = C.decode_topk_noalloc(scores, n, topk)
    torch.cuda.synchronize()
    assert torch.equal(again, C.decode_topk(scores, n, topk))


def _largest_fitting_n_max(C, B, topk, limit=16 << 20):
    lo, hi = 0, 1 << 22
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if C.LIB.cslc_decode_topk_workspace_bytes(B, mid, topk) <= limit:
            lo = mid
        else:
            hi = mid - 1
    return lo


def test_noalloc_at_the_size_limit(C):
    """The largest n_max whose scratch fits the 16 MiB array (B = 8) gives
    exactly the workspace version's indices; one entry more is refused."""
    B, topk = 8, 1024
    n_max = _largest_fitting_n_max(C, B, topk)
    assert n_max == 259068
    n_list = [n_max, n_max - 1, 200000, 1024, 1, 0, 131071, n_max]
    scores, n = _case(B, n_max, n_list, 1203, False)
    ref = C.decode_topk(scores, n, topk)
    got = C.decode_topk_noalloc(scores, n, topk)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
    big = torch.zeros(B, n_max + 1, device="cuda")
    idx = torch.empty(B, topk, dtype=torch.int32, device="cuda")
    st = C.LIB.cslc_decode_topk_noalloc(ctypes.c_void_p(big.data_ptr()), ctypes.c_void_p(n.data_ptr()), B, n_max + 1,
                                        topk, ctypes.c_void_p(idx.data_ptr()), None)
    assert st == 5


def test_noalloc_rejects_oversized_calls(C):
    scores = torch.zeros(64, 40000, device="cuda")
    n = torch.full((64,), 40000, dtype=torch.int32, device="cuda")
    idx = torch.empty(64, 1024, dtype=torch.int32, device="cuda")
    st = C.LIB.cslc_decode_topk_noalloc(ctypes.c_void_p(scores.data_ptr()), ctypes.c_void_p(n.data_ptr()), 64, 40000,
                                        1024, ctypes.c_void_p(idx.data_ptr()), None)
    assert st == 5 and b"static scratch" in C.LIB.cslc_last_error()
