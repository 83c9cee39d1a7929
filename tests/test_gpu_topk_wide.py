"""GPU parity of the prefill top-k on wide rows (a 1M-token CSA context has
262,144 entries) and of the BF16-score variant of the indexer + top-k.

Integer results are bit-exact against the oracle's selection on the same
scores. BF16 scores: each is the bf16 rounding of the kernel's fp32 score, so
it lies within the fp32 score tolerance (max-abs 2e-2) plus half a bf16 ulp of
the oracle's score, and equals the oracle's score rounded to bf16 except where
the two fp32 sums straddle a rounding boundary; the selection is exactly the
top-k of the kernel's own bf16 scores; its recall against the fp32 path's
selection is reported and gated.
"""

import numpy as np
import pytest
import torch

import oracle as O
from compressed_sparse_long_compress_b200 import workloads as W
from tests.helpers import f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def C(cuda_device):
    from compressed_sparse_long_compress_b200 import cslc
    return cslc


def dev(t):
    return t.to("cuda:0")


@pytest.mark.parametrize("Nc,q_pos0,kind", [
    (262144, 4 * 262144 - 6, "plain"),     # the 1M-token context: the last rows see every entry
    (245003, 4 * 245003 - 600, "ties"),    # ragged width; rows see 244,853 .. 245,003 entries
])
def test_topk_on_wide_rows_bitexact(C, Nc, q_pos0, kind):
    L, topk, m = 6, 1024, 4
    s = W.rand_f32((1, L, Nc), seed=1300 + Nc % 97)
    if kind == "ties":
        s = torch.round(s * 8) / 8
    idx = C.csa_topk(dev(s), m=m, topk=topk, q_pos0=q_pos0)
    ref = O.topk_select(f64(s), m, topk, q_pos0)
    assert np.array_equal(idx.cpu().numpy(), ref)
    # the same rows as bf16 scores
    sb = s.to(torch.bfloat16)
    idx_b = C.csa_topk_bf16(dev(sb), m=m, topk=topk, q_pos0=q_pos0)
    assert np.array_equal(idx_b.cpu().numpy(), O.topk_select(f64(sb), m, topk, q_pos0))


def test_indexer_topk_at_262144_entries(C):
    L, Nc, HI, m, topk = 8, 262144, 8, 4, 1024
    q_pos0 = 4 * Nc - L
    s = W.PrefillShape(B=1, L=L, H=16, m=m, HI=HI, topk=topk)
    x = W.prefill_inputs(s, wid=131, with_indexer=True)
    x["k_idx"] = W.randn_bf16((1, Nc, 64), W.seed_of(131, W.T_KIDX))
    qi, w, k = dev(x["q_idx"]), dev(x["w"]), dev(x["k_idx"])
    idx, scores = C.csa_indexer_topk(qi, w, k, m=m, topk=topk, q_pos0=q_pos0, scores=True)
    idx_blocked, _ = C.csa_indexer_topk(qi, w, k, m=m, topk=topk, q_pos0=q_pos0)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx_blocked)
    sc = f64(scores)
    assert np.array_equal(idx.cpu().numpy(), O.topk_select(sc, m, topk, q_pos0))
    ref = O.indexer_scores(f64(x["q_idx"]), f64(x["w"]), f64(x["k_idx"]), m, q_pos0)
    vis = np.isfinite(ref)   # entries past a row's n_vis are left unspecified
    assert vis.sum() > 8 * 262140 and float(np.abs(sc[vis] - ref[vis]).max()) <= 2e-2


@pytest.mark.parametrize("B,L,HI,m,topk,q_pos0,Nc", [
    (1, 4096, 4, 4, 128, 0, None),        # the tiny workload's CSA layer
    (2, 1000, 8, 4, 64, 0, None),
    (1, 777, 6, 4, 100, 37, None),        # H_I not a power of two (mma.sync kernel)
    (1, 300, 8, 4, 1024, 60000, 16384),   # rows of the 65,536-token workload
])
def test_indexer_topk_bf16_scores(C, B, L, HI, m, topk, q_pos0, Nc):
    s = W.PrefillShape(B=B, L=L, H=16, m=m, HI=HI, topk=topk)
    x = W.prefill_inputs(s, wid=132, with_indexer=True)
    if Nc is not None:
        x["k_idx"] = W.randn_bf16((B, Nc, 64), W.seed_of(132, W.T_KIDX))
    n_c = x["k_idx"].shape[1]
    qi, w, k = dev(x["q_idx"]), dev(x["w"]), dev(x["k_idx"])
    idx, sb = C.csa_indexer_topk_bf16(qi, w, k, m=m, topk=topk, q_pos0=q_pos0, scores=True)
    idx_blocked, _ = C.csa_indexer_topk_bf16(qi, w, k, m=m, topk=topk, q_pos0=q_pos0)
    idx32, s32 = C.csa_indexer_topk(qi, w, k, m=m, topk=topk, q_pos0=q_pos0, scores=True)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx_blocked)
    got = f64(sb)
    ref = O.indexer_scores(f64(x["q_idx"]), f64(x["w"]), f64(x["k_idx"]), m, q_pos0)
    vis = np.isfinite(ref)
    ref_b = O.round_bf16(ref)
    # within the fp32 score tolerance (2e-2) of the oracle plus the half bf16
    # ulp of the rounding; equal to the oracle's rounding but where the two
    # fp32 sums straddle a rounding boundary
    half_ulp = np.ldexp(1.0, np.frexp(np.where(vis, np.abs(got), 1.0))[1] - 9)
    diff = np.abs(np.where(vis, got, 0.0) - np.where(vis, ref, 0.0))
    assert np.all(diff <= 2e-2 + half_ulp), float((diff - half_ulp).max())
    assert np.mean(got[vis] == ref_b[vis]) > 0.99
    # the selection is exactly the top-k of the kernel's own bf16 scores
    got_vis = np.where(vis, got, -np.inf)
    idx_np = idx.cpu().numpy()
    assert np.array_equal(idx_np, O.topk_select(got_vis, m, topk, q_pos0))
    # recall against the fp32 path's selection
    i32 = idx32.cpu().numpy()
    kept, total = 0, 0
    for b in range(B):
        for t in range(L):
            a = i32[b, t][i32[b, t] >= 0]
            kept += len(np.intersect1d(a, idx_np[b, t]))
            total += len(a)
    recall = kept / max(1, total)
    print(f"bf16-score recall vs fp32 path: {recall:.4f}")
    assert recall > 0.95
