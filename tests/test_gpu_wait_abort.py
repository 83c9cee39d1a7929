"""The bounded-wait failure path of the pipelined tcgen05 kernels.

With the testing hook setting the wait limit (and the sleep between checks)
to 0 ns, the first wait that is not already satisfied gives up: the CTA's
roles leave their loops together, products and copies already issued
complete, TMEM is released, and cslc_sync_status reports
CSLC_ERR_DEVICE_CHECK. With the default limits restored, the same call then
runs normally and matches the oracle, so nothing was left behind (a CTA that
kept its TMEM would stall the next launch on that SM). No wait is ever left
unbounded: the hook only shortens the limits.
"""

import math

import numpy as np
import pytest
import torch

import oracle as O
from compressed_sparse_long_compress_b200 import workloads as W
from tests.helpers import assert_close, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def C(cuda_device):
    from compressed_sparse_long_compress_b200 import cslc
    return cslc


@pytest.fixture(autouse=True)
def _restore_limits(cuda_device):
    yield
    from compressed_sparse_long_compress_b200 import cslc
    cslc.testing_set_wait_limits(cslc.WAIT_LIMIT_NS_DEFAULT, cslc.WAIT_SLEEP_NS_DEFAULT)


def _aborts(C, run):
    C.testing_set_wait_limits(0, 0)
    run()
    with pytest.raises(C.CslcError) as ei:
        C.sync_status()
    assert ei.value.status == 7 and "timed out" in str(ei.value)
    C.testing_set_wait_limits(C.WAIT_LIMIT_NS_DEFAULT, C.WAIT_SLEEP_NS_DEFAULT)


def test_sparse_attention_wait_abort_then_recovers(C):
    L, H, n_c, k = 512, 64, 16384, 1024
    q = W.randn_bf16((1, L, H, 128), 1401).cuda()
    e = W.randn_bf16((1, n_c, 128), 1402, std=0.4).cuda()
    g = torch.Generator(device="cuda").manual_seed(1403)
    idx = torch.sort(torch.rand(1, L, n_c, device="cuda", generator=g).topk(k, dim=-1).indices.int(),
                     dim=-1).values.contiguous()
    scale = 1 / math.sqrt(128)
    _aborts(C, lambda: C.csa_sparse_attn(q, e, idx, scale))
    out, _ = C.csa_sparse_attn(q, e, idx, scale)
    C.sync_status()
    rows = np.array([0, 17, 255, 511])
    o_ref, _ = O.sparse_attention(f64(q), f64(e), idx.cpu().numpy(), scale, rows=rows)
    assert_close(f64(out)[:, rows], o_ref, what="sparse attention after an abort")


def test_dense_attention_wait_abort_then_recovers(C):
    L, H, m, n_c = 1001, 64, 4, 250
    q = W.randn_bf16((1, L, H, 128), 1411).cuda()
    e = W.randn_bf16((1, n_c, 128), 1412, std=0.4).cuda()
    scale = 1 / math.sqrt(128)
    _aborts(C, lambda: C.hca_dense_attn(q, e, m_prime=m, scale=scale))
    out, _ = C.hca_dense_attn(q, e, m_prime=m, scale=scale)
    C.sync_status()
    o_ref, _ = O.dense_causal_attention(f64(q), f64(e), m, scale)
    assert_close(f64(out), o_ref, what="dense attention after an abort")


def test_indexer_wait_abort_then_recovers(C):
    s = W.WORKLOADS["tiny"].csa
    x = {k: v.cuda() for k, v in W.prefill_inputs(s, 1421, with_indexer=True).items()}
    _aborts(C, lambda: C.csa_indexer_topk(x["q_idx"], x["w"], x["k_idx"], m=s.m, topk=s.topk, scores=True))
    idx, scores = C.csa_indexer_topk(x["q_idx"], x["w"], x["k_idx"], m=s.m, topk=s.topk, scores=True)
    C.sync_status()
    ref = O.indexer_scores(f64(x["q_idx"]), f64(x["w"]), f64(x["k_idx"]), s.m)
    vis = np.isfinite(ref)
    assert_close(np.where(vis, f64(scores), -np.inf), ref, what="indexer scores after an abort")
    assert np.array_equal(idx.cpu().numpy(), O.topk_select(np.where(vis, f64(scores), -np.inf), s.m, s.topk))


def test_front_end_wait_abort_then_recovers(C):
    B, L, dm, m = 1, 2048, 512, 4
    h = W.randn_bf16((B, L, dm), 1431).cuda()
    Wt = W.randn_bf16((4, 128, dm), 1432, std=dm ** -0.5).cuda()
    bias = W.randn_bf16((2 * m, 128), 1433, std=0.1).cuda()
    _aborts(C, lambda: C.compress_front_end(h, Wt, bias, m, True))
    got = C.compress_front_end(h, Wt, bias, m, True)
    C.sync_status()
    ref = O.compressor_front_end(f64(h), f64(Wt), f64(bias), m, True)
    assert_close(f64(got), ref, what="front end after an abort")
