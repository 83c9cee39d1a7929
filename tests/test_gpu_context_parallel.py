"""Context-parallel CSA prefill through the library's kernels on one GPU.

The ranks are emulated in one process, one after the other: every rank's
compress phase runs first, the concatenation of their entries and keys
stands in for the all-gather, then every rank's attend phase runs (no kernel
waits on another rank). The concatenated outputs must equal the
single-sequence GPU pipeline bit for bit: a window's entry, a score and a row's
attention do not depend on where the shard boundaries fall, only on absolute
positions (the halo and q_pos0 carry those). A few rows are also checked
against the oracle.
"""

import numpy as np
import pytest
import torch

import oracle as O
from compressed_sparse_long_compress_b200 import context_parallel as CP
from compressed_sparse_long_compress_b200 import workloads as W
from tests.helpers import assert_close, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def C(cuda_device):
    from compressed_sparse_long_compress_b200 import cslc
    return cslc


def _inputs(L, m, seed):
    s = W.PrefillShape(B=1, L=L, H=64, m=m, HI=8, topk=512)
    x = W.prefill_inputs(s, wid=seed, with_indexer=True)
    x["kc"] = W.randn_bf16((1, L, 64), seed + 5)
    x["kz"] = W.randn_bf16((1, L, 64), seed + 6)
    x["k_pos_bias"] = W.randn_bf16((2 * m, 64), seed + 7, std=0.1)
    return {k: v.cuda() for k, v in x.items() if k != "k_idx"}, s


@pytest.mark.parametrize("world,L,m", [(3, 8195, 4), (4, 6000, 4), (2, 4099, 2)])
def test_emulated_ranks_equal_single_sequence(C, world, L, m):
    x, s = _inputs(L, m, 71)
    ops = CP.library_ops(C)
    # single sequence
    e = C.csa_compress(x["c"], x["z"], x["pos_bias"], m=m)
    k = C.csa_compress(x["kc"], x["kz"], x["k_pos_bias"], m=m)
    idx, _ = C.csa_indexer_topk(x["q_idx"], x["w"], k, m=m, topk=s.topk)
    ref, _ = C.csa_sparse_attn(x["q"], e, idx, s.scale)
    # emulated ranks
    xl = [CP.local_slices(x, L, m, world, r) for r in range(world)]
    parts = [CP.compress_local(xl[r], L, m, world, r, ops) for r in range(world)]
    e_all = torch.cat([p[1] for p in parts], dim=1).contiguous()
    k_all = torch.cat([p[2] for p in parts], dim=1).contiguous()
    out = torch.cat([CP.attend_local(xl[r], parts[r][0], e_all, k_all, m, s.topk, s.scale, ops)
                     for r in range(world)], dim=1)
    C.sync_status()
    assert [p[0].t0 for p in parts][1:] == [p[0].t1 for p in parts][:-1]
    assert torch.equal(e_all, e) and torch.equal(k_all, k)
    assert torch.equal(out, ref)
    # a few rows against the oracle, on the GPU's own selection
    rows = np.array([0, m - 1, parts[-1][0].t0, parts[-1][0].t0 + 1, L - 1])
    o_ref, _ = O.sparse_attention(f64(x["q"]), f64(e), idx.cpu().numpy(), s.scale, rows=rows)
    assert_close(f64(out)[:, rows], o_ref, what="context-parallel rows")
