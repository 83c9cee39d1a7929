"""Context-parallel CSA prefill host logic on CPU (gloo, world sizes 2 and 3).

Each rank runs compressed_sparse_long_compress_b200.context_parallel on its
token shard, with the oracle as the per-rank computation (the plumbing under
test is the sharding, the halo, the all-gather of entries and keys and the
q_pos0 offsets); the concatenated outputs must equal the single-process
oracle pipeline on the whole sequence exactly. No GPU is used.
"""

import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(L, m, seed):
    sys.path.insert(0, ROOT)
    from compressed_sparse_long_compress_b200 import workloads as W
    s = W.PrefillShape(B=1, L=L, H=4, m=m, HI=2, topk=16)
    x = W.prefill_inputs(s, wid=seed, with_indexer=True)
    x["kc"] = W.randn_bf16((1, L, 64), seed + 5)
    x["kz"] = W.randn_bf16((1, L, 64), seed + 6)
    x["k_pos_bias"] = W.randn_bf16((2 * m, 64), seed + 7, std=0.1)
    return {k: v.double() for k, v in x.items() if k != "k_idx"}, s


def _oracle_ops():
    import oracle as O
    from compressed_sparse_long_compress_b200.context_parallel import CspOps
    t = lambda a: torch.from_numpy(np.asarray(a))
    n = lambda a: a.double().numpy()
    return CspOps(
        compress=lambda c, z, bias, m: t(O.compress(n(c), n(z), n(bias), m, True)),
        indexer_topk=lambda qi, w, k, m, topk, q_pos0: t(
            O.topk_select(O.indexer_scores(n(qi), n(w), n(k), m, q_pos0), m, topk, q_pos0)),
        sparse_attn=lambda q, e, idx, scale: t(O.sparse_attention(n(q), n(e), idx.numpy(), scale)[0]),
    )


def _worker(rank, world, port, L, m, out):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        from compressed_sparse_long_compress_b200 import context_parallel as CP
        x, s = _inputs(L, m, 61)
        xl = CP.local_slices(x, L, m, world, rank)
        o, sh = CP.csa_prefill_cp(xl, L, m, s.topk, s.scale, _oracle_ops())
        out[rank] = (sh.t0, sh.t1, o.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,L,m", [(2, 203, 4), (3, 130, 4), (2, 64, 8)])
def test_context_parallel_equals_single_process(world, L, m):
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), L, m, out), nprocs=world, join=True)
    sys.path.insert(0, ROOT)
    import oracle as O
    x, s = _inputs(L, m, 61)
    n = lambda a: a.numpy()
    e = O.compress(n(x["c"]), n(x["z"]), n(x["pos_bias"]), m, True)
    k = O.compress(n(x["kc"]), n(x["kz"]), n(x["k_pos_bias"]), m, True)
    idx = O.topk_select(O.indexer_scores(n(x["q_idx"]), n(x["w"]), k, m), m, s.topk)
    ref, _ = O.sparse_attention(n(x["q"]), e, idx, s.scale)
    got = np.concatenate([out[r][2] for r in range(world)], axis=1)
    assert [out[r][0] for r in range(world)][0] == 0 and out[world - 1][1] == L
    assert all(out[r][1] == out[r + 1][0] for r in range(world - 1))   # shards tile the sequence
    assert np.array_equal(got, ref)


def test_shards_cover_whole_windows():
    sys.path.insert(0, ROOT)
    from compressed_sparse_long_compress_b200.context_parallel import shard_of
    for L, m, world in [(203, 4, 2), (65536, 4, 8), (1000, 128, 3), (5, 4, 4)]:
        sh = [shard_of(L, m, world, r) for r in range(world)]
        assert sh[0].t0 == 0 and sh[-1].t1 == L and sh[0].halo == 0
        assert sum(x.e1 - x.e0 for x in sh) == L // m
        for a, b in zip(sh, sh[1:]):
            assert a.t1 == b.t0 and a.e1 == b.e0 and a.t1 % m == 0
            assert b.halo == (m if b.t0 > 0 else 0)
