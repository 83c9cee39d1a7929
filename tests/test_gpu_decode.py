"""GPU parity of the decode path over the mixed BF16-RoPE / FP8 KV layout
(indexer scores, exact top-k, sparse / dense split-K attention, the fused
multi-layer step) against the CPU oracle, through the C ABI."""

import math

import numpy as np
import pytest
import torch

import oracle as O
from compressed_sparse_long_compress_b200 import workloads as W
from tests.helpers import REL_L2_FP8, assert_close, check_selection, f64, max_differing

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def C(cuda_device):
    from compressed_sparse_long_compress_b200 import cslc
    return cslc


def dev(t):
    return t.to("cuda:0")


@pytest.mark.parametrize("B,n_max,n_list,topk,ties", [
    (5, 70000, [70000, 1000, 1024, 0, 5], 1024, False),
    (3, 262144, [262144, 200000, 131072], 1024, True),
    (2, 9000, [9000, 8999], 2048, True),
    (4, 5000, [5000, 4000, 17, 4999], 7, False),
])
def test_decode_topk_on_given_scores_bitexact(C, B, n_max, n_list, topk, ties):
    s = W.rand_f32((B, n_max), seed=900 + n_max)
    if ties:
        s = torch.round(s * 4) / 4
    n = torch.tensor(n_list, dtype=torch.int32)
    idx = C.decode_topk(dev(s), dev(n), topk).cpu().numpy()
    for b in range(B):
        assert np.array_equal(idx[b], O.topk_select_row(f64(s)[b], n_list[b], topk)), b


def test_decode_topk_degenerate_all_equal(C):
    s = torch.zeros(2, 50000)
    n = torch.tensor([50000, 30000], dtype=torch.int32)
    idx = C.decode_topk(dev(s), dev(n), 1024).cpu().numpy()
    assert np.array_equal(idx, np.tile(np.arange(1024, dtype=np.int32), (2, 1)))


def _layer_inputs(d, layer, wid, n_list):
    x = W.decode_layer_inputs(d, layer, wid)
    return x, torch.tensor(n_list, dtype=torch.int32)


def _oracle_kv(x):
    codes, rope, scale = O.quantize_kv_mixed(f64(x["kv"]))
    return O.dequantize_kv_mixed(codes, rope, scale)


def _gpu_layer(C, d, kind, x, n, topk, want_scores=True):
    nope, rope, sc = C.quantize_kv_mixed(dev(x["kv"]))
    B = d.B
    kw = {}
    if kind == "csa":
        kw = dict(q_idx=dev(x["q_idx"]), w=dev(x["w"]), k_idx=dev(x["k_idx"]), topk=topk,
                  idx_out=torch.empty(B, topk, dtype=torch.int32, device="cuda:0"),
                  scores_out=torch.empty(B, x["kv"].shape[1], device="cuda:0") if want_scores else None)
    return C.DecodeLayer(kind, dev(x["q"]), nope, rope, sc, dev(n), d.scale, **kw)


def _check_csa_layer(layer, x, n_list, topk, kv_hat, seqs=None):
    """Scores within max-abs 2e-2 / rel-L2 1e-2 of the oracle; the selection
    exactly the top-k of the kernel's own scores; the oracle's own selection
    identical but for verified near-ties (at most 1 % of the sequences, at
    least one); the output equal (FP8 tolerance) to the oracle's attention over
    the selection the kernel made, for every sequence."""
    B = len(n_list)
    seqs = range(B) if seqs is None else seqs
    sc = f64(layer.scores_out)
    idx = layer.idx_out.cpu().numpy()
    out = f64(layer.out)
    s_ref = O.decode_indexer_scores(f64(x["q_idx"]), f64(x["w"]), f64(x["k_idx"]), n_list)
    n_diff = 0
    for b in seqs:
        n = n_list[b]
        assert_close(sc[b, :n], s_ref[b, :n], what=f"scores seq {b}")
        # the selection is exactly the top-k of the kernel's own scores
        assert np.array_equal(idx[b], O.topk_select_row(sc[b], n, topk)), b
        ref_idx = O.topk_select_row(s_ref[b], n, topk)
        n_diff += not check_selection(idx[b], ref_idx, s_ref[b], n, topk)
        sel = idx[b][idx[b] >= 0]
        o_ref, _ = O.attend(f64(x["q"])[b], kv_hat[b, sel], layer.scale)
        assert_close(out[b], O.round_bf16(o_ref), rel=REL_L2_FP8, what=f"csa out seq {b}")
    assert n_diff <= max_differing(len(list(seqs))), n_diff


def test_decode_small_csa_and_hca_layers(C):
    d = W.DecodeShape(B=3, H=64, kinds=("csa", "hca"), n_entries=(3000, 3000), topk=512)
    n_list = [3000, 1500, 400]
    xc, n = _layer_inputs(d, 0, 41, n_list)
    xh, _ = _layer_inputs(d, 1, 41, n_list)
    lc = _gpu_layer(C, d, "csa", xc, n, 512)
    lh = _gpu_layer(C, d, "hca", xh, n, 512)
    C.decode_step([lc, lh], HI=8)
    torch.cuda.synchronize()
    _check_csa_layer(lc, xc, n_list, 512, _oracle_kv(xc))
    o_ref = O.decode_hca_layer(f64(xh["q"]), _oracle_kv(xh), n_list, d.scale)
    assert_close(f64(lh.out), o_ref, rel=REL_L2_FP8, what="hca out")


@pytest.mark.parametrize("H,n_max,want_scores,ties", [(64, 6000, True, False), (128, 5003, True, True),
                                                     (16, 4100, False, False)])
def test_decode_csa_large_batch(C, H, n_max, want_scores, ties):
    """A batch large enough for the one-launch cluster tail (select, order,
    attention and combine of a CSA layer, one cluster per sequence), with
    contexts of 0, 1, fewer than k, exactly k, k + 1 and up to n_max entries
    (n_max = 5003 takes the unvectorised score scan), tied scores from
    duplicated keys, and the scores kept in the library's workspace."""
    B, topk = 40, 1024
    d = W.DecodeShape(B=B, H=H, kinds=("csa",), n_entries=(n_max,), topk=topk)
    base = [0, 1, 300, topk, topk + 1, 2000, n_max - 1, n_max]
    n_list = [base[b % len(base)] if b < 2 * len(base) else int(np.random.default_rng(b).integers(0, n_max + 1))
              for b in range(B)]
    x, n = _layer_inputs(d, 0, 47 + H, n_list)
    if ties:
        x["k_idx"][:, 100:400] = x["k_idx"][:, 0:300]
    lc = _gpu_layer(C, d, "csa", x, n, topk, want_scores=want_scores)
    C.decode_step([lc], HI=8)
    torch.cuda.synchronize()
    if want_scores:
        _check_csa_layer(lc, x, n_list, topk, _oracle_kv(x))
    else:
        idx = lc.idx_out.cpu().numpy()
        s_ref = O.decode_indexer_scores(f64(x["q_idx"]), f64(x["w"]), f64(x["k_idx"]), n_list)
        kv_hat, out = _oracle_kv(x), f64(lc.out)
        n_diff = 0
        for b in range(B):
            assert np.sum(idx[b] >= 0) == min(topk, n_list[b]) and np.all(idx[b][idx[b] >= 0] < n_list[b])
            sel = idx[b][idx[b] >= 0]
            assert np.all(np.diff(sel) > 0)
            n_diff += not check_selection(idx[b], O.topk_select_row(s_ref[b], n_list[b], topk), s_ref[b],
                                          n_list[b], topk)
            o_ref, _ = O.attend(f64(x["q"])[b], kv_hat[b, sel], d.scale)
            assert_close(out[b], O.round_bf16(o_ref), rel=REL_L2_FP8, what=f"csa out seq {b}")
        assert n_diff <= max_differing(B), n_diff


def test_decode_csa_topk_covering_everything_equals_dense(C):
    d = W.DecodeShape(B=2, H=16, kinds=("csa",), n_entries=(700,), topk=2048)
    n_list = [700, 650]
    x, n = _layer_inputs(d, 0, 43, n_list)
    lc = _gpu_layer(C, d, "csa", x, n, 2048)
    C.decode_step([lc], HI=8)
    torch.cuda.synchronize()
    idx = lc.idx_out.cpu().numpy()
    for b in range(2):
        assert np.array_equal(idx[b, : n_list[b]], np.arange(n_list[b])) and np.all(idx[b, n_list[b]:] == -1)
    o_ref = O.decode_hca_layer(f64(x["q"]), _oracle_kv(x), n_list, d.scale)
    assert_close(f64(lc.out), o_ref, rel=REL_L2_FP8, what="csa(all) out")


def test_decode_hca_zero_and_tiny_contexts(C):
    d = W.DecodeShape(B=4, H=128, kinds=("hca",), n_entries=(300,))
    n_list = [0, 1, 257, 300]
    x, n = _layer_inputs(d, 0, 44, n_list)
    lh = _gpu_layer(C, d, "hca", x, n, 1)
    C.decode_step([lh], HI=8)
    torch.cuda.synchronize()
    o_ref = O.decode_hca_layer(f64(x["q"]), _oracle_kv(x), n_list, d.scale)
    assert np.all(f64(lh.out)[0] == 0)
    assert_close(f64(lh.out), o_ref, rel=REL_L2_FP8, what="hca out")


def test_decode_hca_several_chunks_per_cta(C):
    # 4 x 157 chunks of 128 entries -> 3 chunks per attention CTA (384 entries
    # per split): a full context, an empty one, one that ends one entry into a
    # split's first chunk, and a ragged one
    d = W.DecodeShape(B=4, H=64, kinds=("hca",), n_entries=(20000,))
    n_list = [20000, 0, 385, 12345]
    x, n = _layer_inputs(d, 0, 46, n_list)
    lh = _gpu_layer(C, d, "hca", x, n, 1)
    C.decode_step([lh], HI=8)
    torch.cuda.synchronize()
    o_ref = O.decode_hca_layer(f64(x["q"]), _oracle_kv(x), n_list, d.scale)
    assert np.all(f64(lh.out)[1] == 0)
    assert_close(f64(lh.out), o_ref, rel=REL_L2_FP8, what="hca out")


def test_decode_step_is_deterministic(C):
    d = W.DecodeShape(B=2, H=64, kinds=("csa",), n_entries=(20000,))
    x, n = _layer_inputs(d, 0, 45, [20000, 12345])
    lc = _gpu_layer(C, d, "csa", x, n, 1024)
    step = C.DecodeStep([lc], HI=8)
    a = [t.clone() for t in step()] + [lc.idx_out.clone()]
    b = [t.clone() for t in step()] + [lc.idx_out.clone()]
    torch.cuda.synchronize()
    assert all(torch.equal(u, v) for u, v in zip(a, b))


@pytest.mark.parametrize("name", ["csa_decode", "hybrid_decode"])
def test_decode_full_size_sampled(C, name):
    wl = W.WORKLOADS[name]
    d = wl.decode
    layers, xs = [], []
    for li, kind in enumerate(d.kinds):
        x = W.decode_layer_inputs(d, li, wl.wid, device="cuda:0")
        n = torch.full((d.B,), d.n_entries[li], dtype=torch.int32, device="cuda:0")
        xs.append(x)
        layers.append(_gpu_layer(C, d, kind, x, n, d.topk))
    C.decode_step(layers, HI=d.HI)
    torch.cuda.synchronize()
    # every sequence of the hybrid step; 16 of the 64 of the CSA decode workload
    seqs = list(range(d.B)) if d.B <= 8 else [0, 1, 2, 3, 4, 5, 6, 7, 17, 31, 40, 47, 55, 61, 62, 63]
    for li, kind in enumerate(d.kinds):
        x = {k: v[seqs] for k, v in xs[li].items()}
        n_list = [d.n_entries[li]] * len(seqs)
        kv_hat = _oracle_kv(x)
        if kind == "csa":
            sub = _Sub(layers[li], seqs)
            _check_csa_layer(sub, x, n_list, d.topk, kv_hat)
        else:
            o_ref = O.decode_hca_layer(f64(x["q"]), kv_hat, n_list, d.scale)
            assert_close(f64(layers[li].out[seqs]), o_ref, rel=REL_L2_FP8, what=f"{name} hca layer {li}")


class _Sub:
    """Rows `seqs` of a decode layer's outputs."""

    def __init__(self, layer, seqs):
        self.scores_out = layer.scores_out[seqs]
        self.idx_out = layer.idx_out[seqs]
        self.out = layer.out[seqs]
        self.scale = layer.scale
