"""GPU parity of decode-time incremental compression (cslc_decode_append).

Token by token, the append must build exactly the cache a prefill pass builds
from the same tokens: entries through csa_compress / hca_compress and
cslc_quantize_kv_mixed (bit-identical codes, RoPE halves and scales), indexer
keys through the D = 64 compressor (bit-identical), n_entries = floor(L / m).
Against the oracle: the dequantised cache within the FP8 tolerance of the
oracle's entries, keys within the bf16 tolerance.
"""

import numpy as np
import pytest
import torch

import oracle as O
from compressed_sparse_long_compress_b200 import workloads as W
from tests.helpers import REL_L2_FP8, assert_close, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def C(cuda_device):
    from compressed_sparse_long_compress_b200 import cslc
    return cslc


def _tokens(B, L, seed, keys):
    x = {"c": W.randn_bf16((B, L, 128), seed), "z": W.randn_bf16((B, L, 128), seed + 1)}
    if keys:
        x["kc"] = W.randn_bf16((B, L, 64), seed + 2)
        x["kz"] = W.randn_bf16((B, L, 64), seed + 3)
    return {k: v.cuda() for k, v in x.items()}


def _run_appends(C, x, lengths, offsets, m, overlap, n_max, bias, kbias):
    B = len(lengths)
    keys = "kc" in x
    st = C.AppendState(B, m, overlap, keys, "cuda")
    nope = torch.zeros(B, n_max, 64, dtype=torch.uint8, device="cuda")
    rope = torch.zeros(B, n_max, 64, dtype=torch.bfloat16, device="cuda")
    scale = torch.zeros(B, n_max, device="cuda")
    k_idx = torch.zeros(B, n_max, 64, dtype=torch.bfloat16, device="cuda") if keys else None
    n_entries = torch.zeros(B, dtype=torch.int32, device="cuda")
    steps = max(o + l for o, l in zip(offsets, lengths))
    ar = torch.arange(B, device="cuda")
    for t in range(steps):
        p = [t - o if 0 <= t - o < l else -1 for o, l in zip(offsets, lengths)]
        tok = torch.tensor([max(v, 0) for v in p], device="cuda")
        pos = torch.tensor(p, dtype=torch.int32, device="cuda")
        c, z = x["c"][ar, tok].contiguous(), x["z"][ar, tok].contiguous()
        kw = {}
        if keys:
            kw = dict(k_c=x["kc"][ar, tok].contiguous(), k_z=x["kz"][ar, tok].contiguous(), k_pos_bias=kbias,
                      k_idx=k_idx)
        C.decode_append(st, c, z, pos, bias, nope, rope, scale, n_entries, **kw)
    torch.cuda.synchronize()
    return nope, rope, scale, k_idx, n_entries


@pytest.mark.parametrize("m,overlap,keys,lengths,offsets", [
    (4, True, True, [203, 150, 3], [0, 5, 2]),     # CSA: ragged, late start, shorter than one window
    (128, False, False, [300, 257], [0, 1]),       # HCA: two entries, one ends one token into a window
    (2, True, True, [41], [0]),
])
def test_append_builds_the_prefill_cache(C, m, overlap, keys, lengths, offsets):
    B, L = len(lengths), max(lengths)
    x = _tokens(B, L, 500 + m, keys)
    W_ = 2 * m if overlap else m
    bias = W.randn_bf16((W_, 128), 510 + m, std=0.1).cuda()
    kbias = W.randn_bf16((W_, 64), 520 + m, std=0.1).cuda() if keys else None
    n_max = L // m + 1
    nope, rope, scale, k_idx, n_entries = _run_appends(C, x, lengths, offsets, m, overlap, n_max, bias, kbias)
    assert n_entries.tolist() == [l // m for l in lengths]
    comp = C.csa_compress if overlap else C.hca_compress
    kwm = {"m": m} if overlap else {"m_prime": m}
    for b, l in enumerate(lengths):
        n = l // m
        if n == 0:
            continue
        # the prefill path on the same tokens
        e = comp(x["c"][b:b + 1, :l].contiguous(), x["z"][b:b + 1, :l].contiguous(), bias, **kwm)
        pn, pr, ps = C.quantize_kv_mixed(e)
        assert torch.equal(nope[b, :n], pn[0]) and torch.equal(rope[b, :n], pr[0]) and torch.equal(scale[b, :n], ps[0])
        # the oracle
        e_ref = O.compress(f64(x["c"][b:b + 1, :l]), f64(x["z"][b:b + 1, :l]), f64(bias), m, overlap)
        hat = O.dequantize_kv_mixed(nope[b:b + 1, :n].cpu().numpy(), f64(rope[b:b + 1, :n]), scale[b:b + 1, :n].cpu().numpy())
        assert_close(hat, e_ref, rel=REL_L2_FP8, max_abs=0.1, what=f"appended entries seq {b}")   # e4m3: half a step is up to 1/16 of |x|
        if keys:
            kp = comp(x["kc"][b:b + 1, :l].contiguous(), x["kz"][b:b + 1, :l].contiguous(), kbias, **kwm)
            assert torch.equal(k_idx[b, :n], kp[0])
            k_ref = O.compress(f64(x["kc"][b:b + 1, :l]), f64(x["kz"][b:b + 1, :l]), f64(kbias), m, overlap)
            assert_close(f64(k_idx[b:b + 1, :n]), k_ref, what=f"appended keys seq {b}")


def test_append_beyond_capacity_is_dropped(C):
    m, L, n_max = 4, 40, 6
    x = _tokens(1, L, 560, True)
    bias = W.randn_bf16((8, 128), 561, std=0.1).cuda()
    kbias = W.randn_bf16((8, 64), 562, std=0.1).cuda()
    nope, rope, scale, k_idx, n_entries = _run_appends(C, x, [L], [0], m, True, n_max, bias, kbias)
    assert n_entries.tolist() == [n_max]
    e = C.csa_compress(x["c"], x["z"], bias, m=m)[:, :n_max].contiguous()
    pn, _, ps = C.quantize_kv_mixed(e)
    assert torch.equal(nope[0], pn[0]) and torch.equal(scale[0], ps[0])


def test_compress_64_dim_keys_matches_oracle(C):
    x = _tokens(2, 1001, 570, True)
    for m, overlap in ((4, True), (128, False)):
        bias = W.randn_bf16((2 * m if overlap else m, 64), 571, std=0.1).cuda()
        comp = C.csa_compress if overlap else C.hca_compress
        got = comp(x["kc"], x["kz"], bias, **({"m": m} if overlap else {"m_prime": m}))
        ref = O.compress(f64(x["kc"]), f64(x["kz"]), f64(bias), m, overlap)
        assert got.shape == (2, 1001 // m, 64)
        assert_close(f64(got), ref, what=f"64-dim compress m={m}")
        assert np.mean(f64(got) == ref) > 0.98
