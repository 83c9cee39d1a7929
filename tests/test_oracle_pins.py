"""Pins of the CPU oracles to things other than themselves (CPU only).

Each test checks an oracle function against a closed form, a special case that
reduces to a library routine (torch float64 matmul / scaled_dot_product_attention
/ logsumexp / float8 casts), an invariant, or brute force on tiny inputs, so that
a dropped term, a wrong sign or index, or a transposed operand fails one of them.
"""

import itertools
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as NUMPY_ORACLE
from oracle import cpp_oracle as CPP_ORACLE

RNG = np.random.default_rng(12345)


@pytest.fixture(params=["numpy", "cpp"])
def O(request):
    """Every pin runs against both oracles: the float64 numpy one and the
    float64 C++ / OpenMP one (neither is pinned by the other)."""
    return NUMPY_ORACLE if request.param == "numpy" else CPP_ORACLE


def bf16_values(shape, std=1.0, rng=RNG):
    x = torch.from_numpy(rng.standard_normal(shape) * std).float().to(torch.bfloat16)
    return x.double().numpy()


# ---------------------------------------------------------------- rounding ---

def test_round_bf16_matches_torch_cast_for_float32_inputs(O):
    x = np.concatenate([
        RNG.standard_normal(20000) * 10.0 ** RNG.integers(-30, 30, 20000),
        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 2.0 ** -130, 3.3e38, 3.4e38]),
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    got = O.round_bf16(x.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_round_bf16_ties_to_even_closed_form(O):
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties to the even mantissa (1.0)
    assert O.round_bf16(np.array([1 + 2 ** -8]))[0] == 1.0
    assert O.round_bf16(np.array([1 + 3 * 2 ** -8]))[0] == 1 + 2 ** -6
    assert np.isinf(O.round_bf16(np.array([3.5e38]))[0])


# ---------------------------------------------------------------- geometry ---

def test_visibility_closed_form(O):
    # an entry is visible once its whole window has ended: (i+1)m - 1 <= p
    m, n_c = 4, 10
    assert [O.n_visible(p, m, n_c) for p in range(0, 12)] == [0, 0, 0, 1, 1, 1, 1, 2, 2, 2, 2, 3]
    assert O.n_visible(10_000, m, n_c) == n_c
    assert O.n_visible(-1, m, n_c) == 0
    # brute force: count entries whose last window token is <= p
    for p in range(0, 60):
        brute = sum(1 for i in range(n_c) if (i + 1) * m - 1 <= p)
        assert O.n_visible(p, m, n_c) == brute


def test_window_membership(O):
    t, s, prev = O.compression_window(0, 4, True)
    assert list(t) == [0, 1, 2, 3] and list(s) == [4, 5, 6, 7] and not prev.any()
    t, s, prev = O.compression_window(3, 4, True)
    assert list(t) == list(range(8, 16)) and list(s) == list(range(8))
    assert list(prev) == [True] * 4 + [False] * 4
    t, s, prev = O.compression_window(2, 128, False)
    assert list(t) == list(range(256, 384)) and list(s) == list(range(128))


# ------------------------------------------------------------- compressor ---

def test_compression_weights_sum_to_one(O):
    zw = RNG.standard_normal((3, 8, 16)) * 5
    bias = RNG.standard_normal((8, 16))
    w = O.compression_weights(zw, bias)
    assert np.all(w >= 0)
    assert np.max(np.abs(w.sum(axis=-2) - 1.0)) < 1e-12


@pytest.mark.parametrize("m,overlap", [(4, True), (128, False), (2, True), (3, False)])
def test_constant_input_stays_constant(O, m, overlap):
    B, L, D = 2, 8 * m + 3, 16
    const = bf16_values((1, 1, D))
    c = np.broadcast_to(const, (B, L, D)).copy()
    z = bf16_values((B, L, D))
    bias = bf16_values((2 * m if overlap else m, D), std=0.1)
    e = O.compress(c, z, bias, m, overlap)
    np.testing.assert_array_equal(e, np.broadcast_to(const, e.shape))


def test_output_inside_window_range(O):
    m, B, L, D = 4, 1, 64, 32
    c, z = bf16_values((B, L, D)), bf16_values((B, L, D)) * 3
    bias = bf16_values((2 * m, D), std=0.1)
    e = O.compress(c, z, bias, m, True, round_output=False)
    for i in range(L // m):
        toks, _, _ = O.compression_window(i, m, True)
        lo, hi = c[:, toks].min(axis=1), c[:, toks].max(axis=1)
        assert np.all(e[:, i] >= lo - 1e-12) and np.all(e[:, i] <= hi + 1e-12)


def test_zero_logits_give_window_mean_csa(O):
    # z = 0, bias = 0: every weight is 1/|window| -> plain mean of the window's c
    m, B, L, D = 4, 2, 40, 8
    c = bf16_values((B, L, D))
    z = np.zeros((B, L, D))
    e = O.compress(c, z, np.zeros((2 * m, D)), m, True, round_output=False)
    np.testing.assert_allclose(e[:, 0], c[:, 0:4].mean(axis=1), rtol=0, atol=1e-14)
    for i in range(1, L // m):
        np.testing.assert_allclose(e[:, i], c[:, (i - 1) * m:(i + 1) * m].mean(axis=1), atol=1e-14)


def test_zero_logits_give_window_mean_hca(O):
    m, B, L, D = 128, 1, 128 * 3 + 5, 4
    c = bf16_values((B, L, D))
    e = O.compress(c, np.zeros((B, L, D)), np.zeros((m, D)), m, False, round_output=False)
    assert e.shape == (B, 3, D)
    for i in range(3):
        np.testing.assert_allclose(e[:, i], c[:, i * m:(i + 1) * m].mean(axis=1), atol=1e-14)


def test_hand_worked_example_csa_m2(O):
    # D = 1, c = 1..6, z = 0, bias = 0, m = 2 (windows of 2m = 4 tokens, entry 0 only C^a)
    c = np.arange(1.0, 7.0).reshape(1, 6, 1)
    e = O.compress(c, np.zeros_like(c), np.zeros((4, 1)), 2, True, round_output=False)
    np.testing.assert_allclose(e[0, :, 0], [1.5, 2.5, 4.5], atol=1e-15)


def test_hand_worked_example_log_weights(O):
    # softmax of log(a) is a / sum(a): HCA m'=3, c = 1..6, z = log([1,3,1, 2,2,4])
    c = np.arange(1.0, 7.0).reshape(1, 6, 1)
    z = np.log(np.array([1.0, 3.0, 1.0, 2.0, 2.0, 4.0])).reshape(1, 6, 1)
    e = O.compress(c, z, np.zeros((3, 1)), 3, False, round_output=False)
    np.testing.assert_allclose(e[0, :, 0], [(1 + 6 + 3) / 5, (8 + 10 + 24) / 8], atol=1e-14)


def test_log_weights_give_weighted_average(O):
    m, B, L, D = 4, 1, 32, 8
    c = bf16_values((B, L, D))
    a = RNG.uniform(0.1, 3.0, (B, L, D))
    bias_w = RNG.uniform(0.5, 2.0, (2 * m, D))
    e = O.compress(c, np.log(a), np.log(bias_w), m, True, round_output=False)
    for i in range(L // m):
        toks, slots, _ = O.compression_window(i, m, True)
        wts = a[:, toks] * bias_w[slots][None]
        ref = (wts * c[:, toks]).sum(axis=1) / wts.sum(axis=1)
        np.testing.assert_allclose(e[:, i], ref, rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("overlap,m", [(True, 4), (False, 8)])
def test_spike_selects_the_token(O, overlap, m):
    # a huge logit on token t, channel j makes every window holding t output c_t[j]
    B, L, D = 1, 8 * m, 4
    c = bf16_values((B, L, D))
    for t in [0, m - 1, m, 3 * m + 1, L - 1]:
        z = np.zeros((B, L, D))
        z[0, t, 1] = 80.0
        e = O.compress(c, z, np.zeros((2 * m if overlap else m, D)), m, overlap, round_output=False)
        holders = {t // m} | ({t // m + 1} if overlap and t // m + 1 < L // m else set())
        for i in range(L // m):
            if i in holders:
                assert abs(e[0, i, 1] - c[0, t, 1]) < 1e-20
            else:
                toks, _, _ = O.compression_window(i, m, overlap)
                np.testing.assert_allclose(e[0, i, 1], c[0, toks, 1].mean(), atol=1e-14)


def test_positional_bias_slots(O):
    # a huge bias on slot s picks the token in that slot: C^b slots 0..m-1, C^a m..2m-1
    m, B, L, D = 4, 1, 24, 2
    c = bf16_values((B, L, D))
    for s in range(2 * m):
        bias = np.zeros((2 * m, D))
        bias[s] = 80.0
        e = O.compress(c, np.zeros((B, L, D)), bias, m, True, round_output=False)
        for i in range(L // m):
            if i == 0 and s < m:      # no C^b for the first entry: uniform over C^a
                np.testing.assert_allclose(e[0, 0], c[0, 0:m].mean(axis=0), atol=1e-14)
                continue
            tok = (i - 1) * m + s
            np.testing.assert_allclose(e[0, i], c[0, tok], atol=1e-20)


def test_separate_prev_stream(O):
    m, B, L, D = 4, 1, 20, 4
    c, cb = bf16_values((B, L, D)), bf16_values((B, L, D))
    zero = np.zeros((B, L, D))
    e = O.compress(c, zero, np.zeros((2 * m, D)), m, True, c_b=cb, z_b=zero, round_output=False)
    np.testing.assert_allclose(e[:, 0], c[:, 0:m].mean(axis=1), atol=1e-14)
    for i in range(1, L // m):
        ref = np.concatenate([cb[:, (i - 1) * m:i * m], c[:, i * m:(i + 1) * m]], axis=1).mean(axis=1)
        np.testing.assert_allclose(e[:, i], ref, atol=1e-14)


def test_m1_is_identity(O):
    B, L, D = 2, 37, 16
    c, z = bf16_values((B, L, D)), bf16_values((B, L, D))
    e = O.compress(c, z, bf16_values((1, D), std=0.1), 1, False)
    np.testing.assert_array_equal(e, c)


# ----------------------------------------------------------------- indexer ---

def test_indexer_single_head_is_relu_gemm(O):
    B, L, n_c, dI, m = 2, 40, 10, 64, 4
    q = bf16_values((B, L, 1, dI))
    k = bf16_values((B, n_c, dI))
    s = O.indexer_scores(q, np.ones((B, L, 1)), k, m)
    ref = torch.clamp(torch.from_numpy(q[:, :, 0]) @ torch.from_numpy(k).transpose(1, 2), min=0).numpy()
    for t in range(L):
        nv = O.n_visible(t, m, n_c)
        np.testing.assert_allclose(s[:, t, :nv], np.float32(ref[:, t, :nv]), rtol=1e-7, atol=1e-30)
        assert np.all(np.isneginf(s[:, t, nv:]))


def test_indexer_head_weighting(O):
    B, L, n_c, HI, dI, m = 1, 32, 8, 4, 64, 4
    q = bf16_values((B, L, HI, dI))
    k = bf16_values((B, n_c, dI))
    w = RNG.uniform(-1, 1, (B, L, HI))
    s = O.indexer_scores(q, w, k, m)
    qt = torch.from_numpy(q)
    kt = torch.from_numpy(k)
    per_head = torch.clamp(torch.einsum("blhd,bnd->blhn", qt, kt), min=0)
    ref = (per_head * torch.from_numpy(w)[..., None]).sum(dim=2).numpy()
    for t in range(L):
        nv = O.n_visible(t, m, n_c)
        np.testing.assert_allclose(s[:, t, :nv], ref[:, t, :nv], rtol=1e-6, atol=1e-6)


def test_indexer_hand_example(O):
    # q heads [1,0] and [0,1]; keys [2,-1] and [-3,4]; w = [0.5, 2]
    q = np.array([[1.0, 0.0], [0.0, 1.0]]).reshape(1, 1, 2, 2)
    k = np.array([[2.0, -1.0], [-3.0, 4.0]]).reshape(1, 2, 2)
    w = np.array([0.5, 2.0]).reshape(1, 1, 2)
    s = O.indexer_scores(q, w, k, m=1, q_pos0=5)
    np.testing.assert_array_equal(s[0, 0], [1.0, 8.0])


def test_indexer_q_pos0_shifts_visibility(O):
    B, L, n_c, HI, dI, m = 1, 16, 12, 2, 64, 4
    q, k = bf16_values((B, L, HI, dI)), bf16_values((B, n_c, dI))
    w = RNG.uniform(0, 1, (B, L, HI))
    s0 = O.indexer_scores(q, w, k, m, q_pos0=20)
    for t in range(L):
        assert np.isfinite(s0[0, t]).sum() == O.n_visible(20 + t, m, n_c)


# ------------------------------------------------------------------- top-k ---

def _dominance_topk(s, k):
    """Brute force: the unique k-subset whose every member beats every
    non-member under (score desc, index asc)."""
    n = len(s)
    beats = lambda a, b: (s[a] > s[b]) or (s[a] == s[b] and a < b)
    found = []
    for sub in itertools.combinations(range(n), k):
        rest = [j for j in range(n) if j not in sub]
        if all(beats(a, b) for a in sub for b in rest):
            found.append(sub)
    assert len(found) == 1
    return list(found[0])


def test_topk_brute_force_tiny(O):
    rng = np.random.default_rng(7)
    for trial in range(200):
        n = int(rng.integers(1, 10))
        k = int(rng.integers(1, 12))
        s = rng.integers(-3, 4, n).astype(np.float64)   # small ints: many ties
        got = O.topk_select_row(s, n, k)
        kk = min(k, n)
        assert list(got[:kk]) == _dominance_topk(s, kk)
        assert np.all(got[kk:] == -1)


def test_topk_hand_example_ties(O):
    s = np.array([3.0, 5.0, 5.0, 1.0, 5.0])
    assert list(O.topk_select_row(s, 5, 2)) == [1, 2]
    assert list(O.topk_select_row(s, 5, 4)) == [0, 1, 2, 4]
    assert list(O.topk_select_row(s, 3, 5)) == [0, 1, 2, -1, -1]
    assert list(O.topk_select_row(s, 0, 3)) == [-1, -1, -1]


def test_topk_invariant_under_monotone_map(O):
    rng = np.random.default_rng(8)
    s = rng.standard_normal(300)
    a = O.topk_select_row(s, 300, 37)
    b = O.topk_select_row(np.exp(s) * 3.0 + 1.0, 300, 37)
    assert np.array_equal(a, b)
    # top-k equals the k largest by a full descending sort when there are no ties
    ref = np.sort(np.argsort(-s, kind="stable")[:37])
    assert np.array_equal(a, ref)


def test_topk_ignores_invisible_tail(O):
    s = np.array([1.0, 2.0, 3.0, 100.0, 200.0])
    assert list(O.topk_select_row(s, 3, 2)) == [1, 2]


# --------------------------------------------------------------- attention ---

def _sdpa(q, k, v, mask, scale):
    return F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale)


def test_attend_matches_sdpa_and_logsumexp(O):
    H, D, n = 6, 32, 20
    q = bf16_values((H, D))
    kv = bf16_values((n, D))
    o, lse = O.attend(q, kv, 0.3)
    qt, kt = torch.from_numpy(q)[None], torch.from_numpy(kv)[None]
    ref = _sdpa(qt, kt, kt, None, 0.3)[0].numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, torch.logsumexp(0.3 * qt[0] @ kt[0].T, dim=1).numpy(), rtol=1e-12)


def test_attend_hand_example(O):
    # scale 1, one head q = [1], entries [0] and [ln 3]: p = [1/4, 3/4]
    o, lse = O.attend(np.array([[1.0]]), np.array([[0.0], [math.log(3)]]), 1.0)
    assert abs(o[0, 0] - 0.75 * math.log(3)) < 1e-15
    assert abs(lse[0] - math.log(4)) < 1e-15
    o, lse = O.attend(np.ones((3, 4)), np.zeros((0, 4)), 1.0)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


def test_m1_hca_is_plain_causal_attention(O):
    # m = 1 without overlap: entries are the tokens' c, visibility is p >= i
    B, L, H, D = 1, 24, 4, 32
    c, z, q = bf16_values((B, L, D)), bf16_values((B, L, D)), bf16_values((B, L, H, D))
    e = O.compress(c, z, bf16_values((1, D), std=0.1), 1, False)
    o, _ = O.dense_causal_attention(q, e, 1, 1 / math.sqrt(D))
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(c)[:, None]
    mask = torch.ones(L, L, dtype=torch.bool).tril()
    ref = _sdpa(qt, kt, kt, mask, 1 / math.sqrt(D)).permute(0, 2, 1, 3).numpy()
    np.testing.assert_array_equal(o, O.round_bf16(ref))


def test_sparse_attention_matches_masked_sdpa(O):
    B, L, H, D, n_c, k = 1, 16, 4, 32, 12, 5
    q, e = bf16_values((B, L, H, D)), bf16_values((B, n_c, D))
    rng = np.random.default_rng(3)
    idx = np.full((B, L, k), -1, dtype=np.int32)
    for t in range(L):
        cnt = int(rng.integers(1, k + 1))
        idx[0, t, :cnt] = np.sort(rng.choice(n_c, cnt, replace=False))
    o, lse = O.sparse_attention(q, e, idx, 0.2)
    mask = torch.zeros(L, n_c, dtype=torch.bool)
    for t in range(L):
        mask[t, idx[0, t][idx[0, t] >= 0]] = True
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(e)[:, None]
    ref = _sdpa(qt, kt, kt, mask, 0.2).permute(0, 2, 1, 3).numpy()
    np.testing.assert_array_equal(o, O.round_bf16(ref))


def test_csa_with_k_covering_all_equals_dense(O):
    m, B, L, H, D, HI = 4, 1, 64, 4, 32, 2
    c, z, q = bf16_values((B, L, D)), bf16_values((B, L, D)), bf16_values((B, L, H, D))
    qi, k = bf16_values((B, L, HI, 64)), bf16_values((B, L // m, 64))
    w = RNG.uniform(0, 1, (B, L, HI))
    e = O.compress(c, z, bf16_values((2 * m, D), std=0.1), m, True)
    s = O.indexer_scores(qi, w, k, m)
    idx = O.topk_select(s, m, L // m)
    o1, l1 = O.sparse_attention(q, e, idx, 0.1)
    o2, l2 = O.dense_causal_attention(q, e, m, 0.1)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    # the first m-1 queries see nothing and output 0
    assert np.all(o1[:, : m - 1] == 0)


def test_causality_of_full_csa_pipeline(O):
    m, B, L, H, D, HI, k = 4, 1, 48, 2, 16, 2, 3
    g = np.random.default_rng(11)
    c, z, q = bf16_values((B, L, D), rng=g), bf16_values((B, L, D), rng=g), bf16_values((B, L, H, D), rng=g)
    qi, kk = bf16_values((B, L, HI, 64), rng=g), bf16_values((B, L // m, 64), rng=g)
    w = g.uniform(0, 1, (B, L, HI))
    bias = bf16_values((2 * m, D), std=0.1, rng=g)

    def run(c, z, q, qi, kk):
        e = O.compress(c, z, bias, m, True)
        idx = O.topk_select(O.indexer_scores(qi, w, kk, m), m, k)
        return O.sparse_attention(q, e, idx, 0.25)[0], idx

    o_ref, idx_ref = run(c, z, q, qi, kk)
    p = 21
    c2, z2, q2, qi2 = c.copy(), z.copy(), q.copy(), qi.copy()
    c2[:, p + 1:] += 5.0
    z2[:, p + 1:] -= 3.0
    q2[:, p + 1:] *= -1
    qi2[:, p + 1:] *= 2
    kk2 = kk.copy()
    kk2[:, O.n_visible(p, m, L // m):] += 7.0     # keys of entries not yet visible at p
    o2, idx2 = run(c2, z2, q2, qi2, kk2)
    np.testing.assert_array_equal(o2[:, : p + 1], o_ref[:, : p + 1])
    np.testing.assert_array_equal(idx2[:, : p + 1], idx_ref[:, : p + 1])
    for t in range(L):
        valid = idx_ref[0, t][idx_ref[0, t] >= 0]
        assert valid.size == min(k, O.n_visible(t, m, L // m))
        assert np.all(valid < O.n_visible(t, m, L // m))


# ---------------------------------------------------------------- FP8 e4m3 ---

def test_e4m3_decode_matches_torch_float8(O):
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = O.e4m3_decode(codes)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    np.testing.assert_array_equal(got[~np.isnan(got)], ref[~np.isnan(ref)])


def test_e4m3_spec_values(O):
    # OCP FP8 E4M3: max normal 448 = S.1111.110, min normal 2^-6, min subnormal 2^-9
    assert O.e4m3_decode(np.array([0x7E]))[0] == 448.0
    assert O.e4m3_decode(np.array([0x08]))[0] == 2.0 ** -6
    assert O.e4m3_decode(np.array([0x01]))[0] == 2.0 ** -9
    assert O.e4m3_decode(np.array([0x38]))[0] == 1.0
    assert O.e4m3_encode(np.array([1000.0, -1e9, 464.0, 0.0, -0.0]))[:5].tolist() == [0x7E, 0xFE, 0x7E, 0x00, 0x80]


def test_e4m3_roundtrip_and_rne_vs_torch(O):
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    np.testing.assert_array_equal(O.e4m3_encode(O.e4m3_decode(codes)), codes)
    x = np.concatenate([RNG.standard_normal(50000) * 10.0 ** RNG.uniform(-4, 2.6, 50000),
                        O.e4m3_decode(codes) * (1 + 2.0 ** -4)])      # exact midpoints
    x = x[np.abs(x) < 464.0].astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(O.e4m3_encode(x.astype(np.float64)), ref)


def test_e4m3_relative_error_bound(O):
    x = RNG.uniform(2.0 ** -6, 448.0, 100000) * np.sign(RNG.standard_normal(100000))
    r = O.e4m3_decode(O.e4m3_encode(x))
    assert np.max(np.abs(r - x) / np.abs(x)) <= 2.0 ** -4


def test_quantize_kv_mixed(O):
    e = bf16_values((3, 50, 128))
    e[1, 7] = 0.0
    codes, rope, scale = O.quantize_kv_mixed(e)
    assert codes.dtype == np.uint8 and scale.dtype == np.float32
    np.testing.assert_array_equal(rope, e[..., 64:])
    assert scale[1, 7] == 1.0 and np.all(codes[1, 7] == 0)
    hat = O.dequantize_kv_mixed(codes, rope, scale)
    amax = np.abs(e[..., :64]).max(axis=-1, keepdims=True)
    # the entry's largest element maps to +-448 exactly; every error <= half a step
    err = np.abs(hat[..., :64] - e[..., :64])
    assert np.all(err <= np.maximum(np.abs(e[..., :64]) * 2.0 ** -4, amax / 448 * 2.0 ** -10) + 1e-12)
    j = np.abs(e[..., :64]).argmax(axis=-1)
    top = np.take_along_axis(codes, j[..., None], axis=-1)[..., 0]
    mask = amax[..., 0] > 0
    assert np.all((top[mask] & 0x7F) == 0x7E)


# ------------------------------------------------- FP8 indexer operands ---
# (numpy oracle only: the FP8 indexer variant is not timed on the CPU, so the
# C++ oracle does not carry it)

def test_quantize_rows_e4m3_against_torch_cast():
    N = NUMPY_ORACLE
    x = bf16_values((5, 33, 64), std=3.0)
    x[2, 4] = 0.0
    codes, scale = N.quantize_rows_e4m3(x)
    assert codes.shape == x.shape and codes.dtype == np.uint8 and scale.dtype == np.float32
    xf = torch.from_numpy(x).float()
    amax = xf.abs().amax(dim=-1)
    s_ref = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))       # fp32 division
    np.testing.assert_array_equal(scale, s_ref.numpy())
    c_ref = (xf / s_ref[..., None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(codes, c_ref)
    assert scale[2, 4] == 1.0 and np.all(codes[2, 4] == 0)
    j = np.abs(x).argmax(axis=-1)
    top = np.take_along_axis(codes, j[..., None], axis=-1)[..., 0]
    assert np.all((top[np.abs(x).max(axis=-1) > 0] & 0x7F) == 0x7E)


def test_indexer_scores_fp8_single_head_is_relu_gemm_of_torch_decoded_values():
    N = NUMPY_ORACLE
    B, L, n_c, m = 2, 24, 9, 2
    q8, qs = N.quantize_rows_e4m3(bf16_values((B, L, 1, 64)))
    k8, ks = N.quantize_rows_e4m3(bf16_values((B, n_c, 64)))
    w = np.ones((B, L, 1))
    got = N.indexer_scores_fp8(q8, qs, w, k8, ks, m)
    qd = torch.from_numpy(q8).view(torch.float8_e4m3fn).double() * torch.from_numpy(qs).double()[..., None]
    kd = torch.from_numpy(k8).view(torch.float8_e4m3fn).double() * torch.from_numpy(ks).double()[..., None]
    ref = torch.relu(torch.matmul(qd[:, :, 0], kd.transpose(1, 2))).float().double().numpy()
    for t in range(L):
        nv = N.n_visible(t, m, n_c)
        np.testing.assert_array_equal(got[:, t, :nv], ref[:, t, :nv])
        assert np.all(got[:, t, nv:] == -np.inf)


def test_indexer_scores_fp8_scale_equivariance_and_bf16_closeness():
    N = NUMPY_ORACLE
    B, L, HI, n_c, m = 1, 40, 4, 12, 3
    q, k = bf16_values((B, L, HI, 64)), bf16_values((B, n_c, 64))
    w = RNG.uniform(0, 1, (B, L, HI))
    q8, qs = N.quantize_rows_e4m3(q)
    k8, ks = N.quantize_rows_e4m3(k)
    s1 = N.indexer_scores_fp8(q8, qs, w, k8, ks, m)
    s2 = N.indexer_scores_fp8(q8, qs, w, k8, 2 * ks, m)
    vis = np.isfinite(s1)
    np.testing.assert_array_equal(s2[vis], 2 * s1[vis])       # power-of-two scale: exact
    # within the e4m3 rounding of both operands of the bf16 path's scores
    ref = N.indexer_scores(q, w, k, m)
    bound = np.einsum("blh,blhd,bnd->bln", w, np.abs(q), np.abs(k)) * (2 * 2.0 ** -4 + 2.0 ** -8)
    assert np.all(np.abs(s1[vis] - ref[vis]) <= bound[vis] + 1e-6)


# ------------------------------------------------------------------ decode ---

def test_decode_layers_reduce_to_dense_and_library(O):
    B, N, H, D, HI = 3, 40, 4, 128, 2
    e = bf16_values((B, N, D))
    codes, rope, scale = O.quantize_kv_mixed(e)
    hat = O.dequantize_kv_mixed(codes, rope, scale)
    q = bf16_values((B, H, D))
    qi, k = bf16_values((B, HI, 64)), bf16_values((B, N, 64))
    w = RNG.uniform(0, 1, (B, HI))
    n_entries = np.array([40, 17, 1])
    o_h = O.decode_hca_layer(q, hat, n_entries, 0.1)
    for b in range(B):
        n = n_entries[b]
        qt, kt = torch.from_numpy(q[b])[None], torch.from_numpy(hat[b, :n])[None]
        np.testing.assert_array_equal(o_h[b], O.round_bf16(_sdpa(qt, kt, kt, None, 0.1)[0].numpy()))
    # top-k covering every entry equals the dense layer
    o_c, idx, s = O.decode_csa_layer(q, qi, w, k, hat, n_entries, 64, 0.1)
    np.testing.assert_array_equal(o_c, o_h)
    # scores: weighted ReLU of a float64 GEMM; entries past n_entries are -inf
    for b in range(B):
        n = n_entries[b]
        ref = (torch.from_numpy(w[b])[:, None] * torch.clamp(torch.from_numpy(qi[b]) @ torch.from_numpy(k[b, :n]).T, min=0)).sum(0)
        np.testing.assert_allclose(s[b, :n], ref.numpy(), rtol=1e-6)
        assert np.all(np.isneginf(s[b, n:]))
        assert np.array_equal(idx[b][: n], np.arange(n)) and np.all(idx[b][n:] == -1)
    # entries past n_entries do not influence anything
    hat2, k2 = hat.copy(), k.copy()
    hat2[1, 17:] += 9.0
    k2[1, 17:] -= 9.0
    o_c2, idx2, _ = O.decode_csa_layer(q, qi, w, k2, hat2, n_entries, 5, 0.1)
    o_c1, idx1, _ = O.decode_csa_layer(q, qi, w, k, hat, n_entries, 5, 0.1)
    np.testing.assert_array_equal(o_c1, o_c2)
    np.testing.assert_array_equal(idx1, idx2)


def test_cpp_compact_rows_match_full_rows():
    """The C++ oracle's compact-row mode (sampled rows' data packed, positions
    given) equals its full-tensor mode on the same rows."""
    q = bf16_values((1, 300, 16, 128))
    e = bf16_values((1, 75, 128), 0.4)
    qi = bf16_values((1, 300, 4, 64))
    w = np.abs(bf16_values((1, 300, 4)))
    k = bf16_values((1, 75, 64))
    rows = np.array([0, 3, 4, 77, 150, 299])
    o_full, l_full = CPP_ORACLE.dense_causal_attention(q, e, 4, 0.088, q_pos0=0, rows=rows)
    o_c, l_c = CPP_ORACLE.dense_causal_attention(q[:, rows], e, 4, 0.088, q_pos0=0, rows=rows, compact=True)
    assert np.array_equal(o_full, o_c) and np.array_equal(l_full, l_c)
    s_full = CPP_ORACLE.indexer_scores(qi, w, k, 4, rows=rows)
    s_c = CPP_ORACLE.indexer_scores(qi[:, rows], w[:, rows], k, 4, rows=rows, compact=True)
    assert np.array_equal(s_full, s_c)


# ------------------------------------------------- compressor front end ---

def test_projection_is_a_float64_matmul(O):
    h = bf16_values((2, 7, 96))
    W = bf16_values((5, 96))
    ref = torch.matmul(torch.from_numpy(h), torch.from_numpy(W).T).numpy()
    assert np.allclose(O.project(h, W), ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("overlap,m", [(True, 4), (False, 8)])
def test_front_end_with_identity_projections_is_compress(O, overlap, m):
    """With every W the identity (d_model = D) the front end is the compressor
    on the hidden states themselves (c = z = h, and c_b = z_b = h for CSA)."""
    D = 16
    h = bf16_values((1, 8 * m, D))
    eye = np.eye(D)
    W = np.stack([eye] * (4 if overlap else 2))
    bias = bf16_values((2 * m if overlap else m, D), 0.1)
    got = O.compressor_front_end(h, W, bias, m, overlap)
    assert np.array_equal(got, O.compress(h, h, bias, m, overlap))


def test_front_end_uses_each_projection_in_its_place(O):
    """W^{b,*} reach only the C^b half and W^{a,*} only the C^a half: with
    zero logit weights (uniform windows) the entry is the mean over the window
    of h W^{b,KV} on the C^b tokens and h W^{a,KV} on the C^a tokens."""
    m, D, dm = 4, 8, 24
    h = bf16_values((1, 6 * m, dm))
    Wa, Wb = bf16_values((D, dm)), bf16_values((D, dm))
    zero = np.zeros((D, dm))
    got = O.compressor_front_end(h, np.stack([Wa, Wb, zero, zero]), np.zeros((2 * m, D)), m, True,
                                 round_output=False)
    ca, cb = h[0] @ Wa.T, h[0] @ Wb.T
    for i in range(6):
        cur = ca[i * m:(i + 1) * m]
        ref = cur.mean(axis=0) if i == 0 else np.concatenate([cb[(i - 1) * m:i * m], cur]).mean(axis=0)
        assert np.allclose(got[0, i], ref, rtol=1e-12, atol=1e-12)
