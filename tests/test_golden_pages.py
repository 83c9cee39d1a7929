"""The oracle's geometry against the numbers the pages print (tests/golden)."""

import json
import os

import numpy as np
import pytest

import oracle as NUMPY_ORACLE
from oracle import cpp_oracle as CPP_ORACLE

@pytest.fixture(params=["numpy", "cpp"])
def O(request):
    return NUMPY_ORACLE if request.param == "numpy" else CPP_ORACLE


G = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_parameters.json")))


def test_csa_entry_count_at_1M(O):
    n = O.n_compressed(1 << 20, G["csa_m"]["value"])
    ref = G["csa_entries_at_1M_approx"]
    assert abs(n - ref["value"]) <= ref["tolerance_rel"] * ref["value"]
    assert n == 262144


def test_csa_window_size(O):
    toks, _, _ = O.compression_window(5, G["csa_m"]["value"], True)
    assert len(toks) == G["csa_window_tokens"]["value"]


def test_hca_reduction(O):
    mp = G["hca_m_prime"]["value"]
    assert (1 << 20) // O.n_compressed(1 << 20, mp) == G["hca_length_reduction"]["value"]


def test_mixed_kv_layout_sizes(O):
    e = np.ones((1, 1, 128))
    codes, rope, scale = O.quantize_kv_mixed(e)
    assert rope.shape[-1] == G["kv_rope_dims_bf16"]["value"]
    bytes_mixed = codes.shape[-1] * 1 + rope.shape[-1] * 2 + 4
    assert bytes_mixed == 196 and bytes_mixed / 256 < 1.0
