"""The C++ float64 oracle (libcslc_oracle.so) behind the numpy oracle's API.

TEST INFRASTRUCTURE ONLY, like the numpy oracle: only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline legs of ``bench.py`` may use
it. Every function here only converts arrays and forwards them to the C++
library (``cslc_oracle.cpp``), which holds all the arithmetic; the names,
arguments and results are those of ``cslc_oracle.py``, so the same pins run
against both oracles. The library is built on first import when missing.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build_oracle

_LIB = ctypes.CDLL(build_oracle.build())

_D = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_I32 = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_I64 = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
_U8 = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_F32 = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_P = ctypes.c_void_p
_ll, _i, _d = ctypes.c_longlong, ctypes.c_int, ctypes.c_double


def _sig(name, res, args):
    f = getattr(_LIB, name)
    f.restype = res
    f.argtypes = args
    return f


_round_bf16 = _sig("orc_round_bf16", None, [_D, _ll, _D])
_round_fp32 = _sig("orc_round_fp32", None, [_D, _ll, _D])
_n_visible = _sig("orc_n_visible", _ll, [_ll, _ll, _ll])
_window = _sig("orc_compression_window", _i, [_ll, _i, _i, _I64, _I32, _U8])
_weights = _sig("orc_compression_weights", None, [_D, _D, _i, _i, _D])
_compress = _sig("orc_compress", None, [_D, _D, _D, _P, _P, _i, _ll, _i, _i, _i, _i, _D])
_indexer = _sig("orc_indexer_scores", None, [_D, _D, _D, _i, _ll, _i, _i, _ll, _i, _ll, _P, _ll, _i, _D])
_topk_row = _sig("orc_topk_select_row", None, [_D, _ll, _i, _I32])
_topk = _sig("orc_topk_select", None, [_D, _i, _ll, _ll, _i, _i, _ll, _P, _I32])
_attend = _sig("orc_attend", None, [_D, _D, _i, _i, _ll, _d, _D, _D])
_sparse = _sig("orc_sparse_attention", None, [_D, _D, _I32, _i, _ll, _i, _i, _ll, _i, _d, _P, _ll, _D, _D])
_dense = _sig("orc_dense_causal_attention", None, [_D, _D, _i, _ll, _i, _i, _ll, _i, _d, _ll, _P, _ll, _i, _D, _D])
_e4m3_dec = _sig("orc_e4m3_decode", None, [_U8, _ll, _D])
_e4m3_enc = _sig("orc_e4m3_encode", None, [_D, _ll, _U8])
_quant = _sig("orc_quantize_kv_mixed", None, [_D, _ll, _U8, _D, _F32])
_dequant = _sig("orc_dequantize_kv_mixed", None, [_U8, _D, _F32, _ll, _D])
_dec_scores = _sig("orc_decode_indexer_scores", None, [_D, _D, _D, _I64, _i, _ll, _i, _i, _D])
_dec_csa = _sig("orc_decode_csa_layer", None, [_D, _D, _D, _I64, _i, _i, _i, _ll, _i, _d, _D, _I32])
_dec_hca = _sig("orc_decode_hca_layer", None, [_D, _D, _I64, _i, _i, _i, _ll, _d, _D])
_project = _sig("orc_project", None, [_D, _D, _ll, _i, _i, _D])
_threads = _sig("orc_threads", _i, [])
_set_threads = _sig("orc_set_threads", None, [_i])

E4M3_MAX = 448.0


def threads() -> int:
    """OpenMP threads the oracle's parallel loops use."""
    return int(_threads())


def set_threads(n: int) -> None:
    _set_threads(int(n))


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _rows_ptr(rows):
    if rows is None:
        return None, None
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, r.ctypes.data_as(_P)


def round_bf16(x):
    x = _f64(x)
    out = np.empty_like(x)
    _round_bf16(x.reshape(-1), x.size, out.reshape(-1))
    return out


def round_fp32(x):
    x = _f64(x)
    out = np.empty_like(x)
    _round_fp32(x.reshape(-1), x.size, out.reshape(-1))
    return out


def n_compressed(L: int, m: int) -> int:
    return L // m


def n_visible(p: int, m: int, n_c: int) -> int:
    return int(_n_visible(int(p), int(m), int(n_c)))


def compression_window(i: int, m: int, overlap: bool):
    tokens = np.zeros(2 * m, dtype=np.int64)
    slots = np.zeros(2 * m, dtype=np.int32)
    prev = np.zeros(2 * m, dtype=np.uint8)
    n = _window(int(i), int(m), int(bool(overlap)), tokens, slots, prev)
    return tokens[:n], slots[:n].astype(np.int64), prev[:n].astype(bool)


def compression_weights(zw, bias_rows):
    zw = _f64(zw)
    bias_rows = _f64(bias_rows)
    W, D = zw.shape[-2:]
    flat = zw.reshape(-1, W, D)
    out = np.empty_like(flat)
    for j in range(flat.shape[0]):
        _weights(np.ascontiguousarray(flat[j]), bias_rows, W, D, out[j])
    return out.reshape(zw.shape)


def compress(c, z, pos_bias, m: int, overlap: bool, c_b=None, z_b=None, round_output: bool = True):
    c, z, pos_bias = _f64(c), _f64(z), _f64(pos_bias)
    B, L, D = c.shape
    out = np.zeros((B, L // m, D))
    cb = None if c_b is None else _f64(c_b)
    zb = None if z_b is None else _f64(z_b)
    _compress(c, z, pos_bias, None if cb is None else cb.ctypes.data_as(_P), None if zb is None else zb.ctypes.data_as(_P),
              B, L, D, m, int(bool(overlap)), int(bool(round_output)), out)
    return out


def project(h, W):
    h, W = _f64(h), _f64(W)
    B, L, dm = h.shape
    D = W.shape[0]
    out = np.empty((B, L, D))
    _project(h.reshape(B * L, dm), W, B * L, dm, D, out.reshape(B * L, D))
    return out


def compressor_front_end(h, W, pos_bias, m: int, overlap: bool, round_output: bool = True):
    W = _f64(W)
    if overlap:
        return compress(project(h, W[0]), project(h, W[2]), pos_bias, m, True,
                        c_b=project(h, W[1]), z_b=project(h, W[3]), round_output=round_output)
    return compress(project(h, W[0]), project(h, W[1]), pos_bias, m, False, round_output=round_output)


def csa_compress(c, z, pos_bias, m: int = 4, c_b=None, z_b=None, round_output=True):
    return compress(c, z, pos_bias, m, True, c_b, z_b, round_output)


def hca_compress(c, z, pos_bias, m_prime: int = 128, round_output=True):
    return compress(c, z, pos_bias, m_prime, False, None, None, round_output)


def indexer_scores(q_idx, w, k_idx, m: int, q_pos0: int = 0, rows=None, compact: bool = False):
    """As the numpy oracle's; with compact=True, q_idx and w hold only the
    requested rows (row r's data at index r, its position rows[r])."""
    q_idx, w, k_idx = _f64(q_idx), _f64(w), _f64(k_idx)
    B, L, HI, dI = q_idx.shape
    n_c = k_idx.shape[1]
    r, rp = _rows_ptr(rows)
    n_rows = L if r is None else len(r)
    out = np.empty((B, n_rows, n_c))
    _indexer(q_idx, w, k_idx, B, L, HI, dI, n_c, m, int(q_pos0), rp, n_rows, int(bool(compact)), out)
    return out


def topk_select_row(s_row, n_vis: int, k: int):
    s = _f64(s_row)
    out = np.empty(k, dtype=np.int32)
    _topk_row(s, int(n_vis), int(k), out)
    return out


def topk_select(scores, m: int, k: int, q_pos0: int = 0, rows=None):
    scores = _f64(scores)
    B, R, n_c = scores.shape
    if rows is None:
        rows = np.arange(R)
    r, rp = _rows_ptr(rows)
    out = np.empty((B, R, k), dtype=np.int32)
    _topk(scores, B, R, n_c, m, k, int(q_pos0), rp, out)
    return out


def attend(qv, kv, scale: float):
    qv, kv = _f64(qv), _f64(kv)
    H, D = qv.shape
    n = kv.shape[0]
    o = np.empty((H, D))
    lse = np.empty(H)
    _attend(qv, kv if n else np.zeros((1, D)), H, D, n, float(scale), o, lse)
    return o, lse


def sparse_attention(q, e, idx, scale: float, rows=None):
    q, e = _f64(q), _f64(e)
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    B, L, H, D = q.shape
    n_c = e.shape[1]
    r, rp = _rows_ptr(rows)
    n_rows = L if r is None else len(r)
    o = np.empty((B, n_rows, H, D))
    lse = np.empty((B, n_rows, H))
    _sparse(q, e if n_c else np.zeros((B, 1, D)), idx, B, L, H, D, n_c, idx.shape[2], float(scale), rp, n_rows, o, lse)
    return o, lse


def dense_causal_attention(q, e, m: int, scale: float, q_pos0: int = 0, rows=None, compact: bool = False):
    """As the numpy oracle's; with compact=True, q holds only the requested
    rows (row r's data at index r, its position rows[r])."""
    q, e = _f64(q), _f64(e)
    B, L, H, D = q.shape
    n_c = e.shape[1]
    r, rp = _rows_ptr(rows)
    n_rows = L if r is None else len(r)
    o = np.empty((B, n_rows, H, D))
    lse = np.empty((B, n_rows, H))
    _dense(q, e if n_c else np.zeros((B, 1, D)), B, L, H, D, n_c, m, float(scale), int(q_pos0), rp, n_rows,
           int(bool(compact)), o, lse)
    return o, lse


def e4m3_decode(codes):
    codes = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
    out = np.empty(codes.shape)
    _e4m3_dec(codes.reshape(-1), codes.size, out.reshape(-1))
    return out


def e4m3_encode(x):
    x = _f64(x)
    out = np.empty(x.shape, dtype=np.uint8)
    _e4m3_enc(x.reshape(-1), x.size, out.reshape(-1))
    return out


def quantize_kv_mixed(e):
    e = _f64(e)
    lead = e.shape[:-1]
    n = int(np.prod(lead)) if lead else 1
    codes = np.empty(lead + (64,), dtype=np.uint8)
    rope = np.empty(lead + (64,))
    scale = np.empty(lead, dtype=np.float32)
    _quant(e.reshape(n, 128), n, codes.reshape(n, 64), rope.reshape(n, 64), scale.reshape(n))
    return codes, rope, scale


def dequantize_kv_mixed(nope_codes, rope, scale):
    codes = np.ascontiguousarray(np.asarray(nope_codes, dtype=np.uint8))
    rope = _f64(rope)
    scale = np.ascontiguousarray(np.asarray(scale, dtype=np.float32))
    lead = codes.shape[:-1]
    n = int(np.prod(lead)) if lead else 1
    out = np.empty(lead + (128,))
    _dequant(codes.reshape(n, 64), rope.reshape(n, 64), scale.reshape(n), n, out.reshape(n, 128))
    return out


def decode_indexer_scores(q_idx, w, k_idx, n_entries):
    q_idx, w, k_idx = _f64(q_idx), _f64(w), _f64(k_idx)
    B, N, dI = k_idx.shape
    HI = q_idx.shape[1]
    n = np.ascontiguousarray(np.asarray(n_entries, dtype=np.int64))
    out = np.empty((B, N))
    _dec_scores(q_idx, w, k_idx, n, B, N, HI, dI, out)
    return out


def decode_csa_layer(q, q_idx, w, k_idx, kv_hat, n_entries, topk: int, scale: float, scores=None):
    if scores is None:
        scores = decode_indexer_scores(q_idx, w, k_idx, n_entries)
    q, kv_hat, sc = _f64(q), _f64(kv_hat), _f64(scores)
    B, H, D = q.shape
    N = kv_hat.shape[1]
    n = np.ascontiguousarray(np.asarray(n_entries, dtype=np.int64))
    o = np.empty((B, H, D))
    idx = np.empty((B, topk), dtype=np.int32)
    _dec_csa(q, sc, kv_hat if N else np.zeros((B, 1, D)), n, B, H, D, N, topk, float(scale), o, idx)
    return o, idx, scores


def decode_hca_layer(q, kv_hat, n_entries, scale: float):
    q, kv_hat = _f64(q), _f64(kv_hat)
    B, H, D = q.shape
    N = kv_hat.shape[1]
    n = np.ascontiguousarray(np.asarray(n_entries, dtype=np.int64))
    o = np.empty((B, H, D))
    _dec_hca(q, kv_hat if N else np.zeros((B, 1, D)), n, B, H, D, N, float(scale), o)
    return o
