"""Python binding of libcslc (argument marshalling only).

Every function here forwards torch tensors' device pointers to the C ABI in
``include/cslc.h`` and raises ``CslcError`` on a non-OK status. All computation
happens in the library's CUDA kernels; there is no fallback path: if the
shared library is missing or fails to load, importing this module raises.
Calls run on torch's current CUDA stream.
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcslc.so")

c_int, c_size_t, c_float, c_void_p = ctypes.c_int, ctypes.c_size_t, ctypes.c_float, ctypes.c_void_p

STATUS = {0: "OK", 1: "ERR_NULL", 2: "ERR_SHAPE", 3: "ERR_ALIGN", 4: "ERR_UNSUPPORTED",
          5: "ERR_WORKSPACE", 6: "ERR_CUDA", 7: "ERR_DEVICE_CHECK"}

# every symbol include/cslc.h declares
ABI_SYMBOLS = [
    "cslc_abi_version", "cslc_last_error", "cslc_sync_status", "csa_compress", "hca_compress",
    "csa_indexer_topk_workspace_bytes", "csa_indexer_topk", "csa_topk", "csa_sparse_attn",
    "hca_dense_attn", "cslc_quantize_kv_mixed", "cslc_decode_workspace_bytes", "cslc_decode_step",
    "cslc_decode_topk_workspace_bytes", "cslc_decode_topk", "cslc_decode_topk_noalloc", "cslc_decode_append",
    "csa_compress_front_end", "hca_compress_front_end",
    "csa_indexer_topk_bf16_workspace_bytes", "csa_indexer_topk_bf16", "csa_topk_bf16",
    "cslc_testing_set_wait_limits", "cslc_quantize_rows_e4m3", "csa_indexer_topk_fp8",
]


class CslcError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class DecodeLayerC(ctypes.Structure):
    _fields_ = [
        ("kind", c_int), ("q", c_void_p), ("q_idx", c_void_p), ("w", c_void_p), ("k_idx", c_void_p),
        ("nope", c_void_p), ("rope", c_void_p), ("kv_scale", c_void_p), ("n_entries", c_void_p),
        ("n_max", c_int), ("topk", c_int), ("scale", c_float), ("out", c_void_p),
        ("idx_out", c_void_p), ("scores_out", c_void_p),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libcslc.so not built at {LIB_PATH}; run "
                          "`python -m compressed_sparse_long_compress_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P = c_void_p
    sig = {
        "cslc_abi_version": (c_int, []),
        "cslc_last_error": (ctypes.c_char_p, []),
        "cslc_sync_status": (c_int, [P]),
        "csa_compress": (c_int, [P, P, P, P, P, c_int, c_int, c_int, c_int, P, P]),
        "hca_compress": (c_int, [P, P, P, c_int, c_int, c_int, c_int, P, P]),
        "csa_indexer_topk_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int, c_int, c_int]),
        "csa_indexer_topk": (c_int, [P, P, P, c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                     P, P, P, c_size_t, P]),
        "csa_topk": (c_int, [P, c_int, c_int, c_int, c_int, c_int, c_int, P, P]),
        "csa_sparse_attn": (c_int, [P, P, P, c_int, c_int, c_int, c_int, c_int, c_int, c_float, P, P, P]),
        "hca_dense_attn": (c_int, [P, P, c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_float, P, P, P]),
        "cslc_quantize_kv_mixed": (c_int, [P, c_int, c_int, P, P, P, P]),
        "cslc_decode_workspace_bytes": (c_size_t, [ctypes.POINTER(DecodeLayerC), c_int, c_int, c_int, c_int]),
        "cslc_decode_step": (c_int, [ctypes.POINTER(DecodeLayerC), c_int, c_int, c_int, c_int, c_int, c_int,
                                     P, c_size_t, P]),
        "cslc_decode_topk_workspace_bytes": (c_size_t, [c_int, c_int, c_int]),
        "cslc_decode_topk": (c_int, [P, P, c_int, c_int, c_int, P, P, c_size_t, P]),
        "cslc_decode_topk_noalloc": (c_int, [P, P, c_int, c_int, c_int, P, P]),
        "cslc_decode_append": (c_int, [P, P, P, P, P, P, P, c_int, c_int, c_int, P, P, P, P, P, P, P, P, c_int, P, P]),
        "csa_compress_front_end": (c_int, [P, P, P, c_int, c_int, c_int, c_int, P, P]),
        "csa_indexer_topk_bf16_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int, c_int, c_int]),
        "csa_indexer_topk_bf16": (c_int, [P, P, P, c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                          P, P, P, c_size_t, P]),
        "csa_topk_bf16": (c_int, [P, c_int, c_int, c_int, c_int, c_int, c_int, P, P]),
        "cslc_testing_set_wait_limits": (c_int, [ctypes.c_uint64, ctypes.c_uint32]),
        "cslc_quantize_rows_e4m3": (c_int, [P, ctypes.c_int64, c_int, P, P, P]),
        "csa_indexer_topk_fp8": (c_int, [P, P, P, P, P, c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                         P, P, P, c_size_t, P]),
        "hca_compress_front_end": (c_int, [P, P, P, c_int, c_int, c_int, c_int, P, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


LIB = _load()


def _check(st: int):
    if st != 0:
        raise CslcError(st, LIB.cslc_last_error().decode(errors="replace"))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, name, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t


BF16, F32, I32, U8 = torch.bfloat16, torch.float32, torch.int32, torch.uint8


def abi_version() -> int:
    return LIB.cslc_abi_version()


def sync_status(stream=None):
    _check(LIB.cslc_sync_status(_stream(stream)))


WAIT_LIMIT_NS_DEFAULT = 2_000_000_000
WAIT_SLEEP_NS_DEFAULT = 200_000


def testing_set_wait_limits(limit_ns: int, sleep_ns: int):
    """Testing hook: see cslc_testing_set_wait_limits in include/cslc.h."""
    _check(LIB.cslc_testing_set_wait_limits(int(limit_ns), int(sleep_ns)))


# ------------------------------------------------------------- compression

def csa_compress(c, z, pos_bias, m: int = 4, c_b=None, z_b=None, out=None, stream=None):
    """D = 128 (KV entries) or 64 (indexer keys)."""
    B, L, D = c.shape
    _need(c, BF16, "c"); _need(z, BF16, "z", c.shape); _need(pos_bias, BF16, "pos_bias", (2 * m, D))
    if c_b is not None:
        _need(c_b, BF16, "c_b", c.shape); _need(z_b, BF16, "z_b", c.shape)
    if out is None:
        out = torch.empty(B, L // m, D, dtype=BF16, device=c.device)
    _need(out, BF16, "out", (B, L // m, D))
    _check(LIB.csa_compress(_ptr(c), _ptr(z), _ptr(c_b), _ptr(z_b), _ptr(pos_bias), B, L, D, m,
                            _ptr(out), _stream(stream)))
    return out


def hca_compress(c, z, pos_bias, m_prime: int = 128, out=None, stream=None):
    B, L, D = c.shape
    _need(c, BF16, "c"); _need(z, BF16, "z", c.shape); _need(pos_bias, BF16, "pos_bias", (m_prime, D))
    if out is None:
        out = torch.empty(B, L // m_prime, D, dtype=BF16, device=c.device)
    _need(out, BF16, "out", (B, L // m_prime, D))
    _check(LIB.hca_compress(_ptr(c), _ptr(z), _ptr(pos_bias), B, L, D, m_prime, _ptr(out), _stream(stream)))
    return out


def compress_front_end(h, W, pos_bias, m: int, overlap: bool, out=None, stream=None):
    """Entries from hidden states h [B, L, d_model]: W [4, 128, d_model] (CSA)
    or [2, 128, d_model] (HCA, m = 128); see csa_compress_front_end."""
    B, L, dm = h.shape
    _need(h, BF16, "h"); _need(W, BF16, "W", (4 if overlap else 2, 128, dm))
    _need(pos_bias, BF16, "pos_bias", (2 * m if overlap else m, 128))
    if out is None:
        out = torch.empty(B, L // m, 128, dtype=BF16, device=h.device)
    _need(out, BF16, "out", (B, L // m, 128))
    fn = LIB.csa_compress_front_end if overlap else LIB.hca_compress_front_end
    _check(fn(_ptr(h), _ptr(W), _ptr(pos_bias), B, L, dm, m, _ptr(out), _stream(stream)))
    return out


# ---------------------------------------------------------- indexer + top-k

def csa_indexer_topk(q_idx, w, k_idx, m: int, topk: int, q_pos0: int = 0, scores=None, idx=None,
                     ws=None, stream=None):
    """Returns (idx [B, L, topk] int32, scores or None). Pass scores=True to
    have a [B, L, Nc] fp32 score tensor allocated and filled."""
    B, L, HI, dI = q_idx.shape
    Nc = k_idx.shape[1]
    _need(q_idx, BF16, "q_idx"); _need(w, BF16, "w", (B, L, HI)); _need(k_idx, BF16, "k_idx", (B, Nc, dI))
    if scores is True:
        scores = torch.empty(B, L, Nc, dtype=F32, device=q_idx.device)
    if scores is not None:
        _need(scores, F32, "scores", (B, L, Nc))
    if idx is None:
        idx = torch.empty(B, L, topk, dtype=I32, device=q_idx.device)
    _need(idx, I32, "idx", (B, L, topk))
    nbytes = LIB.csa_indexer_topk_workspace_bytes(B, L, Nc, HI, topk, int(scores is not None))
    if nbytes and (ws is None or ws.numel() < nbytes):
        ws = torch.empty(nbytes, dtype=U8, device=q_idx.device)
    _check(LIB.csa_indexer_topk(_ptr(q_idx), _ptr(w), _ptr(k_idx), B, L, Nc, HI, dI, m, q_pos0, topk,
                                _ptr(scores), _ptr(idx), _ptr(ws) if nbytes else None,
                                ws.numel() if (nbytes and ws is not None) else 0, _stream(stream)))
    return idx, scores


def indexer_topk_workspace_bytes(B, L, Nc, HI, topk, scores_given=False) -> int:
    return LIB.csa_indexer_topk_workspace_bytes(B, L, Nc, HI, topk, int(scores_given))


def csa_indexer_topk_bf16(q_idx, w, k_idx, m: int, topk: int, q_pos0: int = 0, scores=None, idx=None,
                          ws=None, stream=None):
    """As csa_indexer_topk with bf16-stored scores (scores=True allocates a
    [B, L, Nc] bf16 tensor)."""
    B, L, HI, dI = q_idx.shape
    Nc = k_idx.shape[1]
    _need(q_idx, BF16, "q_idx"); _need(w, BF16, "w", (B, L, HI)); _need(k_idx, BF16, "k_idx", (B, Nc, dI))
    if scores is True:
        scores = torch.empty(B, L, Nc, dtype=BF16, device=q_idx.device)
    if scores is not None:
        _need(scores, BF16, "scores", (B, L, Nc))
    if idx is None:
        idx = torch.empty(B, L, topk, dtype=I32, device=q_idx.device)
    _need(idx, I32, "idx", (B, L, topk))
    nbytes = LIB.csa_indexer_topk_bf16_workspace_bytes(B, L, Nc, HI, topk, int(scores is not None))
    if nbytes and (ws is None or ws.numel() < nbytes):
        ws = torch.empty(nbytes, dtype=U8, device=q_idx.device)
    _check(LIB.csa_indexer_topk_bf16(_ptr(q_idx), _ptr(w), _ptr(k_idx), B, L, Nc, HI, dI, m, q_pos0, topk,
                                     _ptr(scores), _ptr(idx), _ptr(ws) if nbytes else None,
                                     ws.numel() if (nbytes and ws is not None) else 0, _stream(stream)))
    return idx, scores


def quantize_rows_e4m3(x, codes=None, scales=None, stream=None):
    """Rows x [..., 64] bf16 -> (codes uint8 [..., 64], scales fp32 [...])."""
    _need(x, BF16, "x")
    if x.shape[-1] != 64:
        raise ValueError("quantize_rows_e4m3: rows of 64 values")
    rows = x.numel() // 64
    if codes is None:
        codes = torch.empty(x.shape, dtype=U8, device=x.device)
    if scales is None:
        scales = torch.empty(x.shape[:-1], dtype=F32, device=x.device)
    _need(codes, U8, "codes", tuple(x.shape)); _need(scales, F32, "scales", tuple(x.shape[:-1]))
    _check(LIB.cslc_quantize_rows_e4m3(_ptr(x), rows, 64, _ptr(codes), _ptr(scales), _stream(stream)))
    return codes, scales


def csa_indexer_topk_fp8(q8, q_scale, w, k8, k_scale, m: int, topk: int, q_pos0: int = 0, scores=None, idx=None,
                         ws=None, stream=None):
    """csa_indexer_topk on e4m3 operands (codes + per-row scales from
    quantize_rows_e4m3). Returns (idx, scores or None); scores=True allocates
    a [B, L, Nc] fp32 tensor."""
    B, L, HI, dI = q8.shape
    Nc = k8.shape[1]
    _need(q8, U8, "q8"); _need(q_scale, F32, "q_scale", (B, L, HI)); _need(w, BF16, "w", (B, L, HI))
    _need(k8, U8, "k8", (B, Nc, dI)); _need(k_scale, F32, "k_scale", (B, Nc))
    if scores is True:
        scores = torch.empty(B, L, Nc, dtype=F32, device=q8.device)
    if scores is not None:
        _need(scores, F32, "scores", (B, L, Nc))
    if idx is None:
        idx = torch.empty(B, L, topk, dtype=I32, device=q8.device)
    _need(idx, I32, "idx", (B, L, topk))
    nbytes = LIB.csa_indexer_topk_workspace_bytes(B, L, Nc, HI, topk, int(scores is not None))
    if nbytes and (ws is None or ws.numel() < nbytes):
        ws = torch.empty(nbytes, dtype=U8, device=q8.device)
    _check(LIB.csa_indexer_topk_fp8(_ptr(q8), _ptr(q_scale), _ptr(w), _ptr(k8), _ptr(k_scale), B, L, Nc, HI, dI, m,
                                    q_pos0, topk, _ptr(scores), _ptr(idx), _ptr(ws) if nbytes else None,
                                    ws.numel() if (nbytes and ws is not None) else 0, _stream(stream)))
    return idx, scores


def indexer_topk_bf16_workspace_bytes(B, L, Nc, HI, topk, scores_given=False) -> int:
    return LIB.csa_indexer_topk_bf16_workspace_bytes(B, L, Nc, HI, topk, int(scores_given))


def csa_topk_bf16(scores, m: int, topk: int, q_pos0: int = 0, idx=None, stream=None):
    B, L, Nc = scores.shape
    _need(scores, BF16, "scores")
    if idx is None:
        idx = torch.empty(B, L, topk, dtype=I32, device=scores.device)
    _need(idx, I32, "idx", (B, L, topk))
    _check(LIB.csa_topk_bf16(_ptr(scores), B, L, Nc, m, q_pos0, topk, _ptr(idx), _stream(stream)))
    return idx


def csa_topk(scores, m: int, topk: int, q_pos0: int = 0, idx=None, stream=None):
    B, L, Nc = scores.shape
    _need(scores, F32, "scores")
    if idx is None:
        idx = torch.empty(B, L, topk, dtype=I32, device=scores.device)
    _need(idx, I32, "idx", (B, L, topk))
    _check(LIB.csa_topk(_ptr(scores), B, L, Nc, m, q_pos0, topk, _ptr(idx), _stream(stream)))
    return idx


# ---------------------------------------------------------------- attention

def csa_sparse_attn(q, kv, idx, scale: float, out=None, lse=None, stream=None):
    B, L, H, D = q.shape
    Nc = kv.shape[1]
    topk = idx.shape[2]
    _need(q, BF16, "q"); _need(kv, BF16, "kv", (B, Nc, D)); _need(idx, I32, "idx", (B, L, topk))
    if out is None:
        out = torch.empty_like(q)
    _need(out, BF16, "out", q.shape)
    if lse is True:
        lse = torch.empty(B, L, H, dtype=F32, device=q.device)
    if lse is not None:
        _need(lse, F32, "lse", (B, L, H))
    _check(LIB.csa_sparse_attn(_ptr(q), _ptr(kv), _ptr(idx), B, L, H, D, Nc, topk, float(scale),
                               _ptr(out), _ptr(lse), _stream(stream)))
    return out, lse


def hca_dense_attn(q, kv, m_prime: int, scale: float, q_pos0: int = 0, out=None, lse=None, stream=None):
    B, L, H, D = q.shape
    Nc = kv.shape[1]
    _need(q, BF16, "q"); _need(kv, BF16, "kv", (B, Nc, D))
    if out is None:
        out = torch.empty_like(q)
    _need(out, BF16, "out", q.shape)
    if lse is True:
        lse = torch.empty(B, L, H, dtype=F32, device=q.device)
    if lse is not None:
        _need(lse, F32, "lse", (B, L, H))
    _check(LIB.hca_dense_attn(_ptr(q), _ptr(kv), B, L, H, D, Nc, m_prime, q_pos0, float(scale),
                              _ptr(out), _ptr(lse), _stream(stream)))
    return out, lse


# ----------------------------------------------------------------- mixed KV

def quantize_kv_mixed(kv, nope=None, rope=None, scale=None, stream=None):
    B, N, D = kv.shape
    _need(kv, BF16, "kv")
    if D != 128:
        raise ValueError("kv must have 128 dims")
    nope = torch.empty(B, N, 64, dtype=U8, device=kv.device) if nope is None else nope
    rope = torch.empty(B, N, 64, dtype=BF16, device=kv.device) if rope is None else rope
    scale = torch.empty(B, N, dtype=F32, device=kv.device) if scale is None else scale
    _need(nope, U8, "nope", (B, N, 64)); _need(rope, BF16, "rope", (B, N, 64)); _need(scale, F32, "scale", (B, N))
    _check(LIB.cslc_quantize_kv_mixed(_ptr(kv), B, N, _ptr(nope), _ptr(rope), _ptr(scale), _stream(stream)))
    return nope, rope, scale


# ------------------------------------------------------------------- decode

class DecodeLayer:
    """Tensors of one decode layer (see cslc_decode_layer in include/cslc.h)."""

    def __init__(self, kind: str, q, nope, rope, kv_scale, n_entries, scale: float, out=None,
                 q_idx=None, w=None, k_idx=None, topk: int = 1024, idx_out=None, scores_out=None):
        self.kind = kind
        self.q, self.nope, self.rope, self.kv_scale, self.n_entries = q, nope, rope, kv_scale, n_entries
        self.q_idx, self.w, self.k_idx = q_idx, w, k_idx
        self.scale, self.topk = scale, topk
        self.out = torch.empty_like(q) if out is None else out
        self.idx_out, self.scores_out = idx_out, scores_out

    def to_c(self) -> DecodeLayerC:
        B, H, D = self.q.shape
        n_max = self.nope.shape[1]
        _need(self.q, BF16, "q"); _need(self.out, BF16, "out", self.q.shape)
        _need(self.nope, U8, "nope", (B, n_max, 64)); _need(self.rope, BF16, "rope", (B, n_max, 64))
        _need(self.kv_scale, F32, "kv_scale", (B, n_max)); _need(self.n_entries, I32, "n_entries", (B,))
        if self.kind == "csa":
            _need(self.q_idx, BF16, "q_idx"); _need(self.w, BF16, "w"); _need(self.k_idx, BF16, "k_idx")
            if self.idx_out is not None:
                _need(self.idx_out, I32, "idx_out", (B, self.topk))
            if self.scores_out is not None:
                _need(self.scores_out, F32, "scores_out", (B, n_max))
        return DecodeLayerC(0 if self.kind == "csa" else 1, _ptr(self.q), _ptr(self.q_idx), _ptr(self.w),
                            _ptr(self.k_idx), _ptr(self.nope), _ptr(self.rope), _ptr(self.kv_scale),
                            _ptr(self.n_entries), n_max, self.topk, float(self.scale), _ptr(self.out),
                            _ptr(self.idx_out), _ptr(self.scores_out))


class DecodeStep:
    """A prepared decode step: the C layer array and its workspace, reusable
    across calls (the tensors' contents may change between calls)."""

    def __init__(self, layers, HI: int = 8):
        self.layers = list(layers)
        q = self.layers[0].q
        self.B, self.H, self.D = q.shape
        self.HI = HI
        arr_t = DecodeLayerC * len(self.layers)
        self.c_layers = arr_t(*[l.to_c() for l in self.layers])
        nbytes = LIB.cslc_decode_workspace_bytes(self.c_layers, len(self.layers), self.B, self.H, HI)
        self.ws = torch.empty(max(nbytes, 16), dtype=U8, device=q.device)
        self.ws_bytes = nbytes

    def __call__(self, stream=None):
        _check(LIB.cslc_decode_step(self.c_layers, len(self.layers), self.B, self.H, self.D, self.HI, 64,
                                    _ptr(self.ws), self.ws.numel(), _stream(stream)))
        return [l.out for l in self.layers]


def decode_step(layers, HI: int = 8, stream=None):
    return DecodeStep(layers, HI)(stream)


def decode_topk(scores, n_entries, topk: int, idx=None, stream=None):
    B, n_max = scores.shape
    _need(scores, F32, "scores"); _need(n_entries, I32, "n_entries", (B,))
    if idx is None:
        idx = torch.empty(B, topk, dtype=I32, device=scores.device)
    _need(idx, I32, "idx", (B, topk))
    nbytes = LIB.cslc_decode_topk_workspace_bytes(B, n_max, topk)
    ws = torch.empty(max(nbytes, 16), dtype=U8, device=scores.device)
    _check(LIB.cslc_decode_topk(_ptr(scores), _ptr(n_entries), B, n_max, topk, _ptr(idx), _ptr(ws),
                                ws.numel(), _stream(stream)))
    return idx


def decode_topk_noalloc(scores, n_entries, topk: int, idx=None, stream=None):
    """decode_topk using the library's static scratch instead of a workspace
    (for callers that cannot allocate device memory; see include/cslc.h)."""
    B, n_max = scores.shape
    _need(scores, F32, "scores"); _need(n_entries, I32, "n_entries", (B,))
    if idx is None:
        idx = torch.empty(B, topk, dtype=I32, device=scores.device)
    _need(idx, I32, "idx", (B, topk))
    _check(LIB.cslc_decode_topk_noalloc(_ptr(scores), _ptr(n_entries), B, n_max, topk, _ptr(idx), _stream(stream)))
    return idx


class AppendState:
    """Caller-owned state of cslc_decode_append for one layer: the ring of the
    last W tokens' candidates / logits (and key candidates / logits)."""

    def __init__(self, B: int, m: int, overlap: bool, with_keys: bool, device):
        self.m, self.overlap = m, overlap
        self.W = 2 * m if overlap else m
        self.ring_c = torch.zeros(B, self.W, 128, dtype=BF16, device=device)
        self.ring_z = torch.zeros(B, self.W, 128, dtype=BF16, device=device)
        self.ring_kc = torch.zeros(B, self.W, 64, dtype=BF16, device=device) if with_keys else None
        self.ring_kz = torch.zeros(B, self.W, 64, dtype=BF16, device=device) if with_keys else None


def decode_append(state: AppendState, c, z, pos, pos_bias, nope, rope, kv_scale, n_entries, k_c=None, k_z=None,
                  k_pos_bias=None, k_idx=None, stream=None):
    """One appended token per sequence (see cslc_decode_append); pos [B] int32 on the device."""
    B = c.shape[0]
    n_max = nope.shape[1]
    _need(c, BF16, "c", (B, 128)); _need(z, BF16, "z", (B, 128)); _need(pos, I32, "pos", (B,))
    _need(pos_bias, BF16, "pos_bias", (state.W, 128))
    _need(nope, U8, "nope", (B, n_max, 64)); _need(rope, BF16, "rope", (B, n_max, 64))
    _need(kv_scale, F32, "kv_scale", (B, n_max)); _need(n_entries, I32, "n_entries", (B,))
    if k_c is not None:
        _need(k_c, BF16, "k_c", (B, 64)); _need(k_z, BF16, "k_z", (B, 64))
        _need(k_pos_bias, BF16, "k_pos_bias", (state.W, 64)); _need(k_idx, BF16, "k_idx", (B, n_max, 64))
    _check(LIB.cslc_decode_append(_ptr(c), _ptr(z), _ptr(k_c), _ptr(k_z), _ptr(pos_bias), _ptr(k_pos_bias), _ptr(pos),
                                  B, state.m, int(state.overlap), _ptr(state.ring_c), _ptr(state.ring_z),
                                  _ptr(state.ring_kc), _ptr(state.ring_kz), _ptr(nope), _ptr(rope), _ptr(kv_scale),
                                  _ptr(k_idx), n_max, _ptr(n_entries), _stream(stream)))
