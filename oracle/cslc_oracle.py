"""Plain CPU oracle of the hybrid compressed attention path, in float64.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or call
this module. The CUDA library never imports it and shares no code with it.

Every function follows the method as the source pages describe it, written out
in the most direct form (loops over entries / query rows, numpy matmul, sort and
exp as library steps; no blocking, fusion or reordering). Inputs are numpy
arrays holding bf16-exact values as float64; all arithmetic is float64, and
results are rounded only at the path's storage points: compressed entries and
attention outputs to bf16 (round-to-nearest-even), indexer scores to fp32.

Sources (page title, section):
  [EXPL]  "从论文出发，逐层剖析 CSA / HCA 混注意力、mHC 残差连接与 Muon 优化器"
          (dxhjj.kegongbw.com explainer): §1.1 CSA and its "工程细节" paragraph
          (m=4, top-k=1024, overlapped C^a / C^b windows of 2m tokens), §1.2 HCA
          (m'=128, no selection, dense attention), §1.4 "存储格式混" (RoPE dims in
          BF16, the other dims in FP8).
  [READ]  "读完这篇你就搞懂 DeepSeek v4 了": §三 CSA/HCA -- 压缩机制 (CSA step 1:
          groups of m tokens, per-token contributions weighted per dimension, two
          consecutive groups joined, 4 W + 2 B learnable), 闪电索引 (CSA step 2:
          score every token against every compressed entry, weight per head,
          keep top-k; same mechanism as V3.2 DSA), 注意力计算 (CSA step 3:
          ordinary attention over the selected entries, KV shared), HCA 步骤简化
          (single group, no merge of neighbouring groups, dense over all entries).
  [TECH]  "DeepSeek-V4 技术解析：三大核心架构创新如何突破百万Token上下文瓶颈":
          §2.2 (compress then sparse-select), §2.3 (HCA: m' >> m, one entry per
          m' tokens, dense attention).

Readings where the pages leave a step open:
  R1 compression form: entry i, channel j is sum_t softmax_t(z_t[j] + B[s(t)][j]) * c_t[j]
     over the window tokens t, where s(t) is the token's slot in the window.
  R2 CSA window of entry i: C^b = tokens (i-1)m .. im-1 (slots 0..m-1, absent for
     i = 0), C^a = tokens im .. im+m-1 (slots m..2m-1). HCA window: tokens
     im' .. im'+m'-1 (slots 0..m'-1). Trailing tokens that fill no window are not
     compressed.
  R3 causal visibility: query at absolute position p sees entry i iff the
     entry's window ends at or before p, i.e. (i+1)m - 1 <= p, so
     n_vis(p) = min(N_c, floor((p+1)/m)).
  R4 indexer score: S[t,i] = sum_h w[t,h] * ReLU(q_I[t,h,:] . k_I[i,:]) (the DSA
     lightning-indexer form), no scale factor, one shared indexer key head.
  R5 top-k: the k visible entries with the largest fp32 score; ties go to the
     smaller entry index; the set is returned in ascending index order, padded
     with -1 up to k. k_eff = min(k, n_vis).
  R6 attention: K = V = the 128-dim compressed entry, shared by all query heads;
     softmax(scale * q . e) over the selected (CSA) or all visible (HCA)
     entries; a query with no entry outputs 0 (lse = -inf).
  R7 mixed KV: dims 0..63 stored as FP8 e4m3 with one fp32 scale per entry
     (s = amax/448 computed in fp32, s = 1 when amax = 0, codes = RNE with
     saturation of e/s computed in fp32), dims 64..127 (the RoPE part) kept bf16.
  R8 decode: the new token sits after all cached tokens, so all n_entries[b]
     entries are visible.

Parity status: every function here is pinned by tests/test_oracle_pins.py
(closed forms, special cases that reduce to library routines, invariants and
brute force on tiny inputs). The learned compressor's agreement with the
model's real trained weights is not checkable here (no weights exist in this
setting) and is out of scope.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "round_bf16", "round_fp32", "n_compressed", "n_visible",
    "compression_window", "compression_weights", "compress", "hca_compress",
    "csa_compress", "indexer_scores", "topk_select_row", "topk_select",
    "attend", "sparse_attention", "dense_causal_attention",
    "E4M3_MAX", "e4m3_decode", "e4m3_encode", "quantize_kv_mixed",
    "dequantize_kv_mixed", "decode_indexer_scores", "decode_csa_layer",
    "decode_hca_layer", "project", "compressor_front_end", "quantize_rows_e4m3", "indexer_scores_fp8",
]

F64 = np.float64

# ---------------------------------------------------------------------------
# Storage-point rounding
# ---------------------------------------------------------------------------

_BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


def round_bf16(x):
    """Round float64 values to the nearest bfloat16 (ties to even), as float64.

    bfloat16 has 8 significant bits for normal numbers (|x| >= 2**-126) and a
    fixed quantum of 2**-133 below that; values at or beyond the overflow
    midpoint become +-inf.
    """
    x = np.asarray(x, dtype=F64)
    out = x.copy()
    fin = np.isfinite(x) & (x != 0)
    xf = x[fin]
    _, e = np.frexp(xf)                      # xf = m * 2**e, 0.5 <= |m| < 1
    quantum = np.ldexp(1.0, np.maximum(e, -125) - 8)
    r = np.rint(xf / quantum) * quantum      # np.rint rounds half to even
    r = np.where(np.abs(r) > _BF16_MAX, np.copysign(np.inf, r), r)
    out[fin] = r
    return out


def round_fp32(x):
    """Round float64 values to the nearest float32 (IEEE RNE), as float64."""
    return np.asarray(x, dtype=F64).astype(np.float32).astype(F64)


# ---------------------------------------------------------------------------
# Geometry (readings R2, R3)
# ---------------------------------------------------------------------------

def n_compressed(L: int, m: int) -> int:
    """Number of complete compression windows of m tokens in L tokens."""
    return L // m


def n_visible(p: int, m: int, n_c: int) -> int:
    """Entries visible to a query at absolute position p (reading R3)."""
    if p < 0:
        return 0
    return min(n_c, (p + 1) // m)


def compression_window(i: int, m: int, overlap: bool):
    """Token positions and window slots that form compressed entry i.

    CSA ([EXPL] §1.1 工程细节; [READ] §三 压缩机制): the current group C^a
    (tokens im..im+m-1) plus the previous group's m tokens C^b, so each entry
    sees 2m tokens; C^b takes slots 0..m-1, C^a slots m..2m-1; entry 0 has no
    C^b. HCA ([EXPL] §1.2; [READ] §三 HCA 步骤简化): one group of m' tokens,
    slots 0..m'-1. Returns (tokens, slots, is_prev) arrays.
    """
    cur = np.arange(i * m, (i + 1) * m)
    if not overlap:
        return cur, np.arange(m), np.zeros(m, dtype=bool)
    if i == 0:
        return cur, m + np.arange(m), np.zeros(m, dtype=bool)
    prev = np.arange((i - 1) * m, i * m)
    tokens = np.concatenate([prev, cur])
    slots = np.arange(2 * m)
    is_prev = np.concatenate([np.ones(m, dtype=bool), np.zeros(m, dtype=bool)])
    return tokens, slots, is_prev


def compression_weights(zw, bias_rows):
    """Per-channel softmax over the window of (z_t + B[slot(t)]) (reading R1).

    zw: [..., W, D] logits of the window tokens; bias_rows: [W, D] positional
    bias rows of their slots. Returns weights [..., W, D] that sum to 1 over W
    for every channel ([READ] §三 压缩机制: contributions weighted per dimension).
    """
    a = zw + bias_rows
    a = a - a.max(axis=-2, keepdims=True)
    ex = np.exp(a)
    return ex / ex.sum(axis=-2, keepdims=True)


def compress(c, z, pos_bias, m: int, overlap: bool, c_b=None, z_b=None,
             round_output: bool = True):
    """Compressed entries e[b, i, :] for every complete window (readings R1, R2).

    c, z: [B, L, D]; pos_bias: [2m, D] (overlap) or [m, D]; c_b, z_b: optional
    separate candidate / logit streams used for the C^b half of CSA windows
    ([READ] §三 压缩机制 names two weight sets for the two halves); when absent
    the C^b half reads c and z. Returns [B, L // m, D], bf16-rounded unless
    round_output is False.
    """
    c = np.asarray(c, dtype=F64)
    z = np.asarray(z, dtype=F64)
    pos_bias = np.asarray(pos_bias, dtype=F64)
    cb = c if c_b is None else np.asarray(c_b, dtype=F64)
    zb = z if z_b is None else np.asarray(z_b, dtype=F64)
    B, L, D = c.shape
    n_c = n_compressed(L, m)
    out = np.zeros((B, n_c, D), dtype=F64)
    for i in range(n_c):
        tokens, slots, is_prev = compression_window(i, m, overlap)
        cw = np.where(is_prev[None, :, None], cb[:, tokens], c[:, tokens])
        zw = np.where(is_prev[None, :, None], zb[:, tokens], z[:, tokens])
        wts = compression_weights(zw, pos_bias[slots])
        out[:, i] = (wts * cw).sum(axis=1)
    return round_bf16(out) if round_output else out


def project(h, W):
    """One learned projection of the compressor front end: h [B, L, d_model]
    times W^T for W [D, d_model] (the nn.Linear layout), in float64."""
    return np.einsum("bld,nd->bln", np.asarray(h, dtype=F64), np.asarray(W, dtype=F64))


def compressor_front_end(h, W, pos_bias, m: int, overlap: bool, round_output: bool = True):
    """Compressed entries straight from hidden states ([READ] §三 压缩机制: "4 W
    + 2 B" learnable). CSA (overlap): W [4, D, d_model] holds W^{a,KV},
    W^{b,KV}, W^{a,Z}, W^{b,Z}; the C^a half of a window uses c = h W^{a,KV},
    z = h W^{a,Z}, the C^b half c_b = h W^{b,KV}, z_b = h W^{b,Z}; pos_bias
    [2m, D] holds the two B matrices (C^b slots, then C^a slots). HCA: W [2, D,
    d_model] holds W^{KV}, W^{Z}; pos_bias [m', D]. The projections stay in
    float64 (nothing is rounded between the projection and the compression)."""
    W = np.asarray(W, dtype=F64)
    if overlap:
        return compress(project(h, W[0]), project(h, W[2]), pos_bias, m, True,
                        c_b=project(h, W[1]), z_b=project(h, W[3]), round_output=round_output)
    return compress(project(h, W[0]), project(h, W[1]), pos_bias, m, False, round_output=round_output)


def csa_compress(c, z, pos_bias, m: int = 4, c_b=None, z_b=None, round_output=True):
    """CSA compressor: overlapped 2m-token windows ([EXPL] §1.1 工程细节)."""
    return compress(c, z, pos_bias, m, True, c_b, z_b, round_output)


def hca_compress(c, z, pos_bias, m_prime: int = 128, round_output=True):
    """HCA compressor: non-overlapping m'-token windows ([EXPL] §1.2)."""
    return compress(c, z, pos_bias, m_prime, False, None, None, round_output)


# ---------------------------------------------------------------------------
# Lightning indexer and top-k (readings R4, R5)
# ---------------------------------------------------------------------------

def indexer_scores(q_idx, w, k_idx, m: int, q_pos0: int = 0, rows=None):
    """Indexer scores S[b, t, i] ([READ] §三 闪电索引; reading R4).

    q_idx: [B, L, H_I, d_I]; w: [B, L, H_I]; k_idx: [B, N_c, d_I]. Row t is the
    query at absolute position q_pos0 + t. Entries past n_vis are -inf. rows
    restricts the computation to those query rows (output [B, len(rows), N_c]).
    Result is fp32-rounded.
    """
    q_idx = np.asarray(q_idx, dtype=F64)
    w = np.asarray(w, dtype=F64)
    k_idx = np.asarray(k_idx, dtype=F64)
    B, L, HI, dI = q_idx.shape
    n_c = k_idx.shape[1]
    rows = np.arange(L) if rows is None else np.asarray(rows)
    out = np.full((B, len(rows), n_c), -np.inf, dtype=F64)
    for r, t in enumerate(rows):
        nv = n_visible(q_pos0 + int(t), m, n_c)
        if nv == 0:
            continue
        dots = np.einsum("bhd,bnd->bhn", q_idx[:, t], k_idx[:, :nv])
        out[:, r, :nv] = np.einsum("bh,bhn->bn", w[:, t], np.maximum(dots, 0.0))
    return round_fp32(out)


def topk_select_row(s_row, n_vis: int, k: int):
    """Top-k of one score row over its first n_vis entries (reading R5).

    Order: larger score first, ties to the smaller index. Returns int32 [k]:
    the chosen indices ascending, then -1 padding.
    """
    s = np.asarray(s_row, dtype=F64)[:n_vis]
    cand = np.arange(n_vis)
    order = np.lexsort((cand, -s))           # primary key -s, secondary index
    keep = np.sort(order[: min(k, n_vis)])
    out = np.full(k, -1, dtype=np.int32)
    out[: keep.size] = keep
    return out


def topk_select(scores, m: int, k: int, q_pos0: int = 0, rows=None):
    """Top-k rows of an indexer score tensor [B, R, N_c] ([EXPL] §1.1: k entries)."""
    scores = np.asarray(scores, dtype=F64)
    B, R, n_c = scores.shape
    rows = np.arange(R) if rows is None else np.asarray(rows)
    out = np.full((B, R, k), -1, dtype=np.int32)
    for r in range(R):
        nv = n_visible(q_pos0 + int(rows[r]), m, n_c)
        for b in range(B):
            out[b, r] = topk_select_row(scores[b, r], nv, k)
    return out


# ---------------------------------------------------------------------------
# Attention over compressed entries (reading R6)
# ---------------------------------------------------------------------------

def attend(qv, kv, scale: float):
    """Softmax attention of H query heads over a set of entries, K = V.

    qv: [H, D]; kv: [n, D]. Returns (o [H, D] unrounded, lse [H]). With n = 0
    the output is 0 and lse is -inf.
    """
    qv = np.asarray(qv, dtype=F64)
    kv = np.asarray(kv, dtype=F64)
    H, D = qv.shape
    if kv.shape[0] == 0:
        return np.zeros((H, D)), np.full(H, -np.inf)
    logits = scale * (qv @ kv.T)                       # [H, n]
    mx = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - mx)
    denom = p.sum(axis=1, keepdims=True)
    o = (p @ kv) / denom
    return o, mx[:, 0] + np.log(denom[:, 0])


def sparse_attention(q, e, idx, scale: float, rows=None):
    """CSA core attention over the selected entries ([READ] §三 注意力计算).

    q: [B, L, H, D]; e: [B, N_c, D]; idx: [B, L, k] (-1 = empty slot). Returns
    (o bf16-rounded [B, R, H, D], lse fp32 [B, R, H]) for the requested rows.
    """
    q = np.asarray(q, dtype=F64)
    e = np.asarray(e, dtype=F64)
    idx = np.asarray(idx)
    B, L, H, D = q.shape
    rows = np.arange(L) if rows is None else np.asarray(rows)
    o = np.zeros((B, len(rows), H, D))
    lse = np.zeros((B, len(rows), H))
    for r, t in enumerate(rows):
        for b in range(B):
            sel = idx[b, t]
            sel = sel[sel >= 0]
            o[b, r], lse[b, r] = attend(q[b, t], e[b, sel], scale)
    return round_bf16(o), round_fp32(lse)


def dense_causal_attention(q, e, m: int, scale: float, q_pos0: int = 0, rows=None):
    """HCA core attention: dense over all visible entries ([EXPL] §1.2; R3, R6)."""
    q = np.asarray(q, dtype=F64)
    e = np.asarray(e, dtype=F64)
    B, L, H, D = q.shape
    n_c = e.shape[1]
    rows = np.arange(L) if rows is None else np.asarray(rows)
    o = np.zeros((B, len(rows), H, D))
    lse = np.zeros((B, len(rows), H))
    for r, t in enumerate(rows):
        nv = n_visible(q_pos0 + int(t), m, n_c)
        for b in range(B):
            o[b, r], lse[b, r] = attend(q[b, t], e[b, :nv], scale)
    return round_bf16(o), round_fp32(lse)


# ---------------------------------------------------------------------------
# FP8 e4m3 codec (OCP 8-bit floating point specification, E4M3 format) and the
# mixed BF16-RoPE / FP8 KV layout ([EXPL] §1.4 存储格式混; reading R7)
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_decode(codes):
    """Value of each E4M3 code: sign bit, 4 exponent bits (bias 7), 3 mantissa
    bits; exponent 0 is subnormal (mantissa/8 * 2**-6); S.1111.111 is NaN; there
    are no infinities."""
    codes = np.asarray(codes, dtype=np.int64)
    sign = np.where(codes & 0x80, -1.0, 1.0)
    ex = (codes >> 3) & 0xF
    man = codes & 0x7
    normal = (1.0 + man / 8.0) * np.ldexp(1.0, ex - 7)
    sub = (man / 8.0) * 2.0 ** -6
    val = sign * np.where(ex == 0, sub, normal)
    return np.where((ex == 0xF) & (man == 0x7), np.nan, val)


def e4m3_encode(x):
    """E4M3 code of each value: round to nearest, ties to even, saturating
    finite values beyond the range to +-448 (no NaN produced for finite input)."""
    x = np.asarray(x, dtype=F64)
    sign = np.signbit(x).astype(np.int64) << 7
    a = np.abs(x)
    _, e = np.frexp(np.where(a > 0, a, 1.0))
    quantum = np.ldexp(1.0, np.maximum(e, -5) - 4)   # 4 significant bits; 2**-9 below 2**-6
    r = np.minimum(np.rint(a / quantum) * quantum, E4M3_MAX)
    r = np.where(a > 0, r, 0.0)
    # value -> fields
    _, er = np.frexp(np.where(r > 0, r, 1.0))
    is_normal = r >= 2.0 ** -6
    exp_field = np.where(is_normal, er - 1 + 7, 0)
    man_normal = np.rint((r / np.ldexp(1.0, er - 1) - 1.0) * 8.0)
    man_sub = np.rint(r / 2.0 ** -9)
    man_field = np.where(is_normal, man_normal, man_sub).astype(np.int64)
    code = sign | (exp_field.astype(np.int64) << 3) | man_field
    return code.astype(np.uint8)


def quantize_kv_mixed(e):
    """Split compressed entries [B, N, 128] into the mixed decode layout.

    Returns (nope codes uint8 [B, N, 64] for dims 0..63, rope float64 [B, N, 64]
    = dims 64..127 unchanged, scale float32 [B, N]). The scale and the scaled
    values are computed in fp32, the precision in which the codes are decided.
    """
    e = np.asarray(e, dtype=F64)
    nope = e[..., :64].astype(np.float32)
    amax = np.abs(nope).max(axis=-1)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    scaled = (nope / scale[..., None]).astype(np.float32)
    codes = e4m3_encode(scaled.astype(F64))
    return codes, e[..., 64:].copy(), scale


def quantize_rows_e4m3(x):
    """Rows of x [..., d] as e4m3 codes with one fp32 scale per row ([EXPL]
    §1.4: an FP8 form of the lightning indexer's operands). The rule is the
    one of the mixed KV layout (reading R7): s = amax / 448 in fp32 (1 when the
    row is zero), codes = RNE-saturate(x / s) with the division in fp32.
    Returns (codes uint8 [..., d], scale float32 [...]).
    """
    x = np.asarray(x, dtype=F64).astype(np.float32)
    amax = np.abs(x).max(axis=-1)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    scaled = (x / scale[..., None]).astype(np.float32)
    return e4m3_encode(scaled.astype(F64)), scale


def indexer_scores_fp8(q8, q_scale, w, k8, k_scale, m: int, q_pos0: int = 0, rows=None):
    """Indexer scores from e4m3 operands ([EXPL] §1.4; formula of reading R4):
    the scores of the values the codes stand for, q_I = decode(q8) * q_scale
    per (token, head) row and k_I = decode(k8) * k_scale per entry, in float64,
    rounded to fp32.

    q8: [B, L, H_I, d_I] uint8, q_scale: [B, L, H_I]; w: [B, L, H_I];
    k8: [B, N_c, d_I] uint8, k_scale: [B, N_c].
    """
    q = e4m3_decode(q8) * np.asarray(q_scale, dtype=F64)[..., None]
    k = e4m3_decode(k8) * np.asarray(k_scale, dtype=F64)[..., None]
    return indexer_scores(q, w, k, m, q_pos0, rows=rows)


def dequantize_kv_mixed(nope_codes, rope, scale):
    """Entries as the decode path sees them: FP8 value * scale ++ RoPE part."""
    nope = e4m3_decode(nope_codes) * np.asarray(scale, dtype=F64)[..., None]
    return np.concatenate([nope, np.asarray(rope, dtype=F64)], axis=-1)


# ---------------------------------------------------------------------------
# Decode (one new query token per sequence; reading R8)
# ---------------------------------------------------------------------------

def decode_indexer_scores(q_idx, w, k_idx, n_entries):
    """Indexer scores of one query per sequence over its n_entries[b] entries.

    q_idx: [B, H_I, d_I]; w: [B, H_I]; k_idx: [B, N, d_I]. Returns fp32-rounded
    [B, N], -inf past n_entries[b].
    """
    q_idx = np.asarray(q_idx, dtype=F64)
    w = np.asarray(w, dtype=F64)
    k_idx = np.asarray(k_idx, dtype=F64)
    B, N = k_idx.shape[:2]
    out = np.full((B, N), -np.inf)
    for b in range(B):
        n = int(n_entries[b])
        dots = q_idx[b] @ k_idx[b, :n].T                 # [H_I, n]
        out[b, :n] = w[b] @ np.maximum(dots, 0.0)
    return round_fp32(out)


def decode_csa_layer(q, q_idx, w, k_idx, kv_hat, n_entries, topk: int, scale: float,
                     scores=None):
    """One CSA decode layer: indexer, top-k, sparse attention over kv_hat.

    kv_hat: dequantized entries [B, N, 128]. scores, when given, replaces the
    indexer output (so top-k can be checked on the GPU's own fp32 scores).
    Returns (o bf16-rounded [B, H, D], idx int32 [B, topk], scores).
    """
    if scores is None:
        scores = decode_indexer_scores(q_idx, w, k_idx, n_entries)
    q = np.asarray(q, dtype=F64)
    B, H, D = q.shape
    o = np.zeros((B, H, D))
    idx = np.full((B, topk), -1, dtype=np.int32)
    for b in range(B):
        idx[b] = topk_select_row(scores[b], int(n_entries[b]), topk)
        sel = idx[b][idx[b] >= 0]
        o[b], _ = attend(q[b], kv_hat[b, sel], scale)
    return round_bf16(o), idx, scores


def decode_hca_layer(q, kv_hat, n_entries, scale: float):
    """One HCA decode layer: dense attention over all n_entries[b] entries."""
    q = np.asarray(q, dtype=F64)
    B, H, D = q.shape
    o = np.zeros((B, H, D))
    for b in range(B):
        o[b], _ = attend(q[b], kv_hat[b, : int(n_entries[b])], scale)
    return round_bf16(o)
