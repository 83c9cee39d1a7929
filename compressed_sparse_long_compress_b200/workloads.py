"""Workload shapes and seeded synthetic input generators.

This module holds no arithmetic of the attention method: only tensor shapes,
seeds and random draws. It is the one module that both the CUDA path (tests,
bench) and the CPU oracle's tests take their inputs from.

Seeds: tensor ``tensor_id`` of workload number ``wid`` is drawn from a
``torch.Generator`` seeded with ``1000 * wid + tensor_id`` (+ ``100 * layer`` for
the layers of the hybrid decode workload). Draws are fp32 and then rounded to
bf16. Distributions: q, c, z, indexer q/k and decode KV ~ N(0, 1); positional
bias ~ N(0, 0.1^2); indexer head weights ~ U(0, 1).
"""

from __future__ import annotations

from dataclasses import dataclass, field
import math

import torch

# tensor ids (stable across versions: they feed the seeds)
T_Q, T_C, T_Z, T_BIAS, T_QIDX, T_W, T_KIDX, T_KV, T_CB, T_ZB, T_HC, T_HZ, T_HBIAS = range(1, 14)


@dataclass(frozen=True)
class PrefillShape:
    """One prefill layer's shapes. m: compression ratio; H: query heads."""
    B: int
    L: int
    H: int
    D: int = 128
    m: int = 4
    HI: int = 8
    dI: int = 64
    topk: int = 1024
    overlap: bool = True

    @property
    def n_c(self) -> int:
        return self.L // self.m

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


@dataclass(frozen=True)
class DecodeShape:
    """Decode step: B sequences, one new token each, N entries per layer."""
    B: int
    H: int
    kinds: tuple           # per layer: "csa" or "hca"
    n_entries: tuple       # per layer: entries per sequence
    D: int = 128
    HI: int = 8
    dI: int = 64
    topk: int = 1024

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


@dataclass(frozen=True)
class FrontEndShape:
    """Compressor front end: hidden states [B, L, d_model] through the learned
    projections into compressed entries (window ratio m, overlap = CSA)."""
    B: int
    L: int
    d_model: int
    m: int = 4
    overlap: bool = True

    @property
    def n_c(self) -> int:
        return self.L // self.m

    @property
    def n_proj(self) -> int:
        return 4 if self.overlap else 2


@dataclass(frozen=True)
class Workload:
    wid: int
    name: str
    description: str
    csa: PrefillShape | None = None
    hca: PrefillShape | None = None
    decode: DecodeShape | None = None
    extra: dict = field(default_factory=dict)
    front_end: FrontEndShape | None = None


WORKLOADS = {
    "tiny": Workload(
        1, "tiny",
        "batch 1, L=4096; CSA m=4 (overlapped 2m window) -> 1024 entries, 16 heads x 128, "
        "indexer 4 x 64, top-k 128; HCA m'=128 -> 32 entries dense causal",
        csa=PrefillShape(B=1, L=4096, H=16, m=4, HI=4, topk=128, overlap=True),
        hca=PrefillShape(B=1, L=4096, H=16, m=128, overlap=False),
    ),
    "csa_prefill": Workload(
        2, "csa_prefill",
        "CSA prefill, batch 1, L=65536, m=4 -> 16384 entries, 64 heads x 128, "
        "indexer 8 x 64, top-k 1024, causal",
        csa=PrefillShape(B=1, L=65536, H=64, m=4, HI=8, topk=1024, overlap=True),
    ),
    "hca_prefill": Workload(
        3, "hca_prefill",
        "HCA prefill, batch 1, L=1048576, m'=128 -> 8192 entries, 64 heads x 128, dense causal",
        hca=PrefillShape(B=1, L=1048576, H=64, m=128, overlap=False),
    ),
    "csa_decode": Workload(
        4, "csa_decode",
        "CSA decode, 64 sequences x 1 token at context 131072 (32768 entries each), "
        "64 heads x 128, indexer 8 x 64, top-k 1024, mixed BF16-RoPE/FP8 KV",
        decode=DecodeShape(B=64, H=64, kinds=("csa",), n_entries=(32768,)),
    ),
    "hybrid_decode": Workload(
        5, "hybrid_decode",
        "hybrid decode at 1M context, 8 sequences x 1 token, layers CSA,HCA,CSA,HCA; "
        "CSA 262144 entries (top-k 1024), HCA 8192 entries; 64 heads x 128, mixed KV",
        decode=DecodeShape(B=8, H=64, kinds=("csa", "hca", "csa", "hca"),
                           n_entries=(262144, 8192, 262144, 8192)),
    ),
    "front_end_prefill": Workload(
        6, "front_end_prefill",
        "CSA compressor front end, batch 1, L=65536 hidden states of d_model=7168 -> 4 learned projections "
        "(4 x 128) -> overlapped 2m-window compression, m=4 -> 16384 entries",
        front_end=FrontEndShape(B=1, L=65536, d_model=7168, m=4, overlap=True),
    ),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def randn_bf16(shape, seed: int, device="cpu", std: float = 1.0) -> torch.Tensor:
    """N(0, std^2) draws in fp32 from a seeded generator, rounded to bf16."""
    x = torch.randn(*shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def rand_bf16(shape, seed: int, device="cpu") -> torch.Tensor:
    """U(0, 1) draws in fp32 from a seeded generator, rounded to bf16."""
    x = torch.rand(*shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    return x.to(torch.bfloat16)


def rand_f32(shape, seed: int, device="cpu", lo: float = -4.0, hi: float = 4.0) -> torch.Tensor:
    x = torch.rand(*shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    return x.mul_(hi - lo).add_(lo)


def seed_of(wid: int, tensor_id: int, layer: int = 0) -> int:
    return 1000 * wid + tensor_id + 100 * layer


def prefill_inputs(s: PrefillShape, wid: int, device="cpu", with_indexer=None,
                   separate_prev_stream: bool = False, q_scale: float = 1.0):
    """Raw inputs of one prefill layer: c, z, pos_bias, q and (CSA) indexer q/w/k.

    ``q_scale`` multiplies q after the draw (a "peaky" variant for tests).
    """
    B, L, D = s.B, s.L, s.D
    with_indexer = s.overlap if with_indexer is None else with_indexer
    nb = 2 * s.m if s.overlap else s.m
    out = {
        "c": randn_bf16((B, L, D), seed_of(wid, T_C), device),
        "z": randn_bf16((B, L, D), seed_of(wid, T_Z), device),
        "pos_bias": randn_bf16((nb, D), seed_of(wid, T_BIAS), device, std=0.1),
        "q": randn_bf16((B, L, s.H, D), seed_of(wid, T_Q), device),
    }
    if q_scale != 1.0:
        out["q"] = (out["q"].float() * q_scale).to(torch.bfloat16)
    if separate_prev_stream:
        out["c_b"] = randn_bf16((B, L, D), seed_of(wid, T_CB), device)
        out["z_b"] = randn_bf16((B, L, D), seed_of(wid, T_ZB), device)
    if with_indexer:
        out["q_idx"] = randn_bf16((B, L, s.HI, s.dI), seed_of(wid, T_QIDX), device)
        out["w"] = rand_bf16((B, L, s.HI), seed_of(wid, T_W), device)
        out["k_idx"] = randn_bf16((B, s.n_c, s.dI), seed_of(wid, T_KIDX), device)
    return out


T_H, T_W = 14, 15


def front_end_inputs(s: FrontEndShape, wid: int, device="cpu"):
    """Hidden states h ~ N(0, 1), projection weights ~ N(0, 1/d_model) (so the
    projections are ~ N(0, 1)) and positional bias ~ N(0, 0.1^2), all bf16."""
    return {
        "h": randn_bf16((s.B, s.L, s.d_model), seed_of(wid, T_H), device),
        "W": randn_bf16((s.n_proj, 128, s.d_model), seed_of(wid, T_W), device, std=s.d_model ** -0.5),
        "pos_bias": randn_bf16((2 * s.m if s.overlap else s.m, 128), seed_of(wid, T_BIAS), device, std=0.1),
    }


def decode_layer_inputs(d: DecodeShape, layer: int, wid: int, device="cpu", n_max=None):
    """Raw inputs of one decode layer: q, entries e (bf16, to be quantised into
    the mixed layout), and for CSA the indexer q/w/k."""
    B, H, D = d.B, d.H, d.D
    n = d.n_entries[layer] if n_max is None else n_max
    out = {
        "q": randn_bf16((B, H, D), seed_of(wid, T_Q, layer), device),
        "kv": randn_bf16((B, n, D), seed_of(wid, T_KV, layer), device),
    }
    if d.kinds[layer] == "csa":
        out["q_idx"] = randn_bf16((B, d.HI, d.dI), seed_of(wid, T_QIDX, layer), device)
        out["w"] = rand_bf16((B, d.HI), seed_of(wid, T_W, layer), device)
        out["k_idx"] = randn_bf16((B, n, d.dI), seed_of(wid, T_KIDX, layer), device)
    return out
