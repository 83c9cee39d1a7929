"""Context-parallel CSA prefill: one long sequence split across ranks.

The pages name context parallelism for compressed attention as part of the
training framework ("百万令牌的智慧觉醒…", 基础设施). This module is the host
plumbing for one CSA layer over one sequence on `world` ranks (one process per
GPU, torch.distributed over NCCL on GPUs, gloo on CPU):

1. Each rank owns a contiguous run of tokens [t0, t1); every boundary except
   the last falls on a multiple of m, so that every window's C^a group lies on
   one rank. A rank also reads the m tokens before t0 (the C^b group of its
   first window; rank 0 has none).
2. It compresses its windows locally: the entries with index t0/m .. t1/m - 1
   and their indexer keys.
3. One all-gather assembles every entry and key on every rank (the one
   exchange step of the layer: N_c x 256 B of entries and N_c x 128 B of keys).
4. Indexer, top-k and sparse attention then run locally for the rank's query
   rows, with q_pos0 = t0 so that causal visibility uses absolute positions.

The arithmetic lives in the `ops` given to `csa_prefill_cp` (the library's
kernels on GPUs; any implementation of the same four calls elsewhere); this
module only slices, pads and gathers.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Callable

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class Shard:
    """Token range [t0, t1) of one rank and its compressed entries [e0, e1)."""
    t0: int
    t1: int
    e0: int
    e1: int
    halo: int   # tokens read before t0 (the first window's C^b group)


def shard_of(L: int, m: int, world: int, rank: int) -> Shard:
    """Contiguous shard of rank `rank`: whole windows split as evenly as
    possible, the last rank also taking the tokens past the last window."""
    n_c = L // m
    base, extra = divmod(n_c, world)
    e0 = rank * base + min(rank, extra)
    e1 = e0 + base + (1 if rank < extra else 0)
    t0 = e0 * m
    t1 = L if rank == world - 1 else e1 * m
    return Shard(t0, t1, e0, e1, halo=m if t0 > 0 else 0)


@dataclass
class CspOps:
    """The four computations of a CSA layer (tensors [B, ...] as in the C ABI)."""
    compress: Callable      # (c, z, pos_bias, m) -> entries [B, floor(L/m), D]
    indexer_topk: Callable  # (q_idx, w, k_idx, m, topk, q_pos0) -> idx [B, rows, topk]
    sparse_attn: Callable   # (q, entries, idx, scale) -> out [B, rows, H, D]


def _all_gather_rows(local: torch.Tensor, counts, group=None) -> torch.Tensor:
    """Concatenation over ranks of each rank's `local` [B, n_r, D] along dim 1
    (ranks hold different n_r: padded to the largest for the collective)."""
    world = len(counts)
    n_max = max(counts)
    B, _, D = local.shape
    pad = torch.zeros(B, n_max, D, dtype=local.dtype, device=local.device)
    pad[:, : local.shape[1]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad.contiguous(), group=group)
    return torch.cat([p[:, :n] for p, n in zip(parts, counts)], dim=1).contiguous()


def compress_local(x_local: dict, L: int, m: int, world: int, rank: int, ops: CspOps):
    """Steps 1-2 on one rank: its Shard, entries [B, e1 - e0, D] and indexer
    keys [B, e1 - e0, D_I] (the halo's own window, which has no C^b group on
    this rank, is compressed and dropped)."""
    sh = shard_of(L, m, world, rank)
    drop = 1 if sh.halo else 0
    e_loc = ops.compress(x_local["c"], x_local["z"], x_local["pos_bias"], m)[:, drop:]
    k_loc = ops.compress(x_local["kc"], x_local["kz"], x_local["k_pos_bias"], m)[:, drop:]
    assert e_loc.shape[1] == sh.e1 - sh.e0, (e_loc.shape, sh)
    return sh, e_loc, k_loc


def attend_local(x_local: dict, sh: Shard, e_all, k_all, m: int, topk: int, scale: float, ops: CspOps):
    """Step 4 on one rank: indexer, top-k and sparse attention of its query
    rows [t0, t1) over all entries, causal in absolute positions."""
    idx = ops.indexer_topk(x_local["q_idx"], x_local["w"], k_all, m, topk, sh.t0)
    return ops.sparse_attn(x_local["q"], e_all, idx, scale)


def csa_prefill_cp(x_local: dict, L: int, m: int, topk: int, scale: float, ops: CspOps, group=None):
    """One CSA layer of one sequence of L tokens on this rank's shard.

    x_local holds this rank's slices: "c", "z" (and "kc", "kz", the indexer
    key candidates and logits) for tokens [t0 - halo, t1); "q", "q_idx", "w"
    for tokens [t0, t1); "pos_bias" and "k_pos_bias" whole. Returns this rank's
    output rows [B, t1 - t0, H, D] and its Shard.
    """
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    sh, e_loc, k_loc = compress_local(x_local, L, m, world, rank, ops)
    counts = [shard_of(L, m, world, r).e1 - shard_of(L, m, world, r).e0 for r in range(world)]
    e_all = _all_gather_rows(e_loc, counts, group)
    k_all = _all_gather_rows(k_loc, counts, group)
    return attend_local(x_local, sh, e_all, k_all, m, topk, scale, ops), sh


def local_slices(x_full: dict, L: int, m: int, world: int, rank: int) -> dict:
    """This rank's slices of full-sequence inputs (see csa_prefill_cp)."""
    sh = shard_of(L, m, world, rank)
    a = sh.t0 - sh.halo
    out = {k: x_full[k][:, a:sh.t1].contiguous() for k in ("c", "z", "kc", "kz")}
    out.update({k: x_full[k][:, sh.t0:sh.t1].contiguous() for k in ("q", "q_idx", "w")})
    out["pos_bias"] = x_full["pos_bias"]
    out["k_pos_bias"] = x_full["k_pos_bias"]
    return out


def library_ops(C) -> CspOps:
    """The library's kernels (C = compressed_sparse_long_compress_b200.cslc)."""
    return CspOps(
        compress=lambda c, z, bias, m: C.csa_compress(c, z, bias, m=m),
        indexer_topk=lambda qi, w, k, m, topk, q_pos0: C.csa_indexer_topk(qi, w, k, m=m, topk=topk, q_pos0=q_pos0)[0],
        sparse_attn=lambda q, e, idx, scale: C.csa_sparse_attn(q, e, idx, scale)[0],
    )
