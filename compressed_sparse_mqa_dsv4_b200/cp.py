"""Chunked and context-parallel prefill of one CSA / HCA layer, over the library's C ABI.

"CSA And HCA: Definition, State, And Cost Model", s11 (training / long prefill): a sequence
can be split into contiguous token ranges processed separately -- one after the other
(chunked prefill with a start position, as in pypto-lib PR #834's "128 tokens at start-pos
896" workload) or on different GPUs at once (context parallelism). Both reduce to the same
per-range step:

  * compression of the range's tokens [p0, p0 + n): entry i pools block i (stream a) and,
    for CSA, block i - 1 (stream b, s2.1). The first block of a range with p0 > 0 therefore
    needs the preceding m tokens' rows -- a one-block halo. With p0 a multiple of m, the
    range emits exactly entries p0/m .. (p0 + n)/m - 1;
  * the local window of query t is {max(0, t - w + 1) .. t} (s5.1), so the range's queries
    also read up to w - 1 local rows before p0 -- a window halo;
  * index scores, TopK and attention of query t read only entries s < floor((t + 1)/m)
    (s1), i.e. entries of this range and of earlier ones: with the entries of all earlier
    ranges gathered in front (an all-gather across context-parallel ranks), every query of
    the range sees exactly what full prefill gives it.

Every arithmetic step runs in the library's kernels (dsv4_compress, dsv4_index_topk,
dsv4_hybrid_sparse_attn); this module only arranges rows and, for context parallelism,
moves halos and entries with torch.distributed collectives.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import (dsv4_compress, dsv4_hybrid_sparse_attn, dsv4_index_topk,
               dsv4_index_topk_workspace_size)

__all__ = ["compress_range", "window_ring", "prefill_range", "exchange_halo",
           "allgather_rows", "cp_prefill"]


def compress_range(C: torch.Tensor, Z: torch.Tensor, bias: torch.Tensor, m: int, overlap: bool,
                   p0: int, C_halo: Optional[torch.Tensor] = None,
                   Z_halo: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None):
    """Entries emitted by the tokens [p0, p0 + n) of B sequences: [B, (p0+n)//m - p0//m, c].

    C, Z [B, n, S*c] are the range's rows; p0 must be a multiple of m. For CSA (overlap) with
    p0 > 0, C_halo / Z_halo [B, m, 2c] are the rows of tokens [p0 - m, p0): the preceding
    block that entry p0/m pools from stream b."""
    if p0 % m:
        raise ValueError(f"range start {p0} is not a multiple of m={m}")
    if overlap and p0 > 0:
        if C_halo is None or Z_halo is None or C_halo.shape[1] != m:
            raise ValueError("a CSA range after position 0 needs the m-token halo rows")
        Cx = torch.cat([C_halo, C], dim=1).contiguous()
        Zx = torch.cat([Z_halo, Z], dim=1).contiguous()
        full = dsv4_compress(Cx, Zx, bias, m, True)
        ent = full[:, 1:]              # entry 0 of the extended range lacks its own halo
        if out is not None:
            out.copy_(ent)
            return out
        return ent.contiguous()
    return dsv4_compress(C.contiguous(), Z.contiguous(), bias, m, overlap, out=out)


def window_ring(local: torch.Tensor, p0: int, wwin: int,
                local_halo: Optional[torch.Tensor] = None):
    """Local ring for the queries [p0, p0 + n): returns (ring [B, R, c], R) with position j in
    slot j mod R, holding positions [p0 - h, p0 + n), h = min(p0, wwin - 1).

    local [B, n, c] are the range's own rows; local_halo [B, >= h, c] the rows just before
    p0 (its last h rows are used)."""
    B, n, c = local.shape
    h = min(p0, wwin - 1)
    if h > 0:
        if local_halo is None or local_halo.shape[1] < h:
            raise ValueError(f"queries from position {p0} need {h} window-halo rows")
        rows = torch.cat([local_halo[:, local_halo.shape[1] - h:], local], dim=1)
    else:
        rows = local
    R = h + n
    slots = torch.arange(p0 - h, p0 + n, device=local.device) % R
    ring = torch.empty(B, R, c, dtype=local.dtype, device=local.device)
    ring[:, slots] = rows
    return ring, R


def prefill_range(*, Q, local, p0: int, m: int, wwin: int, pool, KI=None, qI=None, w=None,
                  k: int = 0, sink=None, scale=None, local_halo=None, kv_row_off=None,
                  workspace=None):
    """Index TopK (CSA: KI given) and attention of the queries [p0, p0 + n) of B sequences.

    pool [rows, c] (and KI [rows, c_I]) hold every entry these queries may see -- entries
    s < floor((p0 + n)/m) of each sequence, sequence b's from row kv_row_off[b] (default
    b * rows / B). Q [B, n, H, c]; local [B, n, c] plus local_halo (see window_ring); CSA:
    qI [B, n, H_I, c_I], w [B, n, H_I], k. HCA reads all completed entries (dense).
    Returns (O [B, n, H, c], lse [B, n, H], idx or None, counts or None)."""
    B, n = Q.shape[0], Q.shape[1]
    dev = Q.device
    if kv_row_off is None:
        per = pool.shape[0] // B
        kv_row_off = torch.arange(B, dtype=torch.int64, device=dev) * per
    q_pos0 = torch.full((B,), p0, dtype=torch.int32, device=dev)
    ring, _ = window_ring(local, p0, wwin, local_halo)
    idx = counts = None
    if KI is not None:
        max_e = (p0 + n) // m
        ws = workspace
        if ws is None and max_e > 0:
            ws = torch.empty(max(1, dsv4_index_topk_workspace_size(B, n, max_e, k)),
                             dtype=torch.uint8, device=dev)
        idx, counts = dsv4_index_topk(qI, w, KI, kv_row_off, q_pos0, m, k, max_e, workspace=ws)
        O, lse = dsv4_hybrid_sparse_attn(Q, pool, kv_row_off, idx, counts, ring, q_pos0, m, wwin,
                                         sink, scale)
    else:
        O, lse = dsv4_hybrid_sparse_attn(Q, pool, kv_row_off, None, None, ring, q_pos0, m, wwin,
                                         sink, scale)
    return O, lse, idx, counts


# ----------------------------------------------------------------------------- context parallel


def exchange_halo(x: torch.Tensor, rows: int, group=None):
    """Context-parallel halo: each rank sends the last `rows` token rows of its shard x
    [B, n, ...] to the next rank and receives the previous rank's (rank 0 receives zeros,
    which nothing reads). One all-gather of the shards' tails; returns [B, rows, ...]."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    tail = x[:, x.shape[1] - rows:].contiguous()
    parts = [torch.empty_like(tail) for _ in range(world)]
    dist.all_gather(parts, tail, group=group)
    return parts[rank - 1] if rank > 0 else torch.zeros_like(tail)


def allgather_rows(x: torch.Tensor, group=None):
    """All ranks' [B, e, ...] blocks concatenated along dim 1 in rank order (every rank's
    shard emits the same number of entries e)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    parts = [torch.empty_like(x) for _ in range(world)]
    dist.all_gather(parts, x.contiguous(), group=group)
    return torch.cat(parts, dim=1)


def cp_prefill(*, C, Z, bias, Q, local, m: int, wwin: int, overlap: bool, CI=None, ZI=None,
               biasI=None, qI=None, w=None, k: int = 0, sink=None, scale=None, group=None):
    """Context-parallel prefill of one layer: rank r holds the tokens [r*n, (r+1)*n) of B
    sequences (n a multiple of m and >= wwin - 1; shard tensors as in prefill_range). Halos
    travel from rank r-1 to r, the compressed entries of all ranks are all-gathered, and
    every rank computes O / LSE of its own queries, equal to those of full prefill."""
    import torch.distributed as dist
    rank = dist.get_rank(group)
    B, n = Q.shape[0], Q.shape[1]
    if n % m or n < wwin - 1:
        raise ValueError(f"shard length {n} must be a multiple of m={m} and >= w-1={wwin - 1}")
    p0 = rank * n
    Ch, Zh = exchange_halo(C, m, group), exchange_halo(Z, m, group)
    lh = exchange_halo(local, max(wwin - 1, 1), group)
    ent = compress_range(C, Z, bias, m, overlap, p0, Ch, Zh)              # [B, n/m, c]
    pool = allgather_rows(ent, group)                                     # [B, W*n/m, c]
    KI = None
    if CI is not None:
        CIh, ZIh = exchange_halo(CI, m, group), exchange_halo(ZI, m, group)
        KI = allgather_rows(compress_range(CI, ZI, biasI, m, True, p0, CIh, ZIh), group)
    E = pool.shape[1]
    O, lse, idx, counts = prefill_range(
        Q=Q, local=local, p0=p0, m=m, wwin=wwin, pool=pool.reshape(B * E, -1),
        KI=None if KI is None else KI.reshape(B * E, -1), qI=qI, w=w, k=k, sink=sink,
        scale=scale, local_halo=lh if p0 > 0 else None)
    return O, lse, idx, counts
