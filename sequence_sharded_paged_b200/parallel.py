"""Decode Context Parallelism across GPUs: one shard per rank.

"Efficient Decode Context Parallelism with vLLM for Long Context Workloads",
section 4: each GPU of the group keeps the KV cache of the positions it owns;
section 4.1: each GPU attends the query against its local slice, the per-head
LSEs are all-gathered, every GPU reweights its partial output by
exp(LSE_rank - LSE), and a reduce-scatter sums the reweighted partials so that
each GPU ends with the merged output of its share of the heads.

Here the attention, the reweighting and the reduce-scatter layout run in
libdcp (dcp_decode_rank, dcp_lse_rescale); torch.distributed carries the two
collectives (NCCL over NVLink on GPUs, gloo in the CPU tests).  This module only
orders those calls and allocates their buffers.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import DCP_DECODE_RANK, CacheDesc, dcp_decode_rank, dcp_decode_workspace_size_ex, dcp_lse_rescale


def rank_workspace(desc: CacheDesc, batch: int, q_len: int = 1, device=None) -> torch.Tensor:
    """Workspace of dcp_decode_rank for this rank's cache."""
    n = dcp_decode_workspace_size_ex(desc, batch, q_len, DCP_DECODE_RANK)
    if n == 0:
        raise ValueError("unsupported cache descriptor for dcp_decode_rank")
    return torch.empty(n, dtype=torch.uint8, device=device)


def exchange(o: torch.Tensor, lse: torch.Tensor, rank: int, world: int, group=None, rescale=None):
    """All-gather the LSEs, reweight this rank's partial, reduce-scatter over rows.

    o     fp32 [B][H][Dv]   this rank's normalised partial (H query rows)
    lse   fp32 [B][H]       its natural-log LSE (-inf where it owns nothing)
    Returns (out [B][H/world][Dv], lse_all_rows [B][H]): the merged output of rows
    [rank * H/world, (rank + 1) * H/world) and the merged LSE of every row.
    `rescale(lse_all, rank, o, o_rs, lse_out)` defaults to libdcp's dcp_lse_rescale.
    """
    B, H, Dv = o.shape
    if H % world:
        raise ValueError(f"{H} query rows do not split over {world} ranks")
    lse_all = torch.empty((world, B, H), dtype=torch.float32, device=o.device)
    dist.all_gather_into_tensor(lse_all.view(world * B, H), lse.contiguous(), group=group)
    o_rs = torch.empty((world, B, H // world, Dv), dtype=torch.float32, device=o.device)
    lse_out = torch.empty((B, H), dtype=torch.float32, device=o.device)
    (rescale or dcp_lse_rescale)(lse_all, rank, o, o_rs, lse_out)
    out = torch.empty((B, H // world, Dv), dtype=torch.float32, device=o.device)
    dist.reduce_scatter_tensor(out, o_rs.view(world * B, H // world, Dv), op=dist.ReduceOp.SUM, group=group)
    return out, lse_out


def decode_distributed(desc: CacheDesc, rank: int, world: int, q: torch.Tensor, seq_lens: torch.Tensor,
                       ws: torch.Tensor, group=None):
    """One decode step of rank `rank` of a DCP group (desc: this rank's cache, block
    tables [1][B][max_local_pages]): its local partial, then the exchange.
    q bf16 [B][hq][dk] or [B][q_len][hq][dk].  Returns (out, lse) as exchange(), with
    rows = q_len * hq (row j * hq + h is query token j of head h)."""
    B = q.shape[0]
    rows = q.shape[-2] * (1 if q.dim() == 3 else q.shape[1])
    o = torch.empty((B, rows, desc.dv), dtype=torch.float32, device=q.device)
    lse = torch.empty((B, rows), dtype=torch.float32, device=q.device)
    dcp_decode_rank(desc, rank, q, seq_lens, o.view(*q.shape[:-1], desc.dv), lse.view(q.shape[:-1]), ws)
    return exchange(o, lse, rank, world, group)
