"""Assembly of a sharded paged KV cache on the GPU for a synthetic workload.

Used by the tests and the benchmark.  The caller supplies how many pages each
(shard, request) needs (from its own shard counts); pages are dealt from a
seeded permutation of the pool, the pools are allocated with torch, and the
cache is filled through ``dcp_kv_append`` with rows produced on the device by
the seeded generator.  All arithmetic of the path runs in libdcp.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

import synth
import synth.device as sdev

from . import (DCP_BF16, DCP_DECODE_RANK, DCP_FP8_E4M3, DCP_GQA, DCP_MLA, CacheDesc, dcp_decode_workspace_size,
               dcp_decode_workspace_size_ex, dcp_kv_append, dcp_kv_append_rank, dcp_shard_counts, make_cache_desc)


@dataclass
class DeviceWorkload:
    w: synth.Workload
    desc: CacheDesc
    k_pages: torch.Tensor
    v_pages: torch.Tensor | None
    kv_scales: torch.Tensor | None
    block_tables: torch.Tensor
    num_pages: int
    seq_lens: torch.Tensor       # int32 [B] on device
    ws: torch.Tensor             # decode workspace (uint8)
    rank: int | None = None      # rank-local cache: only shard `rank`'s pages and tables

    @property
    def kv_bytes(self) -> int:
        return int(self.seq_lens.sum().item()) * self.w.kv_bytes_per_token


def gpu_shard_counts(lengths: np.ndarray, n_shards: int, interleave: int) -> np.ndarray:
    """Per-shard counts computed by dcp_shard_counts on the device (int64 [N][B])."""
    sl = torch.as_tensor(np.asarray(lengths, dtype=np.int32), device="cuda")
    out = torch.empty((n_shards, sl.numel()), dtype=torch.int32, device="cuda")
    dcp_shard_counts(sl, n_shards, interleave, out)
    return out.cpu().numpy().astype(np.int64)


def pages_needed(counts: np.ndarray, page_size: int) -> np.ndarray:
    return (counts + page_size - 1) // page_size


def build(w: synth.Workload, counts_with_growth: np.ndarray, fill: bool = True, slack_pages: int = 0,
          max_rows_per_append: int = 1 << 21, rank: int | None = None) -> DeviceWorkload:
    """Allocate the pools and block tables for ``w`` (per-shard counts
    ``counts_with_growth`` [N][B] sized for the longest length the run will
    reach) and, if ``fill``, append every position [0, L_b) of every request.
    rank = r: the cache of rank r of an N-GPU group (pages and block tables of
    shard r only, filled through dcp_kv_append_rank from every position)."""
    dev = torch.device("cuda")
    N, B, P = w.n_shards, w.B, w.page_size
    counts_with_growth = np.asarray(counts_with_growth)
    if rank is not None:
        counts_with_growth = counts_with_growth[rank:rank + 1]
    need = pages_needed(counts_with_growth, P)
    bt_np, num_pages = synth.deal_block_tables(w.seed_len, need, slack_pages=slack_pages)
    bt = torch.as_tensor(bt_np, device=dev)
    kind = DCP_GQA if w.kind == "gqa" else DCP_MLA
    dtype = DCP_FP8_E4M3 if w.dtype == "fp8" else DCP_BF16
    if kind == DCP_GQA:
        k_pages = torch.empty((num_pages, w.hkv, P, w.dk), dtype=torch.bfloat16, device=dev)
        v_pages = torch.empty((num_pages, w.hkv, P, w.dv), dtype=torch.bfloat16, device=dev)
        kv_scales = None
    elif dtype == DCP_BF16:
        k_pages = torch.empty((num_pages, P, 576), dtype=torch.bfloat16, device=dev)
        v_pages = None
        kv_scales = None
    else:
        k_pages = torch.empty((num_pages, P, 576), dtype=torch.uint8, device=dev)
        v_pages = None
        kv_scales = torch.empty((num_pages, P), dtype=torch.float32, device=dev)
    desc = make_cache_desc(kind=kind, dtype=dtype, n_shards=N, interleave=w.interleave, page_size=P,
                           num_pages=num_pages, hq=w.hq, hkv=w.hkv, dk=w.dk, dv=w.dv, scale=w.scale, batch=B,
                           block_tables=bt, k_pages=k_pages, v_pages=v_pages, kv_scales=kv_scales)
    seq_lens = torch.as_tensor(np.asarray(w.lengths, dtype=np.int32), device=dev)
    ws_bytes = dcp_decode_workspace_size(desc, B) if rank is None else dcp_decode_workspace_size_ex(desc, B, 1, DCP_DECODE_RANK)
    if ws_bytes == 0:
        raise ValueError("unsupported cache descriptor for decode")
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    dw = DeviceWorkload(w, desc, k_pages, v_pages, kv_scales, bt, num_pages, seq_lens, ws, rank)
    if fill:
        append_positions(dw, np.zeros(B, np.int64), np.asarray(w.lengths, np.int64), max_rows_per_append)
    return dw


def append_positions(dw: DeviceWorkload, start: np.ndarray, stop: np.ndarray, max_rows: int = 1 << 21) -> None:
    """Append positions [start_b, stop_b) of every request b (generated rows)."""
    w = dw.w
    counts = np.maximum(np.asarray(stop) - np.asarray(start), 0).astype(np.int64)
    total = int(counts.sum())
    if total == 0:
        return
    dev = torch.device("cuda")
    req_all = torch.repeat_interleave(torch.arange(w.B, dtype=torch.int32, device=dev),
                                      torch.as_tensor(counts, device=dev))
    offs = np.concatenate([[0], np.cumsum(counts)[:-1]])
    base = torch.repeat_interleave(torch.as_tensor(np.asarray(start, np.int64) - offs, device=dev),
                                   torch.as_tensor(counts, device=dev))
    pos_all = (torch.arange(total, dtype=torch.int64, device=dev) + base).to(torch.int32)
    for lo in range(0, total, max_rows):
        hi = min(total, lo + max_rows)
        req = req_all[lo:hi].contiguous()
        pos = pos_all[lo:hi].contiguous()
        if w.kind == "gqa":
            k, v = sdev.gqa_rows(w.seed_val, req, pos, w.hkv, w.dk)
        else:
            k, v = sdev.latent_rows(w.seed_val, req, pos), None
        if dw.rank is None:
            dcp_kv_append(dw.desc, req, pos, k, v)
        else:
            dcp_kv_append_rank(dw.desc, dw.rank, req, pos, k, v)
    torch.cuda.synchronize()
