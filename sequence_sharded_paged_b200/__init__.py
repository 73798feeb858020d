"""Python binding of libdcp: decode attention over a sequence-sharded paged KV
cache (Decode Context Parallelism) on NVIDIA B200.

This module only marshals arguments: torch tensors become device pointers,
the current torch stream becomes the cudaStream_t, and a non-zero status
becomes :class:`DcpError`.  Every step of the path runs in the CUDA kernels of
``libdcp.so`` (built in-tree from ``csrc/`` by ``build.py``).  There is no
fallback: if the library is missing, importing the entry points raises.

Entry points (same names as ``include/dcp.h``): ``dcp_shard_counts``,
``dcp_shard_map``, ``dcp_kv_append``, ``dcp_decode_workspace_size``,
``dcp_decode_workspace_size_ex``, ``dcp_decode_partial``,
``dcp_decode_partial_multi``, ``dcp_decode_merged``,
``dcp_decode_partial_noalloc``, ``dcp_merge``, ``dcp_get_device_status``, and for
one rank of a multi-GPU group ``dcp_kv_append_rank``, ``dcp_decode_rank``,
``dcp_lse_rescale`` (the collectives around them are in ``parallel.py``).
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdcp.so")

DCP_OK = 0
DCP_ERR_INVALID_ARG = 1
DCP_ERR_UNSUPPORTED = 2
DCP_ERR_UNALLOCATED_PAGE = 3
DCP_ERR_WORKSPACE_TOO_SMALL = 4
DCP_ERR_CUDA = 5
DCP_ERR_MISALIGNED = 6
DCP_ERR_TIMEOUT = 7

DCP_GQA = 0
DCP_MLA = 1
DCP_BF16 = 0
DCP_FP8_E4M3 = 1

DCP_DECODE_PARTIAL = 0
DCP_DECODE_MERGED = 1
DCP_DECODE_RANK = 2

EXPORTED = ("dcp_status_string", "dcp_shard_counts", "dcp_shard_map", "dcp_kv_append",
            "dcp_decode_workspace_size", "dcp_decode_workspace_size_ex", "dcp_decode_partial",
            "dcp_decode_partial_multi", "dcp_decode_merged", "dcp_decode_partial_noalloc", "dcp_merge",
            "dcp_get_device_status", "dcp_kv_append_rank", "dcp_decode_rank", "dcp_lse_rescale")


class DcpError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class CacheDesc(ctypes.Structure):
    """Mirror of ``dcp_cache_desc``."""
    _fields_ = [
        ("kind", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("n_shards", ctypes.c_int32), ("interleave", ctypes.c_int32),
        ("page_size", ctypes.c_int32), ("num_pages", ctypes.c_int32),
        ("hq", ctypes.c_int32), ("hkv", ctypes.c_int32), ("dk", ctypes.c_int32), ("dv", ctypes.c_int32),
        ("scale", ctypes.c_float),
        ("batch", ctypes.c_int32), ("max_local_pages", ctypes.c_int32), ("reserved0", ctypes.c_int32),
        ("k_pages", ctypes.c_void_p), ("v_pages", ctypes.c_void_p),
        ("kv_scales", ctypes.c_void_p), ("block_tables", ctypes.c_void_p),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libdcp.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libdcp.so is not built ({LIB_PATH}); run __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        D = ctypes.POINTER(CacheDesc)
        L.dcp_status_string.argtypes = [ctypes.c_int]
        L.dcp_status_string.restype = ctypes.c_char_p
        L.dcp_shard_counts.argtypes = [i32, P, i32, i32, P, P]
        L.dcp_shard_map.argtypes = [D, i64, P, P, P, P, P, P]
        L.dcp_kv_append.argtypes = [D, i64, P, P, P, P, P]
        L.dcp_decode_workspace_size.argtypes = [D, i32]
        L.dcp_decode_workspace_size.restype = ctypes.c_size_t
        L.dcp_decode_partial.argtypes = [D, i32, P, P, P, P, P, ctypes.c_size_t, P]
        L.dcp_decode_workspace_size_ex.argtypes = [D, i32, i32, i32]
        L.dcp_decode_workspace_size_ex.restype = ctypes.c_size_t
        L.dcp_decode_partial_multi.argtypes = [D, i32, i32, P, P, P, P, P, ctypes.c_size_t, P]
        L.dcp_decode_merged.argtypes = [D, i32, i32, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.dcp_kv_append_rank.argtypes = [D, i32, i64, P, P, P, P, P]
        L.dcp_decode_rank.argtypes = [D, i32, i32, i32, P, P, P, P, P, ctypes.c_size_t, P]
        L.dcp_lse_rescale.argtypes = [i32, i32, i32, i32, i32, P, P, P, P, P]
        L.dcp_decode_partial_noalloc.argtypes = [D, i32, P, P, P, P, P]
        L.dcp_merge.argtypes = [i32, i32, i32, i32, P, P, P, P, P]
        L.dcp_get_device_status.argtypes = [ctypes.POINTER(i32), P]
        L.dcp_selftest_bounded_wait.argtypes = [P, P]
        for name in ("dcp_shard_counts", "dcp_shard_map", "dcp_kv_append", "dcp_decode_partial",
                     "dcp_decode_partial_multi", "dcp_decode_merged", "dcp_decode_partial_noalloc", "dcp_merge",
                     "dcp_get_device_status", "dcp_kv_append_rank", "dcp_decode_rank", "dcp_lse_rescale",
                     "dcp_selftest_bounded_wait"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().dcp_status_string(int(status)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int, where: str):
    if status != DCP_OK:
        raise DcpError(status, where)


def make_cache_desc(*, kind: int, dtype: int, n_shards: int, interleave: int, page_size: int, num_pages: int,
                    hq: int, hkv: int, dk: int, dv: int, scale: float, batch: int, block_tables,
                    k_pages=None, v_pages=None, kv_scales=None) -> CacheDesc:
    """Build a ``dcp_cache_desc`` from torch tensors (block_tables int32
    [N][B][max_local_pages]); the tensors must outlive every call using it."""
    return CacheDesc(kind, dtype, n_shards, interleave, page_size, num_pages, hq, hkv, dk, dv, float(scale), batch,
                     int(block_tables.shape[2]), 0, _ptr(k_pages), _ptr(v_pages), _ptr(kv_scales),
                     _ptr(block_tables))


def dcp_shard_counts(seq_lens, n_shards: int, interleave: int, counts_out, stream=None) -> None:
    _check(lib().dcp_shard_counts(seq_lens.numel(), _ptr(seq_lens), n_shards, interleave, _ptr(counts_out),
                                  _stream(stream)), "dcp_shard_counts")


def dcp_shard_map(desc: CacheDesc, pos, req, rank_out, local_out, slot_out, stream=None) -> None:
    _check(lib().dcp_shard_map(ctypes.byref(desc), pos.numel(), _ptr(pos), _ptr(req), _ptr(rank_out),
                               _ptr(local_out), _ptr(slot_out), _stream(stream)), "dcp_shard_map")


def dcp_kv_append(desc: CacheDesc, req, pos, k_new, v_new=None, stream=None) -> None:
    _check(lib().dcp_kv_append(ctypes.byref(desc), pos.numel(), _ptr(req), _ptr(pos), _ptr(k_new), _ptr(v_new),
                               _stream(stream)), "dcp_kv_append")


def dcp_decode_workspace_size(desc: CacheDesc, batch: int) -> int:
    return int(lib().dcp_decode_workspace_size(ctypes.byref(desc), batch))


def dcp_decode_partial(desc: CacheDesc, q, seq_lens, o_partial, lse, ws, stream=None) -> None:
    _check(lib().dcp_decode_partial(ctypes.byref(desc), q.shape[0], _ptr(q), _ptr(seq_lens), _ptr(o_partial),
                                    _ptr(lse), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "dcp_decode_partial")


def dcp_decode_workspace_size_ex(desc: CacheDesc, batch: int, q_len: int = 1, mode: int = DCP_DECODE_PARTIAL) -> int:
    """Workspace bytes of the decode call of `mode` (DCP_DECODE_PARTIAL, _MERGED or _RANK)."""
    return int(lib().dcp_decode_workspace_size_ex(ctypes.byref(desc), batch, q_len, int(mode)))


def dcp_decode_partial_multi(desc: CacheDesc, q, seq_lens, o_partial, lse, ws, stream=None) -> None:
    """q bf16 [B][q_len][hq][dk] -> o_partial [N][B][q_len][hq][dv], lse [N][B][q_len][hq]."""
    _check(lib().dcp_decode_partial_multi(ctypes.byref(desc), q.shape[0], q.shape[1], _ptr(q), _ptr(seq_lens),
                                          _ptr(o_partial), _ptr(lse), _ptr(ws), ws.numel() * ws.element_size(),
                                          _stream(stream)), "dcp_decode_partial_multi")


def dcp_decode_merged(desc: CacheDesc, q, seq_lens, out, lse_out, ws, finish_ns=None, stream=None) -> None:
    """Partial attention of every shard and the LSE merge in one launch sequence.
    q bf16 [B][hq][dk] (one query token) or [B][q_len][hq][dk]; out / lse_out have
    q's leading dimensions with dv / no trailing dimension; finish_ns int64 [B] or None."""
    q_len = 1 if q.dim() == 3 else q.shape[1]
    _check(lib().dcp_decode_merged(ctypes.byref(desc), q.shape[0], q_len, _ptr(q), _ptr(seq_lens), _ptr(out),
                                   _ptr(lse_out), _ptr(finish_ns), _ptr(ws), ws.numel() * ws.element_size(),
                                   _stream(stream)), "dcp_decode_merged")


def dcp_kv_append_rank(desc: CacheDesc, rank: int, req, pos, k_new, v_new=None, stream=None) -> None:
    _check(lib().dcp_kv_append_rank(ctypes.byref(desc), rank, pos.numel(), _ptr(req), _ptr(pos), _ptr(k_new),
                                    _ptr(v_new), _stream(stream)), "dcp_kv_append_rank")


def dcp_decode_rank(desc: CacheDesc, rank: int, q, seq_lens, o, lse, ws, stream=None) -> None:
    """Rank `rank`'s partial: q bf16 [B][hq][dk] or [B][q_len][hq][dk] -> o, lse with q's leading dims."""
    q_len = 1 if q.dim() == 3 else q.shape[1]
    _check(lib().dcp_decode_rank(ctypes.byref(desc), rank, q.shape[0], q_len, _ptr(q), _ptr(seq_lens), _ptr(o),
                                 _ptr(lse), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "dcp_decode_rank")


def dcp_lse_rescale(lse_all, rank: int, o, o_rs, lse_out=None, stream=None) -> None:
    """lse_all [N][B][H], o [B][H][Dv] -> o_rs [N][B][H/N][Dv] (reduce-scatter layout), lse_out [B][H]."""
    N, B, H = lse_all.shape
    _check(lib().dcp_lse_rescale(N, rank, B, H, o.shape[-1], _ptr(lse_all), _ptr(o), _ptr(o_rs), _ptr(lse_out),
                                 _stream(stream)), "dcp_lse_rescale")


# size of the library's built-in decode scratch (DCP_STATIC_SCRATCH_BYTES in dcp.h)
DCP_STATIC_SCRATCH_BYTES = 64 << 20


def dcp_decode_partial_noalloc(desc: CacheDesc, q, seq_lens, o_partial, lse, stream=None) -> None:
    """dcp_decode_partial on the library's built-in scratch; allocates nothing.
    Calls that can overlap in time race on that scratch."""
    _check(lib().dcp_decode_partial_noalloc(ctypes.byref(desc), q.shape[0], _ptr(q), _ptr(seq_lens),
                                            _ptr(o_partial), _ptr(lse), _stream(stream)),
           "dcp_decode_partial_noalloc")


def dcp_merge(o_partial, lse, out, lse_out=None, stream=None) -> None:
    N, B, H, Dv = o_partial.shape
    _check(lib().dcp_merge(N, B, H, Dv, _ptr(o_partial), _ptr(lse), _ptr(out), _ptr(lse_out), _stream(stream)),
           "dcp_merge")


def dcp_selftest_bounded_wait(result, stream=None) -> None:
    """Launches the bounded-wait self-test: result int64 [>= 3] on the device receives
    (wait completed?, abort flag, nanoseconds waited); the status word then holds DCP_ERR_TIMEOUT."""
    _check(lib().dcp_selftest_bounded_wait(_ptr(result), _stream(stream)), "dcp_selftest_bounded_wait")


def dcp_get_device_status(stream=None) -> int:
    v = ctypes.c_int32(0)
    _check(lib().dcp_get_device_status(ctypes.byref(v), _stream(stream)), "dcp_get_device_status")
    return int(v.value)
