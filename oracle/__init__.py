"""Float64 CPU oracle for sequence-sharded paged decode attention.

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package.  It shares
no code with the CUDA path (``sequence_sharded_paged_b200``); its one shared
input is the seeded generator (``synth``).

The arithmetic lives in ``oracle.c`` (plain C, float64, OpenMP over
(request, head block)); this module loads ``liboracle.so`` and marshals numpy
arrays.  Definitions followed (see the header of ``oracle.c`` for each):

* ownership / local packing / shard counts: "Efficient Decode Context
  Parallelism with vLLM for Long Context Workloads", section 4, and the
  "Decode Context Parallel Guide", Constraints (``cp_kv_cache_interleave_size``);
* partial attention + LSE and the LSE-weighted merge: the blog, section 4.1;
* MLA absorbed latent (key = 576-wide row, value = first 512): section 5.3;
* GQA head broadcast g(h) = h // (Hq/Hkv): section 5.4.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against brute force, closed forms, library routines or invariants; none is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liboracle.so")
SRC = os.path.join(HERE, "oracle.c")

ORC_OK = 0
ORC_ERR_ARG = 1
ORC_ERR_UNALLOCATED = 3


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (IEEE arithmetic: no fast-math, no contraction)."""
    if (not force and os.path.exists(LIB_PATH)
            and os.path.getmtime(LIB_PATH) >= max(os.path.getmtime(SRC),
                                                  os.path.getmtime(os.path.join(HERE, "..", "synth", "synth_hash.h")))):
        return LIB_PATH
    cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-std=c11", "-o", LIB_PATH, SRC, "-lm"]
    subprocess.run(cmd, check=True, cwd=HERE)
    return LIB_PATH


class _Cache(ctypes.Structure):
    _fields_ = [
        ("kind", ctypes.c_int32), ("fp8", ctypes.c_int32),
        ("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
        ("Dk", ctypes.c_int32), ("Dv", ctypes.c_int32),
        ("scale", ctypes.c_double),
        ("use_synth", ctypes.c_int32),
        ("K", ctypes.c_void_p), ("V", ctypes.c_void_p),
        ("Lmax", ctypes.c_int64),
        ("seed", ctypes.c_uint64),
    ]


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        L.orc_owner.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32]
        L.orc_owner.restype = ctypes.c_int32
        L.orc_local_index.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32]
        L.orc_local_index.restype = ctypes.c_int64
        L.orc_shard_count.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
        L.orc_shard_count.restype = ctypes.c_int64
        L.orc_shard_counts.argtypes = [ctypes.c_int32, P, ctypes.c_int32, ctypes.c_int32, P]
        L.orc_shard_counts.restype = None
        L.orc_shard_map.argtypes = [ctypes.c_int64, P, P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, P,
                                    ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, P, P, P]
        L.orc_shard_map.restype = ctypes.c_int
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_encode.argtypes = [ctypes.c_double]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_quantize_row_e4m3.argtypes = [P, ctypes.c_int32, P, P]
        L.orc_quantize_row_e4m3.restype = None
        L.orc_quantize_rows_e4m3.argtypes = [ctypes.c_int64, ctypes.c_int32, P, P, P]
        L.orc_quantize_rows_e4m3.restype = None
        L.orc_decode.argtypes = [ctypes.POINTER(_Cache), P, P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                 P, ctypes.c_int32, P, P]
        L.orc_decode.restype = ctypes.c_int
        L.orc_decode_multi.argtypes = [ctypes.POINTER(_Cache), P, P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                       ctypes.c_int32, P, P]
        L.orc_decode_multi.restype = ctypes.c_int
        L.orc_merge.argtypes = [ctypes.c_int32] * 4 + [P] * 4
        L.orc_merge.restype = None
        L.orc_synth_bf16.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64, P, P]
        L.orc_synth_bf16.restype = None
        L.orc_num_threads.argtypes = []
        L.orc_num_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


# ----------------------------------------------------------------------------
# shard map
# ----------------------------------------------------------------------------

def owner(p: int, N: int, I: int) -> int:
    return lib().orc_owner(p, N, I)


def local_index(p: int, N: int, I: int) -> int:
    return lib().orc_local_index(p, N, I)


def shard_count(L: int, N: int, I: int, n: int) -> int:
    return lib().orc_shard_count(L, N, I, n)


def shard_counts(seq_lens, N: int, I: int) -> np.ndarray:
    sl = np.ascontiguousarray(seq_lens, dtype=np.int64)
    out = np.zeros((N, sl.size), dtype=np.int64)
    lib().orc_shard_counts(sl.size, _p(sl), N, I, _p(out))
    return out


def shard_map(pos, req, N: int, I: int, P: int, block_tables: np.ndarray, num_pages: int):
    """Returns (status, rank int32, local int32, slot int64)."""
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    req = None if req is None else np.ascontiguousarray(req, dtype=np.int32)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    n = pos.size
    rank = np.zeros(n, np.int32)
    local = np.zeros(n, np.int32)
    slot = np.zeros(n, np.int64)
    st = lib().orc_shard_map(n, _p(pos), None if req is None else _p(req), N, I, P, _p(bt), bt.shape[1],
                             bt.shape[2], num_pages, _p(rank), _p(local), _p(slot))
    return st, rank, local, slot


# ----------------------------------------------------------------------------
# e4m3
# ----------------------------------------------------------------------------

def e4m3_decode(code: int) -> float:
    return lib().orc_e4m3_decode(code)


def e4m3_encode(x: float) -> int:
    return lib().orc_e4m3_encode(float(x))


def quantize_row_e4m3(row_bf16: np.ndarray):
    """(codes uint8 [W], scale float32) for one latent row given as bf16 bits."""
    r = np.ascontiguousarray(row_bf16, dtype=np.uint16)
    codes = np.zeros(r.size, np.uint8)
    sc = np.zeros(1, np.float32)
    lib().orc_quantize_row_e4m3(_p(r), r.size, _p(codes), _p(sc))
    return codes, float(sc[0])


def quantize_rows_e4m3(rows_bf16: np.ndarray):
    """Row-wise quantisation of rows [n][W] (bf16 bits): (codes uint8 [n][W], scales float32 [n])."""
    r = np.ascontiguousarray(rows_bf16, dtype=np.uint16)
    n, W = r.shape
    codes = np.zeros((n, W), np.uint8)
    sc = np.zeros(n, np.float32)
    lib().orc_quantize_rows_e4m3(n, W, _p(r), _p(codes), _p(sc))
    return codes, sc


def e4m3_table() -> np.ndarray:
    """float64 value of each of the 256 e4m3 codes (NaN for the NaN codes)."""
    return np.array([e4m3_decode(c) for c in range(256)])


# ----------------------------------------------------------------------------
# decode attention
# ----------------------------------------------------------------------------

def _decode(cache: _Cache, q: np.ndarray, seq_lens, N: int, I: int, shard: int, req_list=None):
    q = np.ascontiguousarray(q, dtype=np.float64)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int64)
    B, Hq, Dv = cache.B, cache.Hq, cache.Dv
    O = np.zeros((B, Hq, Dv), np.float64)
    lse = np.zeros((B, Hq), np.float64)
    rl = None if req_list is None else np.ascontiguousarray(req_list, dtype=np.int32)
    st = lib().orc_decode(ctypes.byref(cache), _p(q), _p(sl), N, I, shard, None if rl is None else _p(rl),
                          0 if rl is None else rl.size, _p(O), _p(lse))
    if st != ORC_OK:
        raise ValueError(f"orc_decode: bad arguments (status {st})")
    return O, lse


def decode_arrays(kind: str, q, K, V, seq_lens, scale: float, hkv: int = 1, dv: int | None = None,
                  N: int = 1, I: int = 1, shard: int = -1, req_list=None):
    """Decode attention from dense logical float64 arrays.

    GQA: K [B][Lmax][Hkv][Dk], V [B][Lmax][Hkv][Dv].  MLA: K = latent rows
    [B][Lmax][Dk] (value = first ``dv`` entries), V ignored.
    shard = -1: unsharded; shard = n: that shard's partial under (N, I)."""
    q = np.asarray(q, np.float64)
    B, Hq, Dk = q.shape
    K = np.ascontiguousarray(K, dtype=np.float64)
    if kind == "mla":
        Vd = dv if dv is not None else Dk
        c = _Cache(1, 0, B, Hq, 1, Dk, Vd, scale, 0, _p(K).value, None, K.shape[1], 0)
        keep = (K,)
    else:
        V = np.ascontiguousarray(V, dtype=np.float64)
        c = _Cache(0, 0, B, Hq, K.shape[2], Dk, V.shape[3], scale, 0, _p(K).value, _p(V).value, K.shape[1], 0)
        keep = (K, V)
    out = _decode(c, q, seq_lens, N, I, shard, req_list)
    del keep
    return out


def decode_synth(kind: str, dtype: str, seed: int, q, seq_lens, scale: float, hkv: int, dk: int, dv: int,
                 N: int = 1, I: int = 1, shard: int = -1, req_list=None):
    """Decode attention with K/V (or latent) rows regenerated on the fly from the
    seeded generator (``synth``); fp8 rows are quantised by the oracle itself."""
    q = np.asarray(q, np.float64)
    B, Hq, Dk = q.shape
    assert Dk == dk
    c = _Cache(1 if kind == "mla" else 0, 1 if dtype == "fp8" else 0, B, Hq, hkv, dk, dv, scale, 1, None, None,
               0, seed)
    return _decode(c, q, seq_lens, N, I, shard, req_list)


def _decode_multi(cache: _Cache, q: np.ndarray, seq_lens, N: int, I: int, shard: int):
    q = np.ascontiguousarray(q, dtype=np.float64)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int64)
    B, QL, Hq, _ = q.shape
    O = np.zeros((B, QL, Hq, cache.Dv), np.float64)
    lse = np.zeros((B, QL, Hq), np.float64)
    st = lib().orc_decode_multi(ctypes.byref(cache), _p(q), _p(sl), QL, N, I, shard, _p(O), _p(lse))
    if st != ORC_OK:
        raise ValueError(f"orc_decode_multi: bad arguments (status {st})")
    return O, lse


def decode_multi_arrays(kind: str, q, K, V, seq_lens, scale: float, dv: int | None = None,
                        N: int = 1, I: int = 1, shard: int = -1):
    """Decode with QL query tokens per request (speculative decoding under DCP, blog section 6):
    q [B][QL][Hq][Dk]; request b holds seq_lens[b] positions, its QL new tokens last, and query
    token j attends positions p <= seq_lens[b] - QL + j.  K, V, dv, N, I and shard as in
    decode_arrays.  Returns O [B][QL][Hq][Dv], lse [B][QL][Hq]."""
    q = np.asarray(q, np.float64)
    B, QL, Hq, Dk = q.shape
    K = np.ascontiguousarray(K, dtype=np.float64)
    if kind == "mla":
        Vd = dv if dv is not None else Dk
        c = _Cache(1, 0, B, Hq, 1, Dk, Vd, scale, 0, _p(K).value, None, K.shape[1], 0)
        keep = (K,)
    else:
        V = np.ascontiguousarray(V, dtype=np.float64)
        c = _Cache(0, 0, B, Hq, K.shape[2], Dk, V.shape[3], scale, 0, _p(K).value, _p(V).value, K.shape[1], 0)
        keep = (K, V)
    out = _decode_multi(c, q, seq_lens, N, I, shard)
    del keep
    return out


def decode_multi_synth(kind: str, dtype: str, seed: int, q, seq_lens, scale: float, hkv: int, dk: int, dv: int,
                       N: int = 1, I: int = 1, shard: int = -1):
    """decode_multi_arrays with K/V (or latent) rows regenerated on the fly from the
    seeded generator, as decode_synth does: q [B][QL][Hq][Dk] -> O [B][QL][Hq][Dv],
    lse [B][QL][Hq]."""
    q = np.asarray(q, np.float64)
    B, QL, Hq, Dk = q.shape
    assert Dk == dk
    c = _Cache(1 if kind == "mla" else 0, 1 if dtype == "fp8" else 0, B, Hq, hkv, dk, dv, scale, 1, None, None,
               0, seed)
    return _decode_multi(c, q, seq_lens, N, I, shard)


def merge(O_part: np.ndarray, lse_part: np.ndarray):
    """LSE-weighted merge: O_part [N][B][H][Dv], lse_part [N][B][H] -> (O, lse)."""
    O_part = np.ascontiguousarray(O_part, dtype=np.float64)
    lse_part = np.ascontiguousarray(lse_part, dtype=np.float64)
    N, B, H, Dv = O_part.shape
    O = np.zeros((B, H, Dv), np.float64)
    lse = np.zeros((B, H), np.float64)
    lib().orc_merge(N, B, H, Dv, _p(O_part), _p(lse_part), _p(O), _p(lse))
    return O, lse


def synth_bf16(seed: int, tensor: int, idx) -> np.ndarray:
    idx = np.ascontiguousarray(idx, dtype=np.uint64)
    out = np.zeros(idx.size, np.uint16)
    lib().orc_synth_bf16(seed, tensor, idx.size, _p(idx), _p(out))
    return out


def num_threads() -> int:
    return lib().orc_num_threads()
