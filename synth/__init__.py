"""Seeded synthetic inputs shared by the oracle, the tests and the benchmark.

This module holds no arithmetic of the attention method.  It provides:

* the counter-based value generator defined in ``synth_hash.h`` (a numpy
  restatement, bit-identical to the C header that the oracle compiles and to
  the CUDA fill kernels in ``synth_fill.cu``);
* request-length generators shaped like the long-context agentic trace
  described in "Efficient Decode Context Parallelism with vLLM for Long Context
  Workloads", section 2.1 (median ~67k input tokens, 47% under 64k, 18% under
  8k, ~8% over 128k, ~3-4% over 256k, tail to ~1M);
* a random page permutation dealt into per-shard block tables (the caller
  supplies how many pages each (shard, request) needs);
* the five workload configurations with their seeds.

Stream layout (tensor ids from ``synth_hash.h``):

* ``q``: tensor ``SYNTH_T_Q + 64*step``, flat index ``(b*Hq + h)*Dk + d``;
* GQA keys/values: tensors ``SYNTH_T_K`` / ``SYNTH_T_V``, index
  ``synth_kv_index(b, p, g, d, Hkv, D)``;
* MLA latent rows: tensor ``SYNTH_T_LATENT``, index
  ``synth_kv_index(b, p, 0, d, 1, 576)``.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass, field

import numpy as np

_M64 = np.uint64(0xFFFFFFFFFFFFFFFF)
GOLDEN = 0x9E3779B97F4A7C15
TMUL = 0xD1B54A32D192ED03
NORM = float.fromhex("0x1.bb67ae86627e7p-16")

T_Q = 1
T_K = 2
T_V = 3
T_LATENT = 4
T_LENGTHS = 100
T_PAGES = 101

HERE = os.path.dirname(os.path.abspath(__file__))


def _mix_np(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.uint64, copy=True)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        z = z ^ (z >> np.uint64(31))
    return z


def mix(z: int) -> int:
    """SplitMix64 finaliser on a Python int (mod 2**64)."""
    m = (1 << 64) - 1
    z &= m
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & m
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & m
    return z ^ (z >> 31)


def key(seed: int, tensor: int) -> int:
    m = (1 << 64) - 1
    return mix(mix((seed + GOLDEN) & m) ^ ((tensor * TMUL) & m))


def bits(k: int, index) -> np.ndarray:
    """64 random bits of stream ``k`` at element indices ``index`` (array)."""
    idx = np.asarray(index, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(k) + (idx + np.uint64(1)) * np.uint64(GOLDEN)
    return _mix_np(z)


def normal_from_bits(b: np.ndarray) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint64)
    mask = np.uint64(0xFFFF)
    s = ((b & mask).astype(np.int64) + ((b >> np.uint64(16)) & mask).astype(np.int64) +
         ((b >> np.uint64(32)) & mask).astype(np.int64) + ((b >> np.uint64(48)) & mask).astype(np.int64))
    return (s - 131070).astype(np.float64) * NORM


def bf16_bits_from_f64(x: np.ndarray) -> np.ndarray:
    """binary64 -> bfloat16 bits, round to nearest even, straight from the binary64 bits."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    u = x.view(np.uint64)
    sign = u >> np.uint64(63)
    mag = u & np.uint64(0x7FFFFFFFFFFFFFFF)
    e = (mag >> np.uint64(52)).astype(np.int64) - 1023
    m = (mag & np.uint64(0xFFFFFFFFFFFFF)) | np.uint64(1 << 52)
    keep = m >> np.uint64(45)
    rem = m & np.uint64((1 << 45) - 1)
    half = np.uint64(1 << 44)
    up = (rem > half) | ((rem == half) & ((keep & np.uint64(1)) == np.uint64(1)))
    keep = keep + up.astype(np.uint64)
    carry = keep == np.uint64(1 << 8)
    keep = np.where(carry, keep >> np.uint64(1), keep)
    e = e + carry.astype(np.int64)
    be = (e + 127).astype(np.uint64)
    out = (sign << np.uint64(15)) | (be << np.uint64(7)) | (keep & np.uint64(0x7F))
    out = np.where(mag == np.uint64(0), sign << np.uint64(15), out)
    return out.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bits to float64."""
    b = np.asarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def bf16_at(k: int, index) -> np.ndarray:
    return bf16_bits_from_f64(normal_from_bits(bits(k, index)))


def kv_index(b, p, g, d, hkv: int, w: int) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint64)
    p = np.asarray(p, dtype=np.uint64)
    g = np.asarray(g, dtype=np.uint64)
    d = np.asarray(d, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return (((b * np.uint64(hkv) + g) << np.uint64(24)) + p) * np.uint64(w) + d


def q_tensor(step: int) -> int:
    return T_Q + 64 * step


def q_bf16(seed: int, B: int, Hq: int, Dk: int, step: int = 0) -> np.ndarray:
    """q[b][h][d] as bf16 bits, shape (B, Hq, Dk)."""
    k = key(seed, q_tensor(step))
    return bf16_at(k, np.arange(B * Hq * Dk, dtype=np.uint64)).reshape(B, Hq, Dk)


def kv_rows_bf16(seed: int, tensor: int, b: int, positions, hkv: int, w: int) -> np.ndarray:
    """Logical rows of request ``b`` at ``positions``: shape (len(pos), hkv, w), bf16 bits."""
    pos = np.asarray(positions, dtype=np.uint64)
    k = key(seed, tensor)
    idx = kv_index(np.uint64(b), pos[:, None, None], np.arange(hkv, dtype=np.uint64)[None, :, None],
                   np.arange(w, dtype=np.uint64)[None, None, :], hkv, w)
    return bf16_at(k, idx)


# ----------------------------------------------------------------------------
# request lengths
# ----------------------------------------------------------------------------

def _unit(b: np.ndarray) -> np.ndarray:
    """53-bit fraction in [0, 1)."""
    return (np.asarray(b, dtype=np.uint64) >> np.uint64(11)).astype(np.float64) * (1.0 / (1 << 53))


def lengths_uniform(seed: int, B: int, lo: int, hi: int) -> np.ndarray:
    """Integer lengths uniform on [lo, hi] (modulo reduction of 64 random bits)."""
    b = bits(key(seed, T_LENGTHS), np.arange(B, dtype=np.uint64))
    span = np.uint64(hi - lo + 1)
    return (np.uint64(lo) + b % span).astype(np.int64)


# Piecewise log-uniform bands that honour every fraction stated for the trace:
# 18% < 8k, 47% < 64k (so 29% in [8k, 64k)), ~8% > 128k, ~3.5% > 256k, max ~1M.
BIMODAL_BANDS = (
    (1_000, 8_000, 0.18),
    (8_000, 64_000, 0.29),
    (64_000, 128_000, 0.45),
    (128_000, 256_000, 0.045),
    (256_000, 1_000_000, 0.035),
)


def lengths_bimodal(seed: int, B: int, cap: int | None = None) -> np.ndarray:
    """Bimodal long-context lengths (piecewise log-uniform), then the cap rule:
    if the total exceeds ``cap``, every length is multiplied by cap/total,
    floored, and kept >= 1."""
    k = key(seed, T_LENGTHS)
    i = np.arange(B, dtype=np.uint64)
    u_band = _unit(bits(k, 2 * i))
    u_in = _unit(bits(k, 2 * i + np.uint64(1)))
    edges = np.cumsum([p for (_, _, p) in BIMODAL_BANDS])
    edges[-1] = 1.0
    band = np.searchsorted(edges, u_band, side="right")
    band = np.minimum(band, len(BIMODAL_BANDS) - 1)
    lo = np.array([b[0] for b in BIMODAL_BANDS], dtype=np.float64)[band]
    hi = np.array([b[1] for b in BIMODAL_BANDS], dtype=np.float64)[band]
    L = np.floor(lo * np.exp(u_in * np.log(hi / lo))).astype(np.int64)
    L = np.clip(L, 1, None)
    if cap is not None:
        tot = int(L.sum())
        if tot > cap:
            L = np.maximum(1, (L.astype(np.float64) * (cap / tot)).astype(np.int64))
    return L


# ----------------------------------------------------------------------------
# block tables
# ----------------------------------------------------------------------------

def page_permutation(seed: int, num_pages: int) -> np.ndarray:
    """A seeded random permutation of page ids 0..num_pages-1."""
    b = bits(key(seed, T_PAGES), np.arange(num_pages, dtype=np.uint64))
    return np.argsort(b, kind="stable").astype(np.int32)


def deal_block_tables(seed: int, pages_needed: np.ndarray, slack_pages: int = 0):
    """Deal a random permutation of pool pages to (shard, request) slots in order.

    ``pages_needed``: int array (N, B) of pages each shard needs per request.
    Returns (block_tables int32 (N, B, max_local_pages) with -1 for unused,
    num_pages).  The pool holds sum(pages_needed) + slack_pages pages."""
    pages_needed = np.asarray(pages_needed, dtype=np.int64)
    N, B = pages_needed.shape
    total = int(pages_needed.sum())
    num_pages = total + int(slack_pages)
    perm = page_permutation(seed, max(num_pages, 1))
    maxp = max(1, int(pages_needed.max()) if pages_needed.size else 1)
    bt = np.full((N, B, maxp), -1, dtype=np.int32)
    flat_n = pages_needed.reshape(-1)
    offs = np.concatenate([[0], np.cumsum(flat_n)])
    for i in range(N * B):
        c = int(flat_n[i])
        if c:
            bt.reshape(N * B, maxp)[i, :c] = perm[offs[i]:offs[i] + c]
    return bt, num_pages


# ----------------------------------------------------------------------------
# workload configurations
# ----------------------------------------------------------------------------

@dataclass
class Workload:
    name: str
    kind: str            # "gqa" or "mla"
    dtype: str           # "bf16" or "fp8"
    B: int
    hq: int
    hkv: int
    dk: int
    dv: int
    page_size: int
    n_shards: int
    interleave: int
    scale: float
    seed_len: int
    seed_val: int
    lengths: np.ndarray = field(repr=False, default=None)

    @property
    def kv_bytes_per_token(self) -> int:
        if self.kind == "gqa":
            return 2 * self.hkv * self.dk * 2
        return 576 * 2 if self.dtype == "bf16" else 576 + 4


def workload(cfg: int, n_shards: int | None = None, interleave: int | None = None) -> Workload:
    """The five workload configurations (1-based), lengths included."""
    if cfg == 1:
        w = Workload("gqa-tiny B2 Hq8/Hkv2 D64 P16", "gqa", "bf16", 2, 8, 2, 64, 64, 16, 2, 1,
                     1.0 / 8.0, 1001, 2001)
        w.lengths = np.array([300, 1000], dtype=np.int64)
    elif cfg == 2:
        w = Workload("mla-v2lite B8 Hq16 576/512 P64", "mla", "bf16", 8, 16, 1, 576, 512, 64, 2, 1,
                     1.0 / math.sqrt(192.0), 1002, 2002)
        w.lengths = lengths_uniform(1002, 8, 8_000, 32_000)
    elif cfg == 3:
        w = Workload("gqa-qwen3 B128 Hq64/Hkv4 D128 P16", "gqa", "bf16", 128, 64, 4, 128, 128, 16, 8, 128,
                     1.0 / math.sqrt(128.0), 1003, 2003)
        w.lengths = lengths_uniform(1003, 128, 32_000, 128_000)
    elif cfg == 4:
        w = Workload("mla-kimi-bf16 B64 Hq64 576/512 P64", "mla", "bf16", 64, 64, 1, 576, 512, 64, 8, 1,
                     1.0 / math.sqrt(192.0), 1004, 2004)
        w.lengths = lengths_bimodal(1004, 64, cap=8_000_000)
    elif cfg == 5:
        w = Workload("mla-kimi-fp8 B512 Hq64 576/512 P64", "mla", "fp8", 512, 64, 1, 576, 512, 64, 8, 1,
                     1.0 / math.sqrt(192.0), 1005, 2005)
        w.lengths = lengths_bimodal(1005, 512, cap=24_000_000)
    else:
        raise ValueError(f"unknown workload config {cfg}")
    if n_shards is not None:
        w.n_shards = int(n_shards)
    if interleave is not None:
        w.interleave = int(interleave)
    return w


# ----------------------------------------------------------------------------
# device fill library (CUDA build of synth_hash.h)
# ----------------------------------------------------------------------------

_LIB = None


def device_lib():
    """Load ``libsynth.so`` (CUDA fill kernels built from synth_fill.cu)."""
    global _LIB
    if _LIB is None:
        path = os.path.join(HERE, "libsynth.so")
        if not os.path.exists(path):
            raise RuntimeError(f"libsynth.so not built ({path}); run __graft_entry__.build()")
        lib = ctypes.CDLL(path)
        lib.synth_fill_flat.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_void_p]
        lib.synth_fill_flat.restype = ctypes.c_int
        lib.synth_fill_kv_rows.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_int32, ctypes.c_int32, ctypes.c_uint64, ctypes.c_void_p]
        lib.synth_fill_kv_rows.restype = ctypes.c_int
        _LIB = lib
    return _LIB
