"""The C-ABI libraries load on a CPU-only host, export every declared entry
point, and reject bad arguments on the host before touching a GPU."""
import ctypes
import os
import re
import subprocess
import tempfile


import sequence_sharded_paged_b200 as dcp
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dcp.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dcp_[a-z_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for n in ("dcp_shard_map", "dcp_shard_counts", "dcp_kv_append", "dcp_decode_workspace_size",
              "dcp_decode_partial", "dcp_merge", "dcp_get_device_status", "dcp_status_string"):
        assert n in names


def test_libdcp_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", dcp.LIB_PATH], capture_output=True, text=True, check=True)
    exported = set(re.findall(r" T (\w+)", out.stdout))
    missing = [n for n in _declared_functions() if n not in exported]
    assert not missing, missing
    lib = dcp.lib()
    for n in _declared_functions():
        assert hasattr(lib, n)


def test_python_binding_names_match_header():
    for n in _declared_functions():
        if n == "dcp_status_string":
            continue
        assert callable(getattr(dcp, n)), n


def test_status_strings():
    assert dcp.status_string(dcp.DCP_OK) == "ok"
    assert dcp.status_string(dcp.DCP_ERR_UNALLOCATED_PAGE) == "unallocated page"
    assert dcp.status_string(99) == "unknown status"


def test_cache_desc_layout_matches_c_struct():
    src = r"""
    #include <stdio.h>
    #include <stddef.h>
    #include "dcp.h"
    int main(void) {
      printf("%zu %zu %zu %zu %zu %zu %zu\n", sizeof(dcp_cache_desc), offsetof(dcp_cache_desc, scale),
             offsetof(dcp_cache_desc, batch), offsetof(dcp_cache_desc, k_pages), offsetof(dcp_cache_desc, v_pages),
             offsetof(dcp_cache_desc, kv_scales), offsetof(dcp_cache_desc, block_tables));
      return 0;
    }
    """
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        vals = [int(x) for x in subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split()]
    D = dcp.CacheDesc
    assert vals == [ctypes.sizeof(D), D.scale.offset, D.batch.offset, D.k_pages.offset, D.v_pages.offset,
                    D.kv_scales.offset, D.block_tables.offset]


def test_host_validation_without_gpu():
    L = dcp.lib()
    # invalid sizes are rejected before any CUDA call
    assert L.dcp_shard_counts(0, None, 2, 1, None, None) == dcp.DCP_ERR_INVALID_ARG
    assert L.dcp_merge(0, 1, 1, 4, None, None, None, None, None) == dcp.DCP_ERR_INVALID_ARG
    assert L.dcp_kv_append(None, 1, None, None, None, None, None) == dcp.DCP_ERR_INVALID_ARG
    assert L.dcp_shard_map(None, 1, None, None, None, None, None, None) == dcp.DCP_ERR_INVALID_ARG
    assert L.dcp_get_device_status(None, None) == dcp.DCP_ERR_INVALID_ARG
    d = dcp.CacheDesc()
    assert L.dcp_decode_workspace_size(ctypes.byref(d), 1) == 0
    d.kind, d.dtype, d.n_shards, d.interleave, d.page_size = dcp.DCP_MLA, dcp.DCP_BF16, 2, 1, 64
    d.num_pages, d.hq, d.hkv, d.dk, d.dv, d.batch, d.max_local_pages = 10, 64, 1, 576, 512, 1, 4
    d.block_tables = 16
    assert L.dcp_decode_partial(ctypes.byref(d), 1, None, None, None, None, None, 0, None) == \
        dcp.DCP_ERR_INVALID_ARG
    d.page_size = 32
    assert L.dcp_shard_map(ctypes.byref(d), 1, 16, None, 16, 16, 16, None) == dcp.DCP_ERR_UNSUPPORTED
    d.page_size, d.dk = 64, 128
    assert L.dcp_shard_map(ctypes.byref(d), 1, 16, None, 16, 16, 16, None) == dcp.DCP_ERR_UNSUPPORTED
    d.dk, d.block_tables = 576, 8
    assert L.dcp_shard_map(ctypes.byref(d), 1, 16, None, 16, 16, 16, None) == dcp.DCP_ERR_MISALIGNED


def _valid_mla_desc(dtype):
    d = dcp.CacheDesc()
    d.kind, d.dtype, d.n_shards, d.interleave, d.page_size = dcp.DCP_MLA, dtype, 2, 1, 64
    d.num_pages, d.hq, d.hkv, d.dk, d.dv, d.batch, d.max_local_pages = 10, 64, 1, 576, 512, 1, 4
    # placeholder addresses: the host checks read pointer values only, never the memory
    d.k_pages, d.block_tables = 256, 16
    d.kv_scales = 512 if dtype == dcp.DCP_FP8_E4M3 else None
    return d


def test_decode_host_validation_without_gpu():
    """dcp_decode_partial and its no-alloc form reject bad descriptors and arguments with the status
    include/dcp.h names, before any CUDA call."""
    L = dcp.lib()
    A = 1024  # a 16-byte-aligned placeholder device address

    def part(d, B=1, q=A, seq=A, o=A, lse=A, ws=A):
        return L.dcp_decode_partial(ctypes.byref(d), B, q, seq, o, lse, ws, 1 << 20, None)

    def noalloc(d, B=1, q=A, seq=A, o=A, lse=A):
        return L.dcp_decode_partial_noalloc(ctypes.byref(d), B, q, seq, o, lse, None)

    for dt in (dcp.DCP_BF16, dcp.DCP_FP8_E4M3):
        d = _valid_mla_desc(dt)
        for f in (part, noalloc):
            assert f(d, B=2) == dcp.DCP_ERR_INVALID_ARG          # B != cache->batch
            assert f(d, q=None) == dcp.DCP_ERR_INVALID_ARG
            assert f(d, lse=None) == dcp.DCP_ERR_INVALID_ARG
            assert f(d, q=A + 8) == dcp.DCP_ERR_MISALIGNED
            assert f(d, o=A + 4) == dcp.DCP_ERR_MISALIGNED
        assert part(d, ws=None) == dcp.DCP_ERR_INVALID_ARG
        assert part(d, ws=A + 8) == dcp.DCP_ERR_MISALIGNED
    cases = [  # (field changes on a valid descriptor, expected status)
        ({"hq": 8}, dcp.DCP_ERR_UNSUPPORTED),                  # MLA heads come in blocks of 16
        ({"dk": 512}, dcp.DCP_ERR_UNSUPPORTED),
        ({"dtype": 7}, dcp.DCP_ERR_INVALID_ARG),
        ({"kind": 5}, dcp.DCP_ERR_INVALID_ARG),
        ({"page_size": 32}, dcp.DCP_ERR_UNSUPPORTED),
        ({"n_shards": 0}, dcp.DCP_ERR_INVALID_ARG),
        ({"max_local_pages": 1 << 26}, dcp.DCP_ERR_INVALID_ARG),  # 2^26 pages x 64 tokens overflows int32
        ({"k_pages": None}, dcp.DCP_ERR_INVALID_ARG),
        ({"k_pages": 264}, dcp.DCP_ERR_MISALIGNED),
        ({"block_tables": 20}, dcp.DCP_ERR_MISALIGNED),
        ({"dtype": dcp.DCP_FP8_E4M3, "kv_scales": None}, dcp.DCP_ERR_INVALID_ARG),
        ({"dtype": dcp.DCP_FP8_E4M3, "kv_scales": 520}, dcp.DCP_ERR_MISALIGNED),
        ({"kind": dcp.DCP_GQA, "hkv": 4, "dk": 128, "dv": 64, "v_pages": 768}, dcp.DCP_ERR_UNSUPPORTED),
        ({"kind": dcp.DCP_GQA, "hkv": 4, "dk": 128, "dv": 128, "v_pages": 768, "dtype": dcp.DCP_FP8_E4M3},
         dcp.DCP_ERR_UNSUPPORTED),
        ({"kind": dcp.DCP_GQA, "hkv": 4, "dk": 128, "dv": 128, "v_pages": None}, dcp.DCP_ERR_INVALID_ARG),
    ]
    for changes, want in cases:
        d = _valid_mla_desc(dcp.DCP_BF16)
        for k, v in changes.items():
            setattr(d, k, v)
        assert part(d) == want, changes
        assert noalloc(d) == want, changes


def test_libsynth_exports():
    lib = synth.device_lib()
    assert hasattr(lib, "synth_fill_flat") and hasattr(lib, "synth_fill_kv_rows")


def test_new_entry_points_host_validation_without_gpu():
    """The multi-query, merged and rank calls reject bad arguments with the status include/dcp.h
    names, before any CUDA call."""
    L = dcp.lib()
    A = 1024
    d = _valid_mla_desc(dcp.DCP_BF16)

    def multi(q_len, B=1, q=A, o=A, lse=A, ws=A):
        return L.dcp_decode_partial_multi(ctypes.byref(d), B, q_len, q, A, o, lse, ws, 1 << 20, None)

    def merged(q_len, fin=None, B=1):
        return L.dcp_decode_merged(ctypes.byref(d), B, q_len, A, A, A, A, fin, A, 1 << 20, None)

    def rank(r, q_len=1):
        return L.dcp_decode_rank(ctypes.byref(d), r, 1, q_len, A, A, A, A, A, 1 << 20, None)

    for f in (multi, merged):
        assert f(0) == dcp.DCP_ERR_INVALID_ARG        # q_len >= 1
        assert f(65) == dcp.DCP_ERR_UNSUPPORTED       # q_len <= 64
        assert f(1, B=2) == dcp.DCP_ERR_INVALID_ARG   # B != cache->batch
    assert multi(2, q=None) == dcp.DCP_ERR_INVALID_ARG
    assert multi(2, o=A + 4) == dcp.DCP_ERR_MISALIGNED
    assert merged(1, fin=A + 8) == dcp.DCP_ERR_MISALIGNED
    assert rank(-1) == dcp.DCP_ERR_INVALID_ARG
    assert rank(2) == dcp.DCP_ERR_INVALID_ARG           # rank < n_shards (2)
    assert L.dcp_kv_append_rank(ctypes.byref(d), 5, 1, None, A, A, None, None) == dcp.DCP_ERR_INVALID_ARG
    # dcp_lse_rescale: N, rank, B, H, Dv, lse_all, o, o_rs, lse_out
    assert L.dcp_lse_rescale(2, 0, 1, 3, 64, A, A, A, None, None) == dcp.DCP_ERR_INVALID_ARG   # H % N
    assert L.dcp_lse_rescale(2, 2, 1, 4, 64, A, A, A, None, None) == dcp.DCP_ERR_INVALID_ARG   # rank < N
    assert L.dcp_lse_rescale(2, 0, 1, 4, 6, A, A, A, None, None) == dcp.DCP_ERR_INVALID_ARG    # Dv % 4
    assert L.dcp_lse_rescale(2, 0, 1, 4, 64, A, A + 4, A, None, None) == dcp.DCP_ERR_MISALIGNED
    assert L.dcp_decode_workspace_size_ex(ctypes.byref(d), 1, 1, 3) == 0  # no such mode


def test_selftest_bounded_wait_host_validation_without_gpu():
    """The bounded-wait self-test checks its result pointer before touching the device."""
    L = dcp.lib()
    assert L.dcp_selftest_bounded_wait(None, None) == dcp.DCP_ERR_INVALID_ARG
    assert L.dcp_selftest_bounded_wait(1024 + 8, None) == dcp.DCP_ERR_MISALIGNED
