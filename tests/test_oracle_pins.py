"""Pins of the float64 oracle to facts other than itself (CPU only).

Each test names what fixes the expected value: the pages' worked example,
brute-force enumeration, a closed form, a library routine, or an invariant
of the mathematics.  A plausible mistake in the oracle (a dropped term, a wrong
sign, a wrong head mapping, the wrong latent slice as value, a transposed
operand, an off-by-one in the local packing) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------
# shard map
# ----------------------------------------------------------------------------

def _owned_positions_brute(L, N, I):
    """Positions owned by each shard, by walking p = 0..L-1 and dealing runs of I
    consecutive positions round-robin to shards 0..N-1."""
    owned = [[] for _ in range(N)]
    shard, run = 0, 0
    for p in range(L):
        owned[shard].append(p)
        run += 1
        if run == I:
            run = 0
            shard = (shard + 1) % N
    return owned


@pytest.mark.parametrize("N", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("I", [1, 2, 3, 16, 50, 64, 128])
def test_shard_map_brute_force(N, I):
    L = 4096 if N * I <= 512 else 3001
    owned = _owned_positions_brute(L, N, I)
    for n in range(N):
        # counts: enumeration
        for Lp in (0, 1, I - 1, I, I * N - 1, I * N, I * N + 1, L // 3, L):
            if Lp < 0:
                continue
            brute = sum(1 for p in owned[n] if p < Lp)
            assert oracle.shard_count(Lp, N, I, n) == brute, (Lp, n)
        # owner and local index: k-th owned position has local index k
        for k, p in enumerate(owned[n][:300] + owned[n][-50:] if len(owned[n]) > 350 else owned[n]):
            kk = owned[n].index(p)
            assert oracle.owner(p, N, I) == n
            assert oracle.local_index(p, N, I) == kk
    counts = oracle.shard_counts([L], N, I)[:, 0]
    assert counts.sum() == L
    assert np.all(np.abs(counts - L / N) <= I)


def test_shard_map_pages_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "blog_sec4_contiguous_ranges.json")))
    L, N, I = g["seq_len"], g["n_shards"], g["interleave"]
    for r, (lo, hi) in enumerate(g["ranges"]):
        assert oracle.shard_count(L, N, I, r) == hi - lo
        for p in (lo, lo + 1, (lo + hi) // 2, hi - 1):
            assert oracle.owner(p, N, I) == r
            assert oracle.local_index(p, N, I) == p - lo


def test_interleave_equal_block_size_gives_whole_pages():
    g = json.load(open(os.path.join(GOLDEN, "guide_interleave_block_size.json")))
    for case in g["cases"]:
        P, I, N = case["page_size"], case["interleave"], case["n_shards"]
        L = 5 * I * N + 7
        owned = _owned_positions_brute(L, N, I)
        for n in range(N):
            for k, p in enumerate(owned[n]):
                # page k // P of shard n holds consecutive positions
                if k % P:
                    assert p == owned[n][k - 1] + 1
                assert oracle.local_index(p, N, I) == k


@pytest.mark.parametrize("N,I,P", [(2, 1, 16), (8, 128, 16), (3, 5, 4), (4, 64, 64), (8, 1, 64)])
def test_shard_map_slots_against_enumeration(N, I, P):
    rng = np.random.default_rng(N * 1000 + I)
    B = 5
    L = rng.integers(1, 700, size=B)
    owned = {b: _owned_positions_brute(int(L[b]), N, I) for b in range(B)}
    need = np.array([[-(-len(owned[b][n]) // P) for b in range(B)] for n in range(N)])
    bt, num_pages = synth.deal_block_tables(77, need, slack_pages=3)
    pos, req, expect = [], [], []
    for b in range(B):
        for n in range(N):
            for k, p in enumerate(owned[b][n]):
                pos.append(p)
                req.append(b)
                expect.append(int(bt[n, b, k // P]) * P + k % P)
    st, rank, local, slot = oracle.shard_map(pos, req, N, I, P, bt, num_pages)
    assert st == oracle.ORC_OK
    assert np.array_equal(slot, np.array(expect, np.int64))
    # every position gets its own physical slot
    assert len(set(slot.tolist())) == len(slot)


def test_shard_map_unallocated_page():
    N, I, P = 2, 1, 16
    bt = np.full((N, 1, 2), -1, np.int32)
    bt[0, 0, 0] = 3
    st, rank, local, slot = oracle.shard_map([0, 1, 2, 40], [0, 0, 0, 0], N, I, P, bt, 4)
    assert st == oracle.ORC_ERR_UNALLOCATED
    assert slot.tolist() == [3 * 16 + 0, -1, 3 * 16 + 1, -1]
    assert rank.tolist() == [0, 1, 0, 0]


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------

def _rand_problem(rng, B, Hq, Hkv, Dk, Dv, Lmax, kind="gqa"):
    q = rng.standard_normal((B, Hq, Dk))
    if kind == "mla":
        K = rng.standard_normal((B, Lmax, Dk))
        V = None
    else:
        K = rng.standard_normal((B, Lmax, Hkv, Dk))
        V = rng.standard_normal((B, Lmax, Hkv, Dv))
    return q, K, V


def _brute(q, K, V, L, scale, kind, dv=None):
    """softmax(q K^T * scale) V with the exponential taken directly (no max
    subtraction), per (b, h); GQA head h reads kv head h // (Hq/Hkv)."""
    B, Hq, Dk = q.shape
    outs, lses = [], []
    for b in range(B):
        ob, lb = [], []
        for h in range(Hq):
            if kind == "mla":
                k = K[b, :L[b], :]
                v = K[b, :L[b], :dv]
            else:
                Hkv = K.shape[2]
                g = h // (Hq // Hkv)
                k = K[b, :L[b], g, :]
                v = V[b, :L[b], g, :]
            s = scale * (k @ q[b, h])
            e = np.exp(s)
            ob.append((e[:, None] * v).sum(0) / e.sum())
            lb.append(math.log(e.sum()))
        outs.append(ob)
        lses.append(lb)
    return np.array(outs), np.array(lses)


@pytest.mark.parametrize("B,Hq,Hkv,D,Lmax", [(2, 4, 2, 8, 13), (3, 6, 3, 5, 40), (1, 8, 1, 16, 64), (2, 4, 4, 3, 7)])
def test_attention_brute_force_gqa(B, Hq, Hkv, D, Lmax):
    rng = np.random.default_rng(B * 100 + Hq)
    q, K, V = _rand_problem(rng, B, Hq, Hkv, D, D + 1, Lmax)
    V = rng.standard_normal((B, Lmax, Hkv, D + 1))
    L = rng.integers(1, Lmax + 1, size=B)
    scale = 0.37
    O, lse = oracle.decode_arrays("gqa", q, K, V, L, scale)
    Ob, lb = _brute(q, K, V, L, scale, "gqa")
    np.testing.assert_allclose(O, Ob, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lb, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("B,Hq,Dk,Dv,Lmax", [(2, 4, 9, 6, 20), (1, 16, 24, 16, 64)])
def test_attention_brute_force_mla(B, Hq, Dk, Dv, Lmax):
    rng = np.random.default_rng(Dk)
    q, K, _ = _rand_problem(rng, B, Hq, 1, Dk, Dv, Lmax, kind="mla")
    L = rng.integers(1, Lmax + 1, size=B)
    scale = 1 / math.sqrt(Dk)
    O, lse = oracle.decode_arrays("mla", q, K, None, L, scale, dv=Dv)
    Ob, lb = _brute(q, K, None, L, scale, "mla", dv=Dv)
    np.testing.assert_allclose(O, Ob, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lb, rtol=1e-12, atol=1e-13)


def test_attention_lse_matches_library_logsumexp():
    rng = np.random.default_rng(5)
    q, K, V = _rand_problem(rng, 1, 2, 1, 32, 32, 500)
    # large scores: direct exp would overflow; scipy's logsumexp is the reference
    scale = 40.0
    O, lse = oracle.decode_arrays("gqa", q, K, V, [500], scale)
    for h in range(2):
        s = scale * (K[0, :, 0, :] @ q[0, h])
        assert abs(lse[0, h] - logsumexp(s)) <= 1e-12 * abs(logsumexp(s))
        w = np.exp(s - logsumexp(s))
        np.testing.assert_allclose(O[0, h], w @ V[0, :, 0, :], rtol=1e-10, atol=1e-12)


def test_attention_special_cases():
    rng = np.random.default_rng(11)
    q, K, V = _rand_problem(rng, 1, 2, 1, 16, 16, 50)
    # L = 1: output is the single value row, LSE is its score
    O, lse = oracle.decode_arrays("gqa", q, K, V, [1], 0.5)
    for h in range(2):
        np.testing.assert_allclose(O[0, h], V[0, 0, 0], rtol=0, atol=1e-15)
        assert abs(lse[0, h] - 0.5 * float(K[0, 0, 0] @ q[0, h])) < 1e-14
    # q = 0: uniform average, LSE = ln L
    O, lse = oracle.decode_arrays("gqa", np.zeros_like(q), K, V, [50], 0.5)
    np.testing.assert_allclose(O[0, 0], V[0, :50, 0].mean(0), rtol=1e-13, atol=1e-15)
    assert abs(lse[0, 0] - math.log(50)) < 1e-14
    # all keys equal: uniform average, LSE = s + ln L
    K2 = np.repeat(K[:, :1], 50, axis=1)
    O, lse = oracle.decode_arrays("gqa", q, K2, V, [50], 0.5)
    np.testing.assert_allclose(O[0, 1], V[0, :50, 0].mean(0), rtol=1e-12, atol=1e-14)
    assert abs(lse[0, 1] - (0.5 * float(K[0, 0, 0] @ q[0, 1]) + math.log(50))) < 1e-12


def test_mla_value_is_leading_slice_of_latent():
    # a latent whose trailing (rope) columns are huge: they may only enter the scores
    rng = np.random.default_rng(3)
    q, K, _ = _rand_problem(rng, 1, 3, 1, 12, 8, 30, kind="mla")
    K[:, :, 8:] *= 1000.0
    q[:, :, 8:] = 0.0
    O, _ = oracle.decode_arrays("mla", q, K, None, [30], 0.2, dv=8)
    assert np.abs(O).max() < 10.0


# ----------------------------------------------------------------------------
# several query tokens per request (speculative decoding under DCP, blog section 6)
# ----------------------------------------------------------------------------

def _brute_multi(q, K, V, L, scale, kind, dv=None):
    """Masked softmax over ALL Lmax stored positions with the exponential taken directly:
    query token j of request b may see position p iff p < L_b and p <= L_b - QL + j."""
    B, QL, Hq, Dk = q.shape
    Lmax = K.shape[1]
    O = np.zeros((B, QL, Hq, dv if kind == "mla" else V.shape[3]))
    lse = np.zeros((B, QL, Hq))
    pos = np.arange(Lmax)
    for b in range(B):
        for j in range(QL):
            visible = (pos < L[b]) & (pos <= L[b] - QL + j)
            for h in range(Hq):
                if kind == "mla":
                    k, v = K[b], K[b, :, :dv]
                else:
                    g = h // (Hq // K.shape[2])
                    k, v = K[b, :, g, :], V[b, :, g, :]
                e = np.where(visible, np.exp(scale * (k @ q[b, j, h])), 0.0)
                O[b, j, h] = (e[:, None] * v).sum(0) / e.sum()
                lse[b, j, h] = math.log(e.sum())
    return O, lse


@pytest.mark.parametrize("QL", [1, 2, 4])
def test_multi_query_brute_force_gqa(QL):
    rng = np.random.default_rng(40 + QL)
    B, Hq, Hkv, D, Lmax = 3, 4, 2, 8, 30
    q = rng.standard_normal((B, QL, Hq, D))
    K = rng.standard_normal((B, Lmax, Hkv, D))
    V = rng.standard_normal((B, Lmax, Hkv, D + 2))
    L = np.array([QL, 17, Lmax])  # the shortest request: its first query sees position 0 only
    O, lse = oracle.decode_multi_arrays("gqa", q, K, V, L, 0.41)
    Ob, lb = _brute_multi(q, K, V, L, 0.41, "gqa")
    np.testing.assert_allclose(O, Ob, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lb, rtol=1e-12, atol=1e-13)


def test_multi_query_brute_force_mla():
    rng = np.random.default_rng(7)
    B, QL, Hq, Dk, Dv, Lmax = 2, 3, 16, 12, 8, 25
    q = rng.standard_normal((B, QL, Hq, Dk))
    K = rng.standard_normal((B, Lmax, Dk))
    L = np.array([9, 25])
    O, lse = oracle.decode_multi_arrays("mla", q, K, None, L, 0.3, dv=Dv)
    Ob, lb = _brute_multi(q, K, None, L, 0.3, "mla", dv=Dv)
    np.testing.assert_allclose(O, Ob, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lb, rtol=1e-12, atol=1e-13)


def test_multi_query_reduces_to_single_query_decode():
    """QL = 1 is plain decode, and the last of QL query tokens sees the whole request."""
    rng = np.random.default_rng(11)
    B, Hq, Hkv, D, Lmax = 3, 6, 3, 5, 40
    q, K, V = _rand_problem(rng, B, Hq, Hkv, D, D, Lmax)
    L = np.array([4, 23, 40])
    O1, l1 = oracle.decode_arrays("gqa", q, K, V, L, 0.5)
    Om, lm = oracle.decode_multi_arrays("gqa", q[:, None], K, V, L, 0.5)
    np.testing.assert_array_equal(Om[:, 0], O1)
    np.testing.assert_array_equal(lm[:, 0], l1)
    q4 = rng.standard_normal((B, 4, Hq, D))
    O4, l4 = oracle.decode_multi_arrays("gqa", q4, K, V, L, 0.5)
    Ol, ll = oracle.decode_arrays("gqa", q4[:, 3], K, V, L, 0.5)
    np.testing.assert_array_equal(O4[:, 3], Ol)
    np.testing.assert_array_equal(l4[:, 3], ll)


@pytest.mark.parametrize("N,I", [(2, 1), (3, 2), (4, 5), (8, 1)])
def test_multi_query_sharded_merge_reproduces_unsharded(N, I):
    """The causal limit composes with the shard filter: per-shard partials of each query token
    LSE-merge to its unsharded result."""
    rng = np.random.default_rng(N * 7 + I)
    B, QL, Hq, Hkv, D, Lmax = 2, 3, 4, 2, 6, 60
    q = rng.standard_normal((B, QL, Hq, D))
    K = rng.standard_normal((B, Lmax, Hkv, D))
    V = rng.standard_normal((B, Lmax, Hkv, D))
    L = np.array([3, 60])
    O, lse = oracle.decode_multi_arrays("gqa", q, K, V, L, 0.3)
    parts = [oracle.decode_multi_arrays("gqa", q, K, V, L, 0.3, N=N, I=I, shard=n) for n in range(N)]
    Op = np.stack([p[0].reshape(B * QL, Hq, D) for p in parts])
    Lp = np.stack([p[1].reshape(B * QL, Hq) for p in parts])
    Om, lm = oracle.merge(Op, Lp)
    np.testing.assert_allclose(Om.reshape(O.shape), O, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lm.reshape(lse.shape), lse, rtol=1e-12, atol=1e-13)


def test_multi_query_rejects_requests_shorter_than_the_query():
    q = np.zeros((1, 3, 2, 4))
    K = np.zeros((1, 5, 1, 4))
    with pytest.raises(ValueError):
        oracle.decode_multi_arrays("gqa", q, K, K, [2], 1.0)


# ----------------------------------------------------------------------------
# sharding + merge invariant (pins the split into shards and chunks)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("N,I", [(1, 1), (2, 1), (3, 2), (4, 5), (8, 1), (8, 16), (5, 64), (7, 3)])
def test_sharded_merge_reproduces_unsharded(N, I):
    rng = np.random.default_rng(N * 31 + I)
    B, Hq, Hkv, D, Lmax = 3, 4, 2, 8, 150
    q, K, V = _rand_problem(rng, B, Hq, Hkv, D, D, Lmax)
    L = np.array([1, 77, 150])
    O, lse = oracle.decode_arrays("gqa", q, K, V, L, 0.3)
    parts = [oracle.decode_arrays("gqa", q, K, V, L, 0.3, N=N, I=I, shard=n) for n in range(N)]
    Op = np.stack([p[0] for p in parts])
    Lp = np.stack([p[1] for p in parts])
    # empty shards carry O = 0 and LSE = -inf
    for n in range(N):
        for b in range(B):
            if oracle.shard_count(int(L[b]), N, I, n) == 0:
                assert np.all(Lp[n, b] == -np.inf) and np.all(Op[n, b] == 0)
    Om, lm = oracle.merge(Op, Lp)
    np.testing.assert_allclose(Om, O, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lm, lse, rtol=1e-12, atol=1e-13)


def test_sharded_partial_equals_attention_over_owned_rows():
    rng = np.random.default_rng(8)
    N, I = 3, 4
    q, K, _ = _rand_problem(rng, 1, 4, 1, 10, 6, 90, kind="mla")
    owned = _owned_positions_brute(90, N, I)
    for n in range(N):
        O, lse = oracle.decode_arrays("mla", q, K, None, [90], 0.3, dv=6, N=N, I=I, shard=n)
        Ks = K[:, owned[n], :]
        Ob, lb = _brute(q, Ks, None, [len(owned[n])], 0.3, "mla", dv=6)
        np.testing.assert_allclose(O, Ob, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse, lb, rtol=1e-12, atol=1e-13)


def test_arbitrary_chunking_merges_exactly():
    """Split one shard's rows into random contiguous chunks (split-KV): the
    merge of the chunk partials equals the shard partial."""
    rng = np.random.default_rng(21)
    q, K, V = _rand_problem(rng, 1, 2, 1, 8, 8, 400)
    O, lse = oracle.decode_arrays("gqa", q, K, V, [400], 0.4)
    cuts = np.sort(rng.choice(np.arange(1, 400), size=9, replace=False))
    bounds = [0, *cuts.tolist(), 400]
    parts = []
    for lo, hi in zip(bounds[:-1], bounds[1:]):
        parts.append(oracle.decode_arrays("gqa", q, K[:, lo:hi], V[:, lo:hi], [hi - lo], 0.4))
    Om, lm = oracle.merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    np.testing.assert_allclose(Om, O, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lm, lse, rtol=1e-12, atol=1e-13)


def test_merge_edge_cases():
    # all shards empty: O = 0, LSE = -inf
    Op = np.ones((3, 1, 2, 4))
    Lp = np.full((3, 1, 2), -np.inf)
    O, l = oracle.merge(Op, Lp)
    assert np.all(O == 0) and np.all(l == -np.inf)
    # one finite shard: the merge returns it unchanged
    Lp[1, 0, :] = [0.25, -3.0]
    Op[1] *= 2.5
    O, l = oracle.merge(Op, Lp)
    np.testing.assert_allclose(O, Op[1], rtol=0, atol=0)
    np.testing.assert_allclose(l, Lp[1], rtol=0, atol=0)
    # two shards with LSE a, b: weights e^a/(e^a+e^b)
    Op = np.stack([np.full((1, 1, 1), 1.0), np.full((1, 1, 1), 3.0)])
    Lp = np.array([[[math.log(1.0)]], [[math.log(3.0)]]])
    O, l = oracle.merge(Op, Lp)
    assert abs(O[0, 0, 0] - (1.0 * 0.25 + 3.0 * 0.75)) < 1e-15
    assert abs(l[0, 0] - math.log(4.0)) < 1e-15


# ----------------------------------------------------------------------------
# e4m3 quantisation
# ----------------------------------------------------------------------------

def test_e4m3_decode_all_codes_match_library():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        v = oracle.e4m3_decode(c)
        if math.isnan(ref[c]):
            assert math.isnan(v)
        else:
            assert v == ref[c], c


def test_e4m3_encode_matches_library_rne():
    rng = np.random.default_rng(0)
    grid = np.array([oracle.e4m3_decode(c) for c in range(0x7F)])  # non-negative finite values
    mids = (grid[1:] + grid[:-1]) / 2           # ties: round half to even
    xs = np.concatenate([grid, mids, -mids, rng.standard_normal(4000) * 30, rng.standard_normal(1000) * 0.01,
                         np.linspace(-447.9, 447.9, 3001)])
    xs = xs.astype(np.float32).astype(np.float64)
    lib_codes = torch.from_numpy(xs.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for x, c in zip(xs, lib_codes):
        assert oracle.e4m3_encode(float(x)) == c, x


def test_e4m3_encode_saturates():
    assert oracle.e4m3_encode(448.0) == 0x7E
    assert oracle.e4m3_encode(1e6) == 0x7E
    assert oracle.e4m3_encode(-500.0) == 0xFE
    assert oracle.e4m3_encode(0.0) == 0x00


def test_quantize_row_properties():
    rng = np.random.default_rng(4)
    for trial in range(50):
        x = (rng.standard_normal(576) * rng.uniform(0.01, 5)).astype(np.float64)
        xb = synth.bf16_bits_from_f64(x)
        xf = synth.bf16_bits_to_f64(xb)
        codes, sc = oracle.quantize_row_e4m3(xb)
        amax = np.abs(xf).max()
        assert sc == float(np.float32(np.float32(amax) / np.float32(448.0)))
        deq = np.array([oracle.e4m3_decode(int(c)) for c in codes]) * sc
        # the largest element lands on +-448
        i = int(np.argmax(np.abs(xf)))
        assert codes[i] & 0x7F == 0x7E
        # RNE: each code is the library's nearest-even e4m3 value of x/scale
        y = (xf.astype(np.float32) / np.float32(sc)).astype(np.float32)
        lib_codes = torch.from_numpy(np.clip(y, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(codes, lib_codes)
        # reconstruction error within half a quantum of e4m3 (relative 2^-4, absolute 2^-10 * scale)
        err = np.abs(deq - xf)
        assert np.all(err <= np.maximum(np.abs(xf) * 2.0 ** -4, 2.0 ** -10 * sc) * (1 + 1e-6))


def test_quantize_row_all_zero():
    codes, sc = oracle.quantize_row_e4m3(np.zeros(576, np.uint16))
    assert sc == 1.0 and not codes.any()


# ----------------------------------------------------------------------------
# oracle on generated rows == oracle on the same rows as arrays
# ----------------------------------------------------------------------------

def test_synth_source_equals_array_source_gqa():
    seed, B, Hq, Hkv, D = 42, 2, 4, 2, 8
    L = np.array([37, 90])
    qb = synth.q_bf16(seed, B, Hq, D)
    q = synth.bf16_bits_to_f64(qb)
    K = np.zeros((B, 90, Hkv, D))
    V = np.zeros((B, 90, Hkv, D))
    for b in range(B):
        K[b] = synth.bf16_bits_to_f64(synth.kv_rows_bf16(seed, synth.T_K, b, np.arange(90), Hkv, D))
        V[b] = synth.bf16_bits_to_f64(synth.kv_rows_bf16(seed, synth.T_V, b, np.arange(90), Hkv, D))
    Oa, la = oracle.decode_arrays("gqa", q, K, V, L, 0.25)
    Os, ls = oracle.decode_synth("gqa", "bf16", seed, q, L, 0.25, Hkv, D, D)
    assert np.array_equal(Oa, Os) and np.array_equal(la, ls)


def test_synth_source_fp8_uses_quantised_rows():
    seed, B, Hq = 9, 1, 2
    L = np.array([20])
    q = synth.bf16_bits_to_f64(synth.q_bf16(seed, B, Hq, 576))
    rows = synth.kv_rows_bf16(seed, synth.T_LATENT, 0, np.arange(20), 1, 576)[:, 0, :]
    deq = np.zeros((1, 20, 576))
    for p in range(20):
        codes, sc = oracle.quantize_row_e4m3(rows[p])
        deq[0, p] = np.array([oracle.e4m3_decode(int(c)) for c in codes]) * sc
    Oa, la = oracle.decode_arrays("mla", q, deq, None, L, 0.1, dv=512)
    Os, ls = oracle.decode_synth("mla", "fp8", seed, q, L, 0.1, 1, 576, 512)
    np.testing.assert_allclose(Os, Oa, rtol=0, atol=1e-15)
    np.testing.assert_allclose(ls, la, rtol=0, atol=1e-15)


def test_quantize_rows_matches_single_rows():
    rng = np.random.default_rng(12)
    rows = synth.bf16_bits_from_f64(rng.standard_normal((40, 576)) * rng.uniform(0.1, 3, (40, 1)))
    rows[3] = 0
    codes, sc = oracle.quantize_rows_e4m3(rows)
    for i in range(40):
        c1, s1 = oracle.quantize_row_e4m3(rows[i])
        assert np.array_equal(codes[i], c1) and sc[i] == np.float32(s1)


def test_multi_query_synth_source_equals_array_source():
    """decode_multi_synth reads the generator as decode_multi_arrays reads the
    same rows materialised; with one query token it is decode_synth."""
    seed, B, QL, Hq, Hkv, D = 17, 2, 3, 4, 2, 8
    L = np.array([5, 70])
    q = synth.bf16_bits_to_f64(synth.q_bf16(seed, B, QL * Hq, D)).reshape(B, QL, Hq, D)
    K = np.zeros((B, 70, Hkv, D))
    V = np.zeros((B, 70, Hkv, D))
    for b in range(B):
        K[b] = synth.bf16_bits_to_f64(synth.kv_rows_bf16(seed, synth.T_K, b, np.arange(70), Hkv, D))
        V[b] = synth.bf16_bits_to_f64(synth.kv_rows_bf16(seed, synth.T_V, b, np.arange(70), Hkv, D))
    for N, I, shard in ((1, 1, -1), (3, 2, 1)):
        Oa, la = oracle.decode_multi_arrays("gqa", q, K, V, L, 0.3, N=N, I=I, shard=shard)
        Os, ls = oracle.decode_multi_synth("gqa", "bf16", seed, q, L, 0.3, Hkv, D, D, N=N, I=I, shard=shard)
        assert np.array_equal(Oa, Os) and np.array_equal(la, ls)
    q1 = synth.bf16_bits_to_f64(synth.q_bf16(seed, B, Hq, D))
    O1, l1 = oracle.decode_synth("gqa", "bf16", seed, q1, L, 0.3, Hkv, D, D)
    Om, lm = oracle.decode_multi_synth("gqa", "bf16", seed, q1[:, None], L, 0.3, Hkv, D, D)
    assert np.array_equal(O1, Om[:, 0]) and np.array_equal(l1, lm[:, 0])
