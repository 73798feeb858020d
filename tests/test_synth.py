"""The seeded input generators (CPU): numpy and C evaluations agree bit for
bit, the bf16 rounding is round-to-nearest-even, the values are approximately
N(0,1), and the request lengths have the trace's stated shape."""
import json
import os
from fractions import Fraction

import numpy as np

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_numpy_and_c_generators_agree():
    rng = np.random.default_rng(1)
    idx = rng.integers(0, 2**62, size=20000, dtype=np.uint64)
    for seed, tensor in [(0, 1), (2005, synth.T_LATENT), (2**40 + 3, 64 * 7 + 1)]:
        a = oracle.synth_bf16(seed, tensor, idx)
        b = synth.bf16_at(synth.key(seed, tensor), idx)
        assert np.array_equal(a, b)


def _nearest_even_bf16(x: float) -> float:
    """Exact rational round-to-nearest-even onto the bf16 grid (8 significant bits)."""
    if x == 0:
        return 0.0
    fx = Fraction(x)
    a = abs(fx)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    q = Fraction(2) ** (e - 7)
    k = a / q
    fl = k.numerator // k.denominator
    rem = k - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    v = fl * q
    return float(v if fx > 0 else -v)


def test_bf16_rounding_is_nearest_even():
    rng = np.random.default_rng(2)
    x = np.concatenate([synth.normal_from_bits(synth.bits(synth.key(3, 3), np.arange(3000))),
                        rng.standard_normal(2000) * 3])
    # exact ties between bf16 neighbours
    base = synth.bf16_bits_to_f64(synth.bf16_bits_from_f64(rng.standard_normal(500)))
    ulp = np.array([2.0 ** (np.floor(np.log2(abs(v))) - 7) for v in base])
    x = np.concatenate([x, base + ulp / 2, base - ulp / 2, [0.0]])
    got = synth.bf16_bits_to_f64(synth.bf16_bits_from_f64(x))
    for xi, gi in zip(x, got):
        assert gi == _nearest_even_bf16(float(xi)), xi


def test_values_approximately_standard_normal():
    x = synth.normal_from_bits(synth.bits(synth.key(11, 2), np.arange(1_000_000)))
    assert abs(x.mean()) < 5e-3
    assert abs(x.var() - 1.0) < 5e-3
    assert np.abs(x).max() <= 3.4642
    # Irwin-Hall(4) kurtosis is 3 - 1.2/4 = 2.7
    k = ((x - x.mean()) ** 4).mean() / x.var() ** 2
    assert abs(k - 2.7) < 0.02


def test_bimodal_lengths_match_trace_shape():
    g = json.load(open(os.path.join(GOLDEN, "blog_sec2_1_length_shape.json")))
    L = synth.lengths_bimodal(12345, 400_000)
    assert abs((L < 8_000).mean() - g["frac_below_8k"]) < 0.005
    assert abs((L < 64_000).mean() - g["frac_below_64k"]) < 0.005
    assert abs((L > 128_000).mean() - g["frac_above_128k"]) < 0.005
    lo, hi = g["frac_above_256k_range"]
    assert lo <= (L > 256_000).mean() <= hi
    assert abs(np.median(L) - g["median_tokens"]) < 1_000
    assert L.max() <= g["max_tokens"] and L.min() >= 1_000


def test_cap_rule_scales_down_proportionally():
    L0 = synth.lengths_bimodal(1005, 512)
    L = synth.lengths_bimodal(1005, 512, cap=24_000_000)
    assert L0.sum() > 24_000_000 >= L.sum()
    assert L.min() >= 1
    f = 24_000_000 / L0.sum()
    assert np.all((L <= np.maximum(1, L0 * f) + 1e-6) & (L >= L0 * f - 1.0))
    # the cap is inert when the total is below it
    assert np.array_equal(synth.lengths_bimodal(7, 8, cap=10**9), synth.lengths_bimodal(7, 8))


def test_uniform_lengths_in_range():
    L = synth.lengths_uniform(1, 10_000, 32_000, 128_000)
    assert L.min() >= 32_000 and L.max() <= 128_000
    assert abs(L.mean() - 80_000) < 1_000


def test_block_tables_are_disjoint_pages():
    need = np.array([[3, 0, 5], [1, 2, 0]])
    bt, num_pages = synth.deal_block_tables(5, need, slack_pages=4)
    assert num_pages == 15
    used = bt[bt >= 0]
    assert used.size == 11 and len(set(used.tolist())) == 11
    assert used.max() < num_pages
    for n in range(2):
        for b in range(3):
            assert np.all(bt[n, b, :need[n, b]] >= 0) and np.all(bt[n, b, need[n, b]:] == -1)


def test_workload_configs():
    w1 = synth.workload(1)
    assert w1.lengths.tolist() == [300, 1000] and w1.kv_bytes_per_token == 2 * 2 * 64 * 2
    w3 = synth.workload(3)
    assert w3.lengths.min() >= 32_000 and w3.lengths.max() <= 128_000 and w3.n_shards == 8
    w5 = synth.workload(5, n_shards=4, interleave=16)
    assert w5.lengths.sum() <= 24_000_000 and w5.n_shards == 4 and w5.interleave == 16
    assert w5.kv_bytes_per_token == 580
