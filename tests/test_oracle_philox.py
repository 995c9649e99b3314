"""Pins for the oracle's Philox4x32-10 and its uniforms (no GPU)."""
import os

import numpy as np
from scipy import stats

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")


def _kat():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        v = [int(x, 16) for x in line.split()]
        rows.append((v[0:4], v[4:6], v[6:10]))
    return rows


def test_known_answer_vectors():
    rows = _kat()
    assert len(rows) == 3
    for ctr, key, want in rows:
        got = oracle.philox4x32_10(ctr, key)
        assert [int(x) for x in got] == want


def test_uniform_is_top24_bits_of_word0():
    seed = 0x0123456789ABCDEF
    for c in range(50):
        w = oracle.philox4x32_10([c, 3, 1, 0], [seed & 0xFFFFFFFF, seed >> 32])
        u = oracle.uniform(seed, c, 3, 1, 0)
        assert u == (int(w[0]) >> 8) / 2.0 ** 24
        assert 0.0 <= u < 1.0
        assert float(np.float32(u)) == u  # exactly representable in fp32


def test_uniform_histogram_is_flat():
    # 200k counters of one key: 100-bin chi-square and a Kolmogorov-Smirnov test.
    n = 200_000
    u = np.array([oracle.uniform(7, b, i, 0, 0) for b in range(n // 50) for i in range(50)])
    hist, _ = np.histogram(u, bins=100, range=(0.0, 1.0))
    assert stats.chisquare(hist).pvalue > 0.001
    assert stats.kstest(u, "uniform").pvalue > 0.001


def test_counter_words_and_key_all_matter():
    base = oracle.uniform(5, 1, 2, 0, 0)
    assert oracle.uniform(5, 2, 2, 0, 0) != base
    assert oracle.uniform(5, 1, 3, 0, 0) != base
    assert oracle.uniform(5, 1, 2, 1, 0) != base
    assert oracle.uniform(6, 1, 2, 0, 0) != base
    assert oracle.uniform(5 + (1 << 32), 1, 2, 0, 0) != base


def test_many_counters_equals_one_at_a_time():
    rng = np.random.default_rng(11)
    ctrs = rng.integers(0, 2**32, size=(64, 4), dtype=np.uint64).astype(np.uint32)
    key = [0x9E3779B9, 0xDEADBEEF]
    many = oracle.philox4x32_10_many(ctrs, key)
    for i in range(len(ctrs)):
        assert list(many[i]) == list(oracle.philox4x32_10(ctrs[i], key))
    # and the known answers through the batched entry
    rows = _kat()
    for ctr, key, want in rows:
        assert [int(x) for x in oracle.philox4x32_10_many(np.array([ctr]), key)[0]] == want
