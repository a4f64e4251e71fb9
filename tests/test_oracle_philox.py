"""Pins for the oracle's Philox4x32-10 and uniform maps (CPU only)."""
import os

import numpy as np
import pytest
from scipy import stats

from oracle import philox

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")


def _kat():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        lhs, rhs = line.split("|")
        ins = [int(w, 16) for w in lhs.split()]
        outs = [int(w, 16) for w in rhs.split()]
        rows.append((ins[:4], ins[4:], outs))
    return rows


@pytest.mark.parametrize("ctr,key,expect", _kat())
def test_known_answer_scalar(ctr, key, expect):
    assert philox.philox4x32_10(ctr, key) == expect


@pytest.mark.parametrize("ctr,key,expect", _kat())
def test_known_answer_vectorised(ctr, key, expect):
    out = philox.philox4x32_10_np(*[np.array([w]) for w in ctr], *[np.array([w]) for w in key])
    assert [int(o[0]) for o in out] == expect


def test_vectorised_equals_scalar_random_counters():
    rng = np.random.default_rng(5)
    words = rng.integers(0, 2**32, size=(300, 6), dtype=np.uint64)
    vec = philox.philox4x32_10_np(*(words[:, i] for i in range(6)))
    for i in range(300):
        ref = philox.philox4x32_10(words[i, :4].tolist(), words[i, 4:].tolist())
        assert [int(v[i]) for v in vec] == ref


def test_counter_layout_uses_every_field():
    base = philox.uniform_scalar(7, 3, 1, 11)
    assert philox.uniform_scalar(7, 3, 1, 12) != base          # index
    assert philox.uniform_scalar(7, 4, 1, 11) != base          # step lo
    assert philox.uniform_scalar(7, 3 + 2**32, 1, 11) != base  # step hi
    assert philox.uniform_scalar(7, 3, 2, 11) != base          # stream
    assert philox.uniform_scalar(8, 3, 1, 11) != base          # seed lo
    assert philox.uniform_scalar(7 + 2**32, 3, 1, 11) != base  # seed hi
    assert philox.uniforms(7, 3, 1, np.array([11]))[0] == base


def test_uniform24_range_and_exactness():
    assert philox.uniform24(0) == 0.0
    assert philox.uniform24(0xFFFFFFFF) == 1.0 - 2.0 ** -24
    assert philox.uniform24(0x1FF) == 2.0 ** -24                # low 8 bits dropped
    u = philox.uniforms(1, 0, 0, np.arange(1 << 16))
    assert np.all((u >= 0) & (u < 1))
    # every value is a multiple of 2^-24 (exact in fp32)
    assert np.all(u * 2**24 == np.floor(u * 2**24))
    assert np.all(u.astype(np.float32).astype(np.float64) == u)


def test_uniformity_chi_square():
    u = philox.uniforms(1234, 0, 1, np.arange(200_000))
    counts, _ = np.histogram(u, bins=64, range=(0, 1))
    assert stats.chisquare(counts).pvalue > 1e-4
    # independence of neighbouring counters: lag-1 correlation ~ 0
    assert abs(np.corrcoef(u[:-1], u[1:])[0, 1]) < 0.01
