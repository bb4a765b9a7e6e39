"""The softmax numerator lookup in the oracle, pinned.

"Towards Proving Frontier-Scale LLM Inference", The arithmetic: the exponential
is a lookup table and the integer softmax has a 9-bit numerator. The table
reads v = score - row maximum (<= 0) with 8 fractional bits and stores
floor(511 e^(v/256) + 1/2), saturating at 511 above 0. The table is pinned by
properties of the exponential (not by retyping the formula); the proof by the
same brute-force restatement as the SiLU lookup (the argument is shared, only
the labels and the verifier's table differ), and the verifier by tampering.
"""

import math

import numpy as np
import pytest

import oracle
from tests import bruteforce as bf

TABLE = np.array([oracle.exp_q(v) for v in range(-32768, 32768)], dtype=np.int64)


def entry(v):
    return int(TABLE[v + 32768])


def test_table_properties():
    assert entry(0) == 511 and all(entry(v) == 511 for v in range(1, 32768, 101))
    assert entry(-256) == 188                          # 511 / e = 187.98
    assert np.all(np.diff(TABLE) >= 0)                 # non-decreasing
    # halving every 256 ln 2 = 177.4 steps, within rounding
    for v in range(-1500, -200, 37):
        a, b = entry(v), entry(v - 177)
        assert abs(2 * b - a) <= 3, v
    # zero once 511 e^(v/256) < 1/2, i.e. v < 256 ln(1/1022) = -1773.9
    assert entry(-1773) == 1 and entry(-1774) == 0 and entry(-32768) == 0
    assert math.isclose(entry(-512), 511 * math.exp(-2), abs_tol=0.5)


def _cols(n, seed):
    rng = np.random.default_rng(seed)
    g = rng.integers(-2500, 1, n).astype(np.int16)
    return g, TABLE[g.astype(np.int64) + 32768].astype(np.int16)


@pytest.mark.parametrize("n", [1, 3, 8])
def test_bytes_match_bruteforce(n):
    g, s = _cols(n, n)
    pf, _ = oracle.exp_prove(6, g, s)
    assert pf == bf.lookup16_prove(6, g, s, "exp", 511)


@pytest.mark.parametrize("n", [1, 100, 4096])
def test_honest_proof_accepted(n):
    g, s = _cols(n, 30 + n)
    pf, _ = oracle.exp_prove(2, g, s)
    assert oracle.exp_verify(2, g, s, pf) == ("accept", (0, 0))


def test_tables_are_not_interchangeable():
    g, s = _cols(64, 7)
    pf, _ = oracle.exp_prove(2, g, s)
    # the SiLU verifier neither shares the labels nor the table
    assert oracle.silu_verify(2, g, s, pf)[0] != "accept"
    s2 = s.copy()
    s2[5] += 1
    pf2, _ = oracle.exp_prove(2, g, s2)
    assert oracle.exp_verify(2, g, s2, pf2)[0] == "lookup_root"
