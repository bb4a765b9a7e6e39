"""The helper-inverse LogUp in the oracle, pinned.

"Towards Proving Frontier-Scale LLM Inference", The proof system: lookups by
LogUp (Haboeck 2022) -- here in its helper-column form, the variant to set
against the GKR fraction tree: the prover commits h_i = 1 / (alpha - f_i),
and one sum-check proves both sum_i h_i and, through a zero-check against
eq(z, .), that every h_i (alpha - f_i) = 1. Pinned byte for byte against a
brute-force restatement, by the LogUp identity, and by tampering; and it
accepts exactly the statements the GKR-based lookup accepts.
"""

import struct

import numpy as np
import pytest

import oracle
from tests import bruteforce as bf

P = oracle.P


def _keys(n, k, seed):
    rng = np.random.default_rng(seed)
    return rng.integers(-(1 << (k - 1)), 1 << (k - 1), n).astype(np.int32)


@pytest.mark.parametrize("n,k", [(1, 3), (2, 4), (3, 5), (8, 4), (11, 6)])
def test_bytes_match_bruteforce(n, k):
    r = _keys(n, k, n + k)
    pf, _ = oracle.lhi_prove(5, r, k)
    assert pf == bf.lhi_prove(5, r, k)
    assert len(pf) == 4 * (1 << k) + 8 + 32 * max(1, bf.log2c(n)) + 16


@pytest.mark.parametrize("n,k", [(1, 7), (1000, 12), (4096, 12), (5000, 18)])
def test_honest_proof_accepted(n, k):
    r = _keys(n, k, 7 * n)
    pf, _ = oracle.lhi_prove(3, r, k)
    assert oracle.lhi_verify(3, r, k, pf) == ("accept", (0, 0))


def test_key_outside_table_rejected():
    k = 7
    r = _keys(300, k, 1)
    r[10] = 1 << (k - 1)  # one past the table's largest row
    pf, _ = oracle.lhi_prove(4, r, k)
    assert oracle.lhi_verify(4, r, k, pf)[0] == "lhi_sum"


def _put(pf, off, val):
    return pf[:off] + struct.pack("<Q", val % P) + pf[off + 8:]


def test_each_check_fires():
    k, n = 5, 40
    r = _keys(n, k, 2)
    pf, _ = oracle.lhi_prove(6, r, k)
    off = 4 * (1 << k)
    S = struct.unpack("<Q", pf[off:off + 8])[0]
    assert oracle.lhi_verify(6, r, k, _put(pf, off, S + 1))[0] == "lhi_sum"
    g0 = off + 8
    x = struct.unpack("<Q", pf[g0:g0 + 8])[0]
    assert oracle.lhi_verify(6, r, k, _put(pf, g0, x + 1)) == ("lhi_round", (0, 0))
    fo = len(pf) - 16
    h, f = struct.unpack("<QQ", pf[fo:fo + 16])
    assert oracle.lhi_verify(6, r, k, _put(pf, fo, h + 1))[0] == "lhi_final"
    r2 = r.copy()
    r2[3] ^= 1
    assert oracle.lhi_verify(6, r2, k, pf)[0] != "accept"
    assert oracle.lhi_verify(6, r, k, pf[:-8])[0] == "format"


def test_agrees_with_the_lookup_identity():
    # with h from the transcript's alpha, sum h equals the table side: the first check the
    # verifier makes, restated with explicit inverses
    k, n = 6, 50
    r = _keys(n, k, 3)
    pf, _ = oracle.lhi_prove(8, r, k)
    T = 1 << k
    m = np.frombuffer(pf[:4 * T], "<u4")
    assert m.sum() == 64  # the padded key count
    assert all(m[int(x) + (1 << (k - 1))] >= 1 for x in r)
