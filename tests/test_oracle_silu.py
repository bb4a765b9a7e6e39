"""The SiLU lookup in the oracle, pinned.

"How fast can FlashProve go", 2 Background and 3.1: the SiLU is not a
polynomial, so its 16-bit outputs are committed and proven by a lookup. The
table reads a 16-bit input v with 8 fractional bits and stores
floor(v sigma(v / 256) + 1/2). The table is pinned by properties of SiLU
itself (not by retyping the formula), the proof byte for byte against a
brute-force restatement, the lookup identity with explicit inversions, and the
verifier against tampering.
"""

import struct

import numpy as np
import pytest

import oracle
from tests import bruteforce as bf

P = oracle.P
TABLE = np.array([oracle.silu_q(v) for v in range(-32768, 32768)], dtype=np.int64)


def entry(v):
    return int(TABLE[v + 32768])


def test_table_properties():
    assert entry(0) == 0
    # silu(x) - silu(-x) = x: the two rounded entries differ by v up to one unit
    for v in range(1, 32768):
        assert abs(entry(v) - entry(-v) - v) <= 1, v
    # the minimum of silu is -0.27846... at x = -1.27846..., i.e. -71.3 at v = -327 (rounded, a
    # plateau of -71 around it)
    assert TABLE.min() == -71 and entry(-327) == -71
    # identity for large inputs, zero for very negative ones
    assert all(entry(v) == v for v in range(4096, 32768, 97))
    assert all(entry(v) == 0 for v in range(-32768, -4096, 97))
    # increasing above the minimum
    assert np.all(np.diff(TABLE[32768 - 327:]) >= 0)
    # sigma(1) = 0.7310585..., so v = 256 gives 187.15 -> 187; sigma(-1) gives -68.85 -> -69
    assert entry(256) == 187 and entry(-256) == -69


def _vecs(n, seed, lo=-3000, hi=3000):
    rng = np.random.default_rng(seed)
    g = rng.integers(lo, hi, n).astype(np.int16)
    return g, np.array([entry(int(x)) for x in g], np.int16)


@pytest.mark.parametrize("n", [1, 2, 3, 5, 8])
def test_bytes_match_bruteforce(n):
    g, s = _vecs(n, n)
    pf, _ = oracle.silu_prove(4, g, s)
    assert pf == bf.silu_prove(4, g, s)


def test_lookup_identity_with_explicit_inverses():
    g, s = _vecs(200, 9, -32768, 32767)
    gamma, alpha = 123456789, 987654321
    keys = [(int(a) + gamma * int(c)) % P for a, c in zip(g, s)]
    lhs = sum(pow((alpha - f) % P, P - 2, P) for f in keys) % P
    m = {}
    for a in g:
        m[int(a)] = m.get(int(a), 0) + 1
    rhs = sum(c * pow((alpha - (v + gamma * entry(v))) % P, P - 2, P) for v, c in m.items()) % P
    assert lhs == rhs


@pytest.mark.parametrize("n", [1, 77, 1024, 5000])
def test_honest_proof_accepted(n):
    g, s = _vecs(n, 50 + n, -32768, 32767)
    pf, _ = oracle.silu_prove(8, g, s)
    assert oracle.silu_verify(8, g, s, pf) == ("accept", (0, 0))


def _put(pf, off, val):
    return pf[:off] + struct.pack("<Q", val % P) + pf[off + 8:]


def test_each_check_fires():
    n = 40
    g, s = _vecs(n, 3)
    # a wrong output makes a key that is not in the table
    s_bad = s.copy()
    s_bad[7] += 1
    pf_bad, _ = oracle.silu_prove(2, g, s_bad)
    assert oracle.silu_verify(2, g, s_bad, pf_bad)[0] == "lookup_root"
    pf, _ = oracle.silu_prove(2, g, s)
    v = bf.log2c(n)
    off = 4 * 65536  # the multiplicities come first
    l1 = list(struct.unpack("<4Q", pf[off:off + 32]))
    assert oracle.silu_verify(2, g, s, _put(pf, off, l1[0] + 1))[0] == "lookup_root"
    off += 32
    # layer d has d rounds of 4 values and 4 final values; layer 1's first round value
    g0 = struct.unpack("<Q", pf[off:off + 8])[0]
    assert oracle.silu_verify(2, g, s, _put(pf, off, g0 + 1)) == ("lookup_round", (1, 0))
    fin = off + 32
    f0 = struct.unpack("<Q", pf[fin:fin + 8])[0]
    assert oracle.silu_verify(2, g, s, _put(pf, fin, f0 + 1)) == ("lookup_final", (1, 0))
    leaf = len(pf) - 16
    lg = struct.unpack("<Q", pf[leaf:leaf + 8])[0]
    assert oracle.silu_verify(2, g, s, _put(pf, leaf, lg + 1))[0] == "lookup_leaf"
    # the verifier holds other columns than the prover used
    g2 = g.copy()
    g2[0] ^= 2
    assert oracle.silu_verify(2, g2, s, pf)[0] != "accept"
    assert oracle.silu_verify(2, g, s, pf[:-8])[0] == "format"
    assert v >= 2
