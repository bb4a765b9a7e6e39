"""The gated-product sum-check in the oracle, pinned to its definition.

"How fast can FlashProve go", 3.1 Committing intermediate values: the gated
product h = s (.) u is a plain product, so a sum-check reduces a claim on h~(z)
to claims on the committed factors s and u without committing h. The oracle's
proof is checked byte for byte against a brute-force restatement (every round
value a hypercube sum of eq s~ u~ at its definition point, no folding), its
verifier against honest and tampered proofs, and the claim against closed
forms (u = 1 gives s~(z); s = 0 gives 0).
"""

import struct

import numpy as np
import pytest

import oracle
from tests import bruteforce as bf

P = oracle.P


def _vecs(n, seed):
    rng = np.random.default_rng(seed)
    return (rng.integers(-128, 128, n).astype(np.int8), rng.integers(-128, 128, n).astype(np.int8))


@pytest.mark.parametrize("n", [1, 2, 3, 5, 8, 13, 16, 32])
def test_bytes_match_bruteforce(n):
    s, u = _vecs(n, n)
    pf, _ = oracle.had_prove(3, s, u)
    assert pf == bf.had_prove(3, s, u)
    assert len(pf) == 8 + 32 * bf.log2c(n) + 16


@pytest.mark.parametrize("n", [1, 7, 64, 1000, 4097])
def test_honest_proof_accepted(n):
    s, u = _vecs(n, 100 + n)
    pf, _ = oracle.had_prove(9, s, u)
    assert oracle.had_verify(9, s, u, pf) == ("accept", (0, 0))


def _claim_of(pf):
    return struct.unpack("<Q", pf[:8])[0]


def test_claim_closed_forms():
    # u = 1: the claim is s~(z); s = 0: the claim and every round value vanish
    n = 21
    s, _ = _vecs(n, 5)
    ones = np.ones(n, np.int8)
    pf, _ = oracle.had_prove(4, s, ones)
    tx = bf.Tx(4)
    tx.absorb("had_site", bf.tree_digest(s.tobytes()) + bf.tree_digest(ones.tobytes()))
    z = [tx.squeeze("had_z") for _ in range(bf.log2c(n))]
    assert _claim_of(pf) == bf.mle(s, z)
    zero = np.zeros(n, np.int8)
    pf0, _ = oracle.had_prove(4, zero, s)
    assert set(pf0[: len(pf0) - 16]) == {0}


def test_tampered_witness_rejected():
    n = 300
    s, u = _vecs(n, 11)
    pf, _ = oracle.had_prove(1, s, u)
    s2 = s.copy()
    s2[17] ^= 1
    assert oracle.had_verify(1, s2, u, pf)[0] != "accept"
    # a proof made from the changed vector does not verify against the committed one
    pf2, _ = oracle.had_prove(1, s2, u)
    assert oracle.had_verify(1, s, u, pf2)[0] != "accept"
    # swapped factors: a different statement
    assert oracle.had_verify(1, u, s, pf)[0] != "accept"
    # another seed: the transcript diverges
    assert oracle.had_verify(2, s, u, pf)[0] != "accept"


def _put(pf, off, val):
    return pf[:off] + struct.pack("<Q", val % P) + pf[off + 8:]


def test_each_check_fires():
    n = 50
    s, u = _vecs(n, 12)
    pf, _ = oracle.had_prove(6, s, u)
    v = bf.log2c(n)
    c = _claim_of(pf)
    assert oracle.had_verify(6, s, u, _put(pf, 0, c + 1))[0] == "had_claim"
    for t in range(v):  # round t's g(0)
        off = 8 + 32 * t
        g0 = struct.unpack("<Q", pf[off:off + 8])[0]
        assert oracle.had_verify(6, s, u, _put(pf, off, g0 + 1)) == ("had_round", (t, 0))
    fo = 8 + 32 * v
    S, U = struct.unpack("<QQ", pf[fo:fo + 16])
    assert oracle.had_verify(6, s, u, _put(pf, fo, S + 1))[0] == "had_final"
    # S k, U / k keeps the product: only the opening check sees it
    k = 12345
    bad = _put(_put(pf, fo, oracle.fmul(S, k)), fo + 8, oracle.fmul(U, oracle.finv(k)))
    assert oracle.had_verify(6, s, u, bad)[0] == "had_open"
    assert oracle.had_verify(6, s, u, pf[:-1])[0] == "format"
    assert oracle.had_verify(6, s, u, pf + b"\0" * 8)[0] == "format"
