"""Extension-field challenges in the oracle (next row f4), pinned.

"How fast can FlashProve go", 4 Tighter Rooflines: for soundness the
challenges are drawn from an extension of the Goldilocks field. The quadratic
extension F_p[phi] / (phi^2 - 7): the arithmetic is pinned by the field's laws
(7 is a non-residue, so every nonzero element is invertible), and the
gated-product sum-check with extension challenges byte for byte against a
brute-force restatement with its own extension arithmetic (Python integers).
"""

import random
import struct

import numpy as np
import pytest

import oracle
from tests import bruteforce as bf

P = oracle.P


def test_seven_is_not_a_square():
    assert pow(7, (P - 1) // 2, P) == P - 1


def test_arithmetic():
    rnd = random.Random(4)
    for _ in range(200):
        x = (rnd.randrange(P), rnd.randrange(P))
        y = (rnd.randrange(P), rnd.randrange(P))
        assert oracle.e2_mul(x, y) == bf.x_mul(x, y)
        if x != (0, 0):
            assert oracle.e2_mul(x, oracle.e2_inv(x)) == (1, 0)
    # phi^2 = 7; the base field embeds as (a, 0)
    assert oracle.e2_mul((0, 1), (0, 1)) == (7, 0)
    assert oracle.e2_mul((3, 0), (5, 0)) == (15, 0)


def _vecs(n, seed):
    rng = np.random.default_rng(seed)
    return rng.integers(-128, 128, n).astype(np.int8), rng.integers(-128, 128, n).astype(np.int8)


@pytest.mark.parametrize("n", [1, 2, 3, 5, 8])
def test_bytes_match_bruteforce(n):
    s, u = _vecs(n, n)
    pf, _ = oracle.had2_prove(2, s, u)
    assert pf == bf.had2_prove(2, s, u)
    assert len(pf) == 16 + 64 * bf.log2c(n) + 32


@pytest.mark.parametrize("n", [1, 100, 1000])
def test_honest_proof_accepted(n):
    s, u = _vecs(n, 9 + n)
    pf, _ = oracle.had2_prove(3, s, u)
    assert oracle.had2_verify(3, s, u, pf) == ("accept", (0, 0))


def _put(pf, off, val):
    return pf[:off] + struct.pack("<Q", val % P) + pf[off + 8:]


def test_each_check_fires():
    s, u = _vecs(40, 5)
    pf, _ = oracle.had2_prove(1, s, u)
    c_im = struct.unpack("<Q", pf[8:16])[0]
    assert oracle.had2_verify(1, s, u, _put(pf, 8, c_im + 1))[0] == "had_claim"
    r0 = 16 + 8  # round 1, g(0)'s second coordinate
    x = struct.unpack("<Q", pf[r0:r0 + 8])[0]
    assert oracle.had2_verify(1, s, u, _put(pf, r0, x + 1)) == ("had_round", (0, 0))
    fo = len(pf) - 32
    a = struct.unpack("<Q", pf[fo:fo + 8])[0]
    assert oracle.had2_verify(1, s, u, _put(pf, fo, a + 1))[0] == "had_final"
    s2 = s.copy()
    s2[0] ^= 1
    assert oracle.had2_verify(1, s2, u, pf)[0] != "accept"
    # the base-field statement is a different one: its proof does not verify here
    pf_base, _ = oracle.had_prove(1, s, u)
    assert oracle.had2_verify(1, s, u, pf_base)[0] != "accept"


# ---- the matmul sum-check over the extension ------------------------------------------

import workloads  # noqa: E402


def _site(M, K, N, bits, scales, seed):
    s = workloads.random_site(seed, M, K, N, bits, 6)
    if scales:
        s.scales = workloads.group_scales(np.random.default_rng(seed), M, K)
    return s, oracle.witness(s)


@pytest.mark.parametrize("M,K,N,bits,scales", [(1, 1, 1, 8, False), (2, 4, 3, 8, False), (3, 5, 2, 4, True)])
def test_mm2_bytes_match_bruteforce(M, K, N, bits, scales):
    s, w = _site(M, K, N, bits, scales, M * 10 + K)
    pf, _ = oracle.mm2_prove(4, s, w)
    assert pf == bf.mm2_prove(4, s, w)


@pytest.mark.parametrize("M,K,N,bits,scales", [(17, 100, 9, 4, True), (64, 256, 32, 8, False)])
def test_mm2_honest_accepted_and_tampering_named(M, K, N, bits, scales):
    s, w = _site(M, K, N, bits, scales, M + N)
    pf, _ = oracle.mm2_prove(7, s, w)
    assert oracle.mm2_verify(7, s, w, pf) == ("accept", (0, 0))
    fo = len(pf) - 32
    a = struct.unpack("<Q", pf[fo:fo + 8])[0]
    assert oracle.mm2_verify(7, s, w, pf[:fo] + struct.pack("<Q", (a + 1) % P) + pf[fo + 8:])[0] == "mm_final"
    x = struct.unpack("<Q", pf[16:24])[0]  # round 1, g(0)'s first coordinate
    assert oracle.mm2_verify(7, s, w, pf[:16] + struct.pack("<Q", (x + 1) % P) + pf[24:]) == ("mm_round", (0, 0))
    q, r, y = (t.copy() for t in w)
    r[1, 2] += 1
    assert oracle.mm2_verify(7, s, (q, r, y), pf)[0] != "accept"


# ---- the helper-inverse LogUp over the extension ----------------------------------------

def _keys(n, k, seed):
    return np.random.default_rng(seed).integers(-(1 << (k - 1)), 1 << (k - 1), n).astype(np.int32)


def test_extension_inverse():
    rng = np.random.default_rng(3)
    for _ in range(20):
        x = (int(rng.integers(0, P, dtype=np.uint64)), int(rng.integers(0, P, dtype=np.uint64)))
        assert bf.x_mul(x, bf.x_inv(x)) == (1, 0)


@pytest.mark.parametrize("n,k", [(1, 1), (3, 4), (5, 7), (8, 3), (13, 5)])
def test_lhi2_bytes_match_bruteforce(n, k):
    r = _keys(n, k, n * 10 + k)
    pf, _ = oracle.lhi2_prove(2, r, k)
    assert pf == bf.lhi2_prove(2, r, k)


def test_lhi2_accepts_and_names_tampering():
    k = 7
    r = _keys(1000, k, 4)
    pf, _ = oracle.lhi2_prove(6, r, k)
    assert oracle.lhi2_verify(6, r, k, pf) == ("accept", (0, 0))
    T = 1 << k
    off = 4 * T  # S
    x = struct.unpack("<Q", pf[off:off + 8])[0]
    assert oracle.lhi2_verify(6, r, k, pf[:off] + struct.pack("<Q", (x + 1) % P) + pf[off + 8:])[0] == "lhi2_sum"
    off = 4 * T + 16  # round 1, g(0)'s first coordinate
    x = struct.unpack("<Q", pf[off:off + 8])[0]
    assert oracle.lhi2_verify(6, r, k, pf[:off] + struct.pack("<Q", (x + 1) % P) + pf[off + 8:]) == ("lhi2_round", (0, 0))
    off = len(pf) - 32  # h(rho)
    x = struct.unpack("<Q", pf[off:off + 8])[0]
    assert oracle.lhi2_verify(6, r, k, pf[:off] + struct.pack("<Q", (x + 1) % P) + pf[off + 8:])[0] == "lhi2_final"
    r2 = r.copy()
    r2[17] = 1 << 20  # outside R_7
    pf2, _ = oracle.lhi2_prove(6, r2, k)
    assert oracle.lhi2_verify(6, r2, k, pf2)[0] == "lhi2_sum"
    # the base-field proof of the same keys is another proof
    base, _ = oracle.lhi_prove(6, r, k)
    assert oracle.lhi2_verify(6, r, k, base)[0] != "accept"


# ---- the 16-bit function lookups (LogUp-GKR tree) over the extension -----------------------

@pytest.mark.parametrize("n", [1, 2, 3, 5, 8])
def test_silu2_bytes_match_bruteforce(n):
    rng = np.random.default_rng(n + 70)
    g = rng.integers(-32768, 32768, n).astype(np.int16)
    s = np.array([oracle.silu_q(int(x)) for x in g], np.int16)
    pf, _ = oracle.silu2_prove(5, g, s)
    assert pf == bf.lookup16x_prove(5, g, s, "silu2", oracle.silu_q(0))


def test_exp2_bytes_match_bruteforce():
    g = np.array([-5, 0, -300, -1800, 7], np.int16)
    s = np.array([oracle.exp_q(int(x)) for x in g], np.int16)
    pf, _ = oracle.exp2_prove(6, g, s)
    assert pf == bf.lookup16x_prove(6, g, s, "exp2", oracle.exp_q(0))


def test_lookup16_over_extension_accepts_and_rejects():
    rng = np.random.default_rng(71)
    g = rng.integers(-32768, 32768, 3000).astype(np.int16)
    s = np.array([oracle.silu_q(int(x)) for x in g], np.int16)
    pf, _ = oracle.silu2_prove(8, g, s)
    assert oracle.silu2_verify(8, g, s, pf) == ("accept", (0, 0))
    bad = s.copy()
    bad[100] += 1  # an output the table does not hold
    pf2, _ = oracle.silu2_prove(8, g, bad)
    assert oracle.silu2_verify(8, g, bad, pf2)[0] == "lookup_root"
    # the base-field proof and the exponent table's proof are other statements
    base, _ = oracle.silu_prove(8, g, s)
    assert oracle.silu2_verify(8, g, s, base)[0] != "accept"
    assert oracle.exp2_verify(8, g, s, pf)[0] != "accept"


# ---- the two-table rescale LogUp over the extension -------------------------------------

def _lu_sites(shapes, seed, k=6):
    sites = [workloads.random_site(seed + i, M, K, N, 8, k) for i, (M, K, N) in enumerate(shapes)]
    return sites, [oracle.witness(s) for s in sites]


@pytest.mark.parametrize("shapes", [[(1, 4, 1)], [(2, 8, 1), (1, 8, 1)], [(3, 5, 2)], [(2, 16, 4)]])
def test_lu2_bytes_match_bruteforce(shapes):
    sites, wits = _lu_sites(shapes, 30)
    pf, _ = oracle.lu2_prove(3, sites, wits)
    assert pf == bf.lu2_prove(3, sites, wits)


def test_lu2_accepts_and_rejects():
    sites, wits = _lu_sites([(32, 64, 16), (16, 64, 8)], 40)
    pf, _ = oracle.lu2_prove(5, sites, wits)
    assert oracle.lu2_verify(5, sites, wits, pf) == ("accept", (0, 0))
    q, r, y = (a.copy() for a in wits[0])
    r[0, 0] += 1 << 6  # a remainder outside R_6
    pf2, _ = oracle.lu2_prove(5, sites, [(q, r, y), wits[1]])
    assert oracle.lu2_verify(5, sites, [(q, r, y), wits[1]], pf2)[0] == "root_rem"
    q, r, y = (a.copy() for a in wits[1])
    y[1, 1] = 100 if y[1, 1] != 100 else 99  # an output that is not clamp(q)
    pf3, _ = oracle.lu2_prove(5, sites, [wits[0], (q, r, y)])
    assert oracle.lu2_verify(5, sites, [wits[0], (q, r, y)], pf3)[0] == "root_clamp"
    off = len(pf) - 48  # r~(z)
    x = struct.unpack("<Q", pf[off:off + 8])[0]
    assert oracle.lu2_verify(5, sites, wits, pf[:off] + struct.pack("<Q", (x + 1) % P) + pf[off + 8:])[0] == "leaf_Q"
