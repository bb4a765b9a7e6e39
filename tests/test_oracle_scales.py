"""The per-group scale reduction in the oracle, pinned to its definition.

A site with per-64-column scales multiplies W_eff[i][k] = S[i][k // 64] w[i][k];
the matmul sum-check ends with a claim on W_eff~, while only w and S are
committed. As for the gated product ("How fast can FlashProve go", 3.1: a
product that is not committed is reduced by sum-check to claims on its
committed factors), a degree-3 product sum-check over (row, column) turns it
into claims on w~ and on S~ at the row point and the high column coordinates.
The oracle's proof is checked byte for byte against a brute-force
restatement, the scale identity Se~(rho) = S~(rho_row, rho_col_hi) directly,
and the verifier against tampering.
"""

import struct

import numpy as np
import pytest

import oracle
import workloads
from tests import bruteforce as bf

P = oracle.P


def _site(M, K, bits, seed):
    rng = np.random.default_rng(seed)
    w = workloads.int4_packed(rng, M, K) if bits == 4 else workloads.int8_uniform(rng, (M, K))
    sc = workloads.group_scales(rng, M, K)
    v = bf.log2c(M) + bf.log2c(K)
    z = [int(x) for x in rng.integers(0, P, size=v, dtype=np.uint64)]
    return w, sc, z


@pytest.mark.parametrize("M,K,bits", [(1, 1, 8), (2, 64, 4), (1, 100, 8), (4, 32, 4), (3, 20, 8), (2, 128, 4)])
def test_bytes_match_bruteforce(M, K, bits):
    w, sc, z = _site(M, K, bits, M * 1000 + K)
    pf, _ = oracle.scl_prove(5, w, bits, sc, M, K, z)
    assert pf == bf.scl_prove(5, w, bits, sc, M, K, z)


def test_scale_factor_mle_is_the_scales_mle():
    # Se(i, k) = S[i][k // 64] ignores the six low column bits, so its MLE at any point is
    # the scales' MLE at the row coordinates and the column coordinates above those six
    M, K = 3, 200
    w, sc, _ = _site(M, K, 4, 9)
    Se, _ = bf.scale_factors(w, 4, sc, M, K)
    vM, vK = bf.log2c(M), bf.log2c(K)
    G = (K + 63) // 64
    rng = np.random.default_rng(2)
    rho = [int(x) for x in rng.integers(0, P, size=vM + vK, dtype=np.uint64)]
    Sp = [0] * ((1 << vM) << (vK - 6))
    for i in range(M):
        for g in range(G):
            Sp[(i << (vK - 6)) + g] = int(sc[i, g])
    assert bf.mle_at(Se, rho) == bf.mle_at(Sp, rho[:vM] + rho[vM:vM + vK - 6])


@pytest.mark.parametrize("M,K,bits", [(1, 1, 4), (5, 130, 4), (64, 256, 4), (17, 1000, 8), (100, 64, 8)])
def test_honest_proof_accepted(M, K, bits):
    w, sc, z = _site(M, K, bits, 7 + M + K)
    pf, _ = oracle.scl_prove(8, w, bits, sc, M, K, z)
    assert len(pf) == 8 + 32 * len(z) + 16
    assert oracle.scl_verify(8, w, bits, sc, M, K, z, pf) == ("accept", (0, 0))


def _put(pf, off, val):
    return pf[:off] + struct.pack("<Q", val % P) + pf[off + 8:]


def test_each_check_fires():
    M, K, bits = 9, 200, 4
    w, sc, z = _site(M, K, bits, 21)
    pf, _ = oracle.scl_prove(2, w, bits, sc, M, K, z)
    v = len(z)
    a = struct.unpack("<Q", pf[:8])[0]
    assert oracle.scl_verify(2, w, bits, sc, M, K, z, _put(pf, 0, a + 1))[0] == "scl_claim"
    for t in (0, v // 2, v - 1):
        off = 8 + 32 * t
        g0 = struct.unpack("<Q", pf[off:off + 8])[0]
        assert oracle.scl_verify(2, w, bits, sc, M, K, z, _put(pf, off, g0 + 1)) == ("scl_round", (t, 0))
    fo = 8 + 32 * v
    S, W = struct.unpack("<QQ", pf[fo:fo + 16])
    assert oracle.scl_verify(2, w, bits, sc, M, K, z, _put(pf, fo, S + 1))[0] == "scl_final"
    k = 777
    bad = _put(_put(pf, fo, oracle.fmul(S, k)), fo + 8, oracle.fmul(W, oracle.finv(k)))
    assert oracle.scl_verify(2, w, bits, sc, M, K, z, bad) == ("scl_open", (0, 0))
    # a changed scale or weight changes the statement: the claim no longer matches
    sc2 = sc.copy()
    sc2[3, 1] += 1
    assert oracle.scl_verify(2, w, bits, sc2, M, K, z, pf)[0] != "accept"
    w2 = w.copy()
    w2[4, 10] ^= 0x10
    assert oracle.scl_verify(2, w2, bits, sc, M, K, z, pf)[0] != "accept"
    assert oracle.scl_verify(2, w, bits, sc, M, K, z, pf[:-8])[0] == "format"
