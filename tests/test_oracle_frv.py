"""The Freivalds check of a weight matmul in the oracle (next row f4's comparison
statement), pinned.

"Towards Proving Frontier-Scale LLM Inference", The proof system: a matrix
product is checked as A (B r) = C r for a random vector r. Here u = X rho^(.)
(the powers of one squeezed rho over the tokens) is checked against
W_eff u = Y rho^(.) with Y = 2^k q + r. u is pinned by a Python restatement
(transcript replayed with hashlib, Horner's rule in integers); the verifier
accepts honest witnesses and names the wrong row of a tampered one.
"""

import struct

import numpy as np
import pytest

import oracle
import workloads
from tests import bruteforce as bf

P = oracle.P


def _site(M, K, N, bits, scales, seed):
    s = workloads.random_site(seed, M, K, N, bits, 8)
    if scales:
        rng = np.random.default_rng(seed)
        s.scales = workloads.group_scales(rng, M, K)
    return s, oracle.witness(s)


@pytest.mark.parametrize("M,K,N,bits,scales", [(4, 8, 3, 8, False), (9, 70, 5, 4, False), (16, 130, 7, 4, True)])
def test_u_matches_restatement(M, K, N, bits, scales):
    s, w = _site(M, K, N, bits, scales, M + K + N)
    pf, _ = oracle.frv_prove(3, s, w)
    d = bf.site_digests([s], [w])[0]
    tx = bf.Tx(3)
    tx.absorb("frv_site", d[:160])  # W, scales, Xt, q, r (y is not part of this statement)
    rho = tx.squeeze("frv_rho")
    X = np.asarray(s.xt, np.int64).T  # K x N
    u = []
    for k in range(K):
        acc = 0
        for j in reversed(range(N)):
            acc = (acc * rho + int(X[k, j])) % P
        u.append(acc)
    assert pf == bf.fe_bytes(u)


@pytest.mark.parametrize("M,K,N,bits,scales", [(1, 1, 1, 8, False), (33, 100, 17, 4, True), (64, 256, 40, 8, False)])
def test_honest_accepted(M, K, N, bits, scales):
    s, w = _site(M, K, N, bits, scales, 5 * M + N)
    pf, _ = oracle.frv_prove(1, s, w)
    assert oracle.frv_verify(1, s, w, pf) == ("accept", (0, 0))


def test_tampering_named():
    s, w = _site(20, 64, 9, 4, False, 4)
    pf, _ = oracle.frv_prove(2, s, w)
    q, r, y = (a.copy() for a in w)
    q[3, 7] += 1  # token 3, output row 7: the committed digests change, so rho changes too
    assert oracle.frv_verify(2, s, (q, r, y), pf)[0] in ("frv_u", "frv_row")
    # a proof made from the tampered witness fails at the row it changed
    pf2, _ = oracle.frv_prove(2, s, (q, r, y))
    assert oracle.frv_verify(2, s, (q, r, y), pf2) == ("frv_row", (7, 0))
    u0 = struct.unpack("<Q", pf[:8])[0]
    bad = struct.pack("<Q", (u0 + 1) % P) + pf[8:]
    assert oracle.frv_verify(2, s, w, bad) == ("frv_u", (0, 0))
