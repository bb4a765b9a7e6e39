"""Pins of the oracle's MoE routing proof (next row f3).

"How fast can FlashProve go", 2 Background (the note on MoE layers: the routing
computation and each token's choice of expert are proven too). Top-1 routing:
token t goes to the first index e_t of its largest router logit. The prover
commits the one-hot choice H and D[t][e] = l[t][e_t] - l[t][e] - [e < e_t]; a
sum-check ties D to H and l and makes H one-hot, and a helper-inverse LogUp
keeps D in [0, 256). Pinned here by: the witness against a Python first-argmax;
the identity the sum-check rests on, checked directly at random points; the
proof bytes against a brute-force prover (every round value a hypercube sum of
MLEs); honest proofs accepted; every way of cheating on the choice rejected for
its named reason.
"""

import struct

import numpy as np
import pytest

import oracle
from tests import bruteforce as bf

P = bf.P


def _logits(T, E, seed, lo=-128, hi=128):
    return np.random.default_rng(seed).integers(lo, hi, (T, E)).astype(np.int8)


@pytest.mark.parametrize("T,E,seed", [(1, 1, 0), (3, 4, 1), (7, 8, 2), (16, 2, 3), (5, 16, 4)])
def test_witness_is_the_first_argmax(T, E, seed):
    l = _logits(T, E, seed, -3, 3)  # few distinct values: many ties
    H, D = oracle.route_witness(l, T, E)
    Hb, Db = bf.route_witness(l, T, E)
    assert np.array_equal(H, Hb) and np.array_equal(D, Db)
    for t in range(T):
        e_t = int(np.argmax(l[t]))  # numpy returns the first maximum
        assert H[t].sum() == 1 and H[t, e_t] == 1
        assert D[t, e_t] == 0 and (D[t] >= 0).all() and (D[t] < 256).all()
        assert all(l[t, e] < l[t, e_t] for e in range(e_t))  # earlier indices are strictly smaller


@pytest.mark.parametrize("T,E", [(3, 4), (4, 8), (5, 2)])
def test_identity_behind_the_first_term(T, E):
    # D~(z) + l~(z) = sum_x eq(z_t, t) H(x) (l(x) - G(e)), G(e) = sum_{e' < e} eq(z_e, e')
    rng = np.random.default_rng(T * E)
    l = _logits(T, E, T + E)
    H, D = oracle.route_witness(l, T, E)
    vT, vE = bf.log2c(T), bf.log2c(E)
    z = [int(x) for x in rng.integers(0, P, vT + vE, dtype=np.uint64)]
    zt, ze = z[:vT], z[vT:]
    lhs = (bf.mle_at(D.reshape(-1), z) + bf.mle_at(l.reshape(-1).astype(np.int64), z)) % P
    rhs = 0
    for t in range(T):
        for e in range(E):
            if H[t, e]:
                G = sum(bf.eq_ml(ze, [(f >> (vE - 1 - b)) & 1 for b in range(vE)]) for f in range(e))
                rhs += bf.eq_ml(zt, [(t >> (vT - 1 - b)) & 1 for b in range(vT)]) * (int(l[t, e]) - G)
    assert lhs == rhs % P


@pytest.mark.parametrize("T,E,seed", [(1, 1, 0), (1, 2, 1), (3, 4, 2), (2, 8, 3), (5, 2, 4)])
def test_bytes_match_bruteforce(T, E, seed):
    l = _logits(T, E, 10 + seed, -4, 4)
    H, D = oracle.route_witness(l, T, E)
    pf, _ = oracle.route_prove(seed, l, H, D, T, E)
    assert pf == bf.route_prove(seed, l, H, D, T, E)


@pytest.mark.parametrize("T,E", [(100, 16), (64, 128), (1, 128)])
def test_honest_accepted(T, E):
    l = _logits(T, E, T + E)
    H, D = oracle.route_witness(l, T, E)
    pf, _ = oracle.route_prove(3, l, H, D, T, E)
    assert oracle.route_verify(3, l, H, D, T, E, pf) == ("accept", (0, 0))


def _reprove_with_choice(l, T, E, t, e_new):
    """The witness of a prover that routes token t to e_new instead, D recomputed honestly."""
    H, D = oracle.route_witness(l, T, E)
    H = H.copy()
    D = D.astype(np.int64).copy()
    H[t] = 0
    H[t, e_new] = 1
    for e in range(E):
        D[t, e] = int(l[t, e_new]) - int(l[t, e]) - (1 if e < e_new else 0)
    return H, D.astype(np.int32)


def test_a_token_sent_to_a_smaller_logit_is_rejected():
    T, E = 32, 16
    l = _logits(T, E, 5)
    t = 7
    second = int(np.argsort(l[t].astype(np.int64), kind="stable")[-2])
    H, D = _reprove_with_choice(l, T, E, t, second)
    assert D.min() < 0  # some difference is negative: a key below the range
    pf, _ = oracle.route_prove(4, l, H, D, T, E)
    assert oracle.route_verify(4, l, H, D, T, E, pf)[0] == "lhi_sum"


def test_a_tie_broken_upwards_is_rejected():
    T, E = 4, 8
    l = _logits(T, E, 6, -50, 50)
    l[2] = np.array([1, 9, 3, 9, 0, 9, -5, 2], np.int8)  # maxima at 1, 3, 5: the choice must be 1
    H, D = oracle.route_witness(l, T, E)
    assert H[2, 1] == 1
    H2, D2 = _reprove_with_choice(l, T, E, 2, 3)
    assert D2[2, 1] == -1
    pf, _ = oracle.route_prove(5, l, H2, D2, T, E)
    assert oracle.route_verify(5, l, H2, D2, T, E, pf)[0] == "lhi_sum"


def test_inconsistent_or_not_one_hot_witnesses_are_rejected():
    T, E = 16, 8
    l = _logits(T, E, 7)
    H, D = oracle.route_witness(l, T, E)
    # D not tied to H and l (still in range)
    D1 = D.copy()
    D1[3, 2] += 1
    pf, _ = oracle.route_prove(6, l, H, D1, T, E)
    assert oracle.route_verify(6, l, H, D1, T, E, pf) == ("route_round", (0, 0))
    # two experts for one token
    H2 = H.copy()
    H2[5, (int(np.argmax(l[5])) + 1) % E] = 1
    pf, _ = oracle.route_prove(6, l, H2, D, T, E)
    assert oracle.route_verify(6, l, H2, D, T, E, pf) == ("route_round", (0, 0))
    # a non-Boolean entry
    H3 = H.copy()
    H3[1] *= 2
    pf, _ = oracle.route_prove(6, l, H3, D, T, E)
    assert oracle.route_verify(6, l, H3, D, T, E, pf) == ("route_round", (0, 0))
    # no expert for one token
    H4 = H.copy()
    H4[0] = 0
    pf, _ = oracle.route_prove(6, l, H4, D, T, E)
    assert oracle.route_verify(6, l, H4, D, T, E, pf) == ("route_round", (0, 0))


def test_tampered_proof_bytes():
    T, E = 8, 4
    l = _logits(T, E, 8)
    H, D = oracle.route_witness(l, T, E)
    pf, _ = oracle.route_prove(9, l, H, D, T, E)

    def put(b, off, v):
        return b[:off] + struct.pack("<Q", v % P) + b[off + 8:]

    x = struct.unpack("<Q", pf[0:8])[0]
    assert oracle.route_verify(9, l, H, D, T, E, put(pf, 0, x + 1)) == ("route_open", (0, 0))
    n = bf.log2c(T) + bf.log2c(E)
    off = 16 + 32 * 2  # round 3's g(0)
    x = struct.unpack("<Q", pf[off:off + 8])[0]
    assert oracle.route_verify(9, l, H, D, T, E, put(pf, off, x + 1)) == ("route_round", (2, 0))
    off = 16 + 32 * n  # H~(rho)
    x = struct.unpack("<Q", pf[off:off + 8])[0]
    assert oracle.route_verify(9, l, H, D, T, E, put(pf, off, x + 1)) == ("route_open", (2, 0))
    assert oracle.route_verify(9, l, H, D, T, E, pf[:-8])[0] == "format"


def test_routing_shares_the_expert_distribution():
    # seeded logits give near-uniform choices over the experts (the workload's routing)
    T, E = 8192, 128
    l = _logits(T, E, 11)
    H, _ = oracle.route_witness(l, T, E)
    counts = H.sum(axis=0)
    assert counts.sum() == T and counts.min() > 20 and counts.max() < 120
