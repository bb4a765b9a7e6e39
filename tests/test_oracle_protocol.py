"""Pins of the oracle's whole proof.

1. On tiny statements an independent brute-force prover (tests/bruteforce.py:
   hashlib, Python integers, every MLE summed over the full hypercube, no
   folding) must produce the oracle's proof byte for byte.
2. On larger statements the transcript is replayed over the oracle's proof
   and the lookup is checked against its defining identity
   ("Towards Proving Frontier-Scale LLM Inference", How the prover works:
   LogUp; "How fast can FlashProve go", 4 Tighter Rooflines: key side as a
   binary tree): sum_i 1/(alpha - f_i) = sum_j m_j/(alpha - t_j), the tree
   root equals the direct fraction sum, multiplicities add up to the padded
   key count, and the leaf claims are the key columns' MLEs.
3. The oracle's verifier accepts every honest proof.
"""

import random

import numpy as np
import pytest

import oracle
import workloads
from tests import bruteforce as bf

P = oracle.P


def _resolved(sites, seed=0):
    return oracle.resolve(workloads.Workload("t", seed, sites))


TINY = [
    [workloads.random_site(1, 3, 5, 2, 8, 3)],
    [workloads.random_site(2, 4, 8, 4, 4, 4)],
    [workloads.random_site(3, 5, 70, 3, 4, 6, scales=True)],
    [workloads.random_site(4, 1, 1, 1, 8, 1)],
    [workloads.random_site(5, 2, 2, 2, 8, 1, act=False)],
    [workloads.random_site(6, 3, 6, 2, 4, 4, scales=True), workloads.random_site(7, 5, 3, 4, 8, 4),
     workloads.random_site(8, 2, 8, 1, 4, 4)],
    [workloads.random_site(9, 6, 4, 3, 8, 2), workloads.random_site(10, 6, 4, 3, 8, 2)],
]


@pytest.mark.parametrize("idx", range(len(TINY)))
@pytest.mark.parametrize("seed", [0, 12345])
def test_brute_force_prover_matches_oracle_bytes(idx, seed):
    R = _resolved(TINY[idx])
    pf, states, off = oracle.prove(seed, R.sites, R.wits)
    assert pf == bf.prove(seed, R.sites, R.wits)
    w = bf.walk(seed, R.sites, R.wits, pf)
    assert w["consumed"] == len(pf)
    assert w["state"] == states[2] and w["state_mm"] == states[1]
    assert oracle.verify(seed, R.sites, R.wits, pf)[0] == "accept"


def _fe_inv(a):
    return pow(a, P - 2, P)


def _check_lookup_identities(R, pf, seed):
    w = bf.walk(seed, R.sites, R.wits, pf)
    v = w["v"]
    L = 1 << v
    k = R.sites[0].k_shift
    fr = np.concatenate([x[1].reshape(-1) for x in R.wits]).astype(np.int64)
    fq = np.concatenate([x[0].reshape(-1) for x in R.wits]).astype(np.int64)
    fy = np.concatenate([x[2].reshape(-1) for x in R.wits]).astype(np.int64)
    pad = L - len(fr)
    assert 0 <= pad < max(2, len(fr))
    fr, fq, fy = (np.concatenate([a, np.zeros(pad, np.int64)]) for a in (fr, fq, fy))
    assert int(w["m_rem"].sum()) == L and int(w["m_clamp"].sum()) == L
    gamma = w["gamma"]
    # multiplicities by direct counting
    assert np.array_equal(w["m_rem"], np.bincount(fr + (1 << (k - 1)), minlength=1 << k))
    assert np.array_equal(w["m_clamp"], np.bincount(fq + 32768, minlength=65536))
    keys = [[int(x) % P for x in fr], [(int(a) + gamma * int(c)) % P for a, c in zip(fq, fy)]]
    tabs = [[(j - (1 << (k - 1))) % P for j in range(1 << k)],
            [((j - 32768) + gamma * max(-128, min(127, j - 32768))) % P for j in range(65536)]]
    ms = [w["m_rem"], w["m_clamp"]]
    for tau in range(2):
        alpha = w["alpha"][tau]
        lhs = sum(_fe_inv((alpha - f) % P) for f in keys[tau]) % P
        rhs = sum(int(m) * _fe_inv((alpha - t) % P) for m, t in zip(ms[tau], tabs[tau]) if m) % P
        assert lhs == rhs
        p0, p1, q0, q1 = w["l1"][4 * tau:4 * tau + 4]
        root_p, root_q = (p0 * q1 + p1 * q0) % P, q0 * q1 % P
        assert root_p * _fe_inv(root_q) % P == lhs            # tree root = direct fraction sum
        half = L // 2                                         # layer-1 nodes cover the two key halves
        assert p0 * _fe_inv(q0) % P == sum(_fe_inv((alpha - f) % P) for f in keys[tau][:half]) % P
        assert p1 * _fe_inv(q1) % P == sum(_fe_inv((alpha - f) % P) for f in keys[tau][half:]) % P
    z = w["z_leaf"]
    e = oracle.eq_table(z)
    for col, val in zip((fr, fq, fy), w["leaf"]):
        assert sum(int(a) * (int(c) % P) for a, c in zip(e, col)) % P == val
    # every layer round is consistent with its predecessor claim
    for lay in w["layers"]:
        for t in range(1, len(lay["rounds"])):
            g_prev = lay["rounds"][t - 1]
            g = lay["rounds"][t]
            assert (g[0] + g[1]) % P == oracle.lagrange(g_prev, lay["chal"][t - 1])


def test_tiny_config_identities_and_verifier():
    R = oracle.resolve(workloads.build(1))
    pf, states, off = oracle.prove(0, R.sites, R.wits)
    _check_lookup_identities(R, pf, 0)
    assert oracle.verify(0, R.sites, R.wits, pf)[0] == "accept"
    # matmul rounds: g_1(0) + g_1(1) = claim, and the claim is Y's MLE (direct)
    w = bf.walk(0, R.sites, R.wits, pf)
    q, r, _ = R.wits[0]
    Y = (q.astype(np.int64) << 7) + r
    assert w["claims"][0] == bf.mle2(Y.T, w["r_row"], w["r_col"])
    assert (w["mm_rounds"][0][0] + w["mm_rounds"][0][1]) % P == w["claims"][0]


@pytest.mark.parametrize("config", [3, 4, 5])
def test_small_layer_configs_verify(config):
    wl = workloads.build(config, seed=1, small=True)
    R = oracle.resolve(wl)
    pf, states, off = oracle.prove(1, R.sites, R.wits)
    assert oracle.verify(1, R.sites, R.wits, pf)[0] == "accept"
    if R.sites and sum(s.M * s.N for s in R.sites) <= 1 << 16:
        _check_lookup_identities(R, pf, 1)


def test_linked_operands_are_views_of_outputs():
    wl = workloads.build(4, seed=2, small=True)
    R = oracle.resolve(wl)
    names = [s.name for s in R.sites]
    q_site = names.index("wq")
    yq = R.wits[q_site][2]
    s0 = R.sites[names.index("s.1.0")]
    assert np.array_equal(s0.w.reshape(-1), yq.reshape(-1)[1 * 640: 1 * 640 + 640])
    wo = R.sites[names.index("wo")]
    ot = R.wits[names.index("ot.2.0")][2]
    assert np.array_equal(wo.xt[2], ot.reshape(-1))


@pytest.mark.slow
def test_projection_config_verifies():
    R = oracle.resolve(workloads.build(2))
    pf, states, off = oracle.prove(0, R.sites, R.wits)
    assert oracle.verify(0, R.sites, R.wits, pf)[0] == "accept"
    w = bf.walk(0, R.sites, R.wits, pf)
    assert w["consumed"] == len(pf) and w["state"] == states[2]
