"""The MoE dispatch statement (oracle dsp_prove / dsp_verify).

"How fast can FlashProve go", 2 Background (the note on MoE layers: the routing
computation and the choice of expert are proven). The routing proof covers the
choice; this statement covers moving each token's activations to its expert:
the experts' inputs stacked expert by expert, D, are the row permutation of the
layer input X that the routing e gives, D~(r, c) = sum_t eq(r, pos(t)) X~(t, c).

Pins: pos(t) against numpy's stable sort; the identity itself at random points
with Python integers; the brute-force restatement (hypercube sums of MLEs,
hashlib) byte for byte; the layer's own experts' inputs accepted; every
dishonest D, routing or proof byte rejected for its named reason.
"""

import numpy as np
import pytest

import oracle
import workloads
from tests import bruteforce as bf

P = bf.P


def statement(seed, T, K, E):
    rng = np.random.default_rng(seed)
    X = rng.integers(-128, 128, (T, K)).astype(np.int8)
    e = rng.integers(0, E, T).astype(np.int32)
    return X, e, X[np.argsort(e, kind="stable")]


def test_positions_and_identity():
    X, e, D = statement(1, 11, 6, 3)
    order = np.argsort(e, kind="stable")
    pos = np.empty(11, np.int64)
    pos[order] = np.arange(11)
    assert np.array_equal(D[pos], X)
    rng = np.random.default_rng(2)
    for _ in range(3):
        r = [int(v) for v in rng.integers(0, P, 4, dtype=np.uint64)]
        c = [int(v) for v in rng.integers(0, P, 3, dtype=np.uint64)]
        lhs = bf.mle2(D.astype(np.int64), r, c)
        rhs = sum(bf.eq_ml(r, [(int(pos[t]) >> (3 - b)) & 1 for b in range(4)]) * bf.mle(X[t].astype(np.int64), c)
                  for t in range(11)) % P
        assert lhs == rhs


@pytest.mark.parametrize("seed,T,K,E", [(3, 1, 1, 1), (4, 5, 3, 2), (5, 16, 8, 4), (6, 13, 7, 5), (7, 32, 16, 8)])
def test_matches_brute_force(seed, T, K, E):
    X, e, D = statement(seed, T, K, E)
    pf, st = oracle.dsp_prove(seed, X, e, D, E)
    assert pf == bf.dsp_prove(seed, X, e, D, E)
    assert len(pf) == 8 + 24 * bf.log2c(T) + 16
    assert oracle.dsp_verify(seed, X, e, D, E, pf) == ("accept", (0, 0))


def test_moe_layer_inputs_accepted():
    X, e, D = workloads.moe_dispatch(0, E=8, d=32, T=64)
    wl = workloads.build(5, seed=0, E=8, d=32, ffn=64, T=64)
    stacked = np.concatenate([s.xt for s in wl.sites if s.name.endswith(".gate")][:-1])
    assert np.array_equal(stacked, D)  # the experts' gate inputs, in expert order
    pf, _ = oracle.dsp_prove(9, X, e, D, 8)
    assert oracle.dsp_verify(9, X, e, D, 8, pf)[0] == "accept"


@pytest.fixture(scope="module")
def honest():
    X, e, D = statement(8, 40, 12, 6)
    pf, _ = oracle.dsp_prove(8, X, e, D, 6)
    return X, e, D, pf


def _reprove(X, e, D):
    pf, _ = oracle.dsp_prove(8, X, e, D, 6)
    return oracle.dsp_verify(8, X, e, D, 6, pf)[0]


def test_rows_of_two_experts_swapped(honest):
    X, e, D, _ = honest
    D2 = D.copy()
    D2[[0, -1]] = D2[[-1, 0]]
    assert _reprove(X, e, D2) == "dsp_round"


def test_a_token_sent_to_another_expert(honest):
    X, e, D, _ = honest
    e2 = e.copy()
    e2[3] = (e2[3] + 1) % 6  # D still holds the original routing
    assert _reprove(X, e2, D) == "dsp_round"


def test_one_activation_changed_after_dispatch(honest):
    X, e, D, _ = honest
    D2 = D.copy()
    D2[7, 2] ^= 1
    assert _reprove(X, e, D2) == "dsp_round"


def test_changed_proof_bytes(honest):
    X, e, D, pf = honest
    b = bytearray(pf)
    b[1] ^= 1
    assert oracle.dsp_verify(8, X, e, D, 6, bytes(b))[0] == "dsp_claim"
    b = bytearray(pf)
    b[8 + 3] ^= 1
    assert oracle.dsp_verify(8, X, e, D, 6, bytes(b))[0] == "dsp_round"
    b = bytearray(pf)
    b[-9] ^= 1
    assert oracle.dsp_verify(8, X, e, D, 6, bytes(b))[0] == "dsp_final"
    assert oracle.dsp_verify(8, X, e, D, 6, pf[:-8])[0] == "format"
    assert oracle.dsp_verify(8, X, e, D, 6, pf + bytes(8))[0] == "format"
    assert oracle.dsp_verify(8, X, e, D, 5, pf)[0] == "args"  # an expert index outside [0, E)
