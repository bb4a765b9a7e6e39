"""Negative controls: each tamper must be rejected, for the reason it was written for.

Idea from "flashprove-consumer-gpu" (Results: flipped proof bit, truncated
proof, wrong statement are refused) and "Towards Proving Frontier-Scale LLM
Inference" (How far to trust it: controls that tamper one witness cell, weight
or root and must be rejected for the reason the control was written for).

Statement tampers are made before proving and given to prover and verifier
alike (the honest prover runs on a dishonest witness); proof tampers change
bytes of an honest proof. The verifier never checks integer facts of the
witness directly, so every rejection here comes from the protocol.
"""

import numpy as np
import pytest

import oracle
import workloads

P = oracle.P


@pytest.fixture(scope="module")
def honest():
    wl = workloads.build(3, seed=4, small=True)
    R = oracle.resolve(wl)
    pf, states, off = oracle.prove(4, R.sites, R.wits)
    assert oracle.verify(4, R.sites, R.wits, pf)[0] == "accept"
    return R, pf, off


def _reprove(R, sites, wits):
    pf, _, _ = oracle.prove(4, sites, wits)
    return oracle.verify(4, sites, wits, pf)


def _copy_wits(R):
    return [tuple(a.copy() for a in w) for w in R.wits]


def test_wrong_seed(honest):
    R, pf, _ = honest
    assert oracle.verify(5, R.sites, R.wits, pf)[0] == "claim"


def test_flip_weight_nibble(honest):
    R, _, _ = honest
    import copy
    sites = [copy.copy(s) for s in R.sites]
    w = sites[0].w.copy()
    w[3, 7] ^= 0x10
    sites[0].w = w
    assert _reprove(R, sites, R.wits)[0] == "mm_round"


def test_flip_activation_byte(honest):
    R, _, _ = honest
    import copy
    sites = [copy.copy(s) for s in R.sites]
    x = sites[2].xt.copy()
    x[5, 11] ^= 1
    sites[2].xt = x
    assert _reprove(R, sites, R.wits)[0] == "mm_round"


def test_change_one_remainder(honest):
    R, _, _ = honest
    wits = _copy_wits(R)
    wits[1][1][2, 3] += 1
    assert _reprove(R, R.sites, wits)[0] == "mm_round"


def test_output_not_clamped(honest):
    R, _, _ = honest
    wits = _copy_wits(R)
    q, r, y = wits[0]
    i = np.argwhere((q > -128) & (q < 127))[0]
    y[tuple(i)] += 1          # y != clamp(q); the matmul claim does not read y
    assert _reprove(R, R.sites, wits)[0] == "root_clamp"


def test_remainder_out_of_range(honest):
    R, _, _ = honest
    wits = _copy_wits(R)
    q, r, y = wits[2]
    k = R.sites[2].k_shift
    i = np.argwhere((q > -120) & (q < 120))[0]
    r[tuple(i)] += 1 << k     # Y = 2^k q + r still holds
    q[tuple(i)] -= 1
    y[tuple(i)] = max(-128, min(127, int(q[tuple(i)])))
    assert _reprove(R, R.sites, wits)[0] == "root_rem"


def _flip(pf, pos):
    b = bytearray(pf)
    b[pos] ^= 0x01
    return bytes(b)


def test_proof_byte_flips(honest):
    R, pf, off = honest
    ns = len(R.sites)
    k = R.sites[0].k_shift
    n = max(oracle.log2_ceil(s.K) for s in R.sites)
    rounds_at = 8 * ns
    final_at = rounds_at + 24 * n
    m_at = off
    l1_at = off + 4 * (1 << k) + 4 * 65536
    cases = {
        "claims": (0, "claim"),
        "first round": (rounds_at, "mm_round"),
        "last round g(2)": (final_at - 8, "mm_final"),
        "finals": (final_at, "mm_final"),
        "multiplicity": (m_at + 4 * 3, "root_rem"),
        "layer one": (l1_at, "root_rem"),
        "first gkr round": (l1_at + 64, "gkr_round"),
        "leaf": (len(pf) - 8, "leaf_Q"),
    }
    for name, (pos, want) in cases.items():
        got = oracle.verify(4, R.sites, R.wits, _flip(pf, pos))[0]
        assert got == want, (name, got)


def test_truncated_trailing_and_noncanonical(honest):
    R, pf, _ = honest
    assert oracle.verify(4, R.sites, R.wits, pf[:-1])[0] == "format"
    assert oracle.verify(4, R.sites, R.wits, pf + b"\x00")[0] == "format"
    b = bytearray(pf)
    b[0:8] = (P + 1).to_bytes(8, "little")      # claims[0] not canonical
    assert oracle.verify(4, R.sites, R.wits, bytes(b))[0] == "format"
