"""The layer proof with the helper-inverse lookup section (oracle prove_hi / verify_hi).

"Towards Proving Frontier-Scale LLM Inference", The proof system: lookups by
LogUp after Haboeck 2022, the key side a committed column of inverses checked by
one sum-check; "How fast can FlashProve go", 4 Tighter Rooflines: the same
lookups as a binary fraction tree with one sum-check per level. This variant
keeps the tree form's tables and keys (remainder table R_k, clamp table C16,
keys q + gamma y) and replaces the tree by two helper columns and one sum-check
of v rounds.

Pins: the brute-force restatement (Python integers, hashlib, every round value a
hypercube sum of MLEs at field points) reproduces the oracle's proof byte for
byte; the matmul section is the tree form's; honest witnesses are accepted;
each dishonest witness or changed proof byte is rejected for its named reason.
"""

import copy

import numpy as np
import pytest

import oracle
import workloads
from tests import bruteforce as bf

P = oracle.P


def tiny_statement(seed: int, shapes):
    sites = [workloads.random_site(300 + 10 * seed + i, M, K, N, b, k, scales=sc)
             for i, (M, K, N, b, k, sc) in enumerate(shapes)]
    return sites, [oracle.witness(s) for s in sites]


@pytest.mark.parametrize("seed,shapes", [
    (1, [(4, 8, 2, 8, 3, False)]),                          # 8 keys, v = 3
    (2, [(3, 5, 3, 4, 9, False), (2, 70, 3, 4, 9, True)]),  # ragged, padded keys, scales
    (3, [(8, 16, 4, 8, 6, False), (5, 9, 2, 4, 6, False), (1, 3, 1, 8, 6, False)]),
])
def test_matches_brute_force(seed, shapes):
    sites, wits = tiny_statement(seed, shapes)
    pf, states, mm = oracle.prove_hi(seed, sites, wits)
    assert pf == bf.prove_hi(seed, sites, wits)
    gkr, gstates, gmm = oracle.prove(seed, sites, wits)
    assert mm == gmm and pf[:mm] == gkr[:mm] and states[:2] == gstates[:2]
    assert oracle.verify_hi(seed, sites, wits, pf) == ("accept", (0, 0))


def test_size_and_round_count():
    # the lookup section: m_rem (2^k u32), m_clamp (2^16 u32), two sums, v rounds of 4, five finals
    wl = workloads.build(1)
    R = oracle.resolve(wl)
    pf, _, mm = oracle.prove_hi(0, R.sites, R.wits)
    v = 10  # 64 x 16 outputs
    assert len(pf) - mm == 4 * (1 << 7) + 4 * 65536 + 16 + 32 * v + 40
    gkr, _, _ = oracle.prove(0, R.sites, R.wits)
    # the tree form sends v (v - 1) / 2 rounds of 4 and a layer end of 8 per layer
    assert len(gkr) - mm == 4 * (1 << 7) + 4 * 65536 + 64 + sum(32 * d + 64 for d in range(1, v)) + 24


@pytest.fixture(scope="module")
def honest():
    wl = workloads.build(5, seed=2, small=True)
    R = oracle.resolve(wl)
    pf, _, mm = oracle.prove_hi(2, R.sites, R.wits)
    assert oracle.verify_hi(2, R.sites, R.wits, pf) == ("accept", (0, 0))
    return R, pf, mm


def _reprove(sites, wits):
    pf, _, _ = oracle.prove_hi(2, sites, wits)
    return oracle.verify_hi(2, sites, wits, pf)


def _copy_wits(R):
    return [tuple(a.copy() for a in w) for w in R.wits]


def test_remainder_outside_its_table(honest):
    # r + 2^k and q - 1 keep Y = 2^k q + r (the matmul section holds); r leaves R_k
    R, _, _ = honest
    wits = _copy_wits(R)
    q, r, y = wits[4]
    k = R.sites[4].k_shift
    r[1, 2] += 1 << k
    q[1, 2] -= 1
    y[1, 2] = np.clip(q[1, 2], -128, 127)
    assert _reprove(R.sites, wits) == ("lhr_sum", (0, 0))


def test_output_not_clamped(honest):
    R, _, _ = honest
    wits = _copy_wits(R)
    q, r, y = wits[0]
    i = np.argwhere((q > -128) & (q < 127))[0]
    y[tuple(i)] += 1  # y != clamp(q): its key q + gamma y is no row of C16
    assert _reprove(R.sites, wits) == ("lhr_sum", (1, 0))


def test_quotient_beyond_sixteen_bits(honest):
    R, _, _ = honest
    wits = _copy_wits(R)
    q, r, y = wits[2]
    k = R.sites[2].k_shift
    q[0, 0] += 1 << 16
    r[0, 0] -= 1 << (16 + k)  # Y unchanged, r far outside R_k as well
    assert _reprove(R.sites, wits)[0] == "lhr_sum"


def _flip(pf, off):
    b = bytearray(pf)
    b[off] ^= 1
    return bytes(b)


def test_changed_round_value(honest):
    R, pf, mm = honest
    k = R.sites[0].k_shift
    first_round = mm + 4 * (1 << k) + 4 * 65536 + 16
    assert oracle.verify_hi(2, R.sites, R.wits, _flip(pf, first_round + 8))[0] == "lhr_round"


def test_changed_final_value(honest):
    R, pf, mm = honest
    for i in range(5):
        assert oracle.verify_hi(2, R.sites, R.wits, _flip(pf, len(pf) - 40 + 8 * i + 1))[0] == "lhr_final"


def test_changed_sum(honest):
    R, pf, mm = honest
    k = R.sites[0].k_shift
    assert oracle.verify_hi(2, R.sites, R.wits, _flip(pf, mm + 4 * (1 << k) + 4 * 65536))[0] == "lhr_sum"


def test_truncated_and_trailing(honest):
    R, pf, _ = honest
    assert oracle.verify_hi(2, R.sites, R.wits, pf[:-8])[0] == "format"
    assert oracle.verify_hi(2, R.sites, R.wits, pf + bytes(8))[0] == "format"


def test_tree_form_proof_is_not_accepted(honest):
    R, _, _ = honest
    gkr, _, _ = oracle.prove(2, R.sites, R.wits)
    assert oracle.verify_hi(2, R.sites, R.wits, gkr)[0] != "accept"


def test_weight_change_caught_in_matmul_section(honest):
    R, _, _ = honest
    sites = [copy.copy(s) for s in R.sites]
    w = sites[1].w.copy()
    w[0, 0] ^= 0x01
    sites[1].w = w
    assert _reprove(sites, R.wits)[0] == "mm_round"
