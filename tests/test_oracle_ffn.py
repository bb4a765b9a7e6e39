"""The FFN layer statement in the oracle (the layer proof continued by the per-group scale
reductions, the rescale of the hidden activations that the down projection reads, the SiLU lookup
of the gate projection's outputs and the gated product with the up projection's outputs; "How
fast can FlashProve go", 3.1). Pins: the rescale against exact rational rounding over every pair
of 8-bit factors; the proof begins with the layer proof byte for byte and is accepted; each
chained link rejects what it must (a scale reduction that does not continue from the matmul
section's weight value, SiLU outputs that are not the table's entries for the gate outputs, an
up output that is not the gated product's factor, a remainder outside R_kh, a rescale that does
not reconstruct the product, a down operand that is not the rescaled product)."""

import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads


@pytest.fixture(scope="module")
def ffn():
    wl = workloads.build(3, seed=1, small=True, chained=True)
    R = oracle.resolve(wl)
    pf, st = oracle.prove_ffn(3, R.sites, R.wits)
    return R, pf


def test_prefix_is_the_layer_proof_and_accepted(ffn):
    R, pf = ffn
    base, _, _ = oracle.prove(3, R.sites, R.wits)
    assert pf[: len(base)] == base
    assert oracle.verify_ffn(3, R.sites, R.wits, pf)[0] == "accept"
    # three scale reductions (8 + 32 v + 16 bytes each) follow the layer proof
    vs = [int(np.ceil(np.log2(s.M))) + int(np.ceil(np.log2(s.K))) for s in R.sites]
    n = R.sites[0].M * R.sites[0].N
    tail = len(pf) - len(base) - sum(8 + 32 * v + 16 for v in vs)
    # the hidden lookup (its multiplicity tables alone 4 (2^7 + 2^16) bytes), the SiLU lookup and
    # the gated product
    assert tail > 4 * (2 ** 7 + 2 ** 16) + 8 + 32 * int(np.ceil(np.log2(n))) + 16


def test_silu_outputs_fit_eight_bits():
    s = oracle.silu_outputs(np.arange(-128, 128))
    assert s.min() == oracle.silu_q(-128) and s.max() == oracle.silu_q(127)
    assert -128 <= s.min() and s.max() <= 127
    # SiLU shrinks: |silu(v)| <= |v|, with silu(0) = 0
    v = np.arange(-128, 128)
    assert np.all(np.abs(s) <= np.abs(v)) and s[128] == 0


def test_scale_reduction_claim_is_tied_to_the_matmul(ffn):
    R, pf = ffn
    base, _, _ = oracle.prove(3, R.sites, R.wits)
    bad = bytearray(pf)
    bad[len(base)] ^= 1  # the first scale reduction's claim
    assert oracle.verify_ffn(3, R.sites, R.wits, bytes(bad))[0] in ("ffn_link", "format")


def test_wrong_silu_output_is_rejected(ffn):
    R, pf = ffn
    s = oracle.silu_outputs(R.wits[0][2]).copy()
    i = int(np.argmax(np.abs(s)))
    s.reshape(-1)[i] += 1
    hid = honest_hidden(R)
    pf2, _ = oracle.prove_ffn(3, R.sites, R.wits, s16=s, hidden=hid)
    # the lookup's root: the keys' fraction sum is not the table side's
    assert oracle.verify_ffn(3, R.sites, R.wits, pf2, s16=s, hidden=hid)[0] == "lookup_root"


def test_wrong_up_output_is_rejected(ffn):
    R, pf = ffn
    wits = [list(w) for w in R.wits]
    y = wits[1][2].copy()
    y.reshape(-1)[5] ^= 1
    wits[1][2] = y
    assert oracle.verify_ffn(3, R.sites, [tuple(w) for w in wits], pf)[0] != "accept"


def test_outputs_outside_eight_bits_are_refused(ffn):
    R, _ = ffn
    s = oracle.silu_outputs(R.wits[0][2]).copy()
    s.reshape(-1)[0] = 300
    with pytest.raises(ValueError):
        oracle.prove_ffn(3, R.sites, R.wits, s16=s)


def honest_hidden(R, kh=7):
    s8 = oracle.silu_outputs(R.wits[0][2]).astype(np.int8)
    return [a.copy() for a in oracle.ffn_hidden(s8, R.wits[1][2], kh)]


@pytest.mark.parametrize("kh", [1, 7, 14])
def test_hidden_rescale_is_exact_rounding(kh):
    # every pair of 8-bit factors: q = floor(h / 2^kh + 1/2) in exact rationals, r = h - 2^kh q,
    # y = q clamped to 8 bits
    a = np.repeat(np.arange(-128, 128), 256).astype(np.int8)
    b = np.tile(np.arange(-128, 128), 256).astype(np.int8)
    q, r, y = oracle.ffn_hidden(a, b, kh)
    for i in range(0, a.size, 97):
        h = int(a[i]) * int(b[i])
        qq = math.floor(Fraction(h, 2 ** kh) + Fraction(1, 2))
        assert (q[i], r[i], y[i]) == (qq, h - qq * 2 ** kh, max(-128, min(127, qq)))
    h = a.astype(np.int64) * b
    assert np.array_equal(q.astype(np.int64) * 2 ** kh + r, h)
    assert r.min() >= -(2 ** (kh - 1)) and r.max() < 2 ** (kh - 1)
    with pytest.raises(ValueError):
        oracle.ffn_hidden(a[:4], b[:4], 17)


def test_down_reads_the_rescaled_hidden(ffn):
    R, _ = ffn
    q, r, y = honest_hidden(R)
    assert np.array_equal(R.sites[2].xt, y)
    # with kh = 7 the products of SiLU outputs (at most 79 in size) and 8-bit up outputs mostly
    # stay inside 8 bits after the rescale
    assert np.mean(q == y) > 0.99


def test_remainder_outside_the_table_is_rejected(ffn):
    R, _ = ffn
    q, r, y = honest_hidden(R)
    i = int(np.argmax(r < 63))
    q.reshape(-1)[i] -= 1
    r.reshape(-1)[i] += 128  # still reconstructs the product, but r is outside R_7
    pf2, _ = oracle.prove_ffn(3, R.sites, R.wits, hidden=(q, r, y))
    assert oracle.verify_ffn(3, R.sites, R.wits, pf2, hidden=(q, r, y))[0] == "root_rem"


def test_rescale_that_misses_the_product_is_rejected(ffn):
    R, _ = ffn
    q, r, y = honest_hidden(R)
    i = int(np.argmax(r < 63))
    r.reshape(-1)[i] += 1  # in R_7, but 2^7 q + r is no longer s u
    pf2, _ = oracle.prove_ffn(3, R.sites, R.wits, hidden=(q, r, y))
    assert oracle.verify_ffn(3, R.sites, R.wits, pf2, hidden=(q, r, y))[0] == "ffn_hidden"


def test_down_operand_other_than_the_hidden_is_rejected(ffn):
    R, pf = ffn
    q, r, y = honest_hidden(R)
    i = int(np.argmax(np.abs(q) < 100))
    q.reshape(-1)[i] += 1
    r.reshape(-1)[i] -= 128
    y.reshape(-1)[i] += 1  # a consistent clamp pair, but not the down site's committed X
    assert oracle.verify_ffn(3, R.sites, R.wits, pf, hidden=(q, r, y))[0] == "ffn_down"


def test_unchained_down_site_is_rejected():
    wl = workloads.build(3, seed=1, small=True)  # the down site's X a seeded stand-in
    R = oracle.resolve(wl)
    pf, _ = oracle.prove_ffn(3, R.sites, R.wits)
    assert oracle.verify_ffn(3, R.sites, R.wits, pf)[0] == "ffn_down"
