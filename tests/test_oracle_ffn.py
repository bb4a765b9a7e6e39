"""The FFN layer statement in the oracle (the layer proof continued by the per-group scale
reductions, the SiLU lookup of the gate projection's outputs and the gated product with the up
projection's outputs; "How fast can FlashProve go", 3.1). Pins: the proof begins with the layer
proof byte for byte and is accepted; each chained link rejects what it must (a scale reduction
that does not continue from the matmul section's weight value, SiLU outputs that are not the
table's entries for the gate outputs, an up output that is not the gated product's factor)."""

import numpy as np
import pytest

import oracle
import workloads


@pytest.fixture(scope="module")
def ffn():
    wl = workloads.build(3, seed=1, small=True)
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
    assert tail > 8 + 32 * int(np.ceil(np.log2(n))) + 16  # the SiLU lookup and the gated product


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
    pf2, _ = oracle.prove_ffn(3, R.sites, R.wits, s16=s)
    # the lookup's root: the keys' fraction sum is not the table side's
    assert oracle.verify_ffn(3, R.sites, R.wits, pf2, s16=s)[0] == "lookup_root"


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
