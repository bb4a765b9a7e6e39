"""GPU parity of the MoE routing proof through the C ABI.

"How fast can FlashProve go", 2 Background (the note on MoE layers: the routing
computation and each token's choice of expert are proven). The CUDA path (one
warp per token for the first argmax and the committed H and D, the factor
vectors, the openings, one resident degree-3 sum-check, then the helper-
inverse LogUp of D - 128) must write the oracle's H and D and give its proof
bytes and transcript state: one token and one expert (no rounds), ragged token
counts, many ties (few distinct logits), fewer experts than a warp's lanes, and
the MoE layer's 8192 tokens x 128 experts, checked by the oracle's verifier.
The file is named so that pytest collects it after the base-field suites.
"""

import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib_env():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sum_check_prover_b200 import build
    build.build()
    import sum_check_prover_b200 as fp
    return torch, fp


@pytest.fixture
def env(lib_env):
    torch, fp = lib_env
    ctx = fp.Context(0)
    yield torch, fp, ctx
    ctx.close()


def _gpu(env, seed, l, T, E):
    torch, fp, ctx = env
    ld = torch.from_numpy(l).cuda()
    H = torch.empty((T, E), dtype=torch.uint8, device="cuda")
    D = torch.empty((T, E), dtype=torch.int32, device="cuda")
    tx = fp.Transcript(seed)
    pf, status = ctx.prove_routing(tx, ld, T, E, H, D)
    torch.cuda.synchronize()
    return pf, tx.state(), status, H.cpu().numpy(), D.cpu().numpy()


@pytest.mark.parametrize("T,E,lo,hi", [(1, 1, -128, 128), (1, 2, -128, 128), (3, 4, -3, 3), (100, 16, -128, 128),
                                       (257, 8, -2, 2), (1000, 64, -128, 128), (33, 128, -5, 5)])
def test_matches_oracle(env, T, E, lo, hi):
    l = np.random.default_rng(T * 131 + E).integers(lo, hi, (T, E)).astype(np.int8)
    pf, st, status, H, D = _gpu(env, 7, l, T, E)
    Ho, Do = oracle.route_witness(l, T, E)
    assert np.array_equal(H, Ho) and np.array_equal(D, Do)
    assert status == 0
    assert (pf, st) == oracle.route_prove(7, l, Ho, Do, T, E)


def test_stepped_and_resident_give_the_same_proof(env):
    torch, fp, ctx = env
    T, E = 512, 32
    l = np.random.default_rng(5).integers(-128, 128, (T, E)).astype(np.int8)
    a = _gpu(env, 3, l, T, E)[:2]
    ctx.set_profiling(True)  # every round its own launch
    b = _gpu(env, 3, l, T, E)[:2]
    stats = ctx.kernel_stats()
    ctx.set_profiling(False)
    assert a == b
    assert stats["route_round"][0] == 14


def test_argument_errors(env):
    torch, fp, ctx = env
    l = torch.zeros((4, 6), dtype=torch.int8, device="cuda")
    H = torch.empty((4, 6), dtype=torch.uint8, device="cuda")
    D = torch.empty((4, 6), dtype=torch.int32, device="cuda")
    with pytest.raises(fp.FpError):  # E not a power of two
        ctx.prove_routing(fp.Transcript(0), l, 4, 6, H, D)


def test_moe_layer_verified(env):
    # the MoE layer: 8192 tokens routed over 128 experts
    T, E = 8192, 128
    l = np.random.default_rng(11).integers(-128, 128, (T, E)).astype(np.int8)
    pf, st, status, H, D = _gpu(env, 31, l, T, E)
    assert status == 0
    assert oracle.route_verify(31, l, H, D, T, E, pf) == ("accept", (0, 0))
    counts = H.sum(axis=0)
    assert counts.sum() == T and counts.min() > 20
