"""GPU parity of the MoE dispatch proof (sumcheck_prove_dispatch) through the C ABI.

"How fast can FlashProve go", 2 Background (the note on MoE layers). The CUDA
path (the claim through the partial evaluation with row weights, positions by a
per-expert stable scan, the layer input's rows dotted with the column eq table,
the rounds on the matmul sum-check's kernel) must give the oracle's proof bytes
and transcript state: tiny and ragged statements, experts with no tokens, the
MoE layer's own routing and inputs at full size; a routing with an expert index
out of range is refused. The file is named so that pytest collects it after the
base-field suites.
"""

import numpy as np
import pytest

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sum_check_prover_b200 import build
    build.build()
    import sum_check_prover_b200 as fp
    ctx = fp.Context(0)
    yield torch, fp, ctx
    ctx.close()


def gpu(env, seed, X, e, D, E, stepped=False):
    torch, fp, ctx = env
    tx = fp.Transcript(seed)
    ctx.set_profiling(stepped)
    try:
        pf = ctx.prove_dispatch(tx, torch.from_numpy(np.ascontiguousarray(X)).cuda(),
                                torch.from_numpy(np.ascontiguousarray(e, dtype=np.int32)).cuda(),
                                torch.from_numpy(np.ascontiguousarray(D)).cuda(), E)
        torch.cuda.synchronize()
    finally:
        ctx.set_profiling(False)
    return pf, tx.state()


def statement(seed, T, K, E):
    rng = np.random.default_rng(seed)
    X = rng.integers(-128, 128, (T, K)).astype(np.int8)
    e = rng.integers(0, E, T).astype(np.int32)
    return X, e, X[np.argsort(e, kind="stable")]


@pytest.mark.parametrize("T,K,E", [(1, 1, 1), (5, 3, 2), (64, 256, 8), (100, 1000, 7), (513, 300, 40), (37, 64, 200)])
def test_matches_oracle(env, T, K, E):
    X, e, D = statement(T + K + E, T, K, E)
    assert gpu(env, 4, X, e, D, E) == oracle.dsp_prove(4, X, e, D, E)


def test_moe_layer_full_size(env):
    X, e, D = workloads.moe_dispatch(0)
    pf, st = gpu(env, 5, X, e, D, 128)
    assert (pf, st) == oracle.dsp_prove(5, X, e, D, 128)
    assert oracle.dsp_verify(5, X, e, D, 128, pf)[0] == "accept"


def test_stepped_and_resident(env):
    X, e, D = statement(9, 300, 128, 16)
    assert gpu(env, 6, X, e, D, 16) == gpu(env, 6, X, e, D, 16, stepped=True)


def test_dishonest_dispatch_is_rejected(env):
    # rows of two experts swapped. The GPU prover takes each round's g(1) from the running claim,
    # so for a false statement its rounds stay consistent and the proof fails at its end; the
    # oracle's prover evaluates g(1) in full and fails at the first round: both are rejected
    X, e, D = statement(10, 200, 96, 6)
    D2 = D.copy()
    D2[[0, -1]] = D2[[-1, 0]]
    pf, st = gpu(env, 7, X, e, D2, 6)
    honest, _ = gpu(env, 7, X, e, D, 6)
    assert pf != honest
    assert oracle.dsp_verify(7, X, e, D2, 6, pf)[0] == "dsp_final"
    assert oracle.dsp_verify(7, X, e, D2, 6, oracle.dsp_prove(7, X, e, D2, 6)[0])[0] == "dsp_round"


def test_expert_index_out_of_range(env):
    torch, fp, ctx = env
    X, e, D = statement(11, 20, 8, 4)
    e = e.copy()
    e[3] = 4
    with pytest.raises(fp.FpError) as ex:
        gpu(env, 8, X, e, D, 4)
    assert ex.value.code == -1
