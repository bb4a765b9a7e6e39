"""GPU parity of the gated-product sum-check through the C ABI.

"How fast can FlashProve go", 3.1 Committing intermediate values: the MLP's
gated product h = s (.) u is proven by sum-check without being committed.
The CUDA path (claim-derived round values from a resident kernel) must give
the oracle's proof bytes (textbook three-vector sum-check) and transcript
state on every size: one entry (no rounds), powers of two, ragged tails
around the kernel's 256-pair blocks, and sizes that spread over many blocks.
The full-size case is the FFN's hidden tensor, checked by the oracle's
verifier.
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


def _vecs(n, seed):
    rng = np.random.default_rng(seed)
    return rng.integers(-128, 128, n).astype(np.int8), rng.integers(-128, 128, n).astype(np.int8)


def _gpu(env, seed, s, u):
    torch, fp, ctx = env
    tx = fp.Transcript(seed)
    pf = ctx.prove_hadamard(tx, torch.from_numpy(s).cuda(), torch.from_numpy(u).cuda())
    torch.cuda.synchronize()
    return pf, tx.state()


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 8, 13, 255, 256, 257, 511, 1000, 4097, 65537, (1 << 20) + 3])
def test_matches_oracle(env, n):
    s, u = _vecs(n, 1000 + n)
    pf, st = _gpu(env, 5, s, u)
    want, wst = oracle.had_prove(5, s, u)
    assert pf == want
    assert st == wst


def test_extreme_values(env):
    n = 3000
    for a, b in ((-128, -128), (127, -128), (0, 77)):
        s = np.full(n, a, np.int8)
        u = np.full(n, b, np.int8)
        pf, st = _gpu(env, 2, s, u)
        assert (pf, st) == oracle.had_prove(2, s, u)


def test_stepped_and_resident_give_the_same_proof(env):
    torch, fp, ctx = env
    s, u = _vecs(70001, 3)
    a = _gpu(env, 9, s, u)
    ctx.set_profiling(True)  # every round its own launch
    b = _gpu(env, 9, s, u)
    stats = ctx.kernel_stats()
    ctx.set_profiling(False)
    assert a == b
    assert stats["had_round"][0] == 17


def test_argument_errors(env):
    torch, fp, ctx = env
    s = torch.zeros(4, dtype=torch.int8, device="cuda")
    u = torch.zeros(5, dtype=torch.int8, device="cuda")
    with pytest.raises(ValueError):
        ctx.prove_hadamard(fp.Transcript(0), s, u)
    empty = torch.zeros(0, dtype=torch.int8, device="cuda")
    with pytest.raises(fp.FpError):
        ctx.prove_hadamard(fp.Transcript(0), empty, empty)


@pytest.mark.slow
def test_ffn_hidden_full_size_verified(env):
    # the FFN's gated product: 4096 tokens x 14336 hidden units, 5.9e7 entries (v = 26)
    n = 4096 * 14336
    s, u = _vecs(n, 77)
    pf, st = _gpu(env, 31, s, u)
    assert len(pf) == 8 + 32 * 26 + 16
    assert oracle.had_verify(31, s, u, pf) == ("accept", (0, 0))
