"""GPU parity of the extension-field gated-product sum-check through the C ABI.

"How fast can FlashProve go", 3.1 (the gated product is proven by sum-check,
never committed) and 4 (the note on soundness: challenges from an extension
field). The CUDA path (round values h_t(0..2) in F_p[phi]/(phi^2 - 7) from a
resident kernel, the claim taken from round 1) must give the oracle's proof
bytes (textbook three-vector sum-check over the extension) and transcript state
on every size: one entry (no rounds), powers of two, ragged tails around the
kernel's 256-pair blocks and its 2^8-entry eq chunks, and sizes that spread over
many blocks. The full-size case is the FFN's hidden tensor, checked by the
oracle's verifier. The file is named so that pytest collects it after the
base-field suites.
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
    pf = ctx.prove_hadamard_ext2(tx, torch.from_numpy(s).cuda(), torch.from_numpy(u).cuda())
    torch.cuda.synchronize()
    return pf, tx.state()


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 8, 13, 255, 256, 257, 511, 513, 1000, 4097, 65537, (1 << 20) + 3])
def test_matches_oracle(env, n):
    s, u = _vecs(n, 2000 + n)
    pf, st = _gpu(env, 5, s, u)
    want, wst = oracle.had2_prove(5, s, u)
    assert pf == want
    assert st == wst


def test_extreme_values(env):
    n = 3000
    for a, b in ((-128, -128), (127, -128), (0, 77)):
        s = np.full(n, a, np.int8)
        u = np.full(n, b, np.int8)
        pf, st = _gpu(env, 2, s, u)
        assert (pf, st) == oracle.had2_prove(2, s, u)


def test_stepped_and_resident_give_the_same_proof(env):
    torch, fp, ctx = env
    s, u = _vecs(70001, 3)
    a = _gpu(env, 9, s, u)
    ctx.set_profiling(True)  # every round its own launch
    b = _gpu(env, 9, s, u)
    stats = ctx.kernel_stats()
    ctx.set_profiling(False)
    assert a == b
    assert stats["had2_round"][0] == 17
    assert oracle.had2_verify(9, s, u, a[0]) == ("accept", (0, 0))


def test_base_and_extension_proofs_differ(env):
    # the same statement with base-field challenges is another proof of another length
    s, u = _vecs(1000, 4)
    torch, fp, ctx = env
    base = ctx.prove_hadamard(fp.Transcript(1), torch.from_numpy(s).cuda(), torch.from_numpy(u).cuda())
    ext, _ = _gpu(env, 1, s, u)
    assert len(base) == 8 + 32 * 10 + 16 and len(ext) == 16 + 64 * 10 + 32


def test_argument_errors(env):
    torch, fp, ctx = env
    s = torch.zeros(4, dtype=torch.int8, device="cuda")
    u = torch.zeros(5, dtype=torch.int8, device="cuda")
    with pytest.raises(ValueError):
        ctx.prove_hadamard_ext2(fp.Transcript(0), s, u)
    empty = torch.zeros(0, dtype=torch.int8, device="cuda")
    with pytest.raises(fp.FpError):
        ctx.prove_hadamard_ext2(fp.Transcript(0), empty, empty)


@pytest.mark.slow
def test_ffn_hidden_full_size_verified(env):
    # the FFN's gated product: 4096 tokens x 14336 hidden units, 5.9e7 entries (v = 26)
    n = 4096 * 14336
    s, u = _vecs(n, 78)
    pf, st = _gpu(env, 32, s, u)
    assert len(pf) == 16 + 64 * 26 + 32
    assert oracle.had2_verify(32, s, u, pf) == ("accept", (0, 0))
