"""GPU parity of the SiLU lookup through the C ABI.

"How fast can FlashProve go", 2 Background and 3.1: the SiLU's committed
outputs are proven by a lookup into a 2^16-entry table. The CUDA path (one
LogUp-GKR tree, resident layer sum-checks with host-assembled round values)
must give the oracle's proof bytes and transcript state for honest and
dishonest outputs alike (the oracle's verifier then accepts only the honest
ones), on ragged sizes, and the same proof in stepped and resident modes.
"""

import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu
TABLE = None


def table():
    global TABLE
    if TABLE is None:
        TABLE = np.array([oracle.silu_q(v) for v in range(-32768, 32768)], dtype=np.int16)
    return TABLE


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


def _cols(n, seed, lo=-32768, hi=32768):
    rng = np.random.default_rng(seed)
    g = rng.integers(lo, hi, n).astype(np.int16)
    return g, table()[g.astype(np.int64) + 32768]


def _gpu(env, seed, g, s):
    torch, fp, ctx = env
    tx = fp.Transcript(seed)
    pf = ctx.prove_silu(tx, torch.from_numpy(g).cuda(), torch.from_numpy(s).cuda())
    torch.cuda.synchronize()
    return pf, tx.state()


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 8, 13, 300, 1000, 4097, 65537])
def test_matches_oracle(env, n):
    g, s = _cols(n, 10 + n)
    pf, st = _gpu(env, 3, g, s)
    assert (pf, st) == oracle.silu_prove(3, g, s)
    if n <= 4097:
        assert oracle.silu_verify(3, g, s, pf) == ("accept", (0, 0))


@pytest.mark.parametrize("case", ["int8_inputs", "uniform_large", "unaligned"])
def test_histogram_shapes(env, case):
    # the 2^16-row multiplicities over a cluster of two blocks: keys concentrated in a few
    # rows (a projection's int8 outputs as inputs: the window around zero), keys spread over
    # the whole table, and an input column that does not start on a 16-byte boundary
    torch, fp, ctx = env
    if case == "int8_inputs":
        g, s = _cols((1 << 20) + 3, 21, -128, 128)
    else:
        g, s = _cols((1 << 20) + 5 if case == "uniform_large" else 70001, 22)
    if case == "unaligned":
        gb = torch.zeros(len(g) + 3, dtype=torch.int16, device="cuda")
        sb = torch.zeros(len(g) + 3, dtype=torch.int16, device="cuda")
        gd, sd = gb[3:], sb[3:]
        gd.copy_(torch.from_numpy(g))
        sd.copy_(torch.from_numpy(s))
        tx = fp.Transcript(3)
        pf = ctx.prove_silu(tx, gd, sd)
        torch.cuda.synchronize()
        st = tx.state()
    else:
        pf, st = _gpu(env, 3, g, s)
    assert (pf, st) == oracle.silu_prove(3, g, s)


def test_dishonest_output_same_bytes_rejected(env):
    g, s = _cols(500, 4, -2000, 2000)
    s = s.copy()
    s[123] += 1
    pf, st = _gpu(env, 7, g, s)
    assert (pf, st) == oracle.silu_prove(7, g, s)
    assert oracle.silu_verify(7, g, s, pf)[0] == "lookup_root"


EXP = None


def exp_cols(n, seed):
    global EXP
    if EXP is None:
        EXP = np.array([oracle.exp_q(v) for v in range(-32768, 32768)], dtype=np.int16)
    rng = np.random.default_rng(seed)
    g = rng.integers(-3000, 1, n).astype(np.int16)
    return g, EXP[g.astype(np.int64) + 32768]


@pytest.mark.parametrize("n", [1, 3, 5, 100, 1000, 4097])
def test_exp_matches_oracle(env, n):
    # padded sizes exercise the numerator table's padding row (0, 511)
    torch, fp, ctx = env
    g, s = exp_cols(n, 20 + n)
    tx = fp.Transcript(9)
    pf = ctx.prove_exp(tx, torch.from_numpy(g).cuda(), torch.from_numpy(s).cuda())
    torch.cuda.synchronize()
    assert (pf, tx.state()) == oracle.exp_prove(9, g, s)
    assert oracle.exp_verify(9, g, s, pf) == ("accept", (0, 0))


def test_stepped_and_resident_give_the_same_proof(env):
    torch, fp, ctx = env
    g, s = _cols(3000, 5)
    a = _gpu(env, 1, g, s)
    ctx.set_profiling(True)
    b = _gpu(env, 1, g, s)
    ctx.set_profiling(False)
    assert a == b
