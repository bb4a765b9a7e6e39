"""GPU parity of the SiLU and softmax numerator lookups over the quadratic extension.

"How fast can FlashProve go", 2 Background and 3.1 (non-polynomial steps are
proven by lookups), 4 (the key side is a fraction tree with every level proven
by sum-check; the note on soundness: challenges from an extension field). The
CUDA path (histogram, the tree of extension fractions one level per launch,
one resident layer sum-check per level, the leaf claims with the padding row's
share) must give the oracle's proof bytes and transcript state for both tables:
one key (padded to two), ragged key counts around the 256-pair blocks, keys on
the table's edges, and 2^20 keys checked by the oracle's verifier. The file is
named so that pytest collects it after the base-field suites.
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


def _cols(n, seed, table):
    rng = np.random.default_rng(seed)
    if table == "silu":
        g = rng.integers(-32768, 32768, n).astype(np.int16)
        tab = np.array([oracle.silu_q(int(v)) for v in range(-32768, 32768)], np.int64)
    else:
        g = rng.integers(-4000, 1, n).astype(np.int16)
        tab = np.array([oracle.exp_q(int(v)) for v in range(-32768, 32768)], np.int64)
    return g, tab[g.astype(np.int64) + 32768].astype(np.int16)


def _gpu(env, seed, g, s, table):
    torch, fp, ctx = env
    tx = fp.Transcript(seed)
    fn = ctx.prove_silu_ext2 if table == "silu" else ctx.prove_exp_ext2
    pf = fn(tx, torch.from_numpy(g).cuda(), torch.from_numpy(s).cuda())
    torch.cuda.synchronize()
    return pf, tx.state()


@pytest.mark.parametrize("table", ["silu", "exp"])
@pytest.mark.parametrize("n", [1, 2, 3, 5, 255, 256, 257, 1000, 4097, 65537])
def test_matches_oracle(env, table, n):
    g, s = _cols(n, 4000 + n, table)
    want = oracle.silu2_prove(7, g, s) if table == "silu" else oracle.exp2_prove(7, g, s)
    assert _gpu(env, 7, g, s, table) == want


def test_table_edges_and_stepped(env):
    torch, fp, ctx = env
    g = np.tile(np.array([-32768, 32767, 0, -1, 1], np.int16), 2000)
    tab = {int(v): oracle.silu_q(int(v)) for v in set(g.tolist())}
    s = np.array([tab[int(v)] for v in g], np.int16)
    a = _gpu(env, 3, g, s, "silu")
    ctx.set_profiling(True)  # every layer round its own launch
    b = _gpu(env, 3, g, s, "silu")
    stats = ctx.kernel_stats()
    ctx.set_profiling(False)
    assert a == b == oracle.silu2_prove(3, g, s)
    # 2^14 keys: layers 1..13, each round its own launch and each layer's end (its child values
    # at the layer's point) one more launch of the same kernel
    assert stats["silu2_round"][0] == sum(range(1, 14)) + 13


def test_many_keys_verified(env):
    g, s = _cols(1 << 20, 99, "silu")
    pf, st = _gpu(env, 11, g, s, "silu")
    assert oracle.silu2_verify(11, g, s, pf) == ("accept", (0, 0))
