"""GPU parity of the helper-inverse LogUp through the C ABI.

"Towards Proving Frontier-Scale LLM Inference", The proof system: LogUp after
Haboeck 2022, the key side a committed helper column of inverses checked by one
sum-check. The CUDA path (histogram, inverses of the table rows, the helper
column as a gather, every round from one resident kernel) must give the
oracle's proof bytes and transcript state: tables of 2 to 2^16 rows (shared-
memory and global histograms), one key (padded to two), ragged key counts
around the kernel's 256-pair blocks, keys on the table's edges, keys outside
the table (status 1, the same bytes, a proof that does not verify), and a
remainder column of the size a 4096-token FFN projection produces, checked by
the oracle's verifier. The file is named so that pytest collects it after the
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


def _keys(n, k, seed):
    rng = np.random.default_rng(seed)
    return rng.integers(-(1 << (k - 1)), 1 << (k - 1), n).astype(np.int32)


def _gpu(env, seed, r, k):
    torch, fp, ctx = env
    tx = fp.Transcript(seed)
    pf, status = ctx.prove_helper_inverse(tx, torch.from_numpy(r).cuda(), k)
    torch.cuda.synchronize()
    return pf, tx.state(), status


@pytest.mark.parametrize("n,k", [(1, 7), (2, 1), (3, 7), (5, 12), (255, 7), (256, 12), (257, 7), (1000, 16),
                                 (4097, 12), (65537, 7), ((1 << 20) + 3, 12)])
def test_matches_oracle(env, n, k):
    r = _keys(n, k, 3000 + n + k)
    pf, st, status = _gpu(env, 5, r, k)
    want, wst = oracle.lhi_prove(5, r, k)
    assert status == 0
    assert pf == want
    assert st == wst


def test_table_edges(env):
    k = 12
    r = np.tile(np.array([-(1 << 11), (1 << 11) - 1, 0, -1], np.int32), 1000)
    pf, st, status = _gpu(env, 2, r, k)
    assert status == 0 and (pf, st) == oracle.lhi_prove(2, r, k)
    assert oracle.lhi_verify(2, r, k, pf) == ("accept", (0, 0))


def test_keys_outside_the_table(env):
    k = 7
    r = _keys(3000, k, 8)
    r[[5, 700, 2999]] = [64, -65, 1 << 30]
    pf, st, status = _gpu(env, 3, r, k)
    assert status == 1
    assert (pf, st) == oracle.lhi_prove(3, r, k)
    assert oracle.lhi_verify(3, r, k, pf)[0] != "accept"


def test_stepped_and_resident_give_the_same_proof(env):
    torch, fp, ctx = env
    r = _keys(70001, 12, 4)
    a = _gpu(env, 9, r, 12)
    ctx.set_profiling(True)  # every round its own launch
    b = _gpu(env, 9, r, 12)
    stats = ctx.kernel_stats()
    ctx.set_profiling(False)
    assert a == b
    assert stats["lhi_round"][0] == 17
    assert oracle.lhi_verify(9, r, 12, a[0]) == ("accept", (0, 0))


def test_argument_errors(env):
    torch, fp, ctx = env
    r = torch.zeros(4, dtype=torch.int32, device="cuda")
    for k in (0, 25):
        with pytest.raises(fp.FpError):
            ctx.prove_helper_inverse(fp.Transcript(0), r, k)
    empty = torch.zeros(0, dtype=torch.int32, device="cuda")
    with pytest.raises(fp.FpError):
        ctx.prove_helper_inverse(fp.Transcript(0), empty, 7)


@pytest.mark.slow
def test_ffn_projection_remainders_verified(env):
    # the remainders of one 4096-token FFN projection of 4096 outputs: 2^24 keys in R_12
    r = _keys(1 << 24, 12, 77)
    pf, st, status = _gpu(env, 31, r, 12)
    assert status == 0
    assert len(pf) == 4 * 4096 + 8 + 32 * 24 + 16
    assert oracle.lhi_verify(31, r, 12, pf) == ("accept", (0, 0))


# ---- the same statement over the quadratic extension --------------------------------------

def _gpu2(env, seed, r, k):
    torch, fp, ctx = env
    tx = fp.Transcript(seed)
    pf, status = ctx.prove_helper_inverse_ext2(tx, torch.from_numpy(r).cuda(), k)
    torch.cuda.synchronize()
    return pf, tx.state(), status


@pytest.mark.parametrize("n,k", [(1, 7), (2, 1), (3, 7), (257, 12), (1000, 16), (4097, 8), (65537, 7)])
def test_ext2_matches_oracle(env, n, k):
    r = _keys(n, k, 5000 + n + k)
    pf, st, status = _gpu2(env, 4, r, k)
    assert status == 0
    assert (pf, st) == oracle.lhi2_prove(4, r, k)


def test_ext2_keys_outside_and_stepped(env):
    torch, fp, ctx = env
    r = _keys(70001, 12, 9)
    r[[3, 60000]] = [5000, -5000]
    a = _gpu2(env, 2, r, 12)
    ctx.set_profiling(True)
    b = _gpu2(env, 2, r, 12)
    stats = ctx.kernel_stats()
    ctx.set_profiling(False)
    assert a == b and a[2] == 1
    assert stats["lhi2_round"][0] == 17
    assert (a[0], a[1]) == oracle.lhi2_prove(2, r, 12)
    assert oracle.lhi2_verify(2, r, 12, a[0])[0] == "lhi2_sum"
