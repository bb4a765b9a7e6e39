"""GPU parity of the rescale LogUp over the quadratic extension through the C ABI.

"How fast can FlashProve go", 3.1 (the rescale's remainder and the clamp are
proven by lookups) and 4 (the key side is a fraction tree with every level
proven by sum-check; the note on soundness: challenges from an extension
field). The CUDA path (the sites' key columns concatenated, both histograms,
two trees of extension fractions, one resident layer sum-check per level for
both trees, the leaf claims) must give the oracle's proof bytes and transcript
state: one site and several, ragged shapes, and keys outside their tables
(status 1, the same bytes, a proof that does not verify). The file is named so
that pytest collects it after the base-field suites.
"""

import numpy as np
import pytest

import oracle
import workloads
from workloads import device

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


def _committed(env, sites):
    torch, fp, ctx = env
    stages, keep = device.upload(workloads.Workload("lu2", 0, sites))
    ds = stages[0]
    ctx.commit_witness(fp.Transcript(0), ds)
    torch.cuda.synchronize()
    return ds, keep


def _prove(env, seed, ds):
    torch, fp, ctx = env
    tx = fp.Transcript(seed)
    pf, status = ctx.prove_logup_ext2(tx, ds)
    torch.cuda.synchronize()
    return pf, tx.state(), status


@pytest.mark.parametrize("shapes,k", [([(1, 4, 1)], 6), ([(2, 8, 1), (1, 8, 1)], 6), ([(3, 5, 2)], 7),
                                      ([(64, 256, 32), (100, 1000, 37)], 12), ([(257, 300, 9)], 10)])
def test_matches_oracle(env, shapes, k):
    sites = [workloads.random_site(600 + i, M, K, N, 8, k) for i, (M, K, N) in enumerate(shapes)]
    ds, keep = _committed(env, sites)
    wits = [(d.q.cpu().numpy(), d.r.cpu().numpy(), d.y.cpu().numpy()) for d in ds]
    pf, st, status = _prove(env, 5, ds)
    assert status == 0
    assert (pf, st) == oracle.lu2_prove(5, sites, wits)


def test_keys_outside_and_verified(env):
    sites = [workloads.random_site(700, 48, 256, 24, 8, 8)]
    ds, keep = _committed(env, sites)
    wits = [(d.q.cpu().numpy(), d.r.cpu().numpy(), d.y.cpu().numpy()) for d in ds]
    pf, st, status = _prove(env, 6, ds)
    assert status == 0 and oracle.lu2_verify(6, sites, wits, pf) == ("accept", (0, 0))
    ds[0].r[3, 5] += 1 << 8  # a remainder outside R_8
    wits = [(d.q.cpu().numpy(), d.r.cpu().numpy(), d.y.cpu().numpy()) for d in ds]
    pf, st, status = _prove(env, 6, ds)
    assert status == 1
    assert (pf, st) == oracle.lu2_prove(6, sites, wits)
    assert oracle.lu2_verify(6, sites, wits, pf)[0] == "root_rem"
