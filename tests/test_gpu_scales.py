"""GPU parity of the per-group scale reduction through the C ABI.

W_eff[i][k] = S[i][k // 64] w[i][k] is a product of two committed factors that
is itself never committed; the matmul sum-check's claim on W_eff~ is reduced to
claims on w~ and S~ by the product sum-check ("How fast can FlashProve go", 3.1).
The CUDA path must give the oracle's proof bytes and transcript state on ragged
shapes (int4 and int8, K below, at and above one 64-column group, M and K not
powers of two, a single row and a single column) and on the FFN's gate
projection (14336 x 4096 int4 with scales), which the oracle's verifier checks
in full. The CUDA path takes the grouped road (the rounds over the rows and the
64-column groups on S and the group sums W', the last six rounds on the host),
so equal bytes also pin that road to the plain product sum-check.
"""

import numpy as np
import pytest

import oracle
import workloads

pytestmark = pytest.mark.gpu
P = oracle.P


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


def _site(M, K, bits, seed):
    rng = np.random.default_rng(seed)
    w = workloads.int4_packed(rng, M, K) if bits == 4 else workloads.int8_uniform(rng, (M, K))
    sc = workloads.group_scales(rng, M, K)
    v = oracle.log2_ceil(M) + oracle.log2_ceil(K)
    z = [int(x) for x in rng.integers(0, P, size=v, dtype=np.uint64)]
    return w, sc, z


def _gpu(env, seed, w, bits, sc, M, K, z):
    torch, fp, ctx = env
    tx = fp.Transcript(seed)
    pf = ctx.reduce_scales(tx, torch.from_numpy(np.ascontiguousarray(w)).cuda(), bits,
                           torch.from_numpy(np.ascontiguousarray(sc)).cuda(), M, K, z)
    torch.cuda.synchronize()
    return pf, tx.state()


@pytest.mark.parametrize("M,K,bits", [(1, 1, 4), (1, 2, 8), (2, 64, 4), (3, 20, 8), (5, 130, 4), (64, 256, 4),
                                      (17, 1000, 8), (100, 64, 8), (300, 4096, 4), (1000, 777, 8), (1, 64, 4),
                                      (1, 65, 8), (2, 1, 8), (7, 33, 4), (129, 127, 4), (4, 2048, 8)])
def test_matches_oracle(env, M, K, bits):
    w, sc, z = _site(M, K, bits, 3 * M + K)
    pf, st = _gpu(env, 6, w, bits, sc, M, K, z)
    assert (pf, st) == oracle.scl_prove(6, w, bits, sc, M, K, z)


def test_committed_digest_gives_the_same_proof(env):
    # D(W) || D(S) committed in advance (the site's weight digest) stands in for digesting here
    torch, fp, ctx = env
    M, K, bits = 37, 300, 4
    w, sc, z = _site(M, K, bits, 5)
    wd = torch.from_numpy(np.ascontiguousarray(w)).cuda()
    sd = torch.from_numpy(np.ascontiguousarray(sc)).cuda()
    dg = ctx.digest(wd, wd.numel()) + ctx.digest(sd, sd.numel())
    tx = fp.Transcript(4)
    pf = ctx.reduce_scales(tx, wd, bits, sd, M, K, z, w_digest=dg)
    assert (pf, tx.state()) == oracle.scl_prove(4, w, bits, sc, M, K, z)
    with pytest.raises(ValueError):
        ctx.reduce_scales(fp.Transcript(4), wd, bits, sd, M, K, z, w_digest=dg[:32])


def test_stepped_and_resident_give_the_same_proof(env):
    torch, fp, ctx = env
    M, K, bits = 500, 3000, 4
    w, sc, z = _site(M, K, bits, 12)
    a = _gpu(env, 1, w, bits, sc, M, K, z)
    ctx.set_profiling(True)
    b = _gpu(env, 1, w, bits, sc, M, K, z)
    stats = ctx.kernel_stats()
    ctx.set_profiling(False)
    assert a == b
    # the rounds over the row and column-group coordinates run on the device, the last six
    # (the columns inside a 64-column group) on the host
    assert stats["had_round"][0] == len(z) - 6
    assert stats["scl_group"][0] == 1


@pytest.mark.slow
def test_ffn_gate_full_size_verified(env):
    M, K, bits = 14336, 4096, 4
    w, sc, z = _site(M, K, bits, 41)
    pf, _ = _gpu(env, 2, w, bits, sc, M, K, z)
    assert len(pf) == 8 + 32 * 26 + 16
    assert oracle.scl_verify(2, w, bits, sc, M, K, z, pf) == ("accept", (0, 0))


def test_argument_errors(env):
    torch, fp, ctx = env
    w, sc, z = _site(4, 64, 4, 1)
    wd = torch.from_numpy(np.ascontiguousarray(w)).cuda()
    sd = torch.from_numpy(np.ascontiguousarray(sc)).cuda()
    with pytest.raises(fp.FpError):  # weights are int4 or int8
        ctx.reduce_scales(fp.Transcript(0), wd, 2, sd, 4, 64, z)
    with pytest.raises(fp.FpError):  # a coordinate that is not a field element
        ctx.reduce_scales(fp.Transcript(0), wd, 4, sd, 4, 64, [P] + z[1:])
    with pytest.raises(ValueError):  # the point has vM + vK coordinates
        ctx.reduce_scales(fp.Transcript(0), wd, 4, sd, 4, 64, z[:-1])
    with pytest.raises(fp.FpError):  # M = 0: the binding asks for the 6 column coordinates, the library refuses
        ctx.reduce_scales(fp.Transcript(0), wd, 4, sd, 0, 64, [1] * 6)
    # the context is still usable afterwards
    pf, _ = _gpu(env, 6, w, 4, sc, 4, 64, z)
    assert pf == oracle.scl_prove(6, w, 4, sc, 4, 64, z)[0]
