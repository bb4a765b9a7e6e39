"""GPU parity of the extension-field matmul sum-check through the C ABI.

"How fast can FlashProve go", 2 Background (the matmul reduced by sum-check to
claims on its operands) and 4 (the note on soundness: challenges from an
extension field). The CUDA path (extension eq tables, row contractions with
16-byte weights for A = W_eff~(r_row, .) and B = X~(., r_col), the claim over
the committed witness, every round from one resident kernel) must give the
oracle's proof bytes and transcript state on a single entry (no rounds), ragged
shapes in all three dimensions, int4 with and without per-64 scales, int8, and
an FFN-sized projection; with the weights' digest computed by the call and
taken from an offline commitment. The file is named so that pytest collects it
after the base-field suites.
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


def _site(M, K, N, bits, scales, seed):
    s = workloads.random_site(seed, M, K, N, bits, 6)
    if scales:
        s.scales = workloads.group_scales(np.random.default_rng(seed), M, K)
    return s


def _prove(env, s, seed, offline_digest=False):
    torch, fp, ctx = env
    stages, keep = device.upload(workloads.Workload("mm2", 0, [s]))
    d = stages[0][0]
    if offline_digest:
        device.weight_digests(ctx, stages)
    ctx.commit_witness(fp.Transcript(0), [d])  # the witness q, r, y on the device
    tx = fp.Transcript(seed)
    pf = ctx.prove_matmul_ext2(tx, d)
    torch.cuda.synchronize()
    return pf, tx.state(), d


@pytest.mark.parametrize("M,K,N,bits,scales", [(1, 1, 1, 8, False), (1, 2, 1, 4, False), (3, 5, 2, 4, True),
                                               (64, 256, 32, 8, False), (100, 1000, 37, 4, True),
                                               (17, 1023, 9, 8, True), (17, 4097, 9, 4, True),
                                               (257, 300, 513, 4, False)])
def test_matches_oracle(env, M, K, N, bits, scales):
    s = _site(M, K, N, bits, scales, 500 + M + K + N)
    wit = oracle.witness(s)
    pf, st, d = _prove(env, s, 6)
    assert np.array_equal(d.q.cpu().numpy(), wit[0]) and np.array_equal(d.r.cpu().numpy(), wit[1])
    want, wst = oracle.mm2_prove(6, s, wit)
    assert pf == want
    assert st == wst


def test_int8_with_scales_past_the_exact_domain_is_refused(env):
    # int8 weights times int8 scales reach 128 * 128 * 128 * K; at K = 4097 that passes 2^31, so the
    # int32 accumulation of the witness could wrap and the call refuses the site as out of domain
    torch, fp, ctx = env
    s = _site(17, 4097, 9, 8, True, 41)
    stages, keep = device.upload(workloads.Workload("mm2", 0, [s]))
    with pytest.raises(fp.FpError) as e:
        ctx.commit_witness(fp.Transcript(0), [stages[0][0]])
    assert e.value.code == -2  # FP_ERR_SHAPE
    s = _site(17, 1023, 9, 8, True, 41)  # the largest K in the domain for int8 with scales
    stages, keep = device.upload(workloads.Workload("mm2", 0, [s]))
    ctx.commit_witness(fp.Transcript(0), [stages[0][0]])


def test_offline_weight_digest_gives_the_same_proof(env):
    s = _site(48, 640, 24, 4, True, 9)
    a = _prove(env, s, 3)[:2]
    b = _prove(env, s, 3, offline_digest=True)[:2]
    assert a == b == oracle.mm2_prove(3, s, oracle.witness(s))


def test_stepped_and_resident_give_the_same_proof(env):
    torch, fp, ctx = env
    s = _site(128, 2048, 64, 4, False, 10)
    a = _prove(env, s, 4)[:2]
    ctx.set_profiling(True)  # every round its own launch
    b = _prove(env, s, 4)[:2]
    stats = ctx.kernel_stats()
    ctx.set_profiling(False)
    assert a == b
    assert stats["mm2_round"][0] == 11
    assert oracle.mm2_verify(4, s, oracle.witness(s), a[0]) == ("accept", (0, 0))


def test_ffn_projection_verified(env):
    # a Llama-3.1-8B FFN down projection slice: W 4096 x 14336 int4 with per-64 scales, 64 tokens
    s = _site(4096, 14336, 64, 4, True, 11)
    pf, st, d = _prove(env, s, 12)
    assert len(pf) == 16 + 48 * 14 + 32
    assert oracle.mm2_verify(12, s, oracle.witness(s), pf) == ("accept", (0, 0))


# ---- Freivalds' check, the prover's side (the comparison statement) ------------------

def _freivalds(env, s, seed, offline_digest=False):
    torch, fp, ctx = env
    stages, keep = device.upload(workloads.Workload("frv", 0, [s]))
    d = stages[0][0]
    if offline_digest:
        device.weight_digests(ctx, stages)
    ctx.commit_witness(fp.Transcript(0), [d])
    tx = fp.Transcript(seed)
    pf = ctx.prove_freivalds(tx, d)
    torch.cuda.synchronize()
    return pf, tx.state()


@pytest.mark.parametrize("M,K,N,bits,scales", [(1, 1, 1, 8, False), (3, 5, 2, 4, True), (64, 256, 300, 8, False),
                                               (100, 1000, 4097, 4, True)])
def test_freivalds_matches_oracle(env, M, K, N, bits, scales):
    s = _site(M, K, N, bits, scales, 700 + M + K + N)
    w = oracle.witness(s)
    pf, st = _freivalds(env, s, 2)
    assert (pf, st) == oracle.frv_prove(2, s, w)
    assert oracle.frv_verify(2, s, w, pf) == ("accept", (0, 0))


def test_freivalds_offline_weight_digest(env):
    s = _site(32, 640, 48, 4, True, 12)
    assert _freivalds(env, s, 5) == _freivalds(env, s, 5, offline_digest=True) == oracle.frv_prove(5, s,
                                                                                                   oracle.witness(s))
