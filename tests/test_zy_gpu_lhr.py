"""GPU parity of the helper-inverse lookup section (logup_prove_rescale_hi) through the C ABI.

"Towards Proving Frontier-Scale LLM Inference", The proof system (LogUp after
Haboeck 2022), set against the fraction tree of "How fast can FlashProve go", 4.
The layer proof with this lookup section (fp.prove(..., lookup="hi")) must give
the oracle's proof bytes and transcript states (prove_hi) on the tiny matmul,
the FFN and MoE layers at reduced sizes, ragged random statements, and a
witness with keys outside both tables; every round as its own launch must give
the same proof as the resident kernel. The file is named so that pytest
collects it after the base-field suites.
"""

import pytest

import oracle
import workloads
from workloads import device

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


def gpu_prove(env, wl, seed, stepped=False):
    torch, fp, ctx = env
    stages, keep = device.upload(wl)
    device.weight_digests(ctx, stages)
    ctx.set_profiling(stepped)
    try:
        proof, states, status = fp.prove(ctx, seed, stages, lookup="hi")
        torch.cuda.synchronize()
    finally:
        ctx.set_profiling(False)
    wits = [(d.q.cpu().numpy(), d.r.cpu().numpy(), d.y.cpu().numpy()) for st in stages for d in st]
    return proof, states, status, wits


@pytest.mark.parametrize("cfg,small", [(1, False), (3, True), (5, True), (4, True)])
def test_layer_proof_matches_oracle(env, cfg, small):
    wl = workloads.build(cfg, seed=3, small=small)
    proof, states, status, wits = gpu_prove(env, wl, 5)
    R = oracle.resolve(wl)
    want, ostates, _ = oracle.prove_hi(5, R.sites, R.wits)
    assert status == 0
    assert states == ostates
    assert proof == want
    assert oracle.verify_hi(5, R.sites, R.wits, proof)[0] == "accept"


@pytest.mark.parametrize("shapes", [[(100, 1000, 37, 4, True)], [(1, 1, 1, 8, False)],
                                    [(64, 256, 32, 8, False), (257, 300, 51, 4, False), (3, 5, 2, 4, True)]])
def test_random_statements(env, shapes):
    sites = [workloads.random_site(900 + i, M, K, N, b, 9, scales=sc) for i, (M, K, N, b, sc) in enumerate(shapes)]
    wl = workloads.Workload("lhr", 0, sites)
    proof, states, status, wits = gpu_prove(env, wl, 6)
    want, ostates, _ = oracle.prove_hi(6, sites, [oracle.witness(s) for s in sites])
    assert proof == want and states == ostates


def test_stepped_and_resident_give_the_same_proof(env):
    wl = workloads.build(5, seed=4, small=True)
    a = gpu_prove(env, wl, 7)[:2]
    b = gpu_prove(env, wl, 7, stepped=True)[:2]
    assert a == b


def test_keys_outside_the_tables(env):
    # a dishonest witness (a remainder outside R_6 with q - 1, an output that is not clamp(q))
    # written into the device buffers, then the lookup section alone on a fresh transcript:
    # the GPU must give what the host half gives with values from their definitions, which
    # the CPU tests pin to the oracle
    torch, fp, ctx = env
    from tests import bruteforce as bf
    from tests.test_lhr_protocol import LhrValues, multiplicities
    site = workloads.random_site(77, 40, 64, 12, 8, 6)
    stages, keep = device.upload(workloads.Workload("lhr_out", 0, [site]))
    d = stages[0][0]
    ctx.commit_witness(fp.Transcript(0), [d])
    q, r, y = (t.cpu().numpy() for t in (d.q, d.r, d.y))
    r[0, 0] += 1 << 6
    q[0, 0] -= 1
    y[1, 1] = 100 if q[1, 1] != 100 else 101
    d.q.copy_(torch.from_numpy(q))
    d.r.copy_(torch.from_numpy(r))
    d.y.copy_(torch.from_numpy(y))
    tx = fp.Transcript(8)
    lu, status = ctx.prove_logup_hi(tx, [d])
    torch.cuda.synchronize()
    assert status == 1  # FP_WARN_KEYS_OUTSIDE_TABLE
    fr, fq, fy, v = bf.lookup_keys([site], [(q, r, y)])
    m, dg = multiplicities((fr, fq, fy), 6)
    tx2 = fp.Transcript(8)
    want = fp.lhr_protocol_drive(tx2, v, 6, m, dg, LhrValues((fr, fq, fy), 6))
    assert lu == want and tx.state() == tx2.state()
