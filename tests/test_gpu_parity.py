"""GPU parity: the CUDA path against the CPU oracle, through the C ABI.

Bit-exact everywhere (integer witness, field elements, digests, proof bytes,
transcript states). Sizes span several tiles and ragged tails; the oracle
finishes each in seconds. The oracle's verifier must accept every GPU proof.
"""

import random

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
    # a fresh context per test: scratch under-reservation cannot hide behind
    # an arena that an earlier test already grew
    torch, fp = lib_env
    ctx = fp.Context(0)
    yield torch, fp, ctx
    ctx.close()


def run_gpu(env, wl, seed, digests=True):
    torch, fp, ctx = env
    stages, keep = device.upload(wl)
    if digests:
        device.weight_digests(ctx, stages)
    proof, states, status = fp.prove(ctx, seed, stages)
    torch.cuda.synchronize()
    return proof, states, status, stages, keep


def check_against_oracle(env, wl, seed, digests=True):
    proof, states, status, stages, keep = run_gpu(env, wl, seed, digests)
    R = oracle.resolve(wl)
    flat = [d for st in stages for d in st]
    for d, (q, r, y) in zip(flat, R.wits):
        assert np.array_equal(d.q.cpu().numpy(), q), d.name
        assert np.array_equal(d.r.cpu().numpy(), r), d.name
        assert np.array_equal(d.y.cpu().numpy(), y), d.name
    opf, ostates, off = oracle.prove(seed, R.sites, R.wits)
    assert states == ostates
    assert proof == opf
    # an honest witness lies in both tables unless some |q| needs more than 16 bits
    k = R.sites[0].k_shift
    in_domain = all(int(q.min()) >= -32768 and int(q.max()) < 32768 for q, r, y in R.wits)
    verdict = oracle.verify(seed, R.sites, R.wits, proof)[0]
    if in_domain:
        assert status == 0 and verdict == "accept"
    else:
        assert status == 1 and verdict == "root_clamp"
    return proof


# ---- building blocks --------------------------------------------------------------

@pytest.mark.parametrize("n", [0, 1, 63, 64, 1000, 1024, 1025, 32 * 1024, 33 * 1024 + 5, 1 << 21, (1 << 21) + 7])
@pytest.mark.parametrize("offset", [0, 3])
def test_digest_matches_oracle(env, n, offset):
    torch, fp, ctx = env
    rnd = np.random.default_rng(n + offset)
    data = rnd.integers(0, 256, size=n + offset, dtype=np.uint8)
    t = torch.from_numpy(data).cuda()
    ptr = t.data_ptr() + offset if n else None
    assert ctx.digest(ptr, n) == oracle.tree_digest(data[offset:].tobytes())


PE_SHAPES = [
    # rows, cols, bits, scales
    (1, 1, 8, False), (5, 37, 8, False), (64, 4096, 4, False), (300, 257, 4, False), (129, 1000, 4, True),
    (4096, 512, 8, False), (17, 96, 8, True), (2000, 2048, 4, True), (3, 7, 4, False), (16384, 64, 4, False),
    # whole 32-byte row slices (the tensor-core path): ragged row chunks, several scale groups
    (1000, 192, 4, True), (33, 32, 8, False), (257, 640, 8, True), (31, 64, 4, False), (300, 1536, 8, False),
]


def test_digests_in_one_pass_match_one_by_one(env):
    torch, fp, ctx = env
    rng = np.random.default_rng(8)
    bufs = [torch.from_numpy(rng.integers(0, 256, n, dtype=np.uint8)).cuda() for n in (1, 1024, 5000, 1 << 20)]
    pairs = [(b, b.numel()) for b in bufs] + [(bufs[2][7:], bufs[2].numel() - 7), (None, 0)]
    got = ctx.digest_many(pairs)
    want = b"".join(ctx.digest(b, n) for b, n in pairs)
    assert got == want
    assert got[:32] == oracle.tree_digest(bufs[0].cpu().numpy().tobytes())


@pytest.mark.parametrize("shape", PE_SHAPES)
def test_partial_eval_matches_oracle(env, shape):
    torch, fp, ctx = env
    rows, cols, bits, sc = shape
    rng = np.random.default_rng(rows * 7 + cols)
    if bits == 4:
        mat = workloads.int4_packed(rng, rows, cols)
    else:
        mat = workloads.int8_uniform(rng, (rows, cols))
    scales = workloads.group_scales(rng, rows, cols) if sc else None
    v = oracle.log2_ceil(rows)
    z = [int(x) for x in rng.integers(0, oracle.P, size=v, dtype=np.uint64)]
    want = oracle.partial_rows(mat, bits, scales, rows, cols, z)
    out = torch.empty(len(want), dtype=torch.int64, device="cuda")
    ctx.partial_eval(torch.from_numpy(mat).cuda(), bits,
                     None if scales is None else torch.from_numpy(scales).cuda(), rows, cols, z, out)
    torch.cuda.synchronize()
    got = out.cpu().numpy().view(np.uint64)
    assert np.array_equal(got, want)


# ---- whole proofs -----------------------------------------------------------------

def test_tiny_config(env):
    check_against_oracle(env, workloads.build(1), 0)


@pytest.mark.parametrize("config", [3, 4, 5])
def test_small_layer_configs(env, config):
    check_against_oracle(env, workloads.build(config, seed=3, small=True), 3)


def test_projection_config(env):
    check_against_oracle(env, workloads.build(2), 0)


def _random_case(i):
    rnd = random.Random(1000 + i)
    k = rnd.choice([1, 3, 7, 12, 18])
    sites = []
    for j in range(rnd.choice([1, 1, 2, 3])):
        bits = rnd.choice([4, 8])
        M = rnd.choice([1, 2, 5, 64, 130, 257])
        K = rnd.choice([1, 3, 32, 64, 100, 160, 513])
        N = rnd.choice([1, 4, 9, 128, 200])
        sc = bits == 4 and rnd.random() < 0.4
        sites.append(workloads.random_site(50 * i + j, M, K, N, bits, k, scales=sc, act=rnd.random() < 0.7))
    return workloads.Workload(f"rand{i}", i, sites)


@pytest.mark.parametrize("i", range(24))
def test_random_shapes_and_seeds(env, i):
    check_against_oracle(env, _random_case(i), 77 + i)


@pytest.mark.parametrize("k", [14, 15, 16, 17, 18])
def test_remainder_tables_over_a_cluster(env, k):
    # k = 15..18: the remainder table is counted in the distributed shared memory of a cluster
    # of 2^(k-15) blocks; k = 14 is the one-block table. Two sites, one unaligned in size.
    sites = [workloads.random_site(3000 + k, 257, 513, 200, 4, k, scales=True),
             workloads.random_site(3100 + k, 130, 160, 9, 8, k)]
    check_against_oracle(env, workloads.Workload(f"cl{k}", 0, sites), 40 + k)


def test_tampered_clamp_over_a_cluster_is_flagged(env):
    torch, fp, ctx = env
    s = workloads.random_site(3200, 64, 96, 33, 8, 16)
    stages, keep = device.upload(workloads.Workload("t16", 0, [s]))
    tx = fp.Transcript(0)
    ctx.commit_witness(tx, stages[0])
    d = stages[0][0]
    d.y[3, 5] = (int(d.y[3, 5]) + 1) if int(d.y[3, 5]) < 127 else 126
    torch.cuda.synchronize()
    ctx.prove_matmul(tx, stages[0])
    lu, status = ctx.prove_logup(tx, stages[0])
    assert status == 1
    tx.close()


def test_inline_weight_digests_give_the_same_proof(env):
    wl = workloads.build(3, seed=5, small=True)
    a = run_gpu(env, wl, 5, digests=True)[0]
    b = run_gpu(env, wl, 5, digests=False)[0]
    assert a == b


def test_unaligned_operands(env):
    torch, fp, ctx = env
    s = workloads.random_site(9, 70, 96, 33, 8, 9)
    wl = workloads.Workload("u", 0, [s])
    R = oracle.resolve(wl)
    wb = torch.zeros(s.M * s.K + 5, dtype=torch.int8, device="cuda")
    xb = torch.zeros(s.N * s.K + 7, dtype=torch.int8, device="cuda")
    w = wb[5:].view(s.M, s.K)
    xt = xb[7:].view(s.N, s.K)
    w.copy_(torch.from_numpy(s.w))
    xt.copy_(torch.from_numpy(s.xt))
    q = torch.empty((s.N, s.M), dtype=torch.int32, device="cuda")
    r = torch.empty_like(q)
    y = torch.empty((s.N, s.M), dtype=torch.int8, device="cuda")
    d = fp.SiteDesc(w, xt, q, r, y, s.M, s.K, s.N, 8, 9)
    proof, states, status = fp.prove(ctx, 1, [[d]])
    assert proof == oracle.prove(1, R.sites, R.wits)[0]


def test_tampered_clamp_is_flagged_and_rejected(env):
    torch, fp, ctx = env
    wl = workloads.build(1)
    stages, keep = device.upload(wl)
    tx = fp.Transcript(0)
    ctx.commit_witness(tx, stages[0])
    d = stages[0][0]
    d.y[3, 5] = (int(d.y[3, 5]) + 1) if int(d.y[3, 5]) < 127 else 126
    torch.cuda.synchronize()
    mm = ctx.prove_matmul(tx, stages[0])
    lu, status = ctx.prove_logup(tx, stages[0])
    assert status == 1
    R = oracle.resolve(wl)
    q, r, y = R.wits[0]
    y = d.y.cpu().numpy()
    name, _ = oracle.verify(0, R.sites, [(q, r, y)], mm + lu)
    assert name in ("root_clamp", "format", "claim")  # the statement's y changed after commit
    tx.close()


def test_argument_errors(env):
    torch, fp, ctx = env
    wl = workloads.build(1)
    stages, keep = device.upload(wl)
    tx = fp.Transcript(0)
    with pytest.raises(fp.FpError):
        ctx.commit_witness(tx, [])
    d = stages[0][0]
    bad = device.DevSite("bad", d.w, None, d.xt, d.q, d.r, d.y, d.M, d.K, d.N, 8, 0)
    with pytest.raises(fp.FpError):
        ctx.commit_witness(tx, [bad])
    big = device.DevSite("big", d.w, None, d.xt, d.q, d.r, d.y, d.M, 200000, d.N, 8, 7)
    with pytest.raises(fp.FpError):
        ctx.commit_witness(tx, [big])
    mix = device.DevSite("mix", d.w, None, d.xt, d.q, d.r, d.y, d.M, d.K, d.N, 8, 6)
    ctx.commit_witness(tx, [d])
    with pytest.raises(fp.FpError):
        ctx.prove_logup(tx, [d, mix])
    tx.close()


def test_stepped_and_resident_rounds_give_the_same_proof(env):
    torch, fp, ctx = env
    wl = workloads.build(3, seed=8, small=True)
    a = run_gpu(env, wl, 8)[0]
    ctx.set_profiling(True)        # profiling launches every round separately
    b = run_gpu(env, wl, 8)[0]
    stats = ctx.kernel_stats()
    ctx.set_profiling(False)
    assert a == b
    assert stats["gkr_round"][0] > 20 and stats["sc_round"][0] >= 8


def test_bounded_wait_times_out_and_context_survives(env):
    torch, fp, ctx = env
    assert ctx.session_selftest() == -4      # FP_ERR_TIMEOUT, reported, not hung
    check_against_oracle(env, workloads.build(1), 0)
