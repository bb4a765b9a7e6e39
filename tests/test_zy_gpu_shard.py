"""One statement shared among ranks, the device half, on one GPU.

"How fast can FlashProve go", 4 Tighter Rooflines (the work spread over the GPUs
of a node). Each rank commits its own sites (witness GEMM, digests), computes
their claims and partial evaluations and its share of every matmul round on its
own fp_ctx, and exchanges site records, claims, round sums and final values
with the other ranks; every rank then runs the lookup section over all keys.
The proof and transcript states of every rank must be the one-rank GPU proof's,
which is the oracle's.

With one GPU the ranks are threads, each with its own context and stream, and
every matmul round runs as its own launch (stepped mode): no kernel waits for
anything another rank produces, only the host threads wait for each other in
the exchange. The file is named so that pytest collects it after the
base-field suites.
"""

import threading

import numpy as np
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
    return torch, fp


class ThreadGather:
    """An all-gather between threads (the virtual ranks' host exchange)."""

    def __init__(self, world: int):
        self.world = world
        self.slots = [None] * world
        self.bar = threading.Barrier(world)

    def for_rank(self, rank: int):
        def ag(data: bytes):
            self.slots[rank] = data
            self.bar.wait(timeout=120)
            out = list(self.slots)
            self.bar.wait(timeout=120)
            return out
        return ag


def desc(fp, d):
    return fp.SiteDesc(d.w, d.xt, d.q, d.r, d.y, d.M, d.K, d.N, d.w_bits, d.k_shift, d.scales, d.w_digest)


def prove_shared(torch, fp, wl, seed, site_lo):
    stages, keep = device.upload(wl)
    assert len(stages) == 1
    world = len(site_lo) - 1
    gather = ThreadGather(world)
    ctxs = [fp.Context(0) for _ in range(world)]
    device.weight_digests(ctxs[0], stages)
    sites = [desc(fp, d) for d in stages[0]]
    out, errs = [None] * world, []

    def run(rank):
        try:
            ctx = ctxs[rank]
            ctx.set_profiling(True)  # every round its own launch
            shard = fp.Shard(rank, world, site_lo, gather.for_rank(rank))
            mine = [s if i in shard.own else fp.SiteDesc(None, None, None, None, None, s.M, s.K, s.N, s.w_bits,
                                                          s.k_shift) for i, s in enumerate(sites)]
            stream = torch.cuda.Stream()
            with torch.cuda.stream(stream):
                tx = fp.Transcript(seed)
                ctx.commit_witness_shard(tx, mine, shard, stream)
                s0 = tx.state()
                mm = ctx.prove_matmul_shard(tx, mine, shard, stream)
                stream.synchronize()
            out[rank] = (tx, mm, s0, tx.state())
        except Exception as e:  # noqa: BLE001 -- reported below
            errs.append((rank, e))
            gather.bar.abort()

    th = [threading.Thread(target=run, args=(r,)) for r in range(world)]
    for t in th:
        t.start()
    for t in th:
        t.join(timeout=600)
    assert not errs, errs
    # the lookup section over all keys, on each rank's context in turn (each rank's sites
    # wrote their own witness into the shared buffers)
    res = []
    for rank in range(world):
        tx, mm, s0, s1 = out[rank]
        ctxs[rank].set_profiling(False)
        lu, status = ctxs[rank].prove_logup(tx, sites)
        torch.cuda.synchronize()
        res.append((mm + lu, [s0, s1, tx.state()], status))
        tx.close()
    wits = [(d.q.cpu().numpy(), d.r.cpu().numpy(), d.y.cpu().numpy()) for d in stages[0]]
    for c in ctxs:
        c.close()
    return res, wits


def one_rank(torch, fp, wl, seed):
    stages, keep = device.upload(wl)
    ctx = fp.Context(0)
    try:
        device.weight_digests(ctx, stages)
        proof, states, status = fp.prove(ctx, seed, stages)
        torch.cuda.synchronize()
    finally:
        ctx.close()
    return proof, states, status


@pytest.mark.parametrize("world,site_lo", [(2, [0, 7, 15]), (2, [0, 14, 15]), (3, [0, 3, 8, 15])])
def test_shared_moe_statement_equals_one_rank_and_oracle(env, world, site_lo):
    torch, fp = env
    wl = workloads.build(5, seed=1, small=True)  # 4 experts + the shared expert: 15 sites
    assert len(wl.sites) == 15
    res, wits = prove_shared(torch, fp, wl, 7, site_lo)
    want = one_rank(torch, fp, wl, 7)
    R = oracle.resolve(wl)
    for i, (q, r, y) in enumerate(R.wits):
        assert np.array_equal(wits[i][0], q) and np.array_equal(wits[i][1], r) and np.array_equal(wits[i][2], y)
    opf, ostates, _ = oracle.prove(7, R.sites, R.wits)
    assert want[0] == opf and want[1] == ostates
    for proof, states, status in res:
        assert status == 0
        assert states == ostates
        assert proof == opf


def test_shared_random_sites(env):
    torch, fp = env
    shapes = [(100, 1000, 37, 4, True), (64, 256, 32, 8, False), (257, 300, 51, 4, False), (17, 4097, 9, 4, True)]
    sites = [workloads.random_site(800 + i, M, K, N, b, 9, scales=sc) for i, (M, K, N, b, sc) in enumerate(shapes)]
    wl = workloads.Workload("shard", 0, sites)
    res, wits = prove_shared(torch, fp, wl, 8, [0, 1, 4])
    R = oracle.resolve(wl)
    opf, ostates, _ = oracle.prove(8, R.sites, R.wits)
    for proof, states, status in res:
        assert proof == opf and states == ostates
