"""One matmul statement proven by several ranks, on the CPU (gloo), through the
host half of sumcheck_prove_matmul_shard with each rank's device values supplied
by a callback.

"How fast can FlashProve go", 4 Tighter Rooflines: the work of a batch is spread
over the GPUs of a node. The sites of a statement are independent until their
claims are combined, so each rank holds some sites and computes, from its own
sites only, the claims, the partial evaluations A_s = W~_s(r_row, .) and
B_s = X~_s(., r_col), and its share of every round's g(0), g(2); the ranks
exchange those small values. Here each rank's values come straight from their
definitions (Python integers, every MLE a direct eq-weighted sum) and the
exchange is a gloo all-gather between processes. The proof bytes and the
transcript state after the matmul section must be the one-rank proof's, which
the CPU oracle writes.
"""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import oracle
import workloads
from tests import bruteforce as bf

P = bf.P

# ragged shapes in all three dimensions, int4 with and without scales, int8
SHAPES = [(6, 40, 3, 4, False), (16, 64, 8, 8, False), (9, 33, 5, 4, True), (3, 70, 2, 4, False),
          (12, 17, 4, 8, False)]


def statement(seed: int):
    sites = [workloads.random_site(100 * seed + i, M, K, N, bits, 6, scales=sc)
             for i, (M, K, N, bits, sc) in enumerate(SHAPES)]
    return sites, [oracle.witness(s) for s in sites]


class RankValues:
    """This rank's device values for its own sites, from the definitions."""

    def __init__(self, sites, wits, own):
        self.sites, self.wits, self.own = sites, wits, list(own)
        self.n = max(bf.log2c(s.K) for s in sites)
        self.r = None

    def start(self, rr, rc):
        L = 1 << self.n
        self.rr, self.rc = rr, rc
        self.A, self.B = [], []
        for i in self.own:
            s = self.sites[i]
            er = [bf.eq_point(rr[:bf.log2c(s.M)], x) for x in range(s.M)]
            ec = [bf.eq_point(rc[:bf.log2c(s.N)], x) for x in range(s.N)]
            W = bf.weights(s)
            A = [sum(er[m] * int(W[m, k]) for m in range(s.M)) % P if k < s.K else 0 for k in range(L)]
            B = [sum(ec[j] * int(s.xt[j, k]) for j in range(s.N)) % P if k < s.K else 0 for k in range(L)]
            self.A.append(A)
            self.B.append(B)

    def claims(self):
        out = []
        for i in self.own:
            s, (q, r, y) = self.sites[i], self.wits[i]
            Yq = (q.astype(np.int64) << s.k_shift) + r.astype(np.int64)
            out.append(bf.mle2(Yq.T, self.rr[:bf.log2c(s.M)], self.rc[:bf.log2c(s.N)]))
        return out

    def weights(self, rho):
        self.rho = list(rho)

    def _fold(self):
        if self.r is None:
            return
        for vecs in (self.A, self.B):
            for j, v in enumerate(vecs):
                h = len(v) // 2
                vecs[j] = [(v[b] + self.r * (v[b + h] - v[b])) % P for b in range(h)]
        self.r = None

    def round(self, t):
        self._fold()
        g0 = g2 = 0
        for w, A, B in zip(self.rho, self.A, self.B):
            h = len(A) // 2
            s0 = sum(A[b] * B[b] for b in range(h))
            s2 = sum((2 * A[b + h] - A[b]) * (2 * B[b + h] - B[b]) for b in range(h))
            g0 += w * s0
            g2 += w * s2
        return [g0 % P, g2 % P]

    def answer(self, t, r):
        self.r = r

    def finals(self):
        self._fold()
        out = []
        for A, B in zip(self.A, self.B):
            out += [A[0], B[0]]
        return out


def shape_sites(sites):
    import sum_check_prover_b200 as fp
    return [fp.SiteDesc(None, None, None, None, None, s.M, s.K, s.N, s.w_bits, s.k_shift) for s in sites]


def absorb_records(tx, sites, wits):
    for d in bf.site_digests(sites, wits):
        tx.absorb("site", d)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, seed: int, site_lo, q):
    import datetime

    import torch.distributed as td

    import sum_check_prover_b200 as fp

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    td.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        sites, wits = statement(seed)
        shard = fp.Shard(rank, world, site_lo, fp.torch_allgather())
        tx = fp.Transcript(seed)
        absorb_records(tx, sites, wits)
        proof = fp.mm_shard_protocol_drive(tx, shape_sites(sites), shard, RankValues(sites, wits, shard.own))
        q.put((rank, proof, tx.state()))
        td.barrier()
    finally:
        td.destroy_process_group()


def run_ranks(world: int, seed: int, site_lo):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, seed, site_lo, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return got


@pytest.mark.parametrize("world,site_lo", [(2, [0, 2, 5]), (2, [0, 4, 5]), (3, [0, 1, 3, 5])])
def test_ranks_write_the_one_rank_proof(world, site_lo):
    seed = 3
    sites, wits = statement(seed)
    want, states, mm_len = oracle.prove(seed, sites, wits)
    got = run_ranks(world, seed, site_lo)
    for rank, proof, state in got:
        assert proof == want[:mm_len], rank
        assert state == states[1], rank


def test_one_rank_without_shard_matches_the_oracle():
    import sum_check_prover_b200 as fp
    seed = 4
    sites, wits = statement(seed)
    want, states, mm_len = oracle.prove(seed, sites, wits)
    tx = fp.Transcript(seed)
    absorb_records(tx, sites, wits)
    assert tx.state() == states[0]
    proof = fp.mm_shard_protocol_drive(tx, shape_sites(sites), None, RankValues(sites, wits, range(len(sites))))
    assert proof == want[:mm_len] and tx.state() == states[1]


def test_a_rank_with_the_wrong_share_changes_the_proof():
    # planted in the callback's values (the host half is unchanged): one rank leaves a site
    # out of its round share; the exchange then sums to other round values
    import sum_check_prover_b200 as fp
    seed = 5
    sites, wits = statement(seed)
    want, states, mm_len = oracle.prove(seed, sites, wits)

    class Dropping(RankValues):
        def round(self, t):
            self.rho = [0] + self.rho[1:]
            return super().round(t)

    tx = fp.Transcript(seed)
    absorb_records(tx, sites, wits)
    proof = fp.mm_shard_protocol_drive(tx, shape_sites(sites), None, Dropping(sites, wits, range(len(sites))))
    assert len(proof) == mm_len and proof != want[:mm_len]
    assert oracle.verify(seed, sites, wits, proof + want[mm_len:])[0] != "accept"


def test_failed_exchange_and_bad_ranges_are_refused():
    import sum_check_prover_b200 as fp
    sites, wits = statement(6)

    def broken(_data):
        raise RuntimeError("peer gone")

    tx = fp.Transcript(6)
    absorb_records(tx, sites, wits)
    sh = fp.Shard(0, 2, [0, 2, 5], broken)
    with pytest.raises(fp.FpError):
        fp.mm_shard_protocol_drive(tx, shape_sites(sites), sh, RankValues(sites, wits, sh.own))
    for lo in ([0, 0, 5], [0, 3, 4], [1, 3, 5]):  # an empty rank, not covering, not starting at 0
        with pytest.raises(fp.FpError):
            fp.mm_shard_protocol_drive(fp.Transcript(6), shape_sites(sites), fp.Shard(0, 2, lo, broken),
                                       RankValues(sites, wits, range(0)))


def test_balanced_site_ranges():
    import sum_check_prover_b200 as fp
    assert fp.balance_sites([1] * 5, 2) == [0, 3, 5]
    assert fp.balance_sites([5, 1, 1, 1], 2) == [0, 1, 4]
    assert fp.balance_sites([1, 1, 1], 3) == [0, 1, 2, 3]
    lo = fp.balance_sites([1] * 387, 8)
    assert lo[0] == 0 and lo[-1] == 387 and all(b > a for a, b in zip(lo, lo[1:]))
