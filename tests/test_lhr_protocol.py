"""The host half of the helper-inverse lookup section (logup_prove_rescale_hi) on the CPU.

"Towards Proving Frontier-Scale LLM Inference", The proof system (LogUp after
Haboeck 2022). The library's host half runs with its device values supplied by
a callback that computes them from their definitions (Python integers: the
helper columns by modular inverses, every round's sums over the cube of the
folded columns, the eq weights as direct products); after the site records and
the matmul section (driven the same way), the whole proof and the final
transcript state must be the oracle's (prove_hi), byte for byte.
"""

import struct

import numpy as np
import pytest

import oracle
import workloads
from tests import bruteforce as bf
from tests.test_shard_protocol import RankValues, absorb_records, shape_sites

P = bf.P


class LhrValues:
    """The device values of the helper-inverse rounds, from the definitions."""

    def __init__(self, keys, k):
        self.R, self.Q, self.Y = ([int(x) % P for x in col] for col in keys)
        self.k = k
        self.r = None

    def column(self, a0, a1, gamma):
        self.a0, self.a1, self.gamma = a0, a1, gamma
        self.H0 = [pow((a0 - x) % P, P - 2, P) for x in self.R]
        self.H1 = [pow((a1 - q - gamma * y) % P, P - 2, P) for q, y in zip(self.Q, self.Y)]
        pack = lambda col: b"".join(struct.pack("<Q", x) for x in col)  # noqa: E731
        self.V = [self.H0, self.H1, self.R, self.Q, self.Y]
        return bf.tree_digest(pack(self.H0)) + bf.tree_digest(pack(self.H1))

    def start(self, z, beta):
        self.z = z

    def _fold(self):
        if self.r is None:
            return
        h = len(self.V[0]) // 2
        self.V = [[(c[b] + self.r * (c[b + h] - c[b])) % P for b in range(h)] for c in self.V]
        self.r = None

    def round(self, t):
        self._fold()
        h = len(self.V[0]) // 2
        H0, H1, R, Q, Y = self.V
        E = [bf.eq_point(self.z[t:], b) for b in range(h)]  # eq(z_{t+1..v}, b)
        out = [sum(H0[:h]), sum(H0[h:]), sum(H1[:h]), sum(H1[h:])]
        for col in (0, 1):
            for X in range(3):
                acc = 0
                for b in range(h):
                    at = [c[b] + X * (c[b + h] - c[b]) for c in self.V]
                    if col == 0:
                        acc += E[b] * at[0] * (self.a0 - at[2])
                    else:
                        acc += E[b] * at[1] * (self.a1 - at[3] - self.gamma * at[4])
                out.append(acc)
        return [x % P for x in out]

    def answer(self, t, rho):
        self.r = rho

    def finals(self):
        self._fold()
        return [c[0] for c in self.V]


def multiplicities(keys, k):
    fr, fq, _ = keys
    m = np.zeros((1 << k) + 65536, np.int64)
    for x in fr:
        if 0 <= x + (1 << (k - 1)) < (1 << k):
            m[x + (1 << (k - 1))] += 1
    for x in fq:
        if 0 <= x + 32768 < 65536:
            m[(1 << k) + x + 32768] += 1
    rem = m[:1 << k].astype("<u4").tobytes()
    cl = m[1 << k:].astype("<u4").tobytes()
    return m.astype(np.uint32), bf.tree_digest(rem) + bf.tree_digest(cl)


def drive(seed, sites, wits):
    import sum_check_prover_b200 as fp
    tx = fp.Transcript(seed)
    absorb_records(tx, sites, wits)
    mm = fp.mm_shard_protocol_drive(tx, shape_sites(sites), None, RankValues(sites, wits, range(len(sites))))
    fr, fq, fy, v = bf.lookup_keys(sites, wits)
    k = sites[0].k_shift
    m, dg = multiplicities((fr, fq, fy), k)
    lu = fp.lhr_protocol_drive(tx, v, k, m, dg, LhrValues((fr, fq, fy), k))
    return mm + lu, tx.state()


@pytest.mark.parametrize("seed,shapes", [
    (1, [(4, 8, 2, 8, 3, False)]),
    (2, [(3, 5, 3, 4, 9, False), (2, 70, 3, 4, 9, True)]),
    (3, [(8, 16, 4, 8, 6, False), (5, 9, 2, 4, 6, False), (1, 3, 1, 8, 6, False)]),
])
def test_host_half_matches_the_oracle(seed, shapes):
    sites = [workloads.random_site(300 + 10 * seed + i, M, K, N, b, k, scales=sc)
             for i, (M, K, N, b, k, sc) in enumerate(shapes)]
    wits = [oracle.witness(s) for s in sites]
    proof, state = drive(seed, sites, wits)
    want, states, _ = oracle.prove_hi(seed, sites, wits)
    assert proof == want
    assert state == states[2]


def test_keys_outside_the_tables_still_give_the_oracle_proof():
    sites = [workloads.random_site(71, 6, 20, 4, 8, 5)]
    wits = [tuple(a.copy() for a in oracle.witness(sites[0]))]
    q, r, y = wits[0]
    r[0, 0] += 1 << 5  # outside R_5
    q[0, 0] -= 1
    y[1, 1] = 99 if q[1, 1] != 99 else 98  # not clamp(q)
    proof, state = drive(4, sites, wits)
    want, states, _ = oracle.prove_hi(4, sites, wits)
    assert proof == want and state == states[2]
    assert oracle.verify_hi(4, sites, wits, proof)[0] == "lhr_sum"


def test_inconsistent_round_values_are_refused():
    import sum_check_prover_b200 as fp

    class Wrong(LhrValues):
        def round(self, t):
            out = super().round(t)
            out[4] = (out[4] + 1) % P
            return out

    sites = [workloads.random_site(72, 4, 8, 2, 8, 3)]
    wits = [oracle.witness(sites[0])]
    fr, fq, fy, v = bf.lookup_keys(sites, wits)
    m, dg = multiplicities((fr, fq, fy), 3)
    with pytest.raises(fp.FpError):
        fp.lhr_protocol_drive(fp.Transcript(1), v, 3, m, dg, Wrong((fr, fq, fy), 3))
