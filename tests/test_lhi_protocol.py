"""The host half of the helper-inverse LogUp, without a GPU.

"Towards Proving Frontier-Scale LLM Inference", The proof system: LogUp after
Haboeck 2022, the key side a committed column of inverses h_i = 1/(alpha - r_i)
checked by one sum-check of h + beta eq(z, .) (h (alpha - f) - 1). The library
splits logup_prove_helper_inverse into device values (the helper column's
digest; per round H_t(0), H_t(1) = sums of h and Q_t(0..2) = eq-weighted sums
of h (alpha - f)) and a host half that squeezes every challenge, takes
S = H_1(0) + H_1(1), forms g_t(X) = H_t(X) + beta eq(z_<t, rho_<t) eq(z_t, X)
(Q_t(X) - 1), checks each round against the running claim and writes the proof.
Here the device values come from their definitions (Python modular inverses,
MLEs by hypercube sums) and the proof and transcript state must be the
oracle's, byte for byte.
"""

import struct

import numpy as np
import pytest

from tests import bruteforce as bf
import oracle

P = bf.P


@pytest.fixture(scope="module")
def fp():
    from sum_check_prover_b200 import build
    build.build()
    import sum_check_prover_b200 as m
    return m


class BruteLhi:
    """Device values of the helper-inverse LogUp by their definitions."""

    def __init__(self, r, k, tamper=None):
        self.r = [int(x) for x in r]
        self.k = k
        self.v = max(1, bf.log2c(len(self.r)))
        L = 1 << self.v
        self.f = [x % P for x in self.r] + [0] * (L - len(self.r))
        self.rho = []
        self.tamper = tamper  # (round, index): add one to that value
        self.calls = []

    def column(self, alpha):
        self.calls.append("column")
        self.alpha = alpha
        self.h = [pow((alpha - x) % P, P - 2, P) for x in self.f]
        return bf.tree_digest(b"".join(struct.pack("<Q", x) for x in self.h))

    def start(self, z, beta):
        self.calls.append("start")
        assert len(z) == self.v
        self.z, self.beta = z, beta

    def round(self, t):
        self.calls.append(("round", t))
        assert len(self.rho) == t - 1
        rest = self.v - t
        H, Q = [], []
        for X in range(3):
            hs = qs = 0
            for b in range(1 << rest):
                bits = [(b >> (rest - 1 - i)) & 1 for i in range(rest)]
                w = self.rho + [X] + bits
                hw, fw = bf.mle_at(self.h, w), bf.mle_at(self.f, w)
                hs += hw
                qs += bf.eq_ml(self.z[t:], bits) * hw * (self.alpha - fw)
            H.append(hs % P)
            Q.append(qs % P)
        out = [H[0], H[1], Q[0], Q[1], Q[2]]
        if self.tamper and self.tamper[0] == t:
            out[self.tamper[1]] = (out[self.tamper[1]] + 1) % P
        return out

    def answer(self, t, rho):
        self.calls.append(("answer", t))
        assert t == len(self.rho) + 1
        self.rho.append(rho)

    def finals(self):
        self.calls.append("finals")
        return [bf.mle_at(self.h, self.rho), bf.mle_at(self.f, self.rho)]


def _mult(r, k, v):
    m = np.zeros(1 << k, np.int64)
    for x in list(r) + [0] * ((1 << v) - len(r)):
        j = int(x) + (1 << (k - 1))
        if 0 <= j < (1 << k):
            m[j] += 1
    return m.astype("<u4")


def _drive(fp, seed, r, k, vals):
    tx = fp.Transcript(seed)
    tx.absorb("lhi_site", bf.tree_digest(np.asarray(r, "<i4").tobytes()))
    m = _mult(r, k, vals.v)
    pf = fp.lhi_protocol_drive(tx, vals.v, k, m, bf.tree_digest(m.tobytes()), vals)
    return pf, tx.state()


def _keys(n, k, seed):
    rng = np.random.default_rng(seed)
    return rng.integers(-(1 << (k - 1)), 1 << (k - 1), n).astype(np.int32)


@pytest.mark.parametrize("n,k", [(1, 1), (2, 3), (3, 7), (5, 7), (8, 4), (13, 7), (16, 12), (27, 5)])
def test_host_half_matches_oracle(fp, n, k):
    r = _keys(n, k, 10 * n + k)
    vals = BruteLhi(r, k)
    pf, st = _drive(fp, 7, r, k, vals)
    want, wst = oracle.lhi_prove(7, r, k)
    assert pf == want
    assert st == wst
    v = vals.v
    assert len(pf) == 4 * (1 << k) + 8 + 32 * v + 16
    assert vals.calls == ["column", "start"] + [c for t in range(1, v + 1)
                                                for c in (("round", t), ("answer", t))] + ["finals"]


def test_table_edges_and_keys_outside(fp):
    k = 4
    r = np.array([-8, 7, 0, -1, 3, 9, -100], np.int32)  # 9 and -100 lie outside R_4
    vals = BruteLhi(r, k)
    pf, st = _drive(fp, 2, r, k, vals)
    assert (pf, st) == oracle.lhi_prove(2, r, k)
    assert oracle.lhi_verify(2, r, k, pf)[0] != "accept"


@pytest.mark.parametrize("t,i", [(1, 2), (1, 3), (2, 0), (2, 1), (3, 3)])
def test_inconsistent_round_is_refused(fp, t, i):
    # a wrong H(0), H(1), Q(0) or Q(1) breaks g_t(0) + g_t(1) = claim (round 1 against S)
    r = _keys(8, 5, 3)
    with pytest.raises(fp.FpError):
        _drive(fp, 1, r, 5, BruteLhi(r, 5, tamper=(t, i)))


def test_callback_errors_and_sizes(fp):
    import ctypes as C

    r = _keys(4, 3, 1)

    class Broken(BruteLhi):
        def column(self, alpha):
            raise RuntimeError("no column")

    with pytest.raises(fp.FpError):
        _drive(fp, 0, r, 3, Broken(r, 3))
    L = fp.lib()
    cb = fp._VALUES_FN(lambda *a: 0)
    m = (C.c_uint32 * 8)()
    md = C.create_string_buffer(32)
    ln = C.c_size_t(10)
    buf = C.create_string_buffer(10)
    assert L.fp_lhi_protocol_drive(fp.Transcript(0).h, 2, 3, m, md, cb, None, buf, C.byref(ln)) != 0
    assert ln.value == 4 * 8 + 8 + 32 * 2 + 16
    assert L.fp_lhi_protocol_drive(fp.Transcript(0).h, 0, 3, m, md, cb, None, buf, C.byref(ln)) != 0
    assert L.fp_lhi_protocol_drive(fp.Transcript(0).h, 2, 25, m, md, cb, None, buf, C.byref(ln)) != 0


# ---- the routing proof's sum-check (its range check is the statement above) ------------

class BruteRoute:
    """Device values of the routing sum-check by their definitions (MLEs by hypercube sums)."""

    def __init__(self, l, T, E, tamper=None):
        self.T, self.E = T, E
        self.vT, self.vE = bf.log2c(T), bf.log2c(E)
        self.n = self.vT + self.vE
        self.l = np.asarray(l, np.int64).reshape(-1)
        H, D = bf.route_witness(l, T, E)
        self.H = H.astype(np.int64).reshape(-1)
        self.D = D.astype(np.int64).reshape(-1)
        self.rho = []
        self.tamper = tamper

    def start(self, z, w, lam1, lam2):
        self.z, self.w, self.lam1, self.lam2 = z, w, lam1, lam2
        ze = z[self.vT:]
        self.G, acc = [], 0
        for e in range(self.E):
            self.G.append(acc)
            acc = (acc + bf.eq_ml(ze, [(e >> (self.vE - 1 - b)) & 1 for b in range(self.vE)])) % P

    def claim(self):
        rowsum = sum(bf.eq_ml(self.w[:self.vT], [(t >> (self.vT - 1 - b)) & 1 for b in range(self.vT)])
                     for t in range(self.T)) % P
        return [bf.mle_at(self.D, self.z), bf.mle_at(self.l, self.z), rowsum]

    def _F(self, x):
        xt, xe = x[:self.vT], x[self.vT:]
        Hx, lx, Gx = bf.mle_at(self.H, x), bf.mle_at(self.l, x), bf.mle_at(self.G, xe)
        return (bf.eq_ml(self.z[:self.vT], xt) * Hx * (lx - Gx) + self.lam1 * bf.eq_ml(self.w, x) * Hx * (1 - Hx)
                + self.lam2 * bf.eq_ml(self.w[:self.vT], xt) * Hx) % P

    def round(self, t):
        rest = self.n - t
        g = [sum(self._F(self.rho + [X] + [(b >> (rest - 1 - i)) & 1 for i in range(rest)])
                 for b in range(1 << rest)) % P for X in range(4)]
        if self.tamper == t:
            g[0] = (g[0] + 1) % P
        return g

    def answer(self, t, rho):
        assert t == len(self.rho) + 1
        self.rho.append(rho)

    def finals(self):
        return [bf.mle_at(self.H, self.rho), bf.mle_at(self.l, self.rho)]


def _route_drive(fp, seed, l, T, E, vals):
    H, D = bf.route_witness(l, T, E)
    tx = fp.Transcript(seed)
    tx.absorb("route_site", bf.tree_digest(np.asarray(l, np.int8).tobytes()) + bf.tree_digest(H.tobytes())
              + bf.tree_digest(np.asarray(D, "<i4").tobytes()))
    return fp.route_protocol_drive(tx, vals.n, vals)


@pytest.mark.parametrize("T,E,seed", [(1, 1, 0), (1, 2, 1), (3, 4, 2), (2, 8, 3), (5, 2, 4)])
def test_route_host_half_matches_oracle(fp, T, E, seed):
    l = np.random.default_rng(seed).integers(-4, 4, (T, E)).astype(np.int8)
    vals = BruteRoute(l, T, E)
    pf = _route_drive(fp, seed, l, T, E, vals)
    H, D = oracle.route_witness(l, T, E)
    want, _ = oracle.route_prove(seed, l, H, D, T, E)
    assert len(pf) == 16 + 32 * vals.n + 16
    assert pf == want[:len(pf)]  # the rest of the oracle's proof is the range LogUp


def test_route_inconsistent_round_is_refused(fp):
    l = np.random.default_rng(9).integers(-4, 4, (3, 4)).astype(np.int8)
    with pytest.raises(fp.FpError):
        _route_drive(fp, 1, l, 3, 4, BruteRoute(l, 3, 4, tamper=2))
