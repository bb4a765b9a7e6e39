"""The host half of the extension-field gated-product proof, without a GPU.

"How fast can FlashProve go", 3.1 (the gated product is proven by sum-check)
and 4 (the note on soundness: challenges from an extension field). The library
splits sumcheck_prove_hadamard_ext2 into device round values h_t(0..2) and a
host half that squeezes the point and the challenges, forms the round
polynomials g_t(X) = eq(z_<t, rho_<t) eq(z_t, X) h_t(X), takes the claim from
round 1, checks every later round against the running claim, and writes the
proof. Here the round values come from a brute-force restatement (every value a
hypercube sum of MLEs at extension points) and the proof and the transcript
state must be the oracle's, byte for byte; the extension arithmetic on the
host side of the library is the same code its kernels use.
"""

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


class BruteValues:
    """Device values of the gated-product sum-check by their definitions."""

    def __init__(self, s, u, tamper=None):
        self.s = [int(x) for x in s]
        self.u = [int(x) for x in u]
        self.v = bf.log2c(len(self.s))
        self.rho = []
        self.tamper = tamper  # (round, X): add one to that value
        self.calls = []

    def start(self, z):
        assert len(z) == self.v
        self.z = z
        self.calls.append("start")

    def single(self):
        self.calls.append("single")
        c = self.s[0] * self.u[0] % P
        return [(c, 0), (self.s[0] % P, 0), (self.u[0] % P, 0)]

    def round(self, t):
        self.calls.append(("round", t))
        assert len(self.rho) == t - 1
        rest = self.v - t
        out = []
        for X in range(3):
            acc = (0, 0)
            for b in range(1 << rest):
                bits = [((b >> (rest - 1 - i)) & 1, 0) for i in range(rest)]
                pt = self.rho + [(X, 0)] + bits
                e = bf.x_eq(self.z[t:], bits)
                acc = bf.x_add(acc, bf.x_mul(e, bf.x_mul(bf.x_mle(self.s, pt), bf.x_mle(self.u, pt))))
            if self.tamper == (t, X):
                acc = ((acc[0] + 1) % P, acc[1])
            out.append(acc)
        return out

    def answer(self, t, rho):
        self.calls.append(("answer", t))
        assert t == len(self.rho) + 1
        self.rho.append(rho)

    def finals(self):
        self.calls.append("finals")
        return [bf.x_mle(self.s, self.rho), bf.x_mle(self.u, self.rho)]


def _site_tx(fp, seed, s, u):
    tx = fp.Transcript(seed)
    tx.absorb("had2_site", bf.tree_digest(np.asarray(s, np.int8).tobytes())
              + bf.tree_digest(np.asarray(u, np.int8).tobytes()))
    return tx


def _vecs(n, seed):
    rng = np.random.default_rng(seed)
    return rng.integers(-128, 128, n).astype(np.int8), rng.integers(-128, 128, n).astype(np.int8)


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 8, 13, 16, 27])
def test_host_half_matches_oracle(fp, n):
    s, u = _vecs(n, 40 + n)
    tx = _site_tx(fp, 9, s, u)
    vals = BruteValues(s, u)
    pf = fp.had2_protocol_drive(tx, vals.v, vals)
    want, wst = oracle.had2_prove(9, s, u)
    assert pf == want
    assert tx.state() == wst
    v = vals.v
    assert len(pf) == 16 + 64 * v + 32
    if v == 0:
        assert vals.calls == ["start", "single"]
    else:
        assert vals.calls == ["start"] + [c for t in range(1, v + 1) for c in (("round", t), ("answer", t))] + ["finals"]


def test_extreme_factors(fp):
    for a, b in ((-128, -128), (127, -128)):
        s = np.full(7, a, np.int8)
        u = np.full(7, b, np.int8)
        tx = _site_tx(fp, 3, s, u)
        vals = BruteValues(s, u)
        assert fp.had2_protocol_drive(tx, vals.v, vals) == oracle.had2_prove(3, s, u)[0]


@pytest.mark.parametrize("t,X", [(2, 0), (2, 1), (3, 0)])
def test_inconsistent_round_is_refused(fp, t, X):
    # a wrong h_t(0) or h_t(1) from round 2 on breaks g_t(0) + g_t(1) = claim; the host stops
    s, u = _vecs(8, 5)
    tx = _site_tx(fp, 1, s, u)
    with pytest.raises(fp.FpError):
        fp.had2_protocol_drive(tx, 3, BruteValues(s, u, tamper=(t, X)))


def test_wrong_h2_gives_a_proof_the_oracle_rejects(fp):
    # h_t(2) is not covered by the sum check of that round; the next round's claim (or the
    # final check) catches it, which is the verifier's job
    s, u = _vecs(8, 6)
    tx = _site_tx(fp, 2, s, u)
    with pytest.raises(fp.FpError):  # round 2 no longer sums to the claim taken from round 1
        fp.had2_protocol_drive(tx, 3, BruteValues(s, u, tamper=(1, 2)))
    tx = _site_tx(fp, 2, s, u)
    pf = fp.had2_protocol_drive(tx, 3, BruteValues(s, u, tamper=(3, 2)))
    assert oracle.had2_verify(2, s, u, pf)[0] != "accept"


def test_callback_errors_and_small_buffers(fp):
    s, u = _vecs(4, 7)

    class Broken(BruteValues):
        def round(self, t):
            raise RuntimeError("no values")

    tx = _site_tx(fp, 0, s, u)
    with pytest.raises(fp.FpError):
        fp.had2_protocol_drive(tx, 2, Broken(s, u))
    import ctypes as C
    L = fp.lib()
    ln = C.c_size_t(10)
    buf = C.create_string_buffer(10)
    cb = fp._VALUES_FN(lambda *a: 0)
    assert L.fp_had2_protocol_drive(fp.Transcript(0).h, 2, cb, None, buf, C.byref(ln)) != 0
    assert ln.value == 16 + 64 * 2 + 32
    assert L.fp_had2_protocol_drive(fp.Transcript(0).h, 31, cb, None, buf, C.byref(ln)) != 0


# ---- the matmul sum-check over the extension ------------------------------------------

import workloads  # noqa: E402


class BruteMm2:
    """Device values of the extension-field matmul sum-check by their definitions: every
    MLE a double hypercube sum at an extension point."""

    def __init__(self, site, wit, tamper=None):
        q, r, _ = wit
        self.M, self.K, self.N = site.M, site.K, site.N
        self.vM, self.vN, self.n = bf.log2c(site.M), bf.log2c(site.N), bf.log2c(site.K)
        self.W = bf.weights(site)
        self.X = np.asarray(site.xt, np.int64).T
        self.Y = ((1 << site.k_shift) * np.asarray(q, np.int64) + np.asarray(r, np.int64)).T
        self.rho = []
        self.tamper = tamper

    @staticmethod
    def _bits(x, v):
        return [((x >> (v - 1 - b)) & 1, 0) for b in range(v)]

    def _A(self, pt):
        acc = (0, 0)
        for i in range(self.M):
            ei = bf.x_eq(self.zr, self._bits(i, self.vM))
            for k in range(self.K):
                e = bf.x_mul(ei, bf.x_eq(pt, self._bits(k, self.n)))
                w = int(self.W[i, k]) % P
                acc = bf.x_add(acc, (e[0] * w % P, e[1] * w % P))
        return acc

    def _B(self, pt):
        acc = (0, 0)
        for j in range(self.N):
            ej = bf.x_eq(self.zc, self._bits(j, self.vN))
            for k in range(self.K):
                e = bf.x_mul(ej, bf.x_eq(pt, self._bits(k, self.n)))
                x = int(self.X[k, j]) % P
                acc = bf.x_add(acc, (e[0] * x % P, e[1] * x % P))
        return acc

    def start(self, zr, zc):
        assert len(zr) == self.vM and len(zc) == self.vN
        self.zr, self.zc = zr, zc

    def claim(self):
        c = (0, 0)
        for i in range(self.M):
            for j in range(self.N):
                e = bf.x_mul(bf.x_eq(self.zr, self._bits(i, self.vM)), bf.x_eq(self.zc, self._bits(j, self.vN)))
                y = int(self.Y[i, j]) % P
                c = bf.x_add(c, (e[0] * y % P, e[1] * y % P))
        return c

    def round(self, t):
        rest = self.n - t
        g = []
        for X in range(3):
            acc = (0, 0)
            for b in range(1 << rest):
                pt = self.rho + [(X, 0)] + self._bits(b, rest)
                acc = bf.x_add(acc, bf.x_mul(self._A(pt), self._B(pt)))
            if self.tamper == (t, X):
                acc = ((acc[0] + 1) % P, acc[1])
            g.append(acc)
        return g

    def answer(self, t, rho):
        assert t == len(self.rho) + 1
        self.rho.append(rho)

    def finals(self):
        return [self._A(self.rho), self._B(self.rho)]


def _mm_site(M, K, N, bits, scales, seed):
    s = workloads.random_site(seed, M, K, N, bits, 6)
    if scales:
        s.scales = workloads.group_scales(np.random.default_rng(seed), M, K)
    return s, oracle.witness(s)


def _mm_drive(fp, seed, s, w, vals):
    tx = fp.Transcript(seed)
    tx.absorb("mm2_site", bf.site_digests([s], [w])[0][:160])
    return fp.mm2_protocol_drive(tx, vals.vM, vals.vN, vals.n, vals), tx.state()


@pytest.mark.parametrize("M,K,N,bits,scales", [(1, 1, 1, 8, False), (2, 4, 3, 8, False), (3, 5, 2, 4, True),
                                               (4, 8, 4, 4, False), (5, 3, 6, 8, True)])
def test_mm2_host_half_matches_oracle(fp, M, K, N, bits, scales):
    s, w = _mm_site(M, K, N, bits, scales, 100 + M * 7 + K)
    vals = BruteMm2(s, w)
    pf, st = _mm_drive(fp, 8, s, w, vals)
    want, wst = oracle.mm2_prove(8, s, w)
    assert pf == want
    assert st == wst
    assert len(pf) == 16 + 48 * vals.n + 32


@pytest.mark.parametrize("t,X", [(1, 0), (1, 1), (2, 1)])
def test_mm2_inconsistent_round_is_refused(fp, t, X):
    s, w = _mm_site(2, 4, 2, 8, False, 5)
    with pytest.raises(fp.FpError):
        _mm_drive(fp, 1, s, w, BruteMm2(s, w, tamper=(t, X)))


# ---- the helper-inverse LogUp over the extension ------------------------------------------

class BruteLhi2:
    """Device values of the extension-field helper-inverse LogUp by their definitions."""

    def __init__(self, r, k, tamper=None):
        self.r = [int(x) for x in r]
        self.v = max(1, bf.log2c(len(self.r)))
        L = 1 << self.v
        self.f = [x % P for x in self.r] + [0] * (L - len(self.r))
        self.rho = []
        self.tamper = tamper

    def column(self, alpha):
        import struct as _s
        self.alpha = alpha
        self.h = [bf.x_inv(((alpha[0] - x) % P, alpha[1])) for x in self.f]
        return bf.tree_digest(b"".join(_s.pack("<QQ", a, b) for a, b in self.h))

    def start(self, z, beta):
        self.z, self.beta = z, beta

    def _h(self, w):
        acc = (0, 0)
        for x in range(len(self.h)):
            acc = bf.x_add(acc, bf.x_mul(bf.x_eq(w, [((x >> (self.v - 1 - i)) & 1, 0) for i in range(self.v)]),
                                         self.h[x]))
        return acc

    def round(self, t):
        rest = self.v - t
        H, Q = [], []
        for X in range(3):
            hs = qs = (0, 0)
            for b in range(1 << rest):
                bits = [((b >> (rest - 1 - i)) & 1, 0) for i in range(rest)]
                w = self.rho + [(X, 0)] + bits
                hw, fw = self._h(w), bf.x_mle(self.f, w)
                hs = bf.x_add(hs, hw)
                am = bf.x_add(self.alpha, ((-fw[0]) % P, (-fw[1]) % P))
                qs = bf.x_add(qs, bf.x_mul(bf.x_eq(self.z[t:], bits), bf.x_mul(hw, am)))
            H.append(hs)
            Q.append(qs)
        out = [H[0], H[1], Q[0], Q[1], Q[2]]
        if self.tamper == t:
            out[2] = ((out[2][0] + 1) % P, out[2][1])
        return out

    def answer(self, t, rho):
        assert t == len(self.rho) + 1
        self.rho.append(rho)

    def finals(self):
        return [self._h(self.rho), bf.x_mle(self.f, self.rho)]


def _lhi2_drive(fp, seed, r, k, vals):
    tx = fp.Transcript(seed)
    tx.absorb("lhi2_site", bf.tree_digest(np.asarray(r, "<i4").tobytes()))
    m = np.zeros(1 << k, np.int64)
    for x in list(r) + [0] * ((1 << vals.v) - len(r)):
        j = int(x) + (1 << (k - 1))
        if 0 <= j < (1 << k):
            m[j] += 1
    m = m.astype("<u4")
    return fp.lhi2_protocol_drive(tx, vals.v, k, m, bf.tree_digest(m.tobytes()), vals), tx.state()


@pytest.mark.parametrize("n,k", [(1, 1), (3, 4), (5, 7), (8, 3), (13, 5)])
def test_lhi2_host_half_matches_oracle(fp, n, k):
    r = np.random.default_rng(n + 50 * k).integers(-(1 << (k - 1)), 1 << (k - 1), n).astype(np.int32)
    vals = BruteLhi2(r, k)
    assert _lhi2_drive(fp, 3, r, k, vals) == oracle.lhi2_prove(3, r, k)


@pytest.mark.parametrize("t", [1, 2])
def test_lhi2_inconsistent_round_is_refused(fp, t):
    r = np.random.default_rng(8).integers(-8, 8, 8).astype(np.int32)
    with pytest.raises(fp.FpError):
        _lhi2_drive(fp, 1, r, 4, BruteLhi2(r, 4, tamper=t))


# ---- the 16-bit function lookups (LogUp-GKR tree) over the extension ----------------------

class BruteLookup16x:
    """Device values of the extension-field 16-bit lookup by their definitions: the tree by
    its recurrence, every round value a hypercube sum over MLEs at extension points."""

    def __init__(self, g, s, pad_s, tamper=None):
        self.g = [int(x) for x in g]
        self.s = [int(x) for x in s]
        n = len(self.g)
        self.v = max(1, bf.log2c(n))
        L = 1 << self.v
        self.gp = self.g + [0] * (L - n)
        self.sp = self.s + [pad_s] * (L - n)
        self.tamper = tamper

    def tree(self, gamma, alpha):
        neg = lambda x: ((-x[0]) % P, (-x[1]) % P)  # noqa: E731
        L = 1 << self.v
        Pl = [[(1, 0)] * L]
        Ql = [[bf.x_add(alpha, neg(bf.x_add((a % P, 0), bf.x_mul(gamma, (c % P, 0))))) for a, c in zip(self.gp, self.sp)]]
        for _ in range(self.v):
            p, q_ = Pl[0], Ql[0]
            Pl.insert(0, [bf.x_add(bf.x_mul(p[2 * x], q_[2 * x + 1]), bf.x_mul(p[2 * x + 1], q_[2 * x]))
                          for x in range(len(p) // 2)])
            Ql.insert(0, [bf.x_mul(q_[2 * x], q_[2 * x + 1]) for x in range(len(p) // 2)])
        self.Pl, self.Ql = Pl, Ql
        return [Pl[1][0], Pl[1][1], Ql[1][0], Ql[1][1]]

    def layer(self, d, z, lam):
        self.d, self.z, self.lam, self.rho = d, z, lam, []
        Pc, Qc = self.Pl[d + 1], self.Ql[d + 1]
        n2 = 1 << d
        self.vecs = ([Pc[2 * x] for x in range(n2)], [Pc[2 * x + 1] for x in range(n2)],
                     [Qc[2 * x] for x in range(n2)], [Qc[2 * x + 1] for x in range(n2)])

    def round(self, t):
        rest = self.d - t
        h = []
        for X in range(3):
            acc = (0, 0)
            for b in range(1 << rest):
                bits = [((b >> (rest - 1 - i)) & 1, 0) for i in range(rest)]
                pt = self.rho + [(X, 0)] + bits
                pL, pR, qL, qR = (bf.xv_mle(vv, pt) for vv in self.vecs)
                F = bf.x_add(bf.x_add(bf.x_mul(pL, qR), bf.x_mul(pR, qL)), bf.x_mul(self.lam, bf.x_mul(qL, qR)))
                acc = bf.x_add(acc, bf.x_mul(bf.x_eq(self.z[t:self.d], bits), F))
            h.append(acc)
        if self.tamper == (self.d, t):
            h[0] = ((h[0][0] + 1) % P, h[0][1])
        return h

    def answer(self, t, rho):
        self.rho.append(rho)

    def finals(self):
        return [bf.xv_mle(vv, self.rho) for vv in self.vecs]

    def leaf(self, z):
        return [bf.x_mle(self.gp, z), bf.x_mle(self.sp, z)]


def _lk_drive(fp, seed, g, s, table, vals):
    prefix = "silu2" if table == 0 else "exp2"
    tx = fp.Transcript(seed)
    tx.absorb(prefix + "_site", bf.tree_digest(np.asarray(g, "<i2").tobytes()) + bf.tree_digest(np.asarray(s, "<i2").tobytes()))
    gamma = (tx.squeeze(prefix + "_gamma")[0], tx.squeeze(prefix + "_gamma")[0])
    m = np.zeros(1 << 16, np.int64)
    for x in vals.gp:
        m[x + 32768] += 1
    m = m.astype("<u4")
    return fp.lookup16x_protocol_drive(tx, table, vals.v, gamma, m, bf.tree_digest(m.tobytes()), vals), tx.state()


@pytest.mark.parametrize("n", [1, 2, 3, 5, 8])
def test_lookup16x_host_half_matches_oracle(fp, n):
    rng = np.random.default_rng(n + 90)
    g = rng.integers(-32768, 32768, n).astype(np.int16)
    s = np.array([oracle.silu_q(int(x)) for x in g], np.int16)
    vals = BruteLookup16x(g, s, oracle.silu_q(0))
    assert _lk_drive(fp, 4, g, s, 0, vals) == oracle.silu2_prove(4, g, s)


def test_lookup16x_exp_table_and_bad_round_rejected(fp):
    g = np.array([-5, 0, -300, -1800, 7], np.int16)
    s = np.array([oracle.exp_q(int(x)) for x in g], np.int16)
    honest = _lk_drive(fp, 6, g, s, 1, BruteLookup16x(g, s, oracle.exp_q(0)))
    assert honest == oracle.exp2_prove(6, g, s)
    assert oracle.exp2_verify(6, g, s, honest[0])[0] == "accept"
    # a layer round's h(1) is the running claim minus h(0), so a wrong device value at X = 0
    # yields a proof (no refusal) that the verifier rejects
    bad = _lk_drive(fp, 6, g, s, 1, BruteLookup16x(g, s, oracle.exp_q(0), tamper=(2, 2)))
    assert bad[0] != honest[0]
    assert oracle.exp2_verify(6, g, s, bad[0])[0] != "accept"


# ---- the two-table rescale LogUp over the extension --------------------------------------

class BruteLu2:
    """Device values of the extension-field rescale LogUp by their definitions."""

    def __init__(self, wits, tamper=None):
        self.r = [int(x) for w in wits for x in np.asarray(w[1]).reshape(-1)]
        self.q = [int(x) for w in wits for x in np.asarray(w[0]).reshape(-1)]
        self.y = [int(x) for w in wits for x in np.asarray(w[2]).reshape(-1)]
        nk = len(self.r)
        self.v = max(1, bf.log2c(nk))
        L = 1 << self.v
        self.rp, self.qp, self.yp = (c + [0] * (L - nk) for c in (self.r, self.q, self.y))
        self.tamper = tamper

    def tree(self, gamma, alpha0, alpha1):
        neg = lambda x: ((-x[0]) % P, (-x[1]) % P)  # noqa: E731
        keys = [[(a % P, 0) for a in self.rp],
                [bf.x_add((a % P, 0), bf.x_mul(gamma, (c % P, 0))) for a, c in zip(self.qp, self.yp)]]
        self.trees = []
        for tau, alpha in enumerate((alpha0, alpha1)):
            Pl = [[(1, 0)] * len(keys[tau])]
            Ql = [[bf.x_add(alpha, neg(f)) for f in keys[tau]]]
            for _ in range(self.v):
                p_, q_ = Pl[0], Ql[0]
                Pl.insert(0, [bf.x_add(bf.x_mul(p_[2 * x], q_[2 * x + 1]), bf.x_mul(p_[2 * x + 1], q_[2 * x]))
                              for x in range(len(p_) // 2)])
                Ql.insert(0, [bf.x_mul(q_[2 * x], q_[2 * x + 1]) for x in range(len(p_) // 2)])
            self.trees.append((Pl, Ql))
        return [v_ for Pl, Ql in self.trees for v_ in (Pl[1][0], Pl[1][1], Ql[1][0], Ql[1][1])]

    def layer(self, d, z, lam):
        self.d, self.z, self.lam, self.rho = d, z, lam, []
        self.lam2 = bf.x_mul(lam, lam)
        self.vecs = []
        for Pl, Ql in self.trees:
            Pc, Qc = Pl[d + 1], Ql[d + 1]
            self.vecs += [[Pc[2 * x] for x in range(1 << d)], [Pc[2 * x + 1] for x in range(1 << d)],
                          [Qc[2 * x] for x in range(1 << d)], [Qc[2 * x + 1] for x in range(1 << d)]]

    def round(self, t):
        rest = self.d - t
        h = []
        for X in range(3):
            acc = (0, 0)
            for b in range(1 << rest):
                bits = [((b >> (rest - 1 - i)) & 1, 0) for i in range(rest)]
                pt = self.rho + [(X, 0)] + bits
                ev = [bf.xv_mle(vv, pt) for vv in self.vecs]
                F = (0, 0)
                for tau, w in ((0, (1, 0)), (1, self.lam2)):
                    pL, pR, qL, qR = ev[4 * tau:4 * tau + 4]
                    f = bf.x_add(bf.x_add(bf.x_mul(pL, qR), bf.x_mul(pR, qL)), bf.x_mul(self.lam, bf.x_mul(qL, qR)))
                    F = bf.x_add(F, bf.x_mul(w, f))
                acc = bf.x_add(acc, bf.x_mul(bf.x_eq(self.z[t:self.d], bits), F))
            h.append(acc)
        if self.tamper == (self.d, t):
            h[0] = ((h[0][0] + 1) % P, h[0][1])
        return h

    def answer(self, t, rho):
        self.rho.append(rho)

    def finals(self):
        return [bf.xv_mle(vv, self.rho) for vv in self.vecs]

    def leaf(self, z):
        return [bf.x_mle(self.rp, z), bf.x_mle(self.qp, z), bf.x_mle(self.yp, z)]


def _lu2_drive(fp, seed, sites, wits, vals):
    k = sites[0].k_shift
    tx = fp.Transcript(seed)
    r = np.concatenate([np.asarray(w[1], np.int64).reshape(-1) for w in wits])
    q = np.concatenate([np.asarray(w[0], np.int64).reshape(-1) for w in wits])
    y = np.concatenate([np.asarray(w[2], np.int64).reshape(-1) for w in wits])
    tx.absorb("lu2_site", bf.tree_digest(r.astype("<i4").tobytes()) + bf.tree_digest(q.astype("<i4").tobytes())
              + bf.tree_digest(y.astype(np.int8).tobytes()))
    mr = np.zeros(1 << k, np.int64)
    mc = np.zeros(65536, np.int64)
    for a in vals.rp:
        if 0 <= a + (1 << (k - 1)) < (1 << k):
            mr[a + (1 << (k - 1))] += 1
    for a in vals.qp:
        if 0 <= a + 32768 < 65536:
            mc[a + 32768] += 1
    mr, mc = mr.astype("<u4"), mc.astype("<u4")
    pf = fp.lu2_protocol_drive(tx, vals.v, k, mr, bf.tree_digest(mr.tobytes()), mc, bf.tree_digest(mc.tobytes()), vals)
    return pf, tx.state()


@pytest.mark.parametrize("shapes", [[(1, 4, 1)], [(2, 8, 1), (1, 8, 1)], [(3, 5, 2)], [(2, 16, 4)]])
def test_lu2_host_half_matches_oracle(fp, shapes):
    sites = [workloads.random_site(30 + i, M, K, N, 8, 6) for i, (M, K, N) in enumerate(shapes)]
    wits = [oracle.witness(s) for s in sites]
    assert _lu2_drive(fp, 3, sites, wits, BruteLu2(wits)) == oracle.lu2_prove(3, sites, wits)


def test_lu2_bad_round_is_rejected(fp):
    sites = [workloads.random_site(31, 2, 16, 4, 8, 6)]
    wits = [oracle.witness(s) for s in sites]
    honest = _lu2_drive(fp, 3, sites, wits, BruteLu2(wits))
    bad = _lu2_drive(fp, 3, sites, wits, BruteLu2(wits, tamper=(2, 1)))
    assert bad[0] != honest[0]
    assert oracle.lu2_verify(3, sites, wits, honest[0])[0] == "accept"
    assert oracle.lu2_verify(3, sites, wits, bad[0])[0] != "accept"
