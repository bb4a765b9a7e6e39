"""Brute-force restatement of the proof, for tiny statements only.

Independent of ``oracle/`` (and of the CUDA library): Python integers for the
field, ``hashlib`` for SHA-256, numpy only for integer matrix products. Every
prover message is computed straight from its definition -- each multilinear
extension is evaluated by summing eq(point, x) f(x) over the whole hypercube,
and each round polynomial by summing the summand over the unbound variables --
instead of by folding vectors as the oracle does. The two must produce the same
bytes; a dropped term, a wrong index, sign or bit order in either shows up.

Cost is exponential on purpose: keep M, K, N and the key count in the tens.
"""

from __future__ import annotations

import hashlib
import struct

import numpy as np

P = 0xFFFFFFFF00000001


def sha(b: bytes) -> bytes:
    return hashlib.sha256(b).digest()


def tree_digest(data: bytes) -> bytes:
    n = len(data)
    lv = [sha(data[i:i + 1024]) for i in range(0, n, 1024)] or [sha(b"")]
    while len(lv) > 1:
        lv = [sha(b"".join(lv[i:i + 32])) for i in range(0, len(lv), 32)]
    return sha(struct.pack("<Q", n) + lv[0])


class Tx:
    def __init__(self, seed: int):
        self.st = sha(b"FPSC-v1" + struct.pack("<Q", seed))

    def absorb(self, label: str, data: bytes):
        lb = label.encode()
        self.st = sha(self.st + struct.pack("<I", len(lb)) + lb + struct.pack("<Q", len(data)) + data)

    def squeeze(self, label: str) -> int:
        lb = label.encode()
        ctr = 0
        while True:
            h = sha(self.st + b"sq" + struct.pack("<I", len(lb)) + lb + struct.pack("<I", ctr))
            v = int.from_bytes(h[:8], "little")
            if v < P:
                self.st = h
                return v
            ctr += 1


def log2c(n: int) -> int:
    v = 0
    while (1 << v) < n:
        v += 1
    return v


def eq_point(z, x: int) -> int:
    """eq(z, x) with z_1 on the most significant bit of x (closed-form product)."""
    v = len(z)
    acc = 1
    for b in range(v):
        bit = (x >> (v - 1 - b)) & 1
        acc = acc * (z[b] if bit else (1 - z[b])) % P
    return acc


def mle(vals, z) -> int:
    """sum over the whole hypercube of eq(z, x) vals[x] (vals zero-padded)."""
    v = len(z)
    return sum(eq_point(z, x) * (int(vals[x]) % P) for x in range(min(len(vals), 1 << v))) % P


def mle2(mat, zrow, zcol) -> int:
    """MLE of a 2-D array (row bits first) by the double hypercube sum."""
    R, Cc = mat.shape
    acc = 0
    for i in range(min(R, 1 << len(zrow))):
        ei = eq_point(zrow, i)
        for j in range(min(Cc, 1 << len(zcol))):
            acc += ei * eq_point(zcol, j) * (int(mat[i, j]) % P)
    return acc % P


def weights(site) -> np.ndarray:
    """W_eff as an int64 M x K array."""
    if site.w_bits == 8:
        w = site.w.astype(np.int64)
    else:
        b = site.w.astype(np.int64)
        lo, hi = b & 15, b >> 4
        full = np.empty((site.M, 2 * b.shape[1]), np.int64)
        full[:, 0::2], full[:, 1::2] = lo, hi
        w = np.where(full >= 8, full - 16, full)[:, :site.K]
    if site.scales is not None:
        cols = np.arange(site.K) // 64
        w = w * site.scales.astype(np.int64)[:, cols]
    return w


def fe_bytes(vals) -> bytes:
    return b"".join(struct.pack("<Q", int(v) % P) for v in vals)


def prove(seed: int, sites, wits) -> bytes:
    """The whole proof (matmul section then lookup section), by definition."""
    tx = Tx(seed)
    out = bytearray()

    def send(label, vals):
        b = fe_bytes(vals)
        out.extend(b)
        tx.absorb(label, b)

    commit_and_matmul(tx, send, sites, wits)
    lookup_gkr(tx, send, out, sites, wits)
    return bytes(out)


def commit_and_matmul(tx, send, sites, wits):
    """The site records, then the matmul section, by definition."""
    for s, (q, r, y) in zip(sites, wits):
        sc = b"" if s.scales is None else s.scales.tobytes()
        d = tree_digest(s.w.tobytes()) + tree_digest(sc) + tree_digest(s.xt.tobytes()) + \
            tree_digest(q.astype("<i4").tobytes()) + tree_digest(r.astype("<i4").tobytes()) + \
            tree_digest(y.astype(np.int8).tobytes())
        tx.absorb("site", d)

    # ---- matmul sum-check ----
    vM = max(log2c(s.M) for s in sites)
    vN = max(log2c(s.N) for s in sites)
    n = max(log2c(s.K) for s in sites)
    rr = [tx.squeeze("r_row") for _ in range(vM)]
    rc = [tx.squeeze("r_col") for _ in range(vN)]
    Ws = [weights(s) for s in sites]
    Xs = [s.xt.astype(np.int64).T for s in sites]          # K x N
    claims = []
    for s, (q, r, y) in zip(sites, wits):
        Yq = (q.astype(np.int64) << s.k_shift) + r.astype(np.int64)   # N x M
        claims.append(mle2(Yq.T, rr[:log2c(s.M)], rc[:log2c(s.N)]))
    send("claims", claims)
    rho = [1] if len(sites) == 1 else [tx.squeeze("rho") for _ in sites]

    def A_at(si, pt):   # W~_s(r_row, pt)
        return mle2(Ws[si], rr[:log2c(sites[si].M)], pt)

    def B_at(si, pt):   # X~_s(pt, r_col)
        return mle2(Xs[si], pt, rc[:log2c(sites[si].N)])

    chal = []
    for t in range(n):
        g = []
        for X in range(3):
            acc = 0
            rest = n - t - 1
            for b in range(1 << rest):
                tail = [(b >> (rest - 1 - i)) & 1 for i in range(rest)]
                pt = chal + [X] + tail
                for si in range(len(sites)):
                    acc += rho[si] * A_at(si, pt) * B_at(si, pt)
            g.append(acc % P)
        send("sc_round", g)
        chal.append(tx.squeeze("sc_chal"))
    fin = []
    for si in range(len(sites)):
        fin += [A_at(si, chal), B_at(si, chal)]
    send("sc_final", fin)


def lookup_keys(sites, wits):
    """The padded key columns r, q, y (int64) of the sites' outputs in storage order."""
    fr = np.concatenate([w[1].reshape(-1) for w in wits]).astype(np.int64)
    fq = np.concatenate([w[0].reshape(-1) for w in wits]).astype(np.int64)
    fy = np.concatenate([w[2].reshape(-1) for w in wits]).astype(np.int64)
    v = max(1, log2c(len(fr)))
    pad = (1 << v) - len(fr)
    return [np.concatenate([a, np.zeros(pad, np.int64)]) for a in (fr, fq, fy)] + [v]


def lookup_gkr(tx, send, out, sites, wits):
    """The lookup section as the fraction tree with one sum-check per layer, by definition."""
    k = sites[0].k_shift
    fr = np.concatenate([w[1].reshape(-1) for w in wits]).astype(np.int64)
    fq = np.concatenate([w[0].reshape(-1) for w in wits]).astype(np.int64)
    fy = np.concatenate([w[2].reshape(-1) for w in wits]).astype(np.int64)
    v = max(1, log2c(len(fr)))
    L = 1 << v
    pad = L - len(fr)
    fr, fq, fy = (np.concatenate([a, np.zeros(pad, np.int64)]) for a in (fr, fq, fy))

    m_rem = np.zeros(1 << k, np.int64)
    for x in fr:
        j = x + (1 << (k - 1))
        if 0 <= j < (1 << k):
            m_rem[j] += 1
    b = m_rem.astype("<u4").tobytes()
    out.extend(b)
    tx.absorb("logup_m_rem", tree_digest(b))
    gamma = tx.squeeze("logup_gamma")
    m_cl = np.zeros(1 << 16, np.int64)
    for x in fq:
        j = x + 32768
        if 0 <= j < 65536:
            m_cl[j] += 1
    b = m_cl.astype("<u4").tobytes()
    out.extend(b)
    tx.absorb("logup_m_clamp", tree_digest(b))
    alpha = [tx.squeeze("logup_alpha"), tx.squeeze("logup_alpha")]

    keys = [[int(x) % P for x in fr], [(int(a) + gamma * int(c)) % P for a, c in zip(fq, fy)]]
    layers = []  # per table: list over depth d of (P list, Q list)
    for tau in range(2):
        Pl = [[1] * L]
        Ql = [[(alpha[tau] - f) % P for f in keys[tau]]]
        for _ in range(v):
            p, q_ = Pl[0], Ql[0]
            Pl.insert(0, [(p[2 * x] * q_[2 * x + 1] + p[2 * x + 1] * q_[2 * x]) % P for x in range(len(p) // 2)])
            Ql.insert(0, [q_[2 * x] * q_[2 * x + 1] % P for x in range(len(p) // 2)])
        layers.append((Pl, Ql))

    l1 = []
    for tau in range(2):
        Pl, Ql = layers[tau]
        l1 += [Pl[1][0], Pl[1][1], Ql[1][0], Ql[1][1]]
    send("gkr_l1", l1)
    z = [tx.squeeze("gkr_mu")]

    def kids(tau, d):
        Pl, Ql = layers[tau]
        Pc, Qc = Pl[d + 1], Ql[d + 1]
        return ([Pc[2 * x] for x in range(1 << d)], [Pc[2 * x + 1] for x in range(1 << d)],
                [Qc[2 * x] for x in range(1 << d)], [Qc[2 * x + 1] for x in range(1 << d)])

    for d in range(1, v):
        lam = tx.squeeze("gkr_lambda")
        vecs = kids(0, d) + kids(1, d)
        rho_l = []
        for t in range(d):
            g = []
            for X in range(4):
                acc = 0
                rest = d - t - 1
                for bb in range(1 << rest):
                    tail = [(bb >> (rest - 1 - i)) & 1 for i in range(rest)]
                    pt = rho_l + [X] + tail
                    e = 1
                    for zi, pi in zip(z, pt):
                        e = e * (zi * pi + (1 - zi) * (1 - pi)) % P
                    ev = [mle(vv, pt) for vv in vecs]
                    F = 0
                    for tau in range(2):
                        pL, pR, qL, qR = ev[4 * tau:4 * tau + 4]
                        F += pow(lam, 2 * tau, P) * (pL * qR + pR * qL + lam * qL * qR)
                    acc += e * F
                g.append(acc % P)
            send("gkr_round", g)
            rho_l.append(tx.squeeze("gkr_chal"))
        send("gkr_final", [mle(vv, rho_l) for vv in vecs])
        z = rho_l + [tx.squeeze("gkr_mu")]

    send("leaf", [mle(fr, z), mle(fq, z), mle(fy, z)])


def prove_hi(seed: int, sites, wits) -> bytes:
    """The layer proof with the helper-inverse lookup section, by definition: the helper
    columns by Python modular inverses, every round value a hypercube sum of the summand
    over MLEs evaluated at field points (no folding)."""
    tx = Tx(seed)
    out = bytearray()

    def send(label, vals):
        b = fe_bytes(vals)
        out.extend(b)
        tx.absorb(label, b)

    commit_and_matmul(tx, send, sites, wits)
    k = sites[0].k_shift
    fr, fq, fy, v = lookup_keys(sites, wits)
    m_rem = np.zeros(1 << k, np.int64)
    for x in fr:
        if 0 <= x + (1 << (k - 1)) < (1 << k):
            m_rem[x + (1 << (k - 1))] += 1
    b = m_rem.astype("<u4").tobytes()
    out.extend(b)
    tx.absorb("lhr_m_rem", tree_digest(b))
    gamma = tx.squeeze("lhr_gamma")
    m_cl = np.zeros(1 << 16, np.int64)
    for x in fq:
        if 0 <= x + 32768 < 65536:
            m_cl[x + 32768] += 1
    b = m_cl.astype("<u4").tobytes()
    out.extend(b)
    tx.absorb("lhr_m_clamp", tree_digest(b))
    a0, a1 = tx.squeeze("lhr_alpha"), tx.squeeze("lhr_alpha")
    R = [int(x) % P for x in fr]
    Q = [int(x) % P for x in fq]
    Y = [int(x) % P for x in fy]
    h0 = [pow((a0 - x) % P, P - 2, P) for x in R]
    h1 = [pow((a1 - q - gamma * y) % P, P - 2, P) for q, y in zip(Q, Y)]
    pack = lambda col: b"".join(struct.pack("<Q", x) for x in col)  # noqa: E731
    tx.absorb("lhr_h", tree_digest(pack(h0)) + tree_digest(pack(h1)))
    z = [tx.squeeze("lhr_z") for _ in range(v)]
    beta = tx.squeeze("lhr_beta")
    send("lhr_sum", [sum(h0) % P, sum(h1) % P])
    rho = []
    for t in range(v):
        rest = v - t - 1
        g = []
        for X in range(4):
            acc = 0
            for bb in range(1 << rest):
                w = rho + [X] + [(bb >> (rest - 1 - i)) & 1 for i in range(rest)]
                H0, H1, r_, q_, y_ = (mle_at(c, w) for c in (h0, h1, R, Q, Y))
                zero = beta ** 2 * (H0 * (a0 - r_) - 1) + beta ** 3 * (H1 * (a1 - q_ - gamma * y_) - 1)
                acc += H0 + beta * H1 + eq_ml(z, w) * zero
            g.append(acc % P)
        send("lhr_round", g)
        rho.append(tx.squeeze("lhr_chal"))
    send("lhr_final", [mle_at(c, rho) for c in (h0, h1, R, Q, Y)])
    return bytes(out)


def site_digests(sites, wits) -> list:
    out = []
    for s, (q, r, y) in zip(sites, wits):
        sc = b"" if s.scales is None else s.scales.tobytes()
        out.append(tree_digest(s.w.tobytes()) + tree_digest(sc) + tree_digest(s.xt.tobytes()) +
                   tree_digest(q.astype("<i4").tobytes()) + tree_digest(r.astype("<i4").tobytes()) +
                   tree_digest(y.astype(np.int8).tobytes()))
    return out


class _Reader:
    def __init__(self, proof: bytes, tx: Tx):
        self.b, self.pos, self.tx = proof, 0, tx

    def fe(self, label: str, n: int):
        raw = self.b[self.pos:self.pos + 8 * n]
        assert len(raw) == 8 * n, "proof truncated"
        self.pos += 8 * n
        self.tx.absorb(label, raw)
        return [int.from_bytes(raw[8 * i:8 * i + 8], "little") for i in range(n)]

    def mult(self, label: str, n: int):
        raw = self.b[self.pos:self.pos + 4 * n]
        assert len(raw) == 4 * n, "proof truncated"
        self.pos += 4 * n
        self.tx.absorb(label, tree_digest(raw))
        return np.frombuffer(raw, dtype="<u4").astype(np.int64)


def walk(seed: int, sites, wits, proof: bytes) -> dict:
    """Replay the transcript over a proof's bytes (no message is recomputed):
    returns every challenge and message, and the final transcript state."""
    tx = Tx(seed)
    for d in site_digests(sites, wits):
        tx.absorb("site", d)
    rd = _Reader(proof, tx)
    out = {}
    vM = max(log2c(s.M) for s in sites)
    vN = max(log2c(s.N) for s in sites)
    n = max(log2c(s.K) for s in sites)
    out["r_row"] = [tx.squeeze("r_row") for _ in range(vM)]
    out["r_col"] = [tx.squeeze("r_col") for _ in range(vN)]
    out["claims"] = rd.fe("claims", len(sites))
    out["rho"] = [1] if len(sites) == 1 else [tx.squeeze("rho") for _ in sites]
    out["mm_rounds"], out["mm_chal"] = [], []
    for _ in range(n):
        out["mm_rounds"].append(rd.fe("sc_round", 3))
        out["mm_chal"].append(tx.squeeze("sc_chal"))
    out["mm_final"] = rd.fe("sc_final", 2 * len(sites))
    out["state_mm"] = tx.st
    k = sites[0].k_shift
    nk = sum(s.M * s.N for s in sites)
    v = max(1, log2c(nk))
    out["v"] = v
    out["m_rem"] = rd.mult("logup_m_rem", 1 << k)
    out["gamma"] = tx.squeeze("logup_gamma")
    out["m_clamp"] = rd.mult("logup_m_clamp", 1 << 16)
    out["alpha"] = [tx.squeeze("logup_alpha"), tx.squeeze("logup_alpha")]
    out["l1"] = rd.fe("gkr_l1", 8)
    z = [tx.squeeze("gkr_mu")]
    out["layers"] = []
    for d in range(1, v):
        lam = tx.squeeze("gkr_lambda")
        rounds, chal = [], []
        for _ in range(d):
            rounds.append(rd.fe("gkr_round", 4))
            chal.append(tx.squeeze("gkr_chal"))
        fin = rd.fe("gkr_final", 8)
        mu = tx.squeeze("gkr_mu")
        out["layers"].append(dict(lam=lam, rounds=rounds, chal=chal, final=fin, z_in=list(z), mu=mu))
        z = chal + [mu]
    out["z_leaf"] = z
    out["leaf"] = rd.fe("leaf", 3)
    out["consumed"] = rd.pos
    out["state"] = tx.st
    return out


# ---- gated product h = s (.) u ---------------------------------------------------

def eq_ml(z, w) -> int:
    """eq(z, w) for field points z, w of equal length: prod (z_i w_i + (1 - z_i)(1 - w_i))."""
    acc = 1
    for a, b in zip(z, w):
        acc = acc * ((a * b + (1 - a) * (1 - b)) % P) % P
    return acc


def mle_at(vals, w) -> int:
    """MLE of vals (zero-padded to 2^len(w)) at a field point w, by the hypercube sum."""
    v = len(w)
    acc = 0
    for x in range(min(len(vals), 1 << v)):
        bits = [(x >> (v - 1 - b)) & 1 for b in range(v)]
        acc += eq_ml(w, bits) * (int(vals[x]) % P)
    return acc % P


def had_prove(seed: int, s, u) -> bytes:
    """The gated-product proof from definitions: every round value is the sum, over the
    unbound Boolean variables b, of eq(z, (rho, X, b)) s~(rho, X, b) u~(rho, X, b), each
    MLE evaluated by its own hypercube sum; no vector is folded."""
    s = [int(x) for x in np.asarray(s).reshape(-1)]
    u = [int(x) for x in np.asarray(u).reshape(-1)]
    n = len(s)
    v = log2c(n)
    tx = Tx(seed)
    tx.absorb("had_site", tree_digest(bytes(np.asarray(s, np.int8).tobytes())) +
              tree_digest(bytes(np.asarray(u, np.int8).tobytes())))
    z = [tx.squeeze("had_z") for _ in range(v)]
    c = sum(eq_point(z, x) * s[x] * u[x] for x in range(n)) % P
    out = fe_bytes([c])
    tx.absorb("had_claim", fe_bytes([c]))
    rho = []
    for t in range(v):
        rest = v - t - 1
        g = []
        for X in range(4):
            acc = 0
            for b in range(1 << rest):
                w = rho + [X] + [(b >> (rest - 1 - i)) & 1 for i in range(rest)]
                acc += eq_ml(z, w) * mle_at(s, w) * mle_at(u, w)
            g.append(acc % P)
        out += fe_bytes(g)
        tx.absorb("had_round", fe_bytes(g))
        rho.append(tx.squeeze("had_chal"))
    fin = [mle_at(s, rho), mle_at(u, rho)]
    out += fe_bytes(fin)
    tx.absorb("had_final", fe_bytes(fin))
    return out


# ---- per-group scale reduction -------------------------------------------------

def _prod3_rounds(tx, z, svals, uvals, lab_round, lab_chal, lab_final) -> bytes:
    """Round values of the product sum-check of eq(z, .) s u from definitions (hypercube sums)."""
    v = len(z)
    out = b""
    rho = []
    for t in range(v):
        rest = v - t - 1
        g = []
        for X in range(4):
            acc = 0
            for b in range(1 << rest):
                w = rho + [X] + [(b >> (rest - 1 - i)) & 1 for i in range(rest)]
                acc += eq_ml(z, w) * mle_at(svals, w) * mle_at(uvals, w)
            g.append(acc % P)
        out += fe_bytes(g)
        tx.absorb(lab_round, fe_bytes(g))
        rho.append(tx.squeeze(lab_chal))
    fin = [mle_at(svals, rho), mle_at(uvals, rho)]
    out += fe_bytes(fin)
    tx.absorb(lab_final, fe_bytes(fin))
    return out, rho


def scale_factors(w, bits: int, scales, M: int, K: int):
    """Se(i, k) = S[i][k // 64] and w(i, k) over the padded (row bits first) grid, as lists."""
    vM, vK = log2c(M), log2c(K)
    G = (K + 63) // 64
    if bits == 8:
        wv = np.asarray(w, np.int64)
    else:
        b = np.asarray(w, np.int64)
        full = np.empty((M, 2 * b.shape[1]), np.int64)
        full[:, 0::2], full[:, 1::2] = b & 15, b >> 4
        wv = np.where(full >= 8, full - 16, full)[:, :K]
    sc = np.asarray(scales, np.int64).reshape(M, G)
    Se, W = [], []
    for i in range(1 << vM):
        for k in range(1 << vK):
            Se.append(int(sc[i, k // 64]) if i < M and k // 64 < G else 0)
            W.append(int(wv[i, k]) if i < M and k < K else 0)
    return Se, W


def scl_prove(seed: int, w, bits: int, scales, M: int, K: int, z) -> bytes:
    """The scale reduction's proof from definitions, at the given point z (row coordinates first)."""
    Se, W = scale_factors(w, bits, scales, M, K)
    tx = Tx(seed)
    wb = np.ascontiguousarray(w).tobytes()
    tx.absorb("scl_site", tree_digest(wb) + tree_digest(np.ascontiguousarray(scales, dtype=np.int8).tobytes()))
    a = sum(eq_ml(z, [(x >> (len(z) - 1 - i)) & 1 for i in range(len(z))]) * Se[x] * W[x]
            for x in range(len(Se))) % P
    tx.absorb("scl_claim", fe_bytes([a]))
    body, _ = _prod3_rounds(tx, list(z), Se, W, "scl_round", "scl_chal", "scl_final")
    return fe_bytes([a]) + body


# ---- SiLU by lookup ----------------------------------------------------------------

def silu_table_entry(v: int) -> int:
    """floor(v / (1 + e^(-v / 256)) + 1/2) in double precision: the table's definition."""
    import math
    return math.floor(v / (1.0 + math.exp(-v / 256.0)) + 0.5)


def silu_prove(seed: int, g, s) -> bytes:
    """The SiLU lookup's proof from definitions (see lookup16_prove)."""
    return lookup16_prove(seed, g, s, "silu", silu_table_entry(0))


def lookup16_prove(seed: int, g, s, prefix: str, pad_s: int) -> bytes:
    """A 16-bit function lookup's proof from definitions: tree layers by their recurrence, every
    layer round value a hypercube sum of eq times the layer summand over MLEs (no folding).
    The table enters only through its row for input 0, which pads the keys."""
    g = [int(x) for x in np.asarray(g).reshape(-1)]
    s = [int(x) for x in np.asarray(s).reshape(-1)]
    n = len(g)
    v = max(1, log2c(n))
    L = 1 << v
    gp = g + [0] * (L - n)
    sp = s + [pad_s] * (L - n)  # padding keys are the table's row for input 0
    out = bytearray()

    def send(label, vals):
        b = fe_bytes(vals)
        out.extend(b)
        tx.absorb(label, b)

    tx = Tx(seed)
    tx.absorb(prefix + "_site", tree_digest(np.asarray(g, "<i2").tobytes()) + tree_digest(np.asarray(s, "<i2").tobytes()))
    gamma = tx.squeeze(prefix + "_gamma")
    m = np.zeros(1 << 16, np.int64)
    for x in gp:
        m[x + 32768] += 1
    b = m.astype("<u4").tobytes()
    out.extend(b)
    tx.absorb(prefix + "_m", tree_digest(b))
    alpha = tx.squeeze(prefix + "_alpha")
    Pl = [[1] * L]
    Ql = [[(alpha - (a + gamma * c)) % P for a, c in zip(gp, sp)]]
    for _ in range(v):
        p, q_ = Pl[0], Ql[0]
        Pl.insert(0, [(p[2 * x] * q_[2 * x + 1] + p[2 * x + 1] * q_[2 * x]) % P for x in range(len(p) // 2)])
        Ql.insert(0, [q_[2 * x] * q_[2 * x + 1] % P for x in range(len(p) // 2)])
    send(prefix + "_l1", [Pl[1][0], Pl[1][1], Ql[1][0], Ql[1][1]])
    z = [tx.squeeze(prefix + "_mu")]
    for d in range(1, v):
        lam = tx.squeeze(prefix + "_lambda")
        Pc, Qc = Pl[d + 1], Ql[d + 1]
        vecs = ([Pc[2 * x] for x in range(1 << d)], [Pc[2 * x + 1] for x in range(1 << d)],
                [Qc[2 * x] for x in range(1 << d)], [Qc[2 * x + 1] for x in range(1 << d)])
        rho_l = []
        for t in range(d):
            gr = []
            for X in range(4):
                acc = 0
                rest = d - t - 1
                for bb in range(1 << rest):
                    pt = rho_l + [X] + [(bb >> (rest - 1 - i)) & 1 for i in range(rest)]
                    pL, pR, qL, qR = (mle(vv, pt) for vv in vecs)
                    acc += eq_ml(z, pt) * (pL * qR + pR * qL + lam * qL * qR)
                gr.append(acc % P)
            send(prefix + "_round", gr)
            rho_l.append(tx.squeeze(prefix + "_chal"))
        send(prefix + "_final", [mle(vv, rho_l) for vv in vecs])
        z = rho_l + [tx.squeeze(prefix + "_mu")]
    send(prefix + "_leaf", [mle(gp, z), mle(sp, z)])
    return bytes(out)


# ---- the helper-inverse LogUp -------------------------------------------------------

def lhi_prove(seed: int, r, k: int) -> bytes:
    """The helper-inverse LogUp proof from definitions: h by Python modular inverses, every
    round value a hypercube sum of h + beta eq (h (alpha - f) - 1) over MLEs (no folding)."""
    return lhi_body(Tx(seed), r, k)


def lhi_body(tx, r, k: int) -> bytes:
    """The helper-inverse LogUp proof continuing the transcript tx."""
    r = [int(x) for x in np.asarray(r).reshape(-1)]
    n = len(r)
    v = max(1, log2c(n))
    L = 1 << v
    f = [x % P for x in r] + [0] * (L - n)
    out = bytearray()

    def send(label, vals):
        b = fe_bytes(vals)
        out.extend(b)
        tx.absorb(label, b)

    tx.absorb("lhi_site", tree_digest(np.asarray(r, "<i4").tobytes()))
    m = np.zeros(1 << k, np.int64)
    for x in r + [0] * (L - n):
        j = x + (1 << (k - 1))
        if 0 <= j < (1 << k):
            m[j] += 1
    b = m.astype("<u4").tobytes()
    out.extend(b)
    tx.absorb("lhi_m", tree_digest(b))
    alpha = tx.squeeze("lhi_alpha")
    h = [pow((alpha - x) % P, P - 2, P) for x in f]
    tx.absorb("lhi_h", tree_digest(b"".join(struct.pack("<Q", x) for x in h)))
    z = [tx.squeeze("lhi_z") for _ in range(v)]
    beta = tx.squeeze("lhi_beta")
    send("lhi_sum", [sum(h) % P])
    rho = []
    for t in range(v):
        rest = v - t - 1
        g = []
        for X in range(4):
            acc = 0
            for bb in range(1 << rest):
                w = rho + [X] + [(bb >> (rest - 1 - i)) & 1 for i in range(rest)]
                hw, fw = mle_at(h, w), mle_at(f, w)
                acc += hw + beta * eq_ml(z, w) * (hw * (alpha - fw) - 1)
            g.append(acc % P)
        send("lhi_round", g)
        rho.append(tx.squeeze("lhi_chal"))
    send("lhi_final", [mle_at(h, rho), mle_at(f, rho)])
    return bytes(out)


# ---- extension-field challenges: F_p[phi] / (phi^2 - 7) -----------------------------

def x_mul(x, y):
    """(a + b phi)(c + d phi) with phi^2 = 7, as polynomials reduced mod phi^2 - 7."""
    a, b = x
    c, d = y
    return ((a * c + 7 * b * d) % P, (a * d + b * c) % P)


def x_add(x, y):
    return ((x[0] + y[0]) % P, (x[1] + y[1]) % P)


def x_eq(z, w):
    acc = (1, 0)
    for zi, wi in zip(z, w):
        one_z, one_w = ((1 - zi[0]) % P, (-zi[1]) % P), ((1 - wi[0]) % P, (-wi[1]) % P)
        acc = x_mul(acc, x_add(x_mul(zi, wi), x_mul(one_z, one_w)))
    return acc


def x_mle(vals, w):
    v = len(w)
    acc = (0, 0)
    for x in range(min(len(vals), 1 << v)):
        bits = [((x >> (v - 1 - b)) & 1, 0) for b in range(v)]
        e = x_eq(w, bits)
        acc = x_add(acc, (e[0] * (int(vals[x]) % P) % P, e[1] * (int(vals[x]) % P) % P))
    return acc


def had2_prove(seed: int, s, u) -> bytes:
    """The extension-field gated-product proof from definitions (hypercube sums, no folding)."""
    s = [int(x) for x in np.asarray(s).reshape(-1)]
    u = [int(x) for x in np.asarray(u).reshape(-1)]
    n = len(s)
    v = log2c(n)
    tx = Tx(seed)
    tx.absorb("had2_site", tree_digest(np.asarray(s, np.int8).tobytes()) + tree_digest(np.asarray(u, np.int8).tobytes()))
    z = []
    for _ in range(v):
        a = tx.squeeze("had2_z")
        z.append((a, tx.squeeze("had2_z")))
    out = bytearray()

    def send(label, xs):
        b = fe_bytes([c for x in xs for c in x])
        out.extend(b)
        tx.absorb(label, b)

    c = (0, 0)
    for x in range(n):
        bits = [((x >> (v - 1 - b)) & 1, 0) for b in range(v)]
        e = x_eq(z, bits)
        pr = s[x] * u[x] % P
        c = x_add(c, (e[0] * pr % P, e[1] * pr % P))
    send("had2_claim", [c])
    rho = []
    for t in range(v):
        rest = v - t - 1
        g = []
        for X in range(4):
            acc = (0, 0)
            for bb in range(1 << rest):
                w = rho + [(X, 0)] + [((bb >> (rest - 1 - i)) & 1, 0) for i in range(rest)]
                acc = x_add(acc, x_mul(x_eq(z, w), x_mul(x_mle(s, w), x_mle(u, w))))
            g.append(acc)
        send("had2_round", g)
        a = tx.squeeze("had2_chal")
        rho.append((a, tx.squeeze("had2_chal")))
    send("had2_final", [x_mle(s, rho), x_mle(u, rho)])
    return bytes(out)


def mm2_prove(seed: int, site, wit) -> bytes:
    """The extension-field matmul sum-check of one site from definitions: every MLE a hypercube
    sum at an extension point, every round value a sum over the unbound variables."""
    q, r, _ = wit
    M, K, N, k = site.M, site.K, site.N, site.k_shift
    vM, vN, n = log2c(M), log2c(N), log2c(K)
    W = weights(site)                      # M x K
    X = np.asarray(site.xt, np.int64).T    # K x N
    Y = ((1 << k) * np.asarray(q, np.int64) + np.asarray(r, np.int64)).T  # M x N
    tx = Tx(seed)
    tx.absorb("mm2_site", site_digests([site], [wit])[0][:160])

    def squeeze_ext(label):
        a = tx.squeeze(label)
        return (a, tx.squeeze(label))

    zr = [squeeze_ext("mm2_row") for _ in range(vM)]
    zc = [squeeze_ext("mm2_col") for _ in range(vN)]
    out = bytearray()

    def send(label, xs):
        b = fe_bytes([c for x in xs for c in x])
        out.extend(b)
        tx.absorb(label, b)

    def bits(x, v):
        return [((x >> (v - 1 - b)) & 1, 0) for b in range(v)]

    def A_at(pt):  # W_eff~(zr, pt) by the double hypercube sum
        acc = (0, 0)
        for i in range(M):
            ei = x_eq(zr, bits(i, vM))
            for kk in range(K):
                e = x_mul(ei, x_eq(pt, bits(kk, n)))
                acc = x_add(acc, (e[0] * (int(W[i, kk]) % P) % P, e[1] * (int(W[i, kk]) % P) % P))
        return acc

    def B_at(pt):
        acc = (0, 0)
        for j in range(N):
            ej = x_eq(zc, bits(j, vN))
            for kk in range(K):
                e = x_mul(ej, x_eq(pt, bits(kk, n)))
                acc = x_add(acc, (e[0] * (int(X[kk, j]) % P) % P, e[1] * (int(X[kk, j]) % P) % P))
        return acc

    c = (0, 0)
    for i in range(M):
        for j in range(N):
            e = x_mul(x_eq(zr, bits(i, vM)), x_eq(zc, bits(j, vN)))
            y = int(Y[i, j]) % P
            c = x_add(c, (e[0] * y % P, e[1] * y % P))
    send("mm2_claim", [c])
    rho = []
    for t in range(n):
        rest = n - t - 1
        g = []
        for Xv in range(3):
            acc = (0, 0)
            for bb in range(1 << rest):
                pt = rho + [(Xv, 0)] + [((bb >> (rest - 1 - i)) & 1, 0) for i in range(rest)]
                acc = x_add(acc, x_mul(A_at(pt), B_at(pt)))
            g.append(acc)
        send("mm2_round", g)
        rho.append(squeeze_ext("mm2_chal"))
    send("mm2_final", [A_at(rho), B_at(rho)])
    return bytes(out)


# ---- MoE routing: the first argmax of every token's router logits ----------------------

def route_witness(l, T: int, E: int):
    """H (one-hot of the first maximum of every row) and D = l[t][e_t] - l[t][e] - [e < e_t]."""
    l = np.asarray(l, np.int64).reshape(T, E)
    H = np.zeros((T, E), np.uint8)
    D = np.zeros((T, E), np.int64)
    for t in range(T):
        best = max(range(E), key=lambda e: (int(l[t, e]), -e))
        H[t, best] = 1
        for e in range(E):
            D[t, e] = int(l[t, best]) - int(l[t, e]) - (1 if e < best else 0)
    return H, D.astype(np.int32)


def route_prove(seed: int, l, H, D, T: int, E: int) -> bytes:
    """The routing proof from definitions: every round value a hypercube sum of F over the
    unbound variables, with H, l, G and the eq factors as MLEs at the point (no folding)."""
    l = np.asarray(l, np.int64).reshape(-1)
    H = np.asarray(H, np.int64).reshape(-1)
    D = np.asarray(D, np.int64).reshape(-1)
    vT, vE = log2c(T), log2c(E)
    n = vT + vE
    tx = Tx(seed)
    tx.absorb("route_site", tree_digest(np.asarray(l, np.int8).tobytes()) + tree_digest(np.asarray(H, np.uint8).tobytes())
              + tree_digest(np.asarray(D, "<i4").tobytes()))
    z = [tx.squeeze("route_z") for _ in range(n)]
    w = [tx.squeeze("route_w") for _ in range(n)]
    lam1 = tx.squeeze("route_lambda")
    lam2 = tx.squeeze("route_lambda")
    out = bytearray()

    def send(label, vals):
        b = fe_bytes(vals)
        out.extend(b)
        tx.absorb(label, b)

    send("route_open", [mle_at(D, z), mle_at(l, z)])
    # G(e) = sum over e' < e of eq(z_e, e'), as a table over the e bits
    ze = z[vT:]
    G = []
    acc = 0
    for e in range(E):
        G.append(acc)
        acc = (acc + eq_ml(ze, [(e >> (vE - 1 - b)) & 1 for b in range(vE)])) % P

    def F(x):  # the summand at a point x of n coordinates
        xt, xe = x[:vT], x[vT:]
        Hx, lx, Gx = mle_at(H, x), mle_at(l, x), mle_at(G, xe)
        return (eq_ml(z[:vT], xt) * Hx * (lx - Gx) + lam1 * eq_ml(w, x) * Hx * (1 - Hx)
                + lam2 * eq_ml(w[:vT], xt) * Hx) % P

    rho = []
    for t in range(n):
        rest = n - t - 1
        g = []
        for X in range(4):
            s = 0
            for bb in range(1 << rest):
                s += F(rho + [X] + [(bb >> (rest - 1 - i)) & 1 for i in range(rest)])
            g.append(s % P)
        send("route_round", g)
        rho.append(tx.squeeze("route_chal"))
    send("route_final", [mle_at(H, rho), mle_at(l, rho)])
    return bytes(out) + lhi_body(tx, (D - 128).astype(np.int32), 8)


def x_inv(x):
    """1 / (a + b phi) = (a - b phi) / (a^2 - 7 b^2), by Python modular inversion."""
    a, b = x
    nrm = (a * a - 7 * b * b) % P
    ni = pow(nrm, P - 2, P)
    return (a * ni % P, (-b) * ni % P)


def lhi2_prove(seed: int, r, k: int) -> bytes:
    """The helper-inverse LogUp over the extension from definitions: h by extension inverses,
    every round value a hypercube sum of h + beta eq (h (alpha - f) - 1) over MLEs at
    extension points (no folding)."""
    r = [int(x) for x in np.asarray(r).reshape(-1)]
    n = len(r)
    v = max(1, log2c(n))
    L = 1 << v
    f = [x % P for x in r] + [0] * (L - n)
    out = bytearray()
    tx = Tx(seed)

    def send(label, xs):
        b = fe_bytes([c for x in xs for c in x])
        out.extend(b)
        tx.absorb(label, b)

    def sq(label):
        a = tx.squeeze(label)
        return (a, tx.squeeze(label))

    tx.absorb("lhi2_site", tree_digest(np.asarray(r, "<i4").tobytes()))
    m = np.zeros(1 << k, np.int64)
    for x in r + [0] * (L - n):
        j = x + (1 << (k - 1))
        if 0 <= j < (1 << k):
            m[j] += 1
    b = m.astype("<u4").tobytes()
    out.extend(b)
    tx.absorb("lhi2_m", tree_digest(b))
    alpha = sq("lhi2_alpha")
    h = [x_inv(((alpha[0] - x) % P, alpha[1])) for x in f]
    tx.absorb("lhi2_h", tree_digest(b"".join(struct.pack("<QQ", a, c) for a, c in h)))
    z = [sq("lhi2_z") for _ in range(v)]
    beta = sq("lhi2_beta")
    S = (0, 0)
    for x in h:
        S = x_add(S, x)
    send("lhi2_sum", [S])
    one = (1, 0)
    rho = []
    for t in range(v):
        rest = v - t - 1
        g = []
        for X in range(4):
            acc = (0, 0)
            for bb in range(1 << rest):
                w = rho + [(X, 0)] + [((bb >> (rest - 1 - i)) & 1, 0) for i in range(rest)]
                hw = (0, 0)
                for x in range(L):
                    e = x_eq(w, [((x >> (v - 1 - i)) & 1, 0) for i in range(v)])
                    hw = x_add(hw, x_mul(e, h[x]))
                fw = x_mle(f, w)
                inner = x_add(x_mul(hw, x_add(alpha, ((-fw[0]) % P, (-fw[1]) % P))), ((-1) % P, 0))
                acc = x_add(acc, x_add(hw, x_mul(beta, x_mul(x_eq(z, w), inner))))
            g.append(acc)
        send("lhi2_round", g)
        rho.append(sq("lhi2_chal"))
    hr = (0, 0)
    for x in range(L):
        hr = x_add(hr, x_mul(x_eq(rho, [((x >> (v - 1 - i)) & 1, 0) for i in range(v)]), h[x]))
    send("lhi2_final", [hr, x_mle(f, rho)])
    return bytes(out)


def xv_mle(vals, w):
    """MLE of extension-valued vals (zero-padded to 2^len(w)) at an extension point w."""
    v = len(w)
    acc = (0, 0)
    for x in range(min(len(vals), 1 << v)):
        acc = x_add(acc, x_mul(x_eq(w, [((x >> (v - 1 - b)) & 1, 0) for b in range(v)]), vals[x]))
    return acc


def lookup16x_prove(seed: int, g, s, prefix: str, pad_s: int) -> bytes:
    """The 16-bit function lookup over the extension from definitions: the fraction tree by its
    recurrence in the extension, every layer round value a hypercube sum of eq times the layer
    summand over MLEs at extension points (no folding)."""
    g = [int(x) for x in np.asarray(g).reshape(-1)]
    s = [int(x) for x in np.asarray(s).reshape(-1)]
    n = len(g)
    v = max(1, log2c(n))
    L = 1 << v
    gp = g + [0] * (L - n)
    sp = s + [pad_s] * (L - n)
    out = bytearray()
    tx = Tx(seed)

    def send(label, xs):
        b = fe_bytes([c for x in xs for c in x])
        out.extend(b)
        tx.absorb(label, b)

    def sq(label):
        a = tx.squeeze(label)
        return (a, tx.squeeze(label))

    def neg(x):
        return ((-x[0]) % P, (-x[1]) % P)

    tx.absorb(prefix + "_site", tree_digest(np.asarray(g, "<i2").tobytes()) + tree_digest(np.asarray(s, "<i2").tobytes()))
    gamma = sq(prefix + "_gamma")
    m = np.zeros(1 << 16, np.int64)
    for x in gp:
        m[x + 32768] += 1
    b = m.astype("<u4").tobytes()
    out.extend(b)
    tx.absorb(prefix + "_m", tree_digest(b))
    alpha = sq(prefix + "_alpha")
    Pl = [[(1, 0)] * L]
    Ql = [[x_add(alpha, neg(x_add((a % P, 0), x_mul(gamma, (c % P, 0))))) for a, c in zip(gp, sp)]]
    for _ in range(v):
        p, q_ = Pl[0], Ql[0]
        Pl.insert(0, [x_add(x_mul(p[2 * x], q_[2 * x + 1]), x_mul(p[2 * x + 1], q_[2 * x])) for x in range(len(p) // 2)])
        Ql.insert(0, [x_mul(q_[2 * x], q_[2 * x + 1]) for x in range(len(p) // 2)])
    send(prefix + "_l1", [Pl[1][0], Pl[1][1], Ql[1][0], Ql[1][1]])
    z = [sq(prefix + "_mu")]
    for d in range(1, v):
        lam = sq(prefix + "_lambda")
        Pc, Qc = Pl[d + 1], Ql[d + 1]
        vecs = ([Pc[2 * x] for x in range(1 << d)], [Pc[2 * x + 1] for x in range(1 << d)],
                [Qc[2 * x] for x in range(1 << d)], [Qc[2 * x + 1] for x in range(1 << d)])
        rho_l = []
        for t in range(d):
            gr = []
            for X in range(4):
                acc = (0, 0)
                rest = d - t - 1
                for bb in range(1 << rest):
                    pt = rho_l + [(X, 0)] + [((bb >> (rest - 1 - i)) & 1, 0) for i in range(rest)]
                    pL, pR, qL, qR = (xv_mle(vv, pt) for vv in vecs)
                    Fv = x_add(x_add(x_mul(pL, qR), x_mul(pR, qL)), x_mul(lam, x_mul(qL, qR)))
                    acc = x_add(acc, x_mul(x_eq(z, pt), Fv))
                gr.append(acc)
            send(prefix + "_round", gr)
            rho_l.append(sq(prefix + "_chal"))
        send(prefix + "_final", [xv_mle(vv, rho_l) for vv in vecs])
        z = rho_l + [sq(prefix + "_mu")]
    send(prefix + "_leaf", [x_mle(gp, z), x_mle(sp, z)])
    return bytes(out)


def lu2_prove(seed: int, sites, wits) -> bytes:
    """The two-table rescale LogUp over the extension from definitions: both fraction trees by
    their recurrence, every layer round value a hypercube sum of eq times the batched summand
    over MLEs at extension points (no folding)."""
    r = np.concatenate([np.asarray(w[1], np.int64).reshape(-1) for w in wits])
    q = np.concatenate([np.asarray(w[0], np.int64).reshape(-1) for w in wits])
    y = np.concatenate([np.asarray(w[2], np.int64).reshape(-1) for w in wits])
    nk = len(r)
    v = max(1, log2c(nk))
    L = 1 << v
    k = sites[0].k_shift
    rp = [int(x) for x in r] + [0] * (L - nk)
    qp = [int(x) for x in q] + [0] * (L - nk)
    yp = [int(x) for x in y] + [0] * (L - nk)
    out = bytearray()
    tx = Tx(seed)

    def send(label, xs):
        b = fe_bytes([c for x in xs for c in x])
        out.extend(b)
        tx.absorb(label, b)

    def sq(label):
        a = tx.squeeze(label)
        return (a, tx.squeeze(label))

    def mult(vals, off, T, label):
        m = np.zeros(T, np.int64)
        for x in vals:
            if 0 <= x + off < T:
                m[x + off] += 1
        b = m.astype("<u4").tobytes()
        out.extend(b)
        tx.absorb(label, tree_digest(b))

    tx.absorb("lu2_site", tree_digest(r.astype("<i4").tobytes()) + tree_digest(q.astype("<i4").tobytes())
              + tree_digest(y.astype(np.int8).tobytes()))
    mult(rp, 1 << (k - 1), 1 << k, "lu2_m_rem")
    gamma = sq("lu2_gamma")
    mult(qp, 32768, 65536, "lu2_m_clamp")
    alpha = [sq("lu2_alpha"), sq("lu2_alpha")]
    neg = lambda x: ((-x[0]) % P, (-x[1]) % P)  # noqa: E731
    keys = [[(a % P, 0) for a in rp], [x_add((a % P, 0), x_mul(gamma, (c % P, 0))) for a, c in zip(qp, yp)]]
    trees = []
    for tau in range(2):
        Pl = [[(1, 0)] * L]
        Ql = [[x_add(alpha[tau], neg(f)) for f in keys[tau]]]
        for _ in range(v):
            p_, q_ = Pl[0], Ql[0]
            Pl.insert(0, [x_add(x_mul(p_[2 * x], q_[2 * x + 1]), x_mul(p_[2 * x + 1], q_[2 * x])) for x in range(len(p_) // 2)])
            Ql.insert(0, [x_mul(q_[2 * x], q_[2 * x + 1]) for x in range(len(p_) // 2)])
        trees.append((Pl, Ql))
    send("lu2_l1", [t_[0][1][0] if j == 0 else t_[0][1][1] if j == 1 else t_[1][1][0] if j == 2 else t_[1][1][1]
                    for t_ in trees for j in range(4)])
    z = [sq("lu2_mu")]
    for d in range(1, v):
        lam = sq("lu2_lambda")
        lam2 = x_mul(lam, lam)
        vecs = []
        for Pl, Ql in trees:
            Pc, Qc = Pl[d + 1], Ql[d + 1]
            vecs += [[Pc[2 * x] for x in range(1 << d)], [Pc[2 * x + 1] for x in range(1 << d)],
                     [Qc[2 * x] for x in range(1 << d)], [Qc[2 * x + 1] for x in range(1 << d)]]
        rho_l = []
        for t in range(d):
            gr = []
            for X in range(4):
                acc = (0, 0)
                rest = d - t - 1
                for bb in range(1 << rest):
                    pt = rho_l + [(X, 0)] + [((bb >> (rest - 1 - i)) & 1, 0) for i in range(rest)]
                    ev = [xv_mle(vv, pt) for vv in vecs]
                    F = (0, 0)
                    for tau, w in ((0, (1, 0)), (1, lam2)):
                        pL, pR, qL, qR = ev[4 * tau:4 * tau + 4]
                        f = x_add(x_add(x_mul(pL, qR), x_mul(pR, qL)), x_mul(lam, x_mul(qL, qR)))
                        F = x_add(F, x_mul(w, f))
                    acc = x_add(acc, x_mul(x_eq(z, pt), F))
                gr.append(acc)
            send("lu2_round", gr)
            rho_l.append(sq("lu2_chal"))
        send("lu2_final", [xv_mle(vv, rho_l) for vv in vecs])
        z = rho_l + [sq("lu2_mu")]
    send("lu2_leaf", [x_mle(rp, z), x_mle(qp, z), x_mle(yp, z)])
    return bytes(out)


def dsp_prove(seed: int, X, e, D, E: int) -> bytes:
    """The MoE dispatch proof from definitions: pos(t) by a stable sort of the tokens by
    expert, every MLE a hypercube sum at field points (no folding)."""
    X = np.asarray(X, dtype=np.int64)
    D = np.asarray(D, dtype=np.int64)
    e = [int(v) for v in np.asarray(e).reshape(-1)]
    T, K = X.shape
    vT, vK = log2c(T), log2c(K)
    order = sorted(range(T), key=lambda t: (e[t], t))  # expert-major, token order within
    pos = [0] * T
    for p, t in enumerate(order):
        pos[t] = p
    tx = Tx(seed)
    out = bytearray()

    def send(label, vals):
        b = fe_bytes(vals)
        out.extend(b)
        tx.absorb(label, b)

    tx.absorb("dsp_site", tree_digest(X.astype(np.int8).tobytes()) +
              tree_digest(np.asarray(e, "<i4").tobytes()) + tree_digest(D.astype(np.int8).tobytes()))
    rr = [tx.squeeze("dsp_row") for _ in range(vT)]
    rc = [tx.squeeze("dsp_col") for _ in range(vK)]
    send("dsp_claim", [mle2(D, rr, rc)])
    Pv = [eq_point(rr, pos[t]) for t in range(T)]
    Bv = [mle(X[t], rc) for t in range(T)]
    rho = []
    for t in range(vT):
        rest = vT - t - 1
        g = []
        for Xp in range(3):
            acc = 0
            for bb in range(1 << rest):
                w = rho + [Xp] + [(bb >> (rest - 1 - i)) & 1 for i in range(rest)]
                acc += mle_at(Pv, w) * mle_at(Bv, w)
            g.append(acc % P)
        send("dsp_round", g)
        rho.append(tx.squeeze("dsp_chal"))
    send("dsp_final", [mle_at(Pv, rho), mle_at(Bv, rho)])
    return bytes(out)
