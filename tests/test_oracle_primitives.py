"""Pins of the oracle's primitives against things other than itself:
Python integers, hashlib, published vectors, closed forms of the Goldilocks
field, and brute-force sums over the hypercube.

Field: Goldilocks p = 2^64 - 2^32 + 1 ("How fast can FlashProve go", 3.1).
"""

import hashlib
import os
import random
import struct

import numpy as np
import pytest

import oracle
from tests import bruteforce as bf

P = oracle.P
EDGE = [0, 1, 2, P - 1, P - 2, 2**32 - 1, 2**32, 2**32 + 1, 2**63, 2**64 - 2**32, P >> 1]


def test_field_ops_match_python_integers():
    rnd = random.Random(1)
    vals = EDGE + [rnd.randrange(P) for _ in range(300)]
    for a in vals:
        for b in (EDGE + [rnd.randrange(P) for _ in range(3)]):
            assert oracle.fmul(a, b) == a * b % P
            assert oracle.fadd(a, b) == (a + b) % P
            assert oracle.fsub(a, b) == (a - b) % P


def test_field_closed_forms():
    # 2^64 = 2^32 - 1 and 2^96 = -1 (mod p); 2 has order 192.
    assert oracle.fpow(2, 64) == 2**32 - 1
    assert oracle.fpow(2, 96) == P - 1
    assert oracle.fpow(2, 192) == 1
    # p - 1 = 2^32 * 3 * 5 * 17 * 257 * 65537 and 7 generates the multiplicative group
    assert (P - 1) == 2**32 * 3 * 5 * 17 * 257 * 65537
    assert oracle.fpow(7, P - 1) == 1
    for f in (2, 3, 5, 17, 257, 65537):
        assert oracle.fpow(7, (P - 1) // f) != 1
    rnd = random.Random(2)
    for _ in range(50):
        a = rnd.randrange(1, P)
        assert oracle.fmul(a, oracle.finv(a)) == 1


def test_integer_lift():
    for v in [0, 1, -1, 127, -128, 2**31 - 1, -(2**31), -(2**63), 2**62]:
        assert oracle.fint(v) == v % P


def test_sha256_matches_hashlib_and_fips_vectors():
    rnd = random.Random(3)
    for n in list(range(0, 140)) + [1023, 1024, 1025, 4099]:
        m = bytes(rnd.randrange(256) for _ in range(n))
        assert oracle.sha256(m) == hashlib.sha256(m).digest()
    path = os.path.join(os.path.dirname(__file__), "golden", "sha256_fips180_4.txt")
    for line in open(path):
        if line.startswith("#"):
            continue
        msg, dig = line.rstrip("\n").split("\t")
        assert oracle.sha256(msg.encode()).hex() == dig


@pytest.mark.parametrize("n", [0, 1, 1000, 1024, 1025, 2048, 33 * 1024, 33 * 1024 + 5, 32 * 32 * 1024 + 1])
def test_tree_digest_special_cases(n):
    rnd = random.Random(n)
    data = bytes(rnd.randrange(256) for _ in range(n))
    h = lambda b: hashlib.sha256(b).digest()
    # the definition's special cases, written with hashlib directly
    if n <= 1024:
        want = h(struct.pack("<Q", n) + h(data))
    else:
        lv = [h(data[i:i + 1024]) for i in range(0, n, 1024)]
        while len(lv) > 1:
            lv = [h(b"".join(lv[i:i + 32])) for i in range(0, len(lv), 32)]
        want = h(struct.pack("<Q", n) + lv[0])
    assert oracle.tree_digest(data) == want
    if n == 2048:  # two chunks, one parent
        assert want == h(struct.pack("<Q", n) + h(h(data[:1024]) + h(data[1024:])))


def test_transcript_encoding():
    t = oracle.Transcript(42)
    s0 = hashlib.sha256(b"FPSC-v1" + struct.pack("<Q", 42)).digest()
    assert t.state() == s0
    t.absorb("abc", b"\x01\x02")
    s1 = hashlib.sha256(s0 + struct.pack("<I", 3) + b"abc" + struct.pack("<Q", 2) + b"\x01\x02").digest()
    assert t.state() == s1
    c = t.squeeze("ch")
    h = hashlib.sha256(s1 + b"sq" + struct.pack("<I", 2) + b"ch" + struct.pack("<I", 0)).digest()
    v = int.from_bytes(h[:8], "little")
    assert v < P  # the rejection branch fires with probability 2^-32 and is not exercised here
    assert c == v and t.state() == h
    ref = bf.Tx(42)
    ref.absorb("abc", b"\x01\x02")
    assert ref.squeeze("ch") == c


def test_eq_table_properties():
    rnd = random.Random(5)
    for v in range(0, 9):
        z = [rnd.randrange(P) for _ in range(v)]
        e = oracle.eq_table(z)
        assert int(sum(int(x) for x in e) % P) == 1          # sum_x eq(z, x) = 1
        for x in range(1 << v):
            assert int(e[x]) == bf.eq_point(z, x)             # closed-form product
        if v:
            bits = [rnd.randrange(2) for _ in range(v)]       # Boolean z: indicator, z_1 = MSB
            e = oracle.eq_table(bits)
            idx = sum(b << (v - 1 - i) for i, b in enumerate(bits))
            assert [int(t) for t in e] == [1 if x == idx else 0 for x in range(1 << v)]


def test_mle_eval_properties():
    rnd = random.Random(6)
    for v in range(1, 7):
        n = rnd.randrange(1, (1 << v) + 1)                     # ragged: zero padding
        vals = [rnd.randrange(P) for _ in range(n)]
        z = [rnd.randrange(P) for _ in range(v)]
        assert oracle.mle_eval(vals, z) == bf.mle(vals, z)    # brute force over the cube
        x = rnd.randrange(1 << v)
        zb = [(x >> (v - 1 - b)) & 1 for b in range(v)]
        assert oracle.mle_eval(vals, zb) == (vals[x] if x < n else 0)
        b = rnd.randrange(v)                                   # multilinear in each coordinate
        f = []
        for t in (0, 1, 2):
            zz = list(z)
            zz[b] = t
            f.append(oracle.mle_eval(vals, zz))
        assert f[2] == (2 * f[1] - f[0]) % P


def test_lagrange_recovers_cubic():
    rnd = random.Random(7)
    c = [rnd.randrange(P) for _ in range(4)]
    poly = lambda x: (c[0] + c[1] * x + c[2] * x * x + c[3] * x ** 3) % P
    g = [poly(i) for i in range(4)]
    for _ in range(10):
        x = rnd.randrange(P)
        assert oracle.lagrange(g, x) == poly(x)
    quad = lambda x: (c[0] + c[1] * x + c[2] * x * x) % P
    q = [quad(i) for i in range(3)]
    for x in (5, P - 3, rnd.randrange(P)):
        assert oracle.lagrange(q, x) == quad(x)
