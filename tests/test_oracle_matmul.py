"""Pins of the oracle's witness, partial evaluations and output claim.

Witness ("How fast can FlashProve go", 3.1): Y = W . X in integers, rescale
q = round(Y / 2^k) with the remainder r = Y - 2^k q committed, y = clamp(q).
Checked against numpy's integer matmul and floor division (library routines).

Sum-check statement ("How fast can FlashProve go", 2 Background): the MLE of
the product at a random point factors through the partial evaluations,
sum_k W~(zr, k) X~(k, zc) = Y~(zr, zc) -- the identity the matmul
sum-check proves. It ties the witness, both partial evaluations and the
claim together, so a dropped term or a transposed operand in any of them
breaks it.
"""

import random

import numpy as np
import pytest

import oracle
import workloads
from tests import bruteforce as bf

P = oracle.P

SHAPES = [
    # M, K, N, w_bits, k, scales
    (1, 1, 1, 8, 1, False),
    (3, 5, 2, 8, 3, False),
    (7, 33, 5, 4, 4, False),      # odd K: padding nibble
    (9, 130, 3, 4, 12, True),     # scales with a ragged last group
    (16, 64, 16, 4, 7, True),
    (5, 200, 9, 8, 18, False),
]


def _numpy_witness(s):
    W = bf.weights(s)
    Y = W @ s.xt.astype(np.int64).T            # M x N
    k = s.k_shift
    q = (Y + (1 << (k - 1))) // (1 << k)      # numpy floor division
    r = Y - q * (1 << k)
    y = np.clip(q, -128, 127)
    return Y.T, q.T, r.T, y.T                 # token-major


@pytest.mark.parametrize("shape", SHAPES)
def test_witness_matches_numpy(shape):
    M, K, N, b, k, sc = shape
    s = workloads.random_site(100 + M + K, M, K, N, b, k, scales=sc)
    q, r, y = oracle.witness(s)
    Y, q2, r2, y2 = _numpy_witness(s)
    assert np.array_equal(q, q2) and np.array_equal(r, r2) and np.array_equal(y, y2)
    assert np.array_equal((q.astype(np.int64) << k) + r, Y)
    assert r.min() >= -(1 << (k - 1)) and r.max() < (1 << (k - 1))


def test_witness_rejects_overflowing_accumulator():
    K = 140000   # 127 * 127 * K > 2^31
    s = workloads.Site("big", 1, K, 1, 8, 7, w=np.full((1, K), 127, np.int8), xt=np.full((1, K), 127, np.int8))
    with pytest.raises(ValueError):
        oracle.witness(s)


def test_witness_round_half_up_ties():
    # Y = 2^(k-1) * (2t+1) are exact ties; round half up sends them to t + 1.
    k = 3
    xs = np.array([[4, -4, 12, -12, 3, -5, 127, -128]], np.int8)
    s = workloads.Site("tie", 1, 8, 1, 8, k, w=np.eye(1, 8, dtype=np.int8), xt=xs)
    for col in range(8):
        w = np.zeros((1, 8), np.int8)
        w[0, col] = 1
        s.w = w
        q, r, y = oracle.witness(s)
        Yv = int(xs[0, col])
        assert int(q[0, 0]) == int(np.floor(Yv / 8 + 0.5))


@pytest.mark.parametrize("shape", SHAPES)
def test_partial_evals_brute_force_and_boolean_points(shape):
    M, K, N, b, k, sc = shape
    if M * K > 400:
        pytest.skip("brute force only on tiny shapes")
    s = workloads.random_site(200 + M, M, K, N, b, k, scales=sc)
    rnd = random.Random(M * K)
    zr = [rnd.randrange(P) for _ in range(oracle.log2_ceil(M))]
    zc = [rnd.randrange(P) for _ in range(oracle.log2_ceil(N))]
    A = oracle.partial_w(s, zr)
    Bv = oracle.partial_x(s, zc)
    W = bf.weights(s)
    X = s.xt.astype(np.int64).T
    for kk in range(K):
        assert int(A[kk]) == bf.mle(W[:, kk], zr)
        assert int(Bv[kk]) == bf.mle(X[kk, :], zc)
    assert all(int(a) == 0 for a in A[K:]) and all(int(v) == 0 for v in Bv[K:])
    i0 = rnd.randrange(M)
    zb = [(i0 >> (len(zr) - 1 - t)) & 1 for t in range(len(zr))]
    A0 = oracle.partial_w(s, zb)
    assert [int(a) for a in A0[:K]] == [int(w) % P for w in W[i0]]   # row selection
    assert np.array_equal(oracle.partial_rows(s.w, b, s.scales, M, K, zr), A)


@pytest.mark.parametrize("shape", SHAPES)
def test_matmul_identity(shape):
    M, K, N, b, k, sc = shape
    s = workloads.random_site(300 + K, M, K, N, b, k, scales=sc)
    q, r, y = oracle.witness(s)
    rnd = random.Random(K)
    for _ in range(3):
        zr = [rnd.randrange(P) for _ in range(oracle.log2_ceil(M))]
        zc = [rnd.randrange(P) for _ in range(oracle.log2_ceil(N))]
        A = oracle.partial_w(s, zr)
        Bv = oracle.partial_x(s, zc)
        lhs = sum(int(a) * int(v) for a, v in zip(A, Bv)) % P
        assert lhs == oracle.claim(q, r, M, N, k, zr, zc)


def test_claim_special_cases():
    s = workloads.random_site(7, 8, 16, 4, 8, 5)
    q, r, y = oracle.witness(s)
    Y = (q.astype(np.int64) << 5) + r
    for i, j in [(0, 0), (7, 3), (5, 1)]:
        zr = [(i >> (2 - t)) & 1 for t in range(3)]
        zc = [(j >> (1 - t)) & 1 for t in range(2)]
        assert oracle.claim(q, r, 8, 4, 5, zr, zc) == int(Y[j, i]) % P     # Boolean point = entry
    # W = I: the claim is X's MLE (K = M)
    s2 = workloads.Site("id", 16, 16, 4, 8, 5, w=np.eye(16, dtype=np.int8), xt=s.xt[:, :16].copy())
    q2, r2, _ = oracle.witness(s2)
    rnd = random.Random(9)
    zr = [rnd.randrange(P) for _ in range(4)]
    zc = [rnd.randrange(P) for _ in range(2)]
    assert oracle.claim(q2, r2, 16, 4, 5, zr, zc) == bf.mle2(s2.xt.astype(np.int64).T, zr, zc)
    # X = 0: everything is zero
    s3 = workloads.Site("zero", 8, 16, 4, 8, 5, w=s.w, xt=np.zeros((4, 16), np.int8))
    q3, r3, _ = oracle.witness(s3)
    assert oracle.claim(q3, r3, 8, 4, 5, zr[:3], zc) == 0
    assert not oracle.partial_x(s3, zc).any()
