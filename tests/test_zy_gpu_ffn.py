"""The FFN layer statement on the GPU (fp.prove_ffn: the layer proof, its down projection reading
the layer's own hidden activations, continued on one transcript by the per-group scale reductions
at the point the matmul section left the weights, the hidden rescale's commitment and lookup, the
SiLU lookup of the gate projection's outputs and the gated product of the SiLU outputs with the up
projection's outputs; "How fast can FlashProve go", 3.1) against the oracle's statement
(oracle.prove_ffn), byte for byte, on small statements live and on the full-size FFN against the
oracle's stored digests."""

import hashlib
import json
from pathlib import Path

import numpy as np
import pytest

import oracle
import workloads
from workloads import device

pytestmark = pytest.mark.gpu

GOLDEN = Path(__file__).resolve().parent / "golden" / "oracle_fullsize.json"


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


def gpu_ffn(env, wl, seed, kh=7):
    torch, fp, ctx = env
    stages, keep = device.upload(wl)
    device.weight_digests(ctx, stages)
    proof, state, status = fp.prove_ffn(ctx, seed, stages, kh=kh)
    torch.cuda.synchronize()
    wits = [(d.q.cpu().numpy(), d.r.cpu().numpy(), d.y.cpu().numpy()) for st in stages for d in st]
    del stages, keep
    torch.cuda.empty_cache()
    return proof, state, status, wits


def ffn_sites(seed, M, K, N, bits, scales, k=9, kh=7):
    """gate and up (M x K), down (K x M) reading the hidden activations: one token block of N,
    common k."""
    gate = workloads.random_site(seed, M, K, N, bits, k, scales=scales)
    up = workloads.random_site(seed + 1, M, K, N, bits, k, scales=scales)
    down = workloads.random_site(seed + 2, K, M, N, bits, k, scales=scales)
    down.xt, down.xt_hidden, down.stage = None, (0, 1, kh), 1
    return workloads.Workload("ffn", 0, [gate, up, down])


def test_small_ffn_config(env):
    wl = workloads.build(3, seed=1, small=True, chained=True)
    proof, state, status, wits = gpu_ffn(env, wl, 3)
    R = oracle.resolve(wl)
    for (q, r, y), (oq, orr, oy) in zip(wits, R.wits):
        assert np.array_equal(q, oq) and np.array_equal(r, orr) and np.array_equal(y, oy)
    opf, ost = oracle.prove_ffn(3, R.sites, R.wits)
    assert proof == opf and state == ost
    assert oracle.verify_ffn(3, R.sites, R.wits, proof)[0] == "accept"


@pytest.mark.parametrize("shape", [(300, 256, 40, 4, False, 9, 7), (257, 512, 33, 4, True, 9, 5),
                                   (129, 768, 17, 8, True, 16, 9), (96, 64, 1, 8, False, 12, 1)])
def test_random_ffn_statements(env, shape):
    M, K, N, bits, sc, k, kh = shape
    wl = ffn_sites(700 + M, M, K, N, bits, sc, k, kh)
    proof, state, status, wits = gpu_ffn(env, wl, 5, kh)
    R = oracle.resolve(wl)
    assert np.array_equal(wits[2][2], R.wits[2][2])  # the down outputs, from the hidden activations
    opf, ost = oracle.prove_ffn(5, R.sites, R.wits, kh=kh)
    assert len(proof) == len(opf)
    assert proof == opf and state == ost


@pytest.mark.slow
def test_full_ffn_statement(env):
    data = json.loads(GOLDEN.read_text())
    g = data.get("config3_ffn_seed0")
    if g is None:
        pytest.skip("the oracle's digest of the full-size FFN statement is not stored")
    wl = workloads.build(3, seed=0, chained=True)
    proof, state, status, wits = gpu_ffn(env, wl, 0)
    h = hashlib.sha256()
    for q, r, y in wits:
        h.update(q.astype("<i4").tobytes())
        h.update(r.astype("<i4").tobytes())
        h.update(y.astype("i1").tobytes())
    assert h.hexdigest() == g["witness_sha256"]
    assert len(proof) == g["proof_len"]
    assert state.hex() == g["state"]
    assert hashlib.sha256(proof).hexdigest() == g["proof_sha256"]


def test_hidden_rescale_kernel(env):
    # every pair of 8-bit factors: aligned with a ragged tail (16 entries a step, then one by one)
    # and at an offset that takes the entry-by-entry path throughout
    torch, fp, ctx = env
    a = np.repeat(np.arange(-128, 128), 256).astype(np.int8)
    b = np.tile(np.arange(-128, 128), 256).astype(np.int8)
    for kh in (1, 7, 16):
        want = oracle.ffn_hidden(a, b, kh)
        for off, cut in ((0, 5), (3, 0)):
            n = a.size - off - cut
            s8 = torch.from_numpy(a[off:][:n].copy()).cuda()
            u = torch.from_numpy(b[off:][:n].copy()).cuda()
            buf_q = torch.empty(n + 4, dtype=torch.int32, device="cuda")
            buf_r = torch.empty(n + 4, dtype=torch.int32, device="cuda")
            buf_y = torch.empty(n + 16, dtype=torch.int8, device="cuda")
            q, r, y = buf_q[off % 4:][:n], buf_r[off % 4:][:n], buf_y[off:][:n]
            ctx.ffn_hidden(s8, u, kh, q, r, y)
            torch.cuda.synchronize()
            for got, w in zip((q, r, y), want):
                assert np.array_equal(got.cpu().numpy(), w[off:][:n])
