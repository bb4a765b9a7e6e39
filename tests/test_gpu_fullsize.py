"""The layer configurations at their full sizes, on the GPU, checked against the oracle.

* decode layer (attention + dense MLP, 1031 sites) and Llama-shaped FFN
  (7.2e11 MACs): the oracle proved the same statements offline
  (tests/golden/make_golden.py writes oracle_fullsize.json); the GPU proof and
  witness must hash to the same SHA-256 digests and end in the same transcript
  states. Where the stored entry is missing, the decode layer is proved by the
  oracle live;
* FFN: the oracle's verifier also checks the GPU proof against the GPU
  witness in full, and witness entries sampled at random are recomputed one
  by one from W and X;
* MoE layer (387 sites, 8 GB of int4 weights): the proof, the transcript states
  and the witness must hash to the oracle's stored digests (byte parity); every
  protocol check of the verifier runs as well, with the direct evaluations of W
  and X for a sample of sites, and sampled witness entries are recomputed one
  by one.
"""

import hashlib
import json
from pathlib import Path

import numpy as np
import pytest

import oracle
import workloads
from tests import bruteforce as bf
from workloads import device

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


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


def gpu_prove(env, wl, seed):
    torch, fp, ctx = env
    stages, keep = device.upload(wl)
    device.weight_digests(ctx, stages)
    proof, states, status = fp.prove(ctx, seed, stages)
    torch.cuda.synchronize()
    wits = [(d.q.cpu().numpy(), d.r.cpu().numpy(), d.y.cpu().numpy()) for st in stages for d in st]
    flat = [d for st in stages for d in st]
    del stages, keep
    torch.cuda.empty_cache()
    return proof, states, status, wits, flat


def spot_check(sites, wits, n=300, seed=0):
    """Recompute sampled outputs one by one: Y = W_eff[i] . X[:, j], then q, r, y."""
    rng = np.random.default_rng(seed)
    for _ in range(n):
        s = int(rng.integers(len(sites)))
        st = sites[s]
        i, j = int(rng.integers(st.M)), int(rng.integers(st.N))
        if st.w_bits == 8:
            w = st.w[i].astype(np.int64)
        else:
            b = st.w[i].astype(np.int64)
            full = np.empty(2 * b.size, np.int64)
            full[0::2], full[1::2] = b & 15, b >> 4
            w = np.where(full >= 8, full - 16, full)[:st.K]
        if st.scales is not None:
            w = w * st.scales[i].astype(np.int64)[np.arange(st.K) // 64]
        Y = int(np.dot(w, st.xt[j].astype(np.int64)))
        k = st.k_shift
        q = (Y + (1 << (k - 1))) >> k
        q_, r_, y_ = wits[s]
        assert int(q_[j, i]) == q and int(r_[j, i]) == Y - (q << k), (st.name, i, j)
        assert int(y_[j, i]) == max(-128, min(127, q))


GOLDEN = Path(__file__).resolve().parent / "golden" / "oracle_fullsize.json"


def golden(cfg: int, seed: int = 0):
    if not GOLDEN.exists():
        return None
    return json.loads(GOLDEN.read_text()).get(f"config{cfg}_seed{seed}")


def witness_digest(wits) -> str:
    h = hashlib.sha256()
    for q, r, y in wits:
        h.update(q.astype("<i4").tobytes())
        h.update(r.astype("<i4").tobytes())
        h.update(y.astype("i1").tobytes())
    return h.hexdigest()


def check_golden(g, proof, states, wits):
    assert witness_digest(wits) == g["witness_sha256"]
    assert [s.hex() for s in states] == g["states"]
    assert len(proof) == g["proof_len"]
    assert hashlib.sha256(proof).hexdigest() == g["proof_sha256"]


def test_decode_layer_full_byte_parity(env):
    wl = workloads.build(4, seed=0)
    proof, states, status, wits, flat = gpu_prove(env, wl, 0)
    assert status == 0
    g = golden(4)
    if g is not None:
        assert g["sites"] == len(flat)
        check_golden(g, proof, states, wits)
        return
    R = oracle.resolve(wl)
    for idx, (q, r, y) in enumerate(R.wits):
        assert np.array_equal(wits[idx][0], q), flat[idx].name
        assert np.array_equal(wits[idx][1], r), flat[idx].name
        assert np.array_equal(wits[idx][2], y), flat[idx].name
    opf, ostates, _ = oracle.prove(0, R.sites, R.wits)
    assert states == ostates and proof == opf
    assert status == 0
    assert oracle.verify(0, R.sites, R.wits, proof)[0] == "accept"


def test_ffn_full_verified(env):
    wl = workloads.build(3, seed=0)
    proof, states, status, wits, flat = gpu_prove(env, wl, 0)
    assert status == 0
    g = golden(3)
    if g is not None:
        check_golden(g, proof, states, wits)
    spot_check(wl.sites, wits)
    w = bf.walk(0, wl.sites, wits, proof)
    assert w["consumed"] == len(proof) and w["state"] == states[2]
    assert oracle.verify(0, wl.sites, wits, proof)[0] == "accept"


def test_moe_full_sampled(env):
    wl = workloads.build(5, seed=0)
    assert len(wl.sites) == 387
    proof, states, status, wits, flat = gpu_prove(env, wl, 0)
    assert status == 0
    g = golden(5)
    if g is not None:  # byte parity with the oracle's proof of the whole layer
        assert g["sites"] == len(flat)
        check_golden(g, proof, states, wits)
    spot_check(wl.sites, wits, n=200)
    rng = np.random.default_rng(5)
    mask = np.zeros(len(wl.sites), np.uint8)
    mask[rng.choice(len(wl.sites) - 3, size=3, replace=False)] = 1
    mask[-3:] = 1  # the shared expert
    verdict, det = oracle.verify(0, wl.sites, wits, proof, site_mask=mask, skip_leaf_open=True)
    assert verdict == "accept", (verdict, det)
