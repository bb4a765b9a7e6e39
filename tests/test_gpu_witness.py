"""The witness GEMM (Y = W_eff X, then q, r, y) on both tensor-core kernels,
against a plain numpy definition: int64 matrix product, floor division with
round-half-up, remainder, clamp ("How fast can FlashProve go", 3.1).

Three kernels: the warp-specialised tcgen05 kernel (the default) takes every site whose
operands TMA can read (16-byte rows), scaled ones through two byte limbs of s * w; the
single-role tcgen05 kernel (FP_TCGEN05=1) takes such sites without scales; the mma.sync
kernel takes the rest, or every site with FP_TCGEN05=0. Shapes cover partial tiles in
every dimension, K below and across k-tiles and scale groups, and one or many tiles per
site.
"""

import numpy as np
import pytest

import workloads
from workloads import device

pytestmark = pytest.mark.gpu

SHAPES = [
    # M, K, N, w_bits, scales
    (300, 128, 200, 8, False), (256, 256, 128, 4, False), (513, 96, 130, 4, False), (64, 16, 1, 8, False),
    (1000, 4096, 77, 4, False), (40, 32, 300, 4, False), (257, 160, 129, 8, False), (256, 1024, 512, 4, False),
    (129, 64, 64, 4, True), (77, 48, 33, 8, False), (33, 40, 17, 8, False),
    # scaled sites across k-tiles and scale groups, int4 and int8 (K < 1024 keeps int8 x scales exact)
    (300, 1024, 200, 4, True), (257, 768, 129, 8, True), (64, 96, 5, 8, True), (2048, 512, 1280, 4, True),
    # enough 256-row tiles to fill the GPU: the tcgen05 kernel's N = 256 variant
    (4096, 256, 1280, 4, False), (2048, 128, 2560, 8, False),
]


def expected(site):
    w = site.w.astype(np.int64)
    if site.w_bits == 4:
        lo, hi = w & 15, w >> 4
        full = np.empty((site.M, 2 * w.shape[1]), np.int64)
        full[:, 0::2], full[:, 1::2] = lo, hi
        w = np.where(full >= 8, full - 16, full)[:, :site.K]
    if site.scales is not None:
        w = w * np.repeat(site.scales.astype(np.int64), 64, axis=1)[:, :site.K]
    Y = site.xt.astype(np.int64) @ w.T  # N x M, token-major like the witness
    k = site.k_shift
    q = (Y + (1 << (k - 1))) >> k
    return q, Y - (q << k), np.clip(q, -128, 127)


@pytest.fixture(scope="module")
def lib():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sum_check_prover_b200 import build
    build.build()
    import sum_check_prover_b200 as fp
    return torch, fp


@pytest.mark.parametrize("tcgen05", ["2", "1", "0"])
@pytest.mark.parametrize("shape", SHAPES)
def test_witness_matches_definition(lib, shape, tcgen05, monkeypatch):
    torch, fp = lib
    M, K, N, bits, sc = shape
    monkeypatch.setenv("FP_TCGEN05", tcgen05)  # read when the context is created
    ctx = fp.Context(0)
    try:
        site = workloads.random_site(M * 31 + K * 7 + N, M, K, N, bits, 12, scales=sc)
        stages, keep = device.upload(workloads.Workload("w", 0, [site]))
        tx = fp.Transcript(0)
        ctx.commit_witness(tx, stages[0])
        torch.cuda.synchronize()
        d = stages[0][0]
        q, r, y = expected(site)
        assert np.array_equal(d.q.cpu().numpy(), q)
        assert np.array_equal(d.r.cpu().numpy(), r)
        assert np.array_equal(d.y.cpu().numpy(), y)
        tx.close()
    finally:
        ctx.close()
