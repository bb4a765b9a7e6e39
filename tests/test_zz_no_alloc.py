"""The no-allocation partial evaluation (mle_partial_eval_noalloc) against the
regular entry point (mle_partial_eval), through the C ABI.

The no-allocation variant serves callers that must not allocate device memory
(allocator hooks, host callbacks, pools that forbid out-of-band cudaMalloc):
it keeps its scratch in one fixed array inside the library. Two calls in a row
must each give exactly the regular entry point's result -- the second call
must not see anything the first left in the shared scratch array. The file is
named so that pytest collects it last.
"""

import ctypes as C

import numpy as np
import pytest

import oracle
import workloads

pytestmark = pytest.mark.gpu

FP_ERR_SHAPE = -2


@pytest.fixture(scope="module")
def env():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sum_check_prover_b200 import build
    build.build()
    import sum_check_prover_b200 as fp
    L = fp.lib()
    L.mle_partial_eval_noalloc.restype = C.c_int
    L.mle_partial_eval_noalloc.argtypes = [C.c_void_p, C.c_int, C.c_void_p, C.c_int, C.c_int,
                                           C.POINTER(C.c_uint64), C.c_int, C.c_void_p, C.c_void_p]
    ctx = fp.Context(0)
    yield torch, fp, L, ctx
    ctx.close()


def _case(seed, rows, cols, bits, scaled):
    rng = np.random.default_rng(seed)
    mat = workloads.int4_packed(rng, rows, cols) if bits == 4 else workloads.int8_uniform(rng, (rows, cols))
    sc = workloads.group_scales(rng, rows, cols) if scaled else None
    z = [int(x) for x in rng.integers(0, oracle.P, size=oracle.log2_ceil(rows), dtype=np.uint64)]
    return mat, sc, z


def _noalloc(torch, L, mat, bits, sc, rows, cols, z):
    out = torch.full((1 << oracle.log2_ceil(cols),), -1, dtype=torch.int64, device="cuda")
    pt = (C.c_uint64 * max(1, len(z)))(*z)
    stream = torch.cuda.current_stream().cuda_stream
    rc = L.mle_partial_eval_noalloc(mat.data_ptr(), bits, None if sc is None else sc.data_ptr(), rows, cols,
                                    pt, len(z), out.data_ptr(), stream)
    torch.cuda.synchronize()
    return rc, out.cpu().numpy().view(np.uint64)


def _regular(torch, ctx, mat, bits, sc, rows, cols, z):
    out = torch.zeros((1 << oracle.log2_ceil(cols),), dtype=torch.int64, device="cuda")
    ctx.partial_eval(mat, bits, sc, rows, cols, z, out)
    torch.cuda.synchronize()
    return out.cpu().numpy().view(np.uint64)


def test_no_alloc_matches_regular_entry_point_twice(env):
    torch, fp, L, ctx = env
    # two different statements back to back: the first leaves the scratch full
    cases = [(1, 3000, 4096, 4, False), (2, 1500, 1000, 4, True), (3, 70, 517, 8, False)]
    for seed, rows, cols, bits, scaled in cases:
        mat, sc, z = _case(seed, rows, cols, bits, scaled)
        dm = torch.from_numpy(mat).cuda()
        ds = None if sc is None else torch.from_numpy(sc).cuda()
        rc1, a = _noalloc(torch, L, dm, bits, ds, rows, cols, z)
        want = _regular(torch, ctx, dm, bits, ds, rows, cols, z)
        assert rc1 == 0
        assert np.array_equal(a, want)
        rc2, b = _noalloc(torch, L, dm, bits, ds, rows, cols, z)
        assert rc2 == 0
        assert np.array_equal(b, want)


def test_no_alloc_rejects_shapes_beyond_its_scratch(env):
    torch, fp, L, ctx = env
    rows, cols = 4096, 1 << 20        # 4 splits x 2^20 columns > 2^21 words
    pt = (C.c_uint64 * 12)(*([5] * 12))
    dummy = torch.zeros(16, dtype=torch.int8, device="cuda")
    out = torch.zeros(16, dtype=torch.int64, device="cuda")
    rc = L.mle_partial_eval_noalloc(dummy.data_ptr(), 8, None, rows, cols, pt, 12, out.data_ptr(), None)
    assert rc == FP_ERR_SHAPE
