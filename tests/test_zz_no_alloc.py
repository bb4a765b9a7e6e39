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


# int4 and int8, with and without per-64 scales (int8 with scales adds the largest offset,
# 2^14, over up to 1024 rows per split); rows a multiple of 1024 and ragged; columns below
# and above one block's 1024 and not a multiple of it
CASES = [(1, 3000, 4096, 4, False), (2, 1500, 1000, 4, True), (3, 70, 517, 8, False),
         (4, 2048, 1000, 8, True), (5, 1024, 1031, 8, False)]


@pytest.mark.parametrize("seed,rows,cols,bits,scaled", CASES)
def test_no_alloc_matches_regular_entry_point_twice(env, seed, rows, cols, bits, scaled):
    torch, fp, L, ctx = env
    mat, sc, z = _case(seed, rows, cols, bits, scaled)
    dm = torch.from_numpy(mat).cuda()
    ds = None if sc is None else torch.from_numpy(sc).cuda()
    rc1, a = _noalloc(torch, L, dm, bits, ds, rows, cols, z)
    want = _regular(torch, ctx, dm, bits, ds, rows, cols, z)
    assert rc1 == 0
    assert np.array_equal(a, want)
    # the second call in a row finds the first call's partials in the shared scratch
    rc2, b = _noalloc(torch, L, dm, bits, ds, rows, cols, z)
    assert rc2 == 0
    assert np.array_equal(b, want)
    if rows * cols <= 1 << 21:  # and both equal the CPU oracle's partial evaluation
        assert np.array_equal(a, oracle.partial_rows(mat, bits, sc, rows, cols, z))


def test_no_alloc_allocates_nothing_after_the_first_call(env):
    torch, fp, L, ctx = env
    rows, cols, bits = 2000, 3000, 4
    mat, sc, z = _case(7, rows, cols, bits, True)
    dm = torch.from_numpy(mat).cuda()
    ds = torch.from_numpy(sc).cuda()
    out = torch.zeros((1 << oracle.log2_ceil(cols),), dtype=torch.int64, device="cuda")
    pt = (C.c_uint64 * len(z))(*z)
    stream = torch.cuda.current_stream().cuda_stream

    def call():
        rc = L.mle_partial_eval_noalloc(dm.data_ptr(), bits, ds.data_ptr(), rows, cols, pt, len(z),
                                        out.data_ptr(), stream)
        torch.cuda.synchronize()
        return rc

    assert call() == 0  # the first call on this device loads the module (and its 16 MiB array)
    free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    assert call() == 0
    assert call() == 0
    assert torch.cuda.mem_get_info()[0] == free0 and torch.cuda.memory_allocated() == alloc0


def test_no_alloc_rejects_shapes_beyond_its_scratch(env):
    torch, fp, L, ctx = env
    rows, cols = 4096, 1 << 20        # 4 splits x 2^20 columns > 2^21 words
    pt = (C.c_uint64 * 12)(*([5] * 12))
    dummy = torch.zeros(16, dtype=torch.int8, device="cuda")
    out = torch.zeros(16, dtype=torch.int64, device="cuda")
    rc = L.mle_partial_eval_noalloc(dummy.data_ptr(), 8, None, rows, cols, pt, 12, out.data_ptr(), None)
    assert rc == FP_ERR_SHAPE
