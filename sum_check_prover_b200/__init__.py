"""Python binding of libfp, the B200 sum-check prover for quantised matrix products.

Argument marshalling only: every step of the proof runs in the CUDA library
(``libfp.so``, built in-tree by ``sum_check_prover_b200.build``). PyTorch is
used by callers for device memory and streams; this module only passes
``data_ptr()`` values and host buffers through the C ABI declared in
``include/fp.h``. It fails loudly when the library is missing: there is no
CPU fallback.
"""

from __future__ import annotations

import ctypes as C
from pathlib import Path
from typing import Optional, Sequence

__all__ = ["FpError", "Context", "Transcript", "SiteDesc", "prove", "prove_shard", "Shard", "lib", "LIB_PATH",
           "kernel_names", "P",
           "had2_protocol_drive", "lhi_protocol_drive", "mm2_protocol_drive", "route_protocol_drive",
           "lhi2_protocol_drive", "lookup16x_protocol_drive", "lu2_protocol_drive"]

P = 0xFFFFFFFF00000001
LIB_PATH = Path(__file__).resolve().with_name("libfp.so")

FP_OK = 0
FP_WARN_KEYS_OUTSIDE_TABLE = 1


class FpError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libfp error {code}: {msg}")
        self.code = code


class _Site(C.Structure):
    _fields_ = [("w", C.c_void_p), ("scales", C.c_void_p), ("xt", C.c_void_p),
                ("q", C.c_void_p), ("r", C.c_void_p), ("y", C.c_void_p),
                ("w_bits", C.c_int32), ("M", C.c_int32), ("K", C.c_int32), ("N", C.c_int32),
                ("k_shift", C.c_int32), ("w_digest", C.c_void_p)]


class _KStat(C.Structure):
    _fields_ = [("kernel", C.c_int32), ("launches", C.c_int32), ("ms", C.c_double), ("bytes", C.c_double)]


class _LRec(C.Structure):
    _fields_ = [("kernel", C.c_int32), ("reserved", C.c_int32), ("ms", C.c_double), ("bytes", C.c_double),
                ("start_ms", C.c_double)]


_lib = None


def lib():
    """Load libfp.so (raises ImportError if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not LIB_PATH.exists():
        raise ImportError(f"{LIB_PATH} is missing: build it with sum_check_prover_b200.build.build() (nvcc, sm_100a)")
    L = C.CDLL(str(LIB_PATH))
    vp, i32, u64, sz = C.c_void_p, C.c_int, C.c_uint64, C.c_size_t
    L.fp_version.restype = i32
    L.fp_ctx_create.restype = vp
    L.fp_ctx_create.argtypes = [i32]
    L.fp_ctx_destroy.argtypes = [vp]
    L.fp_last_error.restype = C.c_char_p
    L.fp_last_error.argtypes = [vp]
    L.fp_tx_create.restype = vp
    L.fp_tx_create.argtypes = [u64]
    L.fp_tx_destroy.argtypes = [vp]
    L.fp_tx_absorb.argtypes = [vp, C.c_char_p, vp, sz]
    L.fp_tx_squeeze.argtypes = [vp, C.c_char_p, C.POINTER(u64), sz]
    L.fp_tx_state.argtypes = [vp, vp]
    L.fp_digest.argtypes = [vp, vp, sz, vp, vp]
    L.fp_digests.argtypes = [vp, vp, vp, i32, vp, vp]
    L.fp_commit_witness.argtypes = [vp, vp, C.POINTER(_Site), i32, vp]
    L.mle_partial_eval.argtypes = [vp, vp, i32, vp, i32, i32, C.POINTER(u64), i32, vp, vp]
    L.sumcheck_prove_matmul.argtypes = [vp, vp, C.POINTER(_Site), i32, vp, C.POINTER(sz), vp]
    L.logup_prove_rescale.argtypes = [vp, vp, C.POINTER(_Site), i32, vp, C.POINTER(sz), vp]
    L.sumcheck_prove_hadamard.argtypes = [vp, vp, vp, vp, C.c_int64, vp, C.POINTER(sz), vp]
    L.sumcheck_prove_hadamard_ext2.argtypes = [vp, vp, vp, vp, C.c_int64, vp, C.POINTER(sz), vp]
    L.fp_had2_protocol_drive.argtypes = [vp, i32, _VALUES_FN, vp, vp, C.POINTER(sz)]
    L.sumcheck_prove_matmul_ext2.argtypes = [vp, vp, C.POINTER(_Site), vp, C.POINTER(sz), vp]
    L.freivalds_prove_matmul.argtypes = [vp, vp, C.POINTER(_Site), vp, C.POINTER(sz), vp]
    L.sumcheck_prove_routing.argtypes = [vp, vp, vp, C.c_int64, i32, vp, vp, vp, C.POINTER(sz), vp]
    L.fp_route_protocol_drive.argtypes = [vp, i32, _VALUES_FN, vp, vp, C.POINTER(sz)]
    L.logup_prove_silu_ext2.argtypes = [vp, vp, vp, vp, C.c_int64, vp, C.POINTER(sz), vp]
    L.logup_prove_exp_ext2.argtypes = [vp, vp, vp, vp, C.c_int64, vp, C.POINTER(sz), vp]
    L.fp_lookup16x_protocol_drive.argtypes = [vp, i32, i32, C.POINTER(u64), vp, vp, _VALUES_FN, vp, vp, C.POINTER(sz)]
    L.logup_prove_rescale_ext2.argtypes = [vp, vp, C.POINTER(_Site), i32, vp, C.POINTER(sz), vp]
    L.fp_lu2_protocol_drive.argtypes = [vp, i32, i32, vp, vp, vp, vp, _VALUES_FN, vp, vp, C.POINTER(sz)]
    L.logup_prove_helper_inverse_ext2.argtypes = [vp, vp, vp, C.c_int64, i32, vp, C.POINTER(sz), vp]
    L.fp_lhi2_protocol_drive.argtypes = [vp, i32, i32, vp, vp, _VALUES_FN, vp, vp, C.POINTER(sz)]
    L.fp_mm2_protocol_drive.argtypes = [vp, i32, i32, i32, _VALUES_FN, vp, vp, C.POINTER(sz)]
    L.logup_prove_helper_inverse.argtypes = [vp, vp, vp, C.c_int64, i32, vp, C.POINTER(sz), vp]
    L.fp_lhi_protocol_drive.argtypes = [vp, i32, i32, vp, vp, _VALUES_FN, vp, vp, C.POINTER(sz)]
    L.sumcheck_reduce_scales.argtypes = [vp, vp, vp, i32, vp, i32, i32, C.POINTER(u64), vp, vp, C.POINTER(sz), vp]
    L.logup_prove_silu.argtypes = [vp, vp, vp, vp, C.c_int64, vp, C.POINTER(sz), vp]
    L.fp_silu_table.argtypes = [vp]
    L.fp_silu_inputs.argtypes = [vp, vp, C.c_int64, vp, vp, vp, vp]
    L.fp_ffn_hidden.argtypes = [vp, vp, vp, C.c_int64, i32, vp, vp, vp, vp]
    L.sumcheck_last_point.argtypes = [vp, vp, i32, C.POINTER(i32), vp, i32, C.POINTER(i32)]
    L.logup_prove_exp.argtypes = [vp, vp, vp, vp, C.c_int64, vp, C.POINTER(sz), vp]
    L.fp_exp_table.argtypes = [vp]
    L.fp_proof_size.argtypes = [C.POINTER(_Site), i32, C.POINTER(sz), C.POINTER(sz)]
    L.fp_commit_witness_shard.argtypes = [vp, vp, C.POINTER(_Site), i32, C.POINTER(_Shard), vp]
    L.sumcheck_prove_matmul_shard.argtypes = [vp, vp, C.POINTER(_Site), i32, C.POINTER(_Shard), vp, C.POINTER(sz),
                                              vp]
    L.fp_mm_shard_protocol_drive.argtypes = [vp, C.POINTER(_Site), i32, C.POINTER(_Shard), _VALUES_FN, vp, vp,
                                             C.POINTER(sz)]
    L.logup_prove_rescale_hi.argtypes = [vp, vp, C.POINTER(_Site), i32, vp, C.POINTER(sz), vp]
    L.sumcheck_prove_dispatch.argtypes = [vp, vp, vp, vp, vp, C.c_int64, C.c_int64, i32, vp, C.POINTER(sz), vp]
    L.fp_lhr_protocol_drive.argtypes = [vp, i32, i32, vp, vp, _VALUES_FN, vp, vp, C.POINTER(sz)]
    L.fp_ctx_set_profiling.argtypes = [vp, i32]
    L.fp_session_selftest.argtypes = [vp, vp]
    L.fp_host_stats.argtypes = [vp, C.POINTER(C.c_double)]
    L.fp_ctx_launches.restype = C.c_int64
    L.fp_ctx_launches.argtypes = [vp]
    L.fp_kernel_stats.argtypes = [vp, C.POINTER(_KStat), i32]
    L.fp_kernel_log.restype = C.c_int64
    L.fp_kernel_log.argtypes = [vp, C.POINTER(_LRec), C.c_int64]
    L.fp_kernel_name.restype = C.c_char_p
    L.fp_kernel_name.argtypes = [i32]
    _lib = L
    return L


# int (*)(void* user, int kind, int t, const uint64_t* in, uint64_t* out)
_VALUES_FN = C.CFUNCTYPE(C.c_int, C.c_void_p, C.c_int, C.c_int, C.POINTER(C.c_uint64), C.POINTER(C.c_uint64))
VAL_START, VAL_SINGLE, VAL_ROUND, VAL_ANSWER, VAL_FINALS, VAL_COLUMN, VAL_CLAIM, VAL_WEIGHTS = range(8)

# int (*)(void* user, const void* mine, size_t bytes, void* all)
_ALLGATHER_FN = C.CFUNCTYPE(C.c_int, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p)


class _Shard(C.Structure):
    _fields_ = [("rank", C.c_int32), ("world", C.c_int32), ("site_lo", C.POINTER(C.c_int32)),
                ("allgather", _ALLGATHER_FN), ("user", C.c_void_p)]


class Shard:
    """This rank's share of one statement proven by several ranks: rank r proves the
    sites [site_lo[r], site_lo[r + 1]). `allgather(data: bytes) -> list of bytes` returns
    every rank's bytes in rank order (the same length on every rank)."""

    def __init__(self, rank: int, world: int, site_lo: Sequence[int], allgather):
        self.rank, self.world, self.site_lo = int(rank), int(world), [int(x) for x in site_lo]

        def cb(_user, mine, nbytes, out):
            try:
                parts = allgather(C.string_at(mine, nbytes))
                if len(parts) != world or any(len(p) != nbytes for p in parts):
                    return 1
                C.memmove(out, b"".join(parts), nbytes * world)
                return 0
            except Exception:  # reported to the caller as FP_ERR_ARG
                return 1

        self._fn = _ALLGATHER_FN(cb)
        self._lo = (C.c_int32 * (world + 1))(*self.site_lo)
        self.c = _Shard(self.rank, self.world, self._lo, self._fn, None)

    @property
    def own(self) -> range:
        return range(self.site_lo[self.rank], self.site_lo[self.rank + 1])


def torch_allgather(group=None):
    """An all-gather of small host byte strings over a torch.distributed process group
    (gloo, or a gloo group beside NCCL): the host-mediated exchange of a shared statement."""
    import torch
    import torch.distributed as td

    def ag(data: bytes):
        world = td.get_world_size(group)
        mine = torch.frombuffer(bytearray(data), dtype=torch.uint8) if data else torch.zeros(0, dtype=torch.uint8)
        out = [torch.empty(len(data), dtype=torch.uint8) for _ in range(world)]
        td.all_gather(out, mine, group=group)
        return [bytes(t.numpy().tobytes()) for t in out]

    return ag


def balance_sites(costs: Sequence[float], world: int) -> list:
    """Contiguous site ranges, one per rank, with about equal cost each (every rank at
    least one site): the site_lo array of a Shard."""
    n = len(costs)
    if world < 1 or n < world:
        raise ValueError("balance_sites: need at least one site per rank")
    total = float(sum(costs))
    lo, acc, r = [0], 0.0, 1
    for i, c in enumerate(costs):
        acc += c
        # close rank r's range once it holds its share, leaving a site for every later rank
        while r < world and acc >= total * r / world and i + 1 <= n - (world - r):
            lo.append(i + 1)
            r += 1
    while len(lo) < world:
        lo.append(n - (world - len(lo)))
    lo.append(n)
    return lo


def lhr_protocol_drive(tx: "Transcript", v: int, k: int, m, m_digests: bytes, values) -> bytes:
    """Run the host half of the helper-inverse lookup section from the multiplicities on, with
    its device values taken from `values` (no GPU work): values.column(alpha0, alpha1, gamma)
    -> D(h0) || D(h1) (64 bytes), values.start(z, beta), values.round(t) -> 10 values,
    values.answer(t, rho), values.finals() -> 5 values. m: the 2^k + 2^16 multiplicities
    (m_rem then m_clamp); m_digests: their two tree digests."""
    import numpy as np
    L = lib()

    def cb(_user, kind, t, inp, out):
        try:
            if kind == VAL_COLUMN:
                d = values.column(int(inp[0]), int(inp[1]), int(inp[2]))
                for i in range(8):
                    out[i] = int.from_bytes(d[8 * i:8 * i + 8], "little")
                return 0
            if kind == VAL_START:
                values.start([int(inp[i]) for i in range(t)], int(inp[t]))
                return 0
            if kind == VAL_ANSWER:
                values.answer(t, int(inp[0]))
                return 0
            res = values.round(t) if kind == VAL_ROUND else values.finals()
            for i, x in enumerate(res):
                out[i] = int(x) % P
            return 0
        except Exception:  # reported to the caller as FP_ERR_ARG
            return 1

    fn = _VALUES_FN(cb)
    mm = np.ascontiguousarray(np.asarray(m, dtype=np.uint32))
    dg = C.create_string_buffer(bytes(m_digests), 64)
    ln = C.c_size_t(0)
    L.fp_lhr_protocol_drive(tx.h, v, k, mm.ctypes.data, dg, fn, None, None, C.byref(ln))
    buf = C.create_string_buffer(max(1, ln.value))
    rc = L.fp_lhr_protocol_drive(tx.h, v, k, mm.ctypes.data, dg, fn, None, buf, C.byref(ln))
    if rc != 0:
        raise FpError(rc, "fp_lhr_protocol_drive failed")
    return buf.raw[: ln.value]


def mm_shard_protocol_drive(tx: "Transcript", sites: Sequence["SiteDesc"], shard: Optional[Shard], values) -> bytes:
    """Run the host half of the (sharded) matmul sum-check with this rank's device values
    taken from `values` (no GPU work): values.start(r_row, r_col), values.claims() -> the own
    sites' c_s, values.weights(rho_own), values.round(t) -> (g(0), g(2)) share,
    values.answer(t, r), values.finals() -> [A_s, B_s, ...] of the own sites. tx must have
    absorbed the site records. Only the sites' shapes are read."""
    L = lib()
    arr, keep = _sites(sites)
    own = len(sites) if shard is None else len(shard.own)
    vM = max((s.M - 1).bit_length() for s in sites)

    def cb(_user, kind, t, inp, out):
        try:
            if kind == VAL_START:
                pts = [int(inp[i]) for i in range(t)]
                values.start(pts[:vM], pts[vM:])
                return 0
            if kind == VAL_WEIGHTS:
                values.weights([int(inp[i]) for i in range(t)])
                return 0
            if kind == VAL_ANSWER:
                values.answer(t, int(inp[0]))
                return 0
            res = {VAL_CLAIM: values.claims, VAL_FINALS: values.finals}.get(kind)
            res = values.round(t) if kind == VAL_ROUND else res()
            for i, x in enumerate(res):
                out[i] = int(x) % P
            return 0
        except Exception:  # reported to the caller as FP_ERR_ARG
            return 1

    fn = _VALUES_FN(cb)
    ln = C.c_size_t(0)
    sh = None if shard is None else C.byref(shard.c)
    L.fp_mm_shard_protocol_drive(tx.h, arr, len(sites), sh, fn, None, None, C.byref(ln))
    buf = C.create_string_buffer(max(1, ln.value))
    rc = L.fp_mm_shard_protocol_drive(tx.h, arr, len(sites), sh, fn, None, buf, C.byref(ln))
    if rc != 0:
        raise FpError(rc, "fp_mm_shard_protocol_drive failed")
    return buf.raw[: ln.value]


def had2_protocol_drive(tx: "Transcript", v: int, values) -> bytes:
    """Run the host half of the extension-field gated-product proof with its device values
    taken from `values` (no GPU work): values.start(z), values.single() -> (c, s0, u0),
    values.round(t) -> (h(0), h(1), h(2)), values.answer(t, rho), values.finals() -> (s, u),
    every extension element a pair (a, b). tx must have absorbed "had2_site"."""
    L = lib()

    def cb(_user, kind, t, inp, out):
        try:
            if kind == VAL_START:
                values.start([(int(inp[2 * i]), int(inp[2 * i + 1])) for i in range(t)])
                return 0
            if kind == VAL_ANSWER:
                values.answer(t, (int(inp[0]), int(inp[1])))
                return 0
            res = {VAL_SINGLE: values.single, VAL_FINALS: values.finals}.get(kind)
            res = values.round(t) if kind == VAL_ROUND else res()
            for i, (a, b) in enumerate(res):
                out[2 * i] = int(a)
                out[2 * i + 1] = int(b)
            return 0
        except Exception:  # reported to the caller as FP_ERR_ARG
            return 1

    fn = _VALUES_FN(cb)
    cap = 16 + 64 * v + 32
    buf = C.create_string_buffer(cap)
    ln = C.c_size_t(cap)
    rc = L.fp_had2_protocol_drive(tx.h, v, fn, None, buf, C.byref(ln))
    if rc != 0:
        raise FpError(rc, "fp_had2_protocol_drive failed")
    return buf.raw[: ln.value]


def mm2_protocol_drive(tx: "Transcript", vM: int, vN: int, n: int, values) -> bytes:
    """Run the host half of the extension-field matmul sum-check with its device values taken
    from `values` (no GPU work): values.start(r_row, r_col), values.claim() -> c,
    values.round(t) -> (g(0), g(1), g(2)), values.answer(t, rho), values.finals() -> (A, B),
    every extension element a pair (a, b). tx must have absorbed "mm2_site"."""
    L = lib()

    def cb(_user, kind, t, inp, out):
        try:
            if kind == VAL_START:
                pts = [(int(inp[2 * i]), int(inp[2 * i + 1])) for i in range(t)]
                values.start(pts[:vM], pts[vM:])
                return 0
            if kind == VAL_ANSWER:
                values.answer(t, (int(inp[0]), int(inp[1])))
                return 0
            if kind == VAL_CLAIM:
                res = [values.claim()]
            elif kind == VAL_ROUND:
                res = values.round(t)
            elif kind == VAL_FINALS:
                res = values.finals()
            else:
                return 1
            for i, (a, b) in enumerate(res):
                out[2 * i] = int(a)
                out[2 * i + 1] = int(b)
            return 0
        except Exception:  # reported to the caller as FP_ERR_ARG
            return 1

    fn = _VALUES_FN(cb)
    cap = 16 + 48 * n + 32
    buf = C.create_string_buffer(cap)
    ln = C.c_size_t(cap)
    rc = L.fp_mm2_protocol_drive(tx.h, vM, vN, n, fn, None, buf, C.byref(ln))
    if rc != 0:
        raise FpError(rc, "fp_mm2_protocol_drive failed")
    return buf.raw[: ln.value]


def route_protocol_drive(tx: "Transcript", n: int, values) -> bytes:
    """Run the host half of the routing proof up to "route_final" with its device values
    taken from `values` (no GPU work): values.start(z, w, lam1, lam2), values.claim() ->
    (D~(z), l~(z), row-sum weight), values.round(t) -> g(0..3), values.answer(t, rho),
    values.finals() -> (H~(rho), l~(rho)). tx must have absorbed "route_site"."""
    L = lib()

    def cb(_user, kind, t, inp, out):
        try:
            if kind == VAL_START:
                vals = [int(inp[i]) for i in range(2 * t + 2)]
                values.start(vals[:t], vals[t:2 * t], vals[2 * t], vals[2 * t + 1])
            elif kind == VAL_ANSWER:
                values.answer(t, int(inp[0]))
            elif kind in (VAL_CLAIM, VAL_ROUND, VAL_FINALS):
                res = values.claim() if kind == VAL_CLAIM else (values.round(t) if kind == VAL_ROUND
                                                                else values.finals())
                for i, x in enumerate(res):
                    out[i] = int(x)
            else:
                return 1
            return 0
        except Exception:  # reported to the caller as FP_ERR_ARG
            return 1

    fn = _VALUES_FN(cb)
    cap = 16 + 32 * n + 16
    buf = C.create_string_buffer(cap)
    ln = C.c_size_t(cap)
    rc = L.fp_route_protocol_drive(tx.h, n, fn, None, buf, C.byref(ln))
    if rc != 0:
        raise FpError(rc, "fp_route_protocol_drive failed")
    return buf.raw[: ln.value]


def lookup16x_protocol_drive(tx: "Transcript", table: int, v: int, gamma, m, m_digest: bytes, values) -> bytes:
    """Run the host half of the extension-field 16-bit lookup (table 0: SiLU, 1: exponent) from
    the multiplicities on, with its device values taken from `values` (no GPU work):
    values.tree(gamma, alpha) -> layer one's (P0, P1, Q0, Q1), values.layer(d, z, lam),
    values.round(t) -> (h(0), h(1), h(2)), values.answer(t, rho), values.finals() -> (pL, pR,
    qL, qR), values.leaf(z) -> (g~(z), s~(z)); extension elements are pairs (a, b). gamma is the
    pair squeezed after the site."""
    import numpy as np

    L = lib()

    def pairs(inp, k):
        return [(int(inp[2 * i]), int(inp[2 * i + 1])) for i in range(k)]

    def cb(_user, kind, t, inp, out):
        try:
            res = None
            if kind == VAL_COLUMN:
                ga = pairs(inp, 2)
                res = values.tree(ga[0], ga[1])
            elif kind == VAL_START:
                pts = pairs(inp, t + 1)
                values.layer(t, pts[:t], pts[t])
            elif kind == VAL_ANSWER:
                values.answer(t, (int(inp[0]), int(inp[1])))
            elif kind == VAL_ROUND:
                res = values.round(t)
            elif kind == VAL_FINALS:
                res = values.finals()
            elif kind == VAL_CLAIM:
                res = values.leaf(pairs(inp, t))
            else:
                return 1
            for i, (a, b) in enumerate(res or []):
                out[2 * i] = int(a)
                out[2 * i + 1] = int(b)
            return 0
        except Exception:  # reported to the caller as FP_ERR_ARG
            return 1

    fn = _VALUES_FN(cb)
    mm = np.ascontiguousarray(np.asarray(m, dtype="<u4"))
    md = C.create_string_buffer(bytes(m_digest), 32)
    gm = (C.c_uint64 * 2)(int(gamma[0]), int(gamma[1]))
    cap = 4 * 65536 + 64 + 32 + sum(64 * d + 64 for d in range(1, v))
    buf = C.create_string_buffer(cap)
    ln = C.c_size_t(cap)
    rc = L.fp_lookup16x_protocol_drive(tx.h, table, v, gm, mm.ctypes.data, md, fn, None, buf, C.byref(ln))
    if rc != 0:
        raise FpError(rc, "fp_lookup16x_protocol_drive failed")
    return buf.raw[: ln.value]


def lu2_protocol_drive(tx: "Transcript", v: int, k: int, m_rem, d_rem: bytes, m_clamp, d_clamp: bytes,
                       values) -> bytes:
    """Run the host half of the extension-field rescale LogUp from the multiplicities on, with
    its device values taken from `values` (no GPU work): values.tree(gamma, alpha0, alpha1) ->
    layer one of both trees (8 pairs), values.layer(d, z, lam), values.round(t) -> (h(0), h(1),
    h(2)), values.answer(t, rho), values.finals() -> 8 pairs, values.leaf(z) -> (r~, q~, y~).
    tx must have absorbed "lu2_site"."""
    import numpy as np

    L = lib()

    def pairs(inp, k_):
        return [(int(inp[2 * i]), int(inp[2 * i + 1])) for i in range(k_)]

    def cb(_user, kind, t, inp, out):
        try:
            res = None
            if kind == VAL_COLUMN:
                ga = pairs(inp, 3)
                res = values.tree(*ga)
            elif kind == VAL_START:
                pts = pairs(inp, t + 1)
                values.layer(t, pts[:t], pts[t])
            elif kind == VAL_ANSWER:
                values.answer(t, (int(inp[0]), int(inp[1])))
            elif kind == VAL_ROUND:
                res = values.round(t)
            elif kind == VAL_FINALS:
                res = values.finals()
            elif kind == VAL_CLAIM:
                res = values.leaf(pairs(inp, t))
            else:
                return 1
            for i, (a, b) in enumerate(res or []):
                out[2 * i] = int(a)
                out[2 * i + 1] = int(b)
            return 0
        except Exception:  # reported to the caller as FP_ERR_ARG
            return 1

    fn = _VALUES_FN(cb)
    mr = np.ascontiguousarray(np.asarray(m_rem, dtype="<u4"))
    mc = np.ascontiguousarray(np.asarray(m_clamp, dtype="<u4"))
    dr = C.create_string_buffer(bytes(d_rem), 32)
    dc = C.create_string_buffer(bytes(d_clamp), 32)
    cap = 4 * (1 << k) + 4 * 65536 + 128 + 48 + sum(64 * d + 128 for d in range(1, v))
    buf = C.create_string_buffer(cap)
    ln = C.c_size_t(cap)
    rc = L.fp_lu2_protocol_drive(tx.h, v, k, mr.ctypes.data, dr, mc.ctypes.data, dc, fn, None, buf, C.byref(ln))
    if rc != 0:
        raise FpError(rc, "fp_lu2_protocol_drive failed")
    return buf.raw[: ln.value]


def lhi2_protocol_drive(tx: "Transcript", v: int, k: int, m, m_digest: bytes, values) -> bytes:
    """As lhi_protocol_drive for the statement over the quadratic extension: every challenge and
    value an extension pair (a, b); values.column(alpha) -> 32-byte digest, values.start(z, beta),
    values.round(t) -> (H(0), H(1), Q(0), Q(1), Q(2)), values.answer(t, rho), values.finals()."""
    import numpy as np

    L = lib()

    def cb(_user, kind, t, inp, out):
        try:
            if kind == VAL_COLUMN:
                d = values.column((int(inp[0]), int(inp[1])))
                for i in range(4):
                    out[i] = int.from_bytes(d[8 * i: 8 * i + 8], "little")
            elif kind == VAL_START:
                pts = [(int(inp[2 * i]), int(inp[2 * i + 1])) for i in range(t + 1)]
                values.start(pts[:t], pts[t])
            elif kind == VAL_ANSWER:
                values.answer(t, (int(inp[0]), int(inp[1])))
            elif kind in (VAL_ROUND, VAL_FINALS):
                res = values.round(t) if kind == VAL_ROUND else values.finals()
                for i, (a, b) in enumerate(res):
                    out[2 * i] = int(a)
                    out[2 * i + 1] = int(b)
            else:
                return 1
            return 0
        except Exception:  # reported to the caller as FP_ERR_ARG
            return 1

    fn = _VALUES_FN(cb)
    mm = np.ascontiguousarray(np.asarray(m, dtype="<u4"))
    md = C.create_string_buffer(bytes(m_digest), 32)
    cap = 4 * (1 << k) + 16 + 64 * v + 32
    buf = C.create_string_buffer(cap)
    ln = C.c_size_t(cap)
    rc = L.fp_lhi2_protocol_drive(tx.h, v, k, mm.ctypes.data, md, fn, None, buf, C.byref(ln))
    if rc != 0:
        raise FpError(rc, "fp_lhi2_protocol_drive failed")
    return buf.raw[: ln.value]


def lhi_protocol_drive(tx: "Transcript", v: int, k: int, m, m_digest: bytes, values) -> bytes:
    """Run the host half of the helper-inverse LogUp from the multiplicities on, with its
    device values taken from `values` (no GPU work): values.column(alpha) -> 32-byte digest
    of the helper column, values.start(z, beta), values.round(t) -> (H(0), H(1), Q(0), Q(1),
    Q(2)), values.answer(t, rho), values.finals() -> (h~(rho), f~(rho)). m: 2^k counts;
    m_digest: the digest of their u32 little-endian bytes. tx must have absorbed "lhi_site"."""
    import numpy as np

    L = lib()

    def cb(_user, kind, t, inp, out):
        try:
            if kind == VAL_COLUMN:
                d = values.column(int(inp[0]))
                for i in range(4):
                    out[i] = int.from_bytes(d[8 * i: 8 * i + 8], "little")
            elif kind == VAL_START:
                values.start([int(inp[i]) for i in range(t)], int(inp[t]))
            elif kind == VAL_ANSWER:
                values.answer(t, int(inp[0]))
            elif kind == VAL_ROUND:
                for i, x in enumerate(values.round(t)):
                    out[i] = int(x)
            elif kind == VAL_FINALS:
                for i, x in enumerate(values.finals()):
                    out[i] = int(x)
            else:
                return 1
            return 0
        except Exception:  # reported to the caller as FP_ERR_ARG
            return 1

    fn = _VALUES_FN(cb)
    mm = np.ascontiguousarray(np.asarray(m, dtype="<u4"))
    md = C.create_string_buffer(bytes(m_digest), 32)
    cap = 4 * (1 << k) + 8 + 32 * v + 16
    buf = C.create_string_buffer(cap)
    ln = C.c_size_t(cap)
    rc = L.fp_lhi_protocol_drive(tx.h, v, k, mm.ctypes.data, md, fn, None, buf, C.byref(ln))
    if rc != 0:
        raise FpError(rc, "fp_lhi_protocol_drive failed")
    return buf.raw[: ln.value]


def kernel_names() -> list:
    L = lib()
    out, k = [], 0
    while True:
        nm = L.fp_kernel_name(k).decode()
        if nm == "?":
            return out
        out.append(nm)
        k += 1


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    return int(t.data_ptr()) if hasattr(t, "data_ptr") else int(t)


def _stream(stream) -> Optional[int]:
    if stream is None:
        try:
            import torch
            return int(torch.cuda.current_stream().cuda_stream)
        except Exception:
            return None
    return int(getattr(stream, "cuda_stream", stream))


class SiteDesc:
    """One product Y = W . X: device tensors (anything with data_ptr()) and sizes.

    w: M x K int8, or M x ceil(K/2) packed int4 bytes; scales: M x ceil(K/64) int8 or None;
    xt: N x K int8 (token-major X); q, r: N x M int32; y: N x M int8.
    w_digest: 64 bytes from Context.digest(w) + Context.digest(scales), or None.
    """

    def __init__(self, w, xt, q, r, y, M, K, N, w_bits, k_shift, scales=None, w_digest: Optional[bytes] = None):
        self.w, self.xt, self.q, self.r, self.y, self.scales = w, xt, q, r, y, scales
        self.M, self.K, self.N, self.w_bits, self.k_shift = int(M), int(K), int(N), int(w_bits), int(k_shift)
        self.w_digest = w_digest


def _site_records(sites):
    """The fp_site records of the sites as one numpy buffer laid out like _Site (filled a column
    at a time: a layer has hundreds of sites), and the buffers they point into."""
    import numpy as np
    fields = [f for f, _ in _Site._fields_]
    dt = np.dtype({"names": fields,
                   "formats": [np.uint64 if t is C.c_void_p else np.int32 for _, t in _Site._fields_],
                   "offsets": [getattr(_Site, f).offset for f in fields], "itemsize": C.sizeof(_Site)})
    n = len(sites)
    rec = np.zeros(max(1, n), dtype=dt)
    keep = [rec]
    for f in ("w", "scales", "xt", "q", "r", "y"):
        rec[f][:n] = [_ptr(getattr(x, f)) or 0 for x in sites]
    for f in ("w_bits", "M", "K", "N", "k_shift"):
        rec[f][:n] = [int(getattr(x, f)) for x in sites]
    dig = [x.w_digest for x in sites]
    if any(d is not None for d in dig):
        if any(d is not None and len(bytes(d)) != 64 for d in dig):
            raise ValueError("a weight digest is 64 bytes: D(W) || D(scales)")
        buf = C.create_string_buffer(b"".join(bytes(d) if d is not None else bytes(64) for d in dig), 64 * n)
        keep.append(buf)
        base = C.addressof(buf)
        rec["w_digest"][:n] = [base + 64 * i if d is not None else 0 for i, d in enumerate(dig)]
    return rec, keep


class SiteArray:
    """Sites marshalled once for the C ABI: the device pointers and sizes are read when it is
    built, so a proof that passes the same sites to several entry points reads them once. It
    behaves as the list of its sites; build a new one after changing a site."""

    def __init__(self, sites, _rec=None, _keep=None):
        self.sites = list(sites)
        if _rec is None:
            _rec, _keep = _site_records(self.sites)
        self.rec, self.keep = _rec, _keep
        self.arr = (_Site * len(_rec)).from_buffer(_rec)

    @staticmethod
    def concat(parts: Sequence["SiteArray"]) -> "SiteArray":
        import numpy as np
        parts = [p for p in parts if len(p)]
        if not parts:
            return SiteArray([])
        rec = np.zeros(sum(len(p) for p in parts), dtype=parts[0].rec.dtype)  # keeps _Site's padding
        o = 0
        for p in parts:
            rec[o:o + len(p)] = p.rec[: len(p)]
            o += len(p)
        return SiteArray([x for p in parts for x in p.sites], rec, [k for p in parts for k in p.keep] + [rec])

    def __len__(self):
        return len(self.sites)

    def __iter__(self):
        return iter(self.sites)

    def __getitem__(self, i):
        return self.sites[i]


def _as_array(sites) -> "SiteArray":
    return sites if isinstance(sites, SiteArray) else SiteArray(sites)


def _sites(sites: Sequence[SiteDesc]):
    sites = _as_array(sites)
    return sites.arr, [sites]


class Transcript:
    """Host Fiat-Shamir transcript (SHA-256), owned by the library."""

    def __init__(self, seed: int):
        self._L = lib()
        self.h = self._L.fp_tx_create(seed)

    def absorb(self, label: str, data: bytes):
        buf = C.create_string_buffer(bytes(data), max(1, len(data)))
        self._L.fp_tx_absorb(self.h, label.encode(), buf, len(data))

    def squeeze(self, label: str, n: int = 1) -> list:
        out = (C.c_uint64 * max(1, n))()
        self._L.fp_tx_squeeze(self.h, label.encode(), out, n)
        return list(out[:n])

    def state(self) -> bytes:
        out = C.create_string_buffer(32)
        self._L.fp_tx_state(self.h, out)
        return out.raw

    def close(self):
        if self.h:
            self._L.fp_tx_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Context:
    """A prover context on one CUDA device (scratch arenas, timing)."""

    def __init__(self, device: int = 0):
        self._L = lib()
        self.h = self._L.fp_ctx_create(device)
        if not self.h:
            raise FpError(-3, f"fp_ctx_create({device}) failed (no usable CUDA device?)")

    def _check(self, rc: int, what: str) -> int:
        if rc < 0:
            raise FpError(rc, f"{what}: {self._L.fp_last_error(self.h).decode()}")
        return rc

    def close(self):
        if self.h:
            self._L.fp_ctx_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def digest(self, dev, nbytes: int, stream=None) -> bytes:
        out = C.create_string_buffer(32)
        self._check(self._L.fp_digest(self.h, _ptr(dev), nbytes, out, _stream(stream)), "fp_digest")
        return out.raw

    def digest_many(self, bufs: Sequence, stream=None) -> bytes:
        """The digests of [(device buffer, nbytes), ...] in one pass, concatenated (32 bytes each)."""
        n = len(bufs)
        devs = (C.c_void_p * n)(*[_ptr(b) for b, _ in bufs])
        lens = (C.c_size_t * n)(*[int(m) for _, m in bufs])
        out = C.create_string_buffer(32 * n)
        self._check(self._L.fp_digests(self.h, devs, lens, n, out, _stream(stream)), "fp_digests")
        return out.raw

    def commit_witness(self, tx: Transcript, sites: Sequence[SiteDesc], stream=None):
        arr, keep = _sites(sites)
        self._check(self._L.fp_commit_witness(self.h, tx.h, arr, len(sites), _stream(stream)), "fp_commit_witness")

    def partial_eval(self, mat, bits: int, scales, rows: int, cols: int, point: Sequence[int], out, stream=None):
        pt = (C.c_uint64 * max(1, len(point)))(*[int(p) for p in point])
        self._check(self._L.mle_partial_eval(self.h, _ptr(mat), bits, _ptr(scales), rows, cols, pt, len(point),
                                             _ptr(out), _stream(stream)), "mle_partial_eval")

    def proof_size(self, sites: Sequence[SiteDesc]):
        arr, keep = _sites(sites)
        a, b = C.c_size_t(0), C.c_size_t(0)
        self._check(self._L.fp_proof_size(arr, len(sites), C.byref(a), C.byref(b)), "fp_proof_size")
        return a.value, b.value

    def prove_matmul(self, tx: Transcript, sites: Sequence[SiteDesc], stream=None) -> bytes:
        sites = _as_array(sites)
        arr, keep = _sites(sites)
        mm, _ = self.proof_size(sites)
        buf = C.create_string_buffer(max(1, mm))
        n = C.c_size_t(mm)
        self._check(self._L.sumcheck_prove_matmul(self.h, tx.h, arr, len(sites), buf, C.byref(n), _stream(stream)),
                    "sumcheck_prove_matmul")
        return buf.raw[: n.value]

    def commit_witness_shard(self, tx: Transcript, sites: Sequence[SiteDesc], shard: Shard, stream=None):
        """fp_commit_witness for this rank's sites of a shared statement; every rank absorbs
        all site records. Only this rank's sites need device tensors."""
        arr, keep = _sites(sites)
        self._check(self._L.fp_commit_witness_shard(self.h, tx.h, arr, len(sites), C.byref(shard.c),
                                                    _stream(stream)), "fp_commit_witness_shard")

    def prove_matmul_shard(self, tx: Transcript, sites: Sequence[SiteDesc], shard: Shard, stream=None) -> bytes:
        """The matmul sum-check of a shared statement: this rank's sites on this GPU, the
        round sums exchanged; every rank returns the one-rank proof bytes."""
        sites = _as_array(sites)
        arr, keep = _sites(sites)
        mm, _ = self.proof_size(sites)
        buf = C.create_string_buffer(max(1, mm))
        n = C.c_size_t(mm)
        self._check(self._L.sumcheck_prove_matmul_shard(self.h, tx.h, arr, len(sites), C.byref(shard.c), buf,
                                                        C.byref(n), _stream(stream)), "sumcheck_prove_matmul_shard")
        return buf.raw[: n.value]

    def prove_hadamard(self, tx: Transcript, s, u, stream=None) -> bytes:
        """Sum-check proof for the gated product of two device int8 tensors of equal size
        (flattened row-major); continues tx."""
        n = int(s.numel())
        if int(u.numel()) != n:
            raise ValueError("prove_hadamard: s and u differ in size")
        v = 0
        while (1 << v) < n:
            v += 1
        cap = 8 + 32 * v + 16
        buf = C.create_string_buffer(cap)
        ln = C.c_size_t(cap)
        self._check(self._L.sumcheck_prove_hadamard(self.h, tx.h, _ptr(s), _ptr(u), n, buf, C.byref(ln),
                                                    _stream(stream)), "sumcheck_prove_hadamard")
        return buf.raw[: ln.value]

    def prove_hadamard_ext2(self, tx: Transcript, s, u, stream=None) -> bytes:
        """As prove_hadamard, with every challenge and every value sent in the quadratic
        extension F_p[phi]/(phi^2 - 7) (16 bytes each); continues tx."""
        n = int(s.numel())
        if int(u.numel()) != n:
            raise ValueError("prove_hadamard_ext2: s and u differ in size")
        v = 0
        while (1 << v) < n:
            v += 1
        cap = 16 + 64 * v + 32
        buf = C.create_string_buffer(cap)
        ln = C.c_size_t(cap)
        self._check(self._L.sumcheck_prove_hadamard_ext2(self.h, tx.h, _ptr(s), _ptr(u), n, buf, C.byref(ln),
                                                         _stream(stream)), "sumcheck_prove_hadamard_ext2")
        return buf.raw[: ln.value]

    def prove_matmul_ext2(self, tx: Transcript, site: "SiteDesc", stream=None) -> bytes:
        """The matmul sum-check of one committed site with every challenge and value in the
        quadratic extension F_p[phi]/(phi^2 - 7); continues tx."""
        arr, keep = _sites([site])
        n = 0
        while (1 << n) < int(site.K):
            n += 1
        cap = 16 + 48 * n + 32
        buf = C.create_string_buffer(cap)
        ln = C.c_size_t(cap)
        self._check(self._L.sumcheck_prove_matmul_ext2(self.h, tx.h, arr, buf, C.byref(ln), _stream(stream)),
                    "sumcheck_prove_matmul_ext2")
        return buf.raw[: ln.value]

    def prove_freivalds(self, tx: Transcript, site: "SiteDesc", stream=None) -> bytes:
        """Freivalds' check of one committed site, the prover's side: u = X rho^(.) (K field
        elements); continues tx."""
        arr, keep = _sites([site])
        cap = 8 * int(site.K)
        buf = C.create_string_buffer(cap)
        ln = C.c_size_t(cap)
        self._check(self._L.freivalds_prove_matmul(self.h, tx.h, arr, buf, C.byref(ln), _stream(stream)),
                    "freivalds_prove_matmul")
        return buf.raw[: ln.value]

    def prove_routing(self, tx: Transcript, logits, T: int, E: int, H, D, stream=None):
        """Top-1 routing proof of the device int8 router logits (T x E, token-major): writes the
        committed choice H (T x E uint8) and differences D (T x E int32) into the given device
        tensors and returns (proof bytes, status); continues tx."""
        vT = 0
        while (1 << vT) < T:
            vT += 1
        vE = 0
        while (1 << vE) < E:
            vE += 1
        v = 0
        while (1 << v) < T * E:
            v += 1
        v = max(v, 1)
        cap = 16 + 32 * (vT + vE) + 16 + 4 * 256 + 8 + 32 * v + 16
        buf = C.create_string_buffer(cap)
        ln = C.c_size_t(cap)
        rc = self._check(self._L.sumcheck_prove_routing(self.h, tx.h, _ptr(logits), T, E, _ptr(H), _ptr(D), buf,
                                                        C.byref(ln), _stream(stream)), "sumcheck_prove_routing")
        return buf.raw[: ln.value], rc

    def prove_logup_ext2(self, tx: Transcript, sites: Sequence["SiteDesc"], stream=None):
        """The rescale LogUp of the committed sites' keys with every challenge and value in the
        quadratic extension; returns (proof bytes, status: 1 if some key lies outside its table)."""
        arr, keep = _sites(sites)
        nk = sum(int(s.M) * int(s.N) for s in sites)
        v = 0
        while (1 << v) < nk:
            v += 1
        v = max(v, 1)
        k = int(sites[0].k_shift)
        cap = 4 * (1 << k) + 4 * 65536 + 128 + 48 + sum(64 * d + 128 for d in range(1, v))
        buf = C.create_string_buffer(cap)
        ln = C.c_size_t(cap)
        rc = self._check(self._L.logup_prove_rescale_ext2(self.h, tx.h, arr, len(sites), buf, C.byref(ln),
                                                          _stream(stream)), "logup_prove_rescale_ext2")
        return buf.raw[: ln.value], rc

    def prove_helper_inverse_ext2(self, tx: Transcript, r, k: int, stream=None):
        """As prove_helper_inverse with every challenge and value in the quadratic extension."""
        n = int(r.numel())
        v = 0
        while (1 << v) < n:
            v += 1
        v = max(v, 1)
        cap = 4 * (1 << k) + 16 + 64 * v + 32
        buf = C.create_string_buffer(cap)
        ln = C.c_size_t(cap)
        rc = self._check(self._L.logup_prove_helper_inverse_ext2(self.h, tx.h, _ptr(r), n, k, buf, C.byref(ln),
                                                                 _stream(stream)), "logup_prove_helper_inverse_ext2")
        return buf.raw[: ln.value], rc

    def prove_helper_inverse(self, tx: Transcript, r, k: int, stream=None):
        """Helper-inverse LogUp proof that every entry of the device int32 tensor r lies in
        the remainder table R_k; continues tx. Returns (proof bytes, status): status 1 means
        some key lies outside the table."""
        n = int(r.numel())
        v = 0
        while (1 << v) < n:
            v += 1
        v = max(v, 1)
        cap = 4 * (1 << k) + 8 + 32 * v + 16
        buf = C.create_string_buffer(cap)
        ln = C.c_size_t(cap)
        rc = self._check(self._L.logup_prove_helper_inverse(self.h, tx.h, _ptr(r), n, k, buf, C.byref(ln),
                                                            _stream(stream)), "logup_prove_helper_inverse")
        return buf.raw[: ln.value], rc

    def reduce_scales(self, tx: Transcript, w, bits: int, scales, M: int, K: int, point: Sequence[int],
                      stream=None, w_digest: Optional[bytes] = None) -> bytes:
        """Sum-check reducing a claim on the scaled weights' MLE at point (row coordinates
        first) to claims on the weights w and the per-64-column scales (device tensors).
        w_digest: D(W) || D(S) when the weights were committed in advance (64 bytes), else
        they are digested here."""
        if w_digest is not None and len(bytes(w_digest)) != 64:
            raise ValueError("reduce_scales: w_digest is 64 bytes, D(W) || D(S)")
        dg = C.create_string_buffer(bytes(w_digest), 64) if w_digest is not None else None
        v = 0
        while (1 << v) < M:
            v += 1
        vk = 0
        while (1 << vk) < K:
            vk += 1
        v += vk
        if len(point) != v:
            raise ValueError(f"reduce_scales: the point needs {v} coordinates")
        pt = (C.c_uint64 * max(1, v))(*[int(p) for p in point])
        cap = 8 + 32 * v + 16
        buf = C.create_string_buffer(cap)
        ln = C.c_size_t(cap)
        self._check(self._L.sumcheck_reduce_scales(self.h, tx.h, _ptr(w), bits, _ptr(scales), M, K, pt, dg, buf,
                                                   C.byref(ln), _stream(stream)), "sumcheck_reduce_scales")
        return buf.raw[: ln.value]

    def silu_inputs(self, y, g, s, s8, stream=None) -> None:
        """g = y (int16), s = silu_q(y) (int16), s8 = s (int8) for the device int8 tensor y
        (the gate projection's outputs); the caller's device buffers of y's size."""
        self._check(self._L.fp_silu_inputs(self.h, _ptr(y), int(y.numel()), _ptr(g), _ptr(s), _ptr(s8),
                                           _stream(stream)), "fp_silu_inputs")

    def ffn_hidden(self, s8, u, kh: int, q, r, y, stream=None) -> None:
        """The FFN's hidden activations rescaled by 2^kh: h = s8 u, q = floor((h + 2^(kh-1)) /
        2^kh), r = h - 2^kh q (int32), y = clamp(q) (int8), for the device int8 tensors s8 (SiLU
        outputs) and u (up outputs) of one shape; the caller's device buffers of that size."""
        if s8.numel() != u.numel() or q.numel() != s8.numel() or r.numel() != s8.numel() or y.numel() != s8.numel():
            raise ValueError("ffn_hidden: buffers differ in size")
        self._check(self._L.fp_ffn_hidden(self.h, _ptr(s8), _ptr(u), int(s8.numel()), kh, _ptr(q), _ptr(r),
                                          _ptr(y), _stream(stream)), "fp_ffn_hidden")

    def last_point(self):
        """(r_row, rho) of the last matmul section proven with this context (host integers)."""
        vr, n = C.c_int32(0), C.c_int32(0)
        self._check(self._L.sumcheck_last_point(self.h, None, 0, C.byref(vr), None, 0, C.byref(n)),
                    "sumcheck_last_point")
        rr = (C.c_uint64 * max(1, vr.value))()
        rho = (C.c_uint64 * max(1, n.value))()
        self._check(self._L.sumcheck_last_point(self.h, rr, vr.value, C.byref(vr), rho, n.value, C.byref(n)),
                    "sumcheck_last_point")
        return list(rr[: vr.value]), list(rho[: n.value])

    def prove_silu(self, tx: Transcript, g, s, stream=None) -> bytes:
        """LogUp proof that every entry of the device int16 tensor s is the SiLU table's entry
        for the same entry of g (flattened row-major); continues tx."""
        return self._lookup16(self._L.logup_prove_silu, "prove_silu", tx, g, s, stream)

    def prove_exp(self, tx: Transcript, g, s, stream=None) -> bytes:
        """As prove_silu, for the softmax numerator table."""
        return self._lookup16(self._L.logup_prove_exp, "prove_exp", tx, g, s, stream)

    def prove_silu_ext2(self, tx: Transcript, g, s, stream=None) -> bytes:
        """As prove_silu with every challenge and value in the quadratic extension."""
        return self._lookup16(self._L.logup_prove_silu_ext2, "prove_silu_ext2", tx, g, s, stream, ext=True)

    def prove_exp_ext2(self, tx: Transcript, g, s, stream=None) -> bytes:
        """As prove_exp with every challenge and value in the quadratic extension."""
        return self._lookup16(self._L.logup_prove_exp_ext2, "prove_exp_ext2", tx, g, s, stream, ext=True)

    def _lookup16(self, fn, what, tx, g, s, stream, ext=False):
        n = int(g.numel())
        if int(s.numel()) != n:
            raise ValueError(f"{what}: g and s differ in size")
        v = 0
        while (1 << v) < n:
            v += 1
        v = max(v, 1)
        w = 2 if ext else 1  # words per value
        cap = 4 * 65536 + w * (32 + 16) + sum(w * (32 * d + 32) for d in range(1, v))
        buf = C.create_string_buffer(cap)
        ln = C.c_size_t(cap)
        self._check(fn(self.h, tx.h, _ptr(g), _ptr(s), n, buf, C.byref(ln), _stream(stream)), what)
        return buf.raw[: ln.value]

    def prove_logup(self, tx: Transcript, sites: Sequence[SiteDesc], stream=None):
        """Returns (proof bytes, status): status 1 means some key lies outside its table."""
        sites = _as_array(sites)
        arr, keep = _sites(sites)
        _, lu = self.proof_size(sites)
        buf = C.create_string_buffer(max(1, lu))
        n = C.c_size_t(lu)
        rc = self._check(self._L.logup_prove_rescale(self.h, tx.h, arr, len(sites), buf, C.byref(n),
                                                     _stream(stream)), "logup_prove_rescale")
        return buf.raw[: n.value], rc

    def prove_logup_hi(self, tx: Transcript, sites: Sequence[SiteDesc], stream=None):
        """The lookup section in the helper-inverse form (logup_prove_rescale_hi). Returns (proof
        bytes, status): status 1 means some key lies outside its table."""
        arr, keep = _sites(sites)
        n = C.c_size_t(0)
        self._L.logup_prove_rescale_hi(self.h, tx.h, arr, len(sites), None, C.byref(n), _stream(stream))
        buf = C.create_string_buffer(max(1, n.value))
        rc = self._check(self._L.logup_prove_rescale_hi(self.h, tx.h, arr, len(sites), buf, C.byref(n),
                                                        _stream(stream)), "logup_prove_rescale_hi")
        return buf.raw[: n.value], rc

    def prove_dispatch(self, tx: Transcript, X, e, D, E: int, stream=None) -> bytes:
        """The MoE dispatch proof: X (T x K int8, the layer input), e (T int32 experts) and D
        (T x K int8, the experts' inputs stacked expert by expert), device tensors; continues tx."""
        T, K = int(X.shape[0]), int(X.shape[1])
        n = C.c_size_t(0)
        self._L.sumcheck_prove_dispatch(self.h, tx.h, _ptr(X), _ptr(e), _ptr(D), T, K, E, None, C.byref(n),
                                        _stream(stream))
        buf = C.create_string_buffer(max(1, n.value))
        self._check(self._L.sumcheck_prove_dispatch(self.h, tx.h, _ptr(X), _ptr(e), _ptr(D), T, K, E, buf, C.byref(n),
                                                    _stream(stream)), "sumcheck_prove_dispatch")
        return buf.raw[: n.value]

    def set_profiling(self, on):
        """False/0: off; True/1: one launch per sum-check round, each timed; 2: time the
        production (resident) launches as they run."""
        level = 2 if on == 2 else (1 if on else 0)
        self._check(self._L.fp_ctx_set_profiling(self.h, level), "fp_ctx_set_profiling")

    def session_selftest(self, stream=None) -> int:
        """Run the bounded-wait self-test; returns the status code (FP_ERR_TIMEOUT = -4 expected)."""
        return int(self._L.fp_session_selftest(self.h, _stream(stream)))

    def host_stats(self):
        """(waits for a device result, seconds spent waiting, seconds from results to the
        next posted challenge, longest such turnaround) since the context was created."""
        out = (C.c_double * 4)()
        self._check(self._L.fp_host_stats(self.h, out), "fp_host_stats")
        return int(out[0]), float(out[1]), float(out[2]), float(out[3])

    def launches(self) -> int:
        """Kernels launched by the library on this context so far."""
        return int(self._L.fp_ctx_launches(self.h))

    def kernel_log(self) -> list:
        """[(kernel name, device ms, algorithmic bytes, start ms from the first timed launch)] per
        timed launch, in launch order."""
        n = self._check(self._L.fp_kernel_log(self.h, None, 0), "fp_kernel_log")
        arr = (_LRec * max(1, n))()
        n = self._check(self._L.fp_kernel_log(self.h, arr, n), "fp_kernel_log")
        return [(self._L.fp_kernel_name(r.kernel).decode(), r.ms, r.bytes, r.start_ms) for r in arr[:n]]

    def kernel_stats(self) -> dict:
        """{kernel name: (launches, total ms, algorithmic bytes)} since the last reset."""
        cap = 64
        arr = (_KStat * cap)()
        n = self._check(self._L.fp_kernel_stats(self.h, arr, cap), "fp_kernel_stats")
        out = {}
        for i in range(min(n, cap)):
            out[self._L.fp_kernel_name(arr[i].kernel).decode()] = (arr[i].launches, arr[i].ms, arr[i].bytes)
        return out


def prove(ctx: Context, seed: int, stages: Sequence[Sequence[SiteDesc]], stream=None, lookup: str = "gkr"):
    """Prove a layer: commit every stage's witness in order (a later stage may read
    an earlier stage's outputs), then the batched matmul sum-check over all sites,
    then the LogUp rescale/clamp proof, as the fraction tree (lookup="gkr") or by
    helper inverses (lookup="hi"). Returns (proof bytes, transcript states after
    commit / matmul / lookup, lookup status)."""
    if lookup not in ("gkr", "hi"):
        raise ValueError("prove: lookup must be 'gkr' or 'hi'")
    tx = Transcript(seed)
    try:
        parts = [SiteArray(st) for st in stages]
        for st in parts:
            ctx.commit_witness(tx, st, stream)
        sites = SiteArray.concat(parts)
        s0 = tx.state()
        mm = ctx.prove_matmul(tx, sites, stream)
        s1 = tx.state()
        lu, status = (ctx.prove_logup if lookup == "gkr" else ctx.prove_logup_hi)(tx, sites, stream)
        return mm + lu, [s0, s1, tx.state()], status
    finally:
        tx.close()


def _log2c(x: int) -> int:
    v = 0
    while (1 << v) < x:
        v += 1
    return v


def prove_ffn(ctx: Context, seed: int, stages: Sequence[Sequence[SiteDesc]], gate: int = 0, up: int = 1,
              down: int = 2, kh: int = 7, stream=None):
    """Prove an FFN layer ("How fast can FlashProve go", 3.1) as one statement on one
    transcript: the layer proof of prove(), its down site reading the layer's own hidden
    activations; the per-group scale reduction of every site with scales, at the point where
    the matmul section left its weights (r_row's first ceil(log2 M) coordinates, the last
    ceil(log2 K) round challenges); the commitment of the hidden rescale (q_h, r_h, y_h of
    SiLU(gate) * up by 2^kh) and its lookup section (r_h in R_kh, y_h = clamp(q_h)); the SiLU
    lookup with the gate site's outputs as its inputs; the gated product of the SiLU outputs
    with the up site's outputs. gate, up and down index the sites in stage order; the down
    site sits in a later stage than gate and up, and its xt buffer (N x M_gate int8) receives
    y_h before its stage is committed. Returns (proof bytes, transcript state after, lookup
    status)."""
    import torch
    sites = [s for st in stages for s in st]
    g_site, u_site, d_site = sites[gate], sites[up], sites[down]
    if (g_site.M, g_site.N) != (u_site.M, u_site.N):
        raise ValueError("prove_ffn: the gate and up sites differ in shape")
    if (d_site.K, d_site.N) != (g_site.M, g_site.N) or d_site.xt.numel() != g_site.M * g_site.N:
        raise ValueError("prove_ffn: the down site does not read the gate's M x N outputs")
    stage_of = {id(s): i for i, st in enumerate(stages) for s in st}
    if stage_of[id(d_site)] <= max(stage_of[id(g_site)], stage_of[id(u_site)]):
        raise ValueError("prove_ffn: the down site must sit in a later stage than gate and up")
    y = g_site.y
    dev = y.device
    g = torch.empty(y.shape, dtype=torch.int16, device=dev)
    s = torch.empty(y.shape, dtype=torch.int16, device=dev)
    s8 = torch.empty(y.shape, dtype=torch.int8, device=dev)
    qh = torch.empty(y.shape, dtype=torch.int32, device=dev)
    rh = torch.empty(y.shape, dtype=torch.int32, device=dev)
    yh = d_site.xt
    n = y.numel()
    tx = Transcript(seed)
    try:
        hidden = False
        arrays = [SiteArray(st) for st in stages]
        for i, st in enumerate(arrays):
            if not hidden and i == stage_of[id(d_site)]:
                ctx.silu_inputs(y, g, s, s8, stream)
                ctx.ffn_hidden(s8, u_site.y, kh, qh, rh, yh, stream)
                hidden = True
            ctx.commit_witness(tx, st, stream)
        sites = SiteArray.concat(arrays)
        parts = [ctx.prove_matmul(tx, sites, stream)]
        lu, status = ctx.prove_logup(tx, sites, stream)
        parts.append(lu)
        r_row, rho = ctx.last_point()
        nr = len(rho)
        for d in sites:
            if d.scales is None:
                continue
            vm, vk = _log2c(d.M), _log2c(d.K)
            parts.append(ctx.reduce_scales(tx, d.w, d.w_bits, d.scales, d.M, d.K, r_row[:vm] + rho[nr - vk:], stream,
                                           w_digest=d.w_digest))
        tx.absorb("ffn_hidden", ctx.digest_many([(qh, 4 * n), (rh, 4 * n), (yh, n)], stream))
        # the hidden rescale's keys as a lookup section's single site (M x N keys, table R_kh);
        # w and xt only satisfy the site checks, the lookup reads q, r and y
        hs = SiteDesc(w=s8, scales=None, xt=u_site.y, q=qh, r=rh, y=yh, M=g_site.M, K=1, N=g_site.N,
                      w_bits=8, k_shift=kh)
        lu_h, _ = ctx.prove_logup(tx, [hs], stream)
        parts.append(lu_h)
        parts.append(ctx.prove_silu(tx, g, s, stream))
        parts.append(ctx.prove_hadamard(tx, s8, u_site.y, stream))
        return b"".join(parts), tx.state(), status
    finally:
        tx.close()


def prove_shard(ctx: Context, seed: int, sites: Sequence[SiteDesc], shard: Shard, gather_witness, stream=None):
    """Prove one layer statement shared among ranks (one stage, sites independent): this
    rank commits and folds its own sites, the ranks exchange the round sums, then
    gather_witness(sites) -> sites with every site's q, r, y on this device, and the
    lookup section runs over all keys. Every rank returns the one-rank proof, states and
    status."""
    tx = Transcript(seed)
    try:
        sa = SiteArray(sites)
        ctx.commit_witness_shard(tx, sa, shard, stream)
        s0 = tx.state()
        mm = ctx.prove_matmul_shard(tx, sa, shard, stream)
        s1 = tx.state()
        full = gather_witness(list(sites))
        lu, status = ctx.prove_logup(tx, SiteArray(full), stream)
        return mm + lu, [s0, s1, tx.state()], status
    finally:
        tx.close()


def torch_gather_witness(shard: Shard, group=None):
    """gather_witness for prove_shard over a torch.distributed group whose backend moves
    device tensors (NCCL): every rank's q, r, y, concatenated per rank, all-gathered into
    fresh device buffers, and the sites pointed at them."""
    import torch
    import torch.distributed as td

    def gather(sites):
        dev = next(s.q for s in sites[shard.site_lo[shard.rank]:shard.site_lo[shard.rank + 1]]).device
        sizes = [sum(sites[i].M * sites[i].N for i in range(shard.site_lo[r], shard.site_lo[r + 1]))
                 for r in range(shard.world)]
        most = max(sizes)
        mine_qr = torch.zeros(2 * most, dtype=torch.int32, device=dev)
        mine_y = torch.zeros(max(1, most), dtype=torch.int8, device=dev)
        o = 0
        for i in shard.own:
            n = sites[i].M * sites[i].N
            mine_qr[o:o + n] = sites[i].q.reshape(-1)
            mine_qr[most + o:most + o + n] = sites[i].r.reshape(-1)
            mine_y[o:o + n] = sites[i].y.reshape(-1)
            o += n
        all_qr = torch.empty(shard.world * 2 * most, dtype=torch.int32, device=dev)
        all_y = torch.empty(shard.world * max(1, most), dtype=torch.int8, device=dev)
        td.all_gather_into_tensor(all_qr, mine_qr, group=group)
        td.all_gather_into_tensor(all_y, mine_y, group=group)
        out = []
        for r in range(shard.world):
            o = 0
            for i in range(shard.site_lo[r], shard.site_lo[r + 1]):
                s = sites[i]
                n = s.M * s.N
                base = r * 2 * most
                d = SiteDesc(s.w, s.xt, all_qr[base + o:base + o + n].view(s.N, s.M),
                             all_qr[base + most + o:base + most + o + n].view(s.N, s.M),
                             all_y[r * max(1, most) + o:r * max(1, most) + o + n].view(s.N, s.M),
                             s.M, s.K, s.N, s.w_bits, s.k_shift, s.scales, s.w_digest)
                out.append(d)
                o += n
        return out

    return gather


def silu_table():
    """The SiLU table's 2^16 entries (inputs -2^15 .. 2^15 - 1), as the library computes them."""
    import numpy as np
    out = np.zeros(65536, dtype=np.int32)
    rc = lib().fp_silu_table(out.ctypes.data)
    if rc != 0:
        raise FpError(rc, "fp_silu_table")
    return out


def exp_table():
    """The softmax numerator table's 2^16 entries, as the library computes them."""
    import numpy as np
    out = np.zeros(65536, dtype=np.int32)
    rc = lib().fp_exp_table(out.ctypes.data)
    if rc != 0:
        raise FpError(rc, "fp_exp_table")
    return out
