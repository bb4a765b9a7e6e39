"""CPU oracle for the quantised-matmul sum-check prover -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may import this package. The product path (the CUDA library
and its binding in ``sum_check_prover_b200``) never imports it and shares no
code with it.

The arithmetic lives in ``oracle.c`` (plain C, single-threaded, every field
operation an ``unsigned __int128`` product or sum reduced with ``% P``). This
module only builds that file with gcc and marshals numpy arrays through
ctypes. The one piece of logic here is wiring a workload's linked sites
(an operand that is another site's output) on the host.
"""

from __future__ import annotations

import ctypes as C
import os
import subprocess
from pathlib import Path

import numpy as np

P = 0xFFFFFFFF00000001
_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "oracle.c"
_LIB = _HERE / "liboracle.so"
_lib = None

REASONS = {
    0: "accept",
    1: "format",
    2: "claim",
    3: "mm_round",
    4: "mm_final",
    5: "mm_A",
    6: "mm_B",
    7: "root_rem",
    8: "root_clamp",
    9: "gkr_round",
    10: "gkr_final",
    11: "leaf_P",
    12: "leaf_Q",
    13: "leaf_open",
    14: "args",
    15: "had_claim",
    16: "had_round",
    17: "had_final",
    18: "had_open",
    19: "scl_claim",
    20: "scl_round",
    21: "scl_final",
    22: "scl_open",
    23: "lookup_root",
    24: "lookup_round",
    25: "lookup_final",
    26: "lookup_leaf",
    27: "lookup_open",
    32: "frv_u",
    33: "frv_row",
    28: "lhi_sum",
    29: "lhi_round",
    30: "lhi_final",
    31: "lhi_open",
    34: "route_open",
    35: "route_round",
    36: "route_final",
    37: "lhi2_sum",
    38: "lhi2_round",
    39: "lhi2_final",
    40: "lhi2_open",
    41: "lhr_sum",
    42: "lhr_round",
    43: "lhr_final",
    44: "lhr_open",
    45: "dsp_claim",
    46: "dsp_round",
    47: "dsp_final",
    48: "dsp_open",
    49: "ffn_link",
    50: "ffn_hidden",
    51: "ffn_down",
}


def build(force: bool = False) -> Path:
    """Compile oracle.c into liboracle.so with gcc (no GPU needed)."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(f".so.{os.getpid()}")
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", str(tmp), str(_SRC), "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Site(C.Structure):
    _fields_ = [("w", C.c_void_p), ("scales", C.c_void_p), ("xt", C.c_void_p),
                ("w_bits", C.c_int32), ("M", C.c_int32), ("K", C.c_int32), ("N", C.c_int32),
                ("k_shift", C.c_int32), ("pad", C.c_int32)]


class _Wit(C.Structure):
    _fields_ = [("q", C.c_void_p), ("r", C.c_void_p), ("y", C.c_void_p)]


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(str(_LIB))
        u64, vp = C.c_uint64, C.c_void_p
        for nm in ("orc_fadd", "orc_fsub", "orc_fmul", "orc_fpow"):
            getattr(L, nm).restype = u64
            getattr(L, nm).argtypes = [u64, u64]
        L.orc_finv.restype = u64
        L.orc_finv.argtypes = [u64]
        L.orc_fint.restype = u64
        L.orc_fint.argtypes = [C.c_int64]
        L.orc_sha256.argtypes = [vp, u64, vp]
        L.orc_tree_digest.argtypes = [vp, u64, vp]
        L.orc_tx_new.restype = vp
        L.orc_tx_new.argtypes = [u64]
        L.orc_tx_free.argtypes = [vp]
        L.orc_tx_state.argtypes = [vp, vp]
        L.orc_tx_absorb_h.argtypes = [vp, C.c_char_p, vp, u64]
        L.orc_tx_squeeze_h.restype = u64
        L.orc_tx_squeeze_h.argtypes = [vp, C.c_char_p]
        L.orc_eq_table.argtypes = [vp, C.c_int, vp]
        L.orc_mle_eval.restype = u64
        L.orc_mle_eval.argtypes = [vp, u64, vp, C.c_int]
        L.orc_lagrange.restype = u64
        L.orc_lagrange.argtypes = [vp, C.c_int, u64]
        L.orc_witness.restype = C.c_int
        L.orc_witness.argtypes = [C.POINTER(_Site), vp, vp, vp]
        L.orc_partial_w.argtypes = [C.POINTER(_Site), vp, C.c_int, vp]
        L.orc_partial_x.argtypes = [C.POINTER(_Site), vp, C.c_int, vp]
        L.orc_partial_rows.argtypes = [vp, C.c_int, vp, C.c_int, C.c_int, vp, C.c_int, vp]
        L.orc_claim.restype = u64
        L.orc_claim.argtypes = [vp, vp, C.c_int, C.c_int, C.c_int, vp, C.c_int, vp, C.c_int]
        L.orc_prove.restype = C.c_int
        L.orc_prove.argtypes = [u64, C.POINTER(_Site), C.c_int, C.POINTER(_Wit), vp, u64,
                                C.POINTER(u64), vp, C.POINTER(u64)]
        L.orc_verify.restype = C.c_int
        L.orc_verify.argtypes = [u64, C.POINTER(_Site), C.c_int, C.POINTER(_Wit), vp, u64, vp]
        L.orc_verify_opts.restype = C.c_int
        L.orc_verify_opts.argtypes = [u64, C.POINTER(_Site), C.c_int, C.POINTER(_Wit), vp, u64, vp, vp, C.c_int]
        L.orc_prove_hi.argtypes = [u64, C.POINTER(_Site), C.c_int, C.POINTER(_Wit), vp, u64,
                                   C.POINTER(u64), vp, C.POINTER(u64)]
        L.orc_verify_hi.argtypes = [u64, C.POINTER(_Site), C.c_int, C.POINTER(_Wit), vp, u64, vp]
        L.orc_prove_ffn.restype = C.c_int
        L.orc_prove_ffn.argtypes = [u64, C.POINTER(_Site), C.c_int, C.POINTER(_Wit), C.c_int, C.c_int, C.c_int,
                                    C.c_int, vp, vp, vp, vp, vp, u64, C.POINTER(u64), vp]
        L.orc_verify_ffn.restype = C.c_int
        L.orc_verify_ffn.argtypes = [u64, C.POINTER(_Site), C.c_int, C.POINTER(_Wit), C.c_int, C.c_int, C.c_int,
                                     C.c_int, vp, vp, vp, vp, vp, u64, vp]
        L.orc_ffn_hidden.restype = C.c_int
        L.orc_ffn_hidden.argtypes = [vp, vp, u64, C.c_int, vp, vp, vp]
        L.orc_dsp_prove.restype = C.c_int
        L.orc_dsp_prove.argtypes = [vp, vp, vp, vp, u64, u64, C.c_int, vp, u64, C.POINTER(u64)]
        L.orc_dsp_verify.restype = C.c_int
        L.orc_dsp_verify.argtypes = [vp, vp, vp, vp, u64, u64, C.c_int, vp, u64, vp]
        L.orc_had_prove.restype = C.c_int
        L.orc_had_prove.argtypes = [vp, vp, vp, u64, vp, u64, C.POINTER(u64)]
        L.orc_had_verify.restype = C.c_int
        L.orc_had_verify.argtypes = [vp, vp, vp, u64, vp, u64, vp]
        L.orc_scl_prove.restype = C.c_int
        L.orc_scl_prove.argtypes = [vp, vp, C.c_int, vp, C.c_int, C.c_int, vp, vp, u64, C.POINTER(u64)]
        L.orc_scl_verify.restype = C.c_int
        L.orc_scl_verify.argtypes = [vp, vp, C.c_int, vp, C.c_int, C.c_int, vp, vp, u64, vp]
        L.orc_silu_q.restype = C.c_int32
        L.orc_silu_q.argtypes = [C.c_int32]
        L.orc_silu_prove.restype = C.c_int
        L.orc_silu_prove.argtypes = [vp, vp, vp, u64, vp, u64, C.POINTER(u64)]
        L.orc_silu_verify.restype = C.c_int
        L.orc_silu_verify.argtypes = [vp, vp, vp, u64, vp, u64, vp]
        L.orc_exp_q.restype = C.c_int32
        L.orc_exp_q.argtypes = [C.c_int32]
        L.orc_exp_prove.restype = C.c_int
        L.orc_exp_prove.argtypes = [vp, vp, vp, u64, vp, u64, C.POINTER(u64)]
        L.orc_exp_verify.restype = C.c_int
        L.orc_exp_verify.argtypes = [vp, vp, vp, u64, vp, u64, vp]
        for nm in ("orc_silu2_prove", "orc_exp2_prove"):
            getattr(L, nm).restype = C.c_int
            getattr(L, nm).argtypes = [vp, vp, vp, u64, vp, u64, C.POINTER(u64)]
        for nm in ("orc_silu2_verify", "orc_exp2_verify"):
            getattr(L, nm).restype = C.c_int
            getattr(L, nm).argtypes = [vp, vp, vp, u64, vp, u64, vp]
        L.orc_lhi_prove.restype = C.c_int
        L.orc_lhi_prove.argtypes = [vp, vp, u64, C.c_int, vp, u64, C.POINTER(u64)]
        L.orc_lhi_verify.restype = C.c_int
        L.orc_lhi_verify.argtypes = [vp, vp, u64, C.c_int, vp, u64, vp]
        L.orc_e2_mul.argtypes = [vp, vp, vp]
        L.orc_e2_inv.argtypes = [vp, vp]
        L.orc_had2_prove.restype = C.c_int
        L.orc_had2_prove.argtypes = [vp, vp, vp, u64, vp, u64, C.POINTER(u64)]
        L.orc_had2_verify.restype = C.c_int
        L.orc_had2_verify.argtypes = [vp, vp, vp, u64, vp, u64, vp]
        L.orc_frv_prove.restype = C.c_int
        L.orc_frv_prove.argtypes = [vp, C.POINTER(_Site), C.POINTER(_Wit), vp, u64, C.POINTER(u64)]
        L.orc_frv_verify.restype = C.c_int
        L.orc_frv_verify.argtypes = [vp, C.POINTER(_Site), C.POINTER(_Wit), vp, u64, vp]
        for nm in ("orc_lhi2_prove",):
            getattr(L, nm).restype = C.c_int
            getattr(L, nm).argtypes = [vp, vp, u64, C.c_int, vp, u64, C.POINTER(u64)]
        L.orc_lhi2_verify.restype = C.c_int
        L.orc_lhi2_verify.argtypes = [vp, vp, u64, C.c_int, vp, u64, vp]
        L.orc_lu2_prove.restype = C.c_int
        L.orc_lu2_prove.argtypes = [vp, vp, C.c_int, vp, vp, u64, C.POINTER(u64)]
        L.orc_lu2_verify.restype = C.c_int
        L.orc_lu2_verify.argtypes = [vp, vp, C.c_int, vp, vp, u64, vp]
        L.orc_route_witness.restype = None
        L.orc_route_witness.argtypes = [vp, u64, C.c_int, vp, vp]
        L.orc_route_prove.restype = C.c_int
        L.orc_route_prove.argtypes = [vp, vp, vp, vp, u64, C.c_int, vp, u64, C.POINTER(u64)]
        L.orc_route_verify.restype = C.c_int
        L.orc_route_verify.argtypes = [vp, vp, vp, vp, u64, C.c_int, vp, u64, vp]
        L.orc_mm2_prove.restype = C.c_int
        L.orc_mm2_prove.argtypes = [vp, C.POINTER(_Site), C.POINTER(_Wit), vp, u64, C.POINTER(u64)]
        L.orc_mm2_verify.restype = C.c_int
        L.orc_mm2_verify.argtypes = [vp, C.POINTER(_Site), C.POINTER(_Wit), vp, u64, vp]
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _u64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.uint64))


def log2_ceil(n: int) -> int:
    v = 0
    while (1 << v) < n:
        v += 1
    return v


# ---- primitives -----------------------------------------------------------

def fadd(a, b): return lib().orc_fadd(a, b)
def fsub(a, b): return lib().orc_fsub(a, b)
def fmul(a, b): return lib().orc_fmul(a, b)
def fpow(a, e): return lib().orc_fpow(a, e)
def finv(a): return lib().orc_finv(a)
def fint(v): return lib().orc_fint(int(v))


def sha256(data: bytes) -> bytes:
    out = C.create_string_buffer(32)
    buf = C.create_string_buffer(bytes(data), len(data) or 1)
    lib().orc_sha256(buf, len(data), out)
    return out.raw


def tree_digest(data) -> bytes:
    b = np.frombuffer(bytes(data), dtype=np.uint8) if isinstance(data, (bytes, bytearray)) else \
        np.ascontiguousarray(data).view(np.uint8).reshape(-1)
    out = C.create_string_buffer(32)
    lib().orc_tree_digest(_ptr(b) if b.size else None, b.size, out)
    return out.raw


class Transcript:
    def __init__(self, seed: int):
        self._h = lib().orc_tx_new(seed)

    def absorb(self, label: str, data: bytes):
        buf = C.create_string_buffer(bytes(data), len(data) or 1)
        lib().orc_tx_absorb_h(self._h, label.encode(), buf, len(data))

    def squeeze(self, label: str) -> int:
        return lib().orc_tx_squeeze_h(self._h, label.encode())

    def state(self) -> bytes:
        out = C.create_string_buffer(32)
        lib().orc_tx_state(self._h, out)
        return out.raw

    def __del__(self):
        if getattr(self, "_h", None) and _lib is not None:
            _lib.orc_tx_free(self._h)
            self._h = None


def eq_table(z) -> np.ndarray:
    z = _u64(z)
    out = np.zeros(1 << len(z), dtype=np.uint64)
    lib().orc_eq_table(_ptr(z) if len(z) else None, len(z), _ptr(out))
    return out


def mle_eval(vals, z) -> int:
    vals, z = _u64(vals), _u64(z)
    return lib().orc_mle_eval(_ptr(vals), len(vals), _ptr(z) if len(z) else None, len(z))


def lagrange(g, x: int) -> int:
    g = _u64(g)
    return lib().orc_lagrange(_ptr(g), len(g), x)


# ---- sites ----------------------------------------------------------------

def _csite(s, keep: list) -> _Site:
    w = np.ascontiguousarray(s.w)
    xt = np.ascontiguousarray(s.xt)
    sc = None if s.scales is None else np.ascontiguousarray(s.scales)
    keep.extend([w, xt, sc])
    return _Site(_ptr(w), _ptr(sc), _ptr(xt), s.w_bits, s.M, s.K, s.N, s.k_shift, 0)


def witness(s):
    """(q, r, y) of one site, each N x M (token-major)."""
    q = np.zeros((s.N, s.M), dtype=np.int32)
    r = np.zeros((s.N, s.M), dtype=np.int32)
    y = np.zeros((s.N, s.M), dtype=np.int8)
    keep = []
    cs = _csite(s, keep)
    rc = lib().orc_witness(C.byref(cs), _ptr(q), _ptr(r), _ptr(y))
    if rc != 0:
        raise ValueError("accumulator exceeds 31 bits for this site")
    return q, r, y


def partial_w(s, z) -> np.ndarray:
    z = _u64(z)
    out = np.zeros(1 << log2_ceil(s.K), dtype=np.uint64)
    keep = []
    cs = _csite(s, keep)
    lib().orc_partial_w(C.byref(cs), _ptr(z) if len(z) else None, len(z), _ptr(out))
    return out


def partial_x(s, z) -> np.ndarray:
    z = _u64(z)
    out = np.zeros(1 << log2_ceil(s.K), dtype=np.uint64)
    keep = []
    cs = _csite(s, keep)
    lib().orc_partial_x(C.byref(cs), _ptr(z) if len(z) else None, len(z), _ptr(out))
    return out


def partial_rows(mat, bits: int, scales, rows: int, cols: int, z) -> np.ndarray:
    z = _u64(z)
    mat = np.ascontiguousarray(mat)
    sc = None if scales is None else np.ascontiguousarray(scales)
    out = np.zeros(1 << log2_ceil(cols), dtype=np.uint64)
    lib().orc_partial_rows(_ptr(mat), bits, _ptr(sc), rows, cols, _ptr(z) if len(z) else None,
                           len(z), _ptr(out))
    return out


def claim(q, r, M, N, k, zr, zc) -> int:
    q = np.ascontiguousarray(q, dtype=np.int32)
    r = np.ascontiguousarray(r, dtype=np.int32)
    zr, zc = _u64(zr), _u64(zc)
    return lib().orc_claim(_ptr(q), _ptr(r), M, N, k, _ptr(zr) if len(zr) else None, len(zr),
                           _ptr(zc) if len(zc) else None, len(zc))


# ---- workloads --------------------------------------------------------------

class Resolved:
    """A workload's sites with every linked operand materialised, plus the witness."""

    def __init__(self, sites, wits, groups):
        self.sites = sites
        self.wits = wits
        self.groups = groups


def resolve(wl) -> Resolved:
    """Compute every site's witness in stage order, placing grouped outputs into
    their shared buffers and reading linked operands out of earlier outputs."""
    import copy
    sites = [copy.copy(s) for s in wl.sites]
    groups = {g: {"q": np.zeros(shp, np.int32), "r": np.zeros(shp, np.int32), "y": np.zeros(shp, np.int8)}
              for g, shp in wl.groups.items()}
    wits = [None] * len(sites)

    def out_buffer(idx):
        s = sites[idx]
        if s.out_group is not None:
            return groups[s.out_group[0]]["y"].reshape(-1), 0
        return wits[idx][2].reshape(-1), 0

    for stage in sorted({s.stage for s in sites}):
        for i, s in enumerate(sites):
            if s.stage != stage:
                continue
            if s.w_link is not None:
                src, off = out_buffer(s.w_link[0])
                s.w = src[off + s.w_link[1]: off + s.w_link[1] + s.M * s.K].reshape(s.M, s.K).copy()
            if s.xt_link is not None:
                src, off = out_buffer(s.xt_link[0])
                s.xt = src[off + s.xt_link[1]: off + s.xt_link[1] + s.N * s.K].reshape(s.N, s.K).copy()
            if getattr(s, "xt_hidden", None) is not None:
                ig, iu, kh = s.xt_hidden
                s16 = silu_outputs(wits[ig][2])
                s.xt = ffn_hidden(s16.astype(np.int8), wits[iu][2], kh)[2].reshape(s.N, s.K)
            q, r, y = witness(s)
            if s.out_group is not None:
                g = groups[s.out_group[0]]
                o = s.out_group[1]
                n = s.M * s.N
                g["q"].reshape(-1)[o:o + n] = q.reshape(-1)
                g["r"].reshape(-1)[o:o + n] = r.reshape(-1)
                g["y"].reshape(-1)[o:o + n] = y.reshape(-1)
            wits[i] = (q, r, y)
    return Resolved(sites, wits, groups)


def _marshal(sites, wits, keep):
    n = len(sites)
    cs = (_Site * n)()
    cw = (_Wit * n)()
    for i, (s, w) in enumerate(zip(sites, wits)):
        cs[i] = _csite(s, keep)
        q, r, y = (np.ascontiguousarray(a) for a in w)
        keep.extend([q, r, y])
        cw[i] = _Wit(_ptr(q), _ptr(r), _ptr(y))
    return cs, cw


def prove(seed: int, sites, wits):
    """Full proof. Returns (proof bytes, [state after commit, after matmul, after lookup], matmul section length)."""
    keep = []
    cs, cw = _marshal(sites, wits, keep)
    n = C.c_uint64(0)
    off = C.c_uint64(0)
    states = C.create_string_buffer(96)
    # a buffer large enough for any statement's proof in one pass (the multiplicities of
    # the two tables, 32 + 48 bytes per round and site, the layer rounds); the prover runs
    # again only if it was not, with the size it reported
    kmax = max(int(s.k_shift) for s in sites)
    cap = (1 << 22) + 4 * (1 << kmax) + 64 * len(sites)
    buf = np.zeros(cap, dtype=np.uint8)
    rc = lib().orc_prove(seed, cs, len(sites), cw, _ptr(buf), cap, C.byref(n), states, C.byref(off))
    if rc == -2:
        buf = np.zeros(max(1, n.value), dtype=np.uint8)
        rc = lib().orc_prove(seed, cs, len(sites), cw, _ptr(buf), n.value, C.byref(n), states, C.byref(off))
    if rc != 0:
        raise ValueError(f"orc_prove failed ({rc})")
    st = states.raw
    return buf[: n.value].tobytes(), [st[0:32], st[32:64], st[64:96]], off.value


def prove_hi(seed: int, sites, wits):
    """The layer proof with the helper-inverse lookup section (orc_prove_hi): the commit and
    matmul section of prove(), then both rescale tables by two committed helper columns and
    one sum-check. Returns (proof bytes, [state after commit, after matmul, after lookup],
    matmul section length)."""
    keep = []
    cs, cw = _marshal(sites, wits, keep)
    n = C.c_uint64(0)
    off = C.c_uint64(0)
    states = C.create_string_buffer(96)
    kmax = max(int(s.k_shift) for s in sites)
    cap = (1 << 22) + 4 * (1 << kmax) + 64 * len(sites)
    buf = np.zeros(cap, dtype=np.uint8)
    rc = lib().orc_prove_hi(seed, cs, len(sites), cw, _ptr(buf), cap, C.byref(n), states, C.byref(off))
    if rc == -2:
        buf = np.zeros(max(1, n.value), dtype=np.uint8)
        rc = lib().orc_prove_hi(seed, cs, len(sites), cw, _ptr(buf), n.value, C.byref(n), states, C.byref(off))
    if rc != 0:
        raise ValueError(f"orc_prove_hi failed ({rc})")
    st = states.raw
    return buf[: n.value].tobytes(), [st[0:32], st[32:64], st[64:96]], off.value


def verify_hi(seed: int, sites, wits, proof: bytes):
    """Verifier of prove_hi's proofs: (reason name, detail), 'accept' for a valid proof."""
    keep = []
    cs, cw = _marshal(sites, wits, keep)
    pb = np.frombuffer(proof, dtype=np.uint8).copy() if len(proof) else np.zeros(1, np.uint8)
    det = np.zeros(2, dtype=np.int64)
    rc = lib().orc_verify_hi(seed, cs, len(sites), cw, _ptr(pb), len(proof), _ptr(det))
    return REASONS.get(rc, str(rc)), (int(det[0]), int(det[1]))


def verify(seed: int, sites, wits, proof: bytes, site_mask=None, skip_leaf_open: bool = False):
    """Returns (reason_name, detail) -- reason 'accept' for a valid proof.

    site_mask (optional, one flag per site) limits the direct recomputation of
    claims and of W/X evaluations to the flagged sites; skip_leaf_open skips the
    recomputation of the key columns' MLEs. Every other check always runs."""
    keep = []
    cs, cw = _marshal(sites, wits, keep)
    pb = np.frombuffer(proof, dtype=np.uint8).copy() if len(proof) else np.zeros(1, np.uint8)
    det = np.zeros(2, dtype=np.int64)
    if site_mask is None and not skip_leaf_open:
        rc = lib().orc_verify(seed, cs, len(sites), cw, _ptr(pb), len(proof), _ptr(det))
    else:
        mask = None if site_mask is None else np.ascontiguousarray(np.asarray(site_mask, dtype=np.uint8))
        rc = lib().orc_verify_opts(seed, cs, len(sites), cw, _ptr(pb), len(proof), _ptr(det), _ptr(mask),
                                   4 if skip_leaf_open else 0)
    return REASONS.get(rc, str(rc)), (int(det[0]), int(det[1]))


# ---- gated product h = s (.) u ------------------------------------------------

def _i8(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int8).reshape(-1))


def had_prove(seed: int, s, u):
    """Sum-check proof that the gated product h = s (.) u has the claimed MLE at the
    transcript's point (see oracle.c). Returns (proof bytes, transcript state after)."""
    L = lib()
    a, b = _i8(s), _i8(u)
    if a.size != b.size or a.size < 1:
        raise ValueError("had_prove: s and u need the same length >= 1")
    out = []
    for cap in (0, None):
        tx = L.orc_tx_new(seed)
        n = C.c_uint64(0)
        buf = np.zeros(max(1, out[0] if out else 1), dtype=np.uint8)
        rc = L.orc_had_prove(tx, _ptr(a), _ptr(b), a.size, _ptr(buf) if out else None, out[0] if out else 0,
                             C.byref(n))
        st = C.create_string_buffer(32)
        L.orc_tx_state(tx, st)
        L.orc_tx_free(tx)
        if out:
            if rc != 0:
                raise ValueError(f"orc_had_prove failed ({rc})")
            return buf[: n.value].tobytes(), st.raw
        if rc not in (0, -2):
            raise ValueError(f"orc_had_prove rejected the statement ({rc})")
        out.append(n.value)


def had_verify(seed: int, s, u, proof: bytes):
    """Returns (reason_name, detail); 'accept' for a valid proof."""
    L = lib()
    a, b = _i8(s), _i8(u)
    pb = np.frombuffer(proof, dtype=np.uint8).copy() if len(proof) else np.zeros(1, np.uint8)
    det = np.zeros(2, dtype=np.int64)
    tx = L.orc_tx_new(seed)
    rc = L.orc_had_verify(tx, _ptr(a), _ptr(b), a.size, _ptr(pb), len(proof), _ptr(det))
    L.orc_tx_free(tx)
    return REASONS.get(rc, str(rc)), (int(det[0]), int(det[1]))


# ---- per-group scale reduction: W_eff = S (.) w to claims on w and S ----------------

def scl_prove(seed: int, w, bits: int, scales, M: int, K: int, z):
    """Sum-check reducing a claim on W_eff~(z) (W_eff[i][k] = S[i][k // 64] w[i][k]) to
    claims on w and S (see oracle.c). z: vM + vK field elements, row coordinates first.
    Returns (proof bytes, transcript state after)."""
    L = lib()
    wa = np.ascontiguousarray(w)
    sa = np.ascontiguousarray(np.asarray(scales, dtype=np.int8))
    za = _u64(z)
    out = []
    for _ in range(2):
        tx = L.orc_tx_new(seed)
        n = C.c_uint64(0)
        buf = np.zeros(max(1, out[0] if out else 1), dtype=np.uint8)
        rc = L.orc_scl_prove(tx, _ptr(wa), bits, _ptr(sa), M, K, _ptr(za), _ptr(buf) if out else None,
                             out[0] if out else 0, C.byref(n))
        st = C.create_string_buffer(32)
        L.orc_tx_state(tx, st)
        L.orc_tx_free(tx)
        if out:
            if rc != 0:
                raise ValueError(f"orc_scl_prove failed ({rc})")
            return buf[: n.value].tobytes(), st.raw
        if rc not in (0, -2):
            raise ValueError(f"orc_scl_prove rejected the statement ({rc})")
        out.append(n.value)


def scl_verify(seed: int, w, bits: int, scales, M: int, K: int, z, proof: bytes):
    """Returns (reason_name, detail); 'accept' for a valid proof."""
    L = lib()
    wa = np.ascontiguousarray(w)
    sa = np.ascontiguousarray(np.asarray(scales, dtype=np.int8))
    za = _u64(z)
    pb = np.frombuffer(proof, dtype=np.uint8).copy() if len(proof) else np.zeros(1, np.uint8)
    det = np.zeros(2, dtype=np.int64)
    tx = L.orc_tx_new(seed)
    rc = L.orc_scl_verify(tx, _ptr(wa), bits, _ptr(sa), M, K, _ptr(za), _ptr(pb), len(proof), _ptr(det))
    L.orc_tx_free(tx)
    return REASONS.get(rc, str(rc)), (int(det[0]), int(det[1]))


# ---- SiLU by lookup -----------------------------------------------------------------

def silu_q(v: int) -> int:
    """The SiLU table's entry for a 16-bit input read with 8 fractional bits (see oracle.c)."""
    return int(lib().orc_silu_q(int(v)))


def _i16(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int16).reshape(-1))


def _lookup16_prove(fn, seed: int, g, s):
    L = lib()
    a, b = _i16(g), _i16(s)
    if a.size != b.size or a.size < 1:
        raise ValueError("lookup: g and s need the same length >= 1")
    out = []
    for _ in range(2):
        tx = L.orc_tx_new(seed)
        n = C.c_uint64(0)
        buf = np.zeros(max(1, out[0] if out else 1), dtype=np.uint8)
        rc = fn(tx, _ptr(a), _ptr(b), a.size, _ptr(buf) if out else None, out[0] if out else 0, C.byref(n))
        st = C.create_string_buffer(32)
        L.orc_tx_state(tx, st)
        L.orc_tx_free(tx)
        if out:
            if rc != 0:
                raise ValueError(f"lookup prover failed ({rc})")
            return buf[: n.value].tobytes(), st.raw
        if rc not in (0, -2):
            raise ValueError(f"lookup prover rejected the statement ({rc})")
        out.append(n.value)


def _lookup16_verify(fn, seed: int, g, s, proof: bytes):
    L = lib()
    a, b = _i16(g), _i16(s)
    pb = np.frombuffer(proof, dtype=np.uint8).copy() if len(proof) else np.zeros(1, np.uint8)
    det = np.zeros(2, dtype=np.int64)
    tx = L.orc_tx_new(seed)
    rc = fn(tx, _ptr(a), _ptr(b), a.size, _ptr(pb), len(proof), _ptr(det))
    L.orc_tx_free(tx)
    return REASONS.get(rc, str(rc)), (int(det[0]), int(det[1]))


def silu_prove(seed: int, g, s):
    """LogUp proof that every s_i is the SiLU table's entry for g_i. Returns (proof, state after)."""
    return _lookup16_prove(lib().orc_silu_prove, seed, g, s)


def silu_verify(seed: int, g, s, proof: bytes):
    """Returns (reason_name, detail); 'accept' for a valid proof."""
    return _lookup16_verify(lib().orc_silu_verify, seed, g, s, proof)


def exp_q(v: int) -> int:
    """The softmax numerator table's entry: floor(511 e^(v / 256) + 1/2) for v <= 0, 511 above."""
    return int(lib().orc_exp_q(int(v)))


def exp_prove(seed: int, g, s):
    """LogUp proof that every s_i is the exponent table's entry for g_i."""
    return _lookup16_prove(lib().orc_exp_prove, seed, g, s)


def exp_verify(seed: int, g, s, proof: bytes):
    return _lookup16_verify(lib().orc_exp_verify, seed, g, s, proof)


def silu2_prove(seed: int, g, s):
    """The SiLU lookup with every challenge and value in the quadratic extension."""
    return _lookup16_prove(lib().orc_silu2_prove, seed, g, s)


def silu2_verify(seed: int, g, s, proof: bytes):
    return _lookup16_verify(lib().orc_silu2_verify, seed, g, s, proof)


def exp2_prove(seed: int, g, s):
    """The softmax numerator lookup with every challenge and value in the quadratic extension."""
    return _lookup16_prove(lib().orc_exp2_prove, seed, g, s)


def exp2_verify(seed: int, g, s, proof: bytes):
    return _lookup16_verify(lib().orc_exp2_verify, seed, g, s, proof)


# ---- the helper-inverse LogUp (the variant to set against the GKR tree) -------------

def lhi_prove(seed: int, r, k: int):
    """Helper-inverse LogUp proof that every key r_i lies in the remainder table R_k."""
    return _lhi_prove(lib().orc_lhi_prove, seed, r, k)


def lhi2_prove(seed: int, r, k: int):
    """The same statement with every challenge and value in the quadratic extension."""
    return _lhi_prove(lib().orc_lhi2_prove, seed, r, k)


def _lhi_prove(fn, seed: int, r, k: int):
    L = lib()
    a = np.ascontiguousarray(np.asarray(r, dtype=np.int32).reshape(-1))
    out = []
    for _ in range(2):
        tx = L.orc_tx_new(seed)
        n = C.c_uint64(0)
        buf = np.zeros(max(1, out[0] if out else 1), dtype=np.uint8)
        rc = fn(tx, _ptr(a), a.size, k, _ptr(buf) if out else None, out[0] if out else 0, C.byref(n))
        st = C.create_string_buffer(32)
        L.orc_tx_state(tx, st)
        L.orc_tx_free(tx)
        if out:
            if rc != 0:
                raise ValueError(f"helper-inverse prover failed ({rc})")
            return buf[: n.value].tobytes(), st.raw
        if rc not in (0, -2):
            raise ValueError(f"helper-inverse prover rejected the statement ({rc})")
        out.append(n.value)


def lhi_verify(seed: int, r, k: int, proof: bytes):
    return _lhi_verify(lib().orc_lhi_verify, seed, r, k, proof)


def lhi2_verify(seed: int, r, k: int, proof: bytes):
    return _lhi_verify(lib().orc_lhi2_verify, seed, r, k, proof)


def _lhi_verify(fn, seed: int, r, k: int, proof: bytes):
    L = lib()
    a = np.ascontiguousarray(np.asarray(r, dtype=np.int32).reshape(-1))
    pb = np.frombuffer(proof, dtype=np.uint8).copy() if len(proof) else np.zeros(1, np.uint8)
    det = np.zeros(2, dtype=np.int64)
    tx = L.orc_tx_new(seed)
    rc = fn(tx, _ptr(a), a.size, k, _ptr(pb), len(proof), _ptr(det))
    L.orc_tx_free(tx)
    return REASONS.get(rc, str(rc)), (int(det[0]), int(det[1]))


# ---- extension-field challenges: F_p[phi] / (phi^2 - 7) -----------------------------

def e2_mul(x, y):
    a, b, out = _u64(x), _u64(y), np.zeros(2, np.uint64)
    lib().orc_e2_mul(_ptr(a), _ptr(b), _ptr(out))
    return int(out[0]), int(out[1])


def e2_inv(x):
    a, out = _u64(x), np.zeros(2, np.uint64)
    lib().orc_e2_inv(_ptr(a), _ptr(out))
    return int(out[0]), int(out[1])


def had2_prove(seed: int, s, u):
    """The gated-product sum-check with challenges in the quadratic extension."""
    return _lookup16_free_prove(lib().orc_had2_prove, seed, _i8(s), _i8(u))


def had2_verify(seed: int, s, u, proof: bytes):
    L = lib()
    a, b = _i8(s), _i8(u)
    pb = np.frombuffer(proof, dtype=np.uint8).copy() if len(proof) else np.zeros(1, np.uint8)
    det = np.zeros(2, dtype=np.int64)
    tx = L.orc_tx_new(seed)
    rc = L.orc_had2_verify(tx, _ptr(a), _ptr(b), a.size, _ptr(pb), len(proof), _ptr(det))
    L.orc_tx_free(tx)
    return REASONS.get(rc, str(rc)), (int(det[0]), int(det[1]))


def _lookup16_free_prove(fn, seed, a, b):
    L = lib()
    out = []
    for _ in range(2):
        tx = L.orc_tx_new(seed)
        n = C.c_uint64(0)
        buf = np.zeros(max(1, out[0] if out else 1), dtype=np.uint8)
        rc = fn(tx, _ptr(a), _ptr(b), a.size, _ptr(buf) if out else None, out[0] if out else 0, C.byref(n))
        st = C.create_string_buffer(32)
        L.orc_tx_state(tx, st)
        L.orc_tx_free(tx)
        if out:
            if rc != 0:
                raise ValueError(f"prover failed ({rc})")
            return buf[: n.value].tobytes(), st.raw
        if rc not in (0, -2):
            raise ValueError(f"prover rejected the statement ({rc})")
        out.append(n.value)


# ---- the Freivalds check of a weight matmul (a comparison statement) ------------------

def frv_prove(seed: int, site, wit):
    """Freivalds proof of one site: u = X rho^(.) sent after absorbing the site's digests."""
    return _site_prove(lib().orc_frv_prove, seed, site, wit)


def frv_verify(seed: int, site, wit, proof: bytes):
    return _site_verify(lib().orc_frv_verify, seed, site, wit, proof)


def mm2_prove(seed: int, site, wit):
    """The matmul sum-check of one site with challenges in the quadratic extension."""
    return _site_prove(lib().orc_mm2_prove, seed, site, wit)


def mm2_verify(seed: int, site, wit, proof: bytes):
    return _site_verify(lib().orc_mm2_verify, seed, site, wit, proof)


def _site_prove(fn, seed: int, site, wit):
    L = lib()
    keep = []
    cs = _csite(site, keep)
    q, r, y = (np.ascontiguousarray(a) for a in wit)
    cw = _Wit(_ptr(q), _ptr(r), _ptr(y))
    n = C.c_uint64(0)
    tx = L.orc_tx_new(seed)
    fn(tx, C.byref(cs), C.byref(cw), None, 0, C.byref(n))
    L.orc_tx_free(tx)
    buf = np.zeros(max(1, n.value), dtype=np.uint8)
    tx = L.orc_tx_new(seed)
    rc = fn(tx, C.byref(cs), C.byref(cw), _ptr(buf), n.value, C.byref(n))
    st = C.create_string_buffer(32)
    L.orc_tx_state(tx, st)
    L.orc_tx_free(tx)
    if rc != 0:
        raise ValueError(f"prover failed ({rc})")
    return buf[: n.value].tobytes(), st.raw


def _site_verify(fn, seed: int, site, wit, proof: bytes):
    L = lib()
    keep = []
    cs = _csite(site, keep)
    q, r, y = (np.ascontiguousarray(a) for a in wit)
    cw = _Wit(_ptr(q), _ptr(r), _ptr(y))
    pb = np.frombuffer(proof, dtype=np.uint8).copy() if len(proof) else np.zeros(1, np.uint8)
    det = np.zeros(2, dtype=np.int64)
    tx = L.orc_tx_new(seed)
    rc = fn(tx, C.byref(cs), C.byref(cw), _ptr(pb), len(proof), _ptr(det))
    L.orc_tx_free(tx)
    return REASONS.get(rc, str(rc)), (int(det[0]), int(det[1]))


# ---- MoE routing (top-1, the first argmax of the router logits) ---------------------

def route_witness(l, T: int, E: int):
    """(H, D): the one-hot first-argmax choice (T x E u8) and D = l[t][e_t] - l[t][e] - [e < e_t]
    (T x E int32) of the router logits l (T x E int8, token-major)."""
    L = lib()
    a = np.ascontiguousarray(np.asarray(l, dtype=np.int8).reshape(-1))
    H = np.zeros(T * E, dtype=np.uint8)
    D = np.zeros(T * E, dtype=np.int32)
    L.orc_route_witness(_ptr(a), T, E, _ptr(H), _ptr(D))
    return H.reshape(T, E), D.reshape(T, E)


def route_prove(seed: int, l, H, D, T: int, E: int):
    """The routing proof (sum-check tying D to H and l, H one-hot; the range of D by the
    helper-inverse LogUp) for the given witness; returns (proof bytes, transcript state)."""
    L = lib()
    a = np.ascontiguousarray(np.asarray(l, dtype=np.int8).reshape(-1))
    h = np.ascontiguousarray(np.asarray(H, dtype=np.uint8).reshape(-1))
    d = np.ascontiguousarray(np.asarray(D, dtype=np.int32).reshape(-1))
    n = C.c_uint64(0)
    tx = L.orc_tx_new(seed)
    L.orc_route_prove(tx, _ptr(a), _ptr(h), _ptr(d), T, E, None, 0, C.byref(n))
    L.orc_tx_free(tx)
    buf = np.zeros(max(1, n.value), dtype=np.uint8)
    tx = L.orc_tx_new(seed)
    rc = L.orc_route_prove(tx, _ptr(a), _ptr(h), _ptr(d), T, E, _ptr(buf), n.value, C.byref(n))
    st = C.create_string_buffer(32)
    L.orc_tx_state(tx, st)
    L.orc_tx_free(tx)
    if rc != 0:
        raise ValueError(f"orc_route_prove failed ({rc})")
    return buf[: n.value].tobytes(), st.raw


def route_verify(seed: int, l, H, D, T: int, E: int, proof: bytes):
    L = lib()
    a = np.ascontiguousarray(np.asarray(l, dtype=np.int8).reshape(-1))
    h = np.ascontiguousarray(np.asarray(H, dtype=np.uint8).reshape(-1))
    d = np.ascontiguousarray(np.asarray(D, dtype=np.int32).reshape(-1))
    pb = np.frombuffer(proof, dtype=np.uint8).copy() if len(proof) else np.zeros(1, np.uint8)
    det = np.zeros(2, dtype=np.int64)
    tx = L.orc_tx_new(seed)
    rc = L.orc_route_verify(tx, _ptr(a), _ptr(h), _ptr(d), T, E, _ptr(pb), len(proof), _ptr(det))
    L.orc_tx_free(tx)
    return REASONS.get(rc, str(rc)), (int(det[0]), int(det[1]))


# ---- MoE dispatch: the experts' stacked inputs are the routed permutation of X ----------

def _dsp_args(X, e, D):
    x = np.ascontiguousarray(np.asarray(X, dtype=np.int8))
    ev = np.ascontiguousarray(np.asarray(e, dtype=np.int32).reshape(-1))
    d = np.ascontiguousarray(np.asarray(D, dtype=np.int8))
    if x.ndim != 2 or d.shape != x.shape or ev.size != x.shape[0]:
        raise ValueError("dispatch: X and D must be T x K and e of length T")
    return x, ev, d


def dsp_prove(seed: int, X, e, D, E: int):
    """The dispatch proof (orc_dsp_prove) for token-major X (T x K int8), experts e (T) and the
    stacked expert inputs D (T x K); returns (proof bytes, transcript state)."""
    L = lib()
    x, ev, d = _dsp_args(X, e, D)
    T, K = x.shape
    n = C.c_uint64(0)
    tx = L.orc_tx_new(seed)
    L.orc_dsp_prove(tx, _ptr(x), _ptr(ev), _ptr(d), T, K, E, None, 0, C.byref(n))
    L.orc_tx_free(tx)
    buf = np.zeros(max(1, n.value), dtype=np.uint8)
    tx = L.orc_tx_new(seed)
    rc = L.orc_dsp_prove(tx, _ptr(x), _ptr(ev), _ptr(d), T, K, E, _ptr(buf), n.value, C.byref(n))
    st = C.create_string_buffer(32)
    L.orc_tx_state(tx, st)
    L.orc_tx_free(tx)
    if rc != 0:
        raise ValueError(f"orc_dsp_prove failed ({rc})")
    return buf[: n.value].tobytes(), st.raw


def dsp_verify(seed: int, X, e, D, E: int, proof: bytes):
    L = lib()
    x, ev, d = _dsp_args(X, e, D)
    T, K = x.shape
    pb = np.frombuffer(proof, dtype=np.uint8).copy() if len(proof) else np.zeros(1, np.uint8)
    det = np.zeros(2, dtype=np.int64)
    tx = L.orc_tx_new(seed)
    rc = L.orc_dsp_verify(tx, _ptr(x), _ptr(ev), _ptr(d), T, K, E, _ptr(pb), len(proof), _ptr(det))
    L.orc_tx_free(tx)
    return REASONS.get(rc, str(rc)), (int(det[0]), int(det[1]))


# ---- the rescale LogUp over the extension -------------------------------------------

def lu2_prove(seed: int, sites, wits):
    """The two-table rescale LogUp of the sites' key columns with every challenge and value in
    the quadratic extension; returns (proof bytes, transcript state)."""
    L = lib()
    keep = []
    cs, cw = _marshal(sites, wits, keep)
    n = C.c_uint64(0)
    tx = L.orc_tx_new(seed)
    L.orc_lu2_prove(tx, cs, len(sites), cw, None, 0, C.byref(n))
    L.orc_tx_free(tx)
    buf = np.zeros(max(1, n.value), dtype=np.uint8)
    tx = L.orc_tx_new(seed)
    rc = L.orc_lu2_prove(tx, cs, len(sites), cw, _ptr(buf), n.value, C.byref(n))
    st = C.create_string_buffer(32)
    L.orc_tx_state(tx, st)
    L.orc_tx_free(tx)
    if rc != 0:
        raise ValueError(f"orc_lu2_prove failed ({rc})")
    return buf[: n.value].tobytes(), st.raw


def lu2_verify(seed: int, sites, wits, proof: bytes):
    L = lib()
    keep = []
    cs, cw = _marshal(sites, wits, keep)
    pb = np.frombuffer(proof, dtype=np.uint8).copy() if len(proof) else np.zeros(1, np.uint8)
    det = np.zeros(2, dtype=np.int64)
    tx = L.orc_tx_new(seed)
    rc = L.orc_lu2_verify(tx, cs, len(sites), cw, _ptr(pb), len(proof), _ptr(det))
    L.orc_tx_free(tx)
    return REASONS.get(rc, str(rc)), (int(det[0]), int(det[1]))


# ---- the FFN layer statement (the layer proof chained with the scale reductions, the SiLU
# lookup of the gate outputs and the gated product with the up outputs) ---------------------

def silu_outputs(y) -> np.ndarray:
    """The committed SiLU outputs for 8-bit inputs: silu_q of every entry, as int16."""
    tab = np.array([silu_q(v) for v in range(-128, 128)], dtype=np.int16)
    return tab[np.asarray(y, dtype=np.int64) + 128]


def ffn_hidden(s, u, kh: int):
    """The rescaled hidden activations (orc_ffn_hidden) of the products s * u (8-bit SiLU outputs
    and up outputs, same shape): (q_h, r_h, y_h) with q_h = floor((h + 2^(kh-1)) / 2^kh),
    r_h = h - 2^kh q_h, y_h = clamp(q_h, -128, 127)."""
    s = np.ascontiguousarray(s, dtype=np.int8)
    u = np.ascontiguousarray(u, dtype=np.int8)
    if s.shape != u.shape:
        raise ValueError("ffn_hidden: s and u differ in shape")
    q = np.zeros(s.shape, np.int32)
    r = np.zeros(s.shape, np.int32)
    y = np.zeros(s.shape, np.int8)
    if lib().orc_ffn_hidden(_ptr(s), _ptr(u), s.size, kh, _ptr(q), _ptr(r), _ptr(y)) != 0:
        raise ValueError(f"ffn_hidden: kh = {kh} outside [1, 16]")
    return q, r, y


def _ffn_inputs(wits, ig, iu, kh, s16, hidden):
    s = np.ascontiguousarray(silu_outputs(wits[ig][2]) if s16 is None else s16, dtype=np.int16)
    if hidden is None:
        if s.min(initial=0) < -128 or s.max(initial=0) > 127:
            raise ValueError("SiLU outputs do not fit 8 bits")
        hidden = ffn_hidden(s.astype(np.int8), wits[iu][2], kh)
    return s, [np.ascontiguousarray(a, dtype=t) for a, t in zip(hidden, (np.int32, np.int32, np.int8))]


def prove_ffn(seed: int, sites, wits, ig: int = 0, iu: int = 1, idn: int = 2, kh: int = 7, s16=None,
              hidden=None):
    """The FFN statement (orc_prove_ffn): gate = sites[ig], up = sites[iu], down = sites[idn] (its X
    the rescaled hidden activations); s16 defaults to the honest SiLU outputs of the gate's y and
    hidden = (q_h, r_h, y_h) to ffn_hidden of those and the up outputs. Returns (proof bytes,
    transcript state after)."""
    L = lib()
    keep = []
    cs, cw = _marshal(sites, wits, keep)
    s, (qh, rh, yh) = _ffn_inputs(wits, ig, iu, kh, s16, hidden)
    n = C.c_uint64(0)
    st = C.create_string_buffer(32)
    args = (seed, cs, len(sites), cw, ig, iu, idn, kh, _ptr(s), _ptr(qh), _ptr(rh), _ptr(yh))
    rc = L.orc_prove_ffn(*args, None, 0, C.byref(n), st)
    if rc not in (0, -2):
        raise ValueError(f"orc_prove_ffn rejected the statement ({rc})")
    buf = np.zeros(max(1, n.value), dtype=np.uint8)
    rc = L.orc_prove_ffn(*args, _ptr(buf), n.value, C.byref(n), st)
    if rc != 0:
        raise ValueError(f"orc_prove_ffn failed ({rc})")
    return buf[: n.value].tobytes(), st.raw


def verify_ffn(seed: int, sites, wits, proof: bytes, ig: int = 0, iu: int = 1, idn: int = 2, kh: int = 7,
               s16=None, hidden=None):
    """Returns (reason_name, detail); 'accept' for a valid proof."""
    L = lib()
    keep = []
    cs, cw = _marshal(sites, wits, keep)
    s, (qh, rh, yh) = _ffn_inputs(wits, ig, iu, kh, s16, hidden)
    pb = np.frombuffer(proof, dtype=np.uint8).copy() if len(proof) else np.zeros(1, np.uint8)
    det = np.zeros(2, dtype=np.int64)
    rc = L.orc_verify_ffn(seed, cs, len(sites), cw, ig, iu, idn, kh, _ptr(s), _ptr(qh), _ptr(rh), _ptr(yh),
                          _ptr(pb), len(proof), _ptr(det))
    return REASONS.get(rc, str(rc)), (int(det[0]), int(det[1]))
