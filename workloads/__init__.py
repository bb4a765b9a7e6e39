"""Seeded synthetic inputs for the matmul sum-check prover.

This module is the only code that both the CPU oracle tests and the CUDA
path use. It holds shapes and random draws only: no field arithmetic, no
rescale, no hashing, nothing of the proving method.

Layouts (the storage order every consumer assumes):

* ``w``: the weight-side operand W, M x K row-major. int4 is packed two per
  byte along K, the low nibble holding the even k, two's complement; a row
  takes ceil(K/2) bytes and an odd K leaves the last high nibble zero.
  int8 is one signed byte per element.
* ``scales``: optional per-64-group int8 scales along K, M x ceil(K/64).
* ``xt``: the activation operand X stored token-major, i.e. X^T as N x K
  row-major int8 (each token's K-vector contiguous).
* outputs q, r (int32) and y (int8) are N x M row-major (token-major).

Distributions follow the workload descriptions of the pages' layer shapes:
int8 weights uniform in [-128, 127]; int4 weights uniform in [-8, 7];
activations round(N(0, 32)) clamped to [-128, 127]; group scales uniform in
[1, 127]; MoE routing top-1 uniform over the experts.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

__all__ = ["Site", "Workload", "build", "CONFIG_NAMES"]


@dataclass
class Site:
    """One matrix product Y = W . X to be proven (one 'site')."""

    name: str
    M: int
    K: int
    N: int
    w_bits: int
    k_shift: int
    w: Optional[np.ndarray] = None
    scales: Optional[np.ndarray] = None
    xt: Optional[np.ndarray] = None
    # A stage-1 site may read its operand out of an earlier site's y output:
    # (site_index, element_offset) into that site's output *group* buffer.
    w_link: Optional[tuple] = None
    xt_link: Optional[tuple] = None
    # An FFN's down projection reads the gated product of the SiLU of the gate site's outputs
    # with the up site's outputs, rescaled by 2^kh: (gate_index, up_index, kh). Only a
    # declaration: the prover computes these activations from the two outputs.
    xt_hidden: Optional[tuple] = None
    # Sites whose outputs live inside one shared N x M buffer: (group, offset).
    out_group: Optional[tuple] = None
    stage: int = 0
    # W is a committed weight (digested once, offline) rather than an activation
    w_is_weight: bool = True

    @property
    def macs(self) -> int:
        return self.M * self.K * self.N

    @property
    def w_row_bytes(self) -> int:
        return (self.K + 1) // 2 if self.w_bits == 4 else self.K


@dataclass
class Workload:
    name: str
    seed: int
    sites: list
    # shared output buffers: name -> (N, M) shape
    groups: dict = field(default_factory=dict)
    description: str = ""

    @property
    def macs(self) -> int:
        return sum(s.macs for s in self.sites)

    @property
    def n_keys(self) -> int:
        return sum(s.M * s.N for s in self.sites)


def _rng(seed: int, tid: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), int(tid)])))


def int4_packed(rng: np.random.Generator, M: int, K: int) -> np.ndarray:
    """M x ceil(K/2) bytes; every nibble uniform over the 16 two's-complement values."""
    rb = (K + 1) // 2
    w = rng.integers(0, 256, size=(M, rb), dtype=np.uint8)
    if K % 2:
        w[:, -1] &= 0x0F
    return w


def int8_uniform(rng: np.random.Generator, shape) -> np.ndarray:
    return rng.integers(-128, 128, size=shape, dtype=np.int8)


def activations(rng: np.random.Generator, shape) -> np.ndarray:
    v = np.rint(rng.normal(0.0, 32.0, size=shape))
    return np.clip(v, -128, 127).astype(np.int8)


def group_scales(rng: np.random.Generator, M: int, K: int) -> np.ndarray:
    return rng.integers(1, 128, size=(M, (K + 63) // 64), dtype=np.int8)


def unpack_int4(w: np.ndarray, K: int) -> np.ndarray:
    """Packed int4 bytes -> int8 array M x K (test and harness convenience)."""
    lo = (w & 0x0F).astype(np.int8)
    hi = (w >> 4).astype(np.int8)
    out = np.empty((w.shape[0], 2 * w.shape[1]), dtype=np.int8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    out = np.where(out >= 8, out - 16, out).astype(np.int8)
    return out[:, :K]


# ---------------------------------------------------------------------------
# configurations
# ---------------------------------------------------------------------------

def _tiny(seed: int) -> Workload:
    """64x64 int8 W, X 64x16 int8 uniform, rescale by 2^7."""
    M, K, N = 64, 64, 16
    s = Site("tiny", M, K, N, 8, 7,
             w=int8_uniform(_rng(seed, 1), (M, K)),
             xt=int8_uniform(_rng(seed, 2), (N, K)))
    return Workload("tiny", seed, [s], description="W 64x64 int8, X 64x16 int8, k=7")


def _projection(seed: int, M=4096, K=4096, N=512, k=12) -> Workload:
    """Single int4 projection, activations ~ round(N(0,32)), rescale by 2^12."""
    s = Site("proj", M, K, N, 4, k,
             w=int4_packed(_rng(seed, 1), M, K),
             xt=activations(_rng(seed, 2), (N, K)))
    return Workload("projection", seed, [s],
                    description=f"W {M}x{K} int4, X {K}x{N} int8 N(0,32), k={k}")


def _dense_ffn(seed: int, d=4096, ffn=14336, T=4096, k=18, chained=False, kh=7) -> Workload:
    """Llama-3.1-8B-shaped FFN: gate/up d->ffn, down ffn->d, int4 + per-64 int8 scales.

    The down projection's activations are a seeded stand-in, or with ``chained`` the layer's
    own hidden activations (SiLU(gate) * up rescaled by 2^kh), which the FFN statement proves."""
    x = activations(_rng(seed, 100), (T, d))
    h = None if chained else activations(_rng(seed, 101), (T, ffn))
    sites = []
    for idx, (nm, M, K, xt) in enumerate([("gate", ffn, d, x), ("up", ffn, d, x), ("down", d, ffn, h)]):
        sites.append(Site(nm, M, K, T, 4, k,
                          w=int4_packed(_rng(seed, 10 * idx + 1), M, K),
                          scales=group_scales(_rng(seed, 10 * idx + 2), M, K),
                          xt=xt))
    if chained:
        sites[2].xt_hidden = (0, 1, kh)
        sites[2].stage = 1
    return Workload("dense_ffn_chained" if chained else "dense_ffn", seed, sites,
                    description=f"d={d} ffn={ffn} T={T} int4+scales k={k}" + (f" chained kh={kh}" if chained else ""))


def _moe(seed: int, E=128, d=5120, ffn=8192, T=8192, k=12, experts=None, shared=True) -> Workload:
    """Top-1 routed MoE with a shared expert; every matmul its own site.

    ``experts`` (a list of expert indices) and ``shared`` keep only those
    experts' sites: the same tensors, drawn from the same seeds, as in the
    whole layer (a sample of the layer's sites for a CPU timing)."""
    x = activations(_rng(seed, 100), (T, d))
    route = _rng(seed, 99).integers(0, E, size=T)
    keep = set(range(E)) if experts is None else set(int(e) for e in experts)
    sites = []
    for e in range(E):
        idx = np.nonzero(route == e)[0]
        ne = len(idx)
        if ne == 0 or e not in keep:
            continue
        xe = np.ascontiguousarray(x[idx])
        he = activations(_rng(seed, 1000 + 10 * e), (ne, ffn))
        for j, (nm, M, K, xt) in enumerate([("gate", ffn, d, xe), ("up", ffn, d, xe), ("down", d, ffn, he)]):
            sites.append(Site(f"e{e}.{nm}", M, K, ne, 4, k,
                              w=int4_packed(_rng(seed, 1000 + 10 * e + 1 + j), M, K), xt=xt))
    if shared:
        hs = activations(_rng(seed, 200), (T, ffn))
        for j, (nm, M, K, xt) in enumerate([("gate", ffn, d, x), ("up", ffn, d, x), ("down", d, ffn, hs)]):
            sites.append(Site(f"shared.{nm}", M, K, T, 4, k,
                              w=int4_packed(_rng(seed, 300 + j), M, K), xt=xt))
    return Workload("moe", seed, sites,
                    description=f"{E} experts d={d} ffn={ffn} T={T} top-1 + shared, k={k}")


def moe_dispatch(seed: int, E=128, d=5120, T=8192, experts=None):
    """The MoE layer's dispatch statement: the layer input X (T x d, the tensor the experts'
    gate and up sites read), the routing e (the expert of every token) and D, the experts'
    inputs stacked expert by expert (each expert's tokens in token order: the rows of those
    sites' activations). The same draws as _moe's (seeds 100 and 99)."""
    x = activations(_rng(seed, 100), (T, d))
    route = _rng(seed, 99).integers(0, E, size=T)
    D = np.concatenate([x[route == e] for e in range(E)])
    return x, route.astype(np.int32), D


def _attn_dense(seed: int, d=5120, nq=40, nkv=8, hd=128, B=64, ctx=2048, ffn=16384, k=12) -> Workload:
    """Decode step of a GQA attention + dense MLP layer, B requests x 1 token.

    Stage 0: Q/K/V projections, O^T_bg = V_bg^T . P_bg^T per (request, KV group),
    gate/up/down. Stage 1: scores S_bg = Q_bg . K_bg^T (Q read out of the Q
    projection's y), and the O projection (input read out of the attention
    outputs' shared y buffer).
    """
    g = nq // nkv
    x = activations(_rng(seed, 100), (B, d))
    m = activations(_rng(seed, 101), (B, d))          # norm output feeding the MLP
    h = activations(_rng(seed, 102), (B, ffn))        # SiLU(gate)*up output
    kc = activations(_rng(seed, 103), (B, nkv, ctx, hd))   # key cache [b][g][t][d]
    vt = activations(_rng(seed, 104), (B, nkv, hd, ctx))   # value cache stored d-major [b][g][d][t]
    pr = activations(_rng(seed, 105), (B, nkv, g, ctx))    # softmax output P [b][g][h][t]
    sites = []
    qi = len(sites)
    sites.append(Site("wq", nq * hd, d, B, 4, k, w=int4_packed(_rng(seed, 1), nq * hd, d), xt=x))
    sites.append(Site("wk", nkv * hd, d, B, 4, k, w=int4_packed(_rng(seed, 2), nkv * hd, d), xt=x))
    sites.append(Site("wv", nkv * hd, d, B, 4, k, w=int4_packed(_rng(seed, 3), nkv * hd, d), xt=x))
    first_o = len(sites)
    for b in range(B):
        for kv in range(nkv):
            sites.append(Site(f"ot.{b}.{kv}", hd, ctx, g, 8, k, w=vt[b, kv], xt=pr[b, kv],
                              out_group=("attn_out", b * d + kv * g * hd), w_is_weight=False))
    sites.append(Site("gate", ffn, d, B, 4, k, w=int4_packed(_rng(seed, 4), ffn, d), xt=m))
    sites.append(Site("up", ffn, d, B, 4, k, w=int4_packed(_rng(seed, 5), ffn, d), xt=m))
    sites.append(Site("down", d, ffn, B, 4, k, w=int4_packed(_rng(seed, 6), d, ffn), xt=h))
    for b in range(B):
        for kv in range(nkv):
            sites.append(Site(f"s.{b}.{kv}", g, hd, ctx, 8, k, xt=kc[b, kv],
                              w_link=(qi, b * nq * hd + kv * g * hd), stage=1, w_is_weight=False))
    sites.append(Site("wo", d, nq * hd, B, 4, k, w=int4_packed(_rng(seed, 7), d, nq * hd),
                      xt_link=(first_o, 0), stage=1))
    return Workload("attn_dense", seed, sites, groups={"attn_out": (B, nq * hd)},
                    description=f"d={d} heads {nq}/{nkv}x{hd} B={B} ctx={ctx} ffn={ffn} k={k}")


CONFIG_NAMES = {
    1: "tiny",
    2: "projection",
    3: "dense_ffn",
    4: "attn_dense",
    5: "moe",
}

# Reduced shapes with the same structure, small enough for the CPU oracle.
_SMALL = {
    3: dict(d=256, ffn=896, T=64),
    4: dict(d=640, nq=5, nkv=1, hd=128, B=4, ctx=256, ffn=1024),
    5: dict(E=4, d=128, ffn=256, T=128),
}


def build(config: int, seed: int = 0, small: bool = False, **overrides) -> Workload:
    """Build a configuration's sites. ``small`` selects a reduced shape of the same structure."""
    if config == 1:
        return _tiny(seed)
    if config == 2:
        return _projection(seed, **overrides)
    kw = dict(_SMALL[config]) if small else {}
    kw.update(overrides)
    if config == 3:
        return _dense_ffn(seed, **kw)
    if config == 4:
        return _attn_dense(seed, **kw)
    if config == 5:
        return _moe(seed, **kw)
    raise ValueError(f"unknown config {config}")


def random_site(rng_seed: int, M: int, K: int, N: int, w_bits: int, k_shift: int,
                scales: bool = False, act: bool = True) -> Site:
    """A single seeded site of arbitrary shape (ragged shapes for edge-case tests)."""
    r = _rng(rng_seed, 7)
    w = int4_packed(r, M, K) if w_bits == 4 else int8_uniform(r, (M, K))
    sc = group_scales(_rng(rng_seed, 8), M, K) if scales else None
    xt = activations(_rng(rng_seed, 9), (N, K)) if act else int8_uniform(_rng(rng_seed, 9), (N, K))
    return Site(f"rand{rng_seed}", M, K, N, w_bits, k_shift, w=w, scales=sc, xt=xt)
