"""Device copies of a workload for the CUDA path (torch tensors on one GPU).

Pointer wiring only: uploads the seeded host arrays, allocates the witness
buffers (q, r, y; N x M token-major), places grouped outputs inside their
shared buffer, makes a linked operand a view of the output it reads, and gives
an FFN's down site an empty activation buffer for the prover to fill. No
arithmetic of the proving method lives here.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np


@dataclass
class DevSite:
    name: str
    w: object
    scales: object
    xt: object
    q: object
    r: object
    y: object
    M: int
    K: int
    N: int
    w_bits: int
    k_shift: int
    w_digest: Optional[bytes] = None
    is_weight: bool = True


def upload(wl, device: str = "cuda"):
    """Returns (stages, keep): stages is a list of lists of DevSite in site order."""
    import torch

    dev = torch.device(device)
    keep = {}
    groups = {}
    for g, (n, m) in wl.groups.items():
        groups[g] = dict(q=torch.zeros((n, m), dtype=torch.int32, device=dev),
                         r=torch.zeros((n, m), dtype=torch.int32, device=dev),
                         y=torch.zeros((n, m), dtype=torch.int8, device=dev))
    cache = {}
    # the witness of the sites without a shared output buffer, one tensor per column in site
    # order, so the lookup section reads its keys in place
    free = [s for s in wl.sites if s.out_group is None]
    nfree = sum(s.M * s.N for s in free)
    col_q = torch.empty(max(1, nfree), dtype=torch.int32, device=dev)
    col_r = torch.empty(max(1, nfree), dtype=torch.int32, device=dev)
    col_y = torch.empty(max(1, nfree), dtype=torch.int8, device=dev)
    keep["columns"] = (col_q, col_r, col_y)
    foff = 0

    def t(a):
        key = id(a)
        if key not in cache:
            cache[key] = (torch.from_numpy(np.ascontiguousarray(a)).to(dev), a)
        return cache[key][0]

    out = []

    def y_buffer(idx):
        s = wl.sites[idx]
        if s.out_group is not None:
            return groups[s.out_group[0]]["y"].view(-1)
        return out[idx].y.view(-1)

    for i, s in enumerate(wl.sites):
        if s.out_group is not None:
            gb, off, n = groups[s.out_group[0]], s.out_group[1], s.M * s.N
            q = gb["q"].view(-1)[off:off + n].view(s.N, s.M)
            r = gb["r"].view(-1)[off:off + n].view(s.N, s.M)
            y = gb["y"].view(-1)[off:off + n].view(s.N, s.M)
        else:
            n = s.M * s.N
            q = col_q[foff:foff + n].view(s.N, s.M)
            r = col_r[foff:foff + n].view(s.N, s.M)
            y = col_y[foff:foff + n].view(s.N, s.M)
            foff += n
        if s.w_link is not None:
            src, off = s.w_link
            w = y_buffer(src)[off:off + s.M * s.K].view(s.M, s.K)
        else:
            w = t(s.w)
        if s.xt_link is not None:
            src, off = s.xt_link
            xt = y_buffer(src)[off:off + s.N * s.K].view(s.N, s.K)
        elif s.xt_hidden is not None:
            # an FFN's hidden activations: fp.prove_ffn writes them before this stage is committed
            xt = torch.zeros((s.N, s.K), dtype=torch.int8, device=dev)
        else:
            xt = t(s.xt)
        sc = t(s.scales) if s.scales is not None else None
        out.append(DevSite(s.name, w, sc, xt, q, r, y, s.M, s.K, s.N, s.w_bits, s.k_shift,
                           is_weight=(s.w_is_weight and s.w_link is None)))
    keep["groups"] = groups
    keep["cache"] = cache
    stages = []
    for st in sorted({s.stage for s in wl.sites}):
        stages.append([d for d, s in zip(out, wl.sites) if s.stage == st])
    return stages, keep


def weight_digests(ctx, stages):
    """Offline commitment of the weights: D(W) || D(scales) for every weight operand."""
    for st in stages:
        for d in st:
            if not d.is_weight:
                continue
            nb = d.M * ((d.K + 1) // 2 if d.w_bits == 4 else d.K)
            dw = ctx.digest(d.w, nb)
            ds = ctx.digest(d.scales, d.M * ((d.K + 63) // 64)) if d.scales is not None else ctx.digest(None, 0)
            d.w_digest = dw + ds
