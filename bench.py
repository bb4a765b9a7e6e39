#!/usr/bin/env python
"""Benchmark of the B200 sum-check prover for quantised matrix products.

One step = one whole proof of one synthetic statement: witness + commitment
(fp_commit_witness), batched matmul sum-check (sumcheck_prove_matmul) and the
LogUp rescale/clamp proof (logup_prove_rescale), from a fresh transcript.
Default workload (--config 5): the MoE layer, 128 experts of 5120 -> 8192 ->
5120 int4 (gate, up, down) with 8192 tokens routed top-1 and a shared expert of
the same shape, rescale by 2^12: 387 sites, 2.06e12 MACs, 3.5e8 lookup keys.
--config 2 is the single projection (W 4096x4096 int4, X 4096x512, 8.6e9 MACs).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config C]

Prints one JSON line (rank 0). value = proved MACs/s of the whole job with
inputs resident in HBM; e2e = the same through the public API with the
activations copied from pinned host memory and the layer output read back
every step; roofline = the kernel with the largest device time, from a
profiled pass of identical steps (CUDA events around every launch on its
stream); cpu_baseline = the CPU oracle timed on this host.
"""

from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "proved matmul MACs/s and sum-check Melem/s at 1 B200; HBM GB/s vs peak"
UNIT = "MAC/s"
DEFAULT_CONFIG = 5
FLUSH_BYTES = 512 << 20  # > 126 MB L2

# kernel -> source file (traffic counters are valid only for the source they were taken on)
KSRC = {"witness_gemm": "witness.cu", "digest_leaf": "digest.cu", "digest_node": "digest.cu",
        "digest_final": "digest.cu", "eq_build": "mle.cu", "partial_acc": "partial.cu", "partial_fin": "partial.cu",
        "claim": "mle.cu", "sc_round": "sumcheck.cu", "sc_final": "sumcheck.cu", "hist": "logup.cu",
        "keys_gather": "logup.cu", "tree_leaf": "logup.cu", "tree_up": "logup.cu", "gkr_round": "logup.cu",
        "gkr_final": "logup.cu", "leaf_eval": "logup.cu", "reduce": "mle.cu"}


def src_hash(kernel: str) -> str:
    f = ROOT / "sum_check_prover_b200" / "csrc" / KSRC.get(kernel, "")
    h = hashlib.sha256()
    for p in [f, *sorted((ROOT / "sum_check_prover_b200" / "csrc").glob("*.cuh"))]:
        if p.is_file():
            h.update(p.read_bytes())
    return h.hexdigest()[:16]


def peaks() -> dict:
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"], "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "src": "fallback"}


def host_cpu() -> dict:
    """The host's logical core count and CPU model (for the oracle baseline)."""
    model = None
    try:
        for ln in Path("/proc/cpuinfo").read_text().splitlines():
            if ln.startswith("model name"):
                model = ln.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


def cpu_sample(config: int, seed: int, step: int = 0):
    """A bounded sample of the configuration's statement for the single-threaded oracle
    (about 10-20 s of CPU work), and what it is. The sample's sites are the workload's
    own sites, drawn from the same seeds."""
    import workloads
    if config in (1, 2):
        return workloads.build(config, seed=seed), "the whole statement (witness + full proof)"
    if config == 5:
        e = [step % 128]
        wl = workloads.build(5, seed=seed, experts=e, shared=False)
        return wl, (f"the sites of expert {e[0]} of the MoE layer (gate, up, down: 3 of 387 sites, "
                    f"{wl.macs:.3g} MACs, {wl.n_keys} keys), witness + full proof of that sub-statement")
    if config == 3:
        wl = workloads.build(3, seed=seed, T=128)
        return wl, "the FFN with 128 of its 4096 tokens (same weights), witness + full proof"
    wl = workloads.build(4, seed=seed, B=2)
    return wl, "the decode layer with 2 of its 64 requests (same weights), witness + full proof"


def sumcheck_elems(wl) -> int:
    """Initial hypercube sizes of every sum-check instance in one proof."""
    n = max((s.K - 1).bit_length() for s in wl.sites)
    mm = len(wl.sites) * (1 << n)
    nk = wl.n_keys
    v = max(1, (nk - 1).bit_length())
    return mm + 2 * ((1 << v) - 2)


class Clocks:
    """SM clock and clock-event reasons sampled every 2 ms during the timed region (NVML
    from a thread, read-only queries; nvidia-smi every 200 ms when NVML is unavailable)."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.f = None
        self.nvml = None
        self.samples = []
        self.stop_flag = False
        self.thread = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nvml = None

    def _poll(self):
        nv = self.nvml
        bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        while not self.stop_flag:
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = (nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                      if hasattr(nv, "nvmlDeviceGetCurrentClocksEventReasons")
                      else nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h))
                self.samples.append((mhz, [k for k, v in bits.items() if rs & v]))
            except Exception:
                pass
            self.started.set()
            time.sleep(0.002)

    def start(self):
        if self.nvml is not None:
            import threading

            self.samples = []
            self.stop_flag = False
            self.started = threading.Event()
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            self.started.wait(timeout=5)
            self.samples = []  # the region starts now
            return
        try:
            self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=5)
            self.thread = None
            sm = [m for m, _ in self.samples]
            reasons = sorted({r for _, rs in self.samples for r in rs})
            return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                    "samples": len(sm), "reasons": reasons, "source": "nvml, every 2 ms"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.f.seek(0)
        rows = [r for r in csv.reader(io.StringIO(self.f.read())) if len(r) >= 9]
        self.f.close()
        os.unlink(self.f.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for nm, val in zip(names, r[5:9]):
                if val.strip().lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "samples": len(sm), "reasons": sorted(reasons), "source": "nvidia-smi, every 200 ms"}


MICRO_ALL = "sc,pe,gkr,lhr,gemm,had,scl,silu,had2,lhi,mm2,frv,lhi2,silu2,lu2,ffn"


def micro_names(which) -> set:
    """The microbench names in a comma-separated list (whole names: "had" is not "had2")."""
    names = set(which.split(",")) if isinstance(which, str) else set(which)
    unknown = names - set(MICRO_ALL.split(","))
    if unknown:
        raise ValueError(f"unknown microbench names: {sorted(unknown)}")
    return names


def run_micro(fp, torch, ctx, dev: str, which: str = MICRO_ALL) -> dict:
    """Kernel rooflines at HBM scale (inputs well above the 126 MB L2), from a
    profiled pass: every round is its own launch, timed with CUDA events.

    sc_round: matmul sum-check rounds over 2 x 2^26-element vectors (64 sites,
      W 1 x 2^20 int4, one token); round 1 reads A and B, later rounds fold
      in place of the next evaluation (read 4, write 2 values per pair).
    partial_acc: eq-weighted row contraction of a 16384 x 16384 int4 matrix (the
      weight side) and of a 16384 x 16384 int8 matrix (the activation side); and
      the batched weight-side launch of a MoE layer's proof (16 experts of
      8192 x 5120 / 5120 x 8192 int4 plus the shared expert: 51 matrices, 1.07 GB).
    gkr_round: LogUp layer rounds over 2^26 keys (one 8192 x 64 x 8192 int8 site).
    had_round: gated-product sum-check rounds over two 2^26-entry int8 factors
      (round 1 reads the int8 factors and writes the eq table, round 2 folds
      them into field vectors, later rounds read 4 and write 2 values of both
      factors and fold the eq table: 120 B per pair).
    scale_reduction: the whole scale reduction of a 14336 x 4096 int4 weight matrix with
      per-64 scales (CUDA events around the call), its per-kernel split, and the group
      contraction W' (the weights read once) against the copy bandwidth.
    silu_round: the SiLU lookup's layer sum-checks over 2^26 keys (one tree; round 1
      reads the tree layer's children, later rounds fold them: 80 and 160 B per pair).
    had2_round: the gated product over 2^26 entries with challenges in the quadratic
      extension (16-byte vector elements: 120 B per pair in round 2, 240 B later).
    lhi_round: the helper-inverse LogUp's sum-check over 2^26 keys of R_12 (round 1 reads
      the helper column and the keys, later rounds fold both: 104 and 120 B per pair).
    mm2_contract: the extension-field matmul's row contraction of a 16384 x 16384 int4
      weight (the matrix once; the eq weights are 16-byte extension elements).
    frv_u: Freivalds' prover, u = X rho^(.) over a 16384-token x 16384 int8 activation
      (the activation once, plus the powers of rho).
    lhi2_round: the helper-inverse LogUp's rounds over 2^26 keys with extension challenges
      (16-byte vectors: 176 B per pair in round 2, 240 B later).
    silu2_round: the SiLU lookup's layer rounds over 2^26 keys with extension challenges
      (16-byte vectors: 160 and 320 B per pair).
    lu2_round: the rescale LogUp's layer rounds over 2^26 keys with extension challenges,
      both tables in one launch (288 and 576 B per pair).
    ffn: the FFN layer statement (fp.prove_ffn) over the Llama-3.1-8B-shaped FFN (d 4096,
      ffn 14336, 4096 tokens, int4 weights with per-64 scales, k 18) with the down projection
      reading the layer's own hidden activations: device time per statement (CUDA events
      around the call, inputs resident), the per-kernel split from a profiled pass, and the
      hidden-rescale kernel against the copy bandwidth.
    witness_gemm: one 14336 x 4096 int4 by 4096 x 4096 int8 product with its rescale
      epilogue (a Llama-3.1-8B FFN projection), against the tensor peak; and the witness
      launches of a 16-expert MoE layer (about 64 tokens per expert, the shared expert over
      1024 tokens), bound by the weight stream, against the copy bandwidth.
    """
    import workloads
    from workloads import device
    pk = peaks()
    out = {}

    def measure(name, kernel, fn, big=1 << 28):
        ctx.set_profiling(True)
        fn()  # warm: module loading and arena growth stay out of the numbers
        torch.cuda.synchronize()
        ctx.set_profiling(True)  # resets the per-kernel counters
        fn()
        torch.cuda.synchronize()
        log = [r for r in ctx.kernel_log() if r[0] == kernel]
        ctx.set_profiling(False)
        # the HBM-scale launches (>= 256 MB of algorithmic traffic); the small
        # rounds at the end of a sum-check are latency, not bandwidth
        sel = [r for r in log if r[2] >= big]
        ms = sum(r[1] for r in sel)
        by = sum(r[2] for r in sel)
        gbs = by / (ms * 1e-3) / 1e9 if ms > 0 else 0.0
        out[name] = {"kernel": kernel, "launches": len(sel), "ms": ms, "bytes": by, "GBps": gbs,
                     "frac": gbs / pk["hbm_gbs"], "peak": pk["hbm_gbs"],
                     "all_launches": len(log), "all_ms": sum(r[1] for r in log)}

    which = micro_names(which)
    if "sc" in which:
        sites = [workloads.random_site(900 + i, 1, 1 << 20, 1, 4, 12) for i in range(64)]
        st, keep = device.upload(workloads.Workload("sc", 0, sites), dev)
        device.weight_digests(ctx, st)
        measure("sc_round_2^26", "sc_round", lambda: fp.prove(ctx, 1, st))
        del st, keep

    if "pe" in which:
        rows = cols = 16384
        rng = __import__("numpy").random.default_rng(3)
        mat = torch.from_numpy(workloads.int4_packed(rng, rows, cols)).to(dev)
        outv = torch.empty(cols, dtype=torch.int64, device=dev)
        z = [int(x) for x in rng.integers(0, fp.P, size=14, dtype="uint64")]
        measure("partial_eval_int4_16384^2", "partial_acc",
                lambda: ctx.partial_eval(mat, 4, None, rows, cols, z, outv), big=1 << 26)
        del mat
        mat = torch.from_numpy(workloads.int8_uniform(rng, (rows, cols))).to(dev)
        measure("partial_eval_int8_16384^2", "partial_acc",
                lambda: ctx.partial_eval(mat, 8, None, rows, cols, z, outv), big=1 << 26)
        del mat, outv
        # the weight side of a MoE layer in one batched launch (the prover's own call)
        wl = workloads.build(5, 0, E=16, T=1024)
        st, keep = device.upload(wl, dev)
        device.weight_digests(ctx, st)
        measure("partial_eval_int4_moe_16x3_experts", "partial_acc", lambda: fp.prove(ctx, 0, st), big=1 << 28)
        del st, keep, wl

    if "gemm" in which:
        # witness GEMM of an FFN-sized site on the tensor cores (2 x MACs integer ops)
        site = workloads.random_site(55, 14336, 4096, 4096, 4, 12)
        st, keep = device.upload(workloads.Workload("gemm", 0, [site]), dev)
        device.weight_digests(ctx, st)
        tx = fp.Transcript(0)
        ctx.commit_witness(tx, st[0])
        torch.cuda.synchronize()
        ctx.set_profiling(True)
        for _ in range(3):
            ctx.commit_witness(tx, st[0])
        torch.cuda.synchronize()
        n, ms, by = ctx.kernel_stats()["witness_gemm"]
        ctx.set_profiling(False)
        tx.close()
        tops = 2.0 * site.macs / (ms / n * 1e-3) / 1e12
        peak = pk["bf16_tflops"] * 2.0
        out["witness_gemm_14336x4096x4096_int4"] = {"kernel": "witness_gemm", "launches": n, "ms": ms / n,
                                                    "TOPS": tops, "frac": tops / peak, "peak": peak,
                                                    "peak_note": "int8 = measured bf16 x 2 (nominal ratio)"}
        del st, keep
        # the witness launches of a MoE layer (16 experts of 8192 x 5120 / 5120 x 8192 int4 with
        # about 64 routed tokens each, and the shared expert over 1024 tokens): bound by the
        # weight stream, so reported against the copy bandwidth
        wl = workloads.build(5, 0, E=16, T=1024)
        st, keep = device.upload(wl, dev)
        device.weight_digests(ctx, st)
        measure("witness_gemm_moe_16x3_experts_T1024", "witness_gemm", lambda: fp.prove(ctx, 0, st), big=1 << 20)
        del st, keep, wl

    if "had" in which:
        # the gated product of an FFN's hidden tensor, 2^26 entries per factor
        rng = __import__("numpy").random.default_rng(9)
        n = 1 << 26
        sv = torch.from_numpy(rng.integers(-128, 128, n).astype("int8")).to(dev)
        uv = torch.from_numpy(rng.integers(-128, 128, n).astype("int8")).to(dev)
        measure("hadamard_round_2^26", "had_round", lambda: ctx.prove_hadamard(fp.Transcript(4), sv, uv))
        del sv, uv

    if "scl" in which:
        # the scale reduction of an FFN gate projection: 14336 x 4096 int4 weights with per-64 scales
        rng = __import__("numpy").random.default_rng(10)
        M, K = 14336, 4096
        wv = torch.from_numpy(workloads.int4_packed(rng, M, K)).to(dev)
        sv = torch.from_numpy(workloads.group_scales(rng, M, K)).to(dev)
        pt = [int(x) for x in rng.integers(0, fp.P, size=26, dtype="uint64")]
        run = lambda: ctx.reduce_scales(fp.Transcript(5), wv, 4, sv, M, K, pt)  # noqa: E731
        run()
        torch.cuda.synchronize()
        times = []
        for _ in range(5):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            run()
            b.record()
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        ctx.set_profiling(True)
        run()
        torch.cuda.synchronize()
        ks = ctx.kernel_stats()
        ctx.set_profiling(False)
        n_g, ms_g, by_g = ks.get("scl_group", (0, 0.0, 0.0))
        gbs = by_g / (ms_g * 1e-3) / 1e9 if ms_g > 0 else 0.0
        out["scale_reduction_14336x4096"] = {
            "ms": statistics.median(times), "ms_all": times,
            "kernels_profiled_ms": {k: round(v[1], 4) for k, v in sorted(ks.items(), key=lambda kv: -kv[1][1])},
            "scl_group": {"kernel": "scl_group", "ms": ms_g, "bytes": by_g, "GBps": gbs, "frac": gbs / pk["hbm_gbs"],
                          "peak": pk["hbm_gbs"]}}
        del wv, sv

    if "gkr" in which:
        s = workloads.random_site(77, 8192, 64, 8192, 8, 12)
        st, keep = device.upload(workloads.Workload("gkr", 0, [s]), dev)
        device.weight_digests(ctx, st)
        measure("gkr_round_2^26_keys", "gkr_round", lambda: fp.prove(ctx, 2, st))
        del st, keep
    if "lhr" in which:
        # the same statement's lookup section by helper inverses: its rounds, and the columns'
        # formation (table inverses, two gathers; the digests are timed as digest kernels)
        try:
            s = workloads.random_site(77, 8192, 64, 8192, 8, 12)
            st, keep = device.upload(workloads.Workload("lhr", 0, [s]), dev)
            device.weight_digests(ctx, st)
            measure("helper_inverse_rescale_round_2^26_keys", "lhr_round",
                    lambda: fp.prove(ctx, 2, st, lookup="hi"))
            measure("helper_inverse_rescale_columns_2^26_keys", "lhr_column",
                    lambda: fp.prove(ctx, 2, st, lookup="hi"))
            del st, keep
        except Exception as e:  # a failure here must not cost the rest of the line
            out["helper_inverse_rescale_round_2^26_keys"] = {"error": f"{type(e).__name__}: {e}"[:300]}
    if "silu" in which:
        # the SiLU lookup of an FFN's gate values: 2^26 16-bit inputs and their table entries
        try:
            np_ = __import__("numpy")
            rng = np_.random.default_rng(11)
            tab = fp.silu_table().astype(np_.int16)
            gv = rng.integers(-32768, 32768, 1 << 26).astype(np_.int16)
            gd = torch.from_numpy(gv).to(dev)
            sd = torch.from_numpy(tab[gv.astype(np_.int64) + 32768]).to(dev)
            measure("silu_lookup_round_2^26", "silu_round", lambda: ctx.prove_silu(fp.Transcript(6), gd, sd))
            del gd, sd
        except Exception as e:  # a failure here must not cost the rest of the line
            out["silu_lookup_round_2^26"] = {"error": f"{type(e).__name__}: {e}"[:300]}
    if "had2" in which:
        # the gated product of the same 2^26-entry factors with extension-field challenges
        try:
            rng = __import__("numpy").random.default_rng(9)
            n = 1 << 26
            sv = torch.from_numpy(rng.integers(-128, 128, n).astype("int8")).to(dev)
            uv = torch.from_numpy(rng.integers(-128, 128, n).astype("int8")).to(dev)
            measure("hadamard_ext2_round_2^26", "had2_round",
                    lambda: ctx.prove_hadamard_ext2(fp.Transcript(4), sv, uv))
            del sv, uv
        except Exception as e:  # a failure here must not cost the rest of the line
            out["hadamard_ext2_round_2^26"] = {"error": f"{type(e).__name__}: {e}"[:300]}
    if "lhi" in which:
        # the helper-inverse LogUp of 2^26 remainders in R_12 (set against gkr_round's tree)
        try:
            rng = __import__("numpy").random.default_rng(12)
            rv = torch.from_numpy(rng.integers(-2048, 2048, 1 << 26).astype("int32")).to(dev)
            measure("helper_inverse_round_2^26_keys", "lhi_round",
                    lambda: ctx.prove_helper_inverse(fp.Transcript(7), rv, 12))
            del rv
        except Exception as e:  # a failure here must not cost the rest of the line
            out["helper_inverse_round_2^26_keys"] = {"error": f"{type(e).__name__}: {e}"[:300]}
    if "mm2" in which:
        # the extension-field matmul sum-check of a 16384 x 16384 int4 weight (128 MiB) and 256
        # tokens: its row contraction with 16-byte eq weights, set against partial_acc
        try:
            s = workloads.random_site(78, 16384, 16384, 256, 4, 12)
            st, keep = device.upload(workloads.Workload("mm2", 0, [s]), dev)
            d = st[0][0]
            ctx.commit_witness(fp.Transcript(0), [d])
            measure("ext2_contract_16384x16384_int4", "mm2_contract",
                    lambda: ctx.prove_matmul_ext2(fp.Transcript(8), d), big=1 << 26)
            del st, keep, d
        except Exception as e:  # a failure here must not cost the rest of the line
            out["ext2_contract_16384x16384_int4"] = {"error": f"{type(e).__name__}: {e}"[:300]}
    if "frv" in which:
        # Freivalds' prover for 16384 tokens of a 16384-wide activation (256 MiB of Xt)
        try:
            s = workloads.random_site(79, 128, 16384, 16384, 4, 12)
            st, keep = device.upload(workloads.Workload("frv", 0, [s]), dev)
            d = st[0][0]
            ctx.commit_witness(fp.Transcript(0), [d])
            measure("freivalds_u_16384x16384", "frv_u", lambda: ctx.prove_freivalds(fp.Transcript(9), d))
            del st, keep, d
        except Exception as e:  # a failure here must not cost the rest of the line
            out["freivalds_u_16384x16384"] = {"error": f"{type(e).__name__}: {e}"[:300]}
    if "lhi2" in which:
        # the helper-inverse LogUp of 2^26 remainders in R_12 with extension-field challenges
        try:
            rng = __import__("numpy").random.default_rng(12)
            rv = torch.from_numpy(rng.integers(-2048, 2048, 1 << 26).astype("int32")).to(dev)
            measure("helper_inverse_ext2_round_2^26_keys", "lhi2_round",
                    lambda: ctx.prove_helper_inverse_ext2(fp.Transcript(7), rv, 12))
            del rv
        except Exception as e:  # a failure here must not cost the rest of the line
            out["helper_inverse_ext2_round_2^26_keys"] = {"error": f"{type(e).__name__}: {e}"[:300]}
    if "silu2" in which:
        # the SiLU lookup of 2^26 gate values with extension-field challenges
        try:
            np_ = __import__("numpy")
            rng = np_.random.default_rng(11)
            tab = fp.silu_table().astype(np_.int16)
            gv = rng.integers(-32768, 32768, 1 << 26).astype(np_.int16)
            gd = torch.from_numpy(gv).to(dev)
            sd = torch.from_numpy(tab[gv.astype(np_.int64) + 32768]).to(dev)
            measure("silu_ext2_lookup_round_2^26", "silu2_round", lambda: ctx.prove_silu_ext2(fp.Transcript(6), gd, sd))
            del gd, sd
        except Exception as e:  # a failure here must not cost the rest of the line
            out["silu_ext2_lookup_round_2^26"] = {"error": f"{type(e).__name__}: {e}"[:300]}
    if "lu2" in which:
        # the rescale LogUp over the extension for the gkr microbench's site (2^26 keys)
        try:
            s = workloads.random_site(77, 8192, 64, 8192, 8, 12)
            st, keep = device.upload(workloads.Workload("lu2", 0, [s]), dev)
            ctx.commit_witness(fp.Transcript(0), st[0])
            measure("rescale_logup_ext2_round_2^26_keys", "lu2_round",
                    lambda: ctx.prove_logup_ext2(fp.Transcript(10), st[0]))
            del st, keep
        except Exception as e:  # a failure here must not cost the rest of the line
            out["rescale_logup_ext2_round_2^26_keys"] = {"error": f"{type(e).__name__}: {e}"[:300]}

    if "ffn" in which:
        try:
            wl = workloads.build(3, 0, chained=True)
            st, keep = device.upload(wl, dev)
            device.weight_digests(ctx, st)
            fp.prove_ffn(ctx, 0, st)  # warm: arena growth and module loading
            torch.cuda.synchronize()
            times = []
            for _ in range(3):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                proof, _, _ = fp.prove_ffn(ctx, 0, st)
                b.record()
                torch.cuda.synchronize()
                times.append(a.elapsed_time(b))
            ctx.set_profiling(True)
            fp.prove_ffn(ctx, 0, st)
            torch.cuda.synchronize()
            ks = ctx.kernel_stats()
            ctx.set_profiling(False)
            macs = sum(x.macs for x in wl.sites)
            ms = statistics.median(times)
            top = sorted(ks.items(), key=lambda kv: -kv[1][1])[:12]
            n_h, ms_h, by_h = ks.get("ffn_hidden", (0, 0.0, 0.0))
            gbs_h = by_h / (ms_h * 1e-3) / 1e9 if ms_h > 0 else 0.0
            out["ffn_statement_d4096_ffn14336_T4096"] = {
                "ms": ms, "ms_all": times, "MACs": macs, "MACps": macs / (ms * 1e-3),
                "keys": sum(x.M * x.N for x in wl.sites) + wl.sites[0].M * wl.sites[0].N,
                "proof_bytes": len(proof),
                "kernels_profiled_ms": {k: round(v[1], 3) for k, v in top},
                "ffn_hidden": {"launches": n_h, "ms": ms_h, "bytes": by_h, "GBps": gbs_h,
                               "frac": gbs_h / pk["hbm_gbs"], "peak": pk["hbm_gbs"]}}
            del st, keep, wl
        except Exception as e:  # a failure here must not cost the rest of the line
            out["ffn_statement_d4096_ffn14336_T4096"] = {"error": f"{type(e).__name__}: {e}"[:300]}

    try:
        torch.cuda.empty_cache()
    except Exception:
        pass
    return out


def max_over_ranks(x: float, pg, device) -> float:
    """The largest x over all ranks (the job is as slow as its slowest rank); x itself
    when there is one rank."""
    if pg is None:
        return x
    import torch

    t = torch.tensor([x], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, steps: int, total_ms_max: float) -> float:
    """Whole-job units per second: every rank processed units_per_rank per step, and the
    job took the slowest rank's time."""
    return world * units_per_rank * steps / (total_ms_max / 1e3)


def dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# The pages' own figures, with their hardware: context for the numbers above, not a target
# (other hardware, whole-model proofs including commitments, which this path does not build).
PAGES_CONTEXT = {
    "flashprove_maverick_h100": "about 100 proved tokens/s for Llama 4 Maverick (4-bit weights, batches of 64 "
                                "1,024-token requests) on one H100, 111 tokens/s at batch 24 "
                                "(How fast can FlashProve go; FlashProve: How AI Answers Become Provable)",
    "layer_rtx5070ti": "3.2-6.1 s prove-to-verify per Maverick-width layer on an RTX 5070 Ti "
                       "(flashprove-consumer-gpu)",
    "llama8b_request_h100": "1.0-1.5 h per 4,096 + 512-token Llama-3.1-8B request on one H100, with a "
                            "different proof system (a Circle STARK over M31) (Towards Proving Frontier-Scale "
                            "LLM Inference)",
}


def run_reference(args):
    """The CPU oracle as it stands, each step on a bounded sample of the same workload."""
    world, rank, local = dist()
    if rank != 0:
        return
    import oracle
    times, macs_done, label = [], 0, ""
    for i in range(args.warmup + args.steps):
        wl, label = cpu_sample(args.config, args.seed, i)
        t0 = time.perf_counter()
        R = oracle.resolve(wl)
        oracle.prove(args.seed, R.sites, R.wits)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
            macs_done += wl.macs
    value = macs_done / sum(times)
    per = statistics.mean(times)
    full = workloads_description(args.config)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u64", "data": "synthetic",
            "config": {"workload": full, "config": args.config, "sample": label},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"each step: {label}; single-threaded C", **host_cpu()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workloads_description(config: int) -> str:
    return {1: "tiny matmul W 64x64 int8, X 64x16 int8, k=7",
            2: "projection W 4096x4096 int4, X 4096x512 int8 N(0,32), k=12",
            3: "dense FFN d=4096 ffn=14336 T=4096 int4 + per-64 int8 scales, k=18 (3 sites)",
            4: "decode layer d=5120, 40/8 heads x 128, B=64, ctx 2048, MLP 16384, int4, k=12 (1031 sites)",
            5: "MoE layer: 128 experts 5120->8192->5120 int4 (gate/up/down), T=8192 top-1 routed, "
               "shared expert, k=12 (387 sites)"}[config]


def run_ours(args):
    import torch

    world, rank, local = dist()
    torch.cuda.set_device(local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as td
        td.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                              device_id=torch.device(f"cuda:{local}"))
        pg = td

    import sum_check_prover_b200 as fp
    import workloads
    from workloads import device

    dev = torch.device(f"cuda:{local}")
    # every rank proves its own independent statement (weak scaling, no data-path collective)
    wl = workloads.build(args.config, seed=args.seed + rank)
    macs = wl.macs
    elems = sumcheck_elems(wl)
    ctx = fp.Context(local)
    stages, keep = device.upload(wl, f"cuda:{local}")
    device.weight_digests(ctx, stages)  # offline weight commitment: not part of a proof
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(seed):
        return fp.prove(ctx, seed, stages, stream)

    def barrier():
        if pg is not None:
            pg.barrier()

    proof_len = 0
    for i in range(args.warmup):
        proof, states, status = step(args.seed + i)
        proof_len = len(proof)
        assert status == 0
    torch.cuda.synchronize()

    # ---- timed pass: value --------------------------------------------------------
    clocks = Clocks(local)
    barrier()
    torch.cuda.synchronize()
    n0 = ctx.launches()
    hw0 = ctx.host_stats()
    clocks.start()
    times = []
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)  # L2 flush between timed steps, outside the event pair
        e0.record(stream)
        step(args.seed + 100 + i)
        e1.record(stream)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    clk = clocks.stop()
    torch.cuda.synchronize()
    barrier()
    launches = ctx.launches() - n0
    hw1 = ctx.host_stats()
    host_waits = (hw1[0] - hw0[0]) / args.steps
    host_wait_ms = (hw1[1] - hw0[1]) * 1e3 / args.steps
    host_turn_us = (hw1[2] - hw0[2]) * 1e6 / max(1.0, hw1[0] - hw0[0])
    total_ms = sum(times)
    total_ms = max_over_ranks(total_ms, pg, dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(macs, world, args.steps, total_ms)

    # ---- per-kernel figures: a pass identical to the timed one with CUDA events around every
    # launch (recording them costs host time, so the timed pass itself carries none; a resident
    # sum-check launch spans its rounds, host exchanges included), then a stepped pass (every
    # round its own launch: the device time of each round alone) ------------------------------
    ctx.set_profiling(2)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        step(args.seed + 100 + i)
    torch.cuda.synchronize()
    tstats = ctx.kernel_stats()
    ctx.set_profiling(False)
    kern = {k: {"launches": v[0] / args.steps, "ms": v[1] / args.steps,
                "GBps": (v[2] / (v[1] * 1e-3) / 1e9) if v[1] > 0 else None} for k, v in tstats.items()}
    ctx.set_profiling(True)
    for i in range(args.prof_steps):
        flush.fill_(i & 0xFF)
        step(args.seed + 200 + i)
    torch.cuda.synchronize()
    sstats = ctx.kernel_stats()
    ctx.set_profiling(False)
    kern_stepped = {k: {"launches": v[0] / args.prof_steps, "ms": v[1] / args.prof_steps,
                        "GBps": (v[2] / (v[1] * 1e-3) / 1e9) if v[1] > 0 else None} for k, v in sstats.items()}
    dom = max(tstats.items(), key=lambda kv: kv[1][1])
    pk = peaks()
    # the scope table's HBM-bound rows inside this proof: algorithmic bytes over device time,
    # each round alone (stepped pass) and as launched in the timed configuration (a resident
    # sum-check launch spans its rounds and their host exchanges)
    rows = {}
    for row, kn in (("a4_claim", "claim"), ("a5_partial_eval", "partial_acc"), ("a7_matmul_rounds", "sc_round"),
                    ("a8_histogram", "hist"), ("a9_tree", "tree_up"), ("a10_gkr_rounds", "gkr_round"),
                    ("a11_leaf_claims", "leaf_eval")):
        if kn not in sstats:
            continue
        n_, ms_, by_ = sstats[kn]
        gbs = by_ / (ms_ * 1e-3) / 1e9 if ms_ > 0 else 0.0
        ent = {"kernel": kn, "bytes_per_step": by_ / args.prof_steps, "ms_per_step": ms_ / args.prof_steps,
               "GBps": gbs, "frac": gbs / pk["hbm_gbs"]}
        if kn in tstats and tstats[kn][1] > 0:
            ent["GBps_as_launched"] = tstats[kn][2] / (tstats[kn][1] * 1e-3) / 1e9
        rows[row] = ent
    dname, (dl, dms, dbytes) = dom
    avg_ms = dms / dl
    traffic, traffic_note = None, None
    tf = ROOT / "profiles" / "traffic.json"
    if tf.exists():
        t = json.loads(tf.read_text()).get(dname)
        if t and t.get("src") == src_hash(dname) and t.get("ratio") is not None:
            # DRAM bytes over algorithmic bytes, from an ncu capture of the same kernel
            # source on a smaller case; scaled to this launch's algorithmic bytes
            traffic = t["ratio"] * dbytes / dl
            traffic_note = t.get("note")
    if dname == "witness_gemm":
        flops = 2.0 * macs / (dl / args.steps)
        peak = pk["bf16_tflops"] * 2.0
        achieved = flops / (avg_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": traffic, "kernel": dname,
                "peak_note": f"int8 = {pk['src']} bf16 x 2 (nominal int8/bf16 ratio)"}
        if traffic_note:
            roof["traffic_note"] = traffic_note
    else:
        achieved = (dbytes / dl) / (avg_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "traffic": traffic, "kernel": dname,
                "traffic_note": traffic_note,
                "avg_launch_us": avg_ms * 1e3, "bytes_per_launch": dbytes / dl,
                "peak_note": f"{pk['src']} copy bandwidth",
                "measured": "CUDA events around each launch, in a pass of the timed steps' inputs and "
                            "launch configuration; a resident sum-check launch spans all its rounds, "
                            "host exchanges included"}

    # ---- the same statement with the lookup section by helper inverses (row f3's comparison
    # with the fraction tree): device time per proof and host round trips ------------------
    variants = None
    if not args.no_variants:
        for i in range(2):
            fp.prove(ctx, args.seed + 400 + i, stages, stream, lookup="hi")
        torch.cuda.synchronize()
        hv0 = ctx.host_stats()
        hi_ms = []
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            e0.record(stream)
            hp, _, hstatus = fp.prove(ctx, args.seed + 500 + i, stages, stream, lookup="hi")
            e1.record(stream)
            e1.synchronize()
            hi_ms.append(e0.elapsed_time(e1))
        hv1 = ctx.host_stats()
        hi_total = max_over_ranks(sum(hi_ms), pg, dev)
        variants = {
            "gkr": {"lookup": "LogUp-GKR fraction tree, one sum-check per layer", "ms_per_step": ms_per_step,
                    "value": value, "host_round_trips_per_step": host_waits, "proof_bytes": proof_len},
            "hi": {"lookup": "helper-inverse LogUp: two committed columns, one sum-check",
                   "ms_per_step": hi_total / args.steps, "value": job_throughput(macs, world, args.steps, hi_total),
                   "host_round_trips_per_step": (hv1[0] - hv0[0]) / args.steps, "proof_bytes": len(hp),
                   "status": hstatus}}

    # ---- e2e pass: activations from pinned host memory, layer output read back ----------
    flat = [d for st in stages for d in st]
    seen = set()
    host_x = []
    for d in flat:  # one copy per activation tensor (the gate and up sites share theirs)
        if d.xt.data_ptr() not in seen:
            seen.add(d.xt.data_ptr())
            host_x.append((d, d.xt.cpu().pin_memory()))
    # the outputs: the column buffer that holds every ungrouped site's y, and each output group
    col_y = keep["columns"][2]
    dev_y = ([col_y] if any(s.out_group is None for s in wl.sites) else []) + [g["y"] for g in keep["groups"].values()]
    host_y = [(y, torch.empty(y.shape, dtype=torch.int8).pin_memory()) for y in dev_y]
    h2d = sum(x.numel() for _, x in host_x)
    d2h = sum(y.numel() for y, _ in host_y) + proof_len
    e2e_ms = []
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        e0.record(stream)
        for d, x in host_x:
            d.xt.copy_(x, non_blocking=True)
        step(args.seed + 300 + i)
        for y, h in host_y:
            h.copy_(y, non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        e2e_ms.append(e0.elapsed_time(e1))
    e2e_total = sum(e2e_ms)
    e2e_total = max_over_ranks(e2e_total, pg, dev)
    e2e_value = job_throughput(macs, world, args.steps, e2e_total)

    # ---- CPU baseline: the oracle on this host (rank 0, one GPU only) ------------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        swl, label = cpu_sample(args.config, args.seed, 0)
        t0 = time.perf_counter()
        R = oracle.resolve(swl)
        oracle.prove(args.seed, R.sites, R.wits)
        dt = time.perf_counter() - t0
        cpu = {"value": swl.macs / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"{label}; single-threaded C", "seconds": dt, **host_cpu()}

    micro = None
    if rank == 0 and world == 1 and not args.no_micro:
        micro = run_micro(fp, torch, ctx, f"cuda:{local}")

    ctx.close()
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "u64", "data": "synthetic",
                "config": {"workload": workloads_description(args.config), "config": args.config,
                           "sites": len(wl.sites), "macs_per_step": macs, "lookup_keys_per_step": wl.n_keys,
                           "l2": "flushed between timed steps (512 MiB write); inputs also exceed L2"
                                 if wl.n_keys * 9 > (126 << 20) else "flushed between timed steps (512 MiB write)",
                           "parallelism": f"{world} independent statements, one per GPU"},
                "rows": rows,
                "sumcheck_melem_s": world * elems * args.steps / (total_ms / 1e3) / 1e6,
                "sumcheck_elems_per_step": elems,
                "roofline": roof,
                "cpu_baseline": cpu,
                "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
                "gpu_launches": launches,
                "host_round_trips_per_step": host_waits,
                "host_turnaround_us_per_round": host_turn_us,
                "host_wait_ms_per_step": host_wait_ms,
                "clocks": clk,
                "proof_bytes": proof_len,
                "pages_context": PAGES_CONTEXT,
                "kernels": kern,
                "kernels_stepped": kern_stepped,
                "lookup_variants": variants,
                "microbench": micro,
                # last, so that a reader who keeps only the end of the output still sees it
                "summary": compact_summary(rows, micro, kern, variants)}
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()


def compact_summary(rows, micro, kern, variants):
    """The figures of the long keys in a few hundred bytes: each scope row's fraction of the HBM
    peak inside the proof, each microbench's time and fraction, the kernels above 0.2 ms per
    proof and the two lookup variants' times."""
    def r3(x):
        return None if x is None else round(float(x), 3)
    out = {"rows_frac": {k: r3(v.get("frac")) for k, v in (rows or {}).items()},
           "micro_ms_frac": {k: [r3(v.get("ms")), r3(v.get("frac"))] for k, v in (micro or {}).items()},
           "kernels_ms": {k: round(v["ms"], 2) for k, v in (kern or {}).items() if v.get("ms", 0) >= 0.2}}
    if variants:
        out["lookup_variants_ms"] = {k: r3(v.get("ms_per_step")) for k, v in variants.items()}
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--prof-steps", type=int, default=3)
    ap.add_argument("--config", type=int, default=DEFAULT_CONFIG, choices=[1, 2, 3, 4, 5],
                    help="the statement one step proves (5: the MoE layer, the largest one-GPU configuration)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-micro", action="store_true")
    ap.add_argument("--no-variants", action="store_true", help="skip the helper-inverse lookup timing")
    ap.add_argument("--micro-only", nargs="?", const=MICRO_ALL, default=None,
                    help="run only the kernel measurements at scale (comma list of sc, pe, gkr, gemm)")
    args = ap.parse_args()
    if args.micro_only:
        import torch

        import sum_check_prover_b200 as fp
        ctx = fp.Context(0)
        print(json.dumps({"microbench": run_micro(fp, torch, ctx, "cuda:0", args.micro_only)}))
        ctx.close()
        return
    if args.warmup < 1:
        args.warmup = 1
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
