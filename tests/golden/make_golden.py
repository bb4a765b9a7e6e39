"""Writes tests/golden/oracle_fullsize.json: the CPU oracle's proofs of the
full-size layer configurations, as SHA-256 digests of the proof bytes and of
the witness, the transcript states and the section length. Calls only
``oracle`` and ``workloads`` (nothing of the CUDA path).

    python tests/golden/make_golden.py [config ...]     # default: 4 3
    python tests/golden/make_golden.py ffn3             # the FFN statement of configuration 3
"""

import hashlib
import json
import sys
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parents[2]
sys.path.insert(0, str(ROOT))

import oracle  # noqa: E402
import workloads  # noqa: E402

OUT = Path(__file__).resolve().parent / "oracle_fullsize.json"


def witness_digest(wits) -> str:
    h = hashlib.sha256()
    for q, r, y in wits:
        h.update(q.astype("<i4").tobytes())
        h.update(r.astype("<i4").tobytes())
        h.update(y.astype("i1").tobytes())
    return h.hexdigest()


def ffn(cfg: int, data: dict):
    """The FFN statement (oracle.prove_ffn: the layer proof of the chained FFN, whose down site
    reads the layer's own hidden activations, continued by the scale reductions, the hidden
    rescale's lookup, the SiLU lookup of the gate outputs and the gated product with the up
    outputs)."""
    seed = 0
    t0 = time.time()
    wl = workloads.build(cfg, seed=seed, chained=True)
    R = oracle.resolve(wl)
    t1 = time.time()
    proof, state = oracle.prove_ffn(seed, R.sites, R.wits)
    t2 = time.time()
    data[f"config{cfg}_ffn_seed{seed}"] = {
        "workload": wl.description,
        "sites": len(wl.sites),
        "proof_sha256": hashlib.sha256(proof).hexdigest(),
        "proof_len": len(proof),
        "state": state.hex(),
        "witness_sha256": witness_digest(R.wits),
        "oracle_seconds": {"witness": round(t1 - t0, 1), "prove": round(t2 - t1, 1)},
    }
    OUT.write_text(json.dumps(data, indent=1, sort_keys=True) + "\n")
    print(f"ffn{cfg}", "done", round(t2 - t0, 1), "s", flush=True)


def main(configs):
    data = json.loads(OUT.read_text()) if OUT.exists() else {}
    for cfg in configs:
        if isinstance(cfg, str) and cfg.startswith("ffn"):
            ffn(int(cfg[3:]), data)
            continue
        seed = 0
        t0 = time.time()
        wl = workloads.build(cfg, seed=seed)
        R = oracle.resolve(wl)
        t1 = time.time()
        proof, states, mm_len = oracle.prove(seed, R.sites, R.wits)
        t2 = time.time()
        data[f"config{cfg}_seed{seed}"] = {
            "workload": wl.description,
            "sites": len(wl.sites),
            "proof_sha256": hashlib.sha256(proof).hexdigest(),
            "proof_len": len(proof),
            "matmul_section_len": mm_len,
            "states": [s.hex() for s in states],
            "witness_sha256": witness_digest(R.wits),
            "oracle_seconds": {"witness": round(t1 - t0, 1), "prove": round(t2 - t1, 1)},
        }
        OUT.write_text(json.dumps(data, indent=1, sort_keys=True) + "\n")
        print(cfg, "done", round(t2 - t0, 1), "s", flush=True)


if __name__ == "__main__":
    main([a if a.startswith("ffn") else int(a) for a in sys.argv[1:]] or [4, 3])
