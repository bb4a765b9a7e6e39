"""Search for a transcript seed whose first squeeze candidate is rejected.

The Fiat-Shamir squeeze (the transcript of the proof format: st0 = SHA256("FPSC-v1"
|| u64le(seed)), candidate ctr = SHA256(st || "sq" || u32le(|label|) || label ||
u32le(ctr)), the challenge is the first candidate whose low 8 bytes, read
little-endian, are below p = 2^64 - 2^32 + 1) rejects a candidate with
probability about 2^-32. This script scans seeds in parallel until the first
candidate of one is at least p, and writes that seed and label to
squeeze_rejection.json; the tests then check that the oracle and the library
both skip to the next candidate. Only an input is stored here: the expected
challenge is computed by the oracle when the test runs.

Run: python tests/golden/find_squeeze_rejection.py [workers]
"""

import hashlib
import json
import multiprocessing as mp
import struct
import sys
from pathlib import Path

LABEL = b"pin_reject"
OUT = Path(__file__).resolve().parent / "squeeze_rejection.json"
SUFFIX = b"sq" + struct.pack("<I", len(LABEL)) + LABEL + struct.pack("<I", 0)
HIGH = b"\xff\xff\xff\xff"


def scan(args):
    start, step, stop_flag = args
    base = hashlib.sha256(b"FPSC-v1")
    seed = start
    while not stop_flag.value:
        for _ in range(1 << 20):
            h0 = base.copy()
            h0.update(struct.pack("<Q", seed))
            h = hashlib.sha256(h0.digest() + SUFFIX).digest()
            # candidate >= p exactly when its high 32 bits are all ones and its low 32 bits are not all zero
            if h[4:8] == HIGH and h[0:4] != b"\x00\x00\x00\x00":
                stop_flag.value = 1
                return seed
            seed += step
    return None


def main():
    workers = int(sys.argv[1]) if len(sys.argv) > 1 else mp.cpu_count()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        flag = mgr.Value("i", 0)
        with ctx.Pool(workers) as pool:
            for res in pool.imap_unordered(scan, [(w, workers, flag) for w in range(workers)]):
                if res is not None:
                    OUT.write_text(json.dumps({"seed": res, "label": LABEL.decode(),
                                               "note": "first squeeze candidate >= p"}, indent=1) + "\n")
                    print("found", res)
                    pool.terminate()
                    return


if __name__ == "__main__":
    main()
