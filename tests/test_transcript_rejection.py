"""The squeeze's rejection branch, pinned.

A challenge is the first candidate SHA256(st || "sq" || u32le(|label|) || label ||
u32le(ctr)) whose low 8 bytes, read little-endian, are below p = 2^64 - 2^32 + 1;
a candidate at or above p (probability about 2^-32) is skipped. No proof in the
other tests ever meets one. tests/golden/squeeze_rejection.json holds a seed and a
label found by tests/golden/find_squeeze_rejection.py whose first candidate is
rejected: the oracle's transcript, an independent restatement (hashlib) and the
library's transcript must all take the next candidate and move to its state.
"""

import hashlib
import json
import struct
from pathlib import Path

import pytest

import oracle
from tests import bruteforce as bf

P = bf.P
FIX = Path(__file__).resolve().parent / "golden" / "squeeze_rejection.json"


@pytest.fixture(scope="module")
def fix():
    if not FIX.exists():
        pytest.skip("no rejection fixture")
    return json.loads(FIX.read_text())


def _candidate(st, label, ctr):
    lb = label.encode()
    return hashlib.sha256(st + b"sq" + struct.pack("<I", len(lb)) + lb + struct.pack("<I", ctr)).digest()


def test_first_candidate_is_rejected_and_the_next_taken(fix):
    seed, label = fix["seed"], fix["label"]
    st0 = hashlib.sha256(b"FPSC-v1" + struct.pack("<Q", seed)).digest()
    c0 = _candidate(st0, label, 0)
    assert int.from_bytes(c0[:8], "little") >= P
    ctr = 1
    while int.from_bytes(_candidate(st0, label, ctr)[:8], "little") >= P:
        ctr += 1
    want = int.from_bytes(_candidate(st0, label, ctr)[:8], "little")
    # the oracle's transcript and the brute-force restatement
    ot = oracle.Transcript(seed)
    assert ot.squeeze(label) == want
    bt = bf.Tx(seed)
    assert bt.squeeze(label) == want
    # both moved to the accepted candidate's state: the next squeezes agree
    assert ot.squeeze("after") == bt.squeeze("after")


def test_library_transcript_skips_the_same_candidate(fix):
    from sum_check_prover_b200 import build
    build.build()
    import sum_check_prover_b200 as fp
    seed, label = fix["seed"], fix["label"]
    lt = fp.Transcript(seed)
    ot = oracle.Transcript(seed)
    assert lt.squeeze(label)[0] == ot.squeeze(label)
    assert lt.squeeze("after")[0] == ot.squeeze("after")
    assert lt.state() == ot.state()
