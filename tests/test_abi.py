"""The C-ABI library builds for sm_100a, loads without a GPU, and exports every
entry point its header declares. Host-only entry points (transcript, proof
sizes) are checked against the oracle here; compute entry points only run in
the GPU tests."""

import ctypes as C
import random
import re
from pathlib import Path

import pytest

import oracle
import workloads

ROOT = Path(__file__).resolve().parent.parent


@pytest.fixture(scope="module")
def L():
    from sum_check_prover_b200 import build
    build.build()
    import sum_check_prover_b200 as fp
    return fp.lib()


def _declared():
    names = set()
    for h in (ROOT / "include").glob("*.h"):
        src = h.read_text()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        for m in re.finditer(r"\b([A-Za-z_]\w*)\s*\(([^;{}()]*)\)\s*;", src):
            names.add(m.group(1))
    return names


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert {"fp_commit_witness", "mle_partial_eval", "sumcheck_prove_matmul", "logup_prove_rescale"} <= names
    for n in sorted(names):
        assert hasattr(L, n), f"{n} declared in include/ but not exported"
    assert L.fp_version() >= 100


def test_transcript_matches_oracle(L):
    import sum_check_prover_b200 as fp
    rnd = random.Random(11)
    for seed in (0, 1, 2**64 - 1):
        a, b = fp.Transcript(seed), oracle.Transcript(seed)
        assert a.state() == b.state()
        for _ in range(40):
            if rnd.random() < 0.5:
                lab = "lab%d" % rnd.randrange(100)
                data = bytes(rnd.randrange(256) for _ in range(rnd.randrange(0, 300)))
                a.absorb(lab, data)
                b.absorb(lab, data)
            else:
                lab = "ch%d" % rnd.randrange(10)
                assert a.squeeze(lab)[0] == b.squeeze(lab)
        assert a.state() == b.state()
        a.close()


def test_proof_sizes_match_oracle(L):
    import sum_check_prover_b200 as fp
    for sites in (workloads.build(1).sites, workloads.build(3, small=True).sites,
                  [workloads.random_site(3, 5, 7, 3, 4, 5)]):
        R = oracle.resolve(workloads.Workload("t", 0, sites))
        pf, _, off = oracle.prove(0, R.sites, R.wits)
        descs = [fp.SiteDesc(1, 1, 1, 1, 1, s.M, s.K, s.N, s.w_bits, s.k_shift) for s in R.sites]
        arr, keep = fp._sites(descs)
        mm, lu = C.c_size_t(), C.c_size_t()
        assert L.fp_proof_size(arr, len(descs), C.byref(mm), C.byref(lu)) == 0
        assert mm.value == off and mm.value + lu.value == len(pf)


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    import sum_check_prover_b200 as fp
    monkeypatch.setattr(fp, "LIB_PATH", tmp_path / "libfp.so")
    monkeypatch.setattr(fp, "_lib", None)
    with pytest.raises(ImportError):
        fp.lib()


def test_portable_sha_path_matches_oracle(L):
    """The host transcript uses the CPU's SHA extensions when present; the
    portable compression (forced here) must give the same states."""
    import subprocess
    import sys
    code = ("import sys; sys.path.insert(0, '.'); import sum_check_prover_b200 as fp, oracle; "
            "a, b = fp.Transcript(7), oracle.Transcript(7)\n"
            "for i in range(300):\n"
            "    d = bytes((i * 37 + j) % 256 for j in range(i % 190))\n"
            "    a.absorb('l%d' % (i % 5), d); b.absorb('l%d' % (i % 5), d)\n"
            "    assert a.squeeze('c')[0] == b.squeeze('c')\n"
            "assert a.state() == b.state(); print('ok')")
    import os
    env = dict(os.environ, FP_NO_SHANI="1")
    r = subprocess.run([sys.executable, "-c", code], cwd=str(ROOT), env=env, capture_output=True, text=True)
    assert r.returncode == 0 and "ok" in r.stdout, r.stderr


def test_silu_table_matches_oracle(L):
    # the library's table (host C++) and the oracle's (plain C), each from the formula
    import numpy as np
    import sum_check_prover_b200 as fp
    lib_t = fp.silu_table()
    ora_t = np.array([oracle.silu_q(v) for v in range(-32768, 32768)], dtype=np.int32)
    assert np.array_equal(lib_t, ora_t)


def test_exp_table_matches_oracle(L):
    import numpy as np
    import sum_check_prover_b200 as fp
    ora_t = np.array([oracle.exp_q(v) for v in range(-32768, 32768)], dtype=np.int32)
    assert np.array_equal(fp.exp_table(), ora_t)
