"""bench.py's compact summary: the figures of the long keys, small enough to survive a reader
that keeps only the end of the output."""

import json

import bench


def test_summary_rounds_and_filters():
    rows = {"a5_partial_eval": {"frac": 0.96512, "ms_per_step": 1.3}, "a9_tree": {"frac": None}}
    micro = {"gkr_round_2^26_keys": {"ms": 2.84512, "frac": 0.56399, "per_launch": [[1.0, 2.0]] * 50},
             "ffn_statement": {"ms": 41.6}}
    kern = {"gkr_round": {"ms": 28.614, "launches": 28}, "reduce": {"ms": 0.013}}
    variants = {"gkr": {"ms_per_step": 47.9839}, "hi": {"ms_per_step": 53.4268}}
    s = bench.compact_summary(rows, micro, kern, variants)
    assert s["rows_frac"] == {"a5_partial_eval": 0.965, "a9_tree": None}
    assert s["micro_ms_frac"] == {"gkr_round_2^26_keys": [2.845, 0.564], "ffn_statement": [41.6, None]}
    assert s["kernels_ms"] == {"gkr_round": 28.61}  # kernels under 0.2 ms per proof are left out
    assert s["lookup_variants_ms"] == {"gkr": 47.984, "hi": 53.427}
    assert "per_launch" not in json.dumps(s)


def test_summary_without_optional_parts():
    s = bench.compact_summary(None, None, {}, None)
    assert s == {"rows_frac": {}, "micro_ms_frac": {}, "kernels_ms": {}}
    assert len(json.dumps(s)) < 100
