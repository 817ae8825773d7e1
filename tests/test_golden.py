"""The oracle still reproduces its stored regression values (tests/golden/). CPU only."""

import json
import os

import numpy as np

import oracle
from gen import make_attn_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "oracle_tiny_fp32.json")


def test_oracle_matches_golden(oracle_lib):
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "make_golden", os.path.join(os.path.dirname(GOLDEN), "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    rec = json.load(open(GOLDEN))
    inp = make_attn_inputs(1)
    assert mg.digest(inp.seq_offsets, inp.timestamps, inp.q, inp.k, inp.v, inp.pos_bias,
                     inp.time_bias) == rec["inputs_sha256"], "generator drifted"
    got = oracle.attn(inp.seq_offsets, inp.q, inp.k, inp.v, inp.timestamps, inp.pos_bias,
                      inp.time_bias, rec["max_seqlen"], rows=rec["rows"], lib=oracle_lib)
    want = np.array([[[float.fromhex(x) for x in head] for head in row] for row in rec["out"]])
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-15)
