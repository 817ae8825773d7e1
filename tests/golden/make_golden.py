"""Write the stored oracle regression values under tests/golden/.

The pages describing HSTU (the arXiv 2402.17152 abstract and the
generative-recommenders README) print no worked example, so no stored value
here comes from them. These fixtures hold oracle outputs on seeded inputs;
they guard the oracle against silent drift (the pins in test_oracle_pins.py
are what tie it to the mathematics). This script calls only ``gen`` and
``oracle``.

    python tests/golden/make_golden.py
"""

import hashlib
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from gen import make_attn_inputs  # noqa: E402


def digest(*arrays) -> str:
    h = hashlib.sha256()
    for a in arrays:
        h.update(np.ascontiguousarray(a).tobytes())
    return h.hexdigest()


def main():
    inp = make_attn_inputs(1)
    rows = sorted({0, 1, int(inp.seq_offsets[1]) - 1, int(inp.seq_offsets[1]), inp.T // 2,
                   inp.T - 2, inp.T - 1})
    out = oracle.attn(inp.seq_offsets, inp.q, inp.k, inp.v, inp.timestamps, inp.pos_bias,
                      inp.time_bias, inp.max_seqlen, rows=rows)
    rec = {
        "what": "HSTU attention forward, fp64 oracle, tiny fp32 workload (seed 1001)",
        "written_by": "tests/golden/make_golden.py (gen + oracle only)",
        "inputs_sha256": digest(inp.seq_offsets, inp.timestamps, inp.q, inp.k, inp.v,
                                inp.pos_bias, inp.time_bias),
        "max_seqlen": inp.max_seqlen,
        "rows": rows,
        "out": [[[float.hex(float(x)) for x in head] for head in row] for row in out],
    }
    with open(os.path.join(HERE, "oracle_tiny_fp32.json"), "w") as f:
        json.dump(rec, f, indent=0)
        f.write("\n")


if __name__ == "__main__":
    main()
