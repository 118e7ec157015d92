"""Write tests/golden/tiny_ragged_oracle.json from the oracle alone.

The release pages print no worked numerical example for attention, so this
directory holds no page values.  What it holds is a regression fixture: the
fp64 oracle's result on the tiny ragged workload (2 sequences, q_len = kv_len
{37, 64}, Hq = 4, Hkv = 1, D = 64, causal, scale = 1/8, seed 1), written by
this script, which calls only ``oracle`` and the seeded generator ``synth``.
Re-run it only when a change to the oracle's arithmetic is justified by a
passage of the pages (name that passage in the commit message).

    python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import synth  # noqa: E402


def compute():
    w = synth.WORKLOADS["tiny_ragged"]
    q, k, v, cu = synth.make_ragged(w, "cpu")
    rows = [(b, h, i) for b, L in enumerate(w.lengths) for h in range(w.Hq) for i in range(L)]
    o, lse = oracle.default().attn_ragged_rows(
        synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v), cu, cu,
        w.Hq, w.Hkv, w.scale, True, rows)
    pick = [0, 1, 36, 37, 100, 147, 148, len(rows) - 1]
    return rows, o, lse, pick


def main():
    rows, o, lse, pick = compute()
    out = {
        "workload": "tiny_ragged (seed 1): lengths {37, 64}, Hq 4, Hkv 1, D 64, causal, scale 1/8",
        "rows": [list(map(int, r)) for r in rows],
        "lse": [float(x) for x in lse],
        "o_rows": {str(i): [float(x) for x in o[i]] for i in pick},
        "checksum_o": float(np.sum(o)),
    }
    with open(os.path.join(HERE, "tiny_ragged_oracle.json"), "w") as f:
        json.dump(out, f, indent=0)


if __name__ == "__main__":
    main()
