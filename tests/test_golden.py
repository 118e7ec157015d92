"""The oracle reproduces its committed regression fixture (tests/golden)."""
import json
import os

import numpy as np

import synth

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_matches_golden_fixture(orc):
    g = json.load(open(os.path.join(HERE, "golden", "tiny_ragged_oracle.json")))
    w = synth.WORKLOADS["tiny_ragged"]
    q, k, v, cu = synth.make_ragged(w, "cpu")
    rows = np.array(g["rows"], dtype=np.int32)
    o, lse = orc.attn_ragged_rows(synth.bf16_bits(q), synth.bf16_bits(k),
                                  synth.bf16_bits(v), cu, cu, w.Hq, w.Hkv, w.scale,
                                  True, rows)
    assert np.allclose(lse, g["lse"], rtol=0, atol=1e-12)
    for i, vals in g["o_rows"].items():
        assert np.allclose(o[int(i)], vals, rtol=0, atol=1e-12)
    assert abs(float(np.sum(o)) - g["checksum_o"]) < 1e-9
