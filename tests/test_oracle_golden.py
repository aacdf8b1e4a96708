"""The oracle still reproduces the frozen toy-decode fixture (regression pin)."""
import json
import os

import numpy as np

import oracle
import synth

HERE = os.path.dirname(os.path.abspath(__file__))


def test_toy_decode_golden():
    doc = json.load(open(os.path.join(HERE, "golden", "toy_decode_4k.json")))
    x = synth.generate(synth.spec(doc["spec"]))
    assert {f"{b},{h}": v.tolist() for (b, h), v in x.needle_pos.items()} == doc["needles"]
    for hd in doc["heads"]:
        r = oracle.layer_rows(x, 0, hd["head"], [0])
        assert int(r.count[0]) == hd["count"]
        assert r.sel[0][:8].tolist() == hd["selected_head"]
        assert r.sel[0][-8:].tolist() == hd["selected_tail"]
        assert np.allclose(r.out[0, :8], hd["out_first8"], rtol=1e-12, atol=1e-14)
        assert abs(float(np.linalg.norm(r.out[0])) - hd["out_l2"]) <= 1e-12 * max(1.0, hd["out_l2"])
