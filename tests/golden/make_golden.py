"""Write tests/golden/toy_decode_4k.json from the fp64 oracle (and nothing else).

The fixture freezes the oracle's answer on the seeded 4K decode toy (8 query heads,
2 KV heads, retrieval heads {0, 5}, W=512, S=4, p=0.9) so that a later change to the
oracle's arithmetic shows up as a failing regression test.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
import synth  # noqa: E402


def main():
    s = synth.spec("toy_decode_4k")
    x = synth.generate(s)
    heads = []
    for h in range(s.n_q_heads):
        r = oracle.layer_rows(x, 0, h, [0])
        heads.append({
            "head": h,
            "retrieval": h in s.retrieval_heads,
            "count": int(r.count[0]),
            "mass": float(r.mass[0]),
            "selected_head": [int(j) for j in r.sel[0][:8]],
            "selected_tail": [int(j) for j in r.sel[0][-8:]],
            "out_first8": [float(z) for z in r.out[0, :8]],
            "out_l2": float((r.out[0] ** 2).sum() ** 0.5),
        })
    doc = {
        "what": "fp64 oracle on the seeded 4K decode toy (seed 0); written by make_golden.py",
        "spec": "toy_decode_4k",
        "needles": {f"{b},{h}": [int(p) for p in v] for (b, h), v in x.needle_pos.items()},
        "heads": heads,
    }
    with open(os.path.join(HERE, "toy_decode_4k.json"), "w") as f:
        json.dump(doc, f, indent=1)


if __name__ == "__main__":
    main()
