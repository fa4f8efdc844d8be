"""Write tests/golden/tiny_oracle_rows.json: oracle outputs for sampled rows of the tiny
workload, so that later edits of the oracle that change its results are noticed.
Calls only ``oracle`` and the seeded input generator."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle      # noqa: E402
import workloads   # noqa: E402


def main():
    s = workloads.TINY
    d = workloads.make_layer(s)
    rows = workloads.sample_rows(s, n_random=4, seed=123)
    out, lse = oracle.forward(d, s.window, parity=True, rows=rows)
    doc = {
        "_about": "oracle (parity mode) rows of the tiny workload (1,256,4,64), full causal, "
                  "seed 0; written by tests/golden/make_golden.py",
        "workload": s.name,
        "input_sha256": workloads.sha256_of(d),
        "rows": rows.tolist(),
        "out": [[float(x) for x in r] for r in out],
        "lse": [float(x) for x in lse],
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle_rows.json")
    with open(path, "w") as f:
        json.dump(doc, f, indent=0)
    print(path)


if __name__ == "__main__":
    main()
