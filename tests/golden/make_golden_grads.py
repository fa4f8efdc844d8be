"""Write tests/golden/small_oracle_grads.json: the oracle's backward (parity mode) and its fused
projection + prologue on one small seeded grouped-query layer with value embeddings, so that later
edits of those oracle functions that change their results are noticed.  Calls only ``oracle`` and
the seeded input generator."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import torch       # noqa: E402

import oracle      # noqa: E402
import workloads   # noqa: E402

SHAPE = workloads.LayerShape(B=1, T=40, H=4, D=16, window=9, ve=True, seed=21, vocab=13, model_dim=64,
                             kv_heads=2, name="small gqa (1,40,4/2,16) W=9 + VE")


def inputs():
    d = workloads.make_layer(SHAPE)
    g = torch.Generator().manual_seed(77)
    dout = torch.randn((SHAPE.B, SHAPE.T, SHAPE.H, SHAPE.D), generator=g).to(torch.bfloat16)
    dlse = torch.randn((SHAPE.B, SHAPE.H, SHAPE.T), generator=g)
    W = (torch.randn(((SHAPE.H + 2 * SHAPE.Hkv) * SHAPE.D, SHAPE.C), generator=g) * 0.125).to(torch.bfloat16)
    return d, dout, dlse, W


def main():
    d, dout, dlse, W = inputs()
    g = oracle.backward(d, dout, SHAPE.window, dlse=dlse, parity=True)
    qh, kh, vp = oracle.qkv_prologue(d["x"], W, SHAPE.H, SHAPE.Hkv, SHAPE.D, ids=d["ids"], table=d["table"],
                                     Wg=d["Wg"], parity=True)
    doc = {
        "_about": "oracle backward (parity mode) and fused projection + prologue of the layer "
                  f"{SHAPE.name}; written by tests/golden/make_golden_grads.py",
        "input_sha256": workloads.sha256_of(d),
        "grads": {k: v.reshape(-1).tolist() for k, v in g.items()},
        "qkv": {"qhat": qh.reshape(-1).tolist(), "khat": kh.reshape(-1).tolist(), "vprime": vp.reshape(-1).tolist()},
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "small_oracle_grads.json")
    with open(path, "w") as f:
        json.dump(doc, f)
    print(path)


if __name__ == "__main__":
    main()
