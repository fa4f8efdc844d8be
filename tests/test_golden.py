"""Golden fixtures: the configuration values the pages print, and a frozen copy of oracle
rows (regression guard for the oracle).  CPU only."""
import json
import os

import numpy as np

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_sssl_schedule_matches_pages():
    pv = _load("page_values.json")
    w = pv["sssl_windows_d24"]["value"]
    layers = workloads.sssl_layer_shapes(16, 2048)
    for i, s in enumerate(layers):
        kind = w["pattern"][i % 4]
        assert s.window == (w["short"] if kind == "S" else w["long"])
        assert s.ve == (i % 2 == 0)            # even layer indices carry value embeddings


def test_single_layer_shapes_match_pages():
    pv = _load("page_values.json")
    g = pv["gpt2_124m_attention"]["value"]
    assert (workloads.GPT2.H * workloads.GPT2.D, workloads.GPT2.H, workloads.GPT2.D, workloads.GPT2.T) == \
        (g["C"], g["H"], g["D"], g["T"])
    m = pv["d24_model_dim"]["value"]
    assert workloads.D24_L_VE.H * workloads.D24_L_VE.D == m["depth"] * m["per_layer_multiplier"] == m["model_dim"]
    assert workloads.D24_S.window == pv["sssl_windows_d24"]["value"]["short"]
    assert workloads.D24_L_VE.window == pv["sssl_windows_d24"]["value"]["long"]
    assert workloads.GATE_CHANNELS == pv["gate"]["value"]["channels"]


def test_frozen_oracle_rows():
    doc = _load("tiny_oracle_rows.json")
    s = workloads.TINY
    d = workloads.make_layer(s)
    assert workloads.sha256_of(d) == doc["input_sha256"], "seeded input generator changed"
    out, lse = oracle.forward(d, s.window, parity=True, rows=doc["rows"])
    assert np.abs(out - np.array(doc["out"])).max() < 1e-12
    assert np.abs(lse - np.array(doc["lse"])).max() < 1e-12


def test_frozen_oracle_gradients_and_projection():
    import tests.golden.make_golden_grads as mg
    doc = _load("small_oracle_grads.json")
    d, dout, dlse, W = mg.inputs()
    assert workloads.sha256_of(d) == doc["input_sha256"], "seeded input generator changed"
    g = oracle.backward(d, dout, mg.SHAPE.window, dlse=dlse, parity=True)
    for k, v in doc["grads"].items():
        assert np.abs(g[k].reshape(-1) - np.array(v)).max() < 1e-12, k
    qh, kh, vp = oracle.qkv_prologue(d["x"], W, mg.SHAPE.H, mg.SHAPE.Hkv, mg.SHAPE.D, ids=d["ids"],
                                     table=d["table"], Wg=d["Wg"], parity=True)
    for k, v in (("qhat", qh), ("khat", kh), ("vprime", vp)):
        assert np.array_equal(v.reshape(-1), np.array(doc["qkv"][k])), k
