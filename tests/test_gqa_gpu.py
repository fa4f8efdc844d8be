"""GPU parity of grouped-query attention (Hkv key/value heads shared by H / Hkv query heads; the
pages size the key/value projection separately, as kv_dim: intelliparadigm "GPT-2 for $73", model
section).  Every element of out and lse against the oracle, and bit-for-bit agreement with the
multi-head call on key/value heads repeated H / Hkv times."""
import pytest
import torch

import causal_sliding_window_swa_b200 as swa
import workloads
from tests import parity

pytestmark = pytest.mark.gpu

CASES = [
    workloads.LayerShape(B=2, T=300, H=4, D=64, window=100, ve=False, seed=21, kv_heads=2, name="gqa D64 H4/2 W100"),
    workloads.LayerShape(B=1, T=520, H=6, D=128, window=0, ve=True, seed=22, kv_heads=2, name="gqa D128 H6/2 full VE"),
    workloads.LayerShape(B=2, T=256, H=4, D=128, window=64, ve=False, seed=23, kv_heads=1, name="gqa D128 H4/1 W64"),
]


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield


@pytest.mark.parametrize("s", CASES, ids=[c.name for c in CASES])
def test_gqa_matches_oracle(s):
    err = parity.check_full(s)
    print(f"{s.name}: {err}")


@pytest.mark.parametrize("s", CASES[:2], ids=[c.name for c in CASES[:2]])
def test_gqa_equals_multihead_on_repeated_kv_heads(s):
    dev = parity.to_device(workloads.make_layer(s))
    G = s.H // s.Hkv
    o_g, l_g = parity.run_gpu(s, dev)
    rep = dict(dev)
    rep["k"] = dev["k"].repeat_interleave(G, dim=2).contiguous()
    rep["v"] = dev["v"].repeat_interleave(G, dim=2).contiguous()
    if dev["ve"] is not None:
        rep["ve"] = dev["ve"].repeat_interleave(G, dim=2).contiguous()
        rep["Wg"] = dev["Wg"].repeat_interleave(G, dim=1).contiguous()
    o_m, l_m = parity.run_gpu(s, rep)
    assert torch.equal(o_g.view(torch.int16), o_m.view(torch.int16))
    assert torch.equal(l_g, l_m)
