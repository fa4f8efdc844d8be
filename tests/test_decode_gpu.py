"""GPU parity of the decode step (one new token per sequence, key/value cache; the cache is listed
among the pieces the "Let's reproduce GPT-2 (124M)" notes leave out, section 19).  A whole
sequence is generated token by token through the C ABI: step `pos` must return the oracle's
forward row `pos` (same tolerances as the prefill path), and the cache entries it writes must be
bit-identical to the oracle's rounded khat / v' -- the prefill path's values for that token."""
import numpy as np
import pytest
import torch

import causal_sliding_window_swa_b200 as swa
import oracle
import workloads
from tests import parity

pytestmark = pytest.mark.gpu

CASES = [
    workloads.LayerShape(B=2, T=160, H=3, D=64, window=0, ve=False, seed=11, name="decode D64 full"),
    workloads.LayerShape(B=2, T=200, H=2, D=128, window=48, ve=True, seed=12, name="decode D128 W48 VE"),
    workloads.LayerShape(B=1, T=300, H=2, D=128, window=1, ve=False, seed=13, name="decode D128 W1"),
    workloads.LayerShape(B=1, T=260, H=1, D=64, window=129, ve=True, seed=14, name="decode D64 W129 VE"),
    # grouped-query layers: caches with Hkv heads, query head h reads key/value head h / (H/Hkv)
    workloads.LayerShape(B=2, T=180, H=4, D=64, window=50, ve=True, seed=15, kv_heads=2, name="decode gqa D64 H4/2 W50 VE"),
    workloads.LayerShape(B=1, T=260, H=6, D=128, window=0, ve=False, seed=16, kv_heads=3, name="decode gqa D128 H6/3 full"),
    # many rows: few chunks per row, each longer than the four-stage tile ring
    workloads.LayerShape(B=8, T=600, H=12, D=128, window=0, ve=True, seed=17, name="decode D128 96 rows full VE"),
    workloads.LayerShape(B=16, T=1000, H=12, D=64, window=700, ve=False, seed=18, name="decode D64 192 rows W700"),
]


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield


def _bits(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16)


def _generate(s, dev):
    B, T, H, D = s.B, s.T, s.H, s.D
    k_cache = torch.zeros((B, T, s.Hkv, D), dtype=torch.bfloat16, device="cuda")
    v_cache = torch.zeros_like(k_cache)
    out = torch.empty((B, T, H, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    ws = torch.empty(swa.swa_attn_decode_workspace_bytes(B, T, H, D, s.ve, s.window), dtype=torch.uint8,
                     device="cuda")
    for pos in range(T):
        tok = {n: (None if dev[n] is None else dev[n][:, pos].contiguous()) for n in ("q", "k", "v", "ve", "gate_x")}
        o, l = swa.decode(tok["q"], tok["k"], tok["v"], k_cache, v_cache, pos, s.window, ve=tok["ve"],
                          gate_x=tok["gate_x"], Wg=dev["Wg"], workspace=ws)
        out[:, pos] = o
        lse[:, :, pos] = l
    swa.check_device_status()
    return out, lse, k_cache, v_cache


@pytest.mark.parametrize("s", CASES, ids=[c.name for c in CASES])
def test_decode_sequence_matches_oracle(s):
    d = workloads.make_layer(s)
    out, lse, k_cache, v_cache = _generate(s, parity.to_device(d))
    ref_o, ref_l = oracle.forward(d, s.window, parity=True)
    err = parity.compare(out.float().cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, s.name)
    print(f"{s.name}: {err}")
    # the cache holds exactly the prologue's rounded khat / v'
    _, kh, vp = oracle.prologue(d, eps=float(np.float32(1e-6)), parity=True)
    assert (k_cache.view(torch.int16).cpu() != _bits(kh)).sum().item() == 0
    assert (v_cache.view(torch.int16).cpu() != _bits(vp)).sum().item() == 0


def test_decode_rejects_position_outside_cache():
    B, T, H, D = 1, 8, 1, 64
    x = torch.zeros((B, H, D), dtype=torch.bfloat16, device="cuda")
    cache = torch.zeros((B, T, H, D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(swa.SwaError):
        swa.decode(x, x, x, cache, cache.clone(), T, 0)
