"""The entry point that allocates nothing (swa_attn_fwd_noalloc), for callers that cannot
allocate device memory on the call path: plugins whose host framework owns all device memory,
or latency-critical loops where an allocation, which may synchronise the device, is not
allowed.  Its scratch is a fixed array inside the library.

Checked here through the C ABI: on two calls in a row its output equals swa_attn_fwd's on the
same inputs bit for bit (the same kernels run on the same inputs, and every output tile is
computed in a fixed order, so any difference would come from stale or shared scratch); and sizes
beyond the fixed scratch are refused before anything runs.  This file is collected last on
purpose."""
import pytest
import torch

import workloads
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield


def _call_noalloc(swa, s, dev, out, lse):
    P = lambda t: None if t is None else t.data_ptr()
    return swa.swa_attn_fwd_noalloc(P(dev["q"]), P(dev["k"]), P(dev["v"]), P(dev["ve"]), P(dev["gate_x"]),
                                    P(dev["Wg"]), out.data_ptr(), lse.data_ptr(), s.B, s.T, s.H, s.D,
                                    s.window, 10000.0, 1e-6, torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("s", [
    workloads.GPT2,
    workloads.LayerShape(B=2, T=1000, H=3, D=128, window=300, ve=True, seed=77, vocab=4096, model_dim=384,
                         name="(2,1000,3,128) W=300 VE"),
], ids=["gpt2_124m", "ve_window"])
def test_noalloc_matches_fwd_on_two_calls_in_a_row(s):
    import causal_sliding_window_swa_b200 as swa
    assert swa.swa_attn_workspace_bytes(s.B, s.T, s.H, s.D, int(s.ve)) <= swa.swa_attn_noalloc_scratch_bytes()
    dev = parity.to_device(workloads.make_layer(s))
    ref_out, ref_lse = swa.forward(dev["q"], dev["k"], dev["v"], s.window, dev["ve"], dev["gate_x"], dev["Wg"])
    swa.check_device_status()
    for _ in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        assert _call_noalloc(swa, s, dev, out, lse) == swa.SWA_OK
        swa.check_device_status()
        assert torch.equal(out, ref_out), "noalloc output differs from swa_attn_fwd's"
        assert torch.equal(lse, ref_lse), "noalloc lse differs from swa_attn_fwd's"


def test_noalloc_refuses_sizes_beyond_its_scratch():
    import causal_sliding_window_swa_b200 as swa
    s = workloads.D24_S
    assert swa.swa_attn_workspace_bytes(s.B, s.T, s.H, s.D, 0) > swa.swa_attn_noalloc_scratch_bytes()
    # Real buffers of the full size, so that even a missing check could not touch foreign memory.
    q = torch.zeros((s.B, s.T, s.H, s.D), dtype=torch.bfloat16, device="cuda")
    out = torch.full_like(q, 3.0)
    lse = torch.full((s.B, s.H, s.T), 3.0, dtype=torch.float32, device="cuda")
    dev = dict(q=q, k=q, v=q, ve=None, gate_x=None, Wg=None)
    assert _call_noalloc(swa, s, dev, out, lse) == swa.SWA_ERR_NO_MEMORY
    torch.cuda.synchronize()
    assert (out == 3.0).all().item() and (lse == 3.0).all().item()
