"""The tensor-level calls refuse tensors whose shape, dtype or device does not match the layer
before any C call: the C ABI takes bare pointers and could not see the mistake, which would turn
into writes outside the caller's buffers.  No kernel is launched here."""
import os
import subprocess
import sys

import pytest
import torch

import causal_sliding_window_swa_b200 as swa

pytestmark = pytest.mark.gpu

B, T, H, D = 1, 32, 2, 64


def _layer():
    g = torch.Generator().manual_seed(0)
    mk = lambda *shape: torch.randn(*shape, generator=g).to(torch.bfloat16).cuda()
    return mk(B, T, H, D), mk(B, T, H, D), mk(B, T, H, D)


def test_forward_refuses_wrong_outputs():
    q, k, v = _layer()
    with pytest.raises(ValueError, match="out must have shape"):
        swa.forward(q, k, v, 0, out=torch.empty((B, T, H, D + 8), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError, match="out must be torch.bfloat16"):
        swa.forward(q, k, v, 0, out=torch.empty((B, T, H, D), dtype=torch.float16, device="cuda"))
    with pytest.raises(ValueError, match="lse must have shape"):
        swa.forward(q, k, v, 0, lse=torch.empty((B, T, H), dtype=torch.float32, device="cuda"))
    with pytest.raises(ValueError, match="contiguous CUDA"):
        swa.forward(q, k, v, 0, out=torch.empty((B, T, D, H), dtype=torch.bfloat16, device="cuda").transpose(2, 3))
    with pytest.raises(ValueError, match="workspace"):
        swa.forward(q, k, v, 0, workspace=torch.empty(1 << 20, dtype=torch.uint8))
    with pytest.raises(ValueError, match="doc must be torch.int32"):
        swa.forward(q, k, v, 0, doc=torch.zeros((B, T), dtype=torch.int64, device="cuda"))


def test_backward_refuses_wrong_tensors():
    q, k, v = _layer()
    out = torch.empty_like(q)
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError, match="dout must have shape"):
        swa.backward(q, k, v, out, lse, out[:, : T - 1])
    with pytest.raises(ValueError, match="dlse must have shape"):
        swa.backward(q, k, v, out, lse, out, dlse=lse[:, :1])
    with pytest.raises(ValueError, match="lse must be torch.float32"):
        swa.backward(q, k, v, out, lse.double(), out)


def test_decode_refuses_wrong_tensors():
    Tmax = 16
    x = torch.zeros((B, H, D), dtype=torch.bfloat16, device="cuda")
    cache = torch.zeros((B, Tmax, H, D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError, match="v_cache must have shape"):
        swa.decode(x, x, x, cache, cache[:, :, :1].contiguous(), 3, 0)
    with pytest.raises(ValueError, match="k must have shape"):
        swa.decode(x, x[:, :1, :32], x, cache, cache.clone(), 3, 0)
    with pytest.raises(ValueError, match="ve, gate_x and Wg go together"):
        swa.decode(x, x, x, cache, cache.clone(), 3, 0, ve=x)
    with pytest.raises(ValueError, match="gate_x must have shape"):
        swa.decode(x, x, x, cache, cache.clone(), 3, 0, ve=x,
                   gate_x=torch.zeros((B, 16), dtype=torch.bfloat16, device="cuda"),
                   Wg=torch.zeros((32, H), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError, match="lse must have shape"):
        swa.decode(x, x, x, cache, cache.clone(), 3, 0, lse=torch.empty((B, H + 1), device="cuda"))
    with pytest.raises(ValueError, match="doc_start must be torch.int32"):
        swa.decode(x, x, x, cache, cache.clone(), 3, 0, doc_start=torch.zeros(B, device="cuda"))


def test_fused_projection_refuses_wrong_weights():
    C = 128
    x = torch.zeros((B, T, C), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((3 * H * D, C), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError, match="Wqkv must have shape"):
        swa.forward_x(x, W[:-1], H, H, D)
    with pytest.raises(ValueError, match="contiguous CUDA"):
        swa.forward_x(x, W.cpu(), H, H, D)
    with pytest.raises(ValueError, match="workspace"):
        swa.forward_x(x, W, H, H, D, workspace=torch.empty(1 << 20, dtype=torch.uint8))


def test_first_calls_from_several_threads():
    # A fresh process whose first library calls come from four threads at once, each on its own
    # stream: the lazy load, the per-device checks and the shared workspace are set up once and
    # every thread gets the serial result bit for bit.
    code = """
import threading, torch
import causal_sliding_window_swa_b200 as swa
torch.cuda.set_device(0)
g = torch.Generator().manual_seed(1)
q, k, v = (torch.randn(2, 300, 2, 64, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
torch.cuda.synchronize()
res = [None] * 4
go = threading.Barrier(4)
def run(i):
    torch.cuda.set_device(0)
    s = torch.cuda.Stream()
    go.wait()
    with torch.cuda.stream(s):
        res[i] = swa.forward(q, k, v, 100)
    s.synchronize()
ts = [threading.Thread(target=run, args=(i,)) for i in range(4)]
[t.start() for t in ts]
[t.join() for t in ts]
ref = swa.forward(q, k, v, 100)
torch.cuda.synchronize()
swa.check_device_status()
assert all(torch.equal(r[0], ref[0]) and torch.equal(r[1], ref[1]) for r in res)
print("threads ok")
"""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "threads ok" in r.stdout, r.stdout + r.stderr
