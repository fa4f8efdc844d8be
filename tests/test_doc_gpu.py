"""GPU parity of the document-boundary mask (swa_attn_fwd_doc through the C ABI) against the
oracle's forward with document ids, element by element.

The pages mention masking at document boundaries only as a change that was tried (intelliparadigm
"GPT-2 for $73", section 7, the variable-length attention item).  Reading: packed documents are
runs of equal ids; key j is visible to query i iff 0 <= i - j < W and doc[j] == doc[i]; RoPE keeps
the sequence positions.  The documents drawn here are contiguous runs numbered in order, for which
the kernel's run starts and the oracle's equal-id test are the same mask."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests import parity

pytestmark = pytest.mark.gpu

swa = pytest.importorskip("causal_sliding_window_swa_b200")


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield


def _docs(B, T, n_cuts, seed):
    """Contiguous documents: ids 0, 1, 2, ... increasing at n_cuts seeded cut points per row."""
    g = torch.Generator().manual_seed(seed)
    doc = torch.zeros((B, T), dtype=torch.int64)
    for b in range(B):
        for c in sorted(set(torch.randint(1, T, (n_cuts,), generator=g).tolist())):
            doc[b, c:] += 1
    return doc


def _run(s, d, doc, window):
    dev = parity.to_device(d)
    out = torch.full((s.B, s.T, s.H, s.D), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((s.B, s.H, s.T), float("nan"), dtype=torch.float32, device="cuda")
    swa.forward(dev["q"], dev["k"], dev["v"], window, dev["ve"], dev["gate_x"], dev["Wg"], out=out, lse=lse,
                doc=doc.to(torch.int32).cuda())
    swa.check_device_status()
    return out, lse


@pytest.mark.parametrize("B,T,H,Hkv,D,window,ve,cuts", [
    (2, 700, 4, 2, 128, 0, True, 5),
    (2, 700, 4, 4, 128, 300, False, 3),
    (1, 1000, 2, 2, 128, 40, True, 12),
    (2, 513, 3, 3, 64, 0, False, 4),
    (1, 900, 4, 1, 64, 129, True, 7),
    (1, 640, 2, 2, 128, 1, False, 6),
])
def test_document_mask_matches_the_oracle(B, T, H, Hkv, D, window, ve, cuts):
    s = workloads.LayerShape(B=B, T=T, H=H, D=D, window=window, ve=ve, seed=T + cuts, vocab=4096,
                             model_dim=max(32, H * D), kv_heads=Hkv)
    d = workloads.make_layer(s)
    doc = _docs(B, T, cuts, seed=cuts)
    out, lse = _run(s, d, doc, window)
    ro, rl = oracle.forward(d, window, parity=True, doc=doc)
    err = parity.compare(out.float().cpu().numpy(), lse.cpu().numpy(), ro, rl,
                         f"doc ({B},{T},{H}/{Hkv},{D}) W={window} ve={ve} cuts={cuts}")
    print(err)


def test_one_document_equals_the_plain_layer_bitwise():
    s = workloads.LayerShape(B=2, T=600, H=2, D=128, window=200, ve=True, seed=3, vocab=4096, model_dim=256)
    d = workloads.make_layer(s)
    dev = parity.to_device(d)
    o0, l0 = swa.forward(dev["q"], dev["k"], dev["v"], s.window, dev["ve"], dev["gate_x"], dev["Wg"])
    o1, l1 = _run(s, d, torch.full((s.B, s.T), 7, dtype=torch.int64), s.window)
    assert torch.equal(o0, o1) and torch.equal(l0, l1)


def test_one_token_documents_return_their_own_value():
    """Every position its own document: each row sees only itself, so out = v' of that row (the
    weights sum to one) and lse = its own score."""
    s = workloads.LayerShape(B=1, T=300, H=2, D=64, window=0, ve=False, seed=9, vocab=4096, model_dim=128)
    d = workloads.make_layer(s)
    doc = torch.arange(s.T, dtype=torch.int64).view(1, -1)
    out, lse = _run(s, d, doc, 0)
    assert torch.equal(out.cpu(), d["v"])
    ro, rl = oracle.forward(d, 0, parity=True, doc=doc)
    assert np.abs(lse.cpu().numpy() - rl).max() <= parity.LSE_MAX_ABS
