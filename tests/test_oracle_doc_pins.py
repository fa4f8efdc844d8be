"""Pins of the oracle's document-boundary mask (key j visible to query i only inside the causal
window and the same document).  CPU only.

The pages mention masking at document boundaries only as something tried and dropped (the
intelliparadigm write-up's list of changes that did not help); the reading taken here keeps the
sequence positions for RoPE and only narrows the set of visible keys.
"""
import numpy as np
import pytest
import torch

import oracle
import oracle.brute as brute
import workloads


def _layer(B, T, H, D, ve, seed):
    s = workloads.LayerShape(B=B, T=T, H=H, D=D, window=0, ve=ve, seed=seed, vocab=97,
                             model_dim=max(32, H * D))
    return workloads.make_layer(s)


def _docs(B, T, n_cuts, seed):
    g = torch.Generator().manual_seed(seed)
    doc = torch.zeros((B, T), dtype=torch.int64)
    for b in range(B):
        cuts = sorted(set(torch.randint(1, T, (n_cuts,), generator=g).tolist()))
        for c in cuts:
            doc[b, c:] += 1
    return doc


def test_one_document_is_the_plain_layer_bit_for_bit():
    d = _layer(2, 60, 3, 16, True, 1)
    o0, l0 = oracle.forward(d, 9)
    o1, l1 = oracle.forward(d, 9, doc=torch.zeros((2, 60), dtype=torch.int64))
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)


@pytest.mark.parametrize("window", [0, 1, 7, 40])
@pytest.mark.parametrize("ve", [False, True])
def test_documents_match_bruteforce(window, ve):
    d = _layer(2, 70, 2, 16, ve, window + 3)
    doc = _docs(2, 70, 4, window)
    o, l = oracle.forward(d, window, parity=False, doc=doc)
    ob, lb = brute.forward(d, window, doc=doc)
    assert np.abs(o - ob).max() < 1e-12 and np.abs(l - lb).max() < 1e-12


def test_each_document_is_the_layer_on_its_own_slice():
    """RoPE makes scores depend on relative positions only, so (in fp64, no bf16 rounding) the
    rows of a document starting at s equal the plain layer run on that document alone, whose
    positions start at 0."""
    B, T, H, D, W = 1, 90, 2, 32, 25
    d = _layer(B, T, H, D, True, 5)
    doc = torch.zeros((B, T), dtype=torch.int64)
    doc[0, 30:] = 1
    doc[0, 71:] = 2
    o, l = oracle.forward(d, W, parity=False, doc=doc)
    for s0, e0 in ((0, 30), (30, 71), (71, 90)):
        part = {k: (v[:, s0:e0].contiguous() if k in ("q", "k", "v", "ids", "x") else v) for k, v in d.items()}
        op, lp = oracle.forward(part, W, parity=False)
        assert np.abs(o[:, s0:e0] - op).max() < 1e-12
        assert np.abs(l[:, :, s0:e0] - lp).max() < 1e-12


def test_first_row_of_each_document_is_its_own_value():
    B, T, H, D = 1, 40, 2, 16
    d = _layer(B, T, H, D, True, 6)
    doc = _docs(B, T, 3, 11)
    o, _ = oracle.forward(d, 0, parity=False, doc=doc)
    _, _, vp = oracle.prologue(d, parity=False)
    starts = [0] + [t for t in range(1, T) if doc[0, t] != doc[0, t - 1]]
    for t in starts:
        assert np.abs(o[0, t] - vp[0, t]).max() < 1e-12


# ------------------------------------------------------------------- the gradient with documents

def _fd_grads(d, window, dout, dlse, doc):
    """Central differences of the brute-force forward with its own document mask."""
    inp = {k: (v.numpy().copy() if k == "ids" else v.double().numpy().copy()) for k, v in d.items()}

    def loss():
        o, l = brute.forward(inp, window, doc=doc)
        return float(np.sum(o * dout) + np.sum(l * dlse))

    out = {}
    for name in ("q", "k", "v"):
        a = inp[name]
        g = np.zeros_like(a)
        for idx in np.ndindex(a.shape):
            old = a[idx]
            h = 1e-5 * max(1.0, abs(old))
            a[idx] = old + h
            lp = loss()
            a[idx] = old - h
            lm = loss()
            a[idx] = old
            g[idx] = (lp - lm) / (2 * h)
        out[name] = g
    return out


@pytest.mark.parametrize("window", [0, 3])
def test_gradient_with_documents_matches_central_differences(window):
    B, T, H, D = 1, 9, 2, 8
    d = _layer(B, T, H, D, False, 40 + window)
    doc = torch.tensor([[0, 0, 0, 1, 1, 1, 1, 2, 2]])
    g = torch.Generator().manual_seed(window)
    dout = torch.randn((B, T, H, D), generator=g, dtype=torch.float64).numpy()
    dlse = torch.randn((B, H, T), generator=g, dtype=torch.float64).numpy()
    got = oracle.backward(d, dout, window, dlse=dlse, doc=doc)
    fd = _fd_grads(d, window, dout, dlse, doc)
    for key, name in (("dq", "q"), ("dk", "k"), ("dv", "v")):
        assert np.all(np.abs(got[key] - fd[name]) <= 1e-7 + 1e-6 * np.abs(fd[name])), key


def test_gradient_with_one_document_is_the_plain_gradient_bit_for_bit():
    B, T, H, D = 2, 30, 3, 16
    d = _layer(B, T, H, D, True, 9)
    g = torch.Generator().manual_seed(2)
    dout = torch.randn((B, T, H, D), generator=g, dtype=torch.float64).numpy()
    dlse = torch.randn((B, H, T), generator=g, dtype=torch.float64).numpy()
    a = oracle.backward(d, dout, 7, dlse=dlse)
    b = oracle.backward(d, dout, 7, dlse=dlse, doc=torch.zeros((B, T), dtype=torch.int64))
    for key in a:
        assert np.array_equal(a[key], b[key]), key


def test_gradient_of_each_document_is_the_gradient_on_its_own_slice():
    """In fp64 the documents are independent layers (relative positions only), so each one's
    gradient equals the plain gradient of the layer run on its slice alone."""
    B, T, H, D, W = 1, 50, 2, 16, 12
    d = _layer(B, T, H, D, True, 13)
    doc = torch.zeros((B, T), dtype=torch.int64)
    doc[0, 22:] = 1
    g = torch.Generator().manual_seed(3)
    dout = torch.randn((B, T, H, D), generator=g, dtype=torch.float64).numpy()
    dlse = torch.randn((B, H, T), generator=g, dtype=torch.float64).numpy()
    full = oracle.backward(d, dout, W, dlse=dlse, doc=doc)
    for s0, e0 in ((0, 22), (22, 50)):
        part = {k: (v[:, s0:e0].contiguous() if k in ("q", "k", "v", "ids", "x") else v) for k, v in d.items()}
        gp = oracle.backward(part, dout[:, s0:e0], W, dlse=dlse[:, :, s0:e0])
        for key in ("dq", "dk", "dv", "dve", "dx"):
            assert np.abs(full[key][:, s0:e0] - gp[key]).max() < 1e-11, (key, s0)
