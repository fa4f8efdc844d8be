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
