"""Pins of the oracle's fused projection + prologue (q, k, v = x Wqkv^T, then RoPE, RMS and the
gated value embedding) against things other than itself.  CPU only.

The projection is the bias-free linear map of the layer input ("Let's reproduce GPT-2 (124M)"
notes, section 3, the attention listing; intelliparadigm "GPT-2 for $73", section 2); the prologue
is the one the forward pins fix (section 2.2 there; PaperWeekly repost, "Value Embeddings").
"""
import numpy as np
import pytest
import torch

import oracle


def _draw(B, T, C, H, Hkv, D, ve, seed, vocab=11):
    g = torch.Generator().manual_seed(seed)
    bf = lambda *shape, std=1.0: (torch.randn(shape, generator=g) * std).to(torch.bfloat16)
    d = dict(x=bf(B, T, C), W=bf((H + 2 * Hkv) * D, C, std=C ** -0.5))
    if ve:
        d.update(ids=torch.randint(0, vocab, (B, T), generator=g), table=bf(vocab, Hkv * D),
                 Wg=bf(32, Hkv, std=0.3))
    return d


def _call(d, H, Hkv, D, **kw):
    return oracle.qkv_prologue(d["x"], d["W"], H, Hkv, D, ids=d.get("ids"), table=d.get("table"),
                               Wg=d.get("Wg"), **kw)


@pytest.mark.parametrize("H,Hkv,D,ve,parity", [(2, 2, 16, True, False), (4, 2, 8, True, True),
                                               (3, 1, 16, False, True), (2, 2, 64, True, True)])
def test_permutation_weights_reduce_to_the_prologue_bit_for_bit(H, Hkv, D, ve, parity):
    """With each projection row picking one input channel (a 0/1 selection matrix), q, k, v are
    exact copies of x's channels, so the fused result equals the already-pinned prologue applied
    to those copies, bit for bit."""
    B, T = 2, 19
    C = max(32, H * D)
    d = _draw(B, T, C, H, Hkv, D, ve, seed=H * 7 + D)
    g = torch.Generator().manual_seed(5)
    n_out = (H + 2 * Hkv) * D
    pick = torch.randint(0, C, (n_out,), generator=g)
    W = torch.zeros((n_out, C), dtype=torch.bfloat16)
    W[torch.arange(n_out), pick] = 1.0
    d["W"] = W
    qh, kh, vp = _call(d, H, Hkv, D, parity=parity)
    sel = d["x"][..., pick]                                   # (B, T, n_out), exact copies
    inputs = dict(q=sel[..., :H * D].reshape(B, T, H, D).contiguous(),
                  k=sel[..., H * D:(H + Hkv) * D].reshape(B, T, Hkv, D).contiguous(),
                  v=sel[..., (H + Hkv) * D:].reshape(B, T, Hkv, D).contiguous())
    if ve:
        inputs.update(ids=d["ids"], table=d["table"], x=d["x"], Wg=d["Wg"])
    rq, rk, rv = oracle.prologue(inputs, parity=parity)
    assert np.array_equal(qh, rq) and np.array_equal(kh, rk) and np.array_equal(vp, rv)


def test_projection_alone_equals_numpy_matmul():
    """RoPE and the norm switched off (test flags), no value embedding: the outputs are the
    projection itself, checked against NumPy's fp64 matrix product."""
    B, T, C, H, Hkv, D = 2, 13, 96, 3, 1, 16
    d = _draw(B, T, C, H, Hkv, D, False, seed=9)
    qh, kh, vp = _call(d, H, Hkv, D, rope=False, qknorm=False)
    y = d["x"].double().numpy() @ d["W"].double().numpy().T
    got = np.concatenate([qh.reshape(B, T, -1), kh.reshape(B, T, -1), vp.reshape(B, T, -1)], -1)
    assert np.abs(got - y).max() <= 1e-12 * np.abs(y).max()


def test_doubling_the_weights_leaves_the_normalised_rows_unchanged():
    """At eps = 0 the RMS norm removes any positive scale; doubling (exact in bf16) changes no bit
    of qhat or khat, while v' (not normalised) doubles its projection part."""
    B, T, C, H, Hkv, D = 1, 11, 64, 2, 2, 16
    d = _draw(B, T, C, H, Hkv, D, False, seed=4)
    q1, k1, v1 = _call(d, H, Hkv, D, eps=0.0)
    d2 = dict(d, W=(d["W"].float() * 2).to(torch.bfloat16))
    q2, k2, v2 = _call(d2, H, Hkv, D, eps=0.0)
    assert np.array_equal(q1, q2) and np.array_equal(k1, k2)
    assert np.array_equal(v2, 2 * v1)


def test_rejects_bad_weight_shape():
    d = _draw(1, 4, 32, 2, 1, 8, False, seed=1)
    with pytest.raises(ValueError):
        oracle.qkv_prologue(d["x"], d["W"][:-1], 2, 1, 8)
