"""Pins of the oracle's backward (the gradient of the layer) against things other than itself:
central finite differences of the brute-force NumPy forward, torch autograd through an
independent fp64 forward, closed forms, and invariants.  CPU only.

The loss is sum(dout * out) + sum(dlse * lse).  The layer is the one the forward pins fix:
RoPE then RMS QK-norm (intelliparadigm "GPT-2 for $73", section 2.2), the gated value
embedding (PaperWeekly repost, "Value Embeddings" paragraph), causal windowed softmax attention
("Let's reproduce GPT-2 (124M)" notes, section 3; window from section 3.2 of the first page).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import oracle.brute as brute


def _draw(B, T, H, D, Hkv=None, ve=False, C=40, seed=0, unique_ids=True):
    """bf16 inputs.  With unique_ids the table has one row per position (ids = b*T + t), so the
    gradient of a table row is the gradient of the looked-up row at that position."""
    Hkv = H if Hkv is None else Hkv
    g = torch.Generator().manual_seed(seed)
    bf = lambda *shape, std=1.0: (torch.randn(shape, generator=g) * std).to(torch.bfloat16)
    d = dict(q=bf(B, T, H, D), k=bf(B, T, Hkv, D), v=bf(B, T, Hkv, D))
    if ve:
        if unique_ids:
            d["ids"] = torch.arange(B * T, dtype=torch.int64).view(B, T)
            vocab = B * T
        else:
            vocab = 5
            d["ids"] = torch.randint(0, vocab, (B, T), generator=g, dtype=torch.int64)
        d["table"] = bf(vocab, Hkv * D)
        d["x"] = bf(B, T, C)
        d["Wg"] = bf(32, Hkv, std=0.5)
    return d


def _cotangents(B, T, H, D, seed, with_lse=True):
    g = torch.Generator().manual_seed(10_000 + seed)
    dout = torch.randn((B, T, H, D), generator=g, dtype=torch.float64).numpy()
    dlse = torch.randn((B, H, T), generator=g, dtype=torch.float64).numpy() if with_lse else None
    return dout, dlse


def _as_f64_inputs(d):
    out = {}
    for key, t in d.items():
        out[key] = t.numpy().copy() if key == "ids" else t.double().numpy().copy()
    return out


# ------------------------------------------------------- central finite differences (brute force)

def _fd_gradients(d, window, dout, dlse, eps, rope, qknorm):
    """Central differences of the brute-force forward, element by element, over every float
    input (q, k, v, the table, all C channels of x, Wg)."""
    inp = _as_f64_inputs(d)

    def loss():
        o, l = brute.forward(inp, window, eps=eps, rope=rope, qknorm=qknorm)
        return float(np.sum(o * dout) + (np.sum(l * dlse) if dlse is not None else 0.0))

    grads = {}
    for name in ("q", "k", "v", "table", "x", "Wg"):
        if name not in inp:
            continue
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
            g[idx] = (lp - lm) / (2.0 * h)
        grads[name] = g
    return grads


def _close(a, b, atol=1e-7, rtol=1e-6):
    return np.all(np.abs(a - b) <= atol + rtol * np.abs(b))


@pytest.mark.parametrize("B,T,H,D,window,ve,rope,qknorm,with_lse", [
    (1, 6, 2, 8, 0, True, True, True, True),
    (1, 7, 1, 8, 3, True, True, True, True),
    (2, 5, 2, 4, 2, False, True, True, True),
    (1, 6, 2, 8, 1, True, True, True, True),
    (1, 6, 1, 8, 0, False, False, True, False),
    (1, 6, 1, 8, 4, False, True, False, True),
    (1, 5, 2, 4, 0, True, False, False, True),
])
def test_backward_matches_central_differences(B, T, H, D, window, ve, rope, qknorm, with_lse):
    d = _draw(B, T, H, D, ve=ve, seed=B * 100 + T * 10 + window)
    dout, dlse = _cotangents(B, T, H, D, seed=T + window, with_lse=with_lse)
    eps = 1e-6
    g = oracle.backward(d, dout, window, dlse=dlse, eps=eps, rope=rope, qknorm=qknorm)
    fd = _fd_gradients(d, window, dout, dlse, eps, rope, qknorm)
    assert _close(g["dq"], fd["q"]), np.abs(g["dq"] - fd["q"]).max()
    assert _close(g["dk"], fd["k"]), np.abs(g["dk"] - fd["k"]).max()
    assert _close(g["dv"], fd["v"]), np.abs(g["dv"] - fd["v"]).max()
    if ve:
        dtable = fd["table"].reshape(B, T, H, D)      # ids = b*T + t: one table row per position
        assert _close(g["dve"], dtable), np.abs(g["dve"] - dtable).max()
        assert _close(g["dx"], fd["x"][..., :32]), np.abs(g["dx"] - fd["x"][..., :32]).max()
        assert np.abs(fd["x"][..., 32:]).max() < 1e-9   # channels past the gate's 32 never reach it
        assert _close(g["dWg"], fd["Wg"]), np.abs(g["dWg"] - fd["Wg"]).max()


# ----------------------------------------------- torch autograd through an independent forward

def _st_round_bf16(x):
    """Round fp64 to the nearest bf16 value (ties to even) on the bit pattern: keep the sign, the
    exponent and the top 7 stored fraction bits; the dropped 45 bits decide, with the lowest kept
    bit breaking ties.  The gradient passes straight through."""
    bits = x.detach().view(torch.int64)
    low = torch.tensor((1 << 45) - 1, dtype=torch.int64)
    keep = (bits >> 45) & 1
    r = ((bits + (low >> 1) + keep) & ~low).view(torch.float64)
    return x + (r - x).detach()


def _torch_layer(q, k, v, window, base, eps, ve=None, x32=None, Wg=None, rope=True, qknorm=True,
                 st_round=False):
    """fp64 layer in torch, autograd-ready.  RoPE as a 2x2 rotation matrix per (position, pair);
    keys/values repeated to H heads; masked softmax and logsumexp from torch."""
    B, T, H, D = q.shape
    Hkv = k.shape[2]
    half = D // 2
    if rope:
        theta = torch.tensor([base ** (-2.0 * i / D) for i in range(half)], dtype=torch.float64)
        ang = torch.arange(T, dtype=torch.float64)[:, None] * theta[None, :]
        c, s = torch.cos(ang), torch.sin(ang)
        R = torch.stack([torch.stack([c, -s], -1), torch.stack([s, c], -1)], -2)  # (T, half, 2, 2)

        def rot(a):
            pairs = torch.stack([a[..., :half], a[..., half:]], -1)              # (B,T,h,half,2)
            r = torch.einsum("tiac,nthic->nthia", R, pairs)
            return torch.cat([r[..., 0], r[..., 1]], -1)
        q, k = rot(q), rot(k)
    if qknorm:
        q = q * torch.rsqrt(q.pow(2).mean(-1, keepdim=True) + eps)
        k = k * torch.rsqrt(k.pow(2).mean(-1, keepdim=True) + eps)
    if ve is not None:
        gate = 2.0 * torch.sigmoid(torch.einsum("btc,ch->bth", x32, Wg))
        v = v + gate[..., None] * ve
    if st_round:
        q, k, v = _st_round_bf16(q), _st_round_bf16(k), _st_round_bf16(v)
    G = H // Hkv
    k = k.repeat_interleave(G, dim=2)
    v = v.repeat_interleave(G, dim=2)
    scores = torch.einsum("bihd,bjhd->bhij", q, k) / math.sqrt(D)
    W = T if (window <= 0 or window >= T) else window
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    mask = (i - j >= 0) & (i - j < W)
    scores = scores.masked_fill(~mask, float("-inf"))
    lse = torch.logsumexp(scores, -1)
    out = torch.einsum("bhij,bjhd->bihd", torch.softmax(scores, -1), v)
    return out, lse


def _autograd_gradients(d, window, dout, dlse, eps, rope=True, qknorm=True, st_round=False):
    leaf = lambda t: t.double().clone().requires_grad_(True)
    q, k, v = leaf(d["q"]), leaf(d["k"]), leaf(d["v"])
    extra = {}
    if "ids" in d:
        B, T, Hkv, D = d["k"].shape
        extra["ve"] = leaf(d["table"][d["ids"]].view(B, T, Hkv, D))
        extra["x32"] = leaf(d["x"][..., :32])
        extra["Wg"] = leaf(d["Wg"])
    out, lse = _torch_layer(q, k, v, window, 10000.0, eps, rope=rope, qknorm=qknorm,
                            st_round=st_round, **extra)
    loss = (out * torch.from_numpy(dout)).sum()
    if dlse is not None:
        loss = loss + (lse * torch.from_numpy(dlse)).sum()
    loss.backward()
    g = dict(dq=q.grad.numpy(), dk=k.grad.numpy(), dv=v.grad.numpy())
    if extra:
        g.update(dve=extra["ve"].grad.numpy(), dx=extra["x32"].grad.numpy(),
                 dWg=extra["Wg"].grad.numpy())
    return g


def _rel_err(a, b):
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


@pytest.mark.parametrize("H,Hkv,window,ve", [(4, 4, 0, True), (4, 4, 5, False), (4, 2, 5, True),
                                             (6, 1, 11, True), (6, 3, 1, True), (2, 2, 36, True)])
def test_backward_matches_torch_autograd(H, Hkv, window, ve):
    B, T, D = 2, 37, 16
    d = _draw(B, T, H, D, Hkv=Hkv, ve=ve, seed=H * 10 + Hkv + window, unique_ids=False)
    dout, dlse = _cotangents(B, T, H, D, seed=window)
    g = oracle.backward(d, dout, window, dlse=dlse, eps=1e-6)
    ref = _autograd_gradients(d, window, dout, dlse, 1e-6)
    for key in ref:
        assert _rel_err(g[key], ref[key]) < 1e-10, (key, _rel_err(g[key], ref[key]))


@pytest.mark.parametrize("Hkv", [4, 2])
def test_parity_mode_backward_is_straight_through_rounding(Hkv):
    """parity=True: the forward rounds qhat, khat, v' to bf16 and the gradient passes straight
    through the rounding (checked against autograd with a bit-level rounding of its own)."""
    B, T, H, D = 1, 40, 4, 32
    d = _draw(B, T, H, D, Hkv=Hkv, ve=True, seed=77 + Hkv, unique_ids=False)
    dout, dlse = _cotangents(B, T, H, D, seed=5)
    g = oracle.backward(d, dout, 9, dlse=dlse, eps=1e-6, parity=True)
    ref = _autograd_gradients(d, 9, dout, dlse, 1e-6, st_round=True)
    for key in ref:
        assert _rel_err(g[key], ref[key]) < 1e-10, (key, _rel_err(g[key], ref[key]))
    pure = oracle.backward(d, dout, 9, dlse=dlse, eps=1e-6, parity=False)
    assert _rel_err(g["dq"], pure["dq"]) > 1e-6      # the rounding is really applied


# ------------------------------------------------------------------ closed forms and invariants

def test_window_one_closed_form():
    """Window 1: out_i = v'_i and lse_i = qhat_i . khat_i / sqrt(D).  Hence dv = dout,
    dve = g * dout, and, with RoPE and the norm off, dq_i = dlse_i k_i / sqrt(D) and
    dk_i = dlse_i q_i / sqrt(D)."""
    B, T, H, D = 2, 9, 3, 8
    d = _draw(B, T, H, D, ve=True, seed=3, unique_ids=False)
    dout, dlse = _cotangents(B, T, H, D, seed=3)
    g = oracle.backward(d, dout, 1, dlse=dlse, rope=False, qknorm=False)
    assert np.array_equal(g["dv"], dout)
    z = np.einsum("btc,ch->bth", d["x"][..., :32].double().numpy(), d["Wg"].double().numpy())
    gate = 2.0 / (1.0 + np.exp(-z))
    assert np.abs(g["dve"] - gate[..., None] * dout).max() < 1e-14
    gl = dlse.transpose(0, 2, 1)[..., None]                        # (B,T,H,1)
    q, k = d["q"].double().numpy(), d["k"].double().numpy()
    assert np.abs(g["dq"] - gl * k / math.sqrt(D)).max() < 1e-14
    assert np.abs(g["dk"] - gl * q / math.sqrt(D)).max() < 1e-14


def test_lse_only_cotangent_leaves_values_untouched():
    """lse does not depend on v', so with dout = 0 the value-side gradients vanish exactly."""
    B, T, H, D = 1, 20, 2, 16
    d = _draw(B, T, H, D, ve=True, seed=8, unique_ids=False)
    _, dlse = _cotangents(B, T, H, D, seed=8)
    g = oracle.backward(d, np.zeros((B, T, H, D)), 6, dlse=dlse)
    for key in ("dv", "dve", "dx", "dWg"):
        assert not np.any(g[key]), key
    assert np.abs(g["dq"]).max() > 1e-3 and np.abs(g["dk"]).max() > 1e-3


def test_uniform_lse_cotangent_on_full_softmax_row_sums():
    """With a constant dlse = c over a full-causal row and dout = 0, dS_ij = c P_ij sums to c;
    without RoPE/norm and with q = 0 the scores are all zero, so P is uniform over the i + 1
    keys and dq_i = c * mean_{j<=i} k_j / sqrt(D)."""
    B, T, H, D = 1, 12, 1, 8
    d = _draw(B, T, H, D, seed=4)
    d["q"] = torch.zeros_like(d["q"])
    c = 0.75
    g = oracle.backward(d, np.zeros((B, T, H, D)), 0, dlse=np.full((B, H, T), c),
                        rope=False, qknorm=False)
    k = d["k"].double().numpy()[0, :, 0]
    expect = c * np.cumsum(k, axis=0) / np.arange(1, T + 1)[:, None] / math.sqrt(D)
    assert np.abs(g["dq"][0, :, 0] - expect).max() < 1e-14


@pytest.mark.parametrize("rope", [True, False])
def test_rms_scale_invariance_makes_dq_orthogonal_to_q(rope):
    """With eps = 0 the normalised row is unchanged by q -> a q (RoPE is linear), so the
    directional derivative along q is zero: dq . q = 0 row by row (likewise for k)."""
    B, T, H, D = 1, 15, 2, 16
    d = _draw(B, T, H, D, seed=12)
    dout, dlse = _cotangents(B, T, H, D, seed=12)
    g = oracle.backward(d, dout, 5, dlse=dlse, eps=0.0, rope=rope)
    q, k = d["q"].double().numpy(), d["k"].double().numpy()
    assert np.abs(np.sum(g["dq"] * q, -1)).max() < 1e-12
    assert np.abs(np.sum(g["dk"] * k, -1)).max() < 1e-12
    assert np.abs(g["dq"]).max() > 1e-2


@pytest.mark.parametrize("H,Hkv", [(6, 2), (4, 1)])
def test_gqa_gradients_are_group_sums_of_repeated_head_gradients(H, Hkv):
    """Grouped-query attention is the multi-head layer with each key/value head (and its table
    slice and gate column) repeated G = H / Hkv times; by the chain rule for tied inputs its
    key/value-side gradients are the sums over each group of the repeated layer's gradients."""
    B, T, D = 2, 19, 8
    G = H // Hkv
    d = _draw(B, T, H, D, Hkv=Hkv, ve=True, seed=H + Hkv, unique_ids=False)
    rep = dict(q=d["q"], k=d["k"].repeat_interleave(G, 2), v=d["v"].repeat_interleave(G, 2),
               ids=d["ids"], x=d["x"], Wg=d["Wg"].repeat_interleave(G, 1),
               table=d["table"].view(-1, Hkv, D).repeat_interleave(G, 1).reshape(-1, H * D))
    dout, dlse = _cotangents(B, T, H, D, seed=H)
    g = oracle.backward(d, dout, 7, dlse=dlse)
    m = oracle.backward(rep, dout, 7, dlse=dlse)
    assert np.abs(g["dq"] - m["dq"]).max() < 1e-12
    assert np.abs(g["dx"] - m["dx"]).max() < 1e-12
    for key in ("dk", "dv", "dve"):
        summed = m[key].reshape(B, T, Hkv, G, D).sum(3)
        assert np.abs(g[key] - summed).max() < 1e-12, key
    assert np.abs(g["dWg"] - m["dWg"].reshape(32, Hkv, G).sum(2)).max() < 1e-12


def test_backward_rejects_bad_arguments():
    d = _draw(1, 4, 2, 8, seed=1)
    with pytest.raises(ValueError):
        oracle.backward(d, np.zeros((1, 4, 2, 4)), 0)
    with pytest.raises(ValueError):
        oracle.backward(d, np.zeros((1, 4, 2, 8)), 0, dlse=np.zeros((1, 4, 2)))
    three = dict(q=_draw(1, 4, 3, 8)["q"], k=d["k"], v=d["v"])   # Hkv = 2 does not divide H = 3
    with pytest.raises(ValueError):
        oracle.backward(three, np.zeros((1, 4, 3, 8)), 0)


# --------------------------------------------------------------- sampled rows = full backward

@pytest.mark.parametrize("B,T,H,Hkv,D,window,ve,parity", [
    (2, 37, 4, 4, 16, 5, True, False),
    (1, 60, 6, 2, 8, 0, True, True),
    (2, 45, 3, 1, 16, 1, False, True),
    (1, 130, 2, 2, 32, 40, True, True),
])
def test_sampled_rows_equal_the_full_backward_bit_for_bit(B, T, H, Hkv, D, window, ve, parity):
    d = _draw(B, T, H, D, Hkv=Hkv, ve=ve, seed=T + H, unique_ids=False)
    dout, dlse = _cotangents(B, T, H, D, seed=T)
    full = oracle.backward(d, dout, window, dlse=dlse, parity=parity)
    g = torch.Generator().manual_seed(T)
    qrows = torch.randint(0, B * H * T, (9,), generator=g).tolist() + [0, B * H * T - 1]
    krows = torch.randint(0, B * Hkv * T, (9,), generator=g).tolist() + [0, B * Hkv * T - 1, 3]
    rows = oracle.backward_rows(d, dout, window, dlse=dlse, qrows=qrows, krows=krows, parity=parity)
    for n, r in enumerate(qrows):
        bh, i = divmod(r, T)
        b, h = divmod(bh, H)
        assert np.array_equal(rows["dq"][n], full["dq"][b, i, h]), ("dq", r)
    for n, r in enumerate(krows):
        bh, j = divmod(r, T)
        b, hk = divmod(bh, Hkv)
        for key in ("dk", "dv") + (("dve",) if ve else ()):
            assert np.array_equal(rows[key][n], full[key][b, j, hk]), (key, r)


def test_sampled_rows_reject_out_of_range_ids():
    d = _draw(1, 8, 2, 8, seed=2)
    dout, _ = _cotangents(1, 8, 2, 8, seed=2)
    with pytest.raises(ValueError):
        oracle.backward_rows(d, dout, 0, qrows=[16])
    with pytest.raises(ValueError):
        oracle.backward_rows(d, dout, 0, krows=[-1])
