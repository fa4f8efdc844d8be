"""Brute-force NumPy fp64 restatement of the attention layer, for small shapes.

TEST INFRASTRUCTURE, written independently of ``swa_oracle.c`` to pin it: the rotation is
done as a complex multiplication z * exp(i t theta) of the pair z = x_i + i x_{i+D/2}; the
whole T x T score matrix is materialised with an explicit boolean mask; the softmax and the
log-sum-exp come from ``scipy.special``.  Same definition, different arithmetic route:
"Let's reproduce GPT-2 (124M)" notes, section 3 (scores, mask including the diagonal,
softmax over keys, weighted sum of values); intelliparadigm "GPT-2 for $73", section 2.2
(norm after RoPE) and 3.2 (window); PaperWeekly repost (value-embedding gate).
"""
from __future__ import annotations

import numpy as np
from scipy.special import expit, logsumexp, softmax


def _f64(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().cpu().double().numpy()


def rope_complex(x: np.ndarray, base: float) -> np.ndarray:
    """x (B,T,H,D) -> rotated; pair i is (x[..., i], x[..., i + D/2])."""
    B, T, H, D = x.shape
    half = D // 2
    theta = base ** (-2.0 * np.arange(half) / D)
    ang = np.arange(T)[:, None] * theta[None, :]                       # (T, half)
    z = x[..., :half] + 1j * x[..., half:]
    z = z * np.exp(1j * ang)[None, :, None, :]
    return np.concatenate([z.real, z.imag], axis=-1)


def rms(x: np.ndarray, eps: float) -> np.ndarray:
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def window_mask(T: int, window: int, convention: int = 0) -> np.ndarray:
    W = T if (window <= 0 or window >= T) else window
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    diff = i - j
    return (diff >= 0) & ((diff < W) if convention == 0 else (diff <= W))


def forward(inputs, window: int, rope_base: float = 10000.0, eps: float = 1e-6, *,
            rope: bool = True, qknorm: bool = True, convention: int = 0, return_weights=False,
            doc=None):
    q, k, v = _f64(inputs["q"]), _f64(inputs["k"]), _f64(inputs["v"])
    B, T, H, D = q.shape
    if rope:
        q, k = rope_complex(q, rope_base), rope_complex(k, rope_base)
    if qknorm:
        q, k = rms(q, eps), rms(k, eps)
    if inputs.get("ids") is not None:
        ids = np.asarray(inputs["ids"].cpu().numpy() if hasattr(inputs["ids"], "cpu") else inputs["ids"])
        table = _f64(inputs["table"])
        x = _f64(inputs["x"])[..., :32]
        Wg = _f64(inputs["Wg"])
        ve = table[ids].reshape(B, T, H, D)
        gate = 2.0 * expit(np.einsum("btc,ch->bth", x, Wg))             # (B,T,H)
        v = v + gate[..., None] * ve
    s = np.einsum("bihd,bjhd->bhij", q, k) / np.sqrt(D)                # (B,H,T,T)
    mask = np.broadcast_to(window_mask(T, window, convention)[None], (B, T, T))
    if doc is not None:                                                 # same document only
        dd = np.asarray(doc.cpu().numpy() if hasattr(doc, "cpu") else doc)
        mask = mask & (dd[:, :, None] == dd[:, None, :])
    s = np.where(mask[:, None], s, -np.inf)
    p = softmax(s, axis=-1)
    out = np.einsum("bhij,bjhd->bihd", p, v)
    lse = logsumexp(s, axis=-1)                                         # (B,H,T)
    if return_weights:
        return out, lse, p
    return out, lse
