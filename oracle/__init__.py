"""fp64 CPU oracle of the causal sliding-window attention layer (RoPE -> RMS QK-norm ->
gated value embedding -> causal windowed softmax attention).

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA library and never
imports it.

Two independent implementations live here.  The C oracle (``swa_oracle.c``, fp64, one query
row at a time) backs the functions of this module:

* ``forward`` / ``prologue``: the layer and its prologue.
* ``qkv_prologue``: the bias-free q, k, v projection of the layer input x followed by the same
  prologue (the fused projection).
* ``backward``: the gradient of the same layer (chain rule through the five steps in
  reverse); ``backward_rows`` gives the same values at sampled rows.

``brute.py`` is the second: a NumPy fp64 restatement that materialises the full T x T score
matrix, used as the brute-force pin of the C oracle on small shapes.

Each function cites the passage of the pages it follows in ``swa_oracle.c``'s header.
Readings taken where the pages are silent (pair layout and sign of RoPE, window boundary,
eps placement, gate shape) are stated there and in the design notes.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import numpy as np

from . import build as _build

_lib = None


def _configure(lib):
    P = ctypes.c_void_p
    lib.swa_oracle_forward.restype = ctypes.c_int
    lib.swa_oracle_forward.argtypes = [P, P, P, P, P, ctypes.c_int, P, ctypes.c_int, P,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_double, ctypes.c_double,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       P, ctypes.c_int64, P, P]
    lib.swa_oracle_prologue.restype = ctypes.c_int
    lib.swa_oracle_prologue.argtypes = [P, P, P, P, P, ctypes.c_int, P, ctypes.c_int, P,
                                        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_double, ctypes.c_double,
                                        ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P]
    lib.swa_oracle_forward_gqa.restype = ctypes.c_int
    lib.swa_oracle_forward_gqa.argtypes = [P, P, P, P, P, ctypes.c_int, P, ctypes.c_int, P,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                           ctypes.c_double, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, P, ctypes.c_int64, P, P]
    lib.swa_oracle_forward_doc_gqa.restype = ctypes.c_int
    lib.swa_oracle_forward_doc_gqa.argtypes = [P, P, P, P, P, ctypes.c_int, P, ctypes.c_int, P,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                               ctypes.c_double, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, P, P, ctypes.c_int64, P, P]
    lib.swa_oracle_prologue_gqa.restype = ctypes.c_int
    lib.swa_oracle_prologue_gqa.argtypes = [P, P, P, P, P, ctypes.c_int, P, ctypes.c_int, P,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_double, ctypes.c_double,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P]
    lib.swa_oracle_backward_gqa.restype = ctypes.c_int
    lib.swa_oracle_backward_gqa.argtypes = [P, P, P, P, P, ctypes.c_int, P, ctypes.c_int, P,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                            ctypes.c_double, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_int, P, P, P, P, P, P, P, P]
    lib.swa_oracle_backward_doc_gqa.restype = ctypes.c_int
    lib.swa_oracle_backward_doc_gqa.argtypes = [P, P, P, P, P, ctypes.c_int, P, ctypes.c_int, P,
                                                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                                ctypes.c_double, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_int, P, P, P, P, P, P, P, P, P]
    lib.swa_oracle_backward_rows_gqa.restype = ctypes.c_int
    lib.swa_oracle_backward_rows_gqa.argtypes = [P, P, P, P, P, ctypes.c_int, P, ctypes.c_int, P,
                                                 ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                 ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                                 ctypes.c_double, ctypes.c_int, ctypes.c_int,
                                                 ctypes.c_int, ctypes.c_int, P, P,
                                                 P, ctypes.c_int64, P, P, ctypes.c_int64, P, P, P]
    lib.swa_oracle_qkv_prologue_gqa.restype = ctypes.c_int
    lib.swa_oracle_qkv_prologue_gqa.argtypes = [P, ctypes.c_int, P, P, P, ctypes.c_int, P,
                                                ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                                ctypes.c_double, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, P, P, P]
    lib.swa_oracle_threads.restype = ctypes.c_int
    lib.swa_oracle_round_bf16.restype = ctypes.c_double
    lib.swa_oracle_round_bf16.argtypes = [ctypes.c_double]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _configure(ctypes.CDLL(_build.build()))
    return _lib


def _swap_library(path: Optional[str]):
    """Test hook: load another build of swa_oracle.c (e.g. one with a planted mistake).
    ``None`` restores the regular build.  Returns the previously loaded library."""
    global _lib
    prev = _lib
    _lib = None if path is None else _configure(ctypes.CDLL(path))
    return prev


def threads() -> int:
    return int(_load().swa_oracle_threads())


def round_bf16(x: float) -> float:
    return float(_load().swa_oracle_round_bf16(float(x)))


def _bits(t) -> np.ndarray:
    """bf16 tensor/array -> contiguous uint16 bit patterns (no value conversion)."""
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        assert t.dtype == np.uint16
        return np.ascontiguousarray(t)
    import torch
    assert t.dtype == torch.bfloat16, t.dtype
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _ve_args(inputs: Dict):
    if inputs.get("ids") is None:
        return None, None, 0, None, 0, None
    import torch
    ids = inputs["ids"]
    ids = ids.cpu().contiguous().numpy().astype(np.int64) if isinstance(ids, torch.Tensor) else np.ascontiguousarray(ids, dtype=np.int64)
    table = _bits(inputs["table"])
    x = _bits(inputs["x"])
    Wg = _bits(inputs["Wg"])
    return ids, table, int(table.shape[0]), x, int(x.shape[-1]), Wg


def forward(inputs: Dict, window: int, rope_base: float = 10000.0, eps: float = 1e-6, *,
            parity: bool = True, rope: bool = True, qknorm: bool = True,
            window_convention: int = 0, rows=None, doc=None):
    """Attention forward of one layer.

    inputs: dict with q bf16 (B,T,H,D), k, v bf16 (B,T,Hkv,D) (Hkv divides H; query head h reads
    key/value head h // (H // Hkv); Hkv == H is the multi-head layer) and, for value-embedding
    layers, ids (B,T), table [vocab, Hkv*D], x (B,T,C), Wg [32,Hkv].
    parity=True rounds qhat, khat, v' to bf16 after the fp64 prologue (pure fp64 otherwise).
    rope/qknorm switch the prologue steps off (test-only, for the library special case).
    rows: None for every row, else flat query ids ((b*H + h)*T + i).
    doc: None, or document ids (B,T): key j is then visible to query i only within the same
    document as well (a document-boundary mask; RoPE positions stay the sequence positions).

    Returns (out, lse): out fp64 (B,T,H,D) and lse fp64 (B,H,T) when rows is None, else
    out [n_rows, D] and lse [n_rows] in the sorted order of ``rows``.
    """
    lib = _load()
    q, k, v = _bits(inputs["q"]), _bits(inputs["k"]), _bits(inputs["v"])
    B, T, H, D = q.shape
    ids, table, vocab, x, C, Wg = _ve_args(inputs)
    if rows is None:
        rows_a = None
        n = 0
        out = np.empty((B, T, H, D), dtype=np.float64)
        lse = np.empty((B, H, T), dtype=np.float64)
    else:
        rows_a = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        if rows_a.size > 1 and np.any(np.diff(rows_a) < 0):
            raise ValueError("rows must be sorted ascending")
        n = int(rows_a.size)
        out = np.empty((n, D), dtype=np.float64)
        lse = np.empty((n,), dtype=np.float64)
    Hkv = int(k.shape[2])
    if doc is not None:
        import torch
        doc_a = doc.cpu().contiguous().numpy().astype(np.int64) if isinstance(doc, torch.Tensor) \
            else np.ascontiguousarray(doc, dtype=np.int64)
        if doc_a.shape != (B, T):
            raise ValueError("doc must be (B, T)")
        rc = lib.swa_oracle_forward_doc_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(ids), _ptr(table), vocab,
                                            _ptr(x), C, _ptr(Wg), B, T, H, Hkv, D, int(window),
                                            float(rope_base), float(eps), int(parity), int(rope),
                                            int(qknorm), int(window_convention), _ptr(doc_a), _ptr(rows_a),
                                            n, _ptr(out), _ptr(lse))
    elif Hkv == H:
        rc = lib.swa_oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(ids), _ptr(table), vocab,
                                    _ptr(x), C, _ptr(Wg), B, T, H, D, int(window),
                                    float(rope_base), float(eps), int(parity), int(rope), int(qknorm),
                                    int(window_convention), _ptr(rows_a), n, _ptr(out), _ptr(lse))
    else:
        rc = lib.swa_oracle_forward_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(ids), _ptr(table), vocab,
                                        _ptr(x), C, _ptr(Wg), B, T, H, Hkv, D, int(window),
                                        float(rope_base), float(eps), int(parity), int(rope),
                                        int(qknorm), int(window_convention), _ptr(rows_a), n,
                                        _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return out, lse


def prologue(inputs: Dict, rope_base: float = 10000.0, eps: float = 1e-6, *,
             parity: bool = False, rope: bool = True, qknorm: bool = True):
    """qhat (B,T,H,D), khat and v' (B,T,Hkv,D) as fp64 arrays (the steps before the attention)."""
    lib = _load()
    q, k, v = _bits(inputs["q"]), _bits(inputs["k"]), _bits(inputs["v"])
    B, T, H, D = q.shape
    Hkv = int(k.shape[2])
    ids, table, vocab, x, C, Wg = _ve_args(inputs)
    qh = np.empty((B, T, H, D), dtype=np.float64)
    kh = np.empty((B, T, Hkv, D), dtype=np.float64)
    vp = np.empty_like(kh)
    if Hkv == H:
        rc = lib.swa_oracle_prologue(_ptr(q), _ptr(k), _ptr(v), _ptr(ids), _ptr(table), vocab,
                                     _ptr(x), C, _ptr(Wg), B, T, H, D, float(rope_base), float(eps),
                                     int(parity), int(rope), int(qknorm), _ptr(qh), _ptr(kh), _ptr(vp))
    else:
        rc = lib.swa_oracle_prologue_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(ids), _ptr(table), vocab,
                                         _ptr(x), C, _ptr(Wg), B, T, H, Hkv, D, float(rope_base),
                                         float(eps), int(parity), int(rope), int(qknorm), _ptr(qh),
                                         _ptr(kh), _ptr(vp))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return qh, kh, vp


def backward(inputs: Dict, dout, window: int, dlse=None, rope_base: float = 10000.0,
             eps: float = 1e-6, *, parity: bool = False, rope: bool = True, qknorm: bool = True,
             window_convention: int = 0, doc=None):
    """Gradient of ``sum(dout * out) + sum(dlse * lse)`` with respect to the layer's inputs.

    inputs as for ``forward``; dout (B,T,H,D) and dlse (B,H,T) (None for zero) are taken as
    fp64.  parity=False (the default) is the exact gradient of the fp64 layer; parity=True
    rounds qhat, khat, v' to bf16 as the forward's parity mode does and passes the gradient
    straight through the rounding.

    Returns a dict of fp64 arrays: dq (B,T,H,D); dk, dv (B,T,Hkv,D); on value-embedding layers
    also dve (B,T,Hkv,D) (gradient of the looked-up table row at each position), dx (B,T,32)
    (the gate's input channels) and dWg [32,Hkv].  doc: document ids (B,T) as in ``forward``.
    """
    lib = _load()
    q, k, v = _bits(inputs["q"]), _bits(inputs["k"]), _bits(inputs["v"])
    B, T, H, D = q.shape
    Hkv = int(k.shape[2])
    ids, table, vocab, x, C, Wg = _ve_args(inputs)
    go = np.ascontiguousarray(_as_f64(dout))
    if go.shape != (B, T, H, D):
        raise ValueError("dout must be (B, T, H, D)")
    gl = None
    if dlse is not None:
        gl = np.ascontiguousarray(_as_f64(dlse))
        if gl.shape != (B, H, T):
            raise ValueError("dlse must be (B, H, T)")
    grads = dict(dq=np.empty((B, T, H, D)), dk=np.empty((B, T, Hkv, D)),
                 dv=np.empty((B, T, Hkv, D)))
    if ids is not None:
        grads.update(dve=np.empty((B, T, Hkv, D)), dx=np.empty((B, T, 32)),
                     dWg=np.empty((32, Hkv)))
    doc_a = None
    if doc is not None:
        import torch
        doc_a = doc.cpu().contiguous().numpy().astype(np.int64) if isinstance(doc, torch.Tensor) \
            else np.ascontiguousarray(doc, dtype=np.int64)
        if doc_a.shape != (B, T):
            raise ValueError("doc must be (B, T)")
    rc = lib.swa_oracle_backward_doc_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(ids), _ptr(table), vocab,
                                     _ptr(x), C, _ptr(Wg), B, T, H, Hkv, D, int(window),
                                     float(rope_base), float(eps), int(parity), int(rope),
                                     int(qknorm), int(window_convention), _ptr(doc_a), _ptr(go), _ptr(gl),
                                     _ptr(grads["dq"]), _ptr(grads["dk"]), _ptr(grads["dv"]),
                                     _ptr(grads.get("dve")), _ptr(grads.get("dx")),
                                     _ptr(grads.get("dWg")))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return grads


def backward_rows(inputs: Dict, dout, window: int, dlse=None, *, qrows=(), krows=(),
                  rope_base: float = 10000.0, eps: float = 1e-6, parity: bool = True,
                  rope: bool = True, qknorm: bool = True, window_convention: int = 0):
    """``backward`` at sampled rows, bit for bit: qrows are flat query ids ((b*H + h)*T + i),
    krows flat key/value ids ((b*Hkv + hk)*T + j).  Returns dq [len(qrows), D] and dk, dv (and dve
    on value-embedding layers) [len(krows), D], in the order of the requests."""
    lib = _load()
    q, k, v = _bits(inputs["q"]), _bits(inputs["k"]), _bits(inputs["v"])
    B, T, H, D = q.shape
    Hkv = int(k.shape[2])
    ids, table, vocab, x, C, Wg = _ve_args(inputs)
    go = np.ascontiguousarray(_as_f64(dout))
    if go.shape != (B, T, H, D):
        raise ValueError("dout must be (B, T, H, D)")
    gl = None if dlse is None else np.ascontiguousarray(_as_f64(dlse))
    if gl is not None and gl.shape != (B, H, T):
        raise ValueError("dlse must be (B, H, T)")
    qa = np.ascontiguousarray(np.asarray(qrows, dtype=np.int64).reshape(-1))
    ka = np.ascontiguousarray(np.asarray(krows, dtype=np.int64).reshape(-1))
    out = dict(dq=np.empty((qa.size, D)), dk=np.empty((ka.size, D)), dv=np.empty((ka.size, D)))
    if ids is not None:
        out["dve"] = np.empty((ka.size, D))
    rc = lib.swa_oracle_backward_rows_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(ids), _ptr(table), vocab,
                                          _ptr(x), C, _ptr(Wg), B, T, H, Hkv, D, int(window),
                                          float(rope_base), float(eps), int(parity), int(rope),
                                          int(qknorm), int(window_convention), _ptr(go), _ptr(gl),
                                          _ptr(qa), int(qa.size), _ptr(out["dq"]), _ptr(ka), int(ka.size),
                                          _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out.get("dve")))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return out


def _as_f64(a) -> np.ndarray:
    if isinstance(a, np.ndarray):
        return a.astype(np.float64, copy=False)
    return a.detach().cpu().double().numpy()


def qkv_prologue(x, Wqkv, H: int, Hkv: int, D: int, ids=None, table=None, Wg=None,
                 rope_base: float = 10000.0, eps: float = 1e-6, *, parity: bool = False,
                 rope: bool = True, qknorm: bool = True):
    """q, k, v = x Wqkv^T (x (B,T,C) bf16, Wqkv [(H + 2 Hkv) D, C] bf16, the linear layer's layout;
    rows: q heads, k heads, v heads), then RoPE / RMS on q and k and the gated value embedding on
    v (ids (B,T), table [vocab, Hkv D], Wg [32, Hkv]; the gate reads x[..., :32]).
    Returns qhat (B,T,H,D), khat and v' (B,T,Hkv,D) as fp64 (rounded to bf16 values if parity)."""
    lib = _load()
    xb, wb = _bits(x), _bits(Wqkv)
    B, T, C = xb.shape
    if wb.shape != ((H + 2 * Hkv) * D, C):
        raise ValueError("Wqkv must be [(H + 2 Hkv) D, C]")
    import torch
    if ids is not None:
        ids_a = ids.cpu().contiguous().numpy().astype(np.int64) if isinstance(ids, torch.Tensor) \
            else np.ascontiguousarray(ids, dtype=np.int64)
        tb, gw = _bits(table), _bits(Wg)
        vocab = int(tb.shape[0])
    else:
        ids_a = tb = gw = None
        vocab = 0
    qh = np.empty((B, T, H, D))
    kh = np.empty((B, T, Hkv, D))
    vp = np.empty((B, T, Hkv, D))
    rc = lib.swa_oracle_qkv_prologue_gqa(_ptr(xb), C, _ptr(wb), _ptr(ids_a), _ptr(tb), vocab, _ptr(gw),
                                         B, T, H, Hkv, D, float(rope_base), float(eps), int(parity),
                                         int(rope), int(qknorm), _ptr(qh), _ptr(kh), _ptr(vp))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return qh, kh, vp
