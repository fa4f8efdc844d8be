"""B200 (sm_100a) causal sliding-window attention (forward, backward, decode): Python binding of the C ABI in
``include/swa_attn.h``.

This module only marshals arguments: every step of the layer (RoPE, RMS QK-norm, the value-
embedding gate, the windowed attention, the log-sum-exp) runs in the CUDA kernels of
``libswa_attn.so``.  There is no CPU path: the first call loads the library and raises if it
is not built (``load()`` does that eagerly).

Functions with the C names take raw device pointers (ints) and return the status code.
``forward`` is the tensor-level convenience call: it checks dtypes and layouts, allocates the
outputs with torch and raises ``SwaError`` on a non-zero status.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libswa_attn.so")

SWA_OK = 0
SWA_ERR_INVALID_ARG = -1
SWA_ERR_UNSUPPORTED = -2
SWA_ERR_MISALIGNED = -3
SWA_ERR_CUDA = -4
SWA_ERR_TIMEOUT = -5
SWA_ERR_NO_MEMORY = -6
SWA_ERR_NO_DEVICE = -7


class SwaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {swa_attn_strerror(status)} (status {status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m causal_sliding_window_swa_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.swa_attn_fwd.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, F, F, P]
    lib.swa_attn_fwd.restype = I
    lib.swa_attn_fwd_ws.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, F, F, P, Z, P]
    lib.swa_attn_fwd_ws.restype = I
    lib.swa_attn_workspace_bytes.argtypes = [I, I, I, I, I]
    lib.swa_attn_workspace_bytes.restype = Z
    lib.swa_attn_fwd_noalloc.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, F, F, P]
    lib.swa_attn_fwd_noalloc.restype = I
    lib.swa_attn_noalloc_scratch_bytes.argtypes = []
    lib.swa_attn_noalloc_scratch_bytes.restype = Z
    lib.swa_attn_workspace_offset.argtypes = [I, I, I, I, I, I]
    lib.swa_attn_workspace_offset.restype = Z
    lib.swa_attn_rope_table.argtypes = [I, I, I, I, I, F, P, Z, P]
    lib.swa_attn_rope_table.restype = I
    lib.swa_attn_prologue.argtypes = [P, P, P, P, P, P, I, I, I, I, F, F, P, Z, P]
    lib.swa_attn_prologue.restype = I
    lib.swa_attn_attention.argtypes = [P, I, P, P, I, I, I, I, I, P, Z, P]
    lib.swa_attn_attention.restype = I
    lib.swa_attn_strerror.argtypes = [I]
    lib.swa_attn_strerror.restype = ctypes.c_char_p
    lib.swa_attn_last_device_status.argtypes = [P, ctypes.POINTER(ctypes.c_uint)]
    lib.swa_attn_last_device_status.restype = I
    lib.swa_attn_fwd_gqa.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, F, P]
    lib.swa_attn_fwd_gqa.restype = I
    lib.swa_attn_fwd_doc.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, F, P]
    lib.swa_attn_fwd_doc.restype = I
    lib.swa_attn_decode_workspace_bytes.argtypes = [I, I, I, I, I, I]
    lib.swa_attn_decode_workspace_bytes.restype = Z
    lib.swa_attn_decode.argtypes = [P, P, P, P, P, P, P, P, I, P, P, I, I, I, I, I, F, F, P, Z, P]
    lib.swa_attn_decode.restype = I
    lib.swa_attn_decode_gqa.argtypes = [P, P, P, P, P, P, P, P, I, P, P, I, I, I, I, I, I, F, F, P, Z, P]
    lib.swa_attn_decode_gqa.restype = I
    lib.swa_attn_decode_doc.argtypes = [P, P, P, P, P, P, P, P, I, P, P, P, I, I, I, I, I, I, F, F, P, Z, P]
    lib.swa_attn_decode_doc.restype = I
    lib.swa_attn_bwd_workspace_bytes.argtypes = [I, I, I, I, I, I]
    lib.swa_attn_bwd_workspace_bytes.restype = Z
    lib.swa_attn_bwd_gqa.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P,
                                     I, I, I, I, I, I, F, F, P, Z, P]
    lib.swa_attn_bwd_gqa.restype = I
    lib.swa_attn_bwd_doc.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P,
                                     I, I, I, I, I, I, F, F, P, Z, P]
    lib.swa_attn_bwd_doc.restype = I
    lib.swa_attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P,
                                 I, I, I, I, I, F, F, P, Z, P]
    lib.swa_attn_bwd.restype = I
    lib.swa_attn_bwd_saved.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P,
                                       I, I, I, I, I, F, F, P, Z, P]
    lib.swa_attn_bwd_saved.restype = I
    lib.swa_attn_fwd_x_workspace_bytes.argtypes = [I, I, I, I, I]
    lib.swa_attn_fwd_x_workspace_bytes.restype = Z
    lib.swa_attn_qkv_prologue.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, F, F, P, Z, P]
    lib.swa_attn_qkv_prologue.restype = I
    lib.swa_attn_fwd_x.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, F, F, P, Z, P]
    lib.swa_attn_fwd_x.restype = I
    lib.swa_attn_selftest_wait.argtypes = [I, P]
    lib.swa_attn_selftest_wait.restype = I
    lib.swa_attn_set_wait_limit_ms.argtypes = [I]
    lib.swa_attn_set_wait_limit_ms.restype = I
    lib.swa_attn_version.argtypes = []
    lib.swa_attn_version.restype = I
    return lib


_lib_handle: Optional[ctypes.CDLL] = None
_lib_lock = threading.Lock()


def load() -> ctypes.CDLL:
    """Load libswa_attn.so (once, also when several threads make their first call together);
    raises ImportError/OSError if it is missing or stale."""
    global _lib_handle
    if _lib_handle is None:
        with _lib_lock:
            if _lib_handle is None:
                _lib_handle = _load()
    return _lib_handle


class _LazyLib:
    def __getattr__(self, name):
        return getattr(load(), name)


_lib = _LazyLib()


# ------------------------------------------------------------------ the C entry points

def swa_attn_fwd(q, k, v, ve, gate_x, Wg, out, lse, B, T, H, D, window, rope_base, eps, stream) -> int:
    return _lib.swa_attn_fwd(q, k, v, ve, gate_x, Wg, out, lse, B, T, H, D, window, rope_base, eps, stream)


def swa_attn_fwd_ws(q, k, v, ve, gate_x, Wg, out, lse, B, T, H, D, window, rope_base, eps,
                    workspace, ws_bytes, stream) -> int:
    return _lib.swa_attn_fwd_ws(q, k, v, ve, gate_x, Wg, out, lse, B, T, H, D, window, rope_base, eps,
                                workspace, ws_bytes, stream)


def swa_attn_fwd_noalloc(q, k, v, ve, gate_x, Wg, out, lse, B, T, H, D, window, rope_base, eps,
                         stream) -> int:
    """swa_attn_fwd for callers that cannot allocate device memory: scratch comes from a fixed
    array inside the library (see include/swa_attn.h); nothing is allocated."""
    return _lib.swa_attn_fwd_noalloc(q, k, v, ve, gate_x, Wg, out, lse, B, T, H, D, window, rope_base,
                                     eps, stream)


def swa_attn_noalloc_scratch_bytes() -> int:
    return int(_lib.swa_attn_noalloc_scratch_bytes())


def swa_attn_workspace_bytes(B, T, H, D, has_ve) -> int:
    return int(_lib.swa_attn_workspace_bytes(B, T, H, D, int(has_ve)))


SWA_WS_QHAT, SWA_WS_KHAT, SWA_WS_VPRIME, SWA_WS_ROPE_TABLE = 0, 1, 2, 3


def swa_attn_workspace_offset(B, T, H, D, has_ve, section) -> int:
    return int(_lib.swa_attn_workspace_offset(B, T, H, D, int(has_ve), int(section)))


def swa_attn_rope_table(B, T, H, D, has_ve, rope_base, workspace, ws_bytes, stream) -> int:
    return _lib.swa_attn_rope_table(B, T, H, D, int(has_ve), rope_base, workspace, ws_bytes, stream)


def swa_attn_prologue(q, k, v, ve, gate_x, Wg, B, T, H, D, rope_base, eps, workspace, ws_bytes, stream) -> int:
    return _lib.swa_attn_prologue(q, k, v, ve, gate_x, Wg, B, T, H, D, rope_base, eps, workspace, ws_bytes, stream)


def swa_attn_attention(v, has_ve, out, lse, B, T, H, D, window, workspace, ws_bytes, stream) -> int:
    return _lib.swa_attn_attention(v, int(has_ve), out, lse, B, T, H, D, window, workspace, ws_bytes, stream)


def swa_attn_strerror(status: int) -> str:
    return _lib.swa_attn_strerror(int(status)).decode()


def swa_attn_last_device_status(stream=None) -> Tuple[int, int]:
    detail = ctypes.c_uint(0)
    rc = _lib.swa_attn_last_device_status(stream, ctypes.byref(detail))
    return int(rc), int(detail.value)


def swa_attn_fwd_gqa(q, k, v, ve, gate_x, Wg, out, lse, B, T, H, Hkv, D, window, rope_base, eps,
                     stream) -> int:
    return _lib.swa_attn_fwd_gqa(q, k, v, ve, gate_x, Wg, out, lse, B, T, H, Hkv, D, window, rope_base,
                                 eps, stream)


def swa_attn_fwd_doc(q, k, v, ve, gate_x, Wg, doc, out, lse, B, T, H, Hkv, D, window, rope_base, eps,
                     stream) -> int:
    return _lib.swa_attn_fwd_doc(q, k, v, ve, gate_x, Wg, doc, out, lse, B, T, H, Hkv, D, window, rope_base,
                                 eps, stream)


def swa_attn_decode_workspace_bytes(B, Tmax, H, D, has_ve, window) -> int:
    return int(_lib.swa_attn_decode_workspace_bytes(B, Tmax, H, D, int(has_ve), window))


def swa_attn_decode(q, k, v, ve, gate_x, Wg, k_cache, v_cache, pos, out, lse, B, Tmax, H, D, window,
                    rope_base, eps, workspace, ws_bytes, stream) -> int:
    return _lib.swa_attn_decode(q, k, v, ve, gate_x, Wg, k_cache, v_cache, pos, out, lse, B, Tmax, H, D,
                                window, rope_base, eps, workspace, ws_bytes, stream)


def swa_attn_decode_gqa(q, k, v, ve, gate_x, Wg, k_cache, v_cache, pos, out, lse, B, Tmax, H, Hkv, D, window,
                        rope_base, eps, workspace, ws_bytes, stream) -> int:
    return _lib.swa_attn_decode_gqa(q, k, v, ve, gate_x, Wg, k_cache, v_cache, pos, out, lse, B, Tmax, H, Hkv,
                                    D, window, rope_base, eps, workspace, ws_bytes, stream)


def swa_attn_decode_doc(q, k, v, ve, gate_x, Wg, k_cache, v_cache, pos, doc_start, out, lse, B, Tmax, H, Hkv, D,
                        window, rope_base, eps, workspace, ws_bytes, stream) -> int:
    return _lib.swa_attn_decode_doc(q, k, v, ve, gate_x, Wg, k_cache, v_cache, pos, doc_start, out, lse, B, Tmax,
                                    H, Hkv, D, window, rope_base, eps, workspace, ws_bytes, stream)


def swa_attn_bwd_workspace_bytes(B, T, H, Hkv, D, has_ve) -> int:
    return int(_lib.swa_attn_bwd_workspace_bytes(B, T, H, Hkv, D, int(has_ve)))


def swa_attn_bwd_gqa(q, k, v, ve, gate_x, Wg, out, lse, dout, dlse, dq, dk, dv, dve, dgate_x, dWg,
                     B, T, H, Hkv, D, window, rope_base, eps, workspace, ws_bytes, stream) -> int:
    return _lib.swa_attn_bwd_gqa(q, k, v, ve, gate_x, Wg, out, lse, dout, dlse, dq, dk, dv, dve, dgate_x,
                                 dWg, B, T, H, Hkv, D, window, rope_base, eps, workspace, ws_bytes, stream)


def swa_attn_bwd(q, k, v, ve, gate_x, Wg, out, lse, dout, dlse, dq, dk, dv, dve, dgate_x, dWg,
                 B, T, H, D, window, rope_base, eps, workspace, ws_bytes, stream) -> int:
    return _lib.swa_attn_bwd(q, k, v, ve, gate_x, Wg, out, lse, dout, dlse, dq, dk, dv, dve, dgate_x, dWg,
                             B, T, H, D, window, rope_base, eps, workspace, ws_bytes, stream)


def swa_attn_bwd_saved(q, k, v, ve, gate_x, Wg, out, lse, dout, dlse, dq, dk, dv, dve, dgate_x, dWg,
                       B, T, H, D, window, rope_base, eps, workspace, ws_bytes, stream) -> int:
    return _lib.swa_attn_bwd_saved(q, k, v, ve, gate_x, Wg, out, lse, dout, dlse, dq, dk, dv, dve, dgate_x, dWg,
                                   B, T, H, D, window, rope_base, eps, workspace, ws_bytes, stream)


def swa_attn_fwd_x_workspace_bytes(B, T, H, Hkv, D) -> int:
    return int(_lib.swa_attn_fwd_x_workspace_bytes(B, T, H, Hkv, D))


def swa_attn_qkv_prologue(x, Wqkv, ve, Wg, qh, kh, vp, B, T, C, H, Hkv, D, rope_base, eps, workspace,
                          ws_bytes, stream) -> int:
    return _lib.swa_attn_qkv_prologue(x, Wqkv, ve, Wg, qh, kh, vp, B, T, C, H, Hkv, D, rope_base, eps,
                                      workspace, ws_bytes, stream)


def swa_attn_fwd_x(x, Wqkv, ve, Wg, out, lse, B, T, C, H, Hkv, D, window, rope_base, eps, workspace,
                   ws_bytes, stream) -> int:
    return _lib.swa_attn_fwd_x(x, Wqkv, ve, Wg, out, lse, B, T, C, H, Hkv, D, window, rope_base, eps,
                               workspace, ws_bytes, stream)


def swa_attn_selftest_wait(limit_ms: int, stream=None) -> int:
    return int(_lib.swa_attn_selftest_wait(int(limit_ms), stream))


def swa_attn_set_wait_limit_ms(ms: int) -> int:
    return int(_lib.swa_attn_set_wait_limit_ms(int(ms)))


def swa_attn_version() -> int:
    return int(_lib.swa_attn_version())


# ------------------------------------------------------------- tensor-level convenience

def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_handle(stream, device=None):
    """The CUDA stream handle of `stream` (None = the current stream).  A torch stream must belong
    to `device`, the inputs' GPU, when that is given."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    if device is not None and getattr(stream, "device", device) != device:
        raise ValueError(f"stream is on {stream.device}, the inputs on {device}")
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _want(name, t, shape, dtype, device=None):
    """t must be a contiguous CUDA tensor of `shape` and `dtype` (on `device` when given): the C
    calls take bare pointers and cannot check sizes, so a wrong tensor is refused here."""
    if t is None:
        raise ValueError(f"{name} is required")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, not {tuple(t.shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, not {t.dtype}")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the layer's inputs on {device}")


def _want_workspace(ws, device):
    if not ws.is_cuda or not ws.is_contiguous() or ws.device != device:
        raise ValueError(f"workspace must be a contiguous CUDA tensor on {device}")


def _check_qkv(q, k, v, ve, gate_x, Wg):
    """Shapes of a layer call: q (B,T,H,D); k, v and ve (B,T,Hkv,D) with Hkv dividing H (Hkv == H
    for the multi-head layer); gate_x (B,T,32); Wg [32,Hkv].  Returns (B, T, H, Hkv, D)."""
    import torch
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q, k, v must be (B, T, H, D)")
    B, T, H, D = q.shape
    Hkv = k.shape[2]
    kv_shape = (B, T, Hkv, D)
    for name, t, shp in (("q", q, tuple(q.shape)), ("k", k, kv_shape), ("v", v, kv_shape), ("ve", ve, kv_shape)):
        if t is None:
            continue
        if tuple(t.shape) != shp or t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor of shape {shp}")
    if Hkv < 1 or H % Hkv != 0:
        raise ValueError("the key/value head count must divide the query head count")
    if ve is not None:
        if gate_x is None or Wg is None:
            raise ValueError("ve, gate_x and Wg go together")
        if tuple(gate_x.shape) != (B, T, 32) or gate_x.dtype != torch.bfloat16 or not gate_x.is_contiguous():
            raise ValueError("gate_x must be a contiguous bf16 (B, T, 32) tensor")
        if tuple(Wg.shape) != (32, Hkv) or Wg.dtype != torch.bfloat16 or not Wg.is_contiguous():
            raise ValueError(f"Wg must be a contiguous bf16 [32, {Hkv}] tensor")
    elif gate_x is not None or Wg is not None:
        raise ValueError("ve, gate_x and Wg go together")
    for name, t in (("k", k), ("v", v), ("ve", ve), ("gate_x", gate_x), ("Wg", Wg)):
        if t is not None and t.device != q.device:
            raise ValueError(f"{name} is on {t.device}, q on {q.device}")
    return B, T, H, Hkv, D


def forward(q, k, v, window: int = 0, ve=None, gate_x=None, Wg=None, rope_base: float = 10000.0,
            eps: float = 1e-6, *, out=None, lse=None, with_lse: bool = True, workspace=None,
            stream=None, doc=None):
    """One attention layer.  q bf16 (B,T,H,D); k, v (and ve) bf16 (B,T,Hkv,D) CUDA tensors, Hkv
    dividing H (grouped-query attention when Hkv < H: C call swa_attn_fwd_gqa); gate_x (B,T,32);
    Wg [32,Hkv].  Returns (out bf16 (B,T,H,D), lse fp32 (B,H,T) or None).
    ``workspace``: optional uint8 CUDA tensor of at least ``swa_attn_workspace_bytes`` bytes
    (then nothing is allocated by the library; multi-head layers only).
    ``doc``: optional int32 CUDA tensor (B, T) of document ids (C call swa_attn_fwd_doc): a key is
    then visible only inside the query's document, a maximal run of equal ids."""
    import torch
    B, T, H, Hkv, D = _check_qkv(q, k, v, ve, gate_x, Wg)
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    _want("out", out, (B, T, H, D), torch.bfloat16, dev)
    if with_lse and lse is None:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=dev)
    if lse is not None:
        _want("lse", lse, (B, H, T), torch.float32, dev)
    if workspace is not None:
        _want_workspace(workspace, dev)
    if doc is not None:
        _want("doc", doc, (B, T), torch.int32, dev)
        if workspace is not None:
            raise ValueError("the document-masked call uses the library workspace")
    if Hkv != H and workspace is not None:
        raise ValueError("a caller workspace is supported for multi-head layers only")
    with torch.cuda.device(dev):
        st = _stream_handle(stream, dev)
        if doc is not None:
            rc = swa_attn_fwd_doc(_ptr(q), _ptr(k), _ptr(v), _ptr(ve), _ptr(gate_x), _ptr(Wg), _ptr(doc),
                                  _ptr(out), _ptr(lse), B, T, H, Hkv, D, int(window), float(rope_base), float(eps),
                                  st)
            name = "swa_attn_fwd_doc"
        elif Hkv != H:
            rc = swa_attn_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(ve), _ptr(gate_x), _ptr(Wg), _ptr(out),
                                  _ptr(lse), B, T, H, Hkv, D, int(window), float(rope_base), float(eps), st)
            name = "swa_attn_fwd_gqa"
        else:
            args = (_ptr(q), _ptr(k), _ptr(v), _ptr(ve), _ptr(gate_x), _ptr(Wg), _ptr(out), _ptr(lse),
                    B, T, H, D, int(window), float(rope_base), float(eps))
            if workspace is None:
                rc = swa_attn_fwd(*args, st)
            else:
                rc = swa_attn_fwd_ws(*args, _ptr(workspace), workspace.numel() * workspace.element_size(), st)
            name = "swa_attn_fwd"
    if rc != SWA_OK:
        raise SwaError(rc, name)
    return out, lse


def decode(q, k, v, k_cache, v_cache, pos: int, window: int, ve=None, gate_x=None, Wg=None,
           rope_base: float = 1e4, eps: float = 1e-6, out=None, lse=None, workspace=None, stream=None,
           doc_start=None):
    """One generation step (C call swa_attn_decode_doc, which with no ``doc_start`` is
    swa_attn_decode, or swa_attn_decode_gqa when k has fewer heads than q) on torch tensors:
    q (B,H,D), k, v (B,Hkv,D) bf16 of the new token at position ``pos``; ve (B,Hkv,D), gate_x
    (B,32), Wg [32,Hkv] on value-embedding layers; k_cache, v_cache (B,Tmax,Hkv,D) bf16, updated
    in place at ``pos``.  Every tensor is checked against these shapes before the call.
    ``doc_start``: optional int32 CUDA tensor (B,) with the first position of each sequence's
    current document (C call swa_attn_decode_doc).
    Returns (out (B,H,D) bf16, lse (B,H) fp32).  Raises SwaError on a nonzero status."""
    import torch
    if q.dim() != 3 or k.dim() != 3 or k_cache.dim() != 4:
        raise ValueError("q must be (B, H, D), k and v (B, Hkv, D), the caches (B, Tmax, Hkv, D)")
    B, H, D = q.shape
    Hkv = k.shape[1]
    Tmax = k_cache.shape[1]
    dev = q.device
    bf = torch.bfloat16
    _want("q", q, (B, H, D), bf)
    for name, t in (("k", k), ("v", v)):
        _want(name, t, (B, Hkv, D), bf, dev)
    for name, t in (("k_cache", k_cache), ("v_cache", v_cache)):
        _want(name, t, (B, Tmax, Hkv, D), bf, dev)
    if (ve is None) != (gate_x is None) or (ve is None) != (Wg is None):
        raise ValueError("ve, gate_x and Wg go together")
    if ve is not None:
        _want("ve", ve, (B, Hkv, D), bf, dev)
        _want("gate_x", gate_x, (B, 32), bf, dev)
        _want("Wg", Wg, (32, Hkv), bf, dev)
    if out is None:
        out = torch.empty_like(q)
    _want("out", out, (B, H, D), bf, dev)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    _want("lse", lse, (B, H), torch.float32, dev)
    need = swa_attn_decode_workspace_bytes(B, Tmax, H, D, ve is not None, window)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _want_workspace(workspace, dev)
    if doc_start is not None:
        _want("doc_start", doc_start, (B,), torch.int32, dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = _stream_handle(stream, dev)
        rc = _lib.swa_attn_decode_doc(_ptr(q), _ptr(k), _ptr(v), _ptr(ve), _ptr(gate_x), _ptr(Wg), _ptr(k_cache),
                                      _ptr(v_cache), int(pos), _ptr(doc_start), _ptr(out), _ptr(lse), B, Tmax, H,
                                      Hkv, D, int(window), float(rope_base), float(eps), _ptr(workspace), ws_bytes,
                                      st)
    if rc != SWA_OK:
        raise SwaError(rc, "swa_attn_decode_doc" if doc_start is not None else "swa_attn_decode")
    return out, lse


def swa_attn_bwd_doc(q, k, v, ve, gate_x, Wg, doc, out, lse, dout, dlse, dq, dk, dv, dve, dgate_x, dWg,
                     B, T, H, Hkv, D, window, rope_base, eps, workspace, ws_bytes, stream) -> int:
    return _lib.swa_attn_bwd_doc(q, k, v, ve, gate_x, Wg, doc, out, lse, dout, dlse, dq, dk, dv, dve, dgate_x,
                                 dWg, B, T, H, Hkv, D, window, rope_base, eps, workspace, ws_bytes, stream)


def backward(q, k, v, out, lse, dout, window: int = 0, dlse=None, ve=None, gate_x=None, Wg=None,
             rope_base: float = 10000.0, eps: float = 1e-6, *, workspace=None, stream=None, doc=None,
             saved: bool = False):
    """Gradient of one layer (C call swa_attn_bwd_gqa) for the loss sum(dout * out) +
    sum(dlse * lse).  q, k, v, ve, gate_x, Wg as for ``forward``; out bf16 (B,T,H,D) and lse fp32
    (B,H,T) are that call's outputs; dout bf16 (B,T,H,D); dlse fp32 (B,H,T) or None.
    Returns a dict: dq bf16 (B,T,H,D), dk, dv bf16 (B,T,Hkv,D) and, on value-embedding layers,
    dve bf16 (B,T,Hkv,D), dgate_x fp32 (B,T,32), dWg fp32 [32,Hkv].  ``doc``: the int32 (B, T)
    document ids of a document-masked forward (C call swa_attn_bwd_doc).  ``saved``: `workspace`
    (swa_attn_bwd_workspace_bytes() bytes) was passed to the ``forward(..., workspace=...)`` call
    that produced out and lse, so the prologue is not recomputed (C call swa_attn_bwd_saved;
    multi-head, no document mask).  Raises SwaError on a nonzero status."""
    import torch
    if saved and (workspace is None or doc is not None):
        raise ValueError("saved=True needs the forward's workspace, Hkv == H and no document mask")
    B, T, H, Hkv, D = _check_qkv(q, k, v, ve, gate_x, Wg)
    dev = q.device
    for name, t in (("out", out), ("dout", dout)):
        _want(name, t, (B, T, H, D), torch.bfloat16, dev)
    _want("lse", lse, (B, H, T), torch.float32, dev)
    if dlse is not None:
        _want("dlse", dlse, (B, H, T), torch.float32, dev)
    if workspace is not None:
        _want_workspace(workspace, dev)
    g = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v))
    if ve is not None:
        g.update(dve=torch.empty_like(ve),
                 dgate_x=torch.empty((B, T, 32), dtype=torch.float32, device=q.device),
                 dWg=torch.empty((32, Hkv), dtype=torch.float32, device=q.device))
    need = swa_attn_bwd_workspace_bytes(B, T, H, Hkv, D, ve is not None)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    if doc is not None:
        _want("doc", doc, (B, T), torch.int32, dev)
    if saved and Hkv != H:
        raise ValueError("saved=True needs the forward's workspace, Hkv == H and no document mask")
    with torch.cuda.device(dev):
        return _backward_call(q, k, v, ve, gate_x, Wg, doc, out, lse, dout, dlse, g, B, T, H, Hkv, D, window,
                              rope_base, eps, workspace, _stream_handle(stream, dev), saved)


def _backward_call(q, k, v, ve, gate_x, Wg, doc, out, lse, dout, dlse, g, B, T, H, Hkv, D, window, rope_base,
                   eps, workspace, st, saved):
    if saved:
        rc = swa_attn_bwd_saved(_ptr(q), _ptr(k), _ptr(v), _ptr(ve), _ptr(gate_x), _ptr(Wg), _ptr(out), _ptr(lse),
                                _ptr(dout), _ptr(dlse), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g.get("dve")),
                                _ptr(g.get("dgate_x")), _ptr(g.get("dWg")), B, T, H, D, int(window), float(rope_base),
                                float(eps), _ptr(workspace), workspace.numel() * workspace.element_size(), st)
        if rc != SWA_OK:
            raise SwaError(rc, "swa_attn_bwd_saved")
        return g
    rc = swa_attn_bwd_doc(_ptr(q), _ptr(k), _ptr(v), _ptr(ve), _ptr(gate_x), _ptr(Wg), _ptr(doc), _ptr(out),
                          _ptr(lse), _ptr(dout), _ptr(dlse), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]),
                          _ptr(g.get("dve")), _ptr(g.get("dgate_x")), _ptr(g.get("dWg")), B, T, H, Hkv, D,
                          int(window), float(rope_base), float(eps), _ptr(workspace),
                          workspace.numel() * workspace.element_size(), st)
    if rc != SWA_OK:
        raise SwaError(rc, "swa_attn_bwd_doc" if doc is not None else "swa_attn_bwd_gqa")
    return g


def _check_x_w(x, Wqkv, H, Hkv, D, ve, Wg):
    import torch
    if x.dim() != 3:
        raise ValueError("x must be a (B, T, C) tensor")
    B, T, C = x.shape
    N = (H + 2 * Hkv) * D
    _want("x", x, (B, T, C), torch.bfloat16)
    _want("Wqkv", Wqkv, (N, C), torch.bfloat16, x.device)
    if (ve is None) != (Wg is None):
        raise ValueError("ve and Wg go together")
    if ve is not None:
        _want("ve", ve, (B, T, Hkv, D), torch.bfloat16, x.device)
        _want("Wg", Wg, (32, Hkv), torch.bfloat16, x.device)
    return B, T, C


def qkv_prologue(x, Wqkv, H: int, Hkv: int, D: int, ve=None, Wg=None, rope_base: float = 10000.0,
                 eps: float = 1e-6, *, stream=None):
    """q, k, v = x Wqkv^T fused with RoPE / RMS / the gated value embedding (C call
    swa_attn_qkv_prologue).  Returns (qhat (B,T,H,D), khat (B,T,Hkv,D), v' (B,T,Hkv,D)), bf16."""
    import torch
    B, T, C = _check_x_w(x, Wqkv, H, Hkv, D, ve, Wg)
    qh = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=x.device)
    kh = torch.empty((B, T, Hkv, D), dtype=torch.bfloat16, device=x.device)
    vp = torch.empty((B, T, Hkv, D), dtype=torch.bfloat16, device=x.device)
    need = swa_attn_fwd_x_workspace_bytes(B, T, H, Hkv, D)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    with torch.cuda.device(x.device):
        rc = swa_attn_qkv_prologue(_ptr(x), _ptr(Wqkv), _ptr(ve), _ptr(Wg), _ptr(qh), _ptr(kh), _ptr(vp), B, T, C,
                                   H, Hkv, D, float(rope_base), float(eps), _ptr(ws), need,
                                   _stream_handle(stream, x.device))
    if rc != SWA_OK:
        raise SwaError(rc, "swa_attn_qkv_prologue")
    return qh, kh, vp


def forward_x(x, Wqkv, H: int, Hkv: int, D: int, window: int = 0, ve=None, Wg=None,
              rope_base: float = 10000.0, eps: float = 1e-6, *, workspace=None, stream=None):
    """The layer from its input x (C call swa_attn_fwd_x): fused projection + prologue, then the
    windowed attention.  Returns (out bf16 (B,T,H,D), lse fp32 (B,H,T))."""
    import torch
    B, T, C = _check_x_w(x, Wqkv, H, Hkv, D, ve, Wg)
    out = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=x.device)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=x.device)
    need = swa_attn_fwd_x_workspace_bytes(B, T, H, Hkv, D)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    _want_workspace(workspace, x.device)
    with torch.cuda.device(x.device):
        rc = swa_attn_fwd_x(_ptr(x), _ptr(Wqkv), _ptr(ve), _ptr(Wg), _ptr(out), _ptr(lse), B, T, C, H, Hkv, D,
                            int(window), float(rope_base), float(eps), _ptr(workspace),
                            workspace.numel() * workspace.element_size(), _stream_handle(stream, x.device))
    if rc != SWA_OK:
        raise SwaError(rc, "swa_attn_fwd_x")
    return out, lse


def check_device_status(stream=None) -> None:
    """Synchronise and raise SwaError if a kernel recorded an error (e.g. a wait timeout)."""
    rc, detail = swa_attn_last_device_status(_stream_handle(stream))
    if rc != SWA_OK:
        raise SwaError(rc, f"device status word 0x{detail:08x}")


__all__ = [
    "forward", "decode", "backward", "qkv_prologue", "forward_x", "check_device_status", "SwaError",
    "LIB_PATH", "load", "swa_attn_fwd", "swa_attn_fwd_ws", "swa_attn_fwd_noalloc",
    "swa_attn_noalloc_scratch_bytes", "swa_attn_workspace_bytes", "swa_attn_workspace_offset",
    "swa_attn_rope_table", "swa_attn_prologue", "swa_attn_attention", "swa_attn_strerror",
    "swa_attn_last_device_status", "swa_attn_set_wait_limit_ms", "swa_attn_selftest_wait", "swa_attn_version",
    "swa_attn_decode", "swa_attn_decode_gqa", "swa_attn_decode_doc", "swa_attn_decode_workspace_bytes",
    "swa_attn_fwd_gqa", "swa_attn_fwd_doc",
    "swa_attn_bwd", "swa_attn_bwd_saved", "swa_attn_bwd_gqa", "swa_attn_bwd_doc",
    "swa_attn_bwd_workspace_bytes", "swa_attn_fwd_x", "swa_attn_qkv_prologue",
    "swa_attn_fwd_x_workspace_bytes",
]
