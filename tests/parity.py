"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI on the seeded
inputs, and compare element by element with the fp64 oracle (parity mode).

Tolerances: out max-abs 2e-2 and relative L2 5e-3 (bf16 I/O, fp32 accumulation), LSE max-abs
1e-3 -- the bar the layer's specification states -- against the oracle's parity mode, which rounds
qhat, khat, v' to bf16 as the tensor-core operands are.

Against the oracle's pure fp64 mode (no rounding of qhat, khat, v') the output keeps the same
bar, but the LSE cannot: rounding the 2D operands of a single score to bf16 (relative 2^-9 each)
moves that score, and so the LSE of a row that sees few keys: for unit-RMS operands the 2D
rounding errors (uniform, up to 2^-9 relative) give the score a standard deviation of
2^-9 sqrt(2/3) ~ 1.6e-3; the oracle's own parity and pure modes differ by up to 6e-3 at row 0 of
the d24 layers.  The pure-mode LSE bar is therefore 1.5e-2 (about nine standard deviations of
that single-score deviation), stated here and asserted alongside the 1e-3 parity-mode bar."""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

import oracle
import workloads

OUT_MAX_ABS = 2e-2
OUT_REL_L2 = 5e-3
LSE_MAX_ABS = 1e-3
LSE_MAX_ABS_PURE = 1.5e-2


def to_device(d: Dict[str, torch.Tensor], device="cuda"):
    g = workloads.gpu_side_inputs(d)
    return {k: (None if v is None else v.to(device)) for k, v in g.items()}


def run_gpu(s: workloads.LayerShape, dev: Dict, *, nan_fill=True, window=None, **kw):
    import causal_sliding_window_swa_b200 as swa
    q = dev["q"]
    out = torch.empty_like(q)
    lse = torch.empty((s.B, s.H, s.T), dtype=torch.float32, device=q.device)
    if nan_fill:
        out.fill_(float("nan"))
        lse.fill_(float("nan"))
    swa.forward(q, dev["k"], dev["v"], s.window if window is None else window, dev["ve"],
                dev["gate_x"], dev["Wg"], out=out, lse=lse, **kw)
    swa.check_device_status()
    return out, lse


def compare(out_gpu: np.ndarray, lse_gpu: np.ndarray, out_ref: np.ndarray, lse_ref: np.ndarray,
            what: str = "", lse_tol: float = LSE_MAX_ABS):
    assert np.isfinite(out_gpu).all(), f"{what}: non-finite output (unwritten element?)"
    assert np.isfinite(lse_gpu).all(), f"{what}: non-finite lse (unwritten element?)"
    err = np.abs(out_gpu - out_ref)
    max_abs = float(err.max()) if err.size else 0.0
    rel_l2 = float(np.linalg.norm(out_gpu - out_ref) / max(np.linalg.norm(out_ref), 1e-30))
    lse_err = float(np.abs(lse_gpu - lse_ref).max()) if lse_ref.size else 0.0
    msg = f"{what}: max_abs={max_abs:.3e} rel_l2={rel_l2:.3e} lse_max_abs={lse_err:.3e}"
    assert max_abs <= OUT_MAX_ABS, msg
    assert rel_l2 <= OUT_REL_L2, msg
    assert lse_err <= lse_tol, msg
    return dict(max_abs=max_abs, rel_l2=rel_l2, lse_max_abs=lse_err)


def check_full(s: workloads.LayerShape, d: Optional[Dict] = None, **kw):
    """Every element of out and lse against the oracle."""
    d = workloads.make_layer(s) if d is None else d
    out, lse = run_gpu(s, to_device(d), **kw)
    ref_o, ref_l = oracle.forward(d, s.window, parity=True)
    return compare(out.float().cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, s.name)


def check_rows(s: workloads.LayerShape, d: Dict, out: torch.Tensor, lse: torch.Tensor, rows, *,
               pure: bool = False):
    """Sampled rows (flat ids (b*H + h)*T + i) against the oracle (parity mode, or pure fp64 mode
    with its LSE bar), plus finiteness everywhere."""
    rows = torch.as_tensor(rows, dtype=torch.int64)
    ref_o, ref_l = oracle.forward(d, s.window, parity=not pure, rows=rows)
    b = rows // (s.H * s.T)
    h = (rows // s.T) % s.H
    i = rows % s.T
    o = out[b.cuda(), i.cuda(), h.cuda()].float().cpu().numpy()
    l = lse[b.cuda(), h.cuda(), i.cuda()].cpu().numpy()
    assert torch.isfinite(out).all().item() and torch.isfinite(lse).all().item(), f"{s.name}: non-finite"
    return compare(o, l, ref_o, ref_l, s.name + (" (sampled rows, pure fp64)" if pure else " (sampled rows)"),
                   lse_tol=LSE_MAX_ABS_PURE if pure else LSE_MAX_ABS)
