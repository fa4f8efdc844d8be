"""Seeded synthetic inputs for the attention layer, shared by the oracle side and the GPU side.

This module holds only shapes, seeds and random draws.  It computes nothing of the
attention layer itself: no RoPE, no normalisation, no gate, no softmax.  Both the CPU
oracle (``oracle/``) and the CUDA path (``causal_sliding_window_swa_b200``) take their
inputs from here, so they see the same bf16 bytes.

Workloads follow the pages' layer shapes:

* GPT-2 124M attention: C = 768, H = 12, D = 64, T = 1024
  ("Let's reproduce GPT-2 (124M)" notes, section 3, the multi-head attention listing).
* nanochat d24: model dim = depth x 64 = 1536, H = 12, D = 128, T = 2048, sliding windows
  S = 1024 / L = 2048 in the S,S,S,L pattern
  (intelliparadigm "GPT-2 for $73", section 3.2; PaperWeekly repost, "Attention" paragraph).
* Value embeddings: table [vocab, kv_dim] gathered by token id; gate reads x[..., :32]
  (PaperWeekly repost, "Value Embeddings" paragraph).

Activations are i.i.d. N(0, 1) drawn in fp32 and rounded to bf16 (round to nearest even);
the pages train on FineWeb-Edu, which is not needed here: random normals stand in for
the activations of that run.
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import Dict, List, Optional, Tuple

import torch

VOCAB = 32768          # nanochat vocabulary size used for the value-embedding table
GATE_CHANNELS = 32     # the gate reads the first 32 channels of x
WG_STD = 0.02          # Wg ~ N(0, 0.02)


@dataclasses.dataclass(frozen=True)
class LayerShape:
    B: int
    T: int
    H: int
    D: int
    window: int          # <= 0 or >= T means full causal
    ve: bool             # value-embedding layer
    seed: int
    name: str = ""
    vocab: int = VOCAB
    model_dim: int = 0   # channels of x (defaults to H*D)
    kv_heads: int = 0    # key/value heads (grouped-query attention); 0 means H

    @property
    def Hkv(self) -> int:
        return self.kv_heads if self.kv_heads > 0 else self.H

    @property
    def C(self) -> int:
        return self.model_dim if self.model_dim > 0 else self.H * self.D

    @property
    def n_elems(self) -> int:
        return self.B * self.T * self.H * self.D

    def eff_window(self) -> int:
        return self.T if (self.window <= 0 or self.window >= self.T) else self.window

    def unmasked_pairs(self) -> int:
        """Visible (query, key) pairs per call: key j visible to query i iff 0 <= i - j < W."""
        W = self.eff_window()
        per_bh = W * (W + 1) // 2 + (self.T - W) * W
        return self.B * self.H * per_bh


# The five workloads.  Index 0..3 are single layers; the SSSL stack is described separately.
TINY = LayerShape(B=1, T=256, H=4, D=64, window=0, ve=False, seed=0, name="tiny (1,256,4,64) full")
GPT2 = LayerShape(B=8, T=1024, H=12, D=64, window=0, ve=False, seed=1, name="gpt2-124m (8,1024,12,64) full")
D24_S = LayerShape(B=16, T=2048, H=12, D=128, window=1024, ve=False, seed=2,
                   name="d24 S (16,2048,12,128) W=1024")
D24_L_VE = LayerShape(B=16, T=2048, H=12, D=128, window=2048, ve=True, seed=3,
                      name="d24 L+VE (16,2048,12,128) W=2048")
SINGLE_LAYERS: List[LayerShape] = [TINY, GPT2, D24_S, D24_L_VE]

SSSL_SEED = 4
SSSL_LAYERS = 24
SSSL_POINTS: List[Tuple[int, int]] = [(32, 1024), (16, 2048), (8, 4096), (4, 8192), (2, 16384)]


def sssl_layer_shapes(B: int, T: int, H: int = 12, D: int = 128,
                      n_layers: int = SSSL_LAYERS) -> List[LayerShape]:
    """Window pattern S,S,S,L (S = T/2, L = T); value embeddings on even layer indices."""
    out = []
    for layer in range(n_layers):
        long_layer = (layer % 4) == 3
        out.append(LayerShape(B=B, T=T, H=H, D=D, window=(T if long_layer else T // 2),
                              ve=(layer % 2 == 0), seed=SSSL_SEED,
                              name=f"sssl B={B} T={T} layer {layer}"))
    return out


def _bf16_normal(gen: torch.Generator, shape, std: float = 1.0) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def draw_layer(gen: torch.Generator, s: LayerShape) -> Dict[str, torch.Tensor]:
    """Draw one layer's inputs from ``gen`` in a fixed order: q, k, v, then (VE) ids, table, x, Wg.

    Returns CPU tensors: q bf16 (B,T,H,D), k, v bf16 (B,T,Hkv,D); for VE layers also ids int64
    (B,T), table bf16 [vocab, Hkv*D], x bf16 (B,T,C), Wg bf16 [32, Hkv].  With Hkv == H (the
    default) the draws are those of the multi-head layer.
    """
    shp = (s.B, s.T, s.H, s.D)
    kv_shp = (s.B, s.T, s.Hkv, s.D)
    d: Dict[str, torch.Tensor] = {}
    d["q"] = _bf16_normal(gen, shp)
    d["k"] = _bf16_normal(gen, kv_shp)
    d["v"] = _bf16_normal(gen, kv_shp)
    if s.ve:
        d["ids"] = torch.randint(0, s.vocab, (s.B, s.T), generator=gen, dtype=torch.int64)
        d["table"] = _bf16_normal(gen, (s.vocab, s.Hkv * s.D))
        d["x"] = _bf16_normal(gen, (s.B, s.T, s.C))
        d["Wg"] = _bf16_normal(gen, (GATE_CHANNELS, s.Hkv), std=WG_STD)
    return d


def make_layer(s: LayerShape) -> Dict[str, torch.Tensor]:
    """Inputs of a single-layer workload, from its own seed."""
    gen = torch.Generator().manual_seed(s.seed)
    return draw_layer(gen, s)


def sssl_stack(B: int, T: int, H: int = 12, D: int = 128, n_layers: int = SSSL_LAYERS):
    """Yield (shape, inputs) for each layer of the SSSL stack, drawn sequentially from one
    generator seeded once, so every layer has its own tensors."""
    gen = torch.Generator().manual_seed(SSSL_SEED)
    for s in sssl_layer_shapes(B, T, H, D, n_layers):
        yield s, draw_layer(gen, s)


def gpu_side_inputs(d: Dict[str, torch.Tensor]) -> Dict[str, Optional[torch.Tensor]]:
    """The tensors the C-ABI call takes: gathered ve = table[ids] (B,T,H,D) and the contiguous
    gate slice x[..., :32].  This is the embedding lookup that sits before the attention call;
    the oracle does its own lookup from ids and table."""
    q, k, v = d["q"], d["k"], d["v"]
    if "ids" not in d:
        return dict(q=q, k=k, v=v, ve=None, gate_x=None, Wg=None)
    B, T, Hkv, D = k.shape
    ve = d["table"][d["ids"]].view(B, T, Hkv, D)
    gate_x = d["x"][..., :GATE_CHANNELS].contiguous()
    return dict(q=q, k=k, v=v, ve=ve, gate_x=gate_x, Wg=d["Wg"].contiguous())


def sha256_of(d: Dict[str, torch.Tensor]) -> str:
    h = hashlib.sha256()
    for key in sorted(d):
        t = d[key]
        if t is None:
            continue
        h.update(key.encode())
        h.update(t.contiguous().view(torch.uint8).numpy().tobytes() if t.dtype != torch.int64
                 else t.contiguous().numpy().tobytes())
    return h.hexdigest()


def sample_rows(s: LayerShape, n_random: int, seed: int, bh_pairs: Optional[List[Tuple[int, int]]] = None):
    """Deterministic query rows to check at full size: the edge rows 0, 1, W-1, W, W+1, 127, 128,
    T-1 plus ``n_random`` seeded rows, for each (b, h) in ``bh_pairs`` (default: all).
    Returns a sorted int64 tensor of flat row ids ((b*H + h)*T + i)."""
    W = s.eff_window()
    g = torch.Generator().manual_seed(seed)
    fixed = [0, 1, W - 1, W, W + 1, 127, 128, s.T - 1]
    if bh_pairs is None:
        bh_pairs = [(b, h) for b in range(s.B) for h in range(s.H)]
    rows = set()
    for (b, h) in bh_pairs:
        cand = [i for i in fixed if 0 <= i < s.T]
        if n_random > 0:
            cand += torch.randint(0, s.T, (n_random,), generator=g).tolist()
        for i in cand:
            rows.add((b * s.H + h) * s.T + i)
    return torch.tensor(sorted(rows), dtype=torch.int64)
