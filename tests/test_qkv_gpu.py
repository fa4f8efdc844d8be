"""GPU parity of the fused q/k/v projection + prologue (swa_attn_qkv_prologue) and of the layer
run from its input x (swa_attn_fwd_x), through the C ABI, against the fp64 oracle.

What is compared:
  * qhat, khat, v' element by element with the oracle (``oracle.qkv_prologue``): the projection
    x Wqkv^T summed in fp64, RoPE, RMS and the gated value embedding.  The kernel keeps the
    projection in an fp32 tensor-memory accumulator, so its q, k, v carry the accumulation error
    of a C-term fp32 sum, |dy| <= C 2^-23 sum_c |x_c W_c| (the textbook bound for any summation
    order, with a factor 2 to spare); an output near zero can therefore be several bf16 ulps of
    itself away while being only a tiny absolute distance from the exact value.  The check is that
    bound carried through the prologue: every element within half a bf16 ulp of the exact value
    (the oracle's pure mode) plus r (|dy_a| + |dy_b|) + |qhat| sum|y||dy| / (ss + D eps) plus a few
    fp32 roundings for q / k heads, and plus |dy| for v heads; the elements that differ from the
    correctly rounded value (the oracle's parity mode) are counted and must stay rare.
  * out and lse of ``swa_attn_fwd_x`` against the oracle's attention on the oracle's own rounded
    qhat, khat, v' (its prologue switched off by the test-only flags), at the forward tolerances
    (max-abs 2e-2, relative L2 5e-3, LSE 1e-3).

The projection is the bias-free linear map of the layer input ("Let's reproduce GPT-2 (124M)"
notes, section 3, the attention listing, where q, k, v come from one 3C projection; the speedrun
write-ups use a narrower key/value width, covered by Hkv < H); the value-embedding gate follows the
PaperWeekly repost, "Value Embeddings".

Shapes cover D 64 and 128, Hkv < H, value embeddings on and off, ragged token counts, and both
tilings of the kernel (BN = 256 when the q and k/v widths are multiples of 256, else BN = 128).
"""
import numpy as np
import pytest
import torch

import oracle
from tests import parity

pytestmark = pytest.mark.gpu

swa = pytest.importorskip("causal_sliding_window_swa_b200")

MISMATCH_MAX_FRACTION = 5e-3


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield


def _draw(B, T, C, H, Hkv, D, ve, seed, vocab=997):
    """x ~ N(0,1) (B,T,C); Wqkv ~ N(0, 1/C) (so q, k, v are about unit scale); value-embedding
    table ~ N(0,1) gathered by uniform ids; Wg ~ N(0, 0.02), all bf16 (round to nearest)."""
    g = torch.Generator().manual_seed(seed)
    bf = lambda *shape, std=1.0: (torch.randn(shape, generator=g) * std).to(torch.bfloat16)
    d = dict(x=bf(B, T, C), W=bf((H + 2 * Hkv) * D, C, std=C ** -0.5))
    if ve:
        d.update(ids=torch.randint(0, vocab, (B, T), generator=g), table=bf(vocab, Hkv * D),
                 Wg=bf(32, Hkv, std=0.02))
        d["ve"] = d["table"][d["ids"]].reshape(B, T, Hkv, D).contiguous()
    return d


def _check_bound(got, exact, rounded, bound, what):
    """|got - exact| <= half a bf16 ulp of got + bound, elementwise; differences from the correctly
    rounded value counted (and rare)."""
    g = got.double().cpu().numpy()
    half_ulp = np.ldexp(1.0, np.frexp(np.abs(g))[1] - 9)
    excess = np.abs(g - exact) - half_ulp - bound
    n_diff = int((g != rounded).sum())
    print(f"{what}: {n_diff} of {g.size} elements differ from the correctly rounded value; "
          f"worst margin to the bound {excess.max():.3e}")
    assert excess.max() <= 0.0, f"{what}: an element is {excess.max():.3e} beyond its bound"
    assert n_diff <= MISMATCH_MAX_FRACTION * g.size, f"{what}: {n_diff} elements differ"


def _check_projection(d, B, T, C, H, Hkv, D, qh, kh, vp, eps=1e-6):
    x = d["x"].double().numpy().reshape(B, T, C)
    Wm = d["W"].double().numpy()
    y = x @ Wm.T                                    # (B, T, N), exact products, fp64 sum
    dy = C * 2.0 ** -23 * (np.abs(x) @ np.abs(Wm).T)
    px = oracle.qkv_prologue(d["x"], d["W"], H, Hkv, D, ids=d.get("ids"), table=d.get("table"),
                             Wg=d.get("Wg"), parity=False)
    pr = oracle.qkv_prologue(d["x"], d["W"], H, Hkv, D, ids=d.get("ids"), table=d.get("table"),
                             Wg=d.get("Wg"), parity=True)
    eps = float(np.float32(eps))
    for name, heads, off, got, ex, rd in (("qhat", H, 0, qh, px[0], pr[0]), ("khat", Hkv, H * D, kh, px[1], pr[1])):
        yh = y[..., off:off + heads * D].reshape(B, T, heads, D)
        dyh = dy[..., off:off + heads * D].reshape(B, T, heads, D)
        swap = lambda a: np.concatenate([a[..., D // 2:], a[..., :D // 2]], axis=-1)   # RoPE partner
        ss = (yh ** 2).sum(-1, keepdims=True)
        r = 1.0 / np.sqrt(ss / D + eps)
        dss = 2.0 * (np.abs(yh) * dyh).sum(-1, keepdims=True)
        bound = (r * (dyh + swap(dyh)) + np.abs(ex) * dss / (ss + D * eps)
                 + 2.0 ** -20 * (r * (np.abs(yh) + np.abs(swap(yh))) + np.abs(ex)))
        _check_bound(got, ex, rd, bound, name)
    yv = y[..., (H + Hkv) * D:].reshape(B, T, Hkv, D)
    dyv = dy[..., (H + Hkv) * D:].reshape(B, T, Hkv, D)
    ve = d["ve"].double().numpy() if "ve" in d else np.zeros_like(yv)
    bound = dyv + 2.0 ** -20 * (np.abs(px[2]) + 2.0 * np.abs(ve))
    _check_bound(vp, px[2], pr[2], bound, "v'")


CASES = [
    # B, T, C, H, Hkv, D, ve             tiling
    (2, 300, 256, 2, 2, 128, True),      # BN 256 (widths 256), ragged T
    (1, 257, 512, 4, 2, 128, False),     # BN 256, grouped-query, ragged
    (2, 200, 384, 4, 2, 64, True),       # BN 128 (k/v width 128), grouped-query
    (1, 129, 192, 3, 3, 64, False),      # BN 128, widths 192, ragged, N not a multiple of 256
    (1, 384, 136, 2, 1, 64, True),       # C not a multiple of 64 (last chunk zero-filled)
]


@pytest.mark.parametrize("B,T,C,H,Hkv,D,ve", CASES)
def test_qkv_prologue_within_the_accumulation_bound(B, T, C, H, Hkv, D, ve):
    d = _draw(B, T, C, H, Hkv, D, ve, seed=B * 1000 + T + C + D)
    g = {k: v.cuda() for k, v in d.items() if k in ("x", "W", "ve", "Wg")}
    qh, kh, vp = swa.qkv_prologue(g["x"], g["W"], H, Hkv, D, ve=g.get("ve"), Wg=g.get("Wg"))
    swa.check_device_status()
    _check_projection(d, B, T, C, H, Hkv, D, qh, kh, vp)


@pytest.mark.parametrize("B,T,C,H,Hkv,D,ve,window", [
    (2, 300, 256, 2, 2, 128, True, 0),
    (1, 257, 512, 4, 2, 128, False, 100),
    (2, 200, 384, 4, 2, 64, True, 64),
    (1, 129, 192, 3, 3, 64, False, 0),
])
def test_forward_x_matches_the_oracle(B, T, C, H, Hkv, D, ve, window):
    d = _draw(B, T, C, H, Hkv, D, ve, seed=7 * B + T + C + window)
    g = {k: v.cuda() for k, v in d.items() if k in ("x", "W", "ve", "Wg")}
    out, lse = swa.forward_x(g["x"], g["W"], H, Hkv, D, window, ve=g.get("ve"), Wg=g.get("Wg"))
    swa.check_device_status()
    rq, rk, rv = oracle.qkv_prologue(d["x"], d["W"], H, Hkv, D, ids=d.get("ids"), table=d.get("table"),
                                     Wg=d.get("Wg"), parity=True)
    as_bf = lambda a: torch.from_numpy(a).to(torch.bfloat16)
    inputs = dict(q=as_bf(rq), k=as_bf(rk), v=as_bf(rv))
    ref_o, ref_l = oracle.forward(inputs, window, parity=True, rope=False, qknorm=False)
    parity.compare(out.float().cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l,
                   f"forward_x ({B},{T},C={C},{H}/{Hkv},{D}) W={window} ve={ve}")


def test_forward_x_equals_forward_on_the_projected_tensors():
    """The layer from x equals the attention stage run on the fused kernel's own qhat, khat, v'
    (the same attention kernel on the same operands), bit for bit."""
    B, T, C, H, Hkv, D = 2, 333, 256, 2, 2, 128
    d = _draw(B, T, C, H, Hkv, D, True, seed=31)
    g = {k: v.cuda() for k, v in d.items() if k in ("x", "W", "ve", "Wg")}
    out, lse = swa.forward_x(g["x"], g["W"], H, Hkv, D, 150, ve=g["ve"], Wg=g["Wg"])
    qh, kh, vp = swa.qkv_prologue(g["x"], g["W"], H, Hkv, D, ve=g["ve"], Wg=g["Wg"])
    # the attention stage alone reads qhat / khat / v' from a workspace laid out by the library
    nbytes = swa.swa_attn_workspace_bytes(B, T, H, D, 1)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    off = lambda sec: swa.swa_attn_workspace_offset(B, T, H, D, 1, sec)
    n = B * T * H * D * 2
    ws[off(swa.SWA_WS_QHAT):off(swa.SWA_WS_QHAT) + n].copy_(qh.view(torch.uint8).reshape(-1))
    ws[off(swa.SWA_WS_KHAT):off(swa.SWA_WS_KHAT) + n].copy_(kh.view(torch.uint8).reshape(-1))
    ws[off(swa.SWA_WS_VPRIME):off(swa.SWA_WS_VPRIME) + n].copy_(vp.view(torch.uint8).reshape(-1))
    o2 = torch.empty_like(out)
    l2 = torch.empty_like(lse)
    st = torch.cuda.current_stream().cuda_stream
    assert swa.swa_attn_attention(None, 1, o2.data_ptr(), l2.data_ptr(), B, T, H, D, 150, ws.data_ptr(),
                                  nbytes, st) == swa.SWA_OK
    swa.check_device_status()
    assert torch.equal(out, o2) and torch.equal(lse, l2)
