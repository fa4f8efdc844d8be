"""GPU parity: the CUDA path, called through the C ABI, against the fp64 oracle on the same
seeded bf16 inputs.  Every element at sizes the oracle finishes in seconds (several tiles and a
ragged tail), sampled rows at the full workload sizes, plus edge cases."""
import numpy as np
import pytest
import torch

import workloads
from tests import parity

pytestmark = pytest.mark.gpu

swa = pytest.importorskip("causal_sliding_window_swa_b200")


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield


def LS(B, T, H, D, window, ve, seed):
    return workloads.LayerShape(B=B, T=T, H=H, D=D, window=window, ve=ve, seed=seed, vocab=4096,
                                model_dim=max(32, H * D), name=f"({B},{T},{H},{D}) W={window} ve={ve}")


# ------------------------------------------------------------- the named workloads

def test_tiny_full():
    parity.check_full(workloads.TINY)


def test_gpt2_124m_full():
    parity.check_full(workloads.GPT2)


@pytest.mark.parametrize("s", [workloads.D24_S, workloads.D24_L_VE], ids=["d24_S", "d24_L_VE"])
def test_d24_full_size_every_element(s):
    """The d24 layers at full size (16, 2048, 12, 128): every element of out and lse against the
    oracle (a few seconds of the oracle on the host's cores)."""
    err = parity.check_full(s)
    print(f"{s.name}: {err}")


@pytest.mark.parametrize("s", [workloads.TINY, workloads.GPT2, workloads.D24_S, workloads.D24_L_VE],
                         ids=["tiny", "gpt2_124m", "d24_S", "d24_L_VE"])
def test_named_workloads_against_pure_fp64_at_sampled_rows(s):
    """Against the oracle's pure fp64 mode (no bf16 rounding of qhat, khat, v' anywhere), at edge
    and random rows of several (b, h) slices: the output within the layer's bar, the LSE within the
    pure-mode bar derived in tests/parity.py.  (The SSSL stack has the same check per layer.)"""
    d = workloads.make_layer(s)
    dev = parity.to_device(d)
    out, lse = parity.run_gpu(s, dev)
    pairs = [(0, 0), (s.B - 1, s.H - 1), (s.B // 2, s.H // 2)]
    rows = workloads.sample_rows(s, n_random=8, seed=17, bh_pairs=pairs)
    err = parity.check_rows(s, d, out, lse, rows, pure=True)
    print(f"{s.name} vs pure fp64: {err}")


# ---------------------------------------------------- full compare on mid-size shapes

@pytest.mark.parametrize("B,T,H,D,window,ve", [
    (2, 1000, 3, 128, 300, True),      # ragged tail, window edge inside tiles, VE
    (1, 1000, 2, 128, 0, False),
    (2, 777, 2, 64, 129, True),
    (1, 640, 4, 64, 0, False),
    (3, 384, 2, 128, 128, False),      # window == tile size
    (1, 1536, 2, 128, 1024, False),    # S-layer shape, scaled down in B/H
])
def test_midsize_full(B, T, H, D, window, ve):
    parity.check_full(LS(B, T, H, D, window, ve, seed=B * 7 + T + window))


# ------------------------------------------------------------------------ edge cases

@pytest.mark.parametrize("T", [1, 2, 7, 127, 128, 129, 255, 256, 257, 383])
@pytest.mark.parametrize("D", [64, 128])
def test_short_sequences(T, D):
    parity.check_full(LS(1, T, 2, D, 0, D == 128, seed=T))


@pytest.mark.parametrize("window", [1, 2, 3, 64, 127, 128, 129, 255, 256, 257, 511])
def test_windows(window):
    parity.check_full(LS(1, 700, 2, 128, window, False, seed=window))


def test_window_ge_T_equals_full_causal_bitwise():
    s = LS(2, 300, 2, 64, 0, True, seed=5)
    d = workloads.make_layer(s)
    dev = parity.to_device(d)
    o_full, l_full = parity.run_gpu(s, dev)
    for w in (300, 301, 10 ** 6, -1):
        o, l = parity.run_gpu(s, dev, window=w)
        assert torch.equal(o, o_full) and torch.equal(l, l_full)


def test_lse_optional_and_ws_and_stages_bitwise_equal():
    s = LS(2, 520, 3, 128, 200, True, seed=11)
    d = workloads.make_layer(s)
    dev = parity.to_device(d)
    o_ref, l_ref = parity.run_gpu(s, dev)
    # lse = NULL
    o2, l2 = swa.forward(dev["q"], dev["k"], dev["v"], s.window, dev["ve"], dev["gate_x"], dev["Wg"],
                         with_lse=False)
    assert l2 is None and torch.equal(o2, o_ref)
    # caller workspace
    nbytes = swa.swa_attn_workspace_bytes(s.B, s.T, s.H, s.D, 1)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    o3, l3 = swa.forward(dev["q"], dev["k"], dev["v"], s.window, dev["ve"], dev["gate_x"], dev["Wg"],
                         workspace=ws)
    assert torch.equal(o3, o_ref) and torch.equal(l3, l_ref)
    # the two stages called separately
    o4 = torch.empty_like(o_ref)
    l4 = torch.empty_like(l_ref)
    st = torch.cuda.current_stream().cuda_stream
    P = lambda t: None if t is None else t.data_ptr()
    rc = swa.swa_attn_rope_table(s.B, s.T, s.H, s.D, 1, 1e4, ws.data_ptr(), nbytes, st)
    assert rc == 0
    rc = swa.swa_attn_prologue(P(dev["q"]), P(dev["k"]), P(dev["v"]), P(dev["ve"]), P(dev["gate_x"]),
                               P(dev["Wg"]), s.B, s.T, s.H, s.D, 1e4, 1e-6, ws.data_ptr(), nbytes, st)
    assert rc == 0
    rc = swa.swa_attn_attention(P(dev["v"]), 1, o4.data_ptr(), l4.data_ptr(), s.B, s.T, s.H, s.D,
                                s.window, ws.data_ptr(), nbytes, st)
    assert rc == 0
    swa.check_device_status()
    assert torch.equal(o4, o_ref) and torch.equal(l4, l_ref)


def test_outputs_stay_inside_their_buffers():
    """Guard bands around out and lse are untouched."""
    s = LS(1, 300, 2, 128, 0, False, seed=3)
    d = workloads.make_layer(s)
    dev = parity.to_device(d)
    n = s.n_elems
    big = torch.full((n + 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
    out = big[2048:2048 + n].view(s.B, s.T, s.H, s.D)
    lbig = torch.full((s.B * s.H * s.T + 2048,), 7.0, dtype=torch.float32, device="cuda")
    lse = lbig[1024:1024 + s.B * s.H * s.T].view(s.B, s.H, s.T)
    swa.forward(dev["q"], dev["k"], dev["v"], 0, out=out, lse=lse)
    swa.check_device_status()
    assert (big[:2048] == 7).all() and (big[2048 + n:] == 7).all()
    assert (lbig[:1024] == 7).all() and (lbig[1024 + s.B * s.H * s.T:] == 7).all()


def test_repeated_calls_are_deterministic():
    s = LS(2, 600, 2, 128, 256, True, seed=13)
    dev = parity.to_device(workloads.make_layer(s))
    o1, l1 = parity.run_gpu(s, dev)
    for _ in range(3):
        o, l = parity.run_gpu(s, dev)
        assert torch.equal(o, o1) and torch.equal(l, l1)


def test_inputs_not_modified():
    s = LS(1, 400, 2, 64, 100, True, seed=17)
    dev = parity.to_device(workloads.make_layer(s))
    before = {k: v.clone() for k, v in dev.items() if v is not None}
    parity.run_gpu(s, dev)
    for k, v in before.items():
        assert torch.equal(v, dev[k]), k


def test_non_default_stream():
    s = LS(1, 500, 2, 128, 0, False, seed=19)
    d = workloads.make_layer(s)
    dev = parity.to_device(d)
    side = torch.cuda.Stream()
    torch.cuda.current_stream().synchronize()
    with torch.cuda.stream(side):
        out, lse = swa.forward(dev["q"], dev["k"], dev["v"], 0)
    side.synchronize()
    swa.check_device_status(side)
    import oracle
    ro, rl = oracle.forward(d, 0)
    parity.compare(out.float().cpu().numpy(), lse.cpu().numpy(), ro, rl, "side stream")


# ------------------------------------------------- prologue: bit-exact against the oracle

def _prologue_on_gpu(s, dev, rope_base=1e4, eps=1e-6):
    has_ve = dev["ve"] is not None
    nbytes = swa.swa_attn_workspace_bytes(s.B, s.T, s.H, s.D, int(has_ve))
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    P = lambda t: None if t is None else t.data_ptr()
    assert swa.swa_attn_rope_table(s.B, s.T, s.H, s.D, int(has_ve), rope_base, ws.data_ptr(), nbytes, st) == 0
    assert swa.swa_attn_prologue(P(dev["q"]), P(dev["k"]), P(dev["v"]), P(dev["ve"]), P(dev["gate_x"]),
                                 P(dev["Wg"]), s.B, s.T, s.H, s.D, rope_base, eps, ws.data_ptr(), nbytes,
                                 st) == 0
    swa.check_device_status()
    n = s.n_elems

    def section(which):
        off = swa.swa_attn_workspace_offset(s.B, s.T, s.H, s.D, int(has_ve), which)
        return ws[off:off + 2 * n].view(torch.int16).view(s.B, s.T, s.H, s.D).cpu()
    out = {"qh": section(swa.SWA_WS_QHAT), "kh": section(swa.SWA_WS_KHAT)}
    out["vp"] = section(swa.SWA_WS_VPRIME) if has_ve else None
    return out


def _bits_of(x64):
    # values the oracle already rounded to bf16 convert exactly
    t = torch.from_numpy(x64).to(torch.float32)
    b = t.to(torch.bfloat16)
    assert torch.equal(b.to(torch.float32), t), "oracle value not bf16-representable"
    return b.view(torch.int16)


@pytest.mark.parametrize("s", [
    LS(2, 1000, 3, 128, 0, True, seed=41),
    LS(3, 513, 4, 64, 0, True, seed=42),
    workloads.D24_L_VE,
], ids=["mid128", "mid64", "d24_L_VE_full"])
def test_prologue_bit_exact(s):
    import oracle
    d = workloads.make_layer(s)
    got = _prologue_on_gpu(s, parity.to_device(d))
    # the C ABI takes eps as fp32: give the oracle that same value
    qh, kh, vp = oracle.prologue(d, eps=float(np.float32(1e-6)), parity=True)
    for name, ref in (("qh", qh), ("kh", kh), ("vp", vp)):
        if got[name] is None:
            continue
        exp = _bits_of(ref)
        mism = (got[name] != exp).sum().item()
        assert mism == 0, f"{name}: {mism} of {exp.numel()} bf16 values differ from the oracle"


@pytest.mark.parametrize("rope_base,eps", [(1e6, 0.0), (500.0, 1e-2)])
def test_prologue_bit_exact_other_constants(rope_base, eps):
    import oracle
    s = LS(1, 700, 2, 128, 0, True, seed=43)
    d = workloads.make_layer(s)
    got = _prologue_on_gpu(s, parity.to_device(d), rope_base=rope_base, eps=eps)
    qh, kh, vp = oracle.prologue(d, rope_base=rope_base, eps=float(np.float32(eps)), parity=True)
    for name, ref in (("qh", qh), ("kh", kh), ("vp", vp)):
        assert (got[name] != _bits_of(ref)).sum().item() == 0, name


def test_prologue_dense_repairs_overflow_the_repair_lists():
    """Every v' element on a bf16 rounding tie: v in [1, 2), ve = 2^-8 (half a bf16 ulp there) and
    Wg = 0 (gate 2 sigmoid(0) = 1, so v' = v + 2^-8 exactly).  The fast path flags all of them, far
    more than a prologue block's repair list holds (ten row chunks per thread at this size, 1024
    list slots per block), so each block recomputes all its chunks in fp64; every element must
    still be v rounded to nearest even, element by element, as the oracle gives."""
    import oracle
    s = LS(1, 4096, 16, 128, 0, True, seed=44)
    d = workloads.make_layer(s)
    g = torch.Generator().manual_seed(44)
    mant = torch.randint(0, 128, d["v"].shape, generator=g, dtype=torch.int32)
    d["v"] = ((0x3F80 | mant).to(torch.int16)).view(torch.bfloat16)          # 1 + m / 128
    d["table"] = torch.full_like(d["table"], 2.0 ** -8)
    d["Wg"] = torch.zeros_like(d["Wg"])
    got = _prologue_on_gpu(s, parity.to_device(d))
    qh, kh, vp = oracle.prologue(d, eps=float(np.float32(1e-6)), parity=True)
    v = d["v"].float()
    even = (mant % 2 == 0)
    expect = torch.where(even, v, v + 2.0 ** -7)                              # ties to even
    assert torch.equal(torch.from_numpy(vp).float(), expect)                 # the oracle agrees
    mism = (got["vp"] != _bits_of(vp)).sum().item()
    assert mism == 0, f"v': {mism} of {vp.size} values differ"
    # the overflowing blocks recompute qhat and khat of all their chunks in fp64 as well
    for name, ref in (("qh", qh), ("kh", kh)):
        mism = (got[name] != _bits_of(ref)).sum().item()
        assert mism == 0, f"{name}: {mism} of {ref.size} values differ"

