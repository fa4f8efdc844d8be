"""Pins of the fp64 oracle against things other than itself: brute force, a library routine,
closed forms and invariants of the definition.  CPU only.

The definition (scores, causal mask including the diagonal, softmax, weighted sum) is the one
of "Let's reproduce GPT-2 (124M)" notes, section 3; the RoPE -> norm order is intelliparadigm
"GPT-2 for $73", section 2.2; the window is section 3.2 there; the gate is the PaperWeekly
repost's "Value Embeddings" paragraph.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from scipy.special import expit

import oracle
import oracle.brute as brute
import workloads


def _rand_layer(B, T, H, D, ve=False, seed=0, vocab=97):
    s = workloads.LayerShape(B=B, T=T, H=H, D=D, window=0, ve=ve, seed=seed, vocab=vocab,
                             model_dim=max(32, H * D))
    return workloads.make_layer(s)


# ---------------------------------------------------------------- brute force (NumPy, T x T)

@pytest.mark.parametrize("B,T,H,D", [(1, 1, 1, 64), (2, 3, 2, 8), (1, 129, 2, 64), (1, 70, 3, 128)])
@pytest.mark.parametrize("window", [0, 1, 5, 64, 1000])
@pytest.mark.parametrize("ve", [False, True])
def test_oracle_matches_bruteforce(B, T, H, D, window, ve):
    d = _rand_layer(B, T, H, D, ve=ve, seed=B * 1000 + T + window)
    o, l = oracle.forward(d, window, parity=False)
    ob, lb = brute.forward(d, window)
    assert np.abs(o - ob).max() < 1e-12
    assert np.abs(l - lb).max() < 1e-12


@pytest.mark.parametrize("window", [1, 7, 33])
def test_window_convention_switch_matches_bruteforce(window):
    d = _rand_layer(1, 50, 2, 16, seed=window)
    o, l = oracle.forward(d, window, parity=False, window_convention=1)
    ob, lb = brute.forward(d, window, convention=1)
    assert np.abs(o - ob).max() < 1e-12 and np.abs(l - lb).max() < 1e-12


# ----------------------------------------------------- library special case: torch SDPA fp64

@pytest.mark.parametrize("window", [0, 1, 9, 40])
def test_no_prologue_equals_torch_sdpa(window):
    """With RoPE and QK-norm switched off (test-only flags) and no value embedding, the layer
    is plain scaled-dot-product attention with a banded causal mask: torch's fp64 CPU SDPA."""
    B, T, H, D = 2, 77, 3, 64
    d = _rand_layer(B, T, H, D, seed=window + 5)
    o, l = oracle.forward(d, window, parity=False, rope=False, qknorm=False)
    q = d["q"].double().permute(0, 2, 1, 3)
    k = d["k"].double().permute(0, 2, 1, 3)
    v = d["v"].double().permute(0, 2, 1, 3)
    W = T if window <= 0 or window >= T else window
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    mask = (i - j >= 0) & (i - j < W)
    ref = F.scaled_dot_product_attention(q, k, v, attn_mask=mask).permute(0, 2, 1, 3)
    assert np.abs(o - ref.numpy()).max() < 1e-12
    s = (q @ k.transpose(-1, -2)) / math.sqrt(D)
    ref_lse = torch.logsumexp(s.masked_fill(~mask, float("-inf")), dim=-1)
    assert np.abs(l - ref_lse.numpy()).max() < 1e-12


# --------------------------------------------------------------------------- window pins

def test_window_ge_T_and_le_0_are_full_causal_bitwise():
    d = _rand_layer(1, 96, 2, 64, ve=True, seed=3)
    full, lfull = oracle.forward(d, 0)
    for w in (-5, 96, 97, 5000):
        o, l = oracle.forward(d, w)
        assert np.array_equal(o, full) and np.array_equal(l, lfull)


def test_rows_before_window_unaffected_by_window():
    T, W = 100, 37
    d = _rand_layer(2, T, 2, 64, seed=11)
    full, lfull = oracle.forward(d, 0)
    o, l = oracle.forward(d, W)
    assert np.array_equal(o[:, :W], full[:, :W])
    assert np.array_equal(l[:, :, :W], lfull[:, :, :W])
    assert not np.allclose(o[:, W:], full[:, W:])


def test_window_one_is_identity_on_v_prime():
    d = _rand_layer(1, 40, 3, 64, ve=True, seed=2)
    o, l = oracle.forward(d, 1, parity=False)
    qh, kh, vp = oracle.prologue(d)
    assert np.abs(o - vp).max() < 1e-14
    s_ii = np.einsum("bthd,bthd->bht", qh, kh) / math.sqrt(64)
    assert np.abs(l - s_ii).max() < 1e-13


# ------------------------------------------------------------------------- closed forms

def test_row_zero_is_gated_v0_and_its_single_score():
    d = _rand_layer(2, 33, 2, 128, ve=True, seed=8)
    o, l = oracle.forward(d, 0, parity=False)
    qh, kh, vp = oracle.prologue(d)
    assert np.abs(o[:, 0] - vp[:, 0]).max() < 1e-14
    s00 = np.einsum("bhd,bhd->bh", qh[:, 0], kh[:, 0]) / math.sqrt(128)
    assert np.abs(l[:, :, 0] - s00).max() < 1e-13


def test_constant_values_give_constant_output_rows_sum_to_one():
    """v = c for every key: each output row is sum_j p_j c = c iff the weights sum to 1."""
    d = _rand_layer(1, 64, 2, 64, seed=4)
    c = torch.randn(1, 1, 2, 64).to(torch.bfloat16)
    d["v"] = c.expand(1, 64, 2, 64).contiguous()
    for w in (0, 10):
        o, _ = oracle.forward(d, w, parity=False)
        assert np.abs(o - c.double().numpy()).max() < 1e-14


def test_zero_queries_give_uniform_weights():
    """q = 0 -> qhat = 0 -> every score is 0: out_i is the mean of v' over the visible keys and
    lse_i = ln |J_i|."""
    T, W = 50, 12
    d = _rand_layer(1, T, 2, 64, ve=True, seed=6)
    d["q"] = torch.zeros_like(d["q"])
    o, l = oracle.forward(d, W, parity=False)
    _, _, vp = oracle.prologue(d)
    for i in range(T):
        lo = max(0, i - W + 1)
        assert np.abs(o[0, i] - vp[0, lo:i + 1].mean(axis=0)).max() < 1e-14
        assert abs(l[0, 0, i] - math.log(i + 1 - lo)) < 1e-14


def test_hand_derived_two_token_case():
    """B=1, T=2, H=1, D=2, eps=0.  D=2 has one pair with theta_0 = 1, so position 1 rotates by
    1 rad.  q0 = q1 = k0 = (1,0), k1 = (0,1): qhat0 = khat0 = sqrt2 (1,0),
    qhat1 = sqrt2 (cos1, sin1), khat1 = sqrt2 (-sin1, cos1).  Scores (scale 1/sqrt2):
    s00 = sqrt2, s10 = sqrt2 cos1, s11 = 0.  Row 0 -> v0, lse0 = sqrt2.
    Row 1 -> (e^{s10} v0 + v1) / (e^{s10} + 1), lse1 = ln(e^{s10} + 1)."""
    bf = torch.bfloat16
    q = torch.tensor([[[[1.0, 0.0]], [[1.0, 0.0]]]], dtype=bf)
    k = torch.tensor([[[[1.0, 0.0]], [[0.0, 1.0]]]], dtype=bf)
    v = torch.tensor([[[[2.0, -1.0]], [[0.5, 3.0]]]], dtype=bf)
    o, l = oracle.forward(dict(q=q, k=k, v=v), 0, rope_base=10000.0, eps=0.0, parity=False)
    s10 = math.sqrt(2.0) * math.cos(1.0)
    e = math.exp(s10)
    row1 = [(e * 2.0 + 0.5) / (e + 1.0), (e * -1.0 + 3.0) / (e + 1.0)]
    assert np.abs(o[0, 0, 0] - [2.0, -1.0]).max() < 1e-15
    assert np.abs(o[0, 1, 0] - row1).max() < 1e-15
    assert abs(l[0, 0, 0] - math.sqrt(2.0)) < 1e-15
    assert abs(l[0, 0, 1] - math.log(e + 1.0)) < 1e-15


# -------------------------------------------------------------------------------- RoPE

def test_rope_d2_is_rotation_by_t_radians():
    """D = 2: theta_0 = base^0 = 1 for every base; (1, 0) at position t -> (cos t, sin t)."""
    T = 300
    q = torch.zeros(1, T, 1, 2)
    q[..., 0] = 1.0
    d = dict(q=q.to(torch.bfloat16), k=q.to(torch.bfloat16), v=q.to(torch.bfloat16))
    for base in (10000.0, 500.0):
        qh, _, _ = oracle.prologue(d, rope_base=base, qknorm=False)
        t = np.arange(T)
        assert np.abs(qh[0, :, 0, 0] - np.cos(t)).max() < 1e-14
        assert np.abs(qh[0, :, 0, 1] - np.sin(t)).max() < 1e-14


def test_rope_d4_second_pair_uses_base_power():
    """D = 4: pairs (0,2) and (1,3); theta_1 = base^(-2/4) = 1/sqrt(base) (0.01 for 1e4)."""
    T = 64
    x = torch.zeros(1, T, 1, 4)
    x[..., 1] = 1.0          # the pair (1, 3) only
    d = dict(q=x.to(torch.bfloat16), k=x.to(torch.bfloat16), v=x.to(torch.bfloat16))
    qh, _, _ = oracle.prologue(d, rope_base=10000.0, qknorm=False)
    t = np.arange(T) * 0.01
    assert np.abs(qh[0, :, 0, 1] - np.cos(t)).max() < 1e-14
    assert np.abs(qh[0, :, 0, 3] - np.sin(t)).max() < 1e-14
    assert np.abs(qh[0, :, 0, 0]).max() == 0 and np.abs(qh[0, :, 0, 2]).max() == 0


def test_rope_preserves_norm_and_is_identity_at_zero():
    d = _rand_layer(2, 200, 3, 128, seed=21)
    qh, kh, _ = oracle.prologue(d, qknorm=False)
    q = d["q"].double().numpy()
    assert np.abs(np.linalg.norm(qh, axis=-1) / np.linalg.norm(q, axis=-1) - 1).max() < 1e-14
    assert np.array_equal(qh[:, 0], q[:, 0])


def test_rope_relative_position():
    """Same raw q at every position, same raw k at every position: rope(q,t).rope(k,s) depends on
    t - s only."""
    T, D = 40, 64
    q1 = torch.randn(1, 1, 1, D).to(torch.bfloat16)
    k1 = torch.randn(1, 1, 1, D).to(torch.bfloat16)
    d = dict(q=q1.expand(1, T, 1, D).contiguous(), k=k1.expand(1, T, 1, D).contiguous(),
             v=q1.expand(1, T, 1, D).contiguous())
    qh, kh, _ = oracle.prologue(d, qknorm=False)
    G = np.einsum("td,sd->ts", qh[0, :, 0], kh[0, :, 0])
    for c in (1, 5, 17):
        assert np.abs(G[c:, c:] - G[:-c, :-c]).max() < 1e-12


def test_rope_matches_complex_rotation_restatement():
    d = _rand_layer(1, 123, 2, 128, seed=31)
    for base in (10000.0, 1e6):
        qh, kh, _ = oracle.prologue(d, rope_base=base, qknorm=False)
        assert np.abs(qh - brute.rope_complex(d["q"].double().numpy(), base)).max() < 1e-12
        assert np.abs(kh - brute.rope_complex(d["k"].double().numpy(), base)).max() < 1e-12


# --------------------------------------------------------------------------------- RMS

def test_rms_unit_when_eps_zero_and_closed_form_otherwise():
    d = _rand_layer(1, 64, 2, 64, seed=41)
    qh, kh, _ = oracle.prologue(d, eps=0.0)
    for x in (qh, kh):
        assert np.abs(np.sqrt(np.mean(x * x, axis=-1)) - 1).max() < 1e-14
    small = dict(q=(d["q"].float() * 1e-3).to(torch.bfloat16), k=d["k"], v=d["v"])
    eps = 1e-6
    qh, _, _ = oracle.prologue(small, eps=eps)
    ms = np.mean(small["q"].double().numpy() ** 2, axis=-1)
    assert np.abs(np.sqrt(np.mean(qh * qh, axis=-1)) - np.sqrt(ms / (ms + eps))).max() < 1e-13


def test_norm_and_rope_commute():
    d = _rand_layer(1, 100, 2, 128, seed=51)
    both, _, _ = oracle.prologue(d)
    norm_only, _, _ = oracle.prologue(d, rope=False)
    assert np.abs(both - brute.rope_complex(norm_only, 10000.0)).max() < 1e-13


# ---------------------------------------------------------------------------- VE gate

def _ve_layer(seed=0, T=20, H=3, D=64):
    return _rand_layer(2, T, H, D, ve=True, seed=seed, vocab=50)


def test_gate_zero_weights_gives_v_plus_ve():
    d = _ve_layer(1)
    d["Wg"] = torch.zeros_like(d["Wg"])
    _, _, vp = oracle.prologue(d)
    B, T, H, D = d["q"].shape
    ve = d["table"][d["ids"]].view(B, T, H, D).double().numpy()
    assert np.abs(vp - (d["v"].double().numpy() + ve)).max() < 1e-14


def test_gate_zero_table_equals_no_ve_path():
    d = _ve_layer(2)
    d["table"] = torch.zeros_like(d["table"])
    o, l = oracle.forward(d, 7)
    o2, l2 = oracle.forward(dict(q=d["q"], k=d["k"], v=d["v"]), 7)
    assert np.array_equal(o, o2) and np.array_equal(l, l2)


def test_gate_is_two_sigmoid_per_head_in_open_interval():
    """The gate of head h equals 2*expit(x[..., :32] @ Wg[:, h]) (scipy's logistic) and lies in
    (0, 2); channels from 32 on do not matter."""
    d = _ve_layer(3, H=4)
    d["x"] = (d["x"].float() * 20).to(torch.bfloat16)     # push some gates near 0 and 2
    B, T, H, D = d["q"].shape
    _, _, vp = oracle.prologue(d)
    ve = d["table"][d["ids"]].view(B, T, H, D).double().numpy()
    g = (vp - d["v"].double().numpy()) / ve               # same ratio for every d of a head
    z = np.einsum("btc,ch->bth", d["x"][..., :32].double().numpy(), d["Wg"].double().numpy())
    assert np.abs(g - 2 * expit(z)[..., None]).max() < 1e-9
    assert (g > 0).all() and (g < 2).all()
    x2 = d["x"].clone()
    x2[..., 32:] = 0
    _, _, vp2 = oracle.prologue(dict(d, x=x2))
    assert np.array_equal(vp, vp2)


def test_gate_symmetry():
    """2 sigma(z) + 2 sigma(-z) = 2: flipping the sign of Wg flips z."""
    d = _ve_layer(4)
    _, _, vp = oracle.prologue(d)
    _, _, vm = oracle.prologue(dict(d, Wg=-d["Wg"]))
    B, T, H, D = d["q"].shape
    ve = d["table"][d["ids"]].view(B, T, H, D).double().numpy()
    v = d["v"].double().numpy()
    assert np.abs((vp - v) + (vm - v) - 2 * ve).max() < 1e-13


# ---------------------------------------------------------------- bf16 rounding (parity mode)

def test_round_bf16_ties_to_even_without_double_rounding():
    r = oracle.round_bf16
    assert r(1.0 + 2 ** -8) == 1.0                       # tie -> even (1.0)
    assert r(1.0 + 3 * 2 ** -8) == 1.0 + 2 ** -6         # tie -> even (mantissa 2)
    assert r(1.0 + 2 ** -8 + 2 ** -30) == 1.0 + 2 ** -7  # just above the tie: up
    assert r(-(1.0 + 2 ** -8 + 2 ** -30)) == -(1.0 + 2 ** -7)
    assert r(3.0) == 3.0 and r(0.0) == 0.0
    xs = np.random.default_rng(0).standard_normal(2000) * 10
    # fp32 inputs round once, so torch's float32 -> bfloat16 is the library reference here.
    xs32 = xs.astype(np.float32)
    ref = torch.from_numpy(xs32).to(torch.bfloat16).double().numpy()
    assert np.array_equal(np.array([r(float(x)) for x in xs32]), ref)


def test_parity_mode_is_within_tolerance_of_pure_mode():
    """Rounding the MMA operands to bf16 moves the result by much less than the parity bar
    (max-abs 2e-2, rel-L2 5e-3, LSE 1e-3) on the tiny workload."""
    s = workloads.TINY
    d = workloads.make_layer(s)
    o_p, l_p = oracle.forward(d, s.window, parity=True)
    o_f, l_f = oracle.forward(d, s.window, parity=False)
    assert np.abs(o_p - o_f).max() < 2e-2
    assert np.linalg.norm(o_p - o_f) / np.linalg.norm(o_f) < 5e-3
    assert np.abs(l_p - l_f).max() < 2e-2


def test_row_subset_equals_full_rows():
    s = workloads.LayerShape(B=2, T=300, H=3, D=64, window=100, ve=True, seed=9, vocab=64)
    d = workloads.make_layer(s)
    full, lfull = oracle.forward(d, s.window)
    rows = workloads.sample_rows(s, n_random=5, seed=1)
    o, l = oracle.forward(d, s.window, rows=rows)
    b = rows // (s.H * s.T)
    h = (rows // s.T) % s.H
    i = rows % s.T
    assert np.array_equal(o, full[b, i, h]) and np.array_equal(l, lfull[b, h, i])


# ---------------------------------------------------------------- grouped-query attention
# With Hkv key/value heads shared by groups of H / Hkv query heads, query head h reads key/value
# head h // (H / Hkv).  Repeating every key/value head (and its value-embedding table block and
# gate column) H / Hkv times gives a multi-head layer with the same arithmetic in the same order:
# the two must agree bit for bit.

def _repeat_kv(d, G):
    r = dict(d)
    r["k"] = d["k"].repeat_interleave(G, dim=2)
    r["v"] = d["v"].repeat_interleave(G, dim=2)
    if "table" in d:
        V, HkvD = d["table"].shape
        Hkv = d["Wg"].shape[1]
        D = HkvD // Hkv
        r["table"] = d["table"].view(V, Hkv, D).repeat_interleave(G, dim=1).reshape(V, Hkv * G * D).contiguous()
        r["Wg"] = d["Wg"].repeat_interleave(G, dim=1).contiguous()
    return r


@pytest.mark.parametrize("H,Hkv,window,ve", [(6, 2, 13, True), (4, 1, 0, False), (6, 3, 1, True)])
def test_gqa_equals_multihead_with_repeated_kv_heads(H, Hkv, window, ve):
    s = workloads.LayerShape(B=2, T=40, H=H, D=16, window=window, ve=ve, seed=31, kv_heads=Hkv, vocab=50,
                             model_dim=48)
    d = workloads.make_layer(s)
    assert d["k"].shape[2] == Hkv and d["q"].shape[2] == H
    o_g, l_g = oracle.forward(d, window, parity=True)
    o_m, l_m = oracle.forward(_repeat_kv(d, H // Hkv), window, parity=True)
    assert np.array_equal(o_g, o_m) and np.array_equal(l_g, l_m)
    qh, kh, vp = oracle.prologue(d, parity=True)
    qm, km, vm = oracle.prologue(_repeat_kv(d, H // Hkv), parity=True)
    assert kh.shape[2] == Hkv and np.array_equal(qh, qm)
    assert np.array_equal(kh, km[:, :, :: H // Hkv]) and np.array_equal(vp, vm[:, :, :: H // Hkv])


def test_gqa_rejects_heads_that_do_not_divide():
    s = workloads.LayerShape(B=1, T=8, H=6, D=16, window=0, ve=False, seed=1, kv_heads=4)
    with pytest.raises(ValueError):
        oracle.forward(workloads.make_layer(s), 0)
