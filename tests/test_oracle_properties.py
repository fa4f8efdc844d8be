"""Randomized pins of the oracle (hypothesis): random small shapes, windows, window conventions and
value-embedding settings against the independent NumPy brute force (forward) and against torch
autograd through an independent fp64 forward (backward).  CPU only.
"""
import numpy as np
import torch
from hypothesis import given, settings, strategies as st

import oracle
import oracle.brute as brute
import tests.test_oracle_backward_pins as bp
import workloads


@settings(max_examples=40, deadline=None)
@given(B=st.integers(1, 2), T=st.integers(1, 40), H=st.integers(1, 3), D=st.sampled_from([2, 4, 8, 16]),
       window=st.integers(0, 45), ve=st.booleans(), convention=st.integers(0, 1), seed=st.integers(0, 10 ** 6))
def test_forward_matches_bruteforce_on_random_shapes(B, T, H, D, window, ve, convention, seed):
    s = workloads.LayerShape(B=B, T=T, H=H, D=D, window=window, ve=ve, seed=seed, vocab=17,
                             model_dim=max(32, H * D))
    d = workloads.make_layer(s)
    o, l = oracle.forward(d, window, parity=False, window_convention=convention)
    ob, lb = brute.forward(d, window, convention=convention)
    assert np.abs(o - ob).max() < 1e-12 and np.abs(l - lb).max() < 1e-12


@settings(max_examples=25, deadline=None)
@given(T=st.integers(1, 24), Hkv=st.integers(1, 2), G=st.integers(1, 3), D=st.sampled_from([4, 8]),
       window=st.integers(0, 26), ve=st.booleans(), with_lse=st.booleans(), seed=st.integers(0, 10 ** 6))
def test_backward_matches_autograd_on_random_shapes(T, Hkv, G, D, window, ve, with_lse, seed):
    H = Hkv * G
    d = bp._draw(1, T, H, D, Hkv=Hkv, ve=ve, seed=seed, unique_ids=False)
    g = torch.Generator().manual_seed(seed + 1)
    dout = torch.randn((1, T, H, D), generator=g, dtype=torch.float64).numpy()
    dlse = torch.randn((1, H, T), generator=g, dtype=torch.float64).numpy() if with_lse else None
    got = oracle.backward(d, dout, window, dlse=dlse)
    ref = bp._autograd_gradients(d, window, dout, dlse, 1e-6)
    for key in ref:
        scale = max(np.abs(ref[key]).max(), 1e-30)
        assert np.abs(got[key] - ref[key]).max() <= 1e-9 * scale + 1e-12, key
