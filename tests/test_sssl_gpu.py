"""GPU parity on the SSSL stack: 24 consecutive attention layers with windows S,S,S,L
(S = T/2, L = T) and value embeddings on even layers, at (B, T) = (32, 1024), (16, 2048),
(8, 4096), (4, 8192), (2, 16384) -- the d24 model's layer pattern (intelliparadigm "GPT-2 for
$73", section 3.2) swept in length.  Every layer runs through the C ABI at full size; its output
is checked against the fp64 oracle on sampled rows (edge rows 0, 1, W-1, W, W+1, 127, 128, T-1
and seeded random rows) of a few (b, h) slices, in parity mode and in pure fp64 mode, and for
finiteness everywhere."""
import pytest
import torch

import workloads
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield


@pytest.mark.parametrize("B,T", workloads.SSSL_POINTS, ids=[f"B{b}_T{t}" for b, t in workloads.SSSL_POINTS])
def test_sssl_stack(B, T):
    worst = dict(max_abs=0.0, rel_l2=0.0, lse_max_abs=0.0)
    worst_pure = dict(worst)
    for layer, (s, d) in enumerate(workloads.sssl_stack(B, T)):
        dev = parity.to_device(d)
        out, lse = parity.run_gpu(s, dev)
        pairs = [(layer % B, (5 * layer) % s.H), ((layer + 1) % B, (5 * layer + 7) % s.H)]
        rows = workloads.sample_rows(s, n_random=4, seed=100 + layer, bh_pairs=pairs)
        err = parity.check_rows(s, d, out, lse, rows)
        pure = parity.check_rows(s, d, out, lse, rows, pure=True)
        for key in worst:
            worst[key] = max(worst[key], err[key])
            worst_pure[key] = max(worst_pure[key], pure[key])
        del dev, out, lse
    print(f"SSSL B={B} T={T}: worst over 24 layers {worst}; against pure fp64 {worst_pure}")
