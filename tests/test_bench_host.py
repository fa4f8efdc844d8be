"""Host-side checks of bench.py's arithmetic (no GPU): the algorithmic flop count of each workload
(4 D flops per unmasked query-key pair, W (W + 1) / 2 + (T - W) W pairs per (b, h)) against the
GFLOP each layer shape gives by hand, the 24-layer S,S,S,L stack totals, and the L2 note of each
workload."""
import pytest

import bench
import workloads


@pytest.mark.parametrize("s,gflop", [
    (workloads.TINY, 0.034),
    (workloads.GPT2, 12.90),
    (workloads.D24_S, 154.67),
    (workloads.D24_L_VE, 206.26),
], ids=["tiny", "gpt2_124m", "d24_S", "d24_L_VE"])
def test_flops_match_the_hand_counts(s, gflop):
    got = bench.flops_per_step(s) / 1e9
    assert abs(got - gflop) <= 0.006 * gflop + 1e-3, (s.name, got, gflop)


def test_unmasked_pairs_closed_form_and_brute_force():
    # brute force over a small (b, h) slice: pairs (i, j) with 0 <= i - j < W
    for T, W in ((7, 3), (16, 16), (130, 40), (257, 1)):
        s = workloads.LayerShape(B=2, T=T, H=3, D=64, window=W, ve=False, seed=0, name="x")
        brute = sum(1 for i in range(T) for j in range(T) if 0 <= i - j < min(W, T))
        assert s.unmasked_pairs() == 2 * 3 * brute


@pytest.mark.parametrize("T,tflop", [(1024, 2.01), (2048, 4.02), (4096, 8.04), (8192, 16.08), (16384, 32.16)])
def test_sssl_stack_flops_match_the_hand_counts(T, tflop):
    shapes = workloads.sssl_layer_shapes(32768 // T, T, 12, 128)
    assert len(shapes) == 24
    got = sum(bench.flops_per_step(s) for s in shapes) / 1e12
    assert abs(got - tflop) <= 0.006 * tflop, (T, got, tflop)


def test_l2_note_follows_the_input_size():
    # d24 inputs (q, k, v, ve: 403 MB) exceed the 126 MB L2, the GPT-2 124M layer's (38 MB) do not
    assert bench.input_bytes(workloads.D24_L_VE) > bench.L2_BYTES
    assert bench.config_of(workloads.D24_L_VE, 1)["l2"].startswith("no flush")
    assert bench.input_bytes(workloads.GPT2) < bench.L2_BYTES
    assert "flushed between steps" in bench.config_of(workloads.GPT2, 1)["l2"]


def _fake_nvml(clocks, reasons_attr, bits):
    import itertools
    import types
    seq = itertools.cycle(clocks)
    nv = types.SimpleNamespace(NVML_CLOCK_SM=1, nvmlInit=lambda: None,
                               nvmlDeviceGetHandleByIndex=lambda i: ("gpu", i),
                               nvmlDeviceGetMaxClockInfo=lambda h, c: 1965,
                               nvmlDeviceGetClockInfo=lambda h, c: next(seq))
    setattr(nv, reasons_attr, lambda h: bits)
    return nv


@pytest.mark.parametrize("reasons_attr", ["nvmlDeviceGetCurrentClocksEventReasons",
                                          "nvmlDeviceGetCurrentClocksThrottleReasons"])
def test_clock_sampler_reads_clocks_and_reasons(monkeypatch, reasons_attr):
    # NVML faked on the host: clocks cycle 1965 / 1965 / 1800 MHz, reasons gpu_idle + sw_power_cap
    # + hw_slowdown; gpu_idle is not a throttle and is dropped, the rest are named.
    import sys
    import time
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1965, 1965, 1800], reasons_attr, 0x1 | 0x4 | 0x8))
    s = bench.ClockSampler(0, period_s=0.001).start()
    assert s.ok
    time.sleep(0.05)
    r = s.stop()
    assert r["sm_max_mhz"] == 1965 and r["samples"] >= 3
    assert r["sm_mhz"] == 1965                      # the median of a 2:1 mix
    assert r["reasons"] == ["hw_slowdown", "sw_power_cap"]


def test_clock_sampler_without_nvml(monkeypatch):
    import sys
    import types

    def fail():
        raise RuntimeError("no NVML")
    monkeypatch.setitem(sys.modules, "pynvml", types.SimpleNamespace(nvmlInit=fail))
    s = bench.ClockSampler(0).start()
    assert not s.ok
    assert s.stop() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_recorded_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    # the committed ncu traffic is reported only for the kernel source it was captured on
    import json
    f = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.recorded_traffic("d24_L_VE") is None                      # no file
    f.write_text(json.dumps({"d24_L_VE": {"kernel_sha256": bench.kernel_hash(), "dram_bytes_per_launch": 123}}))
    assert bench.recorded_traffic("d24_L_VE") == 123
    assert bench.recorded_traffic("gpt2_124m") is None                     # another workload
    f.write_text(json.dumps({"d24_L_VE": {"kernel_sha256": "0" * 64, "dram_bytes_per_launch": 123}}))
    assert bench.recorded_traffic("d24_L_VE") is None                      # the kernel changed since


def _bench(*argv, env=None):
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    e = dict(os.environ)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(root, "bench.py"), *argv], cwd=root, env=e,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_line():
    # The reference arm is the oracle on the host cores, so it runs here: one JSON line with the
    # GPU arm's metric, unit and workload, impl "reference", its CPU sample, and an e2e entry
    # without device copies.
    import json
    r = _bench("--impl", "reference", "--steps", "1", "--warmup", "3")
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["higher_is_better"] is True
    assert line["metric"].startswith("attention fwd TFLOP/s") and line["n_gpus"] == 1
    assert line["config"]["workload"] == "d24 L+VE (16,2048,12,128) W=2048"
    assert line["steps"] == 1 and line["warmup"] == 3 and line["value"] > 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    r = _bench("--impl", "reference", "--steps", "1", "--warmup", "3", "--gpus", "2",
               env=dict(RANK="1", WORLD_SIZE="2", LOCAL_RANK="1"))
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_bench_refuses_short_warmup():
    r = _bench("--steps", "1", "--warmup", "2")
    assert r.returncode != 0 and "--warmup must be >= 3" in r.stderr


def test_gpu_arm_without_a_device_fails_loudly():
    # no CPU path: without CUDA the product arm exits non-zero and prints no result line
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is visible")
    r = _bench("--steps", "1", "--warmup", "3")
    assert r.returncode != 0 and "{" not in r.stdout and "needs a CUDA device" in r.stderr


def test_input_bytes_and_config_by_hand():
    # d24 L+VE reads q, k, v and ve: 4 x 16 x 2048 x 12 x 128 bf16 = 402.65 MB; GPT-2 124M reads
    # q, k, v: 3 x 8 x 1024 x 12 x 64 bf16 = 37.7 MB
    assert bench.input_bytes(workloads.D24_L_VE) == 4 * 16 * 2048 * 12 * 128 * 2
    assert bench.input_bytes(workloads.GPT2) == 3 * 8 * 1024 * 12 * 64 * 2
    c = bench.config_of(workloads.D24_L_VE, 1)
    assert (c["B_per_gpu"], c["T"], c["H"], c["D"], c["window"], c["value_embeddings"]) == (16, 2048, 12, 128, 2048, True)
    assert c["workload"] == "d24 L+VE (16,2048,12,128) W=2048" and c["global_batch"] == 16
    assert "403 MB" in c["l2"]
    assert bench.config_of(workloads.D24_L_VE, 4)["global_batch"] == 64     # weak scaling: B per GPU fixed


def test_sssl_stack_recipe():
    # S,S,S,L windows (S = T/2), value embeddings on even layers, and every layer drawn in turn
    # from one generator: no two layers share inputs, so L2 cannot serve a later layer's data
    shapes = workloads.sssl_layer_shapes(2, 64, 2, 64, n_layers=8)
    assert [s.window for s in shapes] == [32, 32, 32, 64] * 2
    assert [s.ve for s in shapes] == [True, False] * 4
    stack = workloads.sssl_stack(2, 64, 2, 64, n_layers=8)
    hashes = [workloads.sha256_of(d) for _, d in stack]
    assert len(set(hashes)) == 8
    again = [workloads.sha256_of(d) for _, d in workloads.sssl_stack(2, 64, 2, 64, n_layers=8)]
    assert hashes == again                                       # seeded: the same stack every run
