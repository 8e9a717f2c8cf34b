"""Host-side checks of the benchmark's work model and roofline arithmetic (no GPU).

Every roofline fraction that bench.py reports divides by the algorithmic bytes and
flops of `bench.step_work`, which is written from the layer shapes.  These tests tie
that model to the weight tensors the seeded generators actually allocate (a wrong
dimension or a missing matrix in the model fails them), and check the fraction
arithmetic on made-up timings.  The clock summary, which decides whether a timed run
saw a slowdown, is checked on made-up nvidia-smi lines.
"""
from dataclasses import replace

import numpy as np
import pytest

import bench
from hybrid_mamba_attention_b200 import inputs as I

# A small drafter with every part of the full one: M,A,M,A layers, a SwiGLU MLP after
# each mixer and the shared LM head.
SMALL = replace(I.LLAMA_FULL, name="small_full", d=128, Hq=4, Hkv=2, D=32, H=4, P=16, N=8, d_ff=256,
                vocab=1000)
PEAKS = {"hbm_gbs": 6452.8, "bf16_tflops": 1644.4, "bf16_tflops_sustained": 1395.6}

PER_TOKEN = ("W_in", "W_out", "W_qkv", "W_o", "W_gate", "W_up", "W_down")  # applied to every block token


def _launches(sh):
    """Launches of each kernel group in one draft step."""
    nM, nA, nL = sh.layers.count("M"), sh.layers.count("A"), len(sh.layers)
    return {"in_proj": nM, "inject": nM, "ssd_scan": nM, "out_proj": nM, "qkv_proj": nA, "attn_paged": nA,
            "o_proj": nA, "mlp_gate_up": nL, "mlp_down": nL, "lm_head_argmax": 1}


def _weights(sh):
    w = I.make_weights(sh, seed=7)
    per_token = sum(t.numel() for layer in w["layers"] for k, t in layer.items() if k in PER_TOKEN)
    per_token += w["W_lm"].numel()
    per_request = sum(layer["W_inj"].numel() for layer in w["layers"] if "W_inj" in layer)
    esize = w["W_lm"].element_size()
    return per_token, per_request, esize


def test_weight_bytes_equal_the_generated_weights():
    # with no requests only the weights are left to read, once per launch
    per_token, per_request, esize = _weights(SMALL)
    w = bench.step_work(SMALL, 0, 4, np.zeros(0, dtype=np.int64))
    total = sum(n * w[g]["bytes"] for g, n in _launches(SMALL).items())
    assert total == (per_token + per_request) * esize


@pytest.mark.parametrize("C,K", [(1, 1), (3, 4), (16, 16)])
def test_gemm_flops_equal_two_per_weight_and_row(C, K):
    # every block token meets every per-token matrix once; the injection runs once per request
    per_token, per_request, _ = _weights(SMALL)
    ctx = np.full(C, 37, dtype=np.int64)
    w = bench.step_work(SMALL, C, K, ctx)
    gemms = {g: n for g, n in _launches(SMALL).items() if g not in ("attn_paged", "ssd_scan")}
    flops = sum(n * w[g]["flops"] for g, n in gemms.items())
    assert flops == 2.0 * (C * K * per_token + C * per_request)


def test_attention_bytes_grow_with_the_context_read():
    # one more context token of one request adds its K and V rows of every kv head
    sh = SMALL
    ctx = np.array([100, 250], dtype=np.int64)
    a = bench.step_work(sh, 2, 4, ctx)["attn_paged"]["bytes"]
    b = bench.step_work(sh, 2, 4, ctx + np.array([1, 0]))["attn_paged"]["bytes"]
    assert b - a == 2 * sh.Hkv * sh.D * 2  # K and V, bf16


def test_roofline_fraction_is_achieved_over_the_peak():
    # HBM-bound: the peak's bytes in twice the time is half the peak
    r = bench.roofline_of("mlp_down", {"bytes": 6452.8e9, "flops": 1.0}, 2000.0, PEAKS)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(3226.4) and r["frac"] == pytest.approx(0.5)
    # tensor-bound: a millisecond of sustained-peak flops in a millisecond is 1.0
    fl = 1395.6e12 * 1e-3
    r = bench.roofline_of("mlp_gate_up", {"bytes": 1.0, "flops": fl}, 1.0, PEAKS)
    assert r["bound"] == "tensor" and r["frac"] == pytest.approx(1.0)
    # a kernel timed alone is held to the burst peak instead
    r = bench.roofline_of("mlp_gate_up", {"bytes": 1.0, "flops": fl}, 1.0, PEAKS, sustained=False)
    assert r["peak"] == 1644.4 and r["frac"] == pytest.approx(1395.6 / 1644.4, abs=1e-4)
    # the attention and the scan are reported against HBM even where their flops would dominate
    r = bench.roofline_of("attn_paged", {"bytes": 1.0, "flops": fl}, 1.0, PEAKS, traffic=123)
    assert r["bound"] == "hbm" and r["traffic"] == 123


def test_step_roofline_never_shrinks_with_more_work():
    prev = 0.0
    for C in (1, 2, 8, 32):
        t = bench.step_roofline_ms(SMALL, C, 16, np.full(C, 512, dtype=np.int64), PEAKS)
        assert t >= prev
        prev = t
    short = bench.step_roofline_ms(SMALL, 4, 16, np.full(4, 512, dtype=np.int64), PEAKS)
    long = bench.step_roofline_ms(SMALL, 4, 16, np.full(4, 4096, dtype=np.int64), PEAKS)
    assert long > short


class _Done:
    """Stands in for the finished nvidia-smi process and its reader thread."""

    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0

    def kill(self):
        pass

    def join(self, timeout=None):
        pass


def _smi(sm, smax, power_cap="Not Active", hw="Not Active"):
    # the FIELDS order: index, clocks.sm, clocks.max.sm, power.draw, active mask, hw_slowdown,
    # hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
    return f"0, {sm}, {smax}, 950.1, 0x0000000000000004, {hw}, Not Active, Not Active, {power_cap}"


def test_clock_summary_keeps_the_timed_region_only():
    cs = bench.ClockSampler(0)
    cs.proc, cs.thread = _Done(), _Done()
    cs.lines = [(0.0, _smi(1965, 1965)),                       # before the region: not counted
                (1.0, _smi(1500, 1965, power_cap="Active")),
                (1.1, _smi(1520, 1965, power_cap="Active")),
                (1.2, _smi(1540, 1965)),
                (1.3, "garbled line"),                          # skipped
                (9.0, _smi(900, 1965, hw="Active"))]            # after the region: not counted
    cs.window(0.95, 1.25)
    r = cs.stop()
    assert r["sm_mhz"] == 1520 and r["sm_max_mhz"] == 1965 and r["samples"] == 3
    assert r["reasons"] == ["sw_power_cap"] and r["in_timed_region"] is True


def test_clock_summary_reports_a_slowdown_inside_the_region():
    cs = bench.ClockSampler(0)
    cs.proc, cs.thread = _Done(), _Done()
    cs.lines = [(1.0, _smi(1200, 1965, hw="Active")), (1.1, _smi(1250, 1965))]
    cs.window(0.9, 1.2)
    assert bench.ClockSampler.stop(cs)["reasons"] == ["hw_slowdown"]


def test_clock_summary_without_nvidia_smi_says_so():
    assert bench.ClockSampler(0).stop()["reasons"] == ["unavailable"]


def test_reference_line_carries_this_arms_config_and_metric(monkeypatch, capsys):
    # the reference arm (the CPU oracle) reports on the same config, metric and unit as the
    # CUDA arm; its end-to-end figure is its own value with no host-device copies
    import json
    monkeypatch.setattr(I, "make_step_inputs", lambda wl, dev: {})
    monkeypatch.setattr(bench, "oracle_one_request", lambda I_, wl, r, request=0: (2.0, 1000, 8))

    class Args:
        steps, warmup, C, K, draft_vocab = 2, 3, 128, 16, 0

    bench.run_reference(Args(), rank=0, world=1)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["config"] == bench.step_config(I.full_workload(128, 16), 1)
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT and line["higher_is_better"] is True
    assert line["value"] == pytest.approx(16 / 2.0)
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_attention_configs_warms_up_then_times_a_bounded_number_of_calls(monkeypatch):
    # The standalone attention timing runs the call alone for warm_s seconds, then times
    # a number of calls that spans about timed_s seconds (at least 20, at most 2000),
    # and reports the call time from the CUDA events over exactly those calls.  The
    # library, the inputs and the CUDA events are stand-ins on the CPU here; every call
    # "takes" 0.5 ms of host time.
    import time
    import torch

    calls = []

    class FakeH:
        @staticmethod
        def make_cfg(sh):
            return sh

        @staticmethod
        def kv_view(inp):
            return type("KV", (), {"max_pages": 4})()

        @staticmethod
        def hspec_attn_workspace_size(cfg, C, K, max_pages):
            return 256

        @staticmethod
        def alloc_workspace(n, dev):
            return torch.empty(n, dtype=torch.uint8)

        @staticmethod
        def hspec_attn_paged_block(*args):
            calls.append(time.monotonic())
            time.sleep(0.0005)

        @staticmethod
        def hspec_sync_status():
            return 0

    class FakeEvent:
        def __init__(self, enable_timing=False):
            self.n = None

        def record(self, stream=None):
            self.n = len(calls)

        def elapsed_time(self, other):
            return 0.5 * (other.n - self.n)  # ms: 0.5 ms per call between the events

    def fake_inputs(sh, wl, K, seed, dev, shuffle=True, slack=0.1):
        return {"q": torch.zeros(wl.C, K, sh.Hq, sh.D), "ctx_lens": torch.full((wl.C,), 100, dtype=torch.int32),
                "k_blk": None, "v_blk": None}

    monkeypatch.setattr(torch.cuda, "Event", FakeEvent)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "empty_cache", lambda *a, **k: None)
    monkeypatch.setattr(I, "make_attn_inputs", fake_inputs)
    monkeypatch.setattr(bench.ClockSampler, "start", lambda self: None)  # no nvidia-smi here

    out = bench.attention_configs(FakeH, I, "cpu", PEAKS, warm_s=0.05, timed_s=0.02)
    assert set(out) == {"llama_c32", "qwen_c128"}
    for name, r in out.items():
        assert 20 <= r["calls"] <= 2000
        assert r["us_per_call"] == pytest.approx(500.0)
        assert r["clocks"]["reasons"] == ["unavailable"]
    # each workload: 3 untimed calls, at least warm_s of warm-up calls, then the timed calls
    assert len(calls) >= 2 * (3 + 20 + 8)
