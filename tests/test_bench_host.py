"""Host logic of bench.py that needs no GPU: the clock sampler's parsing and
time window, and the rule that rejects a timing taken under throttling."""
import datetime
import os
import sys
import tempfile

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


class _Proc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        pass


def _sampler_with(rows, now):
    """A ClockSampler whose nvidia-smi output is the given (sm_mhz, power_cap) rows,
    one per second from `now`."""
    c = bench.ClockSampler(0)
    fd, c.path = tempfile.mkstemp(suffix=".csv")
    os.close(fd)
    with open(c.path, "w") as f:
        for i, (mhz, cap, hw) in enumerate(rows):
            ts = (now + datetime.timedelta(seconds=i)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
            f.write(f"{ts}, 0, {mhz}, 1965, 900.00, 0x4, {hw}, Not Active, Not Active, {cap}\n")
    c.proc = _Proc()
    c.out = open(os.devnull, "w")
    return c


def test_clock_samples_outside_the_timed_window_are_dropped():
    now = datetime.datetime.now()
    rows = [(1965, "Not Active", "Not Active"), (1400, "Active", "Not Active"),
            (1300, "Active", "Not Active"), (1965, "Not Active", "Not Active")]
    c = _sampler_with(rows, now)
    clk = c.stop(now + datetime.timedelta(seconds=0.5), now + datetime.timedelta(seconds=2.5))
    assert {k: clk[k] for k in ("sm_mhz", "sm_max_mhz", "reasons", "samples")} == {
        "sm_mhz": 1350.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 2}
    assert clk["source"] == "nvidia-smi inside the timed region"


def test_nvml_samples_inside_the_window_take_precedence():
    now = datetime.datetime.now()
    c = _sampler_with([(1965, "Not Active", "Not Active")], now)
    ms = datetime.timedelta(milliseconds=1)
    # NVML polls: two inside [now+10ms, now+20ms] (one with the power-cap bit),
    # one before it with a hardware-slowdown bit that must not count
    c.polls = [(now + 5 * ms, 1900.0, 0x8), (now + 12 * ms, 1500.0, 0x4),
               (now + 15 * ms, 1450.0, 0x0)]
    c.nvml_max = 1965.0
    clk = c.stop(now + 10 * ms, now + 20 * ms)
    assert clk["sm_mhz"] == 1475.0 and clk["sm_min_mhz"] == 1450.0
    assert clk["reasons"] == ["sw_power_cap"] and clk["samples"] == 2
    assert clk["smi_samples_inside"] == 0 and clk["source"].startswith("NVML")


def test_clock_window_with_no_samples_keeps_them_all():
    now = datetime.datetime.now()
    c = _sampler_with([(1800, "Not Active", "Not Active"), (1700, "Not Active", "Active")], now)
    far = now + datetime.timedelta(hours=1)
    clk = c.stop(far, far + datetime.timedelta(seconds=1))
    assert clk["samples"] == 2 and clk["reasons"] == ["hw_slowdown"]


def test_throttled_or_locked_clocks_are_rejected():
    assert not bench.clocks_rejected(None)
    assert not bench.clocks_rejected({"reasons": ["sw_power_cap"], "sm_mhz": 1300,
                                      "sm_max_mhz": 1965})
    for r in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"):
        assert bench.clocks_rejected({"reasons": [r], "sm_mhz": 1900, "sm_max_mhz": 1965})
    # far below max with no reason: a clock lock left by someone else
    assert bench.clocks_rejected({"reasons": [], "sm_mhz": 900, "sm_max_mhz": 1965})
    assert not bench.clocks_rejected({"reasons": [], "sm_mhz": 1900, "sm_max_mhz": 1965})


def test_gemm_peak_follows_the_clock_regime():
    pk = {"bf16_tflops": 1659.1, "bf16_tflops_sustained": 1400.6}
    capped = {"reasons": ["sw_power_cap"], "sm_mhz": 1383, "sm_max_mhz": 1965}
    full = {"reasons": [], "sm_mhz": 1965, "sm_max_mhz": 1965}
    assert bench.tensor_peak(pk, "measured", capped)[0] == 1400.6
    assert "sustained" in bench.tensor_peak(pk, "measured", capped)[1]
    assert bench.tensor_peak(pk, "measured", full) == (1659.1, "measured bf16 burst")
    assert bench.tensor_peak(pk, "fallback", None) == (1659.1, "fallback bf16 burst")


def test_reference_arm_runs_the_oracle_alone():
    """``--impl reference`` builds its sample on the host and runs only the
    oracle: the library is never imported, CUDA never initialised, and its
    ``config`` is the one the library's line prints for the same workload."""
    import json
    import subprocess
    code = (
        "import sys, runpy, json\n"
        "sys.argv = ['bench.py', '--impl', 'reference', '--workload', 'qkv',\n"
        "            '--steps', '1', '--warmup', '1']\n"
        "runpy.run_path('bench.py', run_name='__main__')\n"
        "import torch\n"
        "mods = [m for m in sys.modules if m.startswith('tensor_transformer_linear_b200')]\n"
        "print(json.dumps({'mods': mods, 'cuda': torch.cuda.is_initialized()}))\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    line, probe = lines[0], lines[-1]
    assert probe == {"mods": [], "cuda": False}
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["config"] == bench.workload_config("qkv", 1)
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
