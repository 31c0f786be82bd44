"""The benchmark's contract on the host (no GPU): the algorithmic byte counts
behind every roofline figure, written out term by term from what each step must
move, and the JSON line of the reference arm (the fp64 oracle on host cores)."""
import json
import os
import subprocess
import sys

import torch

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KIB = 1024


def test_prefill_bytes_per_token_head():
    # the method's bytes: q, k, v, g rows in bf16 (4 x 256 B), beta in bf16, o in
    # the input dtype (256 B); the library's fp32 o (512 B) is the labelled variant
    assert bench.BYTES_PER_TOKEN_HEAD == 4 * 256 + 2 + 256 == 1282
    assert bench.BYTES_PER_TOKEN_HEAD_O32 == 4 * 256 + 2 + 512
    assert bench.STATE_BYTES == 64 * KIB
    # the long-context workload: 65,536 tokens x 64 heads, initial and final
    # state per head
    assert 65536 * 64 * bench.BYTES_PER_TOKEN_HEAD + 64 * 2 * bench.STATE_BYTES == 5_385_486_336


def test_prefill_flop_per_token_head():
    # state products 6 K V plus intra-chunk products 7 C K (K = V = 128, C = 64)
    assert bench.FLOP_PER_TOKEN_HEAD == 6 * 128 * 128 + 7 * 64 * 128 == 155_648


class _Inp:
    def __init__(self, n, t, h):
        self.num_seqs, self.total_tokens, self.num_heads = n, t, h


def test_prefill_roofline_fractions():
    roof, tensor = bench.prefill_roofline(_Inp(1, 65536, 64), 6.0, 6500.0, 1600.0, "measured", None, "k")
    assert abs(roof["achieved"] - 5_385_486_336 / 6e-3 / 1e9) < 1e-6
    assert abs(roof["frac"] - roof["achieved"] / 6500.0) < 1e-12
    assert abs(tensor["peak"] - 800.0) < 1e-9
    assert abs(tensor["achieved"] - 65536 * 64 * 155_648 / 6e-3 / 1e12) < 1e-9
    assert roof["o_fp32_variant"]["algorithmic_bytes_per_launch"] == 65536 * 64 * 1538 + 64 * 2 * 65536


def test_gated_prefill_roofline_counts_the_gate():
    """With the fused output epilogue the gate z (256 B per token-head) is read
    and o is written in bf16, as the method's 1,282 B already count it."""
    roof, _ = bench.prefill_roofline(_Inp(1, 65536, 64), 6.0, 6500.0, 1600.0, "measured", None, "k", gated=True)
    assert roof["algorithmic_bytes_per_launch"] == 65536 * 64 * (1282 + 256) + 64 * 2 * 65536
    assert roof["o_fp32_variant"] is None


def test_decode_bytes_per_pair():
    rows_in = 4 * 256            # q, k, v, g of the token, bf16
    o_out = 512                  # fp32
    beta = 2
    cache = 2 * 9 * 256          # 3 tensors x 3 tokens, read and written
    assert bench.dec_bytes_per_pair(4) == 2 * 64 * KIB + rows_in + o_out + beta + cache == 137_218
    assert bench.dec_bytes_per_pair(2) == 2 * 32 * KIB + rows_in + o_out + beta + cache == 71_682


def test_mtp_bytes_per_pair():
    per_row = 2 * 3 * 512 + 4 * 256 + 2 + 512  # deltas written and read back, q k v g, beta, o
    cache = 3 * 9 * 256                         # read by verify and commit, written by commit
    assert bench.MTP_ROWS == 6
    assert bench.mtp_bytes_per_pair(4) == 3 * 64 * KIB + 6 * per_row + cache == 231_180
    assert bench.mtp_bytes_per_pair(2) == 3 * 32 * KIB + 6 * per_row + cache == 132_876


def _run(args, env_extra=None):
    env = dict(os.environ, **(env_extra or {}))
    return subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True, text=True,
                          timeout=600, env=env)


def test_reference_arm_json_line():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "0"], {"RANK": "0", "WORLD_SIZE": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    for key in ("metric", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config"):
        assert key in line, key
    assert line["value"] > 0 and line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["steps"] == 1 and line["warmup"] == 0 and line["n_gpus"] == 1
    assert line["vs_baseline"] is None and line["data"] == "synthetic"
    assert "workload" in line["config"]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_do_no_work():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "0"], {"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


class FakeNvml:
    """Stand-in for the NVML binding: a fixed sequence of SM clocks and one
    active clock-event reason (the power cap)."""
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonSwPowerCap = 0x4
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonHwThermalSlowdown = 0x40

    def __init__(self, clocks=(1965, 1900, 1965, 1950)):
        self.clocks, self.n, self.shut = clocks, 0, False

    def nvmlInit(self):
        pass

    def nvmlShutdown(self):
        self.shut = True

    def nvmlDeviceGetHandleByUUID(self, uuid):
        raise RuntimeError("no such device")

    def nvmlDeviceGetHandleByIndex(self, i):
        return ("gpu", i)

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        assert h == ("gpu", 0) and kind == self.NVML_CLOCK_SM
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        self.n += 1
        return self.clocks[(self.n - 1) % len(self.clocks)]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.nvmlClocksEventReasonSwPowerCap


def test_clock_sampler_polls_nvml_during_the_region():
    import time as _time
    fake = FakeNvml()
    with bench.ClockSampler(0, nvml=fake, period_s=0.002) as clk:
        _time.sleep(0.05)
    s = clk.summary()
    assert s["source"] == "nvml" and s["samples"] >= 5 and fake.shut
    assert s["sm_max_mhz"] == 1965 and 1900 <= s["sm_mhz"] <= 1965
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_sampler_falls_back_when_nvml_fails():
    class Broken(FakeNvml):
        def nvmlInit(self):
            raise RuntimeError("NVML library not found")

    with bench.ClockSampler(0, nvml=Broken()) as clk:
        pass
    s = clk.summary()
    assert s["source"] == "nvidia-smi"
    if s["samples"] == 0:  # no nvidia-smi on this host
        assert s["reasons"] == ["unavailable"]


def test_device_info_never_raises():
    """Without a GPU (or NVML) every field it cannot read stays None."""
    info = bench.device_info(0)
    assert set(info) == {"name", "driver", "cuda_runtime"}
    assert info["cuda_runtime"] == torch.version.cuda
