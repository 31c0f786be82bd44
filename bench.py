#!/usr/bin/env python
"""Benchmark of the KDA sequence-mixing hot path on B200.

One step = one kda_prefill over the long-context workload (1 sequence x
T = 65,536 tokens, 64 heads x 128, bf16 inputs, fp32 state, gates near the -5
floor on 10 % of channels).  `value` is prefill tokens/s over the whole job
(all ranks), timed on the device with CUDA events, inputs resident in HBM.
The same line carries the decode-step state bandwidth (256 sequences x 64
heads, 1 GiB of fp32 state read and written in place) with its own roofline,
the multi-token decode legs (verify + commit of 6 rows, and the fused
commit + verify), the same decode legs with bf16 state storage, the
end-to-end number through the C ABI with host buffers, the oracle's CPU
throughput, and the SM clocks sampled during the timed region.

Multi-GPU: one process per GPU (torchrun); every rank runs its own
independent sequence (the path shards by sequence/head with no exchange), so
scaling is weak; time = max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import kda_inputs as ki  # noqa: E402

METRIC = "KDA prefill tokens/s (64 heads, T=64k) and decode state GB/s vs HBM peak"
WORKLOAD = "kda_prefill long-context: 1 x T=65536, 64 heads x 128, bf16 in / fp32 state / fp32 out, chunk 64"
H, D, T_LONG = 64, 128, 65536
# Algorithmic bytes of a prefill (what the method must move, bf16 workloads):
# per token-head q, k, v, g (4 x 256 B) + beta (2 B) + o (256 B in the input
# dtype) = 1,282 B, plus per (sequence, head) the initial and the final state
# (2 x 64 KiB fp32).  The library writes o in fp32 (512 B per token-head);
# that variant is reported beside it, labelled.
BYTES_PER_TOKEN_HEAD = 4 * D * 2 + 2 + D * 2
BYTES_PER_TOKEN_HEAD_O32 = 4 * D * 2 + 2 + D * 4
STATE_BYTES = D * D * 4
GATE_BYTES_PER_TOKEN_HEAD = D * 2  # the output epilogue's gate z (bf16)
# Useful tensor work of the chunked prefill per token-head: the state products
# (6 K V) and the intra-chunk products (7 C K), C = 64.
FLOP_PER_TOKEN_HEAD = 6 * D * D + 7 * 64 * D
# Every contraction runs as tcgen05 kind::tf32, whose nominal dense rate is
# half the bf16 rate (1.1 of 2.25 PFLOP/s): the tf32 peak is bf16_tflops / 2.
TF32_PER_BF16 = 0.5


# decode: per (sequence, head) the state read + written (4 or 2 bytes per element), q/k/v/g
# in, o out (fp32), beta, the conv cache (3 tokens x q/k/v read, 3 written)
def dec_bytes_per_pair(state_elem_bytes: int) -> int:
    return 2 * D * D * state_elem_bytes + 4 * D * 2 + D * 4 + 2 + 2 * 9 * D * 2


# kernels launched per call: kda_prefill bf16 = chunk_prep + chunk_scan + conv tail
PREFILL_LAUNCHES = 3
DECODE_LAUNCHES = 1
# multi-token decode (verify R rows, commit the kept prefix), per (sequence, head):
# state read by verify, read and written by commit; per row the deltas
# (k_hat, u, alpha fp32) written and read back, q k v g read, beta, o fp32;
# the conv cache read by both calls and written by commit
MTP_ROWS = 6


def mtp_bytes_per_pair(state_elem_bytes: int) -> int:
    return (3 * D * D * state_elem_bytes + MTP_ROWS * (2 * 3 * D * 4 + 4 * D * 2 + 2 + D * 4)
            + 3 * 9 * D * 2)


MTP_LAUNCHES = 2


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    d = os.path.join(ROOT, "linear_attention_sequence_kda_b200", "csrc")
    for f in sorted(os.listdir(d)):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """dram bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if not rec or rec.get("source_hash") != kernel_source_hash():
        return None
    return rec.get("bytes_per_launch")


class ClockSampler:
    """SM clock and clock-event (throttle) reasons of one GPU, sampled while a
    timed region runs: NVML polled every `period_s` from a background thread
    (reads only), or, where NVML cannot be used, nvidia-smi's 200 ms loop.
    `nvml` may be given a stand-in module (tests)."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, nvml=None, period_s: float = 0.01):
        self.idx = device_index
        self.nvml = nvml
        self.period = period_s
        self.rows = []      # (sm MHz, max sm MHz, [active reasons])
        self.proc = None
        self.thread = None
        self.out = ""
        self.source = None

    def _start_nvml(self):
        nv = self.nvml
        if nv is None:
            import pynvml as nv
        nv.nvmlInit()
        self.nvml = nv
        try:  # the CUDA device's own GPU, whatever devices this process sees
            h = nv.nvmlDeviceGetHandleByUUID("GPU-" + str(torch.cuda.get_device_properties(self.idx).uuid))
        except Exception:
            h = nv.nvmlDeviceGetHandleByIndex(self.idx)
        max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        read_mask = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        bits = [(name, getattr(nv, attr)) for name, attr in self.REASONS]

        def sample():
            mhz, mask = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)), int(read_mask(h))
            self.rows.append((mhz, max_mhz, [name for name, b in bits if mask & b]))

        sample()  # a first read here, so that an NVML that cannot sample falls back now
        self._stop = threading.Event()

        def run():
            while not self._stop.wait(self.period):
                try:
                    sample()
                except Exception:
                    return

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()
        self.source = "nvml"

    def __enter__(self):
        try:
            self._start_nvml()
            return self
        except Exception:
            self.thread = None
            self.rows = []
        self.source = "nvidia-smi"
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=2)
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass
            return
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()
        names = [name for name, _ in self.REASONS]
        for line in (self.out or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                self.rows.append((float(parts[1]), float(parts[2]),
                                  [names[i] for i, x in enumerate(parts[5:9]) if x.lower() == "active"]))
            except ValueError:
                continue

    def summary(self):
        rows = list(self.rows)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0,
                    "source": self.source}
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted({n for r in rows for n in r[2]}), "samples": len(rows),
                "source": self.source}


def device_info(dev_index: int) -> dict:
    """The GPU's name, its driver version and the CUDA runtime in use (reads
    only; a field that cannot be read stays None)."""
    info = {"name": None, "driver": None, "cuda_runtime": torch.version.cuda}
    try:
        info["name"] = torch.cuda.get_device_name(dev_index)
    except Exception:
        pass
    try:
        import pynvml
        pynvml.nvmlInit()
        try:
            v = pynvml.nvmlSystemGetDriverVersion()
            info["driver"] = v.decode() if isinstance(v, bytes) else str(v)
        finally:
            pynvml.nvmlShutdown()
    except Exception:
        pass
    return info


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    from linear_attention_sequence_kda_b200.sharding import max_over_ranks as _max
    return x if world == 1 else _max(x, device="cuda")


def timed(fn, steps, warmup, world, stream):
    """W untimed steps, then K steps bracketed by barrier + synchronize, with
    a CUDA event pair per step on the launching stream.  Returns (total ms,
    per-step ms list), the total being the max over ranks."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(steps):
        evs[i][0].record(stream)
        fn()
        evs[i][1].record(stream)
    stop.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    total = max_over_ranks(start.elapsed_time(stop), world)
    return total, [a.elapsed_time(b) for a, b in evs]


def cpu_baseline(tokens: int = 8192):
    """The fp64 oracle as it stands on this host's cores: all 64 heads of the
    long-context workload over its first `tokens` tokens."""
    import oracle  # test infrastructure; only this leg of the benchmark runs it
    inp = ki.make_prefill([tokens], H, torch.bfloat16, ki.BASE_SEED + 2, gate="bimodal")
    probs = [oracle.prefill_problem(inp, 0, h) for h in range(H)]
    cores = os.cpu_count() or 1
    t0 = time.perf_counter()
    used = oracle.run_problems(probs, cores)
    dt = time.perf_counter() - t0
    return {"value": tokens / dt, "unit": "tokens/s", "cores": used, "kind": "oracle",
            "sample": f"first {tokens} tokens x all {H} heads of the T=65536 workload (fp64 C recurrence, "
                      f"{used} threads, {dt:.2f} s wall)"}


def run_reference(args, world, rank):
    """The reference arm: the fp64 oracle (the pages give no implementation to
    run) on this host's cores, each step one bounded sample of the same
    workload (first 1024 tokens x all 64 heads), inputs generated once."""
    if rank != 0:
        return
    import oracle  # test infrastructure; the reference arm is the one other user
    tokens = 1024
    inp = ki.make_prefill([tokens], H, torch.bfloat16, ki.BASE_SEED + 2, gate="bimodal")
    cores = os.cpu_count() or 1
    used = cores

    def one_step():
        nonlocal used
        probs = [oracle.prefill_problem(inp, 0, h) for h in range(H)]
        t0 = time.perf_counter()
        used = oracle.run_problems(probs, cores)
        return time.perf_counter() - t0

    for _ in range(args.warmup):
        one_step()
    times = [one_step() for _ in range(args.steps)]
    total = sum(times)
    value = args.steps * tokens / total
    sample = (f"first {tokens} tokens x all {H} heads of the T=65536 workload per step "
              f"(fp64 C recurrence, {used} threads)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "heads": H, "seq_len": T_LONG, "batch": 1,
                       "sample_tokens_per_step": tokens},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": used, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=16,
                    help="timed steps of the pipelined end-to-end loop (its fill and drain are spread over them); 0 skips it")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-prefill", action="store_true",
                    help="skip the 4 x 4096 and varlen prefill legs")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode leg")
    ap.add_argument("--heads", type=int, default=H,
                    help="reduced head count (profiling only; the reported workload uses 64)")
    ap.add_argument("--seq-len", type=int, default=T_LONG,
                    help="reduced length (profiling only; the reported workload uses 65536)")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill leg (profiling only)")
    ap.add_argument("--decode-seqs", type=int, default=256,
                    help="reduced decode batch (profiling only; the reported workload uses 256)")
    ap.add_argument("--workload", default="long", choices=["long", "4x4096"],
                    help="the prefill leg's workload (profiling only; the reported workload is long)")
    ap.add_argument("--gated", action="store_true",
                    help="run the prefill leg with the fused output epilogue (profiling only)")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))

    if args.impl == "reference":
        run_reference(args, world, rank)
        return

    world, rank, local = dist_setup()
    import linear_attention_sequence_kda_b200 as kda

    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    hbm_peak, bf16_peak, peak_src = peaks()

    if args.no_prefill:  # decode legs only (profiling)
        print(json.dumps({"decode": run_decode(args, world, dev, stream, kda, hbm_peak),
                          "mtp": run_mtp(args, world, dev, stream, kda, hbm_peak),
                          "mtp_fused": run_mtp_fused(args, world, dev, stream, kda, hbm_peak),
                          "decode_bf16_state": run_decode(args, world, dev, stream, kda, hbm_peak, torch.bfloat16),
                          "mtp_fused_bf16_state": run_mtp_fused(args, world, dev, stream, kda, hbm_peak,
                                                                torch.bfloat16)}),
              flush=True)
        return

    # ---------------- prefill: long-context workload, resident in HBM ----------
    heads, T_run = args.heads, args.seq_len
    profiling = args.workload != "long" or args.gated
    if args.workload == "4x4096":
        inp = ki.workload(1, heads)
        T_run = inp.total_tokens
    elif (heads, T_run) == (H, T_LONG):
        inp = ki.workload(2)
    else:  # same recipe, reduced size (for profiler captures)
        inp = ki.make_prefill([T_run], heads, torch.bfloat16, ki.BASE_SEED + 2, gate="bimodal")
    with ClockSampler(torch.cuda.current_device()) as clk:
        head_leg, ctx = run_prefill_leg(args, world, dev, stream, kda, inp, args.steps, hbm_peak, bf16_peak,
                                        peak_src, keep=True, gated=args.gated)
    d, o, S, prefill_into = ctx
    ms = head_leg["ms_per_step"]
    tokens_per_rank = T_run
    value = world * tokens_per_rank * args.steps / (head_leg["total_ms"] / 1e3)

    # ---------------- end to end: host buffers through the C ABI ----------------
    e2e = None
    if args.e2e_steps > 0:
        e2e = run_e2e(args, world, stream, inp, d, o, S, prefill_into, tokens_per_rank)

    # ---------------- decode step: 256 sequences, state in place ----------------
    dec_line = mtp_line = fused_line = dec16_line = mtp16_line = None
    if not args.no_decode:
        dec_line = run_decode(args, world, dev, stream, kda, hbm_peak)
        mtp_line = run_mtp(args, world, dev, stream, kda, hbm_peak)
        fused_line = run_mtp_fused(args, world, dev, stream, kda, hbm_peak)
        dec16_line = run_decode(args, world, dev, stream, kda, hbm_peak, torch.bfloat16)
        mtp16_line = run_mtp_fused(args, world, dev, stream, kda, hbm_peak, torch.bfloat16)

    # ---------------- the other prefill workloads (multi-sequence schedules) ----
    other_legs = {}
    if not args.no_other_prefill and (heads, T_run) == (H, T_LONG) and not profiling:
        other_legs["prefill_4x4096"] = run_prefill_leg(args, world, dev, stream, kda, ki.workload(1),
                                                       args.steps, hbm_peak, bf16_peak, peak_src)[0]
        other_legs["prefill_varlen"] = run_prefill_leg(args, world, dev, stream, kda, ki.workload(3),
                                                       max(3, args.steps // 2), hbm_peak, bf16_peak, peak_src)[0]
        other_legs["prefill_long_gated"] = run_prefill_leg(args, world, dev, stream, kda, inp, args.steps,
                                                           hbm_peak, bf16_peak, peak_src, gated=True)[0]
        other_legs["prefill_long_scan_only"] = run_scan_only(args, world, dev, stream, kda, inp, args.steps)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "heads": heads, "head_dim": D, "seq_len": T_run, "batch_per_gpu": 1,
                   "chunk": 64, "parallelism": f"dp{world} (independent sequences per GPU)",
                   "l2": "inputs larger than L2 (4.3 GB read per step), no flush"},
        "roofline": head_leg["roofline"],
        "tensor": head_leg["tensor"],
        "e2e": e2e,
        "gpu_launches": args.steps * PREFILL_LAUNCHES,
        "clocks": clk.summary(),
        "device": device_info(local),
        "decode": dec_line,
        "mtp": mtp_line,
        "mtp_fused": fused_line,
        "decode_bf16_state": dec16_line,
        "mtp_fused_bf16_state": mtp16_line,
        **other_legs,
    }
    if (heads, T_run) != (H, T_LONG) or profiling:
        line["config"]["note"] = "profiling run, not the reported workload"
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
        line["oracle_per_workload"] = oracle_per_workload()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def prefill_roofline(inp, launch_ms, hbm_peak, bf16_peak, peak_src, traffic, kernel_name, gated=False):
    """HBM roofline of one kda_prefill on the method's bytes (1,282 B per
    token-head + initial and final state per (sequence, head)), the variant
    with o as the library writes it (fp32), and the tensor-pipe fraction of the
    useful chunked work against the tf32 peak.  With the fused output
    epilogue the gate adds 256 B per token-head and o is written in bf16, as
    the method's bytes already count it."""
    tok_heads = inp.total_tokens * inp.num_heads
    pairs = inp.num_seqs * inp.num_heads
    extra = GATE_BYTES_PER_TOKEN_HEAD if gated else 0
    alg = tok_heads * (BYTES_PER_TOKEN_HEAD + extra) + pairs * 2 * STATE_BYTES
    alg32 = alg if gated else tok_heads * BYTES_PER_TOKEN_HEAD_O32 + pairs * 2 * STATE_BYTES
    sec = launch_ms / 1e3
    achieved = alg / sec / 1e9
    flops = tok_heads * FLOP_PER_TOKEN_HEAD
    tf32_peak = bf16_peak * TF32_PER_BF16
    roof = {"kernel": kernel_name, "bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
            "frac": achieved / hbm_peak, "peak_source": f"{peak_src} hbm_gbs (burst)", "traffic": traffic,
            "algorithmic_bytes_per_launch": alg, "launch_ms": launch_ms,
            "o_fp32_variant": None if gated else {
                "algorithmic_bytes_per_launch": alg32, "achieved": alg32 / sec / 1e9,
                "frac": alg32 / sec / 1e9 / hbm_peak,
                "note": "same call, o counted as written (fp32, 512 B per token-head)"}}
    tensor = {"bound": "tensor", "achieved": flops / sec / 1e12, "peak": tf32_peak, "unit": "TFLOP/s",
              "frac": flops / sec / 1e12 / tf32_peak, "flop_per_launch": flops,
              "peak_source": f"{peak_src} bf16_tflops x {TF32_PER_BF16} (nominal tf32 : bf16)"}
    return roof, tensor


def run_prefill_leg(args, world, dev, stream, kda, inp, steps, hbm_peak, bf16_peak, peak_src, keep=False,
                    gated=False):
    """Times kda_prefill (kda_prefill_gated with `gated`: the output epilogue
    fused, synthetic gate and norm weight, bf16 output) on one workload with
    its inputs resident in HBM: W warm-up calls, then `steps` calls between
    barrier + synchronize, a CUDA event pair per call on the launching stream."""
    d = {n: getattr(inp, n).to(dev) for n in ("q", "k", "v", "g", "beta", "conv_w")}
    init_state = None if inp.init_state is None else inp.init_state.to(dev)
    init_conv = None if inp.init_conv is None else inp.init_conv.to(dev)
    cu_dev = torch.from_numpy(inp.cu_seqlens).to(dev)
    N, Hh = inp.num_seqs, inp.num_heads
    o = torch.empty(d["q"].shape, dtype=torch.bfloat16 if gated else torch.float32, device=dev)
    S = torch.empty((N, Hh, D, D), dtype=torch.float32, device=dev)
    norm = {}
    if gated:
        z, w = ki.make_output_norm(inp.total_tokens, Hh, ki.BASE_SEED + 2)
        norm = {"gate": z.to(dev), "norm_weight": w.to(dev), "norm_eps": 1e-6}
    tail = torch.empty((N, 3, 3, Hh * D), dtype=torch.bfloat16, device=dev)
    max_len = int(np.diff(inp.cu_seqlens).max()) if N else 0
    ws_bytes = kda.workspace_size(N, inp.total_tokens, Hh, max_len)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)

    def prefill_into(dd, oo, ss):
        kda.prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["conv_w"], inp.cu_seqlens, cu_dev,
                    init_state, init_conv, o=oo, final_state=ss, conv_tail=tail, workspace=ws, stream=stream,
                    **norm)

    total_ms, per_step = timed(lambda: prefill_into(d, o, S), steps, args.warmup, world, stream)
    assert kda.check_async_status(stream) == 0
    launch_ms = statistics.mean(per_step)
    kernel_name = ("kda_prefill_gated" if gated else "kda_prefill") + " (chunk_prep_kernel + chunk_scan_kernel)"
    chains = N * Hh
    label = "prefill_long" if (N, inp.total_tokens) == (1, T_LONG) else (
        "prefill_4x4096" if (N, inp.total_tokens) == (4, 16384) else "prefill_varlen")
    roof, tensor = prefill_roofline(inp, launch_ms, hbm_peak, bf16_peak, peak_src,
                                    recorded_traffic(f"{kernel_name} {label}"), kernel_name, gated)
    out_desc = "bf16 out through the fused gated RMS normalisation" if gated else "fp32 out"
    leg = {"workload": f"kda_prefill: {N} sequence(s), {inp.total_tokens} tokens, {Hh} heads x 128, bf16 in / "
                       f"fp32 state / {out_desc}, {chains} (sequence, head) chains "
                       f"({'overlapped' if chains <= 96 else 'one after the other'} schedule)",
           "tokens_per_s": world * inp.total_tokens * steps / (total_ms / 1e3), "ms_per_step": total_ms / steps,
           "total_ms": total_ms, "steps": steps, "roofline": roof, "tensor": tensor,
           "gpu_launches": steps * PREFILL_LAUNCHES}
    if keep:
        return leg, (d, o, S, prefill_into)
    del d, o, S, ws
    torch.cuda.empty_cache()
    return leg, None


def run_scan_only(args, world, dev, stream, kda, inp, steps):
    """The state scan alone on the long-context workload: one record-keeping
    call (kda_prefill_records) prepares every chunk record, then `steps`
    kda_prefill_scan calls over those records are timed like the prefill leg.
    With every record ready, the call is the 64 serial chains: its time over
    the chunk count is the chain's time per chunk."""
    d = {n: getattr(inp, n).to(dev) for n in ("q", "k", "v", "g", "beta", "conv_w")}
    cu_dev = torch.from_numpy(inp.cu_seqlens).to(dev)
    N, Hh = inp.num_seqs, inp.num_heads
    o = torch.empty(d["q"].shape, dtype=torch.float32, device=dev)
    S = torch.empty((N, Hh, D, D), dtype=torch.float32, device=dev)
    tail = torch.empty((N, 3, 3, Hh * D), dtype=torch.bfloat16, device=dev)
    max_len = int(np.diff(inp.cu_seqlens).max())
    ws = torch.empty(kda.workspace_size(N, inp.total_tokens, Hh, max_len), dtype=torch.uint8, device=dev)

    def call(mode):
        kda.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["conv_w"], inp.cu_seqlens, cu_dev, None, None,
                    o=o, final_state=S, conv_tail=tail, workspace=ws, stream=stream, mode=mode)

    call("records")
    total_ms, per_step = timed(lambda: call("scan"), steps, args.warmup, world, stream)
    assert kda.check_async_status(stream) == 0
    chunks = -(-max_len // 64)
    ms = total_ms / steps
    out = {"workload": f"kda_prefill_scan over kept records: {N} x {inp.total_tokens} tokens, {Hh} heads x 128 "
                       f"({N * Hh} chains of {chunks} chunks)",
           "ms_per_step": ms, "steps": steps, "us_per_chunk": ms * 1e3 / chunks,
           "gpu_launches": steps * 2}
    del d, o, S, ws
    torch.cuda.empty_cache()
    return out


def oracle_per_workload():
    """The fp64 oracle as it stands, timed on this host's cores for every
    workload (a bounded sample of the large ones), with the thread count, and
    on one core for the tiny and the decode workloads."""
    import oracle  # test infrastructure; only the baseline legs run it
    cores = os.cpu_count() or 1
    out = {}

    def time_probs(probs, threads):
        t0 = time.perf_counter()
        used = oracle.run_problems(probs, threads)
        return time.perf_counter() - t0, used

    def prefill_sample(i, inp, tokens_note):
        probs = [oracle.prefill_problem(inp, n, h) for n in range(inp.num_seqs) for h in range(inp.num_heads)]
        toks = inp.total_tokens
        dt, used = time_probs(probs, cores)
        rec = {"tokens_per_s": toks / dt, "cores": used, "seconds": dt, "sample": tokens_note}
        if i == 0:
            dt1, _ = time_probs([oracle.prefill_problem(inp, n, h) for n in range(inp.num_seqs)
                                 for h in range(inp.num_heads)], 1)
            rec["one_core_tokens_per_s"] = toks / dt1
        return rec

    out["tiny_fp32"] = prefill_sample(0, ki.workload(0), "whole workload (1 x 256 tokens, 2 heads)")
    w1 = ki.workload(1)
    out["prefill_4x4096"] = prefill_sample(1, w1, "whole workload (4 x 4096 tokens, 64 heads)")
    del w1
    w2 = ki.make_prefill([4096], H, torch.bfloat16, ki.BASE_SEED + 2, gate="bimodal")
    out["prefill_long"] = prefill_sample(2, w2, "first 4096 tokens x 64 heads of the T=65536 workload")
    del w2
    lens = ki.varlen_lengths(ki.BASE_SEED + 3)
    w3 = ki.make_prefill([min(lens[0], 4096)], H, torch.bfloat16, ki.BASE_SEED + 3, state_std=0.02,
                         conv_history=True)
    out["prefill_varlen"] = prefill_sample(3, w3, f"first {min(lens[0], 4096)} tokens of segment 0 x 64 heads "
                                                  f"of the varlen workload (same recipe)")
    del w3
    dec = ki.workload(4)
    probs = [oracle.decode_problem(dec, n, h) for n in range(dec.num_seqs) for h in range(H)]
    dt, used = time_probs(probs, cores)
    probs1 = [oracle.decode_problem(dec, n, h) for n in range(16) for h in range(H)]
    dt1, _ = time_probs(probs1, 1)
    out["decode"] = {"tokens_per_s": dec.num_seqs / dt, "cores": used, "seconds": dt,
                     "one_core_tokens_per_s": 16 / dt1,
                     "sample": "whole workload (256 sequences x 64 heads, one step); one core on 16 sequences"}
    return out


def run_e2e(args, world, stream, inp, d, o, S, prefill_into, tokens_per_rank):
    """Same metric through the C ABI with host buffers: every step copies its
    inputs from pinned host memory, runs kda_prefill, and reads o and the final
    state back to pinned host memory.  The steps are pipelined as a serving
    loop would run them: step i+1's inputs travel host-to-device on one copy
    stream while step i computes and step i-1's results travel back on
    another (two device buffer sets alternate).  The timed region starts
    before the first step's input copy and ends after the last step's result
    has reached the host."""
    pin = {n: getattr(inp, n).pin_memory() for n in ("q", "k", "v", "g", "beta")}
    o_host = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    S_host = torch.empty(S.shape, dtype=S.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = o_host.numel() * o_host.element_size() + S_host.numel() * 4
    sets = [(d, o, S), ({**d, **{n: torch.empty_like(d[n]) for n in pin}}, torch.empty_like(o), torch.empty_like(S))]
    up, down = torch.cuda.Stream(device=o.device), torch.cuda.Stream(device=o.device)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready, computed, out_read = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    issued = [False, False]

    def e2e_step(i):
        b = i % 2
        dd, ob, sb = sets[b]
        if issued[b]:  # step i - 2 has finished with this buffer set
            up.wait_event(computed[b])
        with torch.cuda.stream(up):
            for n, t in pin.items():
                dd[n].copy_(t, non_blocking=True)
            in_ready[b].record(up)
        stream.wait_event(in_ready[b])
        if issued[b]:
            stream.wait_event(out_read[b])
        prefill_into(dd, ob, sb)
        computed[b].record(stream)
        down.wait_event(computed[b])
        with torch.cuda.stream(down):
            o_host.copy_(ob, non_blocking=True)
            S_host.copy_(sb, non_blocking=True)
            out_read[b].record(down)
        issued[b] = True

    for i in range(2):  # warm-up
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    up.wait_event(start)
    for i in range(args.e2e_steps):
        e2e_step(i)
    stream.wait_stream(down)
    stop.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(start.elapsed_time(stop), world)
    value = world * tokens_per_rank * args.e2e_steps / (e2e_ms / 1e3)

    # the host link alone: the same copies with nothing else on the device, each
    # direction timed on its own stream (max over ranks)
    def link_gbs(copy_stream, copies, nbytes, reps=3):
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        barrier(world)
        with torch.cuda.stream(copy_stream):
            a.record(copy_stream)
            for _ in range(reps):
                copies()
            z.record(copy_stream)
        torch.cuda.synchronize()
        return nbytes * reps / (max_over_ranks(a.elapsed_time(z), world) / 1e3) / 1e9

    dd0, ob0, sb0 = sets[0]
    ups = lambda: [dd0[n].copy_(t, non_blocking=True) for n, t in pin.items()]  # noqa: E731
    downs = lambda: (o_host.copy_(ob0, non_blocking=True), S_host.copy_(sb0, non_blocking=True))  # noqa: E731
    h2d_alone = link_gbs(up, ups, h2d)
    d2h_alone = link_gbs(down, downs, d2h)
    # both directions at once, as the pipelined loop runs them: the copy-only step time
    reps = 3
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(world)
    a.record(stream)
    up.wait_event(a)
    down.wait_event(a)
    for _ in range(reps):
        with torch.cuda.stream(up):
            ups()
        with torch.cuda.stream(down):
            downs()
    stream.wait_stream(up)
    stream.wait_stream(down)
    z.record(stream)
    torch.cuda.synchronize()
    copy_ms = max_over_ranks(a.elapsed_time(z), world) / reps
    ceiling = world * tokens_per_rank / (copy_ms / 1e3)
    return {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": args.e2e_steps, "pipelined": "inputs of step i+1 up and results of step i-1 down while step i runs",
            "link": {"bound": "host link", "h2d_gbs_alone": h2d_alone, "d2h_gbs_alone": d2h_alone,
                     "copy_ms_per_step": copy_ms, "ceiling": ceiling, "frac": value / ceiling,
                     "h2d_gbs_in_e2e": h2d * args.e2e_steps / (e2e_ms / 1e3) / 1e9,
                     "note": "ceiling = the step's copies alone (pinned host memory, same tensors, both "
                             "directions at once, 3 repeats), no kernel"}}


def run_decode(args, world, dev, stream, kda, hbm_peak, state_dtype=torch.float32):
    """kda_decode_step on the decode workload (256 sequences, state in place,
    stored in `state_dtype`)."""
    dec = ki.workload(4) if args.decode_seqs == 256 else \
        ki.make_decode(args.decode_seqs, H, torch.bfloat16, ki.BASE_SEED + 4)
    dd = {n: getattr(dec, n).to(dev) for n in ("state", "conv_cache", "q", "k", "v", "g", "beta", "conv_w")}
    dd["state"] = dd["state"].to(state_dtype)
    sb = dd["state"].element_size()
    sname = "fp32" if sb == 4 else "bf16"
    o_dec = torch.empty(dd["q"].shape, dtype=torch.float32, device=dev)

    def dstep():
        kda.decode_step(dd["state"], dd["conv_cache"], dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"],
                        dd["conv_w"], o=o_dec, stream=stream)

    _, dec_steps = timed(dstep, args.steps, args.warmup, world, stream)
    npairs = dec.num_seqs * H
    dec_ms = statistics.mean(dec_steps)
    dec_state_gbs = npairs * 2 * D * D * sb / (dec_ms / 1e3) / 1e9
    alg = npairs * dec_bytes_per_pair(sb)
    dec_alg_gbs = alg / (dec_ms / 1e3) / 1e9
    return {"workload": f"kda_decode_step: {dec.num_seqs} sequences x 1 token, 64 heads x 128, "
                        f"{sname} state in place",
            "state_gbs": dec_state_gbs, "ms_per_step": dec_ms, "tokens_per_s": dec.num_seqs / (dec_ms / 1e3),
            "roofline": {"kernel": "kda_decode", "bound": "hbm", "achieved": dec_alg_gbs, "peak": hbm_peak,
                         "unit": "GB/s", "frac": dec_alg_gbs / hbm_peak, "state_frac": dec_state_gbs / hbm_peak,
                         "traffic": recorded_traffic("kda_decode" if sb == 4 else "kda_decode bf16_state"),
                         "algorithmic_bytes_per_launch": alg},
            "gpu_launches": args.steps * DECODE_LAUNCHES}


def run_mtp(args, world, dev, stream, kda, hbm_peak, state_dtype=torch.float32):
    """Multi-token decode for speculative serving: kda_decode_verify of 6 rows
    (5 drafts + 1) per sequence, then kda_decode_commit of the kept prefix
    (2..6 rows, about four on average), 256 sequences x 64 heads, state stored
    in `state_dtype`."""
    N = args.decode_seqs
    mt = ki.make_decode_rows(N, MTP_ROWS, H, torch.bfloat16, ki.BASE_SEED + 5, accept=(2, MTP_ROWS))
    dd = {n: getattr(mt, n).to(dev) for n in ("state", "conv_cache", "q", "k", "v", "g", "beta", "conv_w")}
    dd["state"] = dd["state"].to(state_dtype)
    sb = dd["state"].element_size()
    sname = "fp32" if sb == 4 else "bf16"
    o_m = torch.empty(dd["q"].shape, dtype=torch.float32, device=dev)
    deltas = torch.empty(kda.deltas_size(N, MTP_ROWS, H) // 4, dtype=torch.float32, device=dev)
    n_acc = torch.from_numpy(mt.n_accept).to(dev)

    def mstep():
        kda.decode_verify(dd["state"], dd["conv_cache"], dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"],
                          dd["conv_w"], o=o_m, deltas=deltas, stream=stream)
        kda.decode_commit(dd["state"], dd["conv_cache"], dd["q"], dd["k"], dd["v"], deltas, n_acc, stream=stream)

    _, steps = timed(mstep, args.steps, args.warmup, world, stream)
    assert kda.check_async_status(stream) == 0
    ms = statistics.mean(steps)

    def vstep():
        kda.decode_verify(dd["state"], dd["conv_cache"], dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"],
                          dd["conv_w"], o=o_m, deltas=deltas, stream=stream)

    _, vsteps = timed(vstep, args.steps, args.warmup, world, stream)
    verify_ms = statistics.mean(vsteps)
    npairs = N * H
    alg = npairs * mtp_bytes_per_pair(sb)
    gbs = alg / (ms / 1e3) / 1e9
    return {"workload": f"kda_decode_verify + kda_decode_commit: {N} sequences x {MTP_ROWS} rows, 64 heads x 128, "
                        f"{int(mt.n_accept.sum())} rows kept, {sname} state in place",
            "verified_rows_per_s": N * MTP_ROWS / (ms / 1e3), "kept_tokens_per_s": int(mt.n_accept.sum()) / (ms / 1e3),
            "ms_per_step": ms, "verify_ms": verify_ms, "commit_ms": ms - verify_ms,
            "state_gbs": npairs * 3 * D * D * sb / (ms / 1e3) / 1e9,
            "roofline": {"kernel": "kda_decode_verify + kda_decode_commit", "bound": "hbm", "achieved": gbs,
                         "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                         "traffic": recorded_traffic("kda_decode_verify + kda_decode_commit"
                                                     + ("" if sb == 4 else " bf16_state")),
                         "algorithmic_bytes_per_launch": alg},
            "gpu_launches": args.steps * (MTP_LAUNCHES + 1)}


def run_mtp_fused(args, world, dev, stream, kda, hbm_peak, state_dtype=torch.float32):
    """The same speculative serving loop with one kda_decode_commit_verify per
    step: keep the previous step's accepted rows and verify 6 new rows in one
    pass over the state (steady state: every step commits the step before)."""
    N = args.decode_seqs
    mt = ki.make_decode_rows(N, MTP_ROWS, H, torch.bfloat16, ki.BASE_SEED + 5, accept=(2, MTP_ROWS))
    dd = {n: getattr(mt, n).to(dev) for n in ("state", "conv_cache", "q", "k", "v", "g", "beta", "conv_w")}
    dd["state"] = dd["state"].to(state_dtype)
    sb = dd["state"].element_size()
    o_m = torch.empty(dd["q"].shape, dtype=torch.float32, device=dev)
    bufs = [torch.empty(kda.deltas_size(N, MTP_ROWS, H) // 4, dtype=torch.float32, device=dev) for _ in range(2)]
    n_acc = torch.from_numpy(mt.n_accept).to(dev)
    kda.decode_verify(dd["state"], dd["conv_cache"], dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["conv_w"],
                      o=o_m, deltas=bufs[0], stream=stream)
    cur = [0]

    def fstep():
        prev, new = bufs[cur[0]], bufs[1 - cur[0]]
        kda.decode_commit_verify(dd["state"], dd["conv_cache"], (dd["q"], dd["k"], dd["v"], prev, n_acc), dd["q"],
                                 dd["k"], dd["v"], dd["g"], dd["beta"], dd["conv_w"], o=o_m, deltas=new,
                                 stream=stream)
        cur[0] = 1 - cur[0]

    _, steps = timed(fstep, args.steps, args.warmup, world, stream)
    assert kda.check_async_status(stream) == 0
    ms = statistics.mean(steps)
    npairs = N * H
    kept = float(mt.n_accept.mean())
    # per (sequence, head): state read + written; per new row deltas written,
    # q k v g read, beta, o fp32; per kept previous row its deltas read; the
    # conv cache read and written and the kept raw rows read for it
    per_pair = (2 * D * D * sb + MTP_ROWS * (3 * D * 4 + 4 * D * 2 + 2 + D * 4) + kept * 3 * D * 4
                + 2 * 9 * D * 2 + 9 * D * 2)
    alg = npairs * per_pair
    gbs = alg / (ms / 1e3) / 1e9
    return {"workload": f"kda_decode_commit_verify: {N} sequences x {MTP_ROWS} rows, 64 heads x 128, "
                        f"{int(mt.n_accept.sum())} rows of the previous step kept, "
                        f"{'fp32' if sb == 4 else 'bf16'} state in place",
            "verified_rows_per_s": N * MTP_ROWS / (ms / 1e3), "kept_tokens_per_s": int(mt.n_accept.sum()) / (ms / 1e3),
            "ms_per_step": ms, "state_gbs": npairs * 2 * D * D * sb / (ms / 1e3) / 1e9,
            "roofline": {"kernel": "kda_decode_commit_verify", "bound": "hbm", "achieved": gbs, "peak": hbm_peak,
                         "unit": "GB/s", "frac": gbs / hbm_peak,
                         "traffic": recorded_traffic("kda_decode_commit_verify" + ("" if sb == 4 else " bf16_state")),
                         "algorithmic_bytes_per_launch": alg},
            "gpu_launches": args.steps}


if __name__ == "__main__":
    main()
