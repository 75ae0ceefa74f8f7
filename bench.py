#!/usr/bin/env python
"""Benchmark of exact tiled attention on B200: forward + backward TFLOP/s.

Workload (default): causal bf16 attention, B=1 H=32 S=4096 D=128, scale
1/sqrt(128), seeded N(0,1) synthetic Q, K, V, dO.  One step is the whole hot
path: fa_fwd, then the three backward launches (fa_bwd_preprocess,
fa_bwd_main, fa_bwd_finish).  FLOPs follow the usual convention: forward
4*B*H*S^2*D halved under the causal mask, backward 2.5x that.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 is launched with torchrun (one rank per GPU).  The heads are
independent, so every rank runs its own copy of the workload (weak scaling,
no data-path collective); the NCCL group only carries the barrier and the
max-over-ranks timing.  ``--impl reference`` times the fp64 CPU oracle on a
bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attn fwd & fwd+bwd TFLOP/s, bf16 causal S=4096 D=128; % of B200 dense peak"
DATASHEET_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
WORKLOADS = {
    "b1_h32_s4096_d128_causal": dict(B=1, H=32, S=4096, D=128, causal=True),
    "b4_h16_s8192_d128_causal": dict(B=4, H=16, S=8192, D=128, causal=True),
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="b1_h32_s4096_d128_causal")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--sustained-s", type=float, default=2.0,
                    help="seconds of back-to-back steps for the sustained leg (0 runs a single step)")
    return ap.parse_args()


def flops(w):
    f = 4.0 * w["B"] * w["H"] * w["S"] ** 2 * w["D"] * (0.5 if w["causal"] else 1.0)
    return f, 2.5 * f


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of each
# dominant kernel at the default workload, from the ncu captures summarised in
# profiles/, with a digest of the kernel sources (code only) they were taken on.
# Reported only while that code is unchanged (otherwise null: the counters are stale).
NCU_TRAFFIC = {
    "bwd_main": (289_130_957, "015da12a81d87b63e77598732a9fcbca3eca84d1bbd4ee8eb74bb88f2f4bc66f",
                 ("fa_bwd.cuh", "sm100.cuh")),
    "fwd": (151_631_642, "44bf43a5f4609a34b73445fd2c1ff632a5ceb5b5098a84206308e1354c97d38a",
            ("fa_fwd.cuh", "sm100.cuh")),
    # decode split kernel, B8 Hq32 Hkv8 L8192 D128 bf16, 2 splits merged in-kernel (mean of 13 launches)
    "decode": (268_978_708, "4696a7ff08d2327e8bf9a19eb0d9726cd3c9d323b54f6fb50c07502f9a1c391b",
               ("fa_decode.cuh", "sm100.cuh")),
}


def source_digest(files) -> str:
    """SHA-256 of the kernel sources with comments and blank space removed
    (edits to comments leave the counters valid; any code change does not)."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "exact_tiled_attention_31_b200", "csrc", f)) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update(re.sub(r"\s+", "", text).encode())
    return h.hexdigest()


def captured_traffic(kernel: str):
    nbytes, digest, files = NCU_TRAFFIC[kernel]
    return nbytes if source_digest(files) == digest else None


def max_over_ranks(vals: dict, device=None) -> dict:
    """Per-key maximum over the ranks of the default process group (the
    slowest rank's time); the values themselves when there is no group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return dict(vals)
    keys = sorted(vals)
    t = torch.tensor([float(vals[k]) for k in keys], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return dict(zip(keys, t.tolist()))


def job_tflops(world: int, flop_per_rank: float, ms: float) -> float:
    """Whole-job throughput: every rank runs the same workload (weak scaling),
    timed by the slowest rank."""
    return world * flop_per_rank / (ms * 1e-3) / 1e12


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads") or 0) for i in threadpool_info())
        if n:
            return int(n)
    except Exception:
        pass
    return os.cpu_count() or 1


# ------------------------------------------------------------------ clocks

class NvmlClockSampler:
    """SM clock, power and clock-event reasons read through NVML (read-only
    queries) by a background thread, about once per millisecond, so that even
    a timed region of a few milliseconds gets many samples.  Rows carry a
    time.time() stamp like the nvidia-smi sampler's."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, uuid: str | None, index: int):
        import threading
        import pynvml
        self.nv = pynvml
        pynvml.nvmlInit()
        self.h = (pynvml.nvmlDeviceGetHandleByUUID(uuid) if uuid else pynvml.nvmlDeviceGetHandleByIndex(index))
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        self.bits = [(name, getattr(pynvml, attr)) for name, attr in self.REASONS]
        self.rows, self.stop_evt = [], threading.Event()
        self.t0 = self.t1 = None
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        nv = self.nv
        while not self.stop_evt.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                power = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
            except Exception:
                break
            self.rows.append(dict(ts=time.time(), sm=sm, sm_max=self.max_mhz, power=power,
                                  reasons=[n for n, b in self.bits if reasons & b]))
            self.stop_evt.wait(0.001)

    def stop(self):
        self.stop_evt.set()
        self.thread.join(timeout=5)
        try:
            self.nv.nvmlShutdown()
        except Exception:
            pass
        return self.rows

    def summary(self, rows, t0=None, t1=None):
        return clock_summary(rows, self.t0 if t0 is None else t0, self.t1 if t1 is None else t1, "nvml")


def clock_summary(rows, t0, t1, source):
    """Median SM clock, reasons and sample counts of the rows inside [t0, t1]
    (all rows when none falls inside)."""
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": source}
    inside = [r for r in rows if t0 is not None and t0 <= r["ts"] <= t1]
    use = inside or rows
    reasons = sorted({n for r in use for n in r["reasons"]})
    return {"sm_mhz": statistics.median(r["sm"] for r in use), "sm_max_mhz": max(r["sm_max"] for r in use),
            "reasons": reasons, "samples": len(use), "samples_in_timed_region": len(inside),
            "power_w_max": max((r["power"] or 0.0) for r in use), "source": source}


def start_clock_sampler(gpu_uuid, index):
    try:
        return NvmlClockSampler(gpu_uuid, index)
    except Exception:
        return ClockSampler(gpu_uuid)


class ClockSampler:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id: str | None):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if gpu_id:
            cmd += ["-i", gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        self.t0 = self.t1 = None

    def stop(self):
        if not self.proc:
            return []
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                stamp, _, frac = parts[0].partition(".")
                ts = time.mktime(time.strptime(stamp, "%Y/%m/%d %H:%M:%S")) + (float("0." + frac) if frac else 0.0)
                rows.append(dict(ts=ts, sm=float(parts[1]), sm_max=float(parts[2]),
                                 power=float(parts[3]) if parts[3] not in ("[N/A]", "N/A") else None,
                                 reasons=[n for n, v in zip(self.NAMES, parts[4:8]) if v.lower() == "active"]))
            except (ValueError, IndexError):
                continue
        return rows

    def summary(self, rows, t0=None, t1=None):
        t0 = self.t0 if t0 is None else t0
        t1 = self.t1 if t1 is None else t1
        return clock_summary(rows, None if t0 is None else t0 - 0.15, None if t1 is None else t1 + 0.15, "nvidia-smi")


# ------------------------------------------------------------------ CPU oracle legs

def oracle_sample(w, target_s: float, max_heads: int = 4):
    """Time the fp64 oracle fwd+bwd on whole heads of the workload until
    about ``target_s`` seconds have passed; returns (flops, seconds, heads)."""
    from exact_tiled_attention_31_b200 import inputs
    from oracle import attention as oa
    t = inputs.make_dense(1, 1, w["S"], w["D"], "bf16", seed=42, with_do=True)
    scale = 1.0 / math.sqrt(w["D"])
    f_fwd, f_bwd = flops(dict(w, B=1, H=1))
    done, t_total = 0, 0.0
    while done < max_heads and (done == 0 or t_total < target_s):
        t0 = time.perf_counter()
        oa.attention_forward(t["q"][0, 0], t["k"][0, 0], t["v"][0, 0], scale, w["causal"])
        oa.attention_backward(t["q"][0, 0], t["k"][0, 0], t["v"][0, 0], t["do"][0, 0], scale, w["causal"])
        t_total += time.perf_counter() - t0
        done += 1
    return done * (f_fwd + f_bwd), t_total, done


def run_reference(args, rank, world, w):
    """--impl reference: the fp64 oracle on the host cores, rank 0 only."""
    if rank != 0:
        return
    from exact_tiled_attention_31_b200 import inputs
    from oracle import attention as oa
    scale = 1.0 / math.sqrt(w["D"])
    # each step: fwd+bwd of the causal prefix of length L of head (0, 0), L
    # chosen so the whole run stays within about two minutes
    t = inputs.make_dense(1, 1, w["S"], w["D"], "bf16", seed=42, with_do=True)
    q, k, v, do = (t[x][0, 0] for x in ("q", "k", "v", "do"))

    def step(L):
        oa.attention_forward(q[:L], k[:L], v[:L], scale, w["causal"])
        oa.attention_backward(q[:L], k[:L], v[:L], do[:L], scale, w["causal"])

    L = w["S"]
    t0 = time.perf_counter()
    step(min(L, 512))
    probe = time.perf_counter() - t0
    budget = 120.0 / max(1, args.steps + args.warmup)
    while L > 128 and probe * (L / 512.0) ** 2 > budget:
        L //= 2
    for _ in range(args.warmup):
        step(L)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step(L)
    el = time.perf_counter() - t0
    f_fwd, f_bwd = flops(dict(w, B=1, H=1, S=L))
    val = (f_fwd + f_bwd) * args.steps / el / 1e12
    sample = f"fwd+bwd of the causal prefix of length {L} of 1 of {w['B'] * w['H']} heads per step"
    out = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": {"workload": args.workload, **w},
           "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


# ------------------------------------------------------------------ GPU arm

# Decode leg: one new token per (sequence, query head) against full KV caches,
# grouped-query heads (32 query heads on 8 KV heads), bf16.  Its bound is HBM:
# the algorithmic bytes are the cache rows read once plus q, O and LSE.
DECODE = dict(B=8, Hq=32, Hkv=8, L=8192, D=128)


def decode_bytes(d) -> int:
    cache = 2 * d["B"] * d["Hkv"] * d["L"] * d["D"] * 2
    return cache + 2 * d["B"] * d["Hq"] * d["D"] * 2 + d["B"] * d["Hq"] * 4


def decode_leg(fa, inputs, torch, dev, stream, steps: int, warmup: int, hbm_peak: float, peak_kind: str):
    """Mean device time of fa_decode (split + merge launches) on DECODE.

    Two sets of inputs (2 x 268 MB of caches, each set above the 126 MB L2)
    alternate between steps, so a step never finds the previous step's cache
    rows in L2; no write-flush runs in between (its dirty lines would be
    written back during the next step and bill it for unrelated traffic)."""
    d = DECODE
    sets = []
    for seed in (42, 43):
        host = inputs.make_decode(d["B"], d["Hq"], d["Hkv"], d["L"], d["D"], "bf16", seed=seed)
        sets.append(tuple(host[x].to(dev) for x in ("q", "k", "v")))
    lens = torch.full((d["B"],), d["L"], dtype=torch.int32, device=dev)
    o = torch.empty_like(sets[0][0])
    lse = torch.empty((d["B"], d["Hq"]), device=dev, dtype=torch.float32)
    n = fa.fa_decode_num_splits(d["B"], d["Hkv"], d["L"])
    ws_bytes = fa.fa_decode_workspace_size(d["B"], d["Hq"], n, d["D"])
    ws = torch.empty(ws_bytes, device=dev, dtype=torch.uint8)
    scale = 1.0 / math.sqrt(d["D"])

    def call(i):
        q, k, v = sets[i % 2]
        st = fa.fa_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), lens.data_ptr(), o.data_ptr(), lse.data_ptr(),
                          d["B"], d["Hq"], d["Hkv"], d["L"], d["D"], scale, fa.api.FA_BF16, n, ws.data_ptr(),
                          ws_bytes, stream.cuda_stream)
        if st != 0:
            raise fa.FAError(st, "fa_decode")

    for i in range(max(warmup, 3)):
        call(i)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda._sleep(20_000_000)  # the host queues the timed calls while the GPU spins (~10 ms)
    for i, (e0, e1) in enumerate(evs):
        e0.record(stream)
        call(i)
        e1.record(stream)
    torch.cuda.synchronize()
    fa.check_device_error()
    ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in evs)
    nbytes = decode_bytes(d)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": "decode_b8_hq32_hkv8_l8192_d128_bf16", **d, "n_splits": n, "ms_per_step": ms,
            "value": gbs, "unit": "GB/s", "tokens_per_s": d["B"] / (ms * 1e-3),
            "l2": "two input sets of 268 MB alternate (inputs larger than L2), no flush",
            "roofline": {"kernel": "fa::decode_split_kernel<128,bf16>" + (
                             " (2..4-CTA clusters, merged in-kernel)" if 2 <= n <= 4 else
                             "" if n == 1 else " + fa::decode_merge_kernel<128,bf16>"),
                         "bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                         "traffic": captured_traffic("decode"), "algorithmic_bytes_per_launch": nbytes,
                         "peak_source": f"{peak_kind} copy bandwidth (hbm_gbs)"}}


def main():
    args = parse()
    w = WORKLOADS[args.workload]
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world, w)
        return

    import datetime

    import torch
    import torch.distributed as dist

    import exact_tiled_attention_31_b200 as fa
    from exact_tiled_attention_31_b200 import inputs

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    B, H, S, D, causal = w["B"], w["H"], w["S"], w["D"], w["causal"]
    scale = 1.0 / math.sqrt(D)
    host = inputs.make_dense(B, H, S, D, "bf16", seed=42, with_do=True)
    q, k, v, do = (host[x].to(dev) for x in ("q", "k", "v", "do"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, S), device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = fa.fa_bwd_workspace_size(B, H, S, D)
    ws = torch.empty(ws_bytes, device=dev, dtype=torch.uint8)
    flush = torch.empty(256 * 1024 * 1024, device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream
    dt = fa.api.FA_BF16

    def chk(st, what):
        if st != 0:
            raise fa.FAError(st, what)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        chk(fa.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, S, D, scale,
                      causal, dt, sh), "fa_fwd")
        if ev:
            ev[1].record(stream)
        chk(fa.fa_bwd_preprocess(o.data_ptr(), do.data_ptr(), lse.data_ptr(), B, H, S, D, dt, ws.data_ptr(),
                                 ws_bytes, sh), "fa_bwd_preprocess")
        if ev:
            ev[2].record(stream)
        chk(fa.fa_bwd_main(q.data_ptr(), k.data_ptr(), v.data_ptr(), do.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                           B, H, S, D, scale, causal, dt, 0, ws.data_ptr(), ws_bytes, sh), "fa_bwd_main")
        if ev:
            ev[3].record(stream)
        chk(fa.fa_bwd_finish(dq.data_ptr(), B, H, S, D, scale, dt, 0, ws.data_ptr(), ws_bytes, sh), "fa_bwd_finish")
        if ev:
            ev[4].record(stream)

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    fa.check_device_error()
    torch.cuda.synchronize()

    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = start_clock_sampler(gpu_id, local)
    time.sleep(0.3)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    sampler.t0 = time.time()
    launches0 = fa.fa_launch_count()
    for i in range(args.steps):
        flush.zero_()  # write 256 MiB (> 126 MB L2) between timed steps; not inside any event pair
        step(evs[i])
    torch.cuda.synchronize()
    barrier()
    sampler.t1 = time.time()
    launches = fa.fa_launch_count() - launches0
    fa.check_device_error()

    # ---- warm L2: 20 steps back to back, each between its own events; the
    # median (the L2 holds whatever the previous step left).  Run before the
    # sustained leg, which leaves the GPU at its power-capped clock.
    warm_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(20)]
    barrier()
    torch.cuda.synchronize()
    for e0, e1 in warm_ev:
        e0.record(stream)
        step()
        e1.record(stream)
    torch.cuda.synchronize()
    fa.check_device_error()
    warm_ms = max_over_ranks({"w": statistics.median(a.elapsed_time(b) for a, b in warm_ev)}, device=dev)["w"]

    # ---- sustained: the same step back to back (no flush in between) for
    # about two seconds, clocks sampled over the whole run
    sus_n = max(1, int(args.sustained_s / max(1e-4, statistics.mean(e[0].elapsed_time(e[4]) for e in evs) * 1e-3)))
    sus_e0, sus_e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    sus_t0 = time.time()
    sus_e0.record(stream)
    for _ in range(sus_n):
        step()
    sus_e1.record(stream)
    torch.cuda.synchronize()
    sus_t1 = time.time()
    clock_rows = sampler.stop()
    fa.check_device_error()
    sus_ms = max_over_ranks({"s": sus_e0.elapsed_time(sus_e1) / sus_n}, device=dev)["s"]


    t_fwd = [e[0].elapsed_time(e[1]) for e in evs]
    t_pre = [e[1].elapsed_time(e[2]) for e in evs]
    t_main = [e[2].elapsed_time(e[3]) for e in evs]
    t_fin = [e[3].elapsed_time(e[4]) for e in evs]
    t_step = [e[0].elapsed_time(e[4]) for e in evs]
    ms = {"step": statistics.mean(t_step), "fwd": statistics.mean(t_fwd), "bwd_pre": statistics.mean(t_pre),
          "bwd_main": statistics.mean(t_main), "bwd_finish": statistics.mean(t_fin)}
    ms = max_over_ranks(ms, device=dev)
    f_fwd, f_bwd = flops(w)
    t_bwd = ms["bwd_pre"] + ms["bwd_main"] + ms["bwd_finish"]
    value = job_tflops(world, f_fwd + f_bwd, ms["step"])
    fwd_tf = f_fwd / (ms["fwd"] * 1e-3) / 1e12
    bwd_tf = f_bwd / (t_bwd * 1e-3) / 1e12
    fb_tf = (f_fwd + f_bwd) / ((ms["fwd"] + t_bwd) * 1e-3) / 1e12

    # ---- end to end through the public API from pinned host buffers.  Each
    # step copies its inputs in and its results out; three streams overlap
    # the copy-in of step i + 1, the compute of step i and the copy-out of
    # step i - 1 (device tensors double-buffered), as a training loop fed from
    # host memory would.
    e2e = None
    if not args.no_e2e:
        nset = 2
        hin = [[host[x].clone().pin_memory() for x in ("q", "k", "v", "do")] for _ in range(nset)]
        hout = [[torch.empty_like(host["q"]).pin_memory(), torch.empty((B, H, S), dtype=torch.float32).pin_memory()]
                + [torch.empty_like(host["q"]).pin_memory() for _ in range(3)] for _ in range(nset)]
        din = [[torch.empty_like(x, device=dev) for x in hin[0]] for _ in range(nset)]
        dout = [[torch.empty_like(hout[0][0], device=dev), torch.empty((B, H, S), device=dev, dtype=torch.float32)]
                + [torch.empty_like(hout[0][0], device=dev) for _ in range(3)] for _ in range(nset)]
        h2d = sum(x.numel() * x.element_size() for x in hin[0])
        d2h = sum(x.numel() * x.element_size() for x in hout[0])
        e_steps = max(4, min(args.steps, 100))  # the K timed steps: one pipeline fill and drain over all of them
        s_in, s_comp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def run(n):
            ev_in, ev_comp, ev_out = [], [], []
            for i in range(n):
                b = i % nset
                with torch.cuda.stream(s_in):
                    if i >= nset:  # set b's inputs were consumed by compute i - nset
                        s_in.wait_event(ev_comp[i - nset])
                    for src, dst in zip(hin[b], din[b]):
                        dst.copy_(src, non_blocking=True)
                    ev_in.append(torch.cuda.Event())
                    ev_in[-1].record(s_in)
                with torch.cuda.stream(s_comp):
                    s_comp.wait_event(ev_in[i])
                    if i >= nset:  # set b's outputs were copied out by step i - nset
                        s_comp.wait_event(ev_out[i - nset])
                    qq, kk, vv, dd = din[b]
                    o_, l_ = fa.forward(qq, kk, vv, causal, scale, out=dout[b][0], lse=dout[b][1], stream=s_comp)
                    fa.backward(qq, kk, vv, o_, dd, l_, causal, scale, workspace=ws, stream=s_comp,
                                out=(dout[b][2], dout[b][3], dout[b][4]))
                    ev_comp.append(torch.cuda.Event())
                    ev_comp[-1].record(s_comp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_comp[i])
                    for src, dst in zip(dout[b], hout[b]):
                        dst.copy_(src, non_blocking=True)
                    ev_out.append(torch.cuda.Event())
                    ev_out[-1].record(s_out)
            return ev_out

        run(nset)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        ev_last = run(e_steps)[-1]
        s_out.wait_event(ev_last)
        e1.record(s_out)
        torch.cuda.synchronize()
        fa.check_device_error()
        e_ms = max_over_ranks({"e2e": e0.elapsed_time(e1) / e_steps}, device=dev)["e2e"]
        e2e = {"value": job_tflops(world, f_fwd + f_bwd, e_ms), "unit": "TFLOP/s",
               "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "api": "exact_tiled_attention_31_b200.forward/backward (ctypes over libfa.so)",
               "pipelining": "copy-in of step i+1, compute of step i and copy-out of step i-1 on three streams, "
                             "device tensors double-buffered, the K timed steps (at most 100) in one pipeline; "
                             "every step's copies inside the timed region"}

    # ---- roofline of the dominant kernel
    pk, pk_kind = peaks()
    traffic = captured_traffic("bwd_main" if ms["bwd_main"] >= ms["fwd"] else "fwd")
    dominant = "bwd_main" if ms["bwd_main"] >= ms["fwd"] else "fwd"
    alg = f_bwd if dominant == "bwd_main" else f_fwd
    achieved = alg / (ms[dominant] * 1e-3) / 1e12
    roofline = {"kernel": "fa::bwd_main_kernel<128,bf16,causal>" if dominant == "bwd_main"
                else "fa::fwd_kernel<128,bf16,causal,dense>",
                "bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / pk["bf16_tflops"], "traffic": traffic,
                "peak_source": f"{pk_kind} bf16 dense burst (MEASURED_PEAKS.json bf16_tflops)"
                if pk_kind == "measured" else "fallback 1590 TFLOP/s (no MEASURED_PEAKS.json)",
                "algorithmic_flops_per_launch": alg, "ms_per_launch": ms[dominant]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        fl, sec, nh = oracle_sample(w, target_s=10.0)
        cpu = {"value": fl / sec / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
               "sample": f"fp64 fwd+bwd of {nh} of {B * H} heads (full S={S}), {sec:.1f} s"}

    decode = None
    if not args.no_decode:
        del flush
        decode = decode_leg(fa, inputs, torch, dev, stream, max(10, min(args.steps, 50)), args.warmup,
                            pk["hbm_gbs"], pk_kind)
        d_ms = max_over_ranks({"d": decode["ms_per_step"]}, device=dev)["d"]
        d_gbs = decode_bytes(DECODE) / (d_ms * 1e-3) / 1e9
        decode.update(ms_per_step=d_ms, value=d_gbs, tokens_per_s=DECODE["B"] / (d_ms * 1e-3), per="GPU (max over ranks)")
        decode["roofline"].update(achieved=d_gbs, frac=d_gbs / pk["hbm_gbs"])

    clocks = sampler.summary(clock_rows)
    sus_clocks = sampler.summary(clock_rows, sus_t0, sus_t1)
    warm = {"steps": len(warm_ev), "median_ms_per_step": warm_ms, "value": job_tflops(world, f_fwd + f_bwd, warm_ms),
            "unit": "TFLOP/s", "l2": "warm: steps back to back, no flush; median of 20"}
    sustained = {"steps": sus_n, "ms_per_step": sus_ms, "value": job_tflops(world, f_fwd + f_bwd, sus_ms),
                 "unit": "TFLOP/s", "l2": "not flushed (steps back to back)", "clocks": sus_clocks,
                 "ms_x_sm_mhz": sus_ms * (sus_clocks["sm_mhz"] or 0.0)}
    clocks["ms_x_sm_mhz"] = ms["step"] * (clocks["sm_mhz"] or 0.0)
    if rank == 0:
        out = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms["step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.workload, **w, "scale": scale, "seed": 42,
                       "l2": "flushed between timed steps (256 MiB write)",
                       "parallelism": f"replicas x{world} (independent heads, no data-path collective)"},
            "fwd_tflops": fwd_tf, "bwd_tflops": bwd_tf, "fwd_bwd_tflops": fb_tf,
            "fwd_pct_of_2250": 100 * fwd_tf / DATASHEET_TFLOPS, "bwd_pct_of_2250": 100 * bwd_tf / DATASHEET_TFLOPS,
            "fwd_bwd_pct_of_2250": 100 * fb_tf / DATASHEET_TFLOPS,
            "fwd_frac_of_measured": fwd_tf / pk["bf16_tflops"], "bwd_frac_of_measured": bwd_tf / pk["bf16_tflops"],
            "kernel_ms": ms, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches, "clocks": clocks, "warm_l2": warm, "sustained": sustained, "decode": decode,
        }
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
