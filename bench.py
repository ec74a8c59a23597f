"""Benchmark of the HyperQuant quantize+encode / decode path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

Default workload: the 4096 x 4096 bf16 lattice / rate sweep (N(0, 0.02^2) with
0.1 % x20 outliers, seed 1): 12 operating points {E8, D4, A2, Z} x {3, 4, 5}
bits per scalar, alpha and Rice k per point from tests/golden/rate_points.json.
One step = for every point, hq_quantize (quantize + encode) of the matrix and
hq_dequantize of the stream back to bf16: the whole weights path.  The 32 MiB
input fits in the 126 MB L2, so L2 is flushed (a 256 MiB write) before every
timed kernel and each kernel is timed alone with CUDA events on the stream it
runs on; the step time is the sum.

metric: GB/s of bf16 input through quantize+encode and decode (the value is the
round trip: input bytes / (encode time + decode time); each direction is also
reported), with MSE and bits per scalar per point.

Under torchrun (N > 1) every rank runs the same workload on its own GPU (the
path shards into independent tensors; no collective in the data path): weak
scaling, value = all ranks' bytes / the slowest rank's time.

--impl reference times the CPU oracle (plain C, tests' reference) on a bounded
sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

DEFAULT_WORKLOAD = "weight_4096x4096_rate_sweep"
L2_FLUSH_BYTES = 256 << 20
PROFILE_ENCODE = os.path.join(ROOT, "profiles", "encode_kernel_e8_4bps.md")
SM_COUNT, SMSP_PER_SM = 148, 4
FP32_FMA_PEAK = SM_COUNT * 128 * 1.965e9      # fp32 fma per second at the maximum SM clock


def rate_points():
    with open(os.path.join(ROOT, "tests", "golden", "rate_points.json")) as f:
        return json.load(f)["workloads"]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d["hbm_gbs"], "measured"
    return 6650.0, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in ("hq_encode.cuh", "hq_encode.cu", "hq_device.cuh", "hq_internal.h"):
        with open(os.path.join(ROOT, "lattice_entropy_coded_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_encode():
    """(DRAM bytes per launch, warp instructions per element) of the E8 4 bps encode
    launch from the committed ncu capture, or (None, None) if the kernel source has
    changed since it was taken."""
    if not os.path.exists(PROFILE_ENCODE):
        return None, None
    vals = {}
    with open(PROFILE_ENCODE) as f:
        for line in f:
            for key in ("kernel_source_hash", "traffic_bytes_per_launch", "warp_inst_per_element"):
                if line.startswith(key + ":"):
                    vals[key] = line.split(":", 1)[1].strip()
    if vals.get("kernel_source_hash") != kernel_source_hash():
        return None, None
    return float(vals["traffic_bytes_per_launch"]), float(vals["warp_inst_per_element"])


def reduce_max(values, device):
    """Element-wise max over ranks (identity without a process group)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def weak_scaling_value(bytes_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job GB/s: every rank processes bytes_per_rank; the job takes the slowest rank's time."""
    return world * bytes_per_rank / (max_ms * 1e6)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "100"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        mhz, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(mhz)}


# ------------------------------------------------------------------ workload
def make_points(workload: str):
    pts = rate_points()[workload]["points"]
    return pts


def run_ours(args, rank: int, world: int, device: torch.device):
    import lattice_entropy_coded_b200 as hq
    assert hq.hq_device_check() == hq.HQ_OK, "needs an sm_100 (B200) device"
    w = synth.WORKLOADS[args.workload]
    assert w["kind"] == "weight", "the default bench workload is a single weight matrix"
    rows, cols, seed = w["rows"], w["cols"], w["seed"]
    x = synth.weight(rows, cols, seed=seed, device=device)
    n = x.numel()
    pts = make_points(args.workload)
    stream = torch.cuda.current_stream(device)

    codecs = []
    for p in pts:
        params = hq.make_params(p["lattice"], p["alpha"], p["k"], seed, 0)
        cap = int(n * (p["bps"] + 3.0) / 32) + 8192
        codecs.append(hq.Codec(rows, cols, params, cap_words=cap, device=device))
    outs = [torch.empty(rows, cols, dtype=torch.bfloat16, device=device) for _ in pts]
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    def one_step(record):
        for i, c in enumerate(codecs):
            flush.fill_(float(i))
            e0, e1 = record()
            e0.record(stream)
            comp = c.quantize(x)
            e1.record(stream)
            flush.fill_(float(i) + 0.5)
            d0, d1 = record()
            d0.record(stream)
            c.dequantize(comp, outs[i])
            d1.record(stream)

    events = []

    def rec():
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        events.append((a, b))
        return a, b

    for _ in range(args.warmup):
        one_step(rec)
    torch.cuda.synchronize(device)
    events.clear()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            one_step(rec)
        t1.record(stream)
        torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    wall_ms = t0.elapsed_time(t1)
    ms = np.array([a.elapsed_time(b) for a, b in events]).reshape(args.steps, len(pts), 2)
    enc_ms = ms[:, :, 0].sum(1)      # per step
    dec_ms = ms[:, :, 1].sum(1)
    step_ms = enc_ms + dec_ms

    # per-point results (outside the timed region): rate and MSE of the bf16 reconstruction
    per_point = []
    xf = x.double()
    for i, (p, c) in enumerate(zip(pts, codecs)):
        st = hq.read_stats(c.stats)
        assert st["status"] == 0, (p, st)
        mse = float(((outs[i].double() - xf) ** 2).mean())
        words = int(c.offsets[-1].item())
        per_point.append(dict(lattice=p["lattice"], bps_target=p["bps"], k=p["k"], alpha=p["alpha"],
                              bps_payload=st["payload_bits"] / n, bps_stream=words * 32.0 / n,
                              bps_total=(words * 32.0 + 64.0 * (c.n_chunks + 1)) / n, mse=mse,
                              d_over_sigma2=mse / float(xf.var()),
                              enc_us=float(np.median(ms[:, i, 0]) * 1e3), dec_us=float(np.median(ms[:, i, 1]) * 1e3),
                              enc_gbs=2.0 * n / (np.median(ms[:, i, 0]) * 1e6),
                              dec_gbs=2.0 * n / (np.median(ms[:, i, 1]) * 1e6),
                              stream_words=words))

    # max over ranks of the summed kernel time
    step_sum, enc_sum, dec_sum, wall_max = reduce_max(
        [float(step_ms.sum()), float(enc_ms.sum()), float(dec_ms.sum()), wall_ms], device)
    in_bytes = 2.0 * n * len(pts)               # bf16 input bytes per step, per rank
    value = weak_scaling_value(in_bytes * args.steps, world, step_sum)
    enc_gbs = weak_scaling_value(in_bytes * args.steps, world, enc_sum)
    dec_gbs = weak_scaling_value(in_bytes * args.steps, world, dec_sum)

    # roofline of the dominant kernel: the encoder at the E8 4 bps point (the slowest launch of a step)
    peak, peak_kind = measured_peaks()
    clk = clk.summary()
    alg = [2.0 * n + 4.0 * pp["stream_words"] + 8.0 * (c.n_chunks + 1) for pp, c in zip(per_point, codecs)]
    enc_launch_ms = ms[:, :, 0].mean(0)
    dec_launch_ms = ms[:, :, 1].mean(0)
    e4 = [i for i, p in enumerate(per_point) if p["lattice"] == "E8" and p["bps_target"] == 4.0][0]
    hbm_achieved = alg[e4] / (enc_launch_ms[e4] * 1e6)
    traffic, inst_per_elem = profiled_encode()
    sm_mhz = clk["sm_mhz"] or 1965.0
    issue_peak = SM_COUNT * SMSP_PER_SM * sm_mhz * 1e6 / 1e9          # G warp-instructions / s
    roofline = {"kernel": "hq::encode_kernel<E8> at 4 bps (one launch, 4096x4096)",
                "bound": "alu", "unit": "Ginst/s",
                "achieved": None if inst_per_elem is None else round(inst_per_elem * n / (enc_launch_ms[e4] * 1e6), 1),
                "peak": round(issue_peak, 1),
                "frac": None if inst_per_elem is None else round(inst_per_elem * n / (enc_launch_ms[e4] * 1e6) / issue_peak, 4),
                "peak_kind": f"issue slots: {SM_COUNT} SMs x {SMSP_PER_SM} schedulers x 1 warp-instruction/cycle at the "
                             f"sampled {sm_mhz:.0f} MHz",
                "traffic": traffic,
                "hbm": {"achieved": round(hbm_achieved, 1), "peak": peak, "unit": "GB/s",
                        "frac": round(hbm_achieved / peak, 4),
                        "peak_kind": ("measured, MEASURED_PEAKS.json hbm_gbs (burst copy; kernels are timed alone)"
                                      if peak_kind == "measured" else "fallback 6.65 TB/s"),
                        "algorithmic_bytes": alg[e4]},
                "all_points": {"encode_hbm_achieved": round(float(np.sum(alg) / (np.sum(enc_launch_ms) * 1e6)), 1),
                               "decode_hbm_achieved": round(float(np.sum(alg) / (np.sum(dec_launch_ms) * 1e6)), 1),
                               "unit": "GB/s"}}

    # end to end through the C ABI with host buffers: H2D of the input, quantize+decode per point,
    # D2H of every reconstruction and stats block
    e2e = run_e2e(args, hq, codecs, pts, rows, cols, device, stream, world)

    return dict(value=value, enc_gbs=enc_gbs, dec_gbs=dec_gbs, ms_per_step=step_sum / args.steps,
                wall_ms_per_step=wall_max / args.steps, per_point=per_point, roofline=roofline,
                clocks=clk, e2e=e2e, launches=2 * len(pts) * args.steps, n=n, in_bytes=in_bytes)


def run_e2e(args, hq, codecs, pts, rows, cols, device, stream, world):
    n = rows * cols
    host_x = synth.weight(rows, cols, seed=synth.WORKLOADS[args.workload]["seed"]).pin_memory()
    host_out = [torch.empty(rows, cols, dtype=torch.bfloat16).pin_memory() for _ in pts]
    host_stats = [torch.empty(32, dtype=torch.uint8).pin_memory() for _ in pts]
    dev_x = torch.empty(rows, cols, dtype=torch.bfloat16, device=device)
    dev_out = [torch.empty(rows, cols, dtype=torch.bfloat16, device=device) for _ in pts]
    # device-to-host copies on their own stream, so point i's copy overlaps point i+1's codec work
    copy_stream = torch.cuda.Stream(device)
    done = [torch.cuda.Event() for _ in pts]

    def step():
        dev_x.copy_(host_x, non_blocking=True)
        for i, c in enumerate(codecs):
            comp = c.quantize(dev_x)
            c.dequantize(comp, dev_out[i])
            done[i].record(stream)
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(done[i])
                host_out[i].copy_(dev_out[i], non_blocking=True)
                host_stats[i].copy_(c.stats, non_blocking=True)
        # the step ends when its copies have landed (and the next step may reuse the buffers)
        stream.wait_stream(copy_stream)

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize(device)
    steps = max(1, min(args.steps, 5))
    if world > 1:
        torch.distributed.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(device)
    ms = reduce_max([t0.elapsed_time(t1)], device)[0]
    for i in range(len(pts)):
        assert hq.read_stats(host_stats[i])["status"] == 0
    in_bytes = 2.0 * n * len(pts)
    return {"value": round(weak_scaling_value(in_bytes * steps, world, ms), 3), "unit": "GB/s",
            "h2d_bytes_per_step": 2 * n, "d2h_bytes_per_step": len(pts) * (2 * n + 32),
            "steps": steps, "ms_per_step": round(ms / steps, 3)}


# ------------------------------------------------------------------ CPU oracle (baseline / reference arm)
def oracle_sample_rate(workload: str, rows_sample: int, threads: int, repeat: int = 1):
    """Oracle quantize+decode of the first rows_sample rows at every point, chunk ranges on
    `threads` host threads (ctypes releases the GIL).  -> (GB/s of bf16 input, seconds, elems)."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle as O
    w = synth.WORKLOADS[workload]
    x = synth.weight(w["rows"], w["cols"], seed=w["seed"])[:rows_sample].contiguous()
    xu = np.ascontiguousarray(x.view(torch.int16).numpy().view(np.uint16))
    R, Cc = xu.shape
    nch = O.n_chunks(R, Cc)
    step = max(1, -(-nch // threads))
    ranges = [(a, min(nch, a + step)) for a in range(0, nch, step)]
    pts = make_points(workload)
    O.lib()

    def job(r, p):
        lat = O.LATTICES[p["lattice"]]
        s, off, _ = O.quantize(xu, lat, p["alpha"], p["k"], w["seed"], 0, r[0], r[1])
        O.dequantize(s, off, R, Cc, lat, p["alpha"], p["k"], w["seed"], 0, False, r[0], r[1])

    t = time.perf_counter()
    with ThreadPoolExecutor(threads) as ex:
        for _ in range(repeat):
            list(ex.map(lambda a: job(*a), [(r, p) for p in pts for r in ranges]))
    dt = time.perf_counter() - t
    elems = R * Cc * len(pts) * repeat
    return 2.0 * elems / dt / 1e9, dt, elems


def kv_rotation_seed(workload_seed: int, tensor: str) -> int:
    """Seed of the dense rotation of the K or V cache of a rotated KV workload."""
    return 1000 * workload_seed + (0 if tensor == "K" else 1)


def oracle_workload(workload: str, threads: int, budget_s: float = 60.0, pts=None):
    """The CPU oracle's quantize+encode and decode over a workload's tensors, generated on the
    host, on `threads` threads (chunk ranges, or KV appends, in parallel), until `budget_s` of
    wall time per operating point is spent.  -> one dict per point; where the budget ran out
    first, the rate is over the tensors done and `extrapolated` is true.  pts: the operating
    points (default: the stored ones)."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle as O
    from oracle import rotation as ORot
    w = synth.WORKLOADS[workload]
    pts = rate_points()[workload if workload in rate_points() else w["points_of"]]["points"] if pts is None else pts
    O.lib()

    def u16(t):
        return np.ascontiguousarray(t.contiguous().view(torch.int16).numpy().view(np.uint16))

    def tensors():
        if w["kind"] == "weight":
            yield synth.weight(w["rows"], w["cols"], w["seed"])
        elif w["kind"] == "weight_set":
            for _, m in synth.weight_set(w["seed"], layers=w["layers"]):
                yield m
        elif w["kind"] == "student_t":
            yield from synth.student_t(w["n"], w["rows"], w["cols"], w["seed"])
        else:
            K, V = synth.kv(w["heads"], w["tokens"], w["seed"])
            yield {"K": K, "V": V}

    total = {"weight": w.get("rows", 0) * w.get("cols", 0), "weight_set": synth.weight_set_elems(w.get("layers", 8)),
             "student_t": w.get("n", 0) * w.get("rows", 0) * w.get("cols", 0),
             "kv": w.get("heads", 0) * w.get("tokens", 0) * 128}[w["kind"]]
    out = []
    with ThreadPoolExecutor(threads) as ex:
        for p in pts:
            lat = O.LATTICES[p["lattice"]]
            busy, elems, t_start = 0.0, 0, time.perf_counter()
            for t in tensors():
                if w["kind"] == "kv":
                    xu = u16(t[p["tensor"]])
                    H, T, _ = xu.shape
                    A = w["append"]
                    dec = np.zeros((H, T, 128), np.uint16)     # appends write disjoint token ranges
                    rot = (ORot.haar_rotation(kv_rotation_seed(w["seed"], p["tensor"])) if w.get("rotation")
                           else None)

                    def job(t0, xu=xu, H=H, T=T, A=A, dec=dec, rot=rot):
                        blk = np.ascontiguousarray(xu[:, t0:t0 + A])
                        s_, off, _ = O.kv_append(blk, t0, lat, p["alpha"], p["k"], w["seed"], 1, rot=rot)
                        O.kv_read_append(s_, off, H, blk.shape[1], t0, lat, p["alpha"], p["k"], w["seed"], 1, dec, T,
                                         rot=rot)
                    jobs = list(range(0, T, A))
                    n_el = xu.size
                else:
                    xu = u16(t)
                    R, Cc = xu.shape
                    nch = O.n_chunks(R, Cc)
                    step = max(1, -(-nch // threads))
                    jobs = [(a, min(nch, a + step)) for a in range(0, nch, step)]

                    def job(r, xu=xu, R=R, Cc=Cc):
                        dk = p.get("dk_last", 0)
                        s_, off, _ = O.quantize(xu, lat, p["alpha"], p["k"], w["seed"], 0, r[0], r[1], dk_last=dk)
                        O.dequantize(s_, off, R, Cc, lat, p["alpha"], p["k"], w["seed"], 0, False, r[0], r[1], dk_last=dk)
                    n_el = xu.size
                t0 = time.perf_counter()
                list(ex.map(job, jobs))
                busy += time.perf_counter() - t0
                elems += n_el
                if time.perf_counter() - t_start > budget_s:
                    break
            out.append({"lattice": p["lattice"], "bps_target": p["bps"], "tensor": p.get("tensor"),
                        "gbs": round(2.0 * elems / busy / 1e9, 4), "seconds": round(busy, 2), "elements": elems,
                        "of_elements": total, "extrapolated": elems < total, "threads": threads})
    return out


def host_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(workload: str):
    threads = host_threads()
    rows = min(4096, max(256, 128 * threads))
    gbs, dt, elems = oracle_sample_rate(workload, rows, threads)
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"rows 0..{rows - 1} of the 4096x4096 matrix at all 12 points, quantize+encode and "
                      f"decode ({elems} elements per direction, {dt:.1f} s wall on {threads} threads)"}


def run_reference(args):
    threads = host_threads()
    rows = max(32, min(1024, 32 * threads))
    for _ in range(args.warmup):
        oracle_sample_rate(args.workload, rows, threads)
    gbs, dt, elems = oracle_sample_rate(args.workload, rows, threads, repeat=args.steps)
    base = {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"rows 0..{rows - 1} of the 4096x4096 matrix at all 12 points per step, quantize+encode and "
                      f"decode, {args.steps} steps ({dt:.1f} s wall on {threads} threads)"}
    return {"metric": "quantize+encode / decode GB/s of bf16 input vs B200 HBM peak; MSE at bps",
            "value": base["value"], "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt * 1e3 / args.steps, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic", "impl": "reference",
            "config": {"workload": args.workload, "rows": 4096, "cols": 4096, "points": 12,
                       "sample_rows": rows, "parallelism": "host threads"},
            "cpu_baseline": base,
            "e2e": {"value": base["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------ the other workloads
def _events():
    return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)


def run_bulk(args):
    """Time one of the other workloads end to end on the device (inputs resident in HBM,
    larger than L2, launches back to back on one stream); prints one JSON line."""
    import lattice_entropy_coded_b200 as hq
    device = torch.device("cuda", 0)
    wl = args.workload
    w = synth.WORKLOADS[wl]
    out = {"workload": wl, "steps": args.steps, "warmup": args.warmup}
    peak, _ = measured_peaks()
    if w["kind"] == "kv":
        H, T, A = w["heads"], w["tokens"], w["append"]
        K, V = synth.kv(H, T, w["seed"], device=device)
        flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=device)
        rots = {}
        if w.get("rotation"):
            # a dense Haar rotation per tensor, drawn on the device; alpha and k for each rate
            # calibrated on the device over the whole tensor (untimed setup)
            pts = []
            for name, src in (("K", K), ("V", V)):
                rots[name] = hq.hq_haar_rotation(kv_rotation_seed(w["seed"], name))
                for bps in (2.0, 1.7):
                    pr = hq.make_params("E8", 1.0, 0, w["seed"], 1, rotation=rots[name])
                    cal = hq.hq_calibrate_kv(src, pr, hq.calib_spec(bps, tol=0.002, k_lo=0, k_hi=4),
                                             hq.stats_tensor(device))
                    pts.append({"tensor": name, "lattice": "E8", "bps": bps, "alpha": cal["alpha"], "k": cal["k"]})
        else:
            pts = rate_points()[wl]["points"]
        res = []
        for p in pts:
            src = K if p["tensor"] == "K" else V
            rot = rots.get(p["tensor"])
            params = hq.make_params("E8", 1.0, p["k"], w["seed"], 1)
            if rot is not None:
                params.rotation = rot.data_ptr()
            cache = hq.KVCache(H, T, params, bits_per_scalar=p["bps"] + 4.0, max_appends=T // A + 1,
                               max_append_tokens=A, device=device, rotation=rot)
            slices = [src[:, t:t + A] for t in range(0, T, A)]
            outb = torch.empty(H, T, 128, dtype=torch.bfloat16, device=device)
            app_ms, read_ms = [], []
            for it in range(args.warmup + args.steps):
                flush.fill_(it)   # the K (or V) tensor fits in L2: evict it before each step
                hq.hq_kv_init(cache.cache, H, 128, params, cache.words, cache.offsets, cache.table, cache.tail,
                              cache.stats)
                a0, a1 = _events()
                a0.record()
                for sl in slices:
                    cache.append(sl, p["alpha"])
                a1.record()
                r0, r1 = _events()
                r0.record()
                cache.read(outb)
                r1.record()
                torch.cuda.synchronize()
                if it >= args.warmup:
                    app_ms.append(a0.elapsed_time(a1))
                    read_ms.append(r0.elapsed_time(r1))
            st = hq.read_stats(cache.stats)
            n = src.numel()
            words = int(cache.tail[(len(slices)) & 1].item())
            # attention scores of 4 query heads per KV head straight from the compressed cache,
            # against reading the cache to bf16 and multiplying
            G = 4
            qh = (torch.randn(H * G, 128, device=device) * 0.1).to(torch.bfloat16)
            sc = torch.empty(H * G, T, device=device)
            sc_ms, rd_ms = [], []
            for it in range(args.warmup + args.steps):
                flush.fill_(it)
                s0, s1 = _events()
                s0.record()
                cache.scores(qh, G, sc)
                s1.record()
                flush.fill_(it + 0.5)
                r0, r1 = _events()
                r0.record()
                cache.read(outb)
                torch.matmul(outb.float(), qh.view(H, G, 128).float().transpose(1, 2))
                r1.record()
                torch.cuda.synchronize()
                if it >= args.warmup:
                    sc_ms.append(s0.elapsed_time(s1))
                    rd_ms.append(r0.elapsed_time(r1))
            # the same appends captured once in a CUDA graph and replayed: device time
            # without the per-call host work (Python, argument checks, launch calls)
            graph = torch.cuda.CUDAGraph()
            hq.hq_kv_init(cache.cache, H, 128, params, cache.words, cache.offsets, cache.table, cache.tail,
                          cache.stats)
            with torch.cuda.graph(graph):
                for sl in slices:
                    cache.append(sl, p["alpha"])
            graph_ms = []
            for it in range(args.warmup + args.steps):
                flush.fill_(it)
                hq.hq_kv_init(cache.cache, H, 128, params, cache.words, cache.offsets, cache.table, cache.tail,
                              cache.stats)
                g0, g1 = _events()
                g0.record()
                graph.replay()
                g1.record()
                torch.cuda.synchronize()
                if it >= args.warmup:
                    graph_ms.append(g0.elapsed_time(g1))
            graph_words = int(cache.tail[(len(slices)) & 1].item())
            del graph
            # one append of all T tokens at once (a prefill: H * T / 32 chunks in one launch)
            pre = hq.KVCache(H, T, params, bits_per_scalar=p["bps"] + 4.0, max_appends=2, max_append_tokens=T,
                             device=device, rotation=rot)
            pre_ms = []
            for it in range(args.warmup + args.steps):
                flush.fill_(it)
                hq.hq_kv_init(pre.cache, H, 128, params, pre.words, pre.offsets, pre.table, pre.tail, pre.stats)
                p0, p1 = _events()
                p0.record()
                pre.append(src, p["alpha"])
                p1.record()
                torch.cuda.synchronize()
                if it >= args.warmup:
                    pre_ms.append(p0.elapsed_time(p1))
            pre_words = int(pre.tail[1].item())
            del pre
            # decode steps: 128 appends of one token each (8 one-tile chunks per launch), captured
            # once in a CUDA graph and replayed; the time per append is the per-token latency
            one = hq.KVCache(H, 128, params, bits_per_scalar=p["bps"] + 8.0, max_appends=129, max_append_tokens=1,
                             device=device, rotation=rot)
            toks = [src[:, t:t + 1] for t in range(128)]
            hq.hq_kv_init(one.cache, H, 128, params, one.words, one.offsets, one.table, one.tail, one.stats)
            g1 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g1):
                for tk in toks:
                    one.append(tk, p["alpha"])
            one_ms = []
            for it in range(args.warmup + args.steps):
                hq.hq_kv_init(one.cache, H, 128, params, one.words, one.offsets, one.table, one.tail, one.stats)
                o0, o1 = _events()
                o0.record()
                g1.replay()
                o1.record()
                torch.cuda.synchronize()
                if it >= args.warmup:
                    one_ms.append(o0.elapsed_time(o1))
            one_status = hq.read_stats(one.stats)["status"]
            del g1, one
            mse = float(((outb.double() - src.double()) ** 2).mean())
            am, rm = float(np.median(app_ms)), float(np.median(read_ms))
            alg = 2.0 * n + 4.0 * words + 8.0 * (cache.cache.chunks + 1)
            res.append(dict(tensor=p["tensor"], bps_target=p["bps"], k=p["k"], alpha=p["alpha"], status=st["status"],
                            bps_payload=st["payload_bits"] / n, bps_stream=words * 32.0 / n, mse=mse,
                            d_over_sigma2=mse / float(src.double().var()), appends=len(slices),
                            append_ms=am, read_ms=rm, append_gbs=2.0 * n / (am * 1e6), read_gbs=2.0 * n / (rm * 1e6),
                            graph_append_ms=float(np.median(graph_ms)),
                            graph_append_gbs=2.0 * n / (float(np.median(graph_ms)) * 1e6),
                            graph_stream_words_match=graph_words == words,
                            prefill_append_ms=float(np.median(pre_ms)),
                            prefill_append_gbs=2.0 * n / (float(np.median(pre_ms)) * 1e6),
                            prefill_stream_words=pre_words,
                            token_append_us=float(np.median(one_ms)) * 1e3 / 128, token_append_status=one_status,
                            # with a dense rotation: the rotation's 128 fp32 fma per element (forward
                            # in the append, inverse in the read) against the fp32 fma peak of
                            # 148 SMs x 128 lanes at the 1965 MHz maximum clock
                            **({"prefill_rotation_fma_frac": 128.0 * n / (float(np.median(pre_ms)) * 1e-3) /
                                FP32_FMA_PEAK,
                                "read_rotation_fma_frac": 128.0 * n / (rm * 1e-3) / FP32_FMA_PEAK} if rot is not None
                               else {}),
                            scores_ms=float(np.median(sc_ms)), read_then_matmul_ms=float(np.median(rd_ms)),
                            scores_query_heads=H * G,
                            append_hbm_frac=alg / (am * 1e6) / peak, read_hbm_frac=alg / (rm * 1e6) / peak))
        out["points"] = res
        if rots:
            out["rotation"] = "Haar-uniform 128x128 per tensor (hq_haar_rotation), alpha/k calibrated on the device"
    else:
        pts = rate_points()[wl if wl in rate_points() else w["points_of"]]["points"]
        if w["kind"] == "weight":
            mats = [synth.weight(w["rows"], w["cols"], w["seed"], device=device)]
        elif w["kind"] == "weight_set":
            mats = [m for _, m in synth.weight_set(w["seed"], device=device, layers=w["layers"])]
        else:
            mats = list(synth.student_t(w["n"], w["rows"], w["cols"], w["seed"], device=device))
        n = sum(m.numel() for m in mats)
        if w.get("dk_last"):
            # a second Rice parameter for the last symbol of each block: alpha and k for each
            # target rate calibrated on the device in that mode (untimed); each is timed next to
            # the single-parameter point of the same rate, the same way
            big = torch.cat(mats, dim=0)
            cal_pts = []
            for p in pts:
                dk = w["dk_last"][p["lattice"]]
                cal_pts.append(dict(p, dk_last=0))
                if dk:
                    c = hq.hq_calibrate(big, hq.make_params(p["lattice"], 1.0, 0, w["seed"], 0, dk_last=dk),
                                        hq.calib_spec(p["bps"], tol=0.002, k_lo=0, k_hi=6), hq.stats_tensor(device))
                    cal_pts.append(dict(p, alpha=c["alpha"], k=c["k"], dk_last=dk))
            pts = cal_pts
            del big
        # inputs that fit in L2 are evicted before each step (a buffer larger than L2 is written)
        flush = (torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=device)
                 if 2 * n < L2_FLUSH_BYTES else None)
        res = []
        for p in pts:
            params = hq.make_params(p["lattice"], p["alpha"], p["k"], w["seed"], 0, dk_last=p.get("dk_last", 0))
            codecs = [hq.Codec(m.shape[0], m.shape[1], params, device=device,
                               cap_words=int(m.numel() * (p["bps"] + 3.0) / 32) + 8192) for m in mats]
            outs = [torch.empty_like(m) for m in mats]
            enc_ms, dec_ms = [], []
            for it in range(args.warmup + args.steps):
                if flush is not None:
                    flush.fill_(it)
                e0, e1 = _events()
                e0.record()
                comps = [c.quantize(m) for c, m in zip(codecs, mats)]
                e1.record()
                if flush is not None:
                    flush.fill_(it + 1)
                d0, d1 = _events()
                d0.record()
                for c, cp, o in zip(codecs, comps, outs):
                    c.dequantize(cp, o)
                d1.record()
                torch.cuda.synchronize()
                if it >= args.warmup:
                    enc_ms.append(e0.elapsed_time(e1))
                    dec_ms.append(d0.elapsed_time(d1))
            stats = [hq.read_stats(c.stats) for c in codecs]
            words = sum(int(c.offsets[-1].item()) for c in codecs)
            nch = sum(c.n_chunks + 1 for c in codecs)
            se = sum(float(((o.double() - m.double()) ** 2).sum()) for o, m in zip(outs, mats))
            var = sum(float(m.double().var()) * m.numel() for m in mats) / n
            em, dm = float(np.median(enc_ms)), float(np.median(dec_ms))
            alg = 2.0 * n + 4.0 * words + 8.0 * nch
            res.append(dict(lattice=p["lattice"], bps_target=p["bps"], k=p["k"], alpha=p["alpha"],
                            status=max(st["status"] for st in stats),
                            bps_payload=sum(st["payload_bits"] for st in stats) / n, bps_stream=words * 32.0 / n,
                            mse=se / n, d_over_sigma2=se / n / var, matrices=len(mats), elements=n,
                            encode_ms=em, decode_ms=dm, encode_gbs=2.0 * n / (em * 1e6), decode_gbs=2.0 * n / (dm * 1e6),
                            encode_hbm_frac=alg / (em * 1e6) / peak, decode_hbm_frac=alg / (dm * 1e6) / peak,
                            **({"dk_last": p["dk_last"]} if "dk_last" in p else {})))
            del codecs, outs, comps
            torch.cuda.empty_cache()
        out["points"] = res
        if w["kind"] == "student_t":
            out["calibration"] = calibrate_set(hq, mats, pts, w["seed"])
    if args.oracle:
        threads = host_threads()
        out["oracle"] = {"threads": threads,
                         "points": oracle_workload(wl, threads,
                                                   pts=pts if (w["kind"] == "kv" or w.get("dk_last")) else None)}
        if w["kind"] == "weight":
            out["oracle"]["single_thread"] = oracle_workload(wl, 1, pts=pts if w.get("dk_last") else None)
    print(json.dumps(out), flush=True)


def calibrate_set(hq, mats, pts, seed):
    """alpha and k for every rate point of a matrix set, chosen on the device over the
    whole set (one contiguous tensor), with the time it takes and one rate pass's time."""
    big = torch.cat(mats, dim=0)
    st = hq.stats_tensor(big.device)
    res = []
    for p in pts:
        params = hq.make_params(p["lattice"], p["alpha"], p["k"], seed, 0)
        e0, e1 = _events()
        e0.record()
        hq.hq_rate(big, params, st)
        e1.record()
        torch.cuda.synchronize()
        pass_ms = e0.elapsed_time(e1)
        r = hq.read_stats(st)
        t0 = time.perf_counter()
        c = hq.hq_calibrate(big, hq.make_params(p["lattice"], 1.0, 0, seed, 0), hq.calib_spec(p["bps"], k_lo=0, k_hi=6),
                            st)
        wall = time.perf_counter() - t0
        res.append(dict(lattice=p["lattice"], bps_target=p["bps"], elements=big.numel(),
                        rate_pass_ms=pass_ms, rate_pass_gbs=2.0 * big.numel() / (pass_ms * 1e6),
                        bps_at_sample_alpha=r["payload_bits"] / big.numel(),
                        sample_alpha=p["alpha"], sample_k=p["k"], calibrated_alpha=c["alpha"], calibrated_k=c["k"],
                        calibrated_bps=c["bps"], evaluations=c["evaluations"], calibrate_wall_s=wall))
    del big
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------ single-matrix case (profiling)
def run_case(args):
    """Quantize + decode one R x C synthetic weight matrix (seed 1) at one operating point of
    the rate sweep, back to back, no L2 flush: the small case the ncu captures run on."""
    import lattice_entropy_coded_b200 as hq
    rows, cols = (int(v) for v in args.case.lower().split("x"))
    p = [q for q in rate_points()[DEFAULT_WORKLOAD]["points"]
         if q["lattice"] == args.lattice and q["bps"] == args.bps][0]
    device = torch.device("cuda", 0)
    x = synth.weight(rows, cols, seed=1, device=device)
    params = hq.make_params(p["lattice"], p["alpha"], p["k"], 1, args.dither)
    codec = hq.Codec(rows, cols, params, cap_words=int(x.numel() * (p["bps"] + 3.0) / 32) + 8192, device=device)
    out = torch.empty(rows, cols, dtype=torch.bfloat16, device=device)
    ev = []
    for i in range(args.warmup + args.steps):
        a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        a.record()
        comp = codec.quantize(x)
        b.record()
        codec.dequantize(comp, out)
        c.record()
        if i >= args.warmup:
            ev.append((a, b, c))
    # decode fused into a GEMV vs decode then GEMV vs a plain bf16 GEMV on the uncompressed matrix
    comp = codec.quantize(x)
    xv = (torch.randn(cols, device=device) * 0.5).to(torch.bfloat16)
    y = torch.empty(rows, device=device)
    gev = {"fused": [], "decode_then_gemv": [], "bf16_gemv": []}
    for i in range(args.warmup + args.steps):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        evs[0].record()
        codec.gemv(comp, xv, y)
        evs[1].record()
        evs[2].record()
        codec.dequantize(comp, out)
        torch.mv(out, xv)
        evs[3].record()
        evs[4].record()
        torch.mv(x, xv)
        evs[5].record()
        if i >= args.warmup:
            gev["fused"].append((evs[0], evs[1]))
            gev["decode_then_gemv"].append((evs[2], evs[3]))
            gev["bf16_gemv"].append((evs[4], evs[5]))
    rst = hq.stats_tensor(device)
    rev = []
    for i in range(args.warmup + args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        hq.hq_rate(x, params, rst)
        b.record()
        if i >= args.warmup:
            rev.append((a, b))
    torch.cuda.synchronize()
    st = hq.read_stats(codec.stats)
    rate_ms = float(np.median([a.elapsed_time(b) for a, b in rev]))
    gemv_ms = {k: float(np.median([a.elapsed_time(b) for a, b in v])) for k, v in gev.items()}
    assert hq.read_stats(rst)["payload_bits"] == st["payload_bits"]
    enc = float(np.median([a.elapsed_time(b) for a, b, _ in ev]))
    dec = float(np.median([b.elapsed_time(c) for _, b, c in ev]))
    n = x.numel()
    words = int(codec.offsets[-1].item())
    alg = 2.0 * n + 4.0 * words + 8.0 * (codec.n_chunks + 1)
    peak, _ = measured_peaks()
    print(json.dumps({"case": args.case, "lattice": p["lattice"], "bps": p["bps"], "dither": args.dither,
                      "status": st["status"], "bps_payload": st["payload_bits"] / n,
                      "enc_ms": enc, "dec_ms": dec, "enc_gbs_in": 2.0 * n / enc / 1e6, "dec_gbs_in": 2.0 * n / dec / 1e6,
                      "enc_frac": alg / enc / 1e6 / peak, "dec_frac": alg / dec / 1e6 / peak,
                      "alg_bytes": alg, "rate_ms": rate_ms, "rate_gbs_in": 2.0 * n / rate_ms / 1e6,
                      "gemv_ms": gemv_ms,
                      "gemv_read_bytes": {"fused": 4.0 * words + 8.0 * (codec.n_chunks + 1) + 2.0 * cols,
                                          "bf16_gemv": 2.0 * n + 2.0 * cols}}), flush=True)


def run_token_case(args):
    """One-token KV appends, as a decode step makes them: 8 heads, E8 with dither at the K 2.0 bps
    point of the 8-head KV workload; 128 appends replayed from a CUDA graph, then the same appends
    as plain calls.  Prints the device time per append.  The small case the ncu capture of the
    one-token encoder runs on."""
    import lattice_entropy_coded_b200 as hq
    wl = "kv_8h_32768tok_e8_dither"
    w = synth.WORKLOADS[wl]
    H = w["heads"]
    p = [q for q in rate_points()[wl]["points"] if q["tensor"] == "K" and q["bps"] == 2.0][0]
    device = torch.device("cuda", 0)
    K, _ = synth.kv(H, 128, seed=w["seed"], device=device)
    params = hq.make_params("E8", 1.0, p["k"], w["seed"], 1)
    one = hq.KVCache(H, 128, params, bits_per_scalar=p["bps"] + 8.0, max_appends=129, max_append_tokens=1,
                     device=device)
    toks = [K[:, t:t + 1].contiguous() for t in range(128)]
    # plain calls first (these are the launches an ncu capture sees), then the graph
    for _ in range(args.warmup):
        hq.hq_kv_init(one.cache, H, 128, params, one.words, one.offsets, one.table, one.tail, one.stats)
        for tk in toks:
            one.append(tk, p["alpha"])
    torch.cuda.synchronize()
    hq.hq_kv_init(one.cache, H, 128, params, one.words, one.offsets, one.table, one.tail, one.stats)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for tk in toks:
            one.append(tk, p["alpha"])
    ms = []
    for it in range(args.warmup + args.steps):
        hq.hq_kv_init(one.cache, H, 128, params, one.words, one.offsets, one.table, one.tail, one.stats)
        a, b = _events()
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        if it >= args.warmup:
            ms.append(a.elapsed_time(b))
    st = hq.read_stats(one.stats)
    del g
    print(json.dumps({"case": "kv one-token appends", "heads": H, "appends": 128, "k": p["k"], "alpha": p["alpha"],
                      "status": st["status"], "bps_payload": st["payload_bits"] / (H * 128 * 128),
                      "token_append_us": float(np.median(ms)) * 1e3 / 128}), flush=True)


# ------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--oracle", action="store_true",
                    help="with --workload: also time the CPU oracle on the workload (about a minute per point)")
    ap.add_argument("--case", default=None, help="RxC: time one matrix (profiling case)")
    ap.add_argument("--token-case", action="store_true", help="time one-token KV appends (profiling case)")
    ap.add_argument("--lattice", default="E8")
    ap.add_argument("--bps", type=float, default=4.0)
    ap.add_argument("--dither", type=int, default=0)
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.case:
        run_case(args)
        return
    if args.token_case:
        run_token_case(args)
        return
    if args.workload != DEFAULT_WORKLOAD and args.impl == "ours":
        run_bulk(args)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    try:
        r = run_ours(args, rank, world, device)
        if rank == 0:
            line = {
                "metric": "quantize+encode / decode GB/s of bf16 input vs B200 HBM peak; MSE at bps",
                "value": round(r["value"], 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(r["ms_per_step"], 4), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": {"workload": args.workload, "rows": 4096, "cols": 4096, "dtype_in": "bf16",
                           "points": "E8,D4,A2,Z x 3,4,5 bps", "step": "12 x (hq_quantize + hq_dequantize bf16)",
                           "l2": "flushed (256 MiB write) before every timed kernel; kernels timed alone",
                           "parallelism": f"independent replicas x{world}" if world > 1 else "single GPU"},
                "quantize_encode_gbs": round(r["enc_gbs"], 2), "decode_gbs": round(r["dec_gbs"], 2),
                "roofline": r["roofline"], "clocks": r["clocks"], "e2e": r["e2e"], "gpu_launches": r["launches"],
                "points": r["per_point"],
            }
            if not args.no_cpu_baseline and world == 1:   # the oracle is timed at N = 1 only
                line["cpu_baseline"] = cpu_baseline(args.workload)
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
