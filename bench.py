"""Benchmark of the streaming-frame step (3D RoPE + paged KV append + paged attention).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config C]

One step streams every frame of the workload through a fresh cache: per frame one
lbm_append_frame (fused rotate + append: q rotated in place, k and v into the pages) and one
lbm_attend_frame (paged attention on persistent CTAs, plus the combine of the units several
CTAs share), host page-table bookkeeping included.  (Folding the rotation of q into the
attention instead, lbm_append_frame with q = NULL, moves a third fewer bytes in the append
but costs the attention more than that saves at these sizes, so it is not what is timed.)  The default workload is the 4096-patch stream (configuration 4):
8 heads x head_dim 128, bf16, 6 special + 64x64 patch tokens per frame, 96 keyframes,
scale_frames 4, sliding_window 32.  Inputs are seeded synthetic frames held in HBM before
timing; a pool of up to 64 distinct frames (1.6 GB here) is larger than L2, so no input is
L2-resident when a frame reads it.

The same invocation (N = 1) also measures the 999-patch streams (configurations 2 and 3:
keyframe every 5th frame over 320 frames, and 2000 keyframes) and reports their attention
and append roofline fractions under "other_configs", each with its own clock summary.

With N > 1 (torchrun) every rank streams its own independent copy of the headline workload
(the step has no exchange between GPUs): weak scaling, value = all ranks' frames / max rank
time.

Prints one JSON line (rank 0).  ``--impl reference`` times the fp64 CPU oracle on this
host's cores on a bounded sample of the same workload instead.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

INPUT_POOL = 64
HEADLINE_CONFIG = 4
OTHER_CONFIGS = (2, 3)
METRIC = "streamed frames/s per layer (RoPE+append+paged attn); % of bf16 TC / HBM peak"
UNIT = "frames/s"
# ncu summaries whose DRAM bytes per attention launch give roofline.traffic (per config)
TRAFFIC_PROFILES = {4: "attn_tc_large4096.md", 1: "attn_tc_stream768.md"}


FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def _peak_number(d, key):
    """The number stored under key in the peaks file: a plain number, or a record holding one
    (value / median / mean), at the top level or inside a nested record; None if absent."""
    def as_num(v):
        if isinstance(v, bool):
            return None
        if isinstance(v, (int, float)):
            return float(v)
        if isinstance(v, dict):
            for k in ("value", "median", "mean"):
                if isinstance(v.get(k), (int, float)) and not isinstance(v.get(k), bool):
                    return float(v[k])
        return None
    if not isinstance(d, dict):
        return None
    if key in d and as_num(d[key]) is not None:
        return as_num(d[key])
    for v in d.values():
        r = _peak_number(v, key) if isinstance(v, dict) else None
        if r is not None:
            return r
    return None


def _peaks(path=None):
    """Roofline denominators: MEASURED_PEAKS.json when it holds them, else the fallback figures
    (a figure missing from the file falls back alone, and the source says so)."""
    path = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(path):
        return dict(FALLBACK_PEAKS, source="fallback")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError) as e:
        return dict(FALLBACK_PEAKS, source=f"fallback (MEASURED_PEAKS.json unreadable: {e})")
    out, missing = {}, []
    for key in ("hbm_gbs", "bf16_tflops"):
        v = _peak_number(d, key)
        if v is None or v <= 0:
            missing.append(key)
            v = FALLBACK_PEAKS[key]
        out[key] = v
    sus = _peak_number(d, "bf16_tflops_sustained")
    if sus and sus > 0:
        out["bf16_tflops_sustained"] = sus
    elif "bf16_tflops" in missing:
        out["bf16_tflops_sustained"] = FALLBACK_PEAKS["bf16_tflops_sustained"]
    else:
        out["bf16_tflops_sustained"] = out["bf16_tflops"]
    out["source"] = "measured" if not missing else "measured (fallback for " + ", ".join(missing) + ")"
    return out


def tensor_peak(peaks: dict, clocks: dict) -> tuple[float, str]:
    """The bf16 peak the attention is compared with: the sustained (power-capped) figure when
    the clocks sampled during the timed region show the power cap, else the burst figure."""
    if "sw_power_cap" in (clocks.get("reasons") or []):
        return peaks["bf16_tflops_sustained"], (peaks["source"] + " bf16_tflops_sustained "
                                                "(sw_power_cap seen during the timed region)")
    return peaks["bf16_tflops"], peaks["source"] + " bf16_tflops (burst; no power cap seen)"


def measured_traffic(cid: int, avg_keys: float):
    """DRAM bytes per attention launch from the committed ncu summary of this workload,
    scaled from the captured frame's key count to the stream's average (K/V reads dominate
    and grow with the keys); None when there is no summary or the kernel source differs from
    the one that was profiled."""
    import hashlib
    name = TRAFFIC_PROFILES.get(cid)
    if name is None:
        return None
    prof = os.path.join(ROOT, "profiles", name)
    src = os.path.join(ROOT, "rope_paged_kv_02_b200", "csrc", "attn_tc.cu")
    if not os.path.exists(prof):
        return None
    fields = {}
    for line in open(prof):
        if ":" in line and not line.startswith("|"):
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if fields.get("kernel_source_sha256_16") != sha:
        return None
    try:
        return float(fields["traffic_bytes_per_launch"]) * avg_keys / float(
            fields["algorithmic_keys_of_capture"])
    except (KeyError, ValueError):
        return None


def frame_work(cfg, n_frames: int | None = None):
    """Algorithmic work per frame of a stream: (attention FLOPs, append bytes, keys seen).

    Frame n with m keyframes committed before it sees min(m, S+W)+1 patch pages and 6(m+1)
    special tokens; attention = 4 T N_k H D flops (QK^T and PV); append moves 6 T H D e bytes
    (read q, k, v; write q rotated in place, k and v into the pages).
    """
    T, H, D, e = cfg.tokens, cfg.heads, cfg.head_dim, cfg.elem_bytes
    flops, nbytes, keys = [], [], []
    m = 0
    for key in cfg.keyframes[:n_frames]:
        nk = (min(m, cfg.scale_frames + cfg.sliding_window) + 1) * cfg.patches + 6 * (m + 1)
        flops.append(4.0 * T * nk * H * D)
        nbytes.append(6.0 * T * H * D * e)
        keys.append(nk)
        if key:
            m += 1
    return np.array(flops), np.array(nbytes), np.array(keys)


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = self.smi_id(device_index)
        self.proc = None
        self.lines = []

    @staticmethod
    def smi_id(device_index: int) -> str:
        """nvidia-smi's name for CUDA device device_index: its UUID or PCI bus id (the CUDA
        ordinal and nvidia-smi's index differ under CUDA_VISIBLE_DEVICES), checked by one
        query; the ordinal itself when neither answers."""
        cands = []
        try:
            import torch
            if torch.cuda.is_available():
                pr = torch.cuda.get_device_properties(device_index)
                u = str(getattr(pr, "uuid", "") or "")
                if u:
                    cands.append(u if u.startswith("GPU-") else "GPU-" + u)
                cands.append("%08X:%02X:%02X.0" % (pr.pci_domain_id, pr.pci_bus_id,
                                                   pr.pci_device_id))
        except Exception:
            pass
        for c in cands:
            try:
                r = subprocess.run(["nvidia-smi", f"--id={c}", "--query-gpu=index",
                                    "--format=csv,noheader"], capture_output=True, text=True,
                                   timeout=20)
                if r.returncode == 0 and r.stdout.strip():
                    return c
            except (OSError, subprocess.SubprocessError):
                break
        return str(device_index)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0,
                    "gpu": self.idx}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "gpu": self.idx}


def dist_setup(n_gpus: int):
    """Rank, world size and local rank; initialises the process group for N > 1."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------------------------------
# the fp64 oracle on the host cores (reference arm and cpu_baseline)
# ------------------------------------------------------------------------------------------

def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def _busiest_frame(cfg) -> int:
    """First frame that sees the stream's largest number of patch pages (steady state)."""
    m, best, first = 0, -1, 0
    for f, key in enumerate(cfg.keyframes):
        n_pages = min(m, cfg.scale_frames + cfg.sliding_window) + 1
        if n_pages > best:
            best, first = n_pages, f
        if key:
            m += 1
    return first


class OracleSampler:
    """The fp64 oracle (``oracle.stream.StreamOracle``, as it stands) advanced to the busiest
    frame of the stream, then timed on frames that see that frame's retained keys.

    Query rows are independent, so a frame's attention is timed on a sample of rows: each
    sample steps the oracle over one frame twice, with r1 and then r2 sampled rows (the frame
    index increases and the frames are stepped as non-keyframes, so the retained set and the
    key count stay those of the busiest frame).  Per-frame time = t(r1) + (T - r1) * slope,
    slope = (t(r2) - t(r1)) / (r2 - r1): rotation, page-table work and key gathering are
    counted once, the attention once per row."""

    def __init__(self, cfg):
        from oracle import stream as ostream
        from rope_paged_kv_02_b200 import workloads
        self.cfg = cfg
        self.wl = workloads
        self.so = ostream.StreamOracle(cfg.heads, cfg.head_dim, cfg.pph, cfg.ppw,
                                       cfg.scale_frames, cfg.sliding_window,
                                       max(1, cfg.n_keyframes))
        self.frame = _busiest_frame(cfg)
        for f in range(self.frame):            # untimed: build the retained state
            q, k, v = workloads.frame_qkv(cfg, f)
            self.so.step(f, cfg.keyframes[f], q, k, v, rows=[], attend=False)
        self.next = self.frame
        self.r2 = min(64, cfg.tokens)
        self.r1 = max(1, self.r2 // 2)
        self.rng = np.random.default_rng(12345)

    def _timed(self, n_rows: int) -> float:
        q, k, v = self.wl.frame_qkv(self.cfg, self.next)
        rows = np.sort(self.rng.choice(self.cfg.tokens, n_rows, replace=False))
        t0 = time.perf_counter()
        self.so.step(self.next, False, q, k, v, rows=rows, attend=True)
        dt = time.perf_counter() - t0
        self.next += 1
        return dt

    def frame_seconds(self) -> tuple[float, float]:
        """(estimated seconds per full frame, seconds spent)."""
        t1 = self._timed(self.r1)
        t2 = self._timed(self.r2)
        slope = max(t2 - t1, 0.0) / (self.r2 - self.r1)
        return t1 + (self.cfg.tokens - self.r1) * slope, t1 + t2

    def describe(self) -> str:
        c = self.cfg
        return (f"frames >= {self.frame} (the first to see as many patch pages as the "
                f"stream ever does), stepped as "
                f"non-keyframes so each sees the same keys; {self.r1} and {self.r2} random "
                f"query rows x {c.heads} heads per sample, full fp64 step (rotate q/k, page "
                f"state, attention), per-frame time extrapolated linearly in rows to all "
                f"{c.tokens}")


def run_reference(args, cfg, rank, world):
    """The fp64 oracle on this host's cores, bounded sample of the same workload."""
    if rank != 0:
        return None
    sampler = OracleSampler(cfg)
    for _ in range(args.warmup):
        sampler.frame_seconds()
    times = [sampler.frame_seconds()[0] for _ in range(args.steps)]
    per_frame = float(np.mean(times))
    value = 1.0 / per_frame
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per_frame * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, bf16-valued inputs)",
        "config": _config_dict(cfg, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": _blas_threads(),
                         "kind": "oracle",
                         "sample": "one frame per step: " + sampler.describe()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


def cpu_baseline(cfg):
    """Oracle frames/s on a bounded sample (two frames' worth of row samples)."""
    sampler = OracleSampler(cfg)
    est, spent = [], 0.0
    for _ in range(2):
        e, s = sampler.frame_seconds()
        est.append(e)
        spent += s
    return {"value": 1.0 / float(np.mean(est)), "unit": UNIT, "cores": _blas_threads(),
            "kind": "oracle",
            "sample": "two samples: " + sampler.describe() + f"; {spent:.1f} s of CPU work"}


def _config_dict(cfg, world, n_frames=None):
    F = cfg.n_frames if n_frames is None else n_frames
    pool = min(F, INPUT_POOL)
    d = {"workload": cfg.describe() if n_frames is None else
         f"first {n_frames} frames of " + cfg.describe(),
         "frames_per_step": F,
         "tokens_per_frame": cfg.tokens, "heads": cfg.heads, "head_dim": cfg.head_dim,
         "scale_frames": cfg.scale_frames, "sliding_window": cfg.sliding_window,
         "parallelism": f"replicas x{world} (independent streams, no exchange)",
         "l2": "inputs larger than L2 (%d distinct frames of q/k/v cycled, %.0f MB)" % (
             pool, pool * 3 * cfg.tokens * cfg.heads * cfg.head_dim * cfg.elem_bytes / 1e6)}
    return d


# ------------------------------------------------------------------------------------------
# the CUDA path
# ------------------------------------------------------------------------------------------

class Workload:
    """Device (and pinned host) copies of a stream's input pool, a cache, and the step."""

    def __init__(self, cfg, dev, n_frames=None, host_copies=False):
        import torch
        from rope_paged_kv_02_b200 import _lib, workloads
        self.cfg = cfg
        self.F = cfg.n_frames if n_frames is None else n_frames
        self.pool = min(self.F, INPUT_POOL)
        tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
        self.tdt = tdt
        self.q, self.k, self.v, self.host = [], [], [], []
        for f in range(self.pool):
            ts = [torch.from_numpy(x).to(tdt) for x in workloads.frame_qkv(cfg, f)]
            if host_copies:
                ts = [t.pin_memory() for t in ts]
                self.host.append(ts)
            self.q.append(ts[0].to(dev))
            self.k.append(ts[1].to(dev))
            self.v.append(ts[2].to(dev))
        self.out = [torch.empty_like(self.q[0]) for _ in range(self.pool)]
        self.rope = _lib.Rope3D(cfg.head_dim, max(self.F, cfg.n_frames), cfg.pph, cfg.ppw, 6)
        self.cache = _lib.PagedKVCache(self.rope, cfg.heads, cfg.head_dim, cfg.patches,
                                       cfg.scale_frames, cfg.sliding_window,
                                       max(1, cfg.n_keyframes),
                                       _lib.LBM_BF16 if cfg.dtype == "bf16" else _lib.LBM_F32)
        self.keys = cfg.keyframes

    def step(self, stream, ev=None):
        """One pass over the stream; with ev, an event pair around every append and attend."""
        c = self.cache
        c.reset()
        for f in range(self.F):
            b = f % self.pool
            if ev is not None:
                ev[f][0].record(stream)
            c.append_frame(self.q[b], self.k[b], self.v[b], f, self.keys[f], stream)
            if ev is not None:
                ev[f][1].record(stream)
            c.attend_frame(self.q[b], self.out[b], stream)
            if ev is not None:
                ev[f][2].record(stream)

    def close(self):
        self.cache.close()
        self.rope.close()


def measure(w: Workload, steps: int, warmup: int, world: int, local: int, peaks: dict,
            dev) -> dict:
    """Times `steps` steps of the stream (after `warmup`), then a second pass of the same
    steps with an event pair around every kernel launch; returns the figures of one line."""
    import torch
    cfg = w.cfg
    stream = torch.cuda.current_stream(dev)
    for _ in range(warmup):
        w.step(stream)
    torch.cuda.synchronize()
    w.cache.check()

    # ---- timed region: K steps back to back on the stream, bracketed by two events ----
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = w.cache.state()["kernel_launches"]
    with ClockSampler(local) as clocks:
        barrier(world)
        torch.cuda.synchronize()
        t0.record(stream)
        for _ in range(steps):
            w.step(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    launches = w.cache.state()["kernel_launches"] - launches0
    ms = max_over_ranks(t0.elapsed_time(t1), world)
    w.cache.check()

    # ---- per-kernel durations: the same K steps again with an event pair around every
    # append and every attend launch (attention + combine) on the launching stream ----
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(w.F)]
           for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    for s in range(steps):
        w.step(stream, evs[s])
    torch.cuda.synchronize()
    barrier(world)
    w.cache.check()
    append_ms = np.array([[e[0].elapsed_time(e[1]) for e in st] for st in evs])
    attn_ms = np.array([[e[1].elapsed_time(e[2]) for e in st] for st in evs])

    flops, nbytes, keys = frame_work(cfg, w.F)
    step_ms = ms / steps
    # The events between launches stop a kernel from overlapping its predecessor's tail, so
    # the event-pair sums can exceed the undisturbed step.  The attention time used for the
    # roofline is capped so that attention + append never exceed the timed step.
    attn_step_evt = float(attn_ms.sum(axis=1).mean())
    append_step_evt = float(append_ms.sum(axis=1).mean())
    attn_step = min(attn_step_evt, step_ms - append_step_evt)
    clk = clocks.summary()
    peak, peak_src = tensor_peak(peaks, clk)
    attn_tflops = flops.sum() / (attn_step / 1e3) / 1e12
    append_gbs = nbytes.sum() / (append_step_evt / 1e3) / 1e9
    return {
        "frames_per_s": w.F * steps * world / (ms / 1e3), "ms_per_step": step_ms,
        "steps": steps, "warmup": warmup, "gpu_launches": int(launches),
        "attention": {
            "achieved_tflops": attn_tflops, "peak_tflops": peak, "frac": attn_tflops / peak,
            "peak_source": peak_src, "ms_per_step": attn_step,
            "event_pair_ms_per_step": attn_step_evt,
            "avg_us": attn_step / w.F * 1e3, "flops_per_frame_avg": float(flops.mean()),
            "avg_keys": float(keys.mean())},
        "append": {"achieved_gbs": append_gbs, "peak_gbs": peaks["hbm_gbs"],
                   "frac": append_gbs / peaks["hbm_gbs"], "bytes_per_frame": float(nbytes[0]),
                   "avg_us": append_step_evt / w.F * 1e3},
        "clocks": clk,
    }


def e2e_measure(w: Workload, steps: int, world: int, dev):
    """Same metric through the C ABI with host buffers: per frame, pinned host q/k/v are
    copied to the device on a host-to-device stream, the frame is appended and attended on
    the compute stream, and its output is copied back to pinned host memory on a
    device-to-host stream, so both copies overlap other frames' kernels.  Three device
    buffer sets rotate: a frame's inputs are overwritten only after the frame that last used
    them has been attended, its output only after the previous one has been copied out."""
    import torch
    F, pool, tdt, cache = w.F, w.pool, w.tdt, w.cache
    hq = [h[0] for h in w.host]
    hk = [h[1] for h in w.host]
    hv = [h[2] for h in w.host]
    ho = [torch.empty_like(hq[0]).pin_memory() for _ in range(pool)]
    nbuf = 3
    dq = [torch.empty(hq[0].shape, dtype=tdt, device=dev) for _ in range(nbuf)]
    dk = [torch.empty_like(dq[0]) for _ in range(nbuf)]
    dv = [torch.empty_like(dq[0]) for _ in range(nbuf)]
    do = [torch.empty_like(dq[0]) for _ in range(nbuf)]
    comp = torch.cuda.current_stream(dev)
    h2d = torch.cuda.Stream(dev)
    d2h = torch.cuda.Stream(dev)
    attended = [torch.cuda.Event() for _ in range(nbuf)]  # the frame in buffer b attended
    landed = [torch.cuda.Event() for _ in range(nbuf)]    # inputs of buffer b on the device
    copied = [torch.cuda.Event() for _ in range(nbuf)]    # output of buffer b on the host
    keys = w.keys

    def step(first):
        cache.reset()
        for f in range(F):
            b = f % nbuf
            h = f % pool
            reuse = not first or f >= nbuf
            with torch.cuda.stream(h2d):
                if reuse:
                    h2d.wait_event(attended[b])
                dq[b].copy_(hq[h], non_blocking=True)
                dk[b].copy_(hk[h], non_blocking=True)
                dv[b].copy_(hv[h], non_blocking=True)
                landed[b].record(h2d)
            comp.wait_event(landed[b])
            if reuse:
                comp.wait_event(copied[b])
            cache.append_frame(dq[b], dk[b], dv[b], f, keys[f], comp)
            cache.attend_frame(dq[b], do[b], comp)
            attended[b].record(comp)
            with torch.cuda.stream(d2h):
                d2h.wait_event(attended[b])
                ho[h].copy_(do[b], non_blocking=True)
                copied[b].record(d2h)

    step(True)
    step(False)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    t0.record(comp)
    for _ in range(steps):
        step(False)
    comp.wait_stream(d2h)          # the last outputs are on the host
    t1.record(comp)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), world)
    per = hq[0].numel() * hq[0].element_size()
    return {"value": F * steps * world / (ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": 3 * per * F, "d2h_bytes_per_step": per * F}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=HEADLINE_CONFIG)
    ap.add_argument("--frames", type=int, default=None,
                    help="stream only the first N frames (small profiling cases)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-configs", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()

    rank, world, local = dist_setup(args.gpus)
    from rope_paged_kv_02_b200 import workloads
    cfg = workloads.CONFIGS[args.config]

    if args.impl == "reference":
        line = run_reference(args, cfg, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        _teardown(world)
        return

    import torch
    from rope_paged_kv_02_b200 import _lib
    from rope_paged_kv_02_b200.build import build
    if rank == 0 or not os.path.exists(_lib.LIB_PATH):
        build()
    barrier(world)
    _lib.load()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = _peaks()
    warmup = max(3, args.warmup)

    w = Workload(cfg, dev, args.frames, host_copies=not args.no_e2e)
    head = measure(w, args.steps, warmup, world, local, peaks, dev)
    e2e = None if args.no_e2e else e2e_measure(w, args.steps, world, dev)
    _, _, keys = frame_work(cfg, w.F)
    w.close()
    del w
    torch.cuda.empty_cache()

    att, app = head["attention"], head["append"]
    line = {
        "metric": METRIC, "value": head["frames_per_s"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype,
        "data": "synthetic (seeded q/k/v rounded to bf16)",
        "config": _config_dict(cfg, world, args.frames),
        "roofline": {
            "bound": "tensor", "achieved": att["achieved_tflops"], "peak": att["peak_tflops"],
            "unit": "TFLOP/s", "frac": att["frac"],
            "traffic": measured_traffic(args.config, float(keys.mean())),
            "kernel": "paged attention (attn_tc + stream-K combine), all frames of the stream",
            "kernel_timing": "event pair around every attend launch in a second pass of the "
                             "same K steps; per-step sum capped at ms_per_step minus the "
                             "appends' event-pair time",
            "peak_source": att["peak_source"],
        },
        "append": app,
        "attention": att,
        "e2e": e2e,
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
    }
    if world == 1 and not args.no_other_configs and args.frames is None:
        others = {}
        for cid in OTHER_CONFIGS:
            if cid == args.config:
                continue
            ocfg = workloads.CONFIGS[cid]
            ow = Workload(ocfg, dev)
            # the 2000-frame stream takes ~2 s a step: two timed steps bound its time
            osteps = 2 if ocfg.n_frames > 1000 else min(args.steps, 5)
            r = measure(ow, osteps, 3, world, local, peaks, dev)
            ow.close()
            del ow
            torch.cuda.empty_cache()
            r["workload"] = ocfg.describe()
            others[ocfg.name] = r
        line["other_configs"] = others
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg)
    if rank == 0:
        print(json.dumps(line), flush=True)
    _teardown(world)


def _teardown(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
