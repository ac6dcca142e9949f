"""Benchmark of the streaming-frame step (3D RoPE + paged KV append + paged attention).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config C]

One step streams every frame of the workload through a fresh cache: per frame one
lbm_append_frame (fused rotate + append) and one lbm_attend_frame (paged attention on
persistent CTAs, plus the combine of the units several CTAs share), host page-table
bookkeeping included.  The default workload is the 768-patch stream: 16 heads x head_dim 64, bf16,
6 special + 24x32 patch tokens per frame, 64 keyframes, scale_frames 8, sliding_window 16.
Inputs are seeded synthetic frames; the 64 frames of a step (304 MB of q/k/v) are larger
than L2, so no input is L2-resident between steps.

With N > 1 (torchrun) every rank streams its own independent copy of the workload (the step
has no exchange between GPUs): weak scaling, value = all ranks' frames / max rank time.

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
METRIC = "streamed frames/s per layer (RoPE+append+paged attn); % of bf16 TC / HBM peak"
UNIT = "frames/s"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def measured_traffic(avg_keys: float):
    """DRAM bytes per attention launch from the committed ncu summary, scaled from the
    captured frame's key count to the stream's average (K/V reads dominate and grow with
    the keys); None once the kernel source differs from the one that was profiled."""
    import hashlib
    prof = os.path.join(ROOT, "profiles", "attn_tc_stream768.md")
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


def frame_work(cfg):
    """Algorithmic work per frame of a stream: (attention FLOPs, append bytes, keys seen).

    Frame n with m keyframes committed before it sees min(m, S+W)+1 patch pages and 6(m+1)
    special tokens; attention = 4 T N_k H D flops (QK^T and PV); append moves 6 T H D e bytes
    (read q, k, v; write q, k, v).
    """
    T, H, D, e = cfg.tokens, cfg.heads, cfg.head_dim, cfg.elem_bytes
    flops, nbytes, keys = [], [], []
    m = 0
    for key in cfg.keyframes:
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
        self.idx = device_index
        self.proc = None
        self.lines = []

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
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


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


def run_reference(args, cfg, rank, world):
    """The fp64 oracle on this host's cores, bounded sample of the same workload."""
    if rank != 0:
        return None
    from oracle import stream as ostream
    from rope_paged_kv_02_b200 import workloads
    sample_frames = [cfg.scale_frames + cfg.sliding_window + 1]  # a steady-state frame
    so_frames = sample_frames[-1] + 1

    def one_step():
        so = ostream.StreamOracle(cfg.heads, cfg.head_dim, cfg.pph, cfg.ppw, cfg.scale_frames,
                                  cfg.sliding_window, cfg.n_keyframes,
                                  kv_source=_regen(cfg))
        t_att = 0.0
        for f in range(so_frames):
            q, k, v = workloads.frame_qkv(cfg, f)
            t0 = time.perf_counter()
            so.step(f, cfg.keyframes[f], q, k, v, rows=None if f in sample_frames else [],
                    attend=f in sample_frames)
            if f in sample_frames:
                t_att += time.perf_counter() - t0
        return t_att / len(sample_frames)

    for _ in range(args.warmup):
        one_step()
    times = [one_step() for _ in range(args.steps)]
    per_frame = float(np.mean(times))
    value = 1.0 / per_frame
    cores = _blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per_frame * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, bf16-valued inputs)",
        "config": _config_dict(cfg, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"one steady-state frame ({sample_frames[0]}) of the stream "
                                   f"per step, all {cfg.tokens} query rows x {cfg.heads} heads, "
                                   "rotate + page state + attention in fp64"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


def _regen(cfg):
    from rope_paged_kv_02_b200 import workloads

    def source(frame, region):
        if region == "special":
            return workloads.frame_specials(cfg, frame, 1), workloads.frame_specials(cfg, frame, 2)
        return workloads.frame_tensor(cfg, frame, 1)[6:], workloads.frame_tensor(cfg, frame, 2)[6:]

    return source


def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def _config_dict(cfg, world):
    return {"workload": cfg.describe(), "frames_per_step": cfg.n_frames,
            "tokens_per_frame": cfg.tokens, "heads": cfg.heads, "head_dim": cfg.head_dim,
            "scale_frames": cfg.scale_frames, "sliding_window": cfg.sliding_window,
            "parallelism": f"replicas x{world} (independent streams, no exchange)",
            "l2": "inputs larger than L2 (%d distinct frames of q/k/v cycled, %.0f MB)" % (
                min(cfg.n_frames, INPUT_POOL),
                min(cfg.n_frames, INPUT_POOL) * 3 * cfg.tokens * cfg.heads * cfg.head_dim
                * cfg.elem_bytes / 1e6)}


def cpu_baseline(cfg):
    """Oracle frames/s on a bounded sample (two steady-state frames, all rows)."""
    from oracle import stream as ostream
    from rope_paged_kv_02_b200 import workloads
    targets = [cfg.scale_frames + cfg.sliding_window + 1, cfg.scale_frames + cfg.sliding_window + 2]
    so = ostream.StreamOracle(cfg.heads, cfg.head_dim, cfg.pph, cfg.ppw, cfg.scale_frames,
                              cfg.sliding_window, cfg.n_keyframes, kv_source=_regen(cfg))
    spent = 0.0
    for f in range(targets[-1] + 1):
        q, k, v = workloads.frame_qkv(cfg, f)
        t0 = time.perf_counter()
        so.step(f, cfg.keyframes[f], q, k, v, rows=None if f in targets else [],
                attend=f in targets)
        if f in targets:
            spent += time.perf_counter() - t0
    return {"value": len(targets) / spent, "unit": UNIT, "cores": _blas_threads(),
            "kind": "oracle",
            "sample": f"frames {targets} of the stream (steady state), all {cfg.tokens} rows "
                      f"x {cfg.heads} heads, fp64 rotate + page state + attention; "
                      f"{spent:.1f} s of CPU work"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=1)
    ap.add_argument("--no-cpu-baseline", action="store_true")
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
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32

    # ---- inputs resident in HBM before timing: the frames of the stream, or for streams
    # longer than INPUT_POOL frames a pool of that many distinct frames used in turn (the
    # pool is larger than L2, and the cache's contents do not change the work per frame) ----
    F = cfg.n_frames
    pool = min(F, INPUT_POOL)
    qs, ks, vs = [], [], []
    for f in range(pool):
        q, k, v = workloads.frame_qkv(cfg, f)
        qs.append(torch.from_numpy(q).to(dev, tdt))
        ks.append(torch.from_numpy(k).to(dev, tdt))
        vs.append(torch.from_numpy(v).to(dev, tdt))
    outs = [torch.empty_like(qs[0]) for _ in range(pool)]
    rope = _lib.Rope3D(cfg.head_dim, F, cfg.pph, cfg.ppw, 6)
    cache = _lib.PagedKVCache(rope, cfg.heads, cfg.head_dim, cfg.patches, cfg.scale_frames,
                              cfg.sliding_window, cfg.n_keyframes,
                              _lib.LBM_BF16 if cfg.dtype == "bf16" else _lib.LBM_F32)
    stream = torch.cuda.current_stream(dev)
    keys = cfg.keyframes

    def step(ev=None):
        cache.reset()
        for f in range(F):
            b = f % pool
            if ev is not None:
                ev[f][0].record(stream)
            cache.append_frame(qs[b], ks[b], vs[b], f, keys[f], stream)
            if ev is not None:
                ev[f][1].record(stream)
            cache.attend_frame(qs[b], outs[b], stream)
            if ev is not None:
                ev[f][2].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    cache.check()

    # ---- timed region: K steps back to back on the stream, bracketed by two events ----
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = cache.state()["kernel_launches"]
    with ClockSampler(local) as clocks:
        barrier(world)
        torch.cuda.synchronize()
        t0.record(stream)
        for s in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    launches = cache.state()["kernel_launches"] - launches0
    ms = t0.elapsed_time(t1)
    ms_max = max_over_ranks(ms, world)
    cache.check()

    # ---- per-kernel durations: the same K steps again with an event pair around every
    # append and every attend launch on the launching stream.  The events between launches
    # stop each kernel from overlapping its predecessor's tail (programmatic dependent
    # launch), so these durations are slightly pessimistic; the headline uses the pass above.
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(F)]
           for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for s in range(args.steps):
        step(evs[s])
    torch.cuda.synchronize()
    barrier(world)
    cache.check()
    append_ms = np.array([[e[0].elapsed_time(e[1]) for e in st] for st in evs])
    attn_ms = np.array([[e[1].elapsed_time(e[2]) for e in st] for st in evs])

    flops, nbytes, keys = frame_work(cfg)
    frames_total = F * args.steps * world
    value = frames_total / (ms_max / 1e3)
    peaks = _peaks()
    attn_avg_s = attn_ms.mean() / 1e3
    attn_tflops = flops.mean() / attn_avg_s / 1e12
    append_gbs = nbytes.mean() / (append_ms.mean() / 1e3) / 1e9
    # steady-state frames (window full) for the headline roofline of the attention kernel
    ss = slice(cfg.scale_frames + cfg.sliding_window, F)
    ss_tflops = flops[ss].mean() / (attn_ms[:, ss].mean() / 1e3) / 1e12

    # ---- end to end: host (pinned) inputs -> device -> append/attend -> host output ----
    e2e = e2e_measure(cfg, cache, args, dev, tdt, world)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_max / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype,
        "data": "synthetic (seeded N(0,1) q/k/v rounded to bf16)",
        "config": _config_dict(cfg, world),
        "roofline": {
            "bound": "tensor", "achieved": attn_tflops,
            "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
            "frac": attn_tflops / peaks["bf16_tflops_sustained"],
            "traffic": measured_traffic(float(keys.mean())) if args.config == 1 else None,
            "kernel": "paged attention (attn_tc + stream-K combine), all frames",
            "kernel_timing": "event pair around every attend launch, second pass of the "
                             "same K steps",
            "peak_source": peaks["source"] + " bf16_tflops_sustained",
            "steady_state_achieved": ss_tflops,
        },
        "append": {"achieved_gbs": append_gbs, "peak_gbs": peaks["hbm_gbs"],
                   "frac": append_gbs / peaks["hbm_gbs"], "bytes_per_frame": float(nbytes[0]),
                   "avg_us": float(append_ms.mean() * 1e3)},
        "attention": {"avg_us": float(attn_ms.mean() * 1e3),
                      "steady_state_avg_us": float(attn_ms[:, ss].mean() * 1e3),
                      "flops_per_frame_avg": float(flops.mean())},
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg)
    if rank == 0:
        print(json.dumps(line), flush=True)
    cache.close()
    rope.close()
    _teardown(world)


def e2e_measure(cfg, cache, args, dev, tdt, world):
    """Same metric through the C ABI with host buffers: per frame, pinned host q/k/v are
    copied to the device on a host-to-device stream, the frame is appended and attended on
    the compute stream, and its output is copied back to pinned host memory on a
    device-to-host stream, so both copies overlap other frames' kernels.  Three device
    buffer sets rotate: a frame's inputs are overwritten only after the frame that last used
    them has been attended, its output only after the previous one has been copied out."""
    import torch
    F = cfg.n_frames
    from rope_paged_kv_02_b200 import workloads
    hq, hk, hv, ho = [], [], [], []
    pool = min(F, INPUT_POOL)
    for f in range(pool):
        q, k, v = workloads.frame_qkv(cfg, f)
        hq.append(torch.from_numpy(q).to(tdt).pin_memory())
        hk.append(torch.from_numpy(k).to(tdt).pin_memory())
        hv.append(torch.from_numpy(v).to(tdt).pin_memory())
        ho.append(torch.empty_like(hq[-1]).pin_memory())
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
    keys = cfg.keyframes

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
    for _ in range(args.steps):
        step(False)
    comp.wait_stream(d2h)          # the last outputs are on the host
    t1.record(comp)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), world)
    per = hq[0].numel() * hq[0].element_size()
    return {"value": F * args.steps * world / (ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": 3 * per * F, "d2h_bytes_per_step": per * F}


def _teardown(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
