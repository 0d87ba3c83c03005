"""Benchmark of the STA forward hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

One step = one pass of the whole hot path on the video+text workload
(B=1, 24 heads, d=128, video (30,48,80) in (6,8,8) tiles + 256 text tokens,
text_length 200, window (3,3,3) tiles; inputs q, k, v bf16 N(0,1), seeded),
raster-ordered in and out: KV tile lists + the attention kernel, which reads
each tile block of q, k, v through 5-D TMA boxes (the raster->tile
permutation) and stores every output row at its raster position (the
inverse).  The standalone permutation kernel is timed separately.
The metric is effective TFLOP/s counting only retained (query, key) pairs,
4 * d FLOP each.  Inputs (3 x 710 MB) are larger than L2, so no flush is
needed between steps.

Multi-GPU (torchrun, one rank per GPU): every rank runs its own batch element
of the same workload (independent problems, weak scaling, no data-path
collective); the time is the max over ranks.

--impl reference times the float64 CPU oracle on the host cores on a bounded
sample of the same workload (it is the baseline, not the target).
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "STA forward ms and effective TFLOP/s (retained tiles) as % of B200 BF16 peak"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
ATTN_SOURCES = ("block_sparse_local_b200/csrc/attn_fwd.cuh",
                "block_sparse_local_b200/csrc/device_ptx.cuh")


def workload_config(w, world):
    """The `config` object of the JSON line (both arms)."""
    return {"workload": w.name, "B_per_gpu": w.B, "heads": w.heads, "d": w.d,
            "video": [w.T, w.H, w.W], "tile": list(w.tile), "window": list(w.windows[0]),
            "text_len": w.text_len, "seq_len": w.S, "global_batch": w.B * world,
            "parallelism": f"independent problems x{world}",
            "l2": "inputs larger than L2 (3 x 710 MB), no flush",
            "step": "tile lists + attention with the raster<->tile permutation "
                    "fused into its TMA loads and output stores"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-swa", action="store_true", help="skip the SWA comparison")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the tiny, video-only and 2-D workloads")
    ap.add_argument("--heads", type=int, default=None,
                    help="run the workload with fewer heads (profiling captures only)")
    ap.add_argument("--backward-only", action="store_true",
                    help="time only the backward pass of the workload (profiling captures)")
    ap.add_argument("--profile-workload", default=None,
                    help="run only the forward of this named STA workload (raster order), "
                         "--steps times after --warmup, for profiling captures; "
                         "--heads keeps that many heads")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def source_hash():
    """Hash of the attention kernel's code (comment-only lines and blank lines
    left out, so that editing a comment keeps the measured traffic valid)."""
    h = hashlib.sha256()
    for rel in ATTN_SOURCES:
        with open(os.path.join(ROOT, rel)) as f:
            for line in f:
                t = line.strip()
                if t and not t.startswith("//"):
                    h.update(t.encode())
                    h.update(b"\n")
    return h.hexdigest()[:16]


def attn_traffic(units_per_launch):
    """DRAM bytes per launch of the attention kernel from the committed ncu
    summary, or None when the kernel source changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "attn_fwd_video_text_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("source_hash") != source_hash():
        return None
    # captured on a smaller case; traffic scales with the key blocks processed
    return d["dram_bytes_per_unit"] * units_per_launch


def run_other_configs(dev, stream, peak, flush_bytes=256 << 20, iters=5):
    """The other STA workloads (tiny, video-only with per-head windows, 2-D
    at (5,5) and at the grid-covering (16,16) window), each as the bench step
    runs them: tile lists + the attention kernel on raster-ordered tensors.
    L2 is flushed (a 256 MB write) before every timed call, and each call is
    timed alone with CUDA events on the launching stream."""
    import torch
    import block_sparse_local_b200 as sta
    from block_sparse_local_b200 import workloads
    flush = torch.empty(flush_bytes, dtype=torch.uint8, device=dev)
    res = {}
    for w in (workloads.TINY, workloads.VIDEO_ONLY, workloads.IMAGE_2D, workloads.IMAGE_2D_FULL):
        shape = (w.T, w.H, w.W)
        q, k, v = workloads.sta_inputs(w, device=dev)
        out = torch.empty_like(q)

        def call():
            sta.forward_raster(q, k, v, w.windows, w.text_len, w.has_text, shape, w.tile,
                               out=out)

        for _ in range(2):
            call()
        torch.cuda.synchronize(dev)
        n = iters if w.B * w.heads > 1 else 20
        times = []
        for _ in range(n):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            call()
            b.record(stream)
            torch.cuda.synchronize(dev)
            times.append(a.elapsed_time(b))
        sta.device_status(dev)
        ms = statistics.median(times)
        pairs = sta.retained_pairs(w.B, w.windows, shape, w.tile, w.text_len, w.has_text)
        tf = 4.0 * w.d * pairs / (ms * 1e-3) / 1e12
        res[w.name] = {"B": w.B, "heads": w.heads, "d": w.d, "video": list(shape),
                       "tile": list(w.tile),
                       "window": list(w.windows[0]) if len(set(w.windows)) == 1 else
                       "per head: " + ", ".join(f"{c}x{sum(1 for x in w.windows if x == c)}"
                                                for c in sorted(set(w.windows))),
                       "ms": ms, "effective_tflops": tf, "pct_of_bf16_peak": 100.0 * tf / peak,
                       "kernel": f"attn_fwd_kernel<{w.d},kSta,raster>",
                       "timing": f"median of {n}, L2 flushed before each call"}
        del q, k, v, out
    del flush
    return res


def run_backward(q, k, v, w, shape, pairs, dev, stream):
    """Backward pass of the STA workload (tile order): dQ, dK, dV from the
    saved LSE; algorithmic work 5 matmuls of 2*d per retained pair."""
    import torch
    import block_sparse_local_b200 as sta
    qt, kt, vt = (sta.tile_reorder(x, shape, w.tile, w.has_text) for x in (q, k, v))
    ot, lset = sta.forward(qt, kt, vt, w.windows, w.text_len, w.has_text, shape, w.tile,
                           return_lse=True)
    dot = torch.randn_like(qt, dtype=torch.float32).to(torch.bfloat16)
    for _ in range(2):
        sta.backward(qt, kt, vt, ot, dot, lset, w.windows, w.text_len, w.has_text, shape, w.tile)
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(3):
        sta.backward(qt, kt, vt, ot, dot, lset, w.windows, w.text_len, w.has_text, shape, w.tile)
    b.record(stream)
    torch.cuda.synchronize(dev)
    bms = a.elapsed_time(b) / 3
    sta.device_status(dev)
    return {"workload": w.name, "ms": bms,
            "effective_tflops": 10.0 * w.d * pairs / (bms * 1e-3) / 1e12,
            "flop_model": "10*d per retained pair (5 matmuls)"}


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait()
        sms, maxs, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sms.append(float(parts[1]))
                    maxs.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        load = [s for s in sms if s > 600] or sms
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(maxs) if maxs else None,
                "samples": len(sms), "reasons": sorted(reasons)}


def cpu_oracle_sample(w, q_h, k_h, v_h, seconds):
    """Time the float64 oracle (form B) on query tiles of one head until
    ``seconds`` pass; returns (effective TFLOP/s, description, threads)."""
    import numpy as np
    from oracle import sta_oracle

    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        threads = len(os.sched_getaffinity(0))
    q64, k64, v64 = (x.double().numpy() for x in (q_h, k_h, v_h))
    ct, ch, cw = w.tile
    NT, NH, NW = w.T // ct, w.H // ch, w.W // cw
    tiles_done, pairs, rows_done = 0, 0, 0
    t0 = time.perf_counter()
    for tq in range(NT * NH * NW):
        qt, qh, qw = tq // (NH * NW), (tq // NW) % NH, tq % NW
        tt = np.arange(qt * ct, (qt + 1) * ct)
        hh = np.arange(qh * ch, (qh + 1) * ch)
        ww = np.arange(qw * cw, (qw + 1) * cw)
        rows = ((tt[:, None, None] * w.H + hh[None, :, None]) * w.W + ww[None, None, :]).ravel()
        sta_oracle.sta_forward_rows(q64, k64, v64, w.T, w.H, w.W, w.tile, w.windows[0],
                                    w.text_len, w.has_text, rows=rows)
        keys = len(sta_oracle.allowed_keys(int(rows[0]), w.T, w.H, w.W, w.tile, w.windows[0],
                                           w.text_len, w.has_text))
        pairs += len(rows) * keys
        rows_done += len(rows)
        tiles_done += 1
        if time.perf_counter() - t0 > seconds:
            break
    dt = time.perf_counter() - t0
    tflops = 4.0 * w.d * pairs / dt / 1e12
    desc = (f"float64 oracle (row-gather form) on {tiles_done} video query tiles "
            f"({rows_done} rows) of head 0 of the same workload, {dt:.1f} s")
    return tflops, desc, threads, dt


def run_reference(args):
    """--impl reference: the CPU oracle as it stands, rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import torch
    from block_sparse_local_b200 import workloads

    w = workloads.VIDEO_TEXT
    g = torch.Generator().manual_seed(w.seed * 1000)
    shape = (w.S, w.d)
    q_h, k_h, v_h = (torch.randn(shape, generator=g).mul_(w.std).to(torch.bfloat16)
                     for _ in range(3))
    per_step = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_oracle_sample(w, q_h, k_h, v_h, per_step / 4)
    vals, total = [], 0.0
    for _ in range(args.steps):
        tf, desc, threads, dt = cpu_oracle_sample(w, q_h, k_h, v_h, per_step)
        vals.append(tf)
        total += dt
    value = statistics.median(vals)
    from oracle import sta_oracle
    flops = 4.0 * w.d * sum(sta_oracle.retained_pairs(w.T, w.H, w.W, w.tile, tuple(win),
                                                      w.text_len, w.has_text)
                            for win in w.windows)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": flops / (value * 1e12) * 1e3 if value > 0 else None,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(w, args.gpus),
        "note": "CPU oracle on a bounded sample; ms_per_step extrapolated to the whole workload",
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def run_profile_workload(args):
    """Forward of one named workload only (profiling captures of the d = 64
    kernel and of the other shapes); prints its time, not a bench line."""
    import dataclasses
    import torch
    import block_sparse_local_b200 as sta
    from block_sparse_local_b200 import workloads
    w = workloads.STA_WORKLOADS[args.profile_workload]
    if args.heads is not None:
        w = dataclasses.replace(w, heads=args.heads, windows=w.windows[:args.heads])
    dev = torch.device("cuda", 0)
    shape = (w.T, w.H, w.W)
    q, k, v = workloads.sta_inputs(w, device=dev)
    out = torch.empty_like(q)
    for i in range(args.warmup + args.steps):
        if i == args.warmup:
            torch.cuda.synchronize(dev)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
        sta.forward_raster(q, k, v, w.windows, w.text_len, w.has_text, shape, w.tile, out=out)
    b.record()
    torch.cuda.synchronize(dev)
    sta.device_status(dev)
    ms = a.elapsed_time(b) / max(1, args.steps)
    pairs = sta.retained_pairs(w.B, w.windows, shape, w.tile, w.text_len, w.has_text)
    print(json.dumps({"profile_workload": w.name, "heads": w.heads, "ms": ms,
                      "effective_tflops": 4.0 * w.d * pairs / (ms * 1e-3) / 1e12}))
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist

    import block_sparse_local_b200 as sta
    from block_sparse_local_b200 import workloads
    from block_sparse_local_b200.dist_timing import max_over_ranks, rank_seed

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))

    w = workloads.VIDEO_TEXT
    if args.heads is not None:
        import dataclasses
        w = dataclasses.replace(w, name=f"{w.name}_heads{args.heads}", heads=args.heads,
                                windows=w.windows[:1] * args.heads)
    shape = (w.T, w.H, w.W)
    # each rank draws its own batch element (independent problems)
    gq = torch.Generator(device=dev)
    qkv = []
    for i in range(3):
        gq.manual_seed(rank_seed(w.seed * 1000 + i, rank))
        qkv.append(torch.randn((w.B, w.heads, w.S, w.d), generator=gq, device=dev,
                               dtype=torch.float32).to(torch.bfloat16))
    q, k, v = qkv
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)
    pairs = sta.retained_pairs(w.B, w.windows, shape, w.tile, w.text_len, w.has_text)
    flops = 4.0 * w.d * pairs

    if args.backward_only:
        if rank == 0:
            print(json.dumps({"backward_only": run_backward(q, k, v, w, shape, pairs, dev,
                                                            stream)}))
        if world > 1:
            dist.destroy_process_group()
        return
    attn_ev = []

    def step(record=False):
        if record:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        sta.forward_raster(q, k, v, w.windows, w.text_len, w.has_text, shape, w.tile, out=out)
        if record:
            e1.record(stream)
            attn_ev.append((e0, e1))

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    nvtx = torch.cuda.nvtx
    with nvtx.range("bench.warmup"):
        for _ in range(max(3, args.warmup)):
            step()
    sta.device_status(dev)
    barrier()
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    with nvtx.range("bench.timed_steps"):
        for _ in range(args.steps):
            step(record=True)
    t1.record(stream)
    barrier()
    clk = clocks.stop()
    sta.device_status(dev)
    ms = t0.elapsed_time(t1) / args.steps
    attn_ms = statistics.mean(a.elapsed_time(b) for a, b in attn_ev)
    attn_ms_median = statistics.median(a.elapsed_time(b) for a, b in attn_ev)
    ms, attn_ms = max_over_ranks([ms, attn_ms], device=dev)
    value = world * flops / (ms * 1e-3) / 1e12

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
        hout = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)

        def e2e_step():
            # the README call on host tensors: the library streams chunks of
            # heads through device staging buffers, copies overlapping compute
            sta.sliding_tile_attention_host(hq, hk, hv, w.windows, w.text_len, w.has_text,
                                            shape, w.tile, out=hout, device=dev,
                                            blocking=False)

        for _ in range(2):
            e2e_step()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(3, min(args.steps, 10))
        e0.record(stream)
        with nvtx.range("bench.e2e_steps"):
            for _ in range(n_e2e):
                e2e_step()
        e1.record(stream)
        barrier()
        e2e_ms = e0.elapsed_time(e1) / n_e2e
        (e2e_ms,) = max_over_ranks([e2e_ms], device=dev)
        nbytes = q.numel() * q.element_size()
        e2e = {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": 3 * nbytes,
               "d2h_bytes_per_step": nbytes}

    # ---- the standalone permutation kernel (raster -> tile order), HBM-bound
    perm = None
    if rank == 0:
        qt = torch.empty_like(q)
        for _ in range(3):
            sta.tile_reorder(q, shape, w.tile, w.has_text, out=qt)
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(10):
            sta.tile_reorder(q, shape, w.tile, w.has_text, out=qt)
        b.record(stream)
        torch.cuda.synchronize(dev)
        pms = a.elapsed_time(b) / 10
        nbytes = 2 * q.numel() * q.element_size()
        peaks_p, src_p = load_peaks()
        perm = {"kernel": "tile_permute_kernel<16>", "ms": pms, "gbs": nbytes / pms / 1e6,
                "frac_of_hbm": nbytes / pms / 1e6 / float(peaks_p["hbm_gbs"]),
                "bytes": nbytes, "peak_source": src_p}
        # the same attention on tile-ordered tensors (the permutation timed
        # apart, above): tile lists + attention, 2-D TMA boxes, tile-order out
        kt, vt = (sta.tile_reorder(x, shape, w.tile, w.has_text) for x in (k, v))
        ot = torch.empty_like(qt)
        for _ in range(3):
            sta.forward(qt, kt, vt, w.windows, w.text_len, w.has_text, shape, w.tile, out=ot)
        torch.cuda.synchronize(dev)
        a.record(stream)
        for _ in range(10):
            sta.forward(qt, kt, vt, w.windows, w.text_len, w.has_text, shape, w.tile, out=ot)
        b.record(stream)
        torch.cuda.synchronize(dev)
        sta.device_status(dev)
        tms = a.elapsed_time(b) / 10
        perm["attention_tile_order"] = {"ms": tms, "effective_tflops": flops / (tms * 1e-3) / 1e12,
                                        "pct_of_bf16_peak": 100.0 * flops / (tms * 1e-3) / 1e12 /
                                        float(peaks_p["bf16_tflops"])}
        del qt, kt, vt, ot

    # ---- token-level sliding-window comparison (mixed blocks), same kernel family
    swa = None
    if rank == 0 and not args.no_swa:
        sw = workloads.SWA_GQA
        sq, sk, sv = workloads.swa_inputs(sw, device=dev)
        so = torch.empty_like(sq)
        for _ in range(3):
            sta.swa_forward(sq, sk, sv, sw.window, True, out=so)
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(10):
            sta.swa_forward(sq, sk, sv, sw.window, True, out=so)
        b.record(stream)
        torch.cuda.synchronize(dev)
        swa_ms = a.elapsed_time(b) / 10
        s_pairs = sw.hq * (sw.window * (sw.window + 1) // 2 + (sw.S - sw.window) * sw.window)
        swa_flops = 4.0 * sw.d * s_pairs
        # STA on the same geometry with 3 heads: about the same retained FLOPs
        wins3 = w.windows[:3]
        m_q, m_k, m_v = (x[:, :3].contiguous() for x in (q, k, v))
        m_o = torch.empty_like(m_q)
        for _ in range(3):
            sta.forward_raster(m_q, m_k, m_v, wins3, w.text_len, w.has_text, shape, w.tile,
                               out=m_o)
        torch.cuda.synchronize(dev)
        a.record(stream)
        for _ in range(10):
            sta.forward_raster(m_q, m_k, m_v, wins3, w.text_len, w.has_text, shape, w.tile,
                               out=m_o)
        b.record(stream)
        torch.cuda.synchronize(dev)
        sta3_ms = a.elapsed_time(b) / 10
        sta3_flops = 4.0 * w.d * sta.retained_pairs(1, wins3, shape, w.tile, w.text_len,
                                                    w.has_text)
        # token-level 3-D sliding window with the same (18,24,24)-token
        # window on the same workload: identical retained pairs, mixed blocks
        win_tok = tuple(wa * ta for wa, ta in zip(w.windows[0], w.tile))
        for _ in range(2):
            sta.swa3d_forward(q, k, v, win_tok, w.text_len, w.has_text, shape, w.tile, out=out)
        torch.cuda.synchronize(dev)
        a.record(stream)
        for _ in range(3):
            sta.swa3d_forward(q, k, v, win_tok, w.text_len, w.has_text, shape, w.tile, out=out)
        b.record(stream)
        torch.cuda.synchronize(dev)
        s3_ms = a.elapsed_time(b) / 3
        sta.device_status(dev)
        swa = {"workload": sw.name, "ms": swa_ms,
               "effective_tflops": swa_flops / (swa_ms * 1e-3) / 1e12,
               "sta_matched": {"heads": 3, "ms": sta3_ms,
                               "effective_tflops": sta3_flops / (sta3_ms * 1e-3) / 1e12},
               "token_window_3d": {"workload": w.name, "window_tokens": list(win_tok),
                                   "ms": s3_ms,
                                   "effective_tflops": flops / (s3_ms * 1e-3) / 1e12,
                                   "sta_speedup": s3_ms / ms}}
        del sq, sk, sv, so, m_q, m_k, m_v, m_o

        # Hilbert-order vs raster-order block-sparse 2-D slide attention on the
        # 2-D image workload's shape (256 x 256 tokens, 8 x 16 heads, d=64),
        # 21 x 21 token window; inputs already in each order.
        iw = workloads.IMAGE_2D
        n2, w2 = iw.W, 21
        hq, hk, hv = workloads.sta_inputs(iw, device=dev)
        ho = torch.empty_like(hq)
        pairs2 = iw.B * iw.heads * n2 * n2 * w2 * w2
        hil = {"workload": f"image2d_{n2}x{n2}_slide{w2}", "window": w2}
        for order in ("raster", "hilbert"):
            counts, ids, cls = sta.build_slide_block_lists(n2, w2, order, device=dev)
            nonempty = int(counts.sum())
            partial = int((cls == 1).sum())
            for _ in range(2):
                sta.slide2d_forward(hq, hk, hv, n2, w2, order, out=ho)
            torch.cuda.synchronize(dev)
            a.record(stream)
            for _ in range(5):
                sta.slide2d_forward(hq, hk, hv, n2, w2, order, out=ho)
            b.record(stream)
            torch.cuda.synchronize(dev)
            t2 = a.elapsed_time(b) / 5
            hil[order] = {"ms": t2, "effective_tflops": 4.0 * iw.d * pairs2 / (t2 * 1e-3) / 1e12,
                          "nonempty_blocks": nonempty, "partial_blocks": partial,
                          "full_blocks": nonempty - partial}
        hil["hilbert_speedup"] = hil["raster"]["ms"] / hil["hilbert"]["ms"]
        sta.device_status(dev)
        swa["hilbert_slide2d"] = hil
        del hq, hk, hv, ho

        # backward pass of the same STA workload
        swa["backward"] = run_backward(q, k, v, w, shape, pairs, dev, stream)

    others = None
    if rank == 0 and not args.no_other_configs:
        peaks_o, _ = load_peaks()
        others = run_other_configs(dev, stream, float(peaks_o["bf16_tflops"]))

    peaks, peak_src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    achieved = flops / (attn_ms * 1e-3) / 1e12
    # per-launch key blocks x query blocks processed (units of the traffic file)
    units = pairs / (128 * 128)
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": attn_traffic(units),
                "kernel": "attn_fwd_kernel<128,kSta,raster>",
                "peak_source": peak_src + " burst bf16",
                "attn_ms": attn_ms, "attn_ms_median": attn_ms_median}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, desc, threads, _ = cpu_oracle_sample(w, q[0, 0].cpu(), k[0, 0].cpu(), v[0, 0].cpu(),
                                                 args.cpu_seconds)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": workload_config(w, world),
            "pct_of_bf16_peak": 100.0 * value / peak,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk,
            "gpu_launches": 2 * args.steps, "permutation": perm, "swa_comparison": swa,
            "other_configs": others,
        }
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.profile_workload is not None:
        return run_profile_workload(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
