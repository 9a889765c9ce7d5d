"""Benchmark of the SSTA forward hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = the whole forward on one synthetic problem: tile_reorder of q, k
and v, build_block_mask, attention_fwd and tile_unorder of O, all through the C
ABI on one stream, inputs already resident in HBM.  Steps cycle over the
workload's seeds.  Every input tensor (about 0.9 GB each) is larger than the
126 MB L2, so no flush is needed between steps.

Reported metric: effective TFLOP/s on kept blocks = 4*D*sum over kept
(query tile, key tile) pairs of rows(query tile)*rows(key tile) per step,
divided by the step time.  With N GPUs (torchrun), every rank runs its own
problem (weak scaling, no collective on the data path); the time is the max
over ranks and the FLOPs are summed.

``--impl reference`` times the CPU oracle instead (rank 0 only, a bounded
sample of the same workload per step).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SSTA fwd ms/call & effective TFLOPS (kept blocks) at 720p-10s latent; % bf16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
LAUNCHES_PER_STEP = 8   # 3 reorder + pool + scores + select-and-list + attention + unorder
                        # (+ norms and redundancy with the importance score)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def load_traffic(kernel_file, w):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current kernel
    source and on this workload (name and head count)."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    src = os.path.join(ROOT, "block_sparse_video_ssta_b200", "csrc", kernel_file)
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    e = d.get(kernel_file, {})
    if e.get("source_sha256_16") == h and e.get("workload") == w.name and e.get("heads", 16) == w.H:
        return e.get("dram_bytes_per_launch")
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id):
        self.bus_id = bus_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", self.bus_id], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
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
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def tile_rows(g_nt, g_ntext, N, L_text):
    import numpy as np
    rows = np.full(g_nt + g_ntext, N, dtype=np.float64)
    if g_ntext:
        rows[-1] = L_text - (g_ntext - 1) * N
    return rows


def valid_rows(w, N, nT, nY, nX, n_text):
    import numpy as np
    vt = np.minimum(w.tT, w.T - np.arange(nT) * w.tT)
    vy = np.minimum(w.tY, w.Y - np.arange(nY) * w.tY)
    vx = np.minimum(w.tX, w.X - np.arange(nX) * w.tX)
    v = (vt[:, None, None] * vy[None, :, None] * vx[None, None, :]).reshape(-1).astype(np.float64)
    if n_text:
        t = np.full(n_text, N, dtype=np.float64)
        t[-1] = w.L_text - (n_text - 1) * N
        v = np.concatenate([v, t])
    return v


def kept_flops(w, plan, kv_idx, kv_cnt):
    """(padded, valid) FLOPs of the kept blocks of one problem, from the compact lists."""
    import numpy as np
    N = plan.tile_tokens
    nT, nY, nX = -(-w.T // w.tT), -(-w.Y // w.tY), -(-w.X // w.tX)
    rows = tile_rows(plan.num_tiles, plan.num_text_tiles, N, w.L_text)
    vrows = valid_rows(w, N, nT, nY, nX, plan.num_text_tiles)
    idx = kv_idx.cpu().numpy()
    ok = idx >= 0
    safe = np.where(ok, idx, 0)
    cols = np.where(ok, rows[safe], 0.0).sum(-1)          # [B,H,NQ]
    vcols = np.where(ok, vrows[safe], 0.0).sum(-1)
    padded = 4.0 * w.D * float((cols * rows[None, None, :]).sum())
    valid = 4.0 * w.D * float((vcols * vrows[None, None, :]).sum())
    return padded, valid


def issued_flops(w, plan, kv_idx):
    """FLOPs the tensor-core attention kernel issues for one problem: every query tile
    is computed on all N of its rows (128-row halves), and a kept key tile on each of
    its 128-key chunks that holds at least one valid key (pad-only chunks are skipped).
    4*D*N*128 per (query tile, kept chunk)."""
    import numpy as np
    N = plan.tile_tokens
    nT, nY, nX = -(-w.T // w.tT), -(-w.Y // w.tY), -(-w.X // w.tX)
    o = np.arange(N)
    dt, dy, dx = o // (w.tX * w.tY), (o // w.tX) % w.tY, o % w.tX
    vt = np.minimum(w.tT, w.T - np.arange(nT) * w.tT)
    vy = np.minimum(w.tY, w.Y - np.arange(nY) * w.tY)
    vx = np.minimum(w.tX, w.X - np.arange(nX) * w.tX)
    valid = ((dt[None, None, None, :] < vt[:, None, None, None]) & (dy[None, None, None, :] < vy[None, :, None, None])
             & (dx[None, None, None, :] < vx[None, None, :, None])).reshape(-1, N // 128, 128)
    chunks = valid.any(-1).sum(-1).astype(np.float64)                       # [NT]
    if plan.num_text_tiles:
        rem = w.L_text - np.arange(plan.num_text_tiles) * N
        chunks = np.concatenate([chunks, np.ceil(np.minimum(rem, N) / 128.0)])
    idx = kv_idx.cpu().numpy()
    ok = idx >= 0
    per_row = np.where(ok, chunks[np.where(ok, idx, 0)], 0.0).sum(-1)       # kept chunks per query tile
    return 4.0 * w.D * N * 128.0 * float(per_row.sum())


def pci_bus_id(dev):
    import torch
    p = torch.cuda.get_device_properties(dev)
    try:
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except AttributeError:
        return str(dev)


# --------------------------------------------------------------------------- CPU oracle
def oracle_sample(w, x_cpu, heads=(0,), tile_stride=64, max_seconds=None):
    """Time the CPU oracle on a bounded sample: the full mask of the given heads plus
    attention on every tile_stride-th video query tile and the text tiles.
    Returns (seconds, kept-block FLOPs of the attended sample, description)."""
    import numpy as np
    import oracle
    g = oracle.geometry(w)
    t0 = time.perf_counter()
    conv = lambda t: None if t is None else t.float().numpy().astype(np.float64)
    q, k, v = (conv(x_cpu[n]) for n in ("q", "k", "v"))
    qt, kt, vt = (conv(x_cpu[n]) for n in ("q_text", "k_text", "v_text"))
    qp, kp, vp = oracle.tile_reorder(w, q, qt), oracle.tile_reorder(w, k, kt), oracle.tile_reorder(w, v, vt)
    S64 = oracle.block_scores(w, oracle.tile_pool(w, qp), oracle.tile_pool(w, kp))
    kept = oracle.kept_mask(w, oracle.select_topk(w, S64))
    tiles = list(range(0, g.NT, tile_stride)) + list(range(g.NT, g.NQ))
    oracle.attention(w, qp, kp, vp, kept, q_tiles=tiles)
    secs = time.perf_counter() - t0
    sub = np.zeros_like(kept)
    sub[:, :, tiles] = kept[:, :, tiles]
    flops = oracle.attention_flops(w, sub)
    desc = (f"heads {list(heads)} of seed 0: reorder+pool+scores+top-k+window of the head, attention on "
            f"{len(tiles)} of {g.NQ} query tiles (every {tile_stride}th video tile + text tiles)")
    return secs, flops, desc


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_inputs(w, seed, heads):
    import ssta_inputs as si
    return si.make_inputs(w, seed, device="cpu", heads=heads)


def run_reference(args):
    """--impl reference: the CPU oracle, rank 0 only.  The oracle's mask for head 0
    is built once (reorder, pool, scores, top-k, window, union; timed and
    reported); each step then runs the oracle's attention on two video query
    tiles of that head (a different pair each step) and the value is the
    kept-block FLOPs of those tiles over the step time."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np
    import oracle
    import ssta_inputs as si
    w = workload_of(args)
    wh = si.with_overrides(w, H=1)
    g = oracle.geometry(wh)
    x = cpu_inputs(w, w.seeds[0], (0,))
    conv = lambda t: None if t is None else t.float().numpy().astype(np.float64)
    t0 = time.perf_counter()
    qp, kp, vp = (oracle.tile_reorder(wh, conv(x[n]), conv(x[n + "_text"])) for n in ("q", "k", "v"))
    kept = oracle.kept_mask(wh, oracle.select_topk(wh, oracle.block_scores(
        wh, oracle.tile_pool(wh, qp), oracle.tile_pool(wh, kp))))
    mask_s = time.perf_counter() - t0
    rng = np.random.default_rng(0)
    order = rng.permutation(g.NT)

    def one(i):
        tiles = [int(order[(2 * i) % g.NT]), int(order[(2 * i + 1) % g.NT])]
        t = time.perf_counter()
        oracle.attention(wh, qp, kp, vp, kept, q_tiles=tiles)
        dt = time.perf_counter() - t
        sub = np.zeros_like(kept)
        sub[:, :, tiles] = kept[:, :, tiles]
        return dt, oracle.attention_flops(wh, sub)

    for i in range(args.warmup):
        one(i)
    secs, flops = 0.0, 0.0
    for i in range(args.steps):
        dt, f = one(args.warmup + i)
        secs += dt
        flops += f
    ms = 1000.0 * secs / args.steps
    value = flops / secs / 1e12
    cores = blas_threads()
    desc = (f"{w.name} seed {w.seeds[0]} head 0: oracle attention on 2 random video query tiles per step "
            f"(float64 numpy); the head's oracle mask took {mask_s:.2f} s once, outside the steps")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "sample": desc},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- GPU arm
def workload_of(args):
    """The named workload with the mask-mode flags applied."""
    import ssta_inputs as si
    w = si.get_workload(args.workload)
    ov = {k: v for k, v in (("score_mode", args.score_mode), ("combine", args.combine),
                            ("window_mode", args.window_mode), ("H", args.heads)) if v is not None}
    return si.with_overrides(w, **ov) if ov else w


def rank_seeds(rank, base_seeds):
    """Weak scaling: rank r solves its own independent problems, seeds r*1000 + s."""
    return [rank * 1000 + s for s in base_seeds]


def reduce_over_ranks(times_ms, work, device, world):
    """Whole-job figures: every time is the max over ranks, every amount of work
    the sum over ranks (one all-reduce each; identity for a single rank)."""
    import torch
    import torch.distributed as dist
    tot = torch.tensor(times_ms, dtype=torch.float64, device=device)
    fl = torch.tensor(work, dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(tot, op=dist.ReduceOp.MAX)
        dist.all_reduce(fl, op=dist.ReduceOp.SUM)
    return tot.tolist(), fl.tolist()


def job_value(flops, ms):
    """TFLOP/s of `flops` done in `ms` milliseconds."""
    return flops / (ms / 1000.0) / 1e12


def run_gpu(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import block_sparse_video_ssta_b200 as S
    import ssta_inputs as si

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    w = workload_of(args)
    d = S.desc_from(w)
    plan = S.ssta_plan(d)
    seeds = rank_seeds(rank, w.seeds)
    stream = torch.cuda.current_stream(dev)

    # per-seed resident inputs and preallocated outputs
    probs = []
    for s in seeds:
        x = si.make_inputs(w, s, device=dev)
        qp = torch.empty((w.B, w.H, plan.packed_len, w.D), dtype=torch.bfloat16, device=dev)
        kp, vp, op = torch.empty_like(qp), torch.empty_like(qp), torch.empty_like(qp)
        kv_idx = torch.empty((w.B, w.H, plan.num_q_tiles, plan.max_kept), dtype=torch.int32, device=dev)
        kv_cnt = torch.empty((w.B, w.H, plan.num_q_tiles), dtype=torch.int32, device=dev)
        ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=dev)
        ws_a = torch.empty(plan.attn_workspace_bytes, dtype=torch.uint8, device=dev)
        lse = torch.empty((w.B, w.H, plan.packed_len), dtype=torch.float32, device=dev)
        o = torch.empty_like(x["q"])
        o_t = torch.empty_like(x["q_text"]) if w.L_text else None
        probs.append(dict(x=x, qp=qp, kp=kp, vp=vp, op=op, kv_idx=kv_idx, kv_cnt=kv_cnt, ws=ws, ws_a=ws_a,
                          lse=lse, o=o, o_t=o_t))

    def step(p, ev=None):
        x = p["x"]
        if ev:
            ev[0].record(stream)
        S.ssta_tile_reorder(d, x["q"], x["q_text"], p["qp"])
        S.ssta_tile_reorder(d, x["k"], x["k_text"], p["kp"])
        S.ssta_tile_reorder(d, x["v"], x["v_text"], p["vp"])
        if ev:
            ev[1].record(stream)
        S.ssta_build_block_mask(d, p["qp"], p["kp"], p["kv_idx"], p["kv_cnt"], workspace=p["ws"])
        if ev:
            ev[2].record(stream)
        S.ssta_attention_fwd(d, p["qp"], p["kp"], p["vp"], p["kv_idx"], p["kv_cnt"], p["op"], p["lse"],
                             workspace=p["ws_a"])
        if ev:
            ev[3].record(stream)
        S.ssta_tile_unorder(d, p["op"], p["o"], p["o_t"])
        if ev:
            ev[4].record(stream)

    for i in range(max(args.warmup, 3)):
        step(probs[i % len(probs)])
    torch.cuda.synchronize()
    for p in probs:
        st = (S.ssta_read_device_status(p["ws"]), S.ssta_read_device_status(p["ws_a"]))
        if st != (0, 0):
            raise RuntimeError(f"device status {st}")
    flops = [kept_flops(w, plan, p["kv_idx"], p["kv_cnt"]) for p in probs]
    issued = [issued_flops(w, plan, p["kv_idx"]) if (w.dtype == "bf16" and plan.tile_tokens % 128 == 0) else None
              for p in probs]

    # ---- timed region (device-resident inputs)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(pci_bus_id(dev)) as clk:
        t_start.record(stream)
        for i in range(args.steps):
            step(probs[i % len(probs)], evs[i])
        t_end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    stage = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(4)] for e in evs])   # [K, 4]
    # ---- L2 flushed vs warm samples, outside the timed region: the mask build 20 times with
    # a 256 MB write (twice the L2) before each sample, the attention 3 times flushed and 3
    # times right after a run on the same inputs (warm); medians.
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    p0 = probs[0]
    e_a, e_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(fn, pre=None):
        if pre is not None:
            pre()
        e_a.record(stream)
        fn()
        e_b.record(stream)
        torch.cuda.synchronize()
        return e_a.elapsed_time(e_b)

    mask_call = lambda: S.ssta_build_block_mask(d, p0["qp"], p0["kp"], p0["kv_idx"], p0["kv_cnt"], workspace=p0["ws"])
    attn_call = lambda: S.ssta_attention_fwd(d, p0["qp"], p0["kp"], p0["vp"], p0["kv_idx"], p0["kv_cnt"], p0["op"],
                                             p0["lse"], workspace=p0["ws_a"])
    mask_flushed = statistics.median(timed(mask_call, flush.zero_) for _ in range(20))
    mask_warm = statistics.median(timed(mask_call, mask_call) for _ in range(20))
    attn_flushed = statistics.median(timed(attn_call, flush.zero_) for _ in range(3))
    attn_warm = statistics.median(timed(attn_call, attn_call) for _ in range(3))
    del flush

    my_flops = sum(flops[i % len(probs)][0] for i in range(args.steps))
    my_vflops = sum(flops[i % len(probs)][1] for i in range(args.steps))
    attn_flops = my_flops

    # ---- e2e through the public API with host buffers (pinned): every step uploads its
    # inputs host -> device and downloads its output device -> host inside the timed region.
    # Inputs and outputs are double-buffered on the device, so the upload of step i+1 and the
    # download of step i-1 run on two copy streams while step i computes on a third.
    p0 = probs[0]
    hx = {k: (v.cpu().pin_memory() if v is not None else None) for k, v in p0["x"].items()}
    host_o = [torch.empty(p0["o"].shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    host_ot = [torch.empty(p0["o_t"].shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)] \
        if w.L_text else [None, None]
    h2d = sum(v.numel() * v.element_size() for v in hx.values() if v is not None)
    d2h = host_o[0].numel() * 2 + (host_ot[0].numel() * 2 if w.L_text else 0)
    pb = [p0, dict(p0, x={k: (torch.empty_like(v) if v is not None else None) for k, v in p0["x"].items()},
                   o=torch.empty_like(p0["o"]), o_t=torch.empty_like(p0["o_t"]) if w.L_text else None)]
    s_comp, s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of buffer b uploaded
    ev_comp = [torch.cuda.Event() for _ in range(2)]   # step on buffer b computed
    ev_out = [torch.cuda.Event() for _ in range(2)]    # output of buffer b downloaded

    def e2e_steps(n):
        for i in range(n):
            b, pi = i % 2, pb[i % 2]
            if i >= 2:
                s_h2d.wait_event(ev_comp[b])           # step i-2 has finished reading buffer b
            with torch.cuda.stream(s_h2d):
                for k, v in hx.items():
                    if v is not None:
                        pi["x"][k].copy_(v, non_blocking=True)
                ev_in[b].record(s_h2d)
            s_comp.wait_event(ev_in[b])
            if i >= 2:
                s_comp.wait_event(ev_out[b])           # step i-2's output has left buffer b
            with torch.cuda.stream(s_comp):
                step(pi)
                ev_comp[b].record(s_comp)
            s_d2h.wait_event(ev_comp[b])
            with torch.cuda.stream(s_d2h):
                host_o[b].copy_(pi["o"], non_blocking=True)
                if w.L_text:
                    host_ot[b].copy_(pi["o_t"], non_blocking=True)
                ev_out[b].record(s_d2h)

    e2e_steps(2)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_h2d)
    e2e_steps(args.steps)
    s_h2d.wait_stream(s_d2h)
    e1.record(s_h2d)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    e2e_flops = flops[0][0] * args.steps

    # ---- reduce over ranks
    (max_ms, max_e2e_ms), (all_flops, all_vflops, all_e2e_flops) = reduce_over_ranks(
        [elapsed_ms, e2e_ms], [my_flops, my_vflops, e2e_flops], dev, world)
    value = job_value(all_flops, max_ms)
    e2e_value = job_value(all_e2e_flops, max_e2e_ms)

    if rank == 0:
        peaks, src = load_peaks()
        attn_ms = float(np.median(stage[:, 2]))
        mask_ms = float(np.median(stage[:, 1]))
        reorder_ms = float(np.median(stage[:, 0]))
        unorder_ms = float(np.median(stage[:, 3]))
        attn_ms_mean = float(stage[:, 2].mean())
        per_call_flops = attn_flops / args.steps
        achieved = per_call_flops / (attn_ms_mean / 1000.0) / 1e12
        per_call_issued = (sum(issued[i % len(probs)] for i in range(args.steps)) / args.steps
                           if issued[0] is not None else None)
        peak_sus = float(peaks["bf16_tflops_sustained"])
        peak_burst = float(peaks["bf16_tflops"])
        hbm = float(peaks["hbm_gbs"])
        valid_tokens = w.B * w.H * w.T * w.Y * w.X
        mask_bytes = 2 * valid_tokens * w.D * 2   # valid video q and k rows read once (bf16)
        mask_gbs = mask_bytes / (mask_ms / 1000.0) / 1e9
        reorder_bytes = 3 * 2 * w.B * w.H * (w.T * w.Y * w.X + w.L_text) * w.D * 2 + \
            3 * w.B * w.H * (plan.packed_len - w.T * w.Y * w.X - w.L_text) * w.D * 2
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            xc = cpu_inputs(w, seeds[0], (0,))
            wh = si.with_overrides(w, H=1)
            secs, f, desc = oracle_sample(wh, xc, (0,), tile_stride=12)
            cpu = {"value": f / secs / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                   "sample": desc, "seconds": secs}
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": max_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "heads": w.H, "head_dim": w.D,
                       "grid": [w.T, w.Y, w.X], "tile": [w.tT, w.tY, w.tX], "window": [w.wT, w.wY, w.wX],
                       "topk": w.topk, "text_tokens": w.L_text, "seeds_per_rank": seeds,
                       "mask": {"score": w.score_mode, "combine": w.combine, "window": w.window_mode},
                       "parallelism": f"dp{world} (one independent problem per rank)",
                       "l2": "no flush: every input tensor (0.9-1.0 GB) is larger than the 126 MB L2"},
            "roofline": {"bound": "tensor", "kernel": "ssta_attention_tc_kernel", "achieved": achieved,
                         "peak": peak_burst, "unit": "TFLOP/s", "frac": achieved / peak_burst,
                         "peak_source": (f"{src} bf16_tflops (burst: the kernel runs at the SM clock of "
                                         f"'clocks', not at the power-capped clock of the sustained figure)"),
                         "work": "kept-block FLOPs per launch (4*D*rows*rows per kept tile pair, tiles as laid "
                                 "out) / mean CUDA-event duration of the launch",
                         "frac_of_sustained_peak": achieved / peak_sus,
                         "issued_tflop_per_call": None if per_call_issued is None else per_call_issued / 1e12,
                         "issued_achieved": (None if per_call_issued is None
                                             else per_call_issued / (attn_ms_mean / 1000.0) / 1e12),
                         "issued_frac": (None if per_call_issued is None
                                         else per_call_issued / (attn_ms_mean / 1000.0) / 1e12 / peak_burst),
                         "traffic": load_traffic("ssta_attn_tc.cu", w)},
            "stages_ms": {"tile_reorder_qkv": reorder_ms, "build_block_mask": mask_ms, "attention_fwd": attn_ms,
                          "tile_unorder_o": unorder_ms, "statistic": f"median of {args.steps} steps",
                          "attention_fwd_mean": attn_ms_mean},
            "l2_samples_ms": {"build_block_mask_flushed": mask_flushed, "build_block_mask_warm": mask_warm,
                              "attention_fwd_flushed": attn_flushed, "attention_fwd_warm": attn_warm,
                              "how": "outside the timed region, seed " + str(seeds[0]) + ": 256 MB written "
                                     "before each flushed sample; warm = right after a run on the same inputs; "
                                     "medians of 20 (mask) and 3 (attention)"},
            "mask_roofline": {"bound": "hbm", "achieved": mask_gbs, "peak": hbm, "unit": "GB/s",
                              "frac": mask_gbs / hbm, "algorithmic_bytes": mask_bytes,
                              "peak_source": f"{src} hbm_gbs",
                              "flushed_achieved": mask_bytes / (mask_flushed / 1000.0) / 1e9,
                              "flushed_frac": mask_bytes / (mask_flushed / 1000.0) / 1e9 / hbm},
            "reorder_gbs": (reorder_bytes / (reorder_ms / 1000.0) / 1e9),
            "kept_tflop_per_call": per_call_flops / 1e12,
            "valid_tflop_per_call": (my_vflops / args.steps) / 1e12,
            "valid_tflops": job_value(all_vflops, max_ms),
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": max_e2e_ms / args.steps,
                    "copies": "pinned host buffers; uploads and downloads on two copy streams, overlapped with "
                              "the previous/next step's compute through double-buffered device inputs and outputs"},
            "gpu_launches": (LAUNCHES_PER_STEP + (2 if w.score_mode == "importance" else 0)) * args.steps,
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_backward(args):
    """Time the backward (dQ, dK, dV) on one GPU: inputs, O, LSE, kept lists and dO resident;
    effective TFLOP/s = 2.5 x the forward's kept-block FLOPs (five products instead of two)."""
    import torch
    import block_sparse_video_ssta_b200 as S
    import ssta_inputs as si
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = workload_of(args)
    d = S.desc_from(w)
    plan = S.ssta_plan(d)
    x = si.make_inputs(w, w.seeds[0], device=dev)
    r = S.ssta_forward(d, x["q"], x["k"], x["v"], x["q_text"], x["k_text"], x["v_text"])
    dO = torch.randn(r["O_packed"].shape, device=dev, generator=torch.Generator(device=dev).manual_seed(5)
                     ).to(r["O_packed"].dtype)
    outs = [torch.empty_like(dO) for _ in range(3)]
    ws = torch.empty(plan.bwd_workspace_bytes, dtype=torch.uint8, device=dev)
    call = lambda: S.ssta_attention_bwd(d, r["qp"], r["kp"], r["vp"], r["O_packed"], r["LSE"], dO,
                                        r["kv_idx"], r["kv_cnt"], *outs, workspace=ws)
    for _ in range(max(args.warmup, 3)):
        call()
    torch.cuda.synchronize()
    assert S.ssta_read_device_status(ws) == 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(pci_bus_id(dev)) as clk:
        e0.record()
        for _ in range(args.steps):
            call()
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    fwd_flops, _ = kept_flops(w, plan, r["kv_idx"], r["kv_cnt"])
    tflops = 2.5 * fwd_flops / (ms / 1000.0) / 1e12
    peaks, src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    peak_sus = float(peaks["bf16_tflops_sustained"])
    line = {
        "metric": "SSTA bwd ms/call & effective TFLOPS (2.5x kept-block forward FLOPs)", "value": tflops,
        "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "pass": "backward", "grid": [w.T, w.Y, w.X], "heads": w.H,
                   "mask": {"score": w.score_mode, "combine": w.combine, "window": w.window_mode},
                   "kernels": ("tcgen05 tensor cores (dQ and dK/dV kernels)" if w.dtype == "bf16" and (w.tX * w.tY * w.tT) % 128 == 0
                               else "SIMT (fp32 storage)")},
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s", "frac": tflops / peak,
                     "peak_source": f"{src} bf16_tflops (burst; the clock record is beside it)",
                     "frac_of_sustained_peak": tflops / peak_sus, "traffic": None},
        "gpu_launches": 4 * args.steps, "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ssta", choices=["ssta", "reference"])
    ap.add_argument("--workload", default="p720_10s_bf16")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--score-mode", default=None, choices=["similarity", "importance"],
                    help="block score ranked by top-k (default: the workload's, similarity)")
    ap.add_argument("--combine", default=None, choices=["union", "and"])
    ap.add_argument("--window-mode", default=None, choices=["shift", "truncate"])
    ap.add_argument("--heads", type=int, default=None,
                    help="run the workload with this many heads (small profiling cases; not a headline run)")
    ap.add_argument("--backward", action="store_true",
                    help="time ssta_attention_bwd instead of the forward (prints its own line)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.backward:
        return run_backward(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
