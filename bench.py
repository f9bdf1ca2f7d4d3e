#!/usr/bin/env python
"""Benchmark of the Ca2-VDM cached attention path on B200.

One step = one autoregressive step at steady state of the Open-Sora-v1.0-shaped attention
layer with the full Pmax = 41 queue (B=1, 256 tokens/frame, 16 heads x 72, chunk l = 8,
P' = 3, T = 50 denoising steps): for each of the 28 blocks of the backbone (each with its
own cache, as in the model), T denoising passes of prefix-spatial + causal temporal
attention reading the shared cache, then the cache-writing pass (self-repeat spatial +
temporal), eviction of the 8 oldest frames, the cache write for all blocks, and the
chunk's cyclic TPE indices.  28 per-block caches plus their inputs (~2.4 GB) keep every
read coming from HBM (inputs larger than L2).

Metric: attention query tokens per second -- each pass moves B*l*HW = 2048 query tokens
through one block's spatial + temporal attention, so a step counts (T+1) * 28 * 2048.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]

Under torchrun each rank runs the same step on its own GPU with its own caches (videos
are independent; no data-path collective); value = all ranks' tokens / max rank time.

  python bench.py --shard heads [...]

splits the heads instead (tensor-parallel attention): rank r of N owns the contiguous heads
ca2_head_shard gives it, keeps caches for those heads only and runs them on full-width
activations through the row pitch, again with no collective on the path (attention never
mixes heads); the whole job processes each step's tokens once (strong scaling).  On one
process, --shard-world G --shard-rank r times rank r's share of a G-way split alone.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attn query-tokens/s per denoise step; temporal HBM GB/s; spatial TFLOP/s vs peak"
WORKLOAD = dict(batch=1, hw=256, heads=16, head_dim=72, chunk_len=8, p_max=41, p_spatial=3,
                n_layers=28, denoise_steps=50)
WORKLOAD_NAME = ("Open-Sora-shaped attention layer, Pmax=41 full queue (steady-state AR step of the "
                 "80-frame run), 28 per-block caches")
# The Ca2-VDM settings timed by --config (Open-Sora v1.0 backbone: C = 1152 in 16 heads of 72,
# chunk l = 8, P' = 3, T = 50): one AR step at the configuration's steady state, every block's
# queue at Pmax.  The default is os_p41.
CONFIGS = {
    "os_p41": dict(batch=1, hw=256, p_max=41, name=WORKLOAD_NAME),
    "os_p25": dict(batch=1, hw=256, p_max=25,
                   name="Open-Sora-shaped attention layer, Pmax=25 full queue (P in {1, 9, 17, 25}), "
                        "28 per-block caches"),
    "os_28blk_b4": dict(batch=4, hw=256, p_max=41,
                        name="attention sub-path of the 28-block backbone, B=4 videos, Pmax=41 full queue"),
    "hires": dict(batch=2, hw=1024, p_max=41,
                  name="512x512 video (32x32 = 1024 tokens/frame), B=2, Pmax=41 full queue, "
                       "spatial map 1024 x 4096"),
}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ca2", choices=["ca2", "reference"])
    ap.add_argument("--config", default="os_p41", choices=sorted(CONFIGS),
                    help="which Ca2-VDM setting one step runs (default os_p41, the Pmax=41 layer)")
    ap.add_argument("--layers", type=int, default=WORKLOAD["n_layers"])
    ap.add_argument("--denoise", type=int, default=WORKLOAD["denoise_steps"])
    ap.add_argument("--shard", default="none", choices=["none", "heads"],
                    help="none: every rank runs the whole step (replicas, weak scaling); heads: the ranks "
                         "split the heads of every block (strong scaling)")
    ap.add_argument("--shard-world", type=int, default=0,
                    help="with --shard heads in a single process: the number of head groups to split into")
    ap.add_argument("--shard-rank", type=int, default=0,
                    help="with --shard-world: which group this process runs")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mode", default="step", choices=["step", "recompute", "per-timestep", "cpu-baseline"],
                    help="step: the timed AR step (default); recompute: cached vs recompute-from-scratch "
                         "attention per denoising step along the 80-frame run; per-timestep: one shared "
                         "cache vs one cache per denoising step (memory and AR-step time); cpu-baseline: "
                         "the oracle per call, one thread and all host threads, at every queue length")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


# ------------------------------------------------------------------------------------
class Clocks:
    """nvidia-smi samples every 200 ms while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = tempfile.mktemp(suffix=".csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.Q,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def source_sha(name: str) -> str:
    with open(os.path.join(ROOT, "causal_kv_cache_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def committed_traffic(kernel_file: str):
    """dram bytes per launch from the committed ncu summary, if the kernel is unchanged."""
    try:
        with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
            d = json.load(f)
        e = d.get(kernel_file)
        if e and e.get("source_sha") == source_sha(kernel_file):
            return e.get("bytes_per_launch")
    except Exception:
        pass
    return None


def max_over_ranks(ms: float, dist, world: int, device) -> float:
    """The slowest rank's time: every rank contributes its own device-timed milliseconds and
    all receive the maximum (a no-op on one rank)."""
    if world <= 1:
        return ms
    import torch
    tt = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def job_tokens_per_step(tokens_per_step: int, sharded: bool, world: int, heads: int, heads_all: int) -> float:
    """Query tokens the whole job moves through attention per step: every replica its own; a
    head split over `world` ranks moves each token once over all of them; one group of a split
    timed alone (world 1) counts its heads' share of each token."""
    if not sharded:
        return tokens_per_step * world
    if world > 1:
        return tokens_per_step
    return tokens_per_step * heads / heads_all


def whole_job_rate(tokens_per_step: int, steps: int, world: int, ms: float) -> float:
    """Query tokens per second of the whole job: every rank's tokens over the slowest rank's time."""
    return tokens_per_step * steps * world / (ms / 1e3)


# ------------------------------------------------------------------------------------
def run_ca2(args):
    import torch
    import torch.distributed as dist
    from causal_kv_cache_b200 import ca2

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local)
    cfg = CONFIGS[args.config]
    W = dict(WORKLOAD, n_layers=args.layers, denoise_steps=args.denoise,
             **{k: cfg[k] for k in ("batch", "hw", "p_max")})
    B, HW, H_all, D, l, PM, PS = (W[k] for k in ("batch", "hw", "heads", "head_dim", "chunk_len", "p_max",
                                                  "p_spatial"))
    NL, T = W["n_layers"], W["denoise_steps"]
    # heads this process runs: all of them, or its group of a head split (activations stay
    # full width; the kernels get views at head h0 and the full row pitch)
    if args.shard == "heads":
        groups = world if world > 1 else max(1, args.shard_world)
        grank = rank if world > 1 else args.shard_rank
        h0, H = ca2.ca2_head_shard(H_all, groups, grank)
    else:
        groups, grank, h0, H = 1, 0, 0, H_all
    sharded = args.shard == "heads"
    hv = (lambda t: t[..., h0:h0 + H, :]) if sharded else (lambda t: t)
    plane = B * HW * H * D
    frame_bytes = plane * 2
    cache = ca2.KVCache(NL, B, HW, H, D, l, PM, PS, row_pitch=H_all * D if sharded else 0)
    g = torch.Generator(device=dev)
    g.manual_seed(1234 + (0 if sharded else rank))      # the ranks of a head split share activations

    def rnd(n, token_major=False):
        shape = (B, HW, n, H_all, D) if token_major else (B, n, HW, H_all, D)
        return (torch.randn(shape, generator=g, device=dev) * 0.7).to(torch.bfloat16)

    # per-block inputs, reused across passes: spatial tensors frame-major [B][l][HW][H][D],
    # temporal tensors token-major [B][HW][l][H][D]
    inp = [dict(sq=rnd(l), sk=rnd(l), sv=rnd(l), tq=rnd(l, True), tk=rnd(l, True), tv=rnd(l, True))
           for _ in range(NL)]
    so = [torch.empty((B, l, HW, H_all, D), dtype=torch.bfloat16, device=dev) for _ in range(NL)]
    to = [torch.empty((B, HW, l, H_all, D), dtype=torch.bfloat16, device=dev) for _ in range(NL)]
    stream = torch.cuda.current_stream()
    sp = int(stream.cuda_stream)

    # fill the queue: the first frame, then chunks of l until it holds Pmax frames
    fills = [1]
    while 1 + l * (len(fills) - 1) < PM:
        fills.append(l)
    for n in fills:
        kt = [rnd(n, True) for _ in range(NL)]
        vt = [rnd(n, True) for _ in range(NL)]
        ks = [rnd(n) for _ in range(NL)]
        vs = [rnd(n) for _ in range(NL)]
        cache.evict_for(n)
        cache.write([hv(x) for x in kt], [hv(x) for x in vt], [hv(x) for x in ks], [hv(x) for x in vs], n, sp)
    torch.cuda.synchronize()
    assert cache.state()[1] == PM

    h = cache.handle
    tempo = ca2.ca2_temporal_attn
    spat = ca2.ca2_spatial_prefix_attn
    ptr = lambda t: hv(t).data_ptr()
    P = [{k: ptr(v) for k, v in d.items()} for d in inp]
    SO = [ptr(t) for t in so]
    TO = [ptr(t) for t in to]
    g0 = [1 + l * (len(fills) - 1)]
    # device input/output sets the step can run on (the end-to-end run adds a second one so
    # that copies overlap compute); cur[0] selects the set the next step captures
    sets = [dict(P=P, SO=SO, TO=TO)]
    cur = [0]

    def add_set(inp_b, so_b, to_b):
        sets.append(dict(P=[{k: ptr(v) for k, v in d.items()} for d in inp_b], SO=[ptr(t) for t in so_b],
                         TO=[ptr(t) for t in to_b]))
        return len(sets) - 1

    cap = torch.cuda.Stream(device=dev)
    cap_sp = int(cap.cuda_stream)
    live_graphs = []

    def capture(use_prefix, timed):
        """One pass over the 28 blocks (spatial then temporal attention per block) captured
        into a CUDA graph.  A timed capture groups the pass by kernel instead: the 28
        spatial launches between two event nodes, then the 28 temporal launches before a
        third, so each kernel's mean device time is measured without host gaps or per-launch
        event overhead (the synthetic inputs of different calls do not depend on each other,
        so the order within a pass does not change the work)."""
        graph = torch.cuda.CUDAGraph()
        evs = []
        S = sets[cur[0]]
        P, SO, TO = S["P"], S["SO"], S["TO"]
        with torch.cuda.stream(cap):
            graph.capture_begin()
            if timed:
                e0, e1, e2 = (torch.cuda.Event(enable_timing=True, external=True) for _ in range(3))
                e0.record(cap)
                for L in range(NL):
                    p = P[L]
                    spat(h, L, p["sq"], p["sk"], p["sv"], SO[L], l, use_prefix, cap_sp)
                e1.record(cap)
                for L in range(NL):
                    p = P[L]
                    tempo(h, L, p["tq"], p["tk"], p["tv"], TO[L], l, cap_sp)
                e2.record(cap)
                evs.append(("den" if use_prefix else "self", e0, e1, e2))
            else:
                for L in range(NL):
                    p = P[L]
                    spat(h, L, p["sq"], p["sk"], p["sv"], SO[L], l, use_prefix, cap_sp)
                    tempo(h, L, p["tq"], p["tk"], p["tv"], TO[L], l, cap_sp)
            graph.capture_end()
        live_graphs.append(graph)
        return graph, evs

    def step(ev=None):
        """One AR step: TPE indices, T denoising passes, the cache-writing pass, evict, write.

        The queue state is fixed until the write, so each pass is a CUDA graph captured
        once per step.  Pass 0 and the cache-writing pass replay timed graphs (launches
        grouped by kernel between event nodes); passes 1..T-1 replay the plain denoising
        graph."""
        ca2.ca2_tpe_indices(h, g0[0], 0, l)
        g_den, _ = capture(1, False)
        g_den_t, e_den = capture(1, True)
        g_self_t, e_self = capture(0, True)
        g_den_t.replay()
        for t in range(1, T):
            g_den.replay()
        g_self_t.replay()
        cache.evict_for(l)
        if ev is not None:
            ev.extend(e_den + e_self)
            e3, e4 = (torch.cuda.Event(enable_timing=True) for _ in range(2))
            e3.record(stream)
        P = sets[cur[0]]["P"]
        ca2.ca2_cache_write(h, [P[L]["tk"] for L in range(NL)], [P[L]["tv"] for L in range(NL)],
                            [P[L]["sk"] for L in range(NL)], [P[L]["sv"] for L in range(NL)], l, sp)
        if ev is not None:
            e4.record(stream)
            ev.append(("write", e3, e4, None))
        g0[0] += l

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    live_graphs.clear()          # graphs are released only once their replays are done
    st = ca2.ca2_device_status()
    if st != 0:
        raise RuntimeError("device status %d after warm-up" % st)

    clocks = Clocks(local)
    ev = []
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step(ev)
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    live_graphs.clear()
    ms = max_over_ranks(t0.elapsed_time(t1), dist, world, dev)
    st = ca2.ca2_device_status()
    if st != 0:
        raise RuntimeError("device status %d after the timed region" % st)

    sp_den, sp_self, tp_ms, wr_ms = [], [], [], []
    for kind, a, b_, c in ev:
        if kind == "write":
            wr_ms.append(a.elapsed_time(b_))
            continue
        (sp_den if kind == "den" else sp_self).append(a.elapsed_time(b_) / NL)
        tp_ms.append(b_.elapsed_time(c) / NL)
    resident_gb = (cache.tbuf.numel() + cache.sbuf.numel() + NL * 8 * B * l * HW * H_all * D) * 2 / 1e9
    launches_per_step = (T + 1) * NL * 2 + 1
    tokens_per_step = (T + 1) * NL * B * l * HW
    job_tokens = job_tokens_per_step(tokens_per_step, sharded, world, H, H_all)
    value = whole_job_rate(job_tokens, args.steps, 1, ms)

    # ---- cyclic TPE add (a next-row kernel, timed on its own, outside the step) ----
    # 28 launches (one per block's temporal input) in a CUDA graph, replayed 5 times
    tpe_table = (torch.randn((cache.tpe_len, H_all, D), generator=g, device=dev) * 0.7).to(torch.bfloat16)
    tpe_out = [torch.empty((B, HW, l, H_all, D), dtype=torch.bfloat16, device=dev) for _ in range(NL)]
    gt = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        gt.capture_begin()
        for L in range(NL):
            ca2.ca2_tpe_add(h, g0[0], 0, ptr(tpe_table), P[L]["tq"], ptr(tpe_out[L]), l, cap_sp)
        gt.capture_end()
    gt.replay()
    torch.cuda.synchronize()
    ta, tb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ta.record(stream)
    for _ in range(5):
        gt.replay()
    tb.record(stream)
    torch.cuda.synchronize()
    avg_tpe = ta.elapsed_time(tb) / 1e3 / (5 * NL)
    del gt

    # ---- K/V projection with the cache write fused (a next-row kernel, timed on its own) ----
    # one launch per block: the cache-writing pass's temporal and spatial K/V projections
    # (random weights per block, bias included) stored straight into the ring and spatial
    # cache; 28 launches in a CUDA graph, replayed 5 times.  The queue is full, so 8 frames
    # are evicted first and committed back afterwards (the same queue length as the step).
    # the projection's input rows are the full hidden state (Cin = H_all*D, the row pitch);
    # its outputs are this process's heads' K and V channels
    C, Cin = H * D, H_all * D
    n_sp = min(PS, l)
    wk = [[(torch.randn((2 * C, Cin), generator=g, device=dev) * Cin ** -0.5).to(torch.bfloat16)
           for _ in range(2)] for _ in range(NL)]
    bk = [(torch.randn((2 * C,), generator=g, device=dev) * 0.1).to(torch.bfloat16) for _ in range(NL)]
    cache.evict_for(l)
    gp = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        gp.capture_begin()
        for L in range(NL):
            ca2.ca2_kv_proj_write(h, L, inp[L]["tk"], wk[L][0], bk[L], inp[L]["sk"], wk[L][1], bk[L], l, cap_sp)
        gp.capture_end()
    gp.replay()
    torch.cuda.synchronize()
    ta.record(stream)
    for _ in range(5):
        gp.replay()
    tb.record(stream)
    torch.cuda.synchronize()
    avg_proj = ta.elapsed_time(tb) / 1e3 / (5 * NL)
    cache.commit(l)
    assert ca2.ca2_device_status() == 0
    # context, not the product: the same two products as plain library GEMMs (torch matmul of
    # the rows by the weights, no bias, no cache write), 28 pairs in a graph, replayed 5 times
    xs_rows = [inp[L]["sk"].reshape(B, l, HW, Cin)[:, l - n_sp:].reshape(-1, Cin) for L in range(NL)]
    xt_rows = [inp[L]["tk"].reshape(-1, Cin) for L in range(NL)]
    ref_out = [[torch.empty((t.shape[0], 2 * C), dtype=torch.bfloat16, device=dev) for t in (xt_rows[L], xs_rows[L])]
               for L in range(NL)]
    gm = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        # the library's handle and workspace are created outside the capture
        torch.matmul(xt_rows[0], wk[0][0].t(), out=ref_out[0][0])
        cap.synchronize()
        gm.capture_begin()
        for L in range(NL):
            torch.matmul(xt_rows[L], wk[L][0].t(), out=ref_out[L][0])
            torch.matmul(xs_rows[L], wk[L][1].t(), out=ref_out[L][1])
        gm.capture_end()
    gm.replay()
    torch.cuda.synchronize()
    ta.record(stream)
    for _ in range(5):
        gm.replay()
    tb.record(stream)
    torch.cuda.synchronize()
    avg_lib_gemm = ta.elapsed_time(tb) / 1e3 / (5 * NL)
    del gp, gm, wk, bk, ref_out, xs_rows, xt_rows

    # ---- roofline of each kernel ----
    pk, pk_kind = peaks()
    t_bytes = (2 * PM + 4 * l) * frame_bytes                       # cache K,V + chunk Q,K,V + O
    s_flops_den = 4 * D * HW * (1 + PS) * HW * l * H * B           # denoising mode (P' prefix frames)
    s_flops_self = 4 * D * HW * HW * l * H * B                     # self-repeat mode (own frame once)
    w_bytes = 2 * NL * (2 * l + 2 * PS) * frame_bytes              # read + write of K,V (temporal, spatial)
    tpe_bytes = 2 * l * frame_bytes + l * H * D * 2                 # chunk read + write, n table rows
    proj_flops = 2 * B * HW * (l + n_sp) * 2 * C * Cin             # temporal + spatial [K | V] = x W^T
    avg_t = statistics.mean(tp_ms) / 1e3
    avg_sd = statistics.mean(sp_den) / 1e3
    avg_ss = statistics.mean(sp_self) / 1e3
    avg_w = statistics.mean(wr_ms) / 1e3
    kernels = {
        "temporal": {"bound": "hbm", "us": avg_t * 1e6, "achieved": t_bytes / avg_t / 1e9,
                     "peak": pk["hbm_gbs"], "unit": "GB/s", "bytes_per_launch": t_bytes},
        "spatial": {"bound": "tensor", "us": avg_sd * 1e6, "achieved": s_flops_den / avg_sd / 1e12,
                    "peak": pk["bf16_tflops_sustained"], "unit": "TFLOP/s", "flops_per_launch": s_flops_den},
        "spatial_self": {"bound": "tensor", "us": avg_ss * 1e6, "achieved": s_flops_self / avg_ss / 1e12,
                         "peak": pk["bf16_tflops_sustained"], "unit": "TFLOP/s", "flops_per_launch": s_flops_self},
        "cache_write": {"bound": "hbm", "us": avg_w * 1e6, "achieved": w_bytes / avg_w / 1e9,
                        "peak": pk["hbm_gbs"], "unit": "GB/s", "bytes_per_launch": w_bytes},
        "tpe_add": {"bound": "hbm", "us": avg_tpe * 1e6, "achieved": tpe_bytes / avg_tpe / 1e9,
                    "peak": pk["hbm_gbs"], "unit": "GB/s", "bytes_per_launch": tpe_bytes,
                    "note": "timed apart from the step: 28 launches in a graph, replayed 5 times"},
        "kv_proj_write": {"bound": "tensor", "us": avg_proj * 1e6, "achieved": proj_flops / avg_proj / 1e12,
                          "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "flops_per_launch": proj_flops,
                          "note": "timed apart from the step (28 launches in a graph, replayed 5 times) "
                                  "against the burst bf16 peak",
                          "library_gemm_same_shapes_us": avg_lib_gemm * 1e6,
                          "library_gemm_note": "torch matmul (cuBLAS) of the same two products per block, no "
                                               "bias and no cache write: context for the shape, not the product"},
    }
    for k in kernels.values():
        k["frac"] = k["achieved"] / k["peak"]
    step_s = ms / 1e3 / args.steps
    share_t = avg_t * (T + 1) * NL / step_s
    share_s = (avg_sd * T + avg_ss) * NL / step_s
    share_w = avg_w / step_s
    dom = "temporal" if share_t >= share_s else "spatial"
    dk = kernels[dom]
    # the committed capture is of one Open-Sora-shaped launch (B = 1, Pmax = 41, all heads):
    # other settings' launches move other byte counts
    captured_shape = args.config == "os_p41" and not sharded
    traffic = committed_traffic("k_temporal.cu" if dom == "temporal" else "k_spatial.cu") if captured_shape else None
    roofline = {"kernel": "k_temporal_causal" if dom == "temporal" else "k_spatial_prefix",
                "bound": dk["bound"], "achieved": dk["achieved"], "peak": dk["peak"], "unit": dk["unit"],
                "frac": dk["frac"], "traffic": traffic, "peak_source": pk_kind}

    # ---- end to end through host buffers ----
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, inp, so, to, step, stream, NL, job_tokens, world, dist, add_set, cur, hv)

    out = {
        "metric": METRIC, "value": value, "unit": "query-tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "strong" if sharded else "weak", "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,0.49) bf16 Q/K/V; no weights needed)",
        "config": {"workload": cfg["name"], "config": args.config, "batch": B, "tokens_per_frame": HW,
                   "heads": H_all, "head_dim": D, "chunk_len": l, "p_max": PM, "p_spatial": PS, "blocks": NL,
                   "denoise_steps": T, "queue_len": PM, "parallelism": parallelism(sharded, world, groups, grank,
                                                                                  h0, H, H_all),
                   "l2": "inputs larger than L2: %d per-block caches and inputs, %.2f GB on the device"
                         % (NL, resident_gb),
                   "tokens_per_step": tokens_per_step},
        "roofline": roofline,
        "kernels": kernels,
        "kernel_time_share": {"temporal": share_t, "spatial": share_s, "cache_write": share_w},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
        "e2e": e2e,
    }
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(budget_s=12.0)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out))


def parallelism(sharded, world, groups, grank, h0, H, H_all):
    if not sharded:
        return "replica per GPU (dp%d)" % world
    if world > 1:
        return "heads split over %d ranks (tp%d; rank 0 runs heads %d..%d of %d)" % (world, world, h0, h0 + H - 1,
                                                                                 H_all)
    return ("one group of a %d-way head split timed alone: heads %d..%d of %d (group %d); value counts its "
            "heads' share of each token" % (groups, h0, h0 + H - 1, H_all, grank))


def run_e2e(args, inp, so, to, step_fn, stream, NL, job_tokens, world, dist, add_set, cur, hv):
    """The same step with its inputs copied from pinned host memory and its outputs read
    back, all inside the timed region.  The copies run on two streams of their own against
    two device sets of inputs and outputs: while step k computes on one set, step k+1's
    inputs are copied into the other, and step k's outputs are read back while step k+1
    computes.  Events order every copy against the steps that use its buffers."""
    import torch
    host_in = [{k: hv(v).contiguous().cpu().pin_memory() for k, v in d.items()} for d in inp]
    host_out = [torch.empty(hv((so if i % 2 == 0 else to)[0]).shape, dtype=torch.bfloat16).pin_memory()
                for i in range(2 * NL)]
    h2d = sum(v.numel() * 2 for d in host_in for v in d.values())
    d2h = sum(t.numel() * 2 for t in host_out)
    inp_b = [{k: torch.empty_like(v) for k, v in d.items()} for d in inp]
    so_b = [torch.empty_like(t) for t in so]
    to_b = [torch.empty_like(t) for t in to]
    bufs = [(0, inp, so, to), (add_set(inp_b, so_b, to_b), inp_b, so_b, to_b)]
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev_h2d, ev_comp, ev_d2h = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

    def upload(k):
        i = k % 2
        din = bufs[i][1]
        with torch.cuda.stream(up):
            if k >= 2:
                up.wait_event(ev_comp[i])          # the step that last read this set is done
            for L in range(NL):
                for key, v in host_in[L].items():
                    hv(din[L][key]).copy_(v, non_blocking=True)
            ev_h2d[i].record(up)

    def compute(k):
        i = k % 2
        stream.wait_event(ev_h2d[i])
        if k >= 2:
            stream.wait_event(ev_d2h[i])           # this set's previous outputs are read back
        cur[0] = bufs[i][0]
        step_fn()
        ev_comp[i].record(stream)

    def download(k):
        i = k % 2
        dso, dto = bufs[i][2], bufs[i][3]
        with torch.cuda.stream(down):
            down.wait_event(ev_comp[i])
            for L in range(NL):
                host_out[2 * L].copy_(hv(dso[L]), non_blocking=True)
                host_out[2 * L + 1].copy_(hv(dto[L]), non_blocking=True)
            ev_d2h[i].record(down)

    def run(n_steps, start=None):
        if start is not None:
            up.wait_event(start)
        upload(0)
        for k in range(n_steps):
            if k + 1 < n_steps:
                upload(k + 1)
            compute(k)
            download(k)
        stream.wait_event(ev_d2h[(n_steps - 1) % 2])

    run(2)
    torch.cuda.synchronize()
    # up to 10 steps: the AR steps of the 80-frame run (the first upload and the last read-back
    # are not overlapped)
    steps = max(1, min(args.steps, 10))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    run(steps, a)
    b.record(stream)
    torch.cuda.synchronize()
    cur[0] = 0
    ms = max_over_ranks(a.elapsed_time(b), dist, world, "cuda")
    return {"value": whole_job_rate(job_tokens, steps, 1, ms), "unit": "query-tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": ms / steps,
            "copies": "host<->device copies on two streams of their own, overlapping the steps "
                      "(two device sets of inputs and outputs)"}


# ------------------------------------------------------------------------------------
def oracle_sample(budget_s: float):
    """Time the fp64 oracle on a bounded sample of one block's pass (all host threads).

    Sample: temporal attention for 64 token positions x 16 heads (8 queries, 41 queued +
    8 chunk keys each) and prefix-spatial attention for 2 frame-heads (256 queries x 1024
    keys), scaled to query tokens of one block pass (all heads)."""
    import numpy as np
    import oracle
    from ca2_synth import Generator, WORKLOADS
    wl = WORKLOADS["os_p41"]
    gen = Generator(wl, 0)
    q, k, v = gen.qkv(wl.chunk_len)
    _, pk, pv = gen.qkv(wl.p_max)
    prefix_k = [pk[:, i] for i in range(wl.p_max)]
    prefix_v = [pv[:, i] for i in range(wl.p_max)]
    sk = prefix_k[-3:]
    sv = prefix_v[-3:]
    H = wl.heads
    t_units = np.arange(64 * H)
    s_units = np.arange(2)
    t_time = s_time = 0.0
    reps = 0
    start = time.perf_counter()
    while True:
        a = time.perf_counter()
        oracle.temporal_attn(q, k, v, prefix_k, prefix_v, units=t_units)
        b = time.perf_counter()
        oracle.spatial_attn(q, k, v, sk, sv, repeat=0, units=s_units)
        c = time.perf_counter()
        t_time += b - a
        s_time += c - b
        reps += 1
        if time.perf_counter() - start > budget_s:
            break
    # seconds per query token (all heads): temporal sample = 64 positions x 8 frames,
    # spatial sample = 2/16 of one frame's 256 query tokens
    t_per_tok = (t_time / reps) / (64 * wl.chunk_len)
    s_per_tok = (s_time / reps) / (256 * len(s_units) / H)
    value = 1.0 / (t_per_tok + s_per_tok)
    sample = ("%d reps of: temporal 64 positions x 16 heads x 8 queries over 49 keys; spatial 2 "
              "frame-heads x 256 queries x 1024 keys (Pmax=41, P'=3 shapes); scaled to query tokens "
              "of one block pass" % reps)
    return value, sample, oracle.num_threads(), time.perf_counter() - start


def cpu_baseline(budget_s: float):
    value, sample, cores, _ = oracle_sample(budget_s)
    return {"value": value, "unit": "query-tokens/s", "cores": cores, "kind": "oracle", "sample": sample}


def run_cpu_baseline(args):
    """The fp64 oracle as a reported CPU baseline (never a target), on the machine's host cores.

    Per call of the Open-Sora-shaped layer (B=1, HW=256, 16 x 72, l=8, P'=3) at every queue
    length of the 80-frame run (P_k = 1, 9, ..., 41): temporal attention (B*HW*H units of 8
    queries) and prefix-spatial attention (B*n*H frame-heads; n_sp = 1 at P_k = 1, else 3),
    each timed on a bounded sample of units with one thread and with all threads and scaled
    to the whole call.  Then one 512x512 (1024 tokens/frame, B = 2) prefix-spatial call on all
    threads, from a sample of frame-heads, extrapolated to an AR step of T = 50 denoising calls
    plus the cache-writing pass: an extrapolation, stated as such."""
    rank, _, _ = dist_env()
    if rank != 0:
        return
    import numpy as np
    import oracle
    from ca2_synth import Generator, WORKLOADS
    oracle.build()
    all_threads = oracle.num_threads()
    wl = WORKLOADS["os_p41"]
    gen = Generator(wl, 0)
    q, k, v = gen.qkv(wl.chunk_len)
    _, pk, pv = gen.qkv(wl.p_max)
    H = wl.heads
    t_units_call = wl.batch * wl.hw * H
    s_units_call = wl.batch * wl.chunk_len * H

    def timed(fn, min_s=0.3):
        reps, t0 = 0, time.perf_counter()
        while True:
            fn()
            reps += 1
            dt = time.perf_counter() - t0
            if dt >= min_s:
                return dt / reps

    rows = []
    for P in (1, 9, 17, 25, 33, 41):
        prefix_k = [pk[:, i] for i in range(P)]
        prefix_v = [pv[:, i] for i in range(P)]
        n_sp = 1 if P == 1 else 3
        sk, sv = prefix_k[-n_sp:], prefix_v[-n_sp:]
        row = {"p_k": P, "n_sp": n_sp}
        for label, threads, tu, su in (("1_thread", 1, 16, 1), ("all_threads", all_threads, 16 * all_threads,
                                                                 max(1, min(s_units_call, all_threads)))):
            oracle.set_num_threads(threads)
            t_u = np.arange(tu)
            s_u = np.arange(su)
            tt = timed(lambda: oracle.temporal_attn(q, k, v, prefix_k, prefix_v, units=t_u))
            ts = timed(lambda: oracle.spatial_attn(q, k, v, sk, sv, repeat=0, units=s_u))
            row[label] = {"temporal_call_s": tt * t_units_call / tu, "spatial_call_s": ts * s_units_call / su,
                          "temporal_sample_units": tu, "spatial_sample_units": su}
        rows.append(row)
    # 512x512: one prefix-spatial call (B=2, 8 frames, 16 heads: 256 frame-heads of 1024 x 4096)
    hw = WORKLOADS["hires"]
    hgen = Generator(hw, 0)
    hq, hk, hv = hgen.qkv(hw.chunk_len)
    _, hck, hcv = hgen.qkv(3)
    oracle.set_num_threads(all_threads)
    hs_units = np.arange(all_threads)
    th = timed(lambda: oracle.spatial_attn(hq, hk, hv, [hck[:, i] for i in range(3)], [hcv[:, i] for i in range(3)],
                                           repeat=0, units=hs_units), min_s=0.0)
    units_call = hw.batch * hw.chunk_len * hw.heads
    hires_call = th * units_call / len(hs_units)
    oracle.set_num_threads(all_threads)
    out = {
        "impl": "oracle-cpu-baseline", "kind": "oracle", "cores": all_threads, "host_cpus": os.cpu_count(),
        "precision": "f64 naive (two-pass softmax), gcc -O2, OpenMP over units",
        "per_call": rows,
        "hires_spatial": {"call_s_all_threads": hires_call, "sample_frame_heads": len(hs_units),
                          "frame_heads_per_call": units_call,
                          "ar_step_s_extrapolated": hires_call * 51,
                          "note": "extrapolation: one call's time from a sample of frame-heads, times the "
                                  "T = 50 denoising calls plus the cache-writing pass of one AR step"},
    }
    print(json.dumps(out))


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    oracle.build()
    for _ in range(args.warmup):
        oracle_sample(budget_s=0.5)
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        v, sample, cores, _ = oracle_sample(budget_s=3.0)
        vals.append(v)
    wall = time.perf_counter() - t0
    value = statistics.mean(vals)
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "query-tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": wall * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD_NAME, "sample": "bounded CPU sample per step"},
        "cpu_baseline": {"value": value, "unit": "query-tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "query-tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(out))


def run_recompute(args):
    """Attention time per denoising step of one block along the 80-frame run: with the shared
    cache (Ca2-VDM: the chunk's 8 frames attend to the queue) against recomputing every frame
    of the window from scratch (OS-Ext style: each prefix frame again goes through spatial
    self-attention and causal temporal attention over the frames before it).  The pages report
    cumulative time linear in the AR step for the cached model and quadratic for recompute until
    Pmax is reached ("Ca2-VDM" papernotes page, 实验结果, 关键发现 1; bohrium page, surprising
    findings).  Attention only: projections and MLPs need the weights.  One JSON line."""
    import torch
    from causal_kv_cache_b200 import ca2
    rank, world, _ = dist_env()
    if rank != 0:
        return
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    B, HW, H, D, l, PM, PS = (WORKLOAD[k] for k in ("batch", "hw", "heads", "head_dim", "chunk_len", "p_max", "p_spatial"))
    T = args.denoise
    g = torch.Generator(device=dev)
    g.manual_seed(77)
    rnd = lambda *shape: (torch.randn(shape, generator=g, device=dev) * 0.7).to(torch.bfloat16)
    steps = list(range(1, 11))                                   # AR steps of the 80-frame run
    prefix = [min(8 * (k - 1) + 1, PM) for k in steps]           # queued frames before each step
    qlens = sorted({0} | {q for P in prefix for q in [P] + list(range(1, P, 8))})
    caches = {}
    for q in qlens:                                              # one cache per queue length
        c = ca2.KVCache(1, B, HW, H, D, l, PM, PS)
        sizes = ([1] if q >= 1 else []) + [8] * ((q - 1) // 8 if q > 1 else 0)
        for n in sizes:
            kt, ks = rnd(B, HW, n, H, D), rnd(B, n, HW, H, D)
            c.evict_for(n)
            c.write([kt], [kt], [ks], [ks], n)
        assert c.state()[1] == q
        caches[q] = c
    tq, tk, tv = (rnd(B, HW, l, H, D) for _ in range(3))
    sq, sk, sv = (rnd(B, l, HW, H, D) for _ in range(3))
    to, so = torch.empty_like(tq), torch.empty_like(sq)
    tq1, tk1, tv1 = (rnd(B, HW, 1, H, D) for _ in range(3))
    sq1, sk1, sv1 = (rnd(B, 1, HW, H, D) for _ in range(3))
    to1, so1 = torch.empty_like(tq1), torch.empty_like(sq1)
    cap = torch.cuda.Stream(device=dev)

    def cached_pass(P, sp):
        c = caches[P]
        c.spatial_attn(0, sq, sk, sv, so, l, 1, sp)               # prefix-enhanced, P' cache frames
        c.temporal(0, tq, tk, tv, to, l, sp)

    def recompute_pass(P, sp):
        # the window: frame 0 (no earlier frame), then groups of 8 with queues 1, 9, ..., then the chunk
        caches[0].spatial_attn(0, sq1, sk1, sv1, so1, 1, 0, sp)
        caches[0].temporal(0, tq1, tk1, tv1, to1, 1, sp)
        for q in list(range(1, P, 8)) + [P]:
            caches[q].spatial_attn(0, sq, sk, sv, so, l, 0, sp)
            caches[q].temporal(0, tq, tk, tv, to, l, sp)

    def time_graph(fn, P, reps=20):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.stream(cap):
            gr.capture_begin()
            fn(P, int(cap.cuda_stream))
            gr.capture_end()
        for _ in range(3):
            gr.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            gr.replay()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) * 1e3 / reps                    # us per pass

    cached_us = [time_graph(cached_pass, P) for P in prefix]
    recompute_us = [time_graph(recompute_pass, P) for P in prefix]
    assert ca2.ca2_device_status() == 0
    NL = WORKLOAD["n_layers"]
    cum_c, cum_r, acc_c, acc_r = [], [], 0.0, 0.0
    for c_us, r_us in zip(cached_us, recompute_us):
        acc_c += c_us * T * NL / 1e3                              # ms of attention over the AR step
        acc_r += r_us * T * NL / 1e3
        cum_c.append(round(acc_c, 2))
        cum_r.append(round(acc_r, 2))
    out = {"mode": "recompute", "metric": "attention us per denoising step of one block",
           "unit": "us", "ar_steps": steps, "prefix_frames": prefix,
           "cached_us": [round(x, 2) for x in cached_us], "recompute_us": [round(x, 2) for x in recompute_us],
           "cumulative_ms": {"cached": cum_c, "recompute": cum_r, "blocks": NL, "denoise_steps": T},
           "ratio_last_step": round(recompute_us[-1] / cached_us[-1], 2),
           "config": {"workload": WORKLOAD_NAME, "batch": B, "tokens_per_frame": HW, "heads": H,
                      "head_dim": D, "chunk_len": l, "p_max": PM, "p_spatial": PS},
           "data": "synthetic (seeded N(0,0.49) bf16); attention only (projections and MLPs need weights)"}
    print(json.dumps(out))


def run_per_timestep(args):
    """One cache shared by all T denoising steps (Ca2-VDM: prefix frames at tEmb(0)) against one
    cache per denoising step (a per-timestep KV cache, as when prefix K/V depend on the noise
    level).  Same kernels.  Shared: each AR step is T passes reading the one cache, the
    cache-writing pass and one write.  Per-timestep: T passes, pass t reading cache t, and T
    writes, since each step's K/V are stored at their own noise level ("Ca2-VDM" papernotes page,
    关键设计 2 and 实验结果, 关键发现 4).  Reports the cache bytes and the AR-step time of both."""
    import torch
    from causal_kv_cache_b200 import ca2
    rank, world, _ = dist_env()
    if rank != 0:
        return
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    B, HW, H, D, l, PM, PS = (WORKLOAD[k] for k in ("batch", "hw", "heads", "head_dim", "chunk_len", "p_max", "p_spatial"))
    NL, T = args.layers, args.denoise
    g = torch.Generator(device=dev)
    g.manual_seed(99)
    rnd = lambda *shape: (torch.randn(shape, generator=g, device=dev) * 0.7).to(torch.bfloat16)

    def filled_cache():
        c = ca2.KVCache(NL, B, HW, H, D, l, PM, PS)
        kt, ks = [rnd(B, HW, 1, H, D)] * NL, [rnd(B, 1, HW, H, D)] * NL
        c.evict_for(1)
        c.write(kt, kt, ks, ks, 1)
        kt8, ks8 = [rnd(B, HW, l, H, D)] * NL, [rnd(B, l, HW, H, D)] * NL
        for _ in range(5):                                      # queue of 41 frames
            c.evict_for(l)
            c.write(kt8, kt8, ks8, ks8, l)
        return c

    shared = filled_cache()
    per_t = [filled_cache() for _ in range(T)]
    tq = [rnd(B, HW, l, H, D) for _ in range(NL)]
    sq = [rnd(B, l, HW, H, D) for _ in range(NL)]
    to, so = [torch.empty_like(x) for x in tq], [torch.empty_like(x) for x in sq]
    kt8, ks8 = [rnd(B, HW, l, H, D) for _ in range(NL)], [rnd(B, l, HW, H, D) for _ in range(NL)]
    cap = torch.cuda.Stream(device=dev)

    def one_pass(c, use_prefix, sp):
        for L in range(NL):
            c.spatial_attn(L, sq[L], sq[L], sq[L], so[L], l, use_prefix, sp)
            c.temporal(L, tq[L], tq[L], tq[L], to[L], l, sp)

    def graph_of(fn):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.stream(cap):
            gr.capture_begin()
            fn(int(cap.cuda_stream))
            gr.capture_end()
        return gr

    g_shared = graph_of(lambda sp: one_pass(shared, 1, sp))
    g_shared_self = graph_of(lambda sp: one_pass(shared, 0, sp))
    g_per = [graph_of(lambda sp, c=c: one_pass(c, 1, sp)) for c in per_t]
    stream = torch.cuda.current_stream()
    sp = int(stream.cuda_stream)

    def step_shared():
        for _ in range(T):
            g_shared.replay()
        g_shared_self.replay()
        shared.evict_for(l)                                     # the queue stays full: evict 8, write 8
        shared.write(kt8, kt8, ks8, ks8, l, sp)

    def step_per():
        for t in range(T):
            g_per[t].replay()
        for c in per_t:                                         # each step's K/V into its own cache
            c.evict_for(l)
            c.write(kt8, kt8, ks8, ks8, l, sp)

    def timed(fn, reps=3):
        fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    ms_shared = timed(step_shared)
    ms_per = timed(step_per)
    assert ca2.ca2_device_status() == 0
    assert shared.state()[1] == PM and all(c.state()[1] == PM for c in per_t)
    tb, sbb = ca2.ca2_cache_bytes(shared.cfg)
    bytes_one = tb + sbb
    out = {"mode": "per-timestep", "metric": "AR-step time (ms) and cache bytes", "unit": "ms",
           "shared": {"ms_per_ar_step": round(ms_shared, 3), "cache_bytes": bytes_one, "caches": 1},
           "per_timestep": {"ms_per_ar_step": round(ms_per, 3), "cache_bytes": bytes_one * T, "caches": T},
           "time_ratio": round(ms_per / ms_shared, 3), "memory_ratio": T,
           "config": {"workload": WORKLOAD_NAME, "blocks": NL, "denoise_steps": T, "batch": B,
                      "tokens_per_frame": HW, "heads": H, "head_dim": D, "chunk_len": l, "p_max": PM,
                      "p_spatial": PS},
           "data": "synthetic (seeded N(0,0.49) bf16)"}
    print(json.dumps(out))


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.mode == "recompute":
        run_recompute(args)
    elif args.mode == "per-timestep":
        run_per_timestep(args)
    elif args.mode == "cpu-baseline":
        run_cpu_baseline(args)
    else:
        run_ca2(args)


if __name__ == "__main__":
    main()
