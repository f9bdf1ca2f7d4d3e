"""The multi-rank path of bench.py on CPU (gloo, world size 2): independent replicas, no
data-path collective; the timing is the maximum over ranks and the rate counts every rank's
tokens.  The reference arm runs on rank 0 only."""
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, ms_by_rank, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(ms_by_rank[rank], dist, world, "cpu")
        rate = bench.whole_job_rate(2048, 10, world, ms)
        out.put((rank, ms, rate))
    finally:
        dist.destroy_process_group()


def _free_port():
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_two_ranks_take_the_slowest_time_and_count_all_tokens():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ms_by_rank = [12.5, 31.25]
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, ms_by_rank, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, rate in res:
        assert ms == 31.25                                  # every rank sees the slowest rank's time
        assert rate == pytest.approx(2048 * 10 * 2 / 31.25e-3)   # all ranks' tokens / that time


def test_single_rank_is_unchanged():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.0, None, 1, "cpu") == 7.0
    assert bench.whole_job_rate(100, 3, 1, 1000.0) == pytest.approx(300.0)


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


# ---- head sharding over ranks (tensor-parallel heads; no collective on the data path) -----

def _head_shard_worker(rank, world, port, out):
    import dataclasses
    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from ca2_synth import WORKLOADS, Generator
    from causal_kv_cache_b200 import ca2
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = dataclasses.replace(WORKLOADS["tiny"], heads=5)
        H = wl.heads
        h0, hc = ca2.ca2_head_shard(H, world, rank)
        parts = [None] * world
        dist.all_gather_object(parts, (h0, hc))
        # every rank draws the same full-width inputs; each attends over its own heads only
        g = Generator(wl, 3)
        pre = [g.frames(1) for _ in range(2 * 3)]                  # 3 queued K/V frames
        sc = [g.frames(1) for _ in range(2)]                       # one spatial-cache frame
        q, k, v = g.qkv(wl.chunk_len)
        mine = lambda a: np.ascontiguousarray(a[..., h0:h0 + hc, :])
        pk = [mine(pre[2 * i][:, 0]) for i in range(3)]
        pv = [mine(pre[2 * i + 1][:, 0]) for i in range(3)]
        t = oracle.temporal_attn(mine(q), mine(k), mine(v), pk, pv)
        s = oracle.spatial_attn(mine(q), mine(k), mine(v), [mine(sc[0][:, 0])], [mine(sc[1][:, 0])], repeat=0)
        outs = [None] * world
        dist.all_gather_object(outs, (t, s))
        # the host ring state of each rank's cache (fake device pointers: host calls only)
        c = dict(n_layers=2, batch=wl.batch, hw=wl.hw, heads=hc, head_dim=wl.head_dim, chunk_len=wl.chunk_len,
                 p_max=wl.p_max, p_spatial=wl.p_spatial, tpe_len=0, row_pitch=H * wl.head_dim)
        tb, sb = ca2.ca2_cache_bytes(c)
        hdl = ca2.ca2_cache_init(c, 0x7F0000000000, tb, 0x7F1000000000, sb)
        trace = []
        for n in (1, 4, 4, 4, 3, 4):
            trace.append(ca2.ca2_cache_evict_for(hdl, n))
            ca2.ca2_cache_commit(hdl, n)
            trace.append(ca2.ca2_cache_state(hdl))
        ca2.ca2_cache_destroy(hdl)
        states = [None] * world
        dist.all_gather_object(states, (trace, tb, sb))
        if rank == 0:
            full_t = oracle.temporal_attn(q, k, v, [f[:, 0] for f in pre[0::2]], [f[:, 0] for f in pre[1::2]])
            full_s = oracle.spatial_attn(q, k, v, [sc[0][:, 0]], [sc[1][:, 0]], repeat=0)
            full_c = dict(c, heads=H, row_pitch=0)
            out.put((parts, [np.concatenate([o[i] for o in outs], axis=3) for i in (0, 1)], (full_t, full_s),
                     states, ca2.ca2_cache_bytes(full_c)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_split_heads_and_assemble_the_full_result():
    """World size 2 over gloo: ca2_head_shard gives rank 0 heads 0..2 and rank 1 heads 3..4 of
    5; the oracle run on each rank's heads and gathered along the head axis equals the oracle
    run on all heads exactly (attention never mixes heads); both ranks' host ring states move
    in step; the per-rank caches add up to the whole cache."""
    import numpy as np
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_head_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    parts, got, ref, states, full_bytes = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert parts == [(0, 3), (3, 2)]
    for g, r in zip(got, ref):
        assert g.shape == r.shape and np.array_equal(g, r)
    assert states[0][0] == states[1][0]                          # same evictions and queue states
    import oracle
    ring = oracle.RingModel(9, 1)                                # tiny: Pmax = 9, P' = 1
    expect = []
    for n in (1, 4, 4, 4, 3, 4):
        z = np.zeros((1, n, 1, 1, 1), dtype=np.uint16)
        expect.append(len(ring.write(z, z, z, z)))
        expect.append((ring.head, ring.count, len(ring.spatial_ids), ring.frames_written))
    assert states[0][0] == expect
    assert sum(s[1] for s in states) == full_bytes[0] and sum(s[2] for s in states) == full_bytes[1]


def test_job_tokens_by_parallelism():
    """Replicas count every rank's tokens; a head split over N ranks counts each token once; one
    group of a split timed alone counts its heads' share (the groups of a split add up to one)."""
    sys.path.insert(0, ROOT)
    import bench
    from causal_kv_cache_b200 import ca2
    assert bench.job_tokens_per_step(2048, False, 1, 16, 16) == 2048
    assert bench.job_tokens_per_step(2048, False, 4, 16, 16) == 4 * 2048
    assert bench.job_tokens_per_step(2048, True, 4, 4, 16) == 2048
    shares = [bench.job_tokens_per_step(2048, True, 1, ca2.ca2_head_shard(16, 3, r)[1], 16) for r in range(3)]
    assert sum(shares) == pytest.approx(2048)


def test_reference_arm_line_has_the_contract_keys():
    """Rank 0 of the reference arm (the oracle on the host cores) prints one JSON line with the
    keys the bench contract names, its cpu_baseline and e2e describing the same run."""
    import json
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 1 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
