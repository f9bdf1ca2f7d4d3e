"""CUDA path (through the C ABI) against the fp64 oracle on the same seeded bf16 inputs.

Tolerance for attention outputs: max-abs 2e-2 and relative L2 5e-3 (tests/gpu_util.py);
ring contents, eviction order, queue state and TPE indices must match bit for bit.
"""
import dataclasses

import numpy as np
import pytest

import oracle
from ca2_synth import WORKLOADS, Generator, bf16_bits, bf16_to_f32

pytestmark = pytest.mark.gpu


def _wl(base, **kw):
    return dataclasses.replace(WORKLOADS[base], **kw)


def test_tiny_generation_loop_every_call():
    """The tiny workload end to end: first frame, 3 AR steps x (2 denoising passes + the
    cache-writing pass), every attention output, every cache write, TPE indices."""
    from tests.gpu_util import Loop
    wl = WORKLOADS["tiny"]
    lp = Loop(wl, seed=0, tpe_offset=0)
    lp.first_frame()
    for _ in range(wl.ar_steps):
        lp.ar_step(wl.chunk_len, wl.denoise_steps)
    assert lp.rings[0].evicted == [0, 1, 2, 3]         # the last write evicted the oldest 4
    assert len(lp.stats) == 2 * (1 + 3 * 3)


def test_tiny_peaky_values():
    from tests.gpu_util import Loop
    wl = _wl("tiny", recipe="peaky", name="tiny_peaky")
    lp = Loop(wl, seed=5)
    lp.first_frame()
    for _ in range(3):
        lp.ar_step(wl.chunk_len, 1)


def test_tiny_eight_times_scale():
    """The tiny workload with inputs at 8 times its N(0, 1/16) scale (N(0, 4)): scores of
    several units, near one-hot softmax rows, running maxima that jump between blocks."""
    from tests.gpu_util import Loop
    wl = _wl("tiny", scale=2.0, name="tiny_x8")
    lp = Loop(wl, seed=9)
    lp.first_frame()
    for _ in range(wl.ar_steps):
        lp.ar_step(wl.chunk_len, wl.denoise_steps)
    assert len(lp.stats) == 2 * (1 + 3 * 3)


def test_first_frame_temporal_returns_v_exactly():
    """Single visible key: with an empty queue and one frame the softmax weight is exactly
    1, so the output is V: bit for bit wherever fp16 (the operand type of the P V product)
    represents the bf16 value, i.e. |v| >= 2^-14 or v = 0; smaller values come back as their
    fp16 subnormal, within 2^-25 of v."""
    import torch
    from causal_kv_cache_b200.ca2 import KVCache
    from tests.gpu_util import to_bits, to_dev, token_major
    for name in ("tiny", "os_p41"):
        wl = WORKLOADS[name]
        g = Generator(wl, 3)
        q, k, v = g.qkv(1)
        c = KVCache(1, wl.batch, wl.hw, wl.heads, wl.head_dim, wl.chunk_len, wl.p_max, wl.p_spatial)
        tq, tk, tv = token_major(q), token_major(k), token_major(v)
        out = torch.empty(tq.shape, dtype=torch.bfloat16, device="cuda")
        c.temporal(0, to_dev(tq), to_dev(tk), to_dev(tv), out, 1)
        got = to_bits(out)
        v32 = bf16_to_f32(tv)
        exact = (np.abs(v32) >= 2.0 ** -14) | (v32 == 0)
        assert exact.mean() > 0.99
        assert np.array_equal(got[exact], tv[exact])
        assert np.array_equal(got, bf16_bits(v32.astype(np.float16).astype(np.float32)))
        assert np.abs(bf16_to_f32(got).astype(np.float64) - v32).max() <= 2.0 ** -25


def test_poisoned_buffers_never_reach_outputs():
    """A freshly allocated cache buffer holds anything.  With every element of both cache
    buffers set to a NaN bit pattern before the first write, ring slots that hold no queued
    frame, rows past Pmax of the last 16-slot group (Pmax = 41), and spatial-cache frames
    not yet written must never reach an output: every output is finite and matches the
    oracle while the queue fills."""
    import torch
    from tests.gpu_util import Loop
    wl = _wl("os_p41", n_layers=1)
    lp = Loop(wl, seed=21)
    lp.cache.tbuf.view(torch.int16).fill_(0x7FC0)     # bf16 quiet NaN
    lp.cache.sbuf.view(torch.int16).fill_(0x7FC0)
    lp.first_frame()
    for _ in range(3):
        lp.ar_step(wl.chunk_len, 1)


def test_os_p41_eighty_frames():
    """Open-Sora-shaped layer, Pmax = 41: first frame + 10 chunks of 8 (eviction from the
    7th write on) with a random cyclic TPE offset.  Temporal outputs in full at every call;
    spatial on 16 sampled frame-heads per call (the full spatial map is checked below)."""
    from tests.gpu_util import Loop
    wl = WORKLOADS["os_p41"]
    off = Generator(wl).tpe_offset(seed=1)
    lp = Loop(wl, seed=0, tpe_offset=off)
    rng = np.random.default_rng(7)
    lp.first_frame()
    counts = []
    for _ in range(wl.ar_steps):
        counts.append(lp.rings[0].count)
        s_units = rng.choice(wl.batch * wl.chunk_len * wl.heads, size=16, replace=False)
        lp.ar_step(wl.chunk_len, 1, s_units=s_units)
    assert counts == [1, 9, 17, 25, 33, 41, 41, 41, 41, 41]
    assert lp.rings[0].evicted == list(range(8 * 5))
    assert lp.rings[0].frames_written == 81


def test_os_p41_full_spatial_maps():
    """Full spatial outputs (all 8 frames x 16 heads x 256 tokens) with 3 prefix frames,
    and in self-repeat mode."""
    from tests.gpu_util import Loop
    wl = WORKLOADS["os_p41"]
    lp = Loop(wl, seed=1)
    lp.first_frame()
    lp.ar_step(wl.chunk_len, 0, s_units=np.arange(4))
    assert len(lp.rings[0].spatial_ids) == 3
    q, k, v = lp.gen.qkv(wl.chunk_len)
    lp.spatial(0, q, k, v, use_prefix=1)
    lp.spatial(0, q, k, v, use_prefix=0)


def test_os_p25_queue_fills():
    from tests.gpu_util import Loop
    wl = WORKLOADS["os_p25"]
    lp = Loop(wl, seed=2)
    lp.first_frame()
    for _ in range(wl.ar_steps + 1):
        lp.ar_step(wl.chunk_len, 1, s_units=np.arange(0, 128, 17))
    assert lp.rings[0].count == 25


def test_cache_shared_across_denoising_steps_bit_identical():
    """Cache sharing: T reads of one cache give bit-identical outputs, the cache bytes do
    not change, and a cache rebuilt before each step gives the same bits again."""
    import torch
    from tests.gpu_util import Loop, to_bits, to_dev, token_major
    wl = _wl("os_p41")
    lp = Loop(wl, seed=4)
    lp.first_frame()
    lp.ar_step(wl.chunk_len, 0, s_units=np.arange(2))
    lp.ar_step(wl.chunk_len, 0, s_units=np.arange(2))
    ring_before = lp.cache.tbuf.clone()
    sp_before = lp.cache.sbuf.clone()
    tq, tk, tv = (to_dev(token_major(x)) for x in lp.gen.qkv(wl.chunk_len))
    sq, sk, sv = (to_dev(x) for x in lp.gen.qkv(wl.chunk_len))
    to = torch.empty_like(tq)
    so = torch.empty_like(sq)
    first_t = first_s = None
    for t in range(8):
        lp.cache.spatial_attn(0, sq, sk, sv, so, wl.chunk_len, 1)
        lp.cache.temporal(0, tq, tk, tv, to, wl.chunk_len)
        if first_t is None:
            first_t, first_s = to.clone(), so.clone()
        else:
            assert torch.equal(to.view(torch.int16), first_t.view(torch.int16))
            assert torch.equal(so.view(torch.int16), first_s.view(torch.int16))
    torch.cuda.synchronize()
    assert torch.equal(lp.cache.tbuf.view(torch.int16), ring_before.view(torch.int16))
    assert torch.equal(lp.cache.sbuf.view(torch.int16), sp_before.view(torch.int16))
    # rebuild: a second cache fed the same frames in the same order
    from causal_kv_cache_b200.ca2 import KVCache
    c2 = KVCache(1, wl.batch, wl.hw, wl.heads, wl.head_dim, wl.chunk_len, wl.p_max, wl.p_spatial)
    ring = lp.rings[0]
    frames = sorted(ring.queue)
    # queue frames were written as: [0], [1..8], [9..16]
    for lo, hi in ((0, 1), (1, 9), (9, 17)):
        kt = np.stack([ring.k[g] for g in range(lo, hi)], axis=1)
        vt = np.stack([ring.v[g] for g in range(lo, hi)], axis=1)
        if hi == 17:
            ks = np.zeros_like(kt)
            vs = np.zeros_like(vt)
            for j, g in enumerate(ring.spatial_ids):
                ks[:, hi - lo - len(ring.spatial_ids) + j] = ring.sk[g]
                vs[:, hi - lo - len(ring.spatial_ids) + j] = ring.sv[g]
        else:
            ks, vs = kt, vt
        c2.write([to_dev(token_major(kt))], [to_dev(token_major(vt))], [to_dev(ks)], [to_dev(vs)], hi - lo)
    assert frames == list(range(17))
    to2 = torch.empty_like(tq)
    so2 = torch.empty_like(sq)
    c2.spatial_attn(0, sq, sk, sv, so2, wl.chunk_len, 1)
    c2.temporal(0, tq, tk, tv, to2, wl.chunk_len)
    assert torch.equal(to2.view(torch.int16), first_t.view(torch.int16))
    assert torch.equal(so2.view(torch.int16), first_s.view(torch.int16))


@pytest.mark.parametrize("shape", [
    dict(hw=200, heads=3, head_dim=16, batch=2, chunk_len=5, p_max=13, p_spatial=2),
    dict(hw=130, heads=2, head_dim=24, batch=1, chunk_len=8, p_max=8, p_spatial=1),
    dict(hw=64, heads=4, head_dim=128, batch=1, chunk_len=3, p_max=30, p_spatial=3),
    dict(hw=257, heads=6, head_dim=72, batch=1, chunk_len=4, p_max=9, p_spatial=0),
    dict(hw=40, heads=16, head_dim=64, batch=3, chunk_len=2, p_max=3, p_spatial=2),
])
def test_ragged_shapes(shape):
    """Ragged query/key tiles (HW not a multiple of 128), odd head counts, head dims 16-128,
    short chunks, Pmax = l, P' = 0; several AR steps with eviction."""
    from tests.gpu_util import Loop
    wl = _wl("tiny", recipe="normal", scale=0.5, n_layers=1, name="ragged", **shape)
    lp = Loop(wl, seed=9)
    lp.first_frame()
    for _ in range(4):
        lp.ar_step(wl.chunk_len, 1)
    # a short chunk (fewer frames than l)
    if wl.chunk_len > 1:
        lp.ar_step(wl.chunk_len - 1, 1)


@pytest.mark.parametrize("head_dim", [72, 64, 128])
def test_spatial_max_grows_in_late_blocks(head_dim):
    """Spatial-cache keys scaled up (more for later cache frames and for the second key
    block of each frame), so the running row max jumps well past the lazy-rescale
    threshold after the first blocks and O is rescaled between P V products."""
    from ca2_synth import bf16_bits, bf16_to_f32
    from tests.gpu_util import Loop
    wl = _wl("tiny", recipe="normal", scale=0.5, n_layers=1, hw=256, heads=2, head_dim=head_dim,
             batch=1, chunk_len=3, p_max=6, p_spatial=3, name="lazy_rescale")
    lp = Loop(wl, seed=21)
    kt, vt = lp.gen.frames(3), lp.gen.frames(3)
    ks = bf16_to_f32(lp.gen.frames(3)).copy()
    for i in range(3):
        ks[:, i] *= 3.0 * (i + 1)
    ks[:, :, 128:] *= 2.0
    vs = lp.gen.frames(3)
    lp.write([kt], [vt], [bf16_bits(ks)], [vs])
    q, k, v = lp.gen.qkv(3)
    lp.spatial(0, q, k, v, use_prefix=1)


@pytest.mark.parametrize("name,offset,g0", [("tiny", 0, 0), ("tiny", 3, 7), ("os_p41", 0, 41), ("os_p41", 17, 45)])
def test_tpe_add_bit_exact(name, offset, g0):
    """Chunk + cyclic TPE rows, out of place and in place, bit for bit against the oracle
    (indices wrap past N_tpe for the larger first frames)."""
    import torch
    from causal_kv_cache_b200.ca2 import KVCache
    from tests.gpu_util import to_bits, to_dev, token_major
    wl = WORKLOADS[name]
    g = Generator(wl, 11)
    c = KVCache(1, wl.batch, wl.hw, wl.heads, wl.head_dim, wl.chunk_len, wl.p_max, wl.p_spatial)
    C = wl.heads * wl.head_dim
    table = g.frames(c.tpe_len)[0, :, 0].reshape(c.tpe_len, wl.heads, wl.head_dim)   # [N_tpe][H][D]
    for n in (wl.chunk_len, 1):
        x = token_major(g.frames(n))                                                  # [B][HW][n][H][D]
        ref = oracle.tpe_add(x.reshape(wl.batch, wl.hw, n, C), table.reshape(-1, C), g0, offset)
        xd, td = to_dev(x), to_dev(table)
        out = torch.empty_like(xd)
        c.tpe_add(g0, offset, td, xd, out, n)
        assert np.array_equal(to_bits(out).reshape(ref.shape), ref)
        c.tpe_add(g0, offset, td, xd, xd, n)                                          # in place
        assert np.array_equal(to_bits(xd).reshape(ref.shape), ref)


def test_long_queue_pmax81():
    """A queue of up to 81 frames (six 16-slot ring groups): first frame + 11 AR steps of 8,
    filling the ring and then evicting; every attention output and cache write checked."""
    from tests.gpu_util import Loop
    wl = _wl("tiny", recipe="normal", scale=0.5, n_layers=1, hw=64, heads=2, head_dim=72, batch=1,
             chunk_len=8, p_max=81, p_spatial=3, name="pmax81")
    lp = Loop(wl, seed=31)
    lp.first_frame()
    for _ in range(11):
        lp.ar_step(wl.chunk_len, 1)
    assert lp.rings[0].count == 81


def test_multi_layer_write_bit_exact():
    """One cache-write launch for many layers (more than one launch's layer table)."""
    from tests.gpu_util import Loop
    wl = _wl("tiny", n_layers=70, batch=2, hw=16, heads=2, head_dim=16)
    lp = Loop(wl, seed=12)
    for n in (1, 4, 4, 4, 4):
        kts = [lp.gen.frames(n) for _ in range(wl.n_layers)]
        vts = [lp.gen.frames(n) for _ in range(wl.n_layers)]
        kss = [lp.gen.frames(n) for _ in range(wl.n_layers)]
        vss = [lp.gen.frames(n) for _ in range(wl.n_layers)]
        lp.write(kts, vts, kss, vss)
    assert lp.rings[0].count == 9


def test_hires_sampled():
    """512x512 shape (HW = 1024, B = 2): queue filled to 41, spatial map 1024 x 4096.
    Sampled: 512 temporal (b, s, h) units, 2 full spatial frame-heads per call."""
    from tests.gpu_util import Loop
    wl = WORKLOADS["hires"]
    lp = Loop(wl, seed=0)
    rng = np.random.default_rng(3)
    # pre-fill: first frame then 5 clean chunks (cache writes only)
    for n in (1, 8, 8, 8, 8, 8):
        k, v = lp.gen.frames(n), lp.gen.frames(n)
        lp.write([k], [v], [k], [v])
    assert lp.rings[0].count == 41
    for _ in range(2):
        t_units = rng.choice(wl.batch * wl.hw * wl.heads, size=512, replace=False)
        s_units = rng.choice(wl.batch * wl.chunk_len * wl.heads, size=2, replace=False)
        lp.ar_step(wl.chunk_len, 1, t_units=t_units, s_units=s_units)


def test_bounded_wait_reports_timeout_and_context_survives():
    """A kernel waiting on a barrier nothing completes gives up after ~1 ms, the host reads
    CA2_ERR_TIMEOUT, and the next calls run normally."""
    import torch
    from causal_kv_cache_b200 import ca2
    assert ca2.ca2_device_status() == 0
    ca2.ca2_selftest_timeout(1000)
    assert ca2.ca2_device_status() == -6
    assert ca2.ca2_device_status() == 0
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0


def _bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (8 significant bits), for normal x."""
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return np.exp2(e - 7)


def _check_projection(got_bits, exact, bound, C, what, fp16=False):
    """|got - exact| <= half a bf16 ulp (the one rounding) + the fp32 accumulation bound
    C * 2^-23 * sum|x w| (twice the textbook gamma_C of recursive summation).  fp16: the
    stored values are fp16 bit patterns (the spatial cache's V), the same bf16 values."""
    if fp16:
        got = got_bits.view(np.float16).astype(np.float64)
    else:
        got = (got_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.isfinite(got).all(), "%s: non-finite value" % what
    tol = 0.5 * _bf16_ulp(np.maximum(np.abs(exact), np.abs(got))) + C * 2.0 ** -23 * bound
    err = np.abs(got - exact)
    assert (err <= tol).all(), "%s: max excess %g" % (what, float((err - tol).max()))


@pytest.mark.parametrize("shape,bias", [
    (dict(n_layers=2, batch=1, hw=256, heads=16, head_dim=72, chunk_len=8, p_max=41, p_spatial=3), True),
    (dict(n_layers=2, batch=2, hw=200, heads=3, head_dim=16, chunk_len=5, p_max=13, p_spatial=2), False),
    (dict(n_layers=2, batch=1, hw=130, heads=4, head_dim=128, chunk_len=3, p_max=7, p_spatial=3, n=2), True),
])
def test_kv_proj_write_matches_oracle(shape, bias):
    """The cache-writing stage's K/V projection stored straight into the caches: every
    written element against the exact projection, every other ring slot, spatial frame and
    layer untouched (still the poison), with the write wrapping past the ring's end."""
    import torch
    from causal_kv_cache_b200.ca2 import KVCache
    s = dict(shape)
    NL, B, HW, H, D, l, PM, PS = (s[k] for k in ("n_layers", "batch", "hw", "heads", "head_dim", "chunk_len",
                                                "p_max", "p_spatial"))
    n = s.get("n", l)                       # a short chunk: fewer frames than P' reach the spatial cache
    C = H * D
    rng = np.random.default_rng(31)
    bits = lambda a: (np.asarray(a, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)
    n_sp = min(PS, n)
    x_t = bits(rng.standard_normal((B, HW, n, C)))
    x_s = bits(rng.standard_normal((B, n, HW, C)))
    w_t = bits(rng.standard_normal((2 * C, C)) / np.sqrt(C))
    w_s = bits(rng.standard_normal((2 * C, C)) / np.sqrt(C))
    b_t = bits(rng.standard_normal(2 * C)) if bias else None
    b_s = bits(rng.standard_normal(2 * C)) if bias else None
    dev = lambda a: None if a is None else torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    cache = KVCache(NL, B, HW, H, D, l, PM, PS)
    cache.tbuf.view(torch.int16).fill_(0x7FC0)
    cache.sbuf.view(torch.int16).fill_(0x7FC0)
    # move the ring head so that the chunk's slots wrap past the end of the ring
    def advance(k):
        while k > 0:
            cache.commit(min(l, k))
            k -= min(l, k)
    advance(n)
    cache.evict(n)
    advance(max(1, PM - n - 1))
    head, count = cache.state()[0], cache.state()[1]
    if count + n > PM:
        cache.evict(count + n - PM)
    head, count = cache.state()[0], cache.state()[1]
    slot0 = (head + count) % PM
    cache.kv_proj_write(1, dev(x_t), dev(w_t), dev(b_t), dev(x_s), dev(w_s), dev(b_s), n)
    torch.cuda.synchronize()
    from causal_kv_cache_b200 import ca2
    assert ca2.ca2_device_status() == 0
    ring = [cache.ring(1, kv).view(torch.int16).cpu().numpy().view(np.uint16) for kv in (0, 1)]
    spat = [cache.spatial(1, kv).view(torch.int16).cpu().numpy().view(np.uint16) for kv in (0, 1)]
    # temporal: rows (b, s, f)
    k, v = oracle.kv_projection(x_t.reshape(-1, C), w_t, b_t)
    bound = oracle.kv_projection_bound(x_t.reshape(-1, C), w_t, b_t)
    slots = [(slot0 + f) % PM for f in range(n)]
    for kv, exact, bnd in ((0, k, bound[:, :C]), (1, v, bound[:, C:])):
        got = ring[kv][:, :, :, slots, :]                       # [B][HW][H][n][D]
        got = got.transpose(0, 1, 3, 2, 4).reshape(-1, C)       # rows (b, s, f), channels (h, d)
        _check_projection(got, exact, bnd, C, "temporal %s" % "KV"[kv], fp16=kv == 1)
        rest = np.delete(ring[kv], slots, axis=3)
        assert (rest == 0x7FC0).all(), "temporal: a slot outside the chunk's was written"
    # spatial: the chunk's last n_sp frames, rows (b, s) per frame
    xs_last = x_s[:, n - n_sp:]                                 # [B][n_sp][HW][C]
    k, v = oracle.kv_projection(xs_last.reshape(-1, C), w_s, b_s)
    bound = oracle.kv_projection_bound(xs_last.reshape(-1, C), w_s, b_s)
    for kv, exact, bnd in ((0, k, bound[:, :C]), (1, v, bound[:, C:])):
        got = spat[kv][:n_sp].transpose(1, 0, 2, 3, 4).reshape(-1, C)   # [B][n_sp][HW] rows
        _check_projection(got, exact, bnd, C, "spatial %s" % "KV"[kv], fp16=kv == 1)
        if kv == 1:   # exactly the fp16 form of a bf16 value
            g32 = got.view(np.float16).astype(np.float32)
            assert np.array_equal(g32, bf16_to_f32(bf16_bits(g32))), "spatial V is not a bf16 value"
    for got in (ring[1][:, :, :, slots, :],):                  # the ring's V as well
        g32 = np.ascontiguousarray(got).view(np.float16).astype(np.float32)
        assert np.array_equal(g32, bf16_to_f32(bf16_bits(g32))), "ring V is not a bf16 value"
        assert (spat[kv][n_sp:] == 0x7FC0).all(), "spatial: a frame past n_sp was written"
    # layer 0 untouched
    for kv in (0, 1):
        assert (cache.ring(0, kv).view(torch.int16) == 0x7FC0).all().item()
        assert (cache.spatial(0, kv).view(torch.int16) == 0x7FC0).all().item()
    cache.commit(n)
    assert cache.state()[1] == count + n and cache.state()[2] == n_sp


def test_out_of_range_v_is_reported():
    """The attention's P V products run in fp16, so V must lie within the fp16 range: a larger
    V value written to the caches, in the frame's own V of a spatial call or in the chunk's V
    of a temporal call is reported as CA2_ERR_RANGE by ca2_device_status, which then clears;
    in-range calls report nothing."""
    import torch
    from causal_kv_cache_b200 import ca2
    from causal_kv_cache_b200.ca2 import KVCache
    from tests.gpu_util import to_dev, token_major
    wl = WORKLOADS["tiny"]
    g = Generator(wl, 17)
    c = KVCache(1, wl.batch, wl.hw, wl.heads, wl.head_dim, wl.chunk_len, wl.p_max, wl.p_spatial)
    assert ca2.ca2_device_status() == 0
    k, v = g.frames(1), g.frames(1)
    c.write([to_dev(token_major(k))], [to_dev(token_major(v))], [to_dev(k)], [to_dev(v)], 1)
    assert ca2.ca2_device_status() == 0
    big = v.copy()
    big[0, 0, 3, 1, 5] = bf16_bits(np.array([70000.0], dtype=np.float32))[0]
    c.evict_for(1)
    c.write([to_dev(token_major(k))], [to_dev(token_major(big))], [to_dev(k)], [to_dev(big)], 1)
    assert ca2.ca2_device_status() == -7
    assert ca2.ca2_device_status() == 0
    q, kk, vv = g.qkv(wl.chunk_len)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    vv[0, 1, 2, 0, 3] = bf16_bits(np.array([-1e6], dtype=np.float32))[0]
    c.spatial_attn(0, to_dev(q), to_dev(kk), to_dev(vv), out, wl.chunk_len, 0)
    assert ca2.ca2_device_status() == -7
    assert ca2.ca2_device_status() == 0
    tq, tk, tv = (token_major(x) for x in g.qkv(wl.chunk_len))
    tout = torch.empty(tq.shape, dtype=torch.bfloat16, device="cuda")
    c.temporal(0, to_dev(tq), to_dev(tk), to_dev(tv), tout, wl.chunk_len)
    assert ca2.ca2_device_status() == 0
    tv[0, 5, 2, 1, 7] = bf16_bits(np.array([-3e5], dtype=np.float32))[0]
    c.temporal(0, to_dev(tq), to_dev(tk), to_dev(tv), tout, wl.chunk_len)
    assert ca2.ca2_device_status() == -7
    assert ca2.ca2_device_status() == 0
