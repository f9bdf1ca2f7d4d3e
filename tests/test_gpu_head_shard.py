"""Head sharding on one GPU.  The heads of every layer are split into G contiguous groups by
ca2_head_shard and each group runs through a cache handle of its own, on the full-width
activations: row pitch H*D, every pointer offset to element h0*D of the first row.  Every
(token, head) history and every (frame, head) map is independent of the other heads, so each
group's attention outputs, cache contents, TPE sums and projected K/V must equal the
unsharded run's bit for bit; the unsharded run itself is checked against the oracle.

Shape: 6 heads of 72 (G = 4 gives the uneven groups 2, 2, 1, 1), B = 2, 40 tokens per frame
(a ragged tile), l = 8, Pmax = 17 (the last AR step reads a queue that has evicted), P' = 3,
2 layers, lnhead values.
"""
import dataclasses

import numpy as np
import pytest

import oracle
from ca2_synth import WORKLOADS, Generator

pytestmark = pytest.mark.gpu

SHARD = dataclasses.replace(WORKLOADS["os_p25"], name="shard6", batch=2, heads=6, hw=40, p_max=17,
                            n_layers=2, ar_steps=4, denoise_steps=1)


def test_head_shards_equal_the_unsharded_run():
    import torch
    from causal_kv_cache_b200.ca2 import KVCache, ca2_head_shard
    from tests.gpu_util import check_close, f16_bits_of_bf16, to_bits, to_dev, token_major
    wl = SHARD
    NL, B, HW, H, D, l, PM, PS = (wl.n_layers, wl.batch, wl.hw, wl.heads, wl.head_dim, wl.chunk_len, wl.p_max,
                                  wl.p_spatial)
    C = H * D
    gen = Generator(wl, 7)
    full = KVCache(NL, B, HW, H, D, l, PM, PS)
    groups = {}
    for G in (2, 4):
        parts = [ca2_head_shard(H, G, r) for r in range(G)]
        groups[G] = [(h0, hc, KVCache(NL, B, HW, hc, D, l, PM, PS, row_pitch=C)) for h0, hc in parts]
    assert [(h0, hc) for h0, hc, _ in groups[4]] == [(0, 2), (2, 2), (4, 1), (5, 1)]
    assert [(h0, hc) for h0, hc, _ in groups[2]] == [(0, 3), (3, 3)]
    rings = [oracle.RingModel(PM, PS) for _ in range(NL)]
    nan = lambda t: torch.full_like(t, float("nan"))     # a head no group wrote stays NaN

    def sharded(call, ins, out_like):
        """Run `call(cache, *inputs, out)` per group on head views; yield each G's output."""
        for G, shards in groups.items():
            o = nan(out_like)
            for h0, hc, c in shards:
                call(c, *[t[..., h0:h0 + hc, :] for t in ins], o[..., h0:h0 + hc, :])
            yield G, o

    def spatial(L, q, k, v, n, use_prefix):
        dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
        out = torch.empty_like(dq)
        full.spatial_attn(L, dq, dk, dv, out, n, use_prefix)
        ref_bits = to_bits(out)
        for G, o in sharded(lambda c, a, b, d, e: c.spatial_attn(L, a, b, d, e, n, use_prefix), (dq, dk, dv), dq):
            assert np.array_equal(to_bits(o), ref_bits), "spatial, %d groups, layer %d" % (G, L)
        if use_prefix:
            sk, sv = rings[L].spatial()
            ref = oracle.spatial_attn(q, k, v, sk, sv, repeat=0)
        else:
            ref = oracle.spatial_attn(q, k, v, [], [], repeat=PS + 1)
        check_close(ref_bits, ref, "shard6 spatial")

    def temporal(L, q, k, v, n):
        dq, dk, dv = (to_dev(token_major(a)) for a in (q, k, v))
        out = torch.empty_like(dq)
        full.temporal(L, dq, dk, dv, out, n)
        ref_bits = to_bits(out)
        for G, o in sharded(lambda c, a, b, d, e: c.temporal(L, a, b, d, e, n), (dq, dk, dv), dq):
            assert np.array_equal(to_bits(o), ref_bits), "temporal, %d groups, layer %d" % (G, L)
        pk, pv = rings[L].prefix()
        check_close(np.ascontiguousarray(np.swapaxes(ref_bits, 1, 2)), oracle.temporal_attn(q, k, v, pk, pv),
                    "shard6 temporal")

    def all_caches():
        yield full, 0, H
        for shards in groups.values():
            for h0, hc, c in shards:
                yield c, h0, hc

    def check_caches():
        """Queued ring slots and the spatial cache: the unsharded cache against the oracle's
        frames, every group's against the unsharded cache's heads, bit for bit."""
        torch.cuda.synchronize()
        for c, _, _ in all_caches():
            assert c.state() == full.state()
        for L, ring in enumerate(rings):
            assert full.state() == (ring.head, ring.count, len(ring.spatial_ids), ring.frames_written)
            slots = [ring.slot_of(g) for g in ring.queue]
            fr = [to_bits(full.ring(L, kv))[:, :, :, slots] for kv in (0, 1)]       # [B][HW][H][q][D]
            fs = [to_bits(full.spatial(L, kv))[:len(ring.spatial_ids)] for kv in (0, 1)]
            for i, g in enumerate(ring.queue):
                assert np.array_equal(fr[0][:, :, :, i], ring.k[g])
                assert np.array_equal(fr[1][:, :, :, i], f16_bits_of_bf16(ring.v[g]))
            for j, g in enumerate(ring.spatial_ids):
                assert np.array_equal(fs[0][j], ring.sk[g])
                assert np.array_equal(fs[1][j], f16_bits_of_bf16(ring.sv[g]))
            for c, h0, hc in all_caches():
                for kv in (0, 1):
                    assert np.array_equal(to_bits(c.ring(L, kv))[:, :, :, slots], fr[kv][:, :, h0:h0 + hc]), \
                        "ring %s of heads %d..%d, layer %d" % ("KV"[kv], h0, h0 + hc, L)
                    assert np.array_equal(to_bits(c.spatial(L, kv))[:len(ring.spatial_ids)],
                                          fs[kv][:, :, :, h0:h0 + hc]), \
                        "spatial %s of heads %d..%d, layer %d" % ("KV"[kv], h0, h0 + hc, L)

    def write(kv_frames, n):
        evicted = {c.evict_for(n) for c, _, _ in all_caches()}
        assert len(evicted) == 1
        kt = [to_dev(token_major(f[0])) for f in kv_frames]
        vt = [to_dev(token_major(f[1])) for f in kv_frames]
        ks = [to_dev(f[2]) for f in kv_frames]
        vs = [to_dev(f[3]) for f in kv_frames]
        for c, h0, hc in all_caches():
            view = lambda ts: [t[..., h0:h0 + hc, :] for t in ts]
            c.write(view(kt), view(vt), view(ks), view(vs), n)
        e = evicted.pop()
        for L, f in enumerate(kv_frames):
            assert len(rings[L].write(f[0], f[1], f[2], f[3])) == e
        check_caches()

    def pass_(n, use_prefix):
        frames = []
        for L in range(NL):
            sq, sk, sv = gen.qkv(n)
            tq, tk, tv = gen.qkv(n)
            spatial(L, sq, sk, sv, n, use_prefix)
            temporal(L, tq, tk, tv, n)
            frames.append((tk, tv, sk, sv))
        return frames

    write(pass_(1, 0), 1)
    for _ in range(wl.ar_steps):
        pass_(l, 1)
        write(pass_(l, 0), l)
    assert rings[0].evicted == list(range(16))          # frames 0..7, then 8..15

    # cyclic TPE add: table and chunk rows C apart, each group adding its heads' columns
    g0 = rings[0].frames_written
    table = to_dev(gen.frames(full.tpe_len)[0, :, 0].reshape(full.tpe_len, H, D))
    x = to_dev(token_major(gen.frames(l)))
    out = torch.empty_like(x)
    full.tpe_add(g0, 3, table, x, out, l)
    ref = oracle.tpe_add(to_bits(x).reshape(B, HW, l, C), to_bits(table).reshape(-1, C), g0, 3)
    assert np.array_equal(to_bits(out).reshape(ref.shape), ref)
    for G, shards in groups.items():
        o = nan(x)
        for h0, hc, c in shards:
            c.tpe_add(g0, 3, table[:, h0:h0 + hc], x[..., h0:h0 + hc, :], o[..., h0:h0 + hc, :], l)
        assert np.array_equal(to_bits(o), to_bits(out)), "TPE add, %d groups" % G

    # K/V projection into the caches: full-width inputs (Cin = C), each group's weight rows
    # are the K channels and then the V channels of its heads
    rng = np.random.default_rng(5)
    dev = lambda a: torch.from_numpy(a).cuda().to(torch.bfloat16)
    x_t = dev(rng.standard_normal((B, HW, l, C), dtype=np.float32))
    x_s = dev(rng.standard_normal((B, l, HW, C), dtype=np.float32))
    w = [dev(rng.standard_normal((2 * C, C), dtype=np.float32) / np.sqrt(C)) for _ in range(2 * NL)]
    b = [dev(rng.standard_normal(2 * C, dtype=np.float32) * 0.1) for _ in range(2 * NL)]
    evicted = {c.evict_for(l) for c, _, _ in all_caches()}
    assert evicted == {8}
    for c, h0, hc in all_caches():
        rows = torch.cat([torch.arange(h0 * D, (h0 + hc) * D), C + torch.arange(h0 * D, (h0 + hc) * D)]).cuda()
        for L in range(NL):
            c.kv_proj_write(L, x_t, w[2 * L][rows].contiguous(), b[2 * L][rows].contiguous(),
                            x_s, w[2 * L + 1][rows].contiguous(), b[2 * L + 1][rows].contiguous(), l)
        c.commit(l)
    torch.cuda.synchronize()
    head, count, sp, fw = full.state()
    slots = [(head + count - l + f) % PM for f in range(l)]
    for L in range(NL):
        fr = [to_bits(full.ring(L, kv))[:, :, :, slots] for kv in (0, 1)]
        fs = [to_bits(full.spatial(L, kv))[:sp] for kv in (0, 1)]
        for c, h0, hc in all_caches():
            assert c.state() == (head, count, sp, fw)
            for kv in (0, 1):
                assert np.array_equal(to_bits(c.ring(L, kv))[:, :, :, slots], fr[kv][:, :, h0:h0 + hc]), \
                    "projected ring %s of heads %d..%d" % ("KV"[kv], h0, h0 + hc)
                assert np.array_equal(to_bits(c.spatial(L, kv))[:sp], fs[kv][:, :, :, h0:h0 + hc]), \
                    "projected spatial %s of heads %d..%d" % ("KV"[kv], h0, h0 + hc)
    from causal_kv_cache_b200 import ca2
    assert ca2.ca2_device_status() == 0
