"""Pins that tie the CPU oracle to what the pages and the mathematics fix.

Each ``pin_*`` takes a loaded oracle library handle and raises AssertionError when the
oracle disagrees with an independent statement of the same fact: a brute-force
full-sequence masked attention written as matrices, torch's scaled_dot_product_attention
in fp64 for the unmasked special cases, closed forms, and the pages' own numbers.
``test_oracle_pins.py`` runs them on the real oracle and on planted mutants of it.
"""
from __future__ import annotations

import math

import numpy as np

import oracle
from ca2_synth import Generator, WORKLOADS, Workload, bf16_bits, bf16_to_f32

TINY = WORKLOADS["tiny"]


def _f64(bits):
    return bf16_to_f32(bits).astype(np.float64)


def _wl(**kw) -> Workload:
    base = dict(name="pin", batch=2, heads=2, head_dim=16, hw=3, chunk_len=4, p_max=9,
                p_spatial=2, n_layers=1, ar_steps=1, denoise_steps=1, recipe="normal", scale=0.6)
    base.update(kw)
    return Workload(**base)


def brute_causal(q_seq, k_seq, v_seq):
    """softmax(Q K^T / sqrt(D) + M) V for one (b, s, h) with M_ij = -inf when i < j.

    q_seq, k_seq, v_seq: [L][D] float64.  Written as whole matrices on purpose, unlike the
    oracle's per-query loops.
    """
    L, D = q_seq.shape
    logits = q_seq @ k_seq.T / math.sqrt(D)
    mask = np.triu(np.full((L, L), -np.inf), k=1)
    logits = logits + mask
    logits -= logits.max(axis=1, keepdims=True)
    w = np.exp(logits)
    w /= w.sum(axis=1, keepdims=True)
    return w @ v_seq


def _sequence(prefix, chunk, b, s, h):
    """Stack the (b, s, h) D-vectors of prefix frames then chunk frames into [L][D]."""
    rows = [_f64(f[b, s, h]) for f in prefix]
    rows += [_f64(chunk[b, c, s, h]) for c in range(chunk.shape[1])]
    return np.stack(rows)


def pin_temporal_full_sequence(lib, seed=3, P=5, n=4, recipe="normal"):
    """Invariant (a): attention of a chunk over the cached prefix equals the chunk rows of
    full-sequence masked attention recomputed from scratch over [prefix || chunk]."""
    wl = _wl(recipe=recipe)
    g = Generator(wl, seed)
    pq, pk, pv = g.qkv(P)              # prefix frames (their queries only fill the matrix)
    q, k, v = g.qkv(n)
    prefix_k = [pk[:, p] for p in range(P)]
    prefix_v = [pv[:, p] for p in range(P)]
    got = oracle.temporal_attn(q, k, v, prefix_k, prefix_v, lib=lib)
    for b in range(wl.batch):
        for s in range(wl.hw):
            for h in range(wl.heads):
                Q = _sequence([pq[:, p] for p in range(P)], q, b, s, h)
                K = _sequence(prefix_k, k, b, s, h)
                V = _sequence(prefix_v, v, b, s, h)
                ref = brute_causal(Q, K, V)[P:]
                np.testing.assert_allclose(got[b, :, s, h], ref, rtol=1e-12, atol=1e-13)


def pin_temporal_no_prefix(lib):
    """Invariant (a) with an empty queue: plain causal attention inside the chunk."""
    pin_temporal_full_sequence(lib, seed=11, P=0, n=4)


def pin_temporal_peaky(lib):
    """Invariant (a) with sharp softmax rows (values x2): the max subtraction must hold."""
    pin_temporal_full_sequence(lib, seed=5, P=3, n=3, recipe="peaky")


def pin_single_visible_key(lib):
    """Invariant (d): the first frame's pass (empty queue, one frame) returns V exactly."""
    wl = _wl(batch=1, hw=5)
    g = Generator(wl, 7)
    q, k, v = g.qkv(1)
    got = oracle.temporal_attn(q, k, v, [], [], lib=lib)
    assert np.array_equal(got, _f64(v)), "single visible key must return V exactly"


def pin_causal_closed_form(lib):
    """Closed form.  D = 16, so logits are q.k / 4.  Query of chunk frame 0 with one cached
    frame: q = 2 e0, k_prefix = 0, k_chunk0 = 2 e0 -> logits (0, 1), weights
    (1, e) / (1 + e).  A later chunk frame 1 must not leak into frame 0 (causal mask)."""
    B, HW, H, D = 1, 1, 1, 16
    e0 = np.zeros(D, np.float32)
    e0[0] = 1.0
    q = np.zeros((B, 2, HW, H, D), np.float32)
    k = np.zeros_like(q)
    v = np.zeros_like(q)
    q[0, 0, 0, 0] = 2 * e0
    k[0, 0, 0, 0] = 2 * e0
    v[0, 0, 0, 0] = np.arange(D, dtype=np.float32) * 0.5
    k[0, 1, 0, 0] = 50 * e0          # would dominate frame 0 if the mask leaked
    v[0, 1, 0, 0] = 1000.0
    pkf = np.zeros((B, HW, H, D), np.float32)
    pvf = np.full((B, HW, H, D), -3.0, np.float32)
    got = oracle.temporal_attn(bf16_bits(q), bf16_bits(k), bf16_bits(v),
                               [bf16_bits(pkf)], [bf16_bits(pvf)], lib=lib)
    w1 = math.e / (1.0 + math.e)
    expect = (1.0 - w1) * -3.0 + w1 * (np.arange(D) * 0.5)
    np.testing.assert_allclose(got[0, 0, 0, 0], expect, rtol=1e-14, atol=1e-14)


def pin_eviction_last_pmax(lib):
    """Invariant (b): after the queue has evicted, cached attention equals full-sequence
    attention over only the last Pmax prefix frames, and differs from attention over the
    whole history."""
    wl = _wl(batch=1, hw=2, p_max=9, chunk_len=4, p_spatial=1)
    g = Generator(wl, 21)
    ring = oracle.RingModel(wl.p_max, wl.p_spatial)
    hist_q, hist_k, hist_v = [], [], []
    # first frame, then chunks of 4 until the queue has evicted
    for n in (1, 4, 4, 4):
        q, k, v = g.qkv(n)
        ring.write(k, v, k, v)
        hist_q.append(q)
        hist_k.append(k)
        hist_v.append(v)
    assert ring.count == wl.p_max and ring.evicted == [0, 1, 2, 3]
    q, k, v = g.qkv(wl.chunk_len)
    pk, pv = ring.prefix()
    got = oracle.temporal_attn(q, k, v, pk, pv, lib=lib)
    allq = np.concatenate(hist_q, axis=1)
    allk = np.concatenate(hist_k, axis=1)
    allv = np.concatenate(hist_v, axis=1)
    keep = slice(allk.shape[1] - wl.p_max, None)
    for s in range(wl.hw):
        for h in range(wl.heads):
            Q = _sequence([f for f in np.moveaxis(allq[:, keep], 1, 0)], q, 0, s, h)
            K = _sequence([f for f in np.moveaxis(allk[:, keep], 1, 0)], k, 0, s, h)
            V = _sequence([f for f in np.moveaxis(allv[:, keep], 1, 0)], v, 0, s, h)
            ref = brute_causal(Q, K, V)[wl.p_max:]
            np.testing.assert_allclose(got[0, :, s, h], ref, rtol=1e-12, atol=1e-13)
            Qa = _sequence([f for f in np.moveaxis(allq, 1, 0)], q, 0, s, h)
            Ka = _sequence([f for f in np.moveaxis(allk, 1, 0)], k, 0, s, h)
            Va = _sequence([f for f in np.moveaxis(allv, 1, 0)], v, 0, s, h)
            full = brute_causal(Qa, Ka, Va)[allk.shape[1]:]
            assert np.abs(full - got[0, :, s, h]).max() > 1e-6, "eviction had no effect"


def pin_cache_sharing(lib):
    """Invariant (c): the prefix K/V do not depend on the denoising step, so reading one
    cache at every step equals rebuilding it before every step, bit for bit."""
    wl = _wl(batch=1, hw=3)
    g = Generator(wl, 31)
    ring = oracle.RingModel(wl.p_max, wl.p_spatial)
    q0, k0, v0 = g.qkv(5)
    ring.write(k0, v0, k0, v0)
    chunk = g.qkv(4)
    pk, pv = ring.prefix()
    first = oracle.temporal_attn(*chunk, pk, pv, lib=lib)
    for _t in range(3):
        again = oracle.temporal_attn(*chunk, pk, pv, lib=lib)
        assert np.array_equal(first, again)
        fresh = oracle.RingModel(wl.p_max, wl.p_spatial)
        fresh.write(k0.copy(), v0.copy(), k0.copy(), v0.copy())
        rebuilt = oracle.temporal_attn(*chunk, *fresh.prefix(), lib=lib)
        assert np.array_equal(first, rebuilt)


def _sdpa(qf, kf, vf):
    import torch
    import torch.nn.functional as F
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    return F.scaled_dot_product_attention(t(qf), t(kf), t(vf)).numpy()


def pin_spatial_self_is_sdpa(lib):
    """Invariant (e): with no prefix frames (P' = 0) spatial attention is plain per-frame
    self-attention; self-repeat R times gives the same result (the repeated keys scale
    numerator and denominator alike).  Checked against torch SDPA in fp64."""
    wl = _wl(batch=2, hw=7, heads=3, head_dim=16, recipe="normal", scale=0.7)
    g = Generator(wl, 41)
    q, k, v = g.qkv(3)
    for R in (1, 4):
        got = oracle.spatial_attn(q, k, v, [], [], repeat=R, lib=lib)
        for b in range(wl.batch):
            for f in range(3):
                for h in range(wl.heads):
                    ref = _sdpa(_f64(q[b, f, :, h]), _f64(k[b, f, :, h]), _f64(v[b, f, :, h]))
                    np.testing.assert_allclose(got[b, f, :, h], ref, rtol=1e-11, atol=1e-13)


def pin_spatial_prefix_is_sdpa_concat(lib):
    """Prefix-enhanced spatial attention: keys/values are the own frame's tokens followed by
    each cached prefix frame's tokens along the spatial axis; map size HW x (1+n)HW."""
    wl = _wl(batch=2, hw=6, heads=2, head_dim=16, recipe="normal", scale=0.7)
    g = Generator(wl, 43)
    q, k, v = g.qkv(2)
    _, ck, cv = g.qkv(3)
    sk = [ck[:, p] for p in range(3)]
    sv = [cv[:, p] for p in range(3)]
    got = oracle.spatial_attn(q, k, v, sk, sv, repeat=0, lib=lib)
    for b in range(wl.batch):
        for f in range(2):
            for h in range(wl.heads):
                K = np.concatenate([_f64(k[b, f, :, h])] + [_f64(x[b, :, h]) for x in sk])
                V = np.concatenate([_f64(v[b, f, :, h])] + [_f64(x[b, :, h]) for x in sv])
                assert K.shape[0] == (1 + 3) * wl.hw
                ref = _sdpa(_f64(q[b, f, :, h]), K, V)
                np.testing.assert_allclose(got[b, f, :, h], ref, rtol=1e-11, atol=1e-13)


def pin_sampled_units(lib):
    """Unit-sampled calls return exactly the rows of the full call."""
    wl = _wl(batch=2, hw=4, heads=2)
    g = Generator(wl, 51)
    q, k, v = g.qkv(3)
    _, pk, pv = g.qkv(2)
    pkl, pvl = [pk[:, 0], pk[:, 1]], [pv[:, 0], pv[:, 1]]
    full = oracle.temporal_attn(q, k, v, pkl, pvl, lib=lib)
    units = np.array([0, 5, 13, 15])
    part = oracle.temporal_attn(q, k, v, pkl, pvl, units=units, lib=lib)
    for i, u in enumerate(units):
        h, s, b = u % 2, (u // 2) % 4, u // 8
        assert np.array_equal(part[i], full[b, :, s, h])
    fulls = oracle.spatial_attn(q, k, v, pkl, pvl, lib=lib)
    units = np.array([1, 4, 11])
    parts = oracle.spatial_attn(q, k, v, pkl, pvl, units=units, lib=lib)
    for i, u in enumerate(units):
        h, f, b = u % 2, (u // 2) % 3, u // 6
        assert np.array_equal(parts[i], fulls[b, f, :, h])


ALL_PINS = [
    pin_temporal_full_sequence, pin_temporal_no_prefix, pin_temporal_peaky,
    pin_single_visible_key, pin_causal_closed_form, pin_eviction_last_pmax,
    pin_cache_sharing, pin_spatial_self_is_sdpa, pin_spatial_prefix_is_sdpa_concat,
    pin_sampled_units,
]
