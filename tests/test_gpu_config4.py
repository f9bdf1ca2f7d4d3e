"""The 28-block setting (B = 4 videos, 28 attention blocks, C = 1152 in 16 heads of 72, l = 8,
Pmax = 41, P' = 3) run as a spatial-temporal chain, teacher-forced per layer against the oracle.

Each block is spatial attention then temporal attention, each x += W_o attn(W_q y, W_k y, W_v y)
with y = LayerNorm(x) (no affine part: the pre-norm of the Open-Sora backbone's blocks, which
keeps every layer's Q, K, V at unit scale while the residual stream grows) and random bf16
weights ~ N(0, 1/C) (the harness around the path; the projections are torch matmuls, not the
product).  The hidden state of the first frame and of every chunk is
N(0, 1).  Per layer, the oracle takes the exact bf16 Q, K, V the GPU kernels received and checks
the attention outputs of fixed samples: 256 (b, s, h) temporal rows and 4 (b, h) spatial
frame-heads (all tokens of one chunk frame).  The oracle keeps its own FIFO of those samples'
K/V frames by global frame id (it never reads the GPU's ring), fed the same bf16 K/V the cache
write receives.  First frame, then 5 AR steps of one denoising pass and the cache-writing pass:
queue lengths 1, 9, 17, 25, 33.
"""
import numpy as np
import pytest

import oracle
from ca2_synth import WORKLOADS

pytestmark = pytest.mark.gpu


def test_28_blocks_b4_teacher_forced_sampled():
    import torch
    from causal_kv_cache_b200.ca2 import KVCache
    from tests.gpu_util import check_close, to_bits
    wl = WORKLOADS["os_28blk"]
    B, H, D, HW, l, PM, PS, NL = (wl.batch, wl.heads, wl.head_dim, wl.hw, wl.chunk_len, wl.p_max, wl.p_spatial,
                                  wl.n_layers)
    C = H * D
    dev = torch.device("cuda", torch.cuda.current_device())
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    bf = torch.bfloat16
    # per layer: spatial (q, k, v, o) and temporal (q, k, v, o) weights [C_out][C_in]
    W = [[(torch.randn((C, C), generator=g, device=dev) * C ** -0.5).to(bf) for _ in range(8)] for _ in range(NL)]
    cache = KVCache(NL, B, HW, H, D, l, PM, PS)
    rng = np.random.default_rng(4)
    t_units = [rng.choice(B * HW * H, size=256, replace=False) for _ in range(NL)]    # (b*HW + s)*H + h
    s_pairs = [rng.choice(B * H, size=4, replace=False) for _ in range(NL)]          # b*H + h
    rings = [oracle.RingModel(PM, PS) for _ in range(NL)]
    checked = {"temporal": 0, "spatial": 0}

    def heads(t):                       # [..., C] -> [..., H, D]
        return t.reshape(*t.shape[:-1], H, D)

    def norm(t):                        # LayerNorm over the channels, fp32, no affine part
        return torch.nn.functional.layer_norm(t.float(), (C,)).to(bf)

    # sample indices on the device: only the samples are copied to the host
    t_idx = [tuple(torch.as_tensor(a, device=dev) for a in (u // (HW * H), (u // H) % HW, u % H)) for u in t_units]
    s_idx = [tuple(torch.as_tensor(a, device=dev) for a in (pr // H, pr % H)) for pr in s_pairs]

    def t_sample(x_tm, L):
        """token-major [B][HW][n][H][D] -> the layer's temporal sample as [1][n][256][1][D] bits."""
        b, s, h = t_idx[L]
        a = to_bits(x_tm[b, s, :, h, :])                                   # [256][n][D]
        return np.ascontiguousarray(a.transpose(1, 0, 2)[None, :, :, None, :])

    def s_sample(x_fm, L):
        """frame-major [B][n][HW][H][D] -> the layer's spatial sample as [4][n][HW][1][D] bits."""
        b, h = s_idx[L]
        a = to_bits(x_fm[b, :, :, h, :])                                   # [4][n][HW][D]
        return np.ascontiguousarray(a[:, :, :, None, :])

    def run_pass(n, use_prefix):
        """One forward pass of the 28 blocks over n frames; returns each layer's K/V for the cache."""
        x = torch.randn((B, n, HW, C), generator=g, device=dev).to(bf)
        kv = []
        for L in range(NL):
            wq, wk, wv, wo, tq_, tk_, tv_, to_ = W[L]
            # spatial: frame-major [B][n][HW][H][D]
            y = norm(x)
            q, k, v = (heads(y @ w.t()).contiguous() for w in (wq, wk, wv))
            o = torch.empty_like(q)
            cache.spatial_attn(L, q, k, v, o, n, use_prefix)
            ring = rings[L]
            sq, sk_, sv_ = s_sample(q, L), s_sample(k, L), s_sample(v, L)
            f = int(rng.integers(0, n))                                    # one chunk frame per call
            if use_prefix:
                ck, cv = ring.spatial()                                    # [4][HW][1][D] per cache frame
                ref = oracle.spatial_attn(sq[:, f:f + 1], sk_[:, f:f + 1], sv_[:, f:f + 1], ck, cv, repeat=0)
            else:
                ref = oracle.spatial_attn(sq[:, f:f + 1], sk_[:, f:f + 1], sv_[:, f:f + 1], [], [], repeat=PS + 1)
            got = s_sample(o, L)[:, f:f + 1]
            check_close(got, ref, "os_28blk spatial")
            checked["spatial"] += 1
            x = x + (o.reshape(B, n, HW, C) @ wo.t()).to(bf)
            # temporal: token-major [B][HW][n][H][D]
            yt = norm(x.transpose(1, 2).contiguous())
            q, k2, v2 = (heads(yt @ w.t()).contiguous() for w in (tq_, tk_, tv_))
            o2 = torch.empty_like(q)
            cache.temporal(L, q, k2, v2, o2, n)
            pk, pv = ring.prefix()                                         # [1][256][1][D] per queued frame
            ref = oracle.temporal_attn(t_sample(q, L), t_sample(k2, L), t_sample(v2, L), pk, pv)
            check_close(t_sample(o2, L), ref, "os_28blk temporal")
            checked["temporal"] += 1
            x = x + (o2.reshape(B, HW, n, C) @ to_.t()).to(bf).transpose(1, 2)
            kv.append((k2, v2, k, v))
        return kv

    def write(kv, n):
        e = cache.evict_for(n)
        cache.write([a[0] for a in kv], [a[1] for a in kv], [a[2] for a in kv], [a[3] for a in kv], n)
        for L, (k2, v2, k, v) in enumerate(kv):
            # the oracle's frames: the temporal sample [1][n][256][1][D], the spatial one [4][n][HW][1][D]
            gone = rings[L].write(t_sample(k2, L), t_sample(v2, L), s_sample(k, L), s_sample(v, L))
            assert len(gone) == e

    write(run_pass(1, 0), 1)                       # the first frame (a clean prefix frame)
    queue = []
    for _ in range(wl.ar_steps):
        queue.append(rings[0].count)
        run_pass(l, 1)                             # a denoising pass reading the cache
        write(run_pass(l, 0), l)                   # the cache-writing pass over the clean chunk
    torch.cuda.synchronize()
    from causal_kv_cache_b200 import ca2
    assert ca2.ca2_device_status() == 0
    assert queue == [1, 9, 17, 25, 33]
    assert cache.state()[1] == 41 and rings[0].count == 41
    assert checked == {"temporal": NL * 11, "spatial": NL * 11}
