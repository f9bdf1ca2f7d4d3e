"""The C ABI of libca2.so on the host: exports, validation and host-only state (no GPU)."""
import ctypes
import os
import re

import pytest

import oracle
from causal_kv_cache_b200 import ca2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE_T = 0x7F0000000000          # 16-byte aligned stand-ins; never dereferenced on the host
FAKE_S = 0x7F1000000000


def cfg(**kw):
    base = dict(n_layers=1, batch=1, hw=256, heads=16, head_dim=72, chunk_len=8, p_max=41,
                p_spatial=3, tpe_len=0, row_pitch=0)
    base.update(kw)
    return base


def make(**kw):
    c = cfg(**kw)
    tb, sb = ca2.ca2_cache_bytes(c)
    return ca2.ca2_cache_init(c, FAKE_T, tb, FAKE_S if sb else None, sb), c


def test_library_exports_every_declared_symbol():
    with open(os.path.join(ROOT, "include", "ca2.h")) as f:
        header = f.read()
    declared = set(re.findall(r"^(?:int|const char \*)\s*(ca2_\w+)\s*\(", header, re.M))
    assert {"ca2_cache_init", "ca2_cache_write", "ca2_temporal_attn", "ca2_spatial_prefix_attn",
            "ca2_cache_evict"} <= declared
    lib = ctypes.CDLL(ca2.LIBRARY_PATH)
    for name in sorted(declared):
        assert hasattr(lib, name), name
    assert set(ca2.__all__) >= declared


def test_cache_bytes_matches_oracle_and_memory_table():
    for kw in (dict(), dict(n_layers=28, batch=4, p_max=41), dict(n_layers=28, p_max=25),
               dict(hw=16, heads=2, head_dim=16, chunk_len=4, p_max=9, p_spatial=1)):
        c = cfg(**kw)
        t, s = ca2.ca2_cache_bytes(c)
        assert t + s == oracle.cache_bytes(c["n_layers"], c["batch"], c["hw"], c["heads"], c["head_dim"],
                                           c["p_max"], c["p_spatial"])
        assert s == oracle.cache_bytes(c["n_layers"], c["batch"], c["hw"], c["heads"], c["head_dim"], 0,
                                       c["p_spatial"])
    # the Ca2-VDM memory-table setting: 0.86 GiB with prefix enhancement
    t, s = ca2.ca2_cache_bytes(cfg(n_layers=28, p_max=25))
    assert t + s == 924_844_032


@pytest.mark.parametrize("bad,code", [
    (dict(head_dim=12), -2), (dict(head_dim=136), -2), (dict(head_dim=0), -2),
    (dict(chunk_len=9), -2), (dict(chunk_len=0), -2), (dict(p_max=7), -2),
    (dict(p_spatial=9), -2), (dict(p_spatial=-1), -2), (dict(n_layers=0), -2),
    (dict(batch=0), -2), (dict(hw=0), -2), (dict(heads=0), -2), (dict(tpe_len=-1), -2),
])
def test_invalid_configs_rejected(bad, code):
    with pytest.raises(ca2.Ca2Error) as e:
        ca2.ca2_cache_bytes(cfg(**bad))
    assert e.value.status == code


def test_init_validation():
    c = cfg()
    tb, sb = ca2.ca2_cache_bytes(c)
    with pytest.raises(ca2.Ca2Error) as e:
        ca2.ca2_cache_init(c, FAKE_T, tb - 1, FAKE_S, sb)
    assert e.value.status == -3
    with pytest.raises(ca2.Ca2Error) as e:
        ca2.ca2_cache_init(c, FAKE_T, tb, FAKE_S, sb - 16)
    assert e.value.status == -3
    with pytest.raises(ca2.Ca2Error) as e:
        ca2.ca2_cache_init(c, FAKE_T + 8, tb, FAKE_S, sb)
    assert e.value.status == -4
    with pytest.raises(ca2.Ca2Error) as e:
        ca2.ca2_cache_init(c, None, tb, FAKE_S, sb)
    assert e.value.status == -1
    with pytest.raises(ca2.Ca2Error) as e:
        ca2.ca2_cache_init(c, FAKE_T, tb, None, sb)
    assert e.value.status == -1
    # P' = 0 needs no spatial buffer
    c0 = cfg(p_spatial=0)
    tb0, sb0 = ca2.ca2_cache_bytes(c0)
    assert sb0 == 0
    h = ca2.ca2_cache_init(c0, FAKE_T, tb0, None, 0)
    ca2.ca2_cache_destroy(h)
    ca2.ca2_cache_destroy(None)


def test_fresh_state_and_evict_bounds():
    h, c = make()
    assert ca2.ca2_cache_state(h) == (0, 0, 0, 0)
    ca2.ca2_cache_evict(h, 0)
    with pytest.raises(ca2.Ca2Error) as e:
        ca2.ca2_cache_evict(h, 1)
    assert e.value.status == -3
    with pytest.raises(ca2.Ca2Error) as e:
        ca2.ca2_cache_evict(h, -1)
    assert e.value.status == -3
    ca2.ca2_cache_destroy(h)


def test_call_validation_before_any_launch():
    h, c = make()
    al = 0x7E0000000000
    # temporal / spatial argument checks
    for fn in (lambda *a: ca2.ca2_temporal_attn(h, *a, stream=0),
               lambda *a: ca2.ca2_spatial_prefix_attn(h, *a, 1, stream=0)):
        with pytest.raises(ca2.Ca2Error) as e:
            fn(1, al, al, al, al, 8)
        assert e.value.status == -1          # layer out of range
        with pytest.raises(ca2.Ca2Error) as e:
            fn(0, None, al, al, al, 8)
        assert e.value.status == -1
        with pytest.raises(ca2.Ca2Error) as e:
            fn(0, al, al, al, al, 9)
        assert e.value.status == -2          # more frames than the chunk length
        with pytest.raises(ca2.Ca2Error) as e:
            fn(0, al, al, al, al, 0)
        assert e.value.status == -2
        with pytest.raises(ca2.Ca2Error) as e:
            fn(0, al + 2, al, al, al, 8)
        assert e.value.status == -4
    with pytest.raises(ca2.Ca2Error) as e:
        ca2.ca2_spatial_prefix_attn(h, 0, al, al, al, al, 8, 2, stream=0)
    assert e.value.status == -1
    # cache write checks: shape, missing spatial tensors, alignment, capacity
    with pytest.raises(ca2.Ca2Error) as e:
        ca2.ca2_cache_write(h, [al], [al], [al], [al], 9, stream=0)
    assert e.value.status == -2
    with pytest.raises(ca2.Ca2Error) as e:
        ca2.ca2_cache_write(h, [al], [al], None, None, 8, stream=0)
    assert e.value.status == -1
    with pytest.raises(ca2.Ca2Error) as e:
        ca2.ca2_cache_write(h, [al + 4], [al], [al], [al], 8, stream=0)
    assert e.value.status == -4
    # TPE add checks: null pointers, negative frame/offset, frame count, alignment
    for args, code in (((0, 0, None, al, al, 8), -1), ((0, 0, al, al, None, 8), -1), ((-1, 0, al, al, al, 8), -1),
                       ((0, -3, al, al, al, 8), -1), ((0, 0, al, al, al, 0), -2), ((0, 0, al, al, al, 9), -2),
                       ((0, 0, al + 8, al, al, 8), -4), ((0, 0, al, al, al + 2, 8), -4)):
        with pytest.raises(ca2.Ca2Error) as e:
            ca2.ca2_tpe_add(h, *args, stream=0)
        assert e.value.status == code, args
    ca2.ca2_cache_destroy(h)
    # capacity: Pmax = 8 = l; a full chunk fits once, the next needs eviction first
    h2, _ = make(p_max=8)
    with pytest.raises(ca2.Ca2Error):
        ca2.ca2_cache_write(h2, [al], [al], [al], [al], 9, stream=0)
    ca2.ca2_cache_destroy(h2)


def test_tpe_indices_match_oracle():
    h, c = make()
    n_tpe = c["p_max"] + c["chunk_len"]       # tpe_len 0 selects Pmax + l
    for g0 in (0, 1, 41, 45, 49, 1000, 10 ** 12):
        for off in (0, 7, 48):
            assert ca2.ca2_tpe_indices(h, g0, off, 8) == oracle.tpe_indices(g0, off, 8, n_tpe)
    assert ca2.ca2_tpe_indices(h, 5, 0, 0) == []
    with pytest.raises(ca2.Ca2Error):
        ca2.ca2_tpe_indices(h, -1, 0, 1)
    ca2.ca2_cache_destroy(h)
    h, c = make(tpe_len=16)
    assert ca2.ca2_tpe_indices(h, 14, 1, 4) == oracle.tpe_indices(14, 1, 4, 16)
    ca2.ca2_cache_destroy(h)


def test_status_strings():
    for code in range(-8, 1):
        assert ca2.ca2_status_string(code) != "unknown status"
    assert ca2.ca2_status_string(-99) == "unknown status"


def test_kv_proj_write_validation_and_commit():
    """The fused projection write rejects bad arguments before any device work, and
    ca2_cache_commit advances the queue exactly as a cache write of n frames does."""
    h, c = make()
    X, W, B = FAKE_T + 0x100000, FAKE_T + 0x200000, FAKE_T + 0x300000
    bad = [
        (dict(x_t=None), -1), (dict(w_t=None), -1), (dict(layer=1), -1), (dict(layer=-1), -1),
        (dict(n=0), -2), (dict(n=9), -2), (dict(x_t=X + 8), -4), (dict(w_t=W + 2), -4),
        (dict(b_t=B + 4), -4), (dict(x_s=None), -1), (dict(w_s=None), -1), (dict(x_s=X + 8), -4),
    ]
    for kw, status in bad:
        a = dict(layer=0, x_t=X, w_t=W, b_t=B, x_s=X, w_s=W, b_s=None, n=8)
        a.update(kw)
        with pytest.raises(ca2.Ca2Error) as e:
            ca2.ca2_kv_proj_write(h, a["layer"], a["x_t"], a["w_t"], a["b_t"], a["x_s"], a["w_s"], a["b_s"], a["n"])
        assert e.value.status == status, (kw, e.value.status)
    # commit: count += n, the spatial cache holds min(P', n) frames
    ca2.ca2_cache_commit(h, 1)
    assert ca2.ca2_cache_state(h) == (0, 1, 1, 1)
    ca2.ca2_cache_commit(h, 8)
    assert ca2.ca2_cache_state(h) == (0, 9, 3, 9)
    for n, status in ((0, -2), (9, -2)):
        with pytest.raises(ca2.Ca2Error) as e:
            ca2.ca2_cache_commit(h, n)
        assert e.value.status == status
    ca2.ca2_cache_destroy(h)
    # a write or commit past Pmax needs an eviction first
    h, c = make(p_max=8)
    ca2.ca2_cache_commit(h, 8)
    with pytest.raises(ca2.Ca2Error) as e:
        ca2.ca2_kv_proj_write(h, 0, X, W, None, X, W, None, 1)
    assert e.value.status == -3
    with pytest.raises(ca2.Ca2Error) as e:
        ca2.ca2_cache_commit(h, 1)
    assert e.value.status == -3
    ca2.ca2_cache_evict(h, 1)
    ca2.ca2_cache_commit(h, 1)
    assert ca2.ca2_cache_state(h) == (1, 8, 1, 9)
    ca2.ca2_cache_destroy(h)
    # P' = 0: the spatial operands are not needed
    h, c = make(p_spatial=0)
    with pytest.raises(ca2.Ca2Error) as e:
        ca2.ca2_kv_proj_write(h, 0, X + 8, W, None, None, None, None, 8)
    assert e.value.status == -4
    ca2.ca2_cache_destroy(h)


def test_evict_for_matches_oracle_fifo():
    """ca2_cache_evict_for evicts exactly the frames the oracle's FIFO drops when n_new more
    are appended (papernotes page, 关键设计 4), over a random schedule of chunk lengths; the
    queue is advanced on the host with ca2_cache_commit (no device work)."""
    import numpy as np
    rng = np.random.default_rng(5)
    for p_max, l in ((41, 8), (9, 4), (8, 8), (13, 5)):
        h, c = make(p_max=p_max, chunk_len=l, p_spatial=min(3, l))
        ring = oracle.RingModel(p_max, min(3, l))
        z = np.zeros((1, 1, 1, 1, 1), dtype=np.uint16)
        for step in range(40):
            n = int(rng.integers(1, l + 1)) if step else 1
            e = ca2.ca2_cache_evict_for(h, n)
            ca2.ca2_cache_commit(h, n)
            zz = np.zeros((1, n, 1, 1, 1), dtype=np.uint16)
            gone = ring.write(zz, zz, zz, zz)
            assert e == len(gone), (p_max, l, step)
            head, count, sp, fw = ca2.ca2_cache_state(h)
            assert (head, count, sp, fw) == (ring.head, ring.count, len(ring.spatial_ids), ring.frames_written)
        for bad in (-1, p_max + 1):
            with pytest.raises(ca2.Ca2Error) as err:
                ca2.ca2_cache_evict_for(h, bad)
            assert err.value.status == -2
        assert ca2.ca2_cache_evict_for(h, 0) == 0
        ca2.ca2_cache_destroy(h)


def test_config_defaults_resolved_by_the_library():
    h, c = make()
    got = ca2.ca2_cache_config(h)
    assert (got.tpe_len, got.row_pitch) == (c["p_max"] + c["chunk_len"], c["heads"] * c["head_dim"])
    assert (got.n_layers, got.batch, got.hw, got.heads, got.head_dim) == (1, 1, 256, 16, 72)
    ca2.ca2_cache_destroy(h)
    h, c = make(tpe_len=16, row_pitch=16 * 72 * 4)
    got = ca2.ca2_cache_config(h)
    assert (got.tpe_len, got.row_pitch) == (16, 16 * 72 * 4)
    ca2.ca2_cache_destroy(h)


@pytest.mark.parametrize("pitch,ok", [(0, True), (1152, True), (1152 + 8, True), (4608, True),
                                      (1144, False), (1156, False), (-8, False)])
def test_row_pitch_validation(pitch, ok):
    if ok:
        ca2.ca2_cache_bytes(cfg(row_pitch=pitch))
    else:
        with pytest.raises(ca2.Ca2Error) as e:
            ca2.ca2_cache_bytes(cfg(row_pitch=pitch))
        assert e.value.status == -2


def test_layer_offsets_follow_the_documented_layout():
    """Offsets of each layer's K/V ring and spatial cache: temporal [N_L][2][B][HW][H][Pmax][D]
    and spatial [N_L][2][P'][B][HW][H][D] bf16, as include/ca2.h states."""
    h, c = make(n_layers=3, batch=2)
    plane = c["batch"] * c["hw"] * c["heads"] * c["head_dim"] * 2
    for L in range(3):
        for kv in (0, 1):
            t, s = ca2.ca2_cache_layer_offsets(h, L, kv)
            assert t == (L * 2 + kv) * c["p_max"] * plane
            assert s == (L * 2 + kv) * c["p_spatial"] * plane
    for bad in ((3, 0), (-1, 0), (0, 2)):
        with pytest.raises(ca2.Ca2Error):
            ca2.ca2_cache_layer_offsets(h, *bad)
    ca2.ca2_cache_destroy(h)


def test_head_shard_partition():
    """ca2_head_shard: for every head count up to 32 and every world size up to it, the ranks'
    ranges are contiguous, in rank order, cover [0, H) once, and differ in size by at most one
    (the larger ones first); bad arguments are rejected."""
    for H in range(1, 33):
        for world in range(1, H + 1):
            parts = [ca2.ca2_head_shard(H, world, r) for r in range(world)]
            assert parts[0][0] == 0
            for (a0, ac), (b0, _) in zip(parts, parts[1:]):
                assert b0 == a0 + ac
            assert parts[-1][0] + parts[-1][1] == H
            sizes = [hc for _, hc in parts]
            assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
    for bad in ((4, 0, 0), (4, 5, 0), (4, 2, 2), (4, 2, -1), (0, 1, 0)):
        with pytest.raises(ca2.Ca2Error) as e:
            ca2.ca2_head_shard(*bad)
        assert e.value.status == -2


def test_header_is_plain_c_and_links(tmp_path):
    """include/ca2.h compiles as C99 with warnings as errors, and a C program that calls the
    library through it links against libca2.so and runs the host-only calls."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_ca2.c"
    src.write_text(r'''
#include <stdio.h>
#include "ca2.h"
int main(void)
{
    ca2_config c = {2, 1, 16, 2, 16, 4, 9, 1, 0, 0};
    size_t tb = 0, sb = 0;
    int h0 = -1, hc = -1;
    if (ca2_cache_bytes(&c, &tb, &sb) != CA2_OK) return 1;
    if (ca2_head_shard(5, 2, 1, &h0, &hc) != CA2_OK || h0 != 3 || hc != 2) return 2;
    if (ca2_head_shard(1, 2, 0, &h0, &hc) != CA2_ERR_SHAPE) return 3;
    printf("%zu %zu %s\n", tb, sb, ca2_status_string(CA2_ERR_RANGE));
    return 0;
}
''')
    exe = tmp_path / "use_ca2"
    lib_dir = os.path.dirname(ca2.LIBRARY_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                    str(exe), "-L", lib_dir, "-lca2", "-Wl,-rpath," + lib_dir], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    tb, sb = ca2.ca2_cache_bytes(cfg(n_layers=2, hw=16, heads=2, head_dim=16, chunk_len=4, p_max=9, p_spatial=1))
    assert r.stdout.split()[:2] == [str(tb), str(sb)]
