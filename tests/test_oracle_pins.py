"""The CPU oracle against its pins (runs without a GPU)."""
import os
import subprocess

import numpy as np
import pytest

import oracle
from tests import oracle_pins as pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def lib():
    return oracle.load()


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(lib, pin):
    pin(lib)


def _read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split("|"))
    return rows


def test_memory_table_pins_cache_bytes():
    """The pages' KV-cache memory (0.86 GB with prefix enhancement, 0.77 GB without) is the
    size of one shared cache of Pmax = 25 temporal frames (+ P' = 3 spatial frames) over
    the 28 Open-Sora v1.0 blocks at C = 1152, 256 tokens per frame, bf16 K and V, batch 1,
    in GiB.  A dropped K/V factor, a per-timestep copy or a wrong frame count misses it."""
    rows = {r[0]: float(r[1]) for r in _read_table("memory_table.txt")}
    gib = 2.0 ** 30
    with_pe = oracle.cache_bytes(28, 1, 256, 16, 72, 25, 3)
    without = oracle.cache_bytes(28, 1, 256, 16, 72, 25, 0)
    assert round(with_pe / gib, 2) == rows["Ca2-VDM w/ PE"]
    assert round(without / gib, 2) == rows["Ca2-VDM w/o PE"]
    assert with_pe == 924_844_032
    # one cache per denoising step (no sharing) would be 50x larger: far above 0.86
    assert round(50 * with_pe / gib, 2) > rows["Live2diff (T=50)"]
    # the Pmax = 41 queue does not fit the printed figure (the table's Pmax is 25)
    assert round(oracle.cache_bytes(28, 1, 256, 16, 72, 41, 3) / gib, 2) != rows["Ca2-VDM w/ PE"]


def test_prefix_schedule_from_pages():
    """First frame, then chunks of l: the queue lengths seen before each AR step are the
    prefix lengths {1, 1+l, ..., Pmax} the pages train with, then stay at Pmax."""
    for l, pmax, seq in _read_table("prefix_schedule.txt"):
        l, pmax = int(l), int(pmax)
        expect = [int(x) for x in seq.split(",")]
        ring = oracle.RingModel(pmax, 3)
        z = np.zeros((1, 1, 1, 1, 1), np.uint16)
        ring.write(z, z, z, z)
        seen = []
        for _ in range(len(expect) + 3):
            seen.append(ring.count)
            zc = np.zeros((1, l, 1, 1, 1), np.uint16)
            ring.write(zc, zc, zc, zc)
        assert seen[: len(expect)] == expect
        assert seen[len(expect):] == [pmax] * 3


def test_ring_fifo_against_explicit_ring():
    """The queue's age order and the slot closed form g mod Pmax against a ring simulated
    with an explicit head pointer and count."""
    rng = np.random.default_rng(0)
    for pmax in (1, 5, 9, 41):
        ring = oracle.RingModel(pmax, 1)
        head, count, slots = 0, 0, [None] * pmax
        g_next = 0
        for _ in range(60):
            n = int(rng.integers(1, pmax + 1))
            e = max(0, count + n - pmax)
            head, count = (head + e) % pmax, count - e
            for j in range(n):
                slots[(head + count + j) % pmax] = g_next + j
            count += n
            z = np.zeros((1, n, 1, 1, 1), np.uint16)
            ring.write(z, z, z, z)
            g_next += n
            assert ring.count == count and ring.head == head
            assert list(ring.queue) == [slots[(head + i) % pmax] for i in range(count)]
            assert all(ring.slot_of(g) == (head + i) % pmax for i, g in enumerate(ring.queue))
        assert ring.evicted == list(range(len(ring.evicted)))   # oldest first


def test_spatial_cache_keeps_last_pspatial():
    ring = oracle.RingModel(9, 3)
    k = np.arange(8, dtype=np.uint16).reshape(1, 8, 1, 1, 1)
    ring.write(k[:, :1], k[:, :1], k[:, :1], k[:, :1])
    assert ring.spatial_ids == [0]
    ring.write(k, k, k, k)
    assert ring.spatial_ids == [6, 7, 8]
    assert [int(x.ravel()[0]) for x in ring.spatial()[0]] == [5, 6, 7]


def test_tpe_cyclic():
    n_tpe = 49
    # inside the table: consecutive indices; past its end they start again from 0
    assert oracle.tpe_indices(41, 0, 8, n_tpe) == list(range(41, 49))
    assert oracle.tpe_indices(49, 0, 8, n_tpe) == list(range(0, 8))
    assert oracle.tpe_indices(45, 0, 8, n_tpe) == [45, 46, 47, 48, 0, 1, 2, 3]
    # with offset 0, N_tpe = Pmax + l = 49 and chunks starting at 1 + 8k, restarting per
    # frame and restarting per chunk give the same indices
    for kk in range(12):
        g0 = 1 + 8 * kk
        per_frame = oracle.tpe_indices(g0, 0, 8, n_tpe)
        start = g0 % n_tpe
        per_chunk = [start + c if start + 8 <= n_tpe else c for c in range(8)]
        assert per_frame == per_chunk
    # a random cyclic shift rotates the whole index sequence
    base = oracle.tpe_indices(0, 0, 200, n_tpe)
    for off in (1, 17, 48):
        assert oracle.tpe_indices(0, off, 200, n_tpe) == [(x + off) % n_tpe for x in base]
    with pytest.raises(ValueError):
        oracle.tpe_indices(0, 0, 1, 0)


# --- planted mistakes: each must make at least one pin fail ---------------------------
MUTANTS = [
    ("mask includes the diagonal", "const double mask = (i < j)", "const double mask = (i <= j)", 0),
    ("mask transposed", "const double mask = (i < j)", "const double mask = (i > j)", 0),
    ("temporal scale 1/D", "const double inv_sqrt_d = 1.0 / sqrt((double)D);",
     "const double inv_sqrt_d = 1.0 / (double)D;", 0),
    ("spatial scale dropped", "const double inv_sqrt_d = 1.0 / sqrt((double)D);",
     "const double inv_sqrt_d = 1.0;", 1),
    ("cached keys used as values", "? pv[j] + fo", "? pk[j] + fo", 0),
    ("prefix order reversed for keys", "? pk[j] + fo", "? pk[P - 1 - j] + fo", 0),
    ("softmax denominator dropped", "const double w = logit[j] / den;", "const double w = logit[j];", 0),
    ("spatial normaliser dropped", "const double w = logit[j] / den;", "const double w = logit[j];", 1),
    ("only the first cached spatial frame", "krow[j] = sk[blk - 1] + off;", "krow[j] = sk[0] + off;", 0),
    ("token and head swapped", "return (((long long)b * HW + s) * H + h) * (long long)D;",
     "return (((long long)b * HW + h) * H + s) * (long long)D;", 0),
    ("no max subtraction guard", "logit[j] = exp(logit[j] - m);", "logit[j] = exp(logit[j] - m) + 1e-9;", 0),
]


def _apply(src, old, new, occurrence):
    parts = src.split(old)
    assert len(parts) > occurrence + 1, "mutation target not found: %r" % old
    return old.join(parts[: occurrence + 1]) + new + old.join(parts[occurrence + 1:])


@pytest.mark.parametrize("name,old,new,occ", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmp_path, name, old, new, occ):
    with open(oracle._SRC) as f:
        src = f.read()
    mutated = _apply(src, old, new, occ)
    assert mutated != src
    c = tmp_path / "mutant.c"
    c.write_text(mutated)
    so = str(tmp_path / "libmutant.so")
    subprocess.check_call(["gcc", *oracle.CFLAGS, str(c), "-o", so, "-lm"])
    lib = oracle.load(so)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(lib)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, "planted mistake %r passed every pin" % name


def _bits(vals):
    return np.asarray(vals, dtype=np.float32).view(np.uint32).__rshift__(16).astype(np.uint16)


def test_tpe_add_zero_table_is_identity():
    rng = np.random.default_rng(4)
    x = rng.integers(0, 0x7F00, size=(2, 5, 3, 16), dtype=np.uint16)
    table = np.zeros((7, 16), dtype=np.uint16)
    assert np.array_equal(oracle.tpe_add(x, table, 5, 2), x)


def test_tpe_add_on_zero_input_gathers_cyclic_rows():
    """x = 0: the result is the table rows at (offset + g0 + f) mod N_tpe, wrap included."""
    n_tpe, C = 7, 16
    table = _bits(np.arange(n_tpe * C, dtype=np.float32).reshape(n_tpe, C) + 1.0)   # exact in bf16
    x = np.zeros((1, 3, 4, C), dtype=np.uint16)
    out = oracle.tpe_add(x, table, 5, 3)          # frames 5..8, offset 3 -> rows 1, 2, 3, 4
    for f, row in enumerate([1, 2, 3, 4]):
        assert np.array_equal(out[0, :, f], np.broadcast_to(table[row], (3, C)))
    out = oracle.tpe_add(x, table, 12, 0)         # rows 5, 6, 0, 1
    assert [int(np.argmax(np.all(out[0, 0, f] == table, axis=1))) for f in range(4)] == [5, 6, 0, 1]


def test_tpe_add_rounds_ties_to_even():
    """1 + 2^-8 lies halfway between 1 and 1 + 2^-7 in bf16: ties go to the even mantissa."""
    table = _bits([[2.0 ** -8, 2.0 ** -8, 3.0 * 2.0 ** -9]])
    x = _bits([1.0, 1.0078125, 1.0]).reshape(1, 1, 1, 3)
    out = oracle.tpe_add(x, table, 0, 0)
    assert out.reshape(-1).tolist() == [0x3F80, 0x3F82, 0x3F81]   # 1.0, 1.015625, 1.0078125


def _bf16_bits(vals):
    """Small exactly representable values -> bf16 bits."""
    f = np.asarray(vals, dtype=np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def _projection_matches_loops(proj) -> bool:
    """Y[r][o] = sum_i x[r][i] w[o][i] + b[o] written out as loops on a tiny case (integer
    values: exact in any order); K is output channels 0..C-1, V channels C..2C-1."""
    rng = np.random.default_rng(5)
    rows, C = 3, 4
    x = rng.integers(-4, 5, size=(rows, C))
    w = rng.integers(-3, 4, size=(2 * C, C))
    b = rng.integers(-8, 9, size=(2 * C,))
    try:
        k, v = proj(_bf16_bits(x), _bf16_bits(w), _bf16_bits(b))
    except Exception:
        return False
    for r in range(rows):
        for o in range(2 * C):
            acc = float(b[o])
            for i in range(C):
                acc += float(x[r][i]) * float(w[o][i])
            got = k[r][o] if o < C else v[r][o - C]
            if got != acc:
                return False
    return True


def test_kv_projection_matches_brute_force_loops():
    """The oracle's projection against the written-out loops."""
    assert _projection_matches_loops(oracle.kv_projection)


def test_kv_projection_planted_mistakes_are_caught():
    """Plausible mistakes in a projection -- K and V halves swapped, the bias dropped, the
    weight read transposed, an input channel off by one -- each fail the loop pin."""
    f64 = lambda a: (np.asarray(a).astype(np.uint32) << 16).view(np.float32).astype(np.float64)

    def swapped(x, w, b):
        k, v = oracle.kv_projection(x, w, b)
        return v, k

    def no_bias(x, w, b):
        return oracle.kv_projection(x, w, None)

    def transposed(x, w, b):
        y = f64(x) @ f64(w)[: f64(x).shape[1]]        # w's first C rows as a C x C matrix
        y = np.concatenate([y, y], axis=1) + f64(b)[None, :]
        C = f64(x).shape[1]
        return y[:, :C], y[:, C:]

    def shifted(x, w, b):
        xs = np.roll(f64(x), 1, axis=1)
        y = xs @ f64(w).T + f64(b)[None, :]
        C = xs.shape[1]
        return y[:, :C], y[:, C:]

    for bad in (swapped, no_bias, transposed, shifted):
        assert not _projection_matches_loops(bad), bad.__name__


def test_kv_projection_identity_and_bias_only():
    """W = [I; 2I] with no bias returns K = x and V = 2x exactly; W = 0 returns the bias."""
    rng = np.random.default_rng(6)
    C = 8
    x = _bf16_bits(rng.integers(-64, 65, size=(5, C)) / 16.0)
    eye = np.eye(C, dtype=np.float32)
    k, v = oracle.kv_projection(x, _bf16_bits(np.concatenate([eye, 2 * eye])))
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(k, xf) and np.array_equal(v, 2 * xf)
    b = rng.integers(-8, 9, size=(2 * C,)).astype(np.float32)
    k, v = oracle.kv_projection(x, _bf16_bits(np.zeros((2 * C, C))), _bf16_bits(b))
    assert np.array_equal(k, np.broadcast_to(b[:C], (5, C))) and np.array_equal(v, np.broadcast_to(b[C:], (5, C)))


def test_kv_projection_bound_is_the_magnitude_sum():
    """The bound is sum_i |x_i w_oi| + |b_o|: on sign-mixed integers it exceeds |Y| and
    equals it when every term is positive."""
    x = _bf16_bits([[1, -2, 3]])
    w = _bf16_bits([[1, 1, 1], [2, 0, -1], [-1, -1, -1], [0, 1, 0], [1, 2, 3], [3, 2, 1]])
    b = _bf16_bits([1, -1, 0, 2, 0, 0])
    bound = oracle.kv_projection_bound(x, w, b)
    assert bound.tolist() == [[7.0, 6.0, 6.0, 4.0, 14.0, 10.0]]
    k, v = oracle.kv_projection(x, w, b)
    assert np.all(np.abs(np.concatenate([k, v], axis=1)) <= bound)
