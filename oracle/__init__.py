"""CPU oracle for the Ca2-VDM cached attention path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import this package.  It shares no code with the CUDA library in
``causal_kv_cache_b200/`` and never imports it.

What it holds (all plain definitions, fp64 for floating point, integers exact):

* ``temporal_attn``  -- causal temporal attention over [cached prefix frames || chunk],
  CausalAttn = Softmax(QK^T/sqrt(C') + M)V with M_ij = -inf for i < j
  ("Ca2-VDM" papernotes page, 关键设计 1; bohrium arXiv 2411.16375 page, formula
  section).  Runs in ``ca2_oracle.c``.
* ``spatial_attn``   -- prefix-enhanced spatial attention, own frame || last P' prefix
  frames, or the own frame self-repeated P'+1 times for clean prefix frames
  (papernotes page, 关键设计 3).  Runs in ``ca2_oracle.c``.
* ``RingModel``      -- the temporal KV-cache queue: frames kept by global frame id, FIFO,
  at most Pmax, oldest dequeued first; plus the one-chunk spatial cache overwritten at
  every write (papernotes page, 关键设计 4 and 5).
* ``tpe_indices``    -- cyclic temporal-position indices (papernotes page, 关键设计 4,
  "Cyclic-TPEs"): index of global frame g is (offset + g) mod N_tpe.
* ``tpe_add``        -- the chunk input plus each frame's TPE row at its cyclic index,
  added to every token's channel vector (the reading taken: the embedding is added to the
  temporal branch's input, as the pages' Open-Sora backbone does).  Sum in float32, one
  rounding to bf16 (nearest, ties to even), the precision the kernel computes in.
* ``cache_bytes``    -- bytes of the shared KV cache (K and V, 2-byte elements,
  Pmax temporal frames plus P' spatial frames per layer).
* ``kv_projection``  -- the K and V a layer stores in the cache-writing stage: the clean
  chunk's hidden states times the layer's K and V projection weights, plus a bias
  (papernotes page, 整体框架: one forward pass over the denoised chunk computes the new KV
  cache; 关键设计 1: attention over Q, K, V).  The weight is one [2C][C] matrix, K rows
  first (the nn.Linear layout).  Exact in fp64; ``kv_projection_bound`` gives the
  magnitude sum an fp32 accumulation error is measured against.

Parity status: every function is pinned by tests in ``tests/test_oracle_pins.py``
(brute-force full-sequence attention, library SDPA special cases, closed forms, the
pages' memory table and prefix-length schedule, and planted-mutation checks).
"""
from __future__ import annotations

import collections
import ctypes
import os
import subprocess
import threading
from typing import Dict, List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ca2_oracle.c")
_LIB = os.path.join(_HERE, "libca2_oracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off"]


def build(src: str = _SRC, out: str = _LIB, force: bool = False) -> str:
    """Compile the C oracle with gcc (plain -O2, no fast-math)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, src, "-o", tmp, "-lm"])
        os.replace(tmp, out)
    return out


def load(path: Optional[str] = None):
    """Load (building first if needed) the oracle library; returns the ctypes handle."""
    global _lib
    with _lock:
        if path is not None:
            return _bind(ctypes.CDLL(path))
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
        return _lib


def _bind(lib):
    P = ctypes.c_void_p
    i = ctypes.c_int
    ll = ctypes.c_longlong
    lib.oracle_temporal_attn.argtypes = [i, i, i, i, i, i, P, P, P, P, P, P, ll, P]
    lib.oracle_temporal_attn.restype = None
    lib.oracle_spatial_attn.argtypes = [i, i, i, i, i, P, P, P, P, P, i, i, P, ll, P]
    lib.oracle_spatial_attn.restype = None
    lib.oracle_num_threads.restype = i
    lib.oracle_set_num_threads.argtypes = [i]
    return lib


def num_threads() -> int:
    return load().oracle_num_threads()


def set_num_threads(n: int) -> None:
    load().oracle_set_num_threads(int(n))


def _u16(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are raw bf16 bits (uint16), got %s" % a.dtype)
    return a


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _ptr_array(frames: Sequence[np.ndarray]):
    arr = (ctypes.c_void_p * max(1, len(frames)))()
    for j, f in enumerate(frames):
        arr[j] = _ptr(f)
    return arr


def temporal_attn(q, k, v, prefix_k: Sequence[np.ndarray], prefix_v: Sequence[np.ndarray],
                  units: Optional[np.ndarray] = None, lib=None) -> np.ndarray:
    """Causal temporal attention of a chunk over [prefix frames || chunk].

    q, k, v: uint16 [B][n][HW][H][D]; prefix_k/v: lists of [B][HW][H][D] frames, oldest first.
    Returns fp64 [B][n][HW][H][D] (units=None) or [len(units)][n][D] for the units
    u = (b*HW + s)*H + h listed.
    """
    lib = lib or load()
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, n, HW, H, D = q.shape
    pk = [_u16(f) for f in prefix_k]
    pv = [_u16(f) for f in prefix_v]
    assert len(pk) == len(pv)
    for f in pk + pv:
        assert f.shape == (B, HW, H, D), f.shape
    P = len(pk)
    if units is None:
        out = np.empty((B * HW * H, n, D), dtype=np.float64)
        lib.oracle_temporal_attn(B, HW, H, D, n, P, _ptr(q), _ptr(k), _ptr(v),
                                 _ptr_array(pk), _ptr_array(pv), None, 0, _ptr(out))
        return out.reshape(B, HW, H, n, D).transpose(0, 3, 1, 2, 4).copy()
    u = np.ascontiguousarray(units, dtype=np.int64)
    out = np.empty((len(u), n, D), dtype=np.float64)
    lib.oracle_temporal_attn(B, HW, H, D, n, P, _ptr(q), _ptr(k), _ptr(v),
                             _ptr_array(pk), _ptr_array(pv), _ptr(u), len(u), _ptr(out))
    return out


def spatial_attn(q, k, v, cache_k: Sequence[np.ndarray], cache_v: Sequence[np.ndarray],
                 repeat: int = 0, units: Optional[np.ndarray] = None, lib=None) -> np.ndarray:
    """Prefix-enhanced spatial attention, per frame.

    repeat=0: keys = own frame || every frame in cache_k (denoising mode).
    repeat=R>0: keys = own frame written out R times (self-repeat mode; cache unused).
    Returns fp64 [B][n][HW][H][D] (units=None) or [len(units)][HW][D] for the units
    u = (b*n + f)*H + h listed.
    """
    lib = lib or load()
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, n, HW, H, D = q.shape
    sk = [_u16(f) for f in cache_k] if repeat == 0 else []
    sv = [_u16(f) for f in cache_v] if repeat == 0 else []
    for f in sk + sv:
        assert f.shape == (B, HW, H, D), f.shape
    if units is None:
        out = np.empty((B * n * H, HW, D), dtype=np.float64)
        lib.oracle_spatial_attn(B, HW, H, D, n, _ptr(q), _ptr(k), _ptr(v), _ptr_array(sk),
                                _ptr_array(sv), len(sk), int(repeat), None, 0, _ptr(out))
        return out.reshape(B, n, H, HW, D).transpose(0, 1, 3, 2, 4).copy()
    u = np.ascontiguousarray(units, dtype=np.int64)
    out = np.empty((len(u), HW, D), dtype=np.float64)
    lib.oracle_spatial_attn(B, HW, H, D, n, _ptr(q), _ptr(k), _ptr(v), _ptr_array(sk),
                            _ptr_array(sv), len(sk), int(repeat), _ptr(u), len(u), _ptr(out))
    return out


def tpe_indices(first_global_frame: int, offset: int, n: int, n_tpe: int) -> List[int]:
    """Cyclic TPE index of each of n frames starting at a global frame index.

    Global frame g gets (offset + g) mod N_tpe: once the table runs out the indices start
    again from the beginning, and a random cyclic shift is the offset (papernotes page,
    关键设计 4 "Cyclic-TPEs" and the training strategy's random cyclic TPE shift).
    """
    if n_tpe <= 0:
        raise ValueError("n_tpe must be positive")
    return [(offset + first_global_frame + c) % n_tpe for c in range(n)]


def bf16_round_bits(x: np.ndarray) -> np.ndarray:
    """float32 values -> bfloat16 bits, rounded to nearest with ties to even (IEEE)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    r[nan] = ((u[nan] >> 16) | 0x40).astype(np.uint16)    # keep NaN a (quiet) NaN
    return r


def tpe_add(x: np.ndarray, table: np.ndarray, first_global_frame: int, offset: int) -> np.ndarray:
    """x + TPE for one chunk, token-major: x [B][HW][n][C] bf16 bits, table [N_tpe][C] bf16 bits.

    Frame f of the chunk (global frame first_global_frame + f) gets row
    tpe_indices(first_global_frame, offset, n, N_tpe)[f] of the table added to every token's
    C-vector ("Ca2-VDM" papernotes page, 关键设计 4 "Cyclic-TPEs").  Each element is the
    float32 sum of the two bf16 values rounded once to bf16 (ties to even).
    """
    x = _u16(x)
    table = _u16(table)
    n, C = x.shape[2], x.shape[3]
    if table.ndim != 2 or table.shape[1] != C:
        raise ValueError("table must be [N_tpe][C] with the chunk's C")
    idx = tpe_indices(first_global_frame, offset, n, table.shape[0])
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    tf = (table.astype(np.uint32) << 16).view(np.float32)[idx]          # [n][C]
    return bf16_round_bits(xf + tf[None, None, :, :])


def kv_projection(x: np.ndarray, w: np.ndarray, b: Optional[np.ndarray] = None):
    """K and V of one layer from its input rows: x [rows][C], w [2C][C], b [2C] or None,
    all bf16 bits.  Returns (K, V), each [rows][C] float64: Y = x w^T + b, K = Y[:, :C],
    V = Y[:, C:] (papernotes page, 整体框架 and 关键设计 1).  Every product of two bf16
    values is exact in fp64 and the sum carries fp64 rounding only (2^-53 relative per
    term), far below the fp32 accumulation error the kernel is compared with.
    """
    xf = _bits_to_f64(x)
    wf = _bits_to_f64(w)
    C = xf.shape[1]
    if wf.shape != (2 * C, C):
        raise ValueError("w must be [2C][C] with the rows' C")
    y = xf @ wf.T
    if b is not None:
        bf = _bits_to_f64(b)
        if bf.shape != (2 * C,):
            raise ValueError("b must be [2C]")
        y = y + bf[None, :]
    return y[:, :C], y[:, C:]


def kv_projection_bound(x: np.ndarray, w: np.ndarray, b: Optional[np.ndarray] = None) -> np.ndarray:
    """sum_i |x_i w_oi| + |b_o| for every output element, [rows][2C] float64: the scale of
    the rounding error of any summation order of the projection."""
    y = np.abs(_bits_to_f64(x)) @ np.abs(_bits_to_f64(w)).T
    if b is not None:
        y = y + np.abs(_bits_to_f64(b))[None, :]
    return y


def _bits_to_f64(a: np.ndarray) -> np.ndarray:
    a = _u16(a)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def cache_bytes(n_layers: int, batch: int, hw: int, heads: int, head_dim: int,
                p_max: int, p_spatial: int, elem_bytes: int = 2) -> int:
    """Bytes of the shared KV cache: K and V of Pmax temporal + P' spatial frames per layer.

    One cache serves every denoising step (papernotes page, 关键设计 2), so T does not
    appear.  The temporal queue holds at most Pmax frames (关键设计 4); the spatial cache
    holds the P' prefix frames that spatial attention reads (关键设计 3, 5).
    """
    per_frame = batch * hw * heads * head_dim * elem_bytes
    return 2 * n_layers * per_frame * (p_max + p_spatial)


class RingModel:
    """The temporal KV-cache queue and the spatial KV cache, kept by global frame id.

    Frames are appended in generation order with consecutive global ids 0, 1, 2, ...
    The queue is FIFO with capacity Pmax: once it would hold more, the oldest frames are
    dequeued (papernotes page, 关键设计 4).  The spatial cache keeps the last
    min(P', n) frames of the newest write and is replaced by every write (关键设计 5).

    ``slot_of(g)`` states where a ring buffer that starts at slot 0 and advances one slot
    per frame keeps frame g: slot g mod Pmax.  It is the layout contract the GPU ring is
    checked against; it is not used by the attention functions above.
    """

    def __init__(self, p_max: int, p_spatial: int):
        if p_max <= 0 or p_spatial < 0:
            raise ValueError("bad capacity")
        self.p_max = p_max
        self.p_spatial = p_spatial
        self.queue: collections.deque = collections.deque()
        self.k: Dict[int, np.ndarray] = {}
        self.v: Dict[int, np.ndarray] = {}
        self.spatial_ids: List[int] = []
        self.sk: Dict[int, np.ndarray] = {}
        self.sv: Dict[int, np.ndarray] = {}
        self.frames_written = 0
        self.evicted: List[int] = []

    # -- state ---------------------------------------------------------------------
    @property
    def count(self) -> int:
        return len(self.queue)

    @property
    def head(self) -> int:
        """Ring slot of the oldest queued frame (0 while the queue is empty and unused)."""
        return (self.queue[0] if self.queue else self.frames_written) % self.p_max

    def slot_of(self, g: int) -> int:
        return g % self.p_max

    def prefix(self):
        """Queued (K, V) frame-planes, oldest first."""
        return [self.k[g] for g in self.queue], [self.v[g] for g in self.queue]

    def spatial(self):
        return [self.sk[g] for g in self.spatial_ids], [self.sv[g] for g in self.spatial_ids]

    # -- updates -------------------------------------------------------------------
    def write(self, k_t, v_t, k_s, v_s, layer_axis: bool = False) -> List[int]:
        """Append the n frames of a chunk ([B][n][HW][H][D]); returns the evicted ids."""
        n = k_t.shape[1]
        gone = []
        for c in range(n):
            g = self.frames_written + c
            self.queue.append(g)
            self.k[g] = np.ascontiguousarray(k_t[:, c])
            self.v[g] = np.ascontiguousarray(v_t[:, c])
        while len(self.queue) > self.p_max:
            g = self.queue.popleft()
            gone.append(g)
            del self.k[g], self.v[g]
        keep = min(self.p_spatial, n)
        self.sk, self.sv = {}, {}
        self.spatial_ids = [self.frames_written + c for c in range(n - keep, n)]
        for c in range(n - keep, n):
            g = self.frames_written + c
            self.sk[g] = np.ascontiguousarray(k_s[:, c])
            self.sv[g] = np.ascontiguousarray(v_s[:, c])
        self.frames_written += n
        self.evicted.extend(gone)
        return gone
