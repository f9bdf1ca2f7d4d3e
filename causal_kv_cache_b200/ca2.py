"""ctypes binding of libca2.so -- argument marshalling only.

Every function keeps the name of its C entry point in ``include/ca2.h`` and forwards to
it; device pointers may be passed as integers or as objects with ``data_ptr()`` (torch
tensors), streams as integers, ``torch.cuda.Stream`` objects or None (torch's current
stream when torch has a CUDA device, else the legacy default stream).  A non-zero
status raises ``Ca2Error``.

``KVCache`` is a convenience owner: it allocates the two cache buffers with torch on the
current device (PyTorch is used for device memory and streams only) and wraps a handle.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence, Tuple

__all__ = [
    "Ca2Error", "ca2_config", "load_library", "LIBRARY_PATH",
    "ca2_cache_bytes", "ca2_cache_init", "ca2_cache_destroy", "ca2_cache_evict", "ca2_cache_evict_for",
    "ca2_cache_config", "ca2_cache_layer_offsets",
    "ca2_cache_write", "ca2_kv_proj_write", "ca2_cache_commit", "ca2_temporal_attn", "ca2_spatial_prefix_attn",
    "ca2_tpe_indices", "ca2_tpe_add",
    "ca2_cache_state", "ca2_device_status", "ca2_selftest_timeout", "ca2_status_string", "ca2_head_shard",
    "ca2_debug_build",
    "ca2_last_error_string",
    "KVCache", "STATUS",
]

LIBRARY_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libca2.so")

STATUS = {
    0: "CA2_OK", -1: "CA2_ERR_ARG", -2: "CA2_ERR_SHAPE", -3: "CA2_ERR_CAPACITY",
    -4: "CA2_ERR_ALIGN", -5: "CA2_ERR_CUDA", -6: "CA2_ERR_TIMEOUT", -7: "CA2_ERR_RANGE",
    -8: "CA2_ERR_BOUNDS",
}


class Ca2Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = _string(status)
        if status == -5:
            try:
                detail += ": " + load_library().ca2_last_error_string().decode()
            except Exception:  # pragma: no cover
                pass
        super().__init__("%s failed: %s (%s)" % (where, STATUS.get(status, status), detail))


class ca2_config(ctypes.Structure):
    _fields_ = [
        ("n_layers", ctypes.c_int), ("batch", ctypes.c_int), ("hw", ctypes.c_int),
        ("heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("chunk_len", ctypes.c_int),
        ("p_max", ctypes.c_int), ("p_spatial", ctypes.c_int), ("tpe_len", ctypes.c_int),
        ("row_pitch", ctypes.c_int),
    ]


_lib = None


def load_library(path: Optional[str] = None):
    """Load libca2.so (no fallback: a missing library is an error).

    The environment variable CA2_LIBRARY, when set, names another build of the library
    to load instead of the in-tree one."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or os.environ.get("CA2_LIBRARY") or LIBRARY_PATH
    if not os.path.exists(p):
        raise RuntimeError("libca2.so is not built (%s); run `python -m causal_kv_cache_b200.build`" % p)
    lib = ctypes.CDLL(p)
    vp, i, ll, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t
    cfgp = ctypes.POINTER(ca2_config)
    pp = ctypes.POINTER(ctypes.c_void_p)
    sig = {
        "ca2_cache_bytes": ([cfgp, ctypes.POINTER(sz), ctypes.POINTER(sz)], i),
        "ca2_cache_init": ([cfgp, vp, sz, vp, sz, ctypes.POINTER(vp)], i),
        "ca2_cache_destroy": ([vp], i),
        "ca2_cache_evict": ([vp, i], i),
        "ca2_cache_evict_for": ([vp, i, ctypes.POINTER(i)], i),
        "ca2_cache_config": ([vp, cfgp], i),
        "ca2_cache_layer_offsets": ([vp, i, i, ctypes.POINTER(sz), ctypes.POINTER(sz)], i),
        "ca2_cache_write": ([vp, pp, pp, pp, pp, i, vp], i),
        "ca2_kv_proj_write": ([vp, i, vp, vp, vp, vp, vp, vp, i, vp], i),
        "ca2_cache_commit": ([vp, i], i),
        "ca2_temporal_attn": ([vp, i, vp, vp, vp, vp, i, vp], i),
        "ca2_spatial_prefix_attn": ([vp, i, vp, vp, vp, vp, i, i, vp], i),
        "ca2_tpe_indices": ([vp, ll, i, i, ctypes.POINTER(ctypes.c_int)], i),
        "ca2_tpe_add": ([vp, ll, i, vp, vp, vp, i, vp], i),
        "ca2_cache_state": ([vp, ctypes.POINTER(i), ctypes.POINTER(i), ctypes.POINTER(i), ctypes.POINTER(ll)], i),
        "ca2_device_status": ([], i),
        "ca2_selftest_timeout": ([i, vp], i),
        "ca2_head_shard": ([i, i, i, ctypes.POINTER(i), ctypes.POINTER(i)], i),
        "ca2_debug_build": ([], i),
        "ca2_status_string": ([i], ctypes.c_char_p),
        "ca2_last_error_string": ([], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    if path is None:
        _lib = lib
    return lib


def _string(status: int) -> str:
    try:
        return load_library().ca2_status_string(int(status)).decode()
    except Exception:  # pragma: no cover - the library itself is missing
        return "?"


def _check(status: int, where: str) -> None:
    if status != 0:
        raise Ca2Error(status, where)


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return int(x.data_ptr())
    raise TypeError("expected a device pointer (int) or a tensor, got %r" % type(x))


def _stream(s) -> Optional[int]:
    if s is None:
        try:
            import torch
            if torch.cuda.is_available():
                return int(torch.cuda.current_stream().cuda_stream)
        except ImportError:  # pragma: no cover
            pass
        return None
    if isinstance(s, int):
        return s
    if hasattr(s, "cuda_stream"):
        return int(s.cuda_stream)
    raise TypeError("bad stream %r" % (s,))


def _ptr_array(xs: Optional[Sequence]):
    if xs is None:
        return None
    arr = (ctypes.c_void_p * max(1, len(xs)))()
    for j, x in enumerate(xs):
        arr[j] = _ptr(x)
    return arr


def _cfg(cfg) -> ca2_config:
    if isinstance(cfg, ca2_config):
        return cfg
    return ca2_config(**cfg) if isinstance(cfg, dict) else ca2_config(*cfg)


# ---- the C entry points ---------------------------------------------------------------
def ca2_cache_bytes(cfg) -> Tuple[int, int]:
    t, s = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(load_library().ca2_cache_bytes(ctypes.byref(_cfg(cfg)), ctypes.byref(t), ctypes.byref(s)),
           "ca2_cache_bytes")
    return t.value, s.value


def ca2_cache_init(cfg, temporal_buf, temporal_bytes: int, spatial_buf, spatial_bytes: int) -> int:
    h = ctypes.c_void_p(None)
    _check(load_library().ca2_cache_init(ctypes.byref(_cfg(cfg)), _ptr(temporal_buf), int(temporal_bytes),
                                         _ptr(spatial_buf), int(spatial_bytes), ctypes.byref(h)),
           "ca2_cache_init")
    return h.value


def ca2_cache_destroy(handle) -> None:
    _check(load_library().ca2_cache_destroy(handle), "ca2_cache_destroy")


def ca2_cache_evict(handle, n_frames: int) -> None:
    _check(load_library().ca2_cache_evict(handle, int(n_frames)), "ca2_cache_evict")


def ca2_cache_evict_for(handle, n_new: int) -> int:
    e = ctypes.c_int(0)
    _check(load_library().ca2_cache_evict_for(handle, int(n_new), ctypes.byref(e)), "ca2_cache_evict_for")
    return e.value


def ca2_cache_config(handle) -> ca2_config:
    c = ca2_config()
    _check(load_library().ca2_cache_config(handle, ctypes.byref(c)), "ca2_cache_config")
    return c


def ca2_cache_layer_offsets(handle, layer: int, kv: int) -> Tuple[int, int]:
    t, s_ = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(load_library().ca2_cache_layer_offsets(handle, int(layer), int(kv), ctypes.byref(t), ctypes.byref(s_)),
           "ca2_cache_layer_offsets")
    return t.value, s_.value


def ca2_cache_write(handle, k_t, v_t, k_s, v_s, n_frames: int, stream=None) -> None:
    _check(load_library().ca2_cache_write(handle, _ptr_array(k_t), _ptr_array(v_t), _ptr_array(k_s),
                                          _ptr_array(v_s), int(n_frames), _stream(stream)),
           "ca2_cache_write")


def ca2_kv_proj_write(handle, layer: int, x_t, w_t, b_t, x_s, w_s, b_s, n_frames: int, stream=None) -> None:
    _check(load_library().ca2_kv_proj_write(handle, int(layer), _ptr(x_t), _ptr(w_t), _ptr(b_t), _ptr(x_s),
                                            _ptr(w_s), _ptr(b_s), int(n_frames), _stream(stream)),
           "ca2_kv_proj_write")


def ca2_cache_commit(handle, n_frames: int) -> None:
    _check(load_library().ca2_cache_commit(handle, int(n_frames)), "ca2_cache_commit")


def ca2_temporal_attn(handle, layer: int, q, k, v, out, n_frames: int, stream=None) -> None:
    _check(load_library().ca2_temporal_attn(handle, int(layer), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                            int(n_frames), _stream(stream)),
           "ca2_temporal_attn")


def ca2_spatial_prefix_attn(handle, layer: int, q, k, v, out, n_frames: int, use_prefix: int,
                            stream=None) -> None:
    _check(load_library().ca2_spatial_prefix_attn(handle, int(layer), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                                  int(n_frames), int(use_prefix), _stream(stream)),
           "ca2_spatial_prefix_attn")


def ca2_tpe_add(handle, first_global_frame: int, offset: int, table, x, out, n_frames: int, stream=None) -> None:
    _check(load_library().ca2_tpe_add(handle, int(first_global_frame), int(offset), _ptr(table), _ptr(x), _ptr(out),
                                      int(n_frames), _stream(stream)),
           "ca2_tpe_add")


def ca2_tpe_indices(handle, first_global_frame: int, offset: int, n: int) -> List[int]:
    buf = (ctypes.c_int * max(1, n))()
    _check(load_library().ca2_tpe_indices(handle, int(first_global_frame), int(offset), int(n),
                                          buf if n > 0 else None),
           "ca2_tpe_indices")
    return list(buf[:n])


def ca2_cache_state(handle) -> Tuple[int, int, int, int]:
    h, c, s = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    fw = ctypes.c_longlong(0)
    _check(load_library().ca2_cache_state(handle, ctypes.byref(h), ctypes.byref(c), ctypes.byref(s),
                                          ctypes.byref(fw)),
           "ca2_cache_state")
    return h.value, c.value, s.value, fw.value


def ca2_device_status() -> int:
    """Returns the status code (0, CA2_ERR_TIMEOUT, CA2_ERR_RANGE or CA2_ERR_CUDA) without raising."""
    return int(load_library().ca2_device_status())


def ca2_selftest_timeout(wait_us: int, stream=None) -> None:
    _check(load_library().ca2_selftest_timeout(int(wait_us), _stream(stream)), "ca2_selftest_timeout")


def ca2_head_shard(heads: int, world: int, rank: int) -> Tuple[int, int]:
    """(first head, number of heads) that `rank` of `world` owns."""
    h0, hc = ctypes.c_int(0), ctypes.c_int(0)
    _check(load_library().ca2_head_shard(int(heads), int(world), int(rank), ctypes.byref(h0), ctypes.byref(hc)),
           "ca2_head_shard")
    return h0.value, hc.value


def ca2_debug_build() -> bool:
    """True when the loaded library is the bounds-checked debug build."""
    return bool(load_library().ca2_debug_build())


def ca2_status_string(status: int) -> str:
    return load_library().ca2_status_string(int(status)).decode()


def ca2_last_error_string() -> str:
    return load_library().ca2_last_error_string().decode()


def _numel(shape) -> int:
    n = 1
    for d in shape:
        n *= int(d)
    return n


# ---- convenience owner ------------------------------------------------------------------
class KVCache:
    """Cache buffers allocated with torch on the current CUDA device, plus the handle.

    ``ring(layer, kv)`` ([B][HW][H][Pmax][D]) and ``spatial(layer, kv)`` ([P'][B][HW][H][D])
    are bf16 views of the buffers with the layout documented in include/ca2.h, at the
    offsets the library reports.  ``row_pitch`` (elements, 0 = H*D) is the distance between
    consecutive rows of the caller's chunk tensors.
    """

    def __init__(self, n_layers, batch, hw, heads, head_dim, chunk_len, p_max, p_spatial,
                 tpe_len=0, device=None, row_pitch=0):
        import torch
        cfg = ca2_config(n_layers, batch, hw, heads, head_dim, chunk_len, p_max, p_spatial, tpe_len, row_pitch)
        tb, sb = ca2_cache_bytes(cfg)
        dev = device or torch.device("cuda", torch.cuda.current_device())
        self.tbuf = torch.empty(tb // 2, dtype=torch.bfloat16, device=dev)
        self.sbuf = torch.empty(max(sb // 2, 8), dtype=torch.bfloat16, device=dev)
        self.handle = ca2_cache_init(cfg, self.tbuf, tb, self.sbuf if sb else None, sb)
        self.cfg = ca2_cache_config(self.handle)         # defaults resolved by the library
        self.tpe_len = self.cfg.tpe_len                   # rows of the TPE table

    def close(self):
        if self.handle:
            ca2_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def ring(self, layer: int, kv: int):
        """Ring of one layer, token-major and head-major within a token: [B][HW][H][Pmax][D]."""
        c = self.cfg
        off = ca2_cache_layer_offsets(self.handle, layer, kv)[0] // 2
        shape = (c.batch, c.hw, c.heads, c.p_max, c.head_dim)
        return self.tbuf[off:off + _numel(shape)].view(*shape)

    def spatial(self, layer: int, kv: int):
        c = self.cfg
        off = ca2_cache_layer_offsets(self.handle, layer, kv)[1] // 2
        shape = (c.p_spatial, c.batch, c.hw, c.heads, c.head_dim)
        return self.sbuf[off:off + _numel(shape)].view(*shape)

    def state(self):
        return ca2_cache_state(self.handle)

    def evict(self, n):
        ca2_cache_evict(self.handle, n)

    def evict_for(self, n_new: int) -> int:
        """Evict just enough of the oldest frames for n_new more to fit; returns that count."""
        return ca2_cache_evict_for(self.handle, n_new)

    def write(self, k_t, v_t, k_s, v_s, n, stream=None):
        ca2_cache_write(self.handle, k_t, v_t, k_s, v_s, n, stream)

    def kv_proj_write(self, layer, x_t, w_t, b_t, x_s, w_s, b_s, n, stream=None):
        ca2_kv_proj_write(self.handle, layer, x_t, w_t, b_t, x_s, w_s, b_s, n, stream)

    def commit(self, n):
        ca2_cache_commit(self.handle, n)

    def temporal(self, layer, q, k, v, out, n, stream=None):
        ca2_temporal_attn(self.handle, layer, q, k, v, out, n, stream)

    def spatial_attn(self, layer, q, k, v, out, n, use_prefix, stream=None):
        ca2_spatial_prefix_attn(self.handle, layer, q, k, v, out, n, use_prefix, stream)

    def tpe(self, first_global_frame, offset, n):
        return ca2_tpe_indices(self.handle, first_global_frame, offset, n)

    def tpe_add(self, first_global_frame, offset, table, x, out, n, stream=None):
        ca2_tpe_add(self.handle, first_global_frame, offset, table, x, out, n, stream)
