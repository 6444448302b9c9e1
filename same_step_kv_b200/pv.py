"""Thin ctypes binding of libpv (include/pv.h), argument marshalling only.

Function names and argument order follow the C ABI.  Tensors may be passed as
torch tensors (their data_ptr() is used) or as raw integer addresses; the
CUDA stream defaults to torch's current stream.  Every pv_* call checks the
returned status and raises PVError with the library's message on failure.
There is no fallback: if libpv.so is missing, importing this module fails.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# PV_LIB may name another build of the same library (e.g. a tuning variant).
LIB_PATH = os.environ.get("PV_LIB") or os.path.join(_HERE, "libpv.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python -m same_step_kv_b200.build`")
lib = ctypes.CDLL(LIB_PATH)

PV_OK = 0
PV_ERR_INVALID_ARG = 1
PV_ERR_SHAPE = 2
PV_ERR_CAPACITY = 3
PV_ERR_STATE = 4
PV_ERR_UNSUPPORTED_ARCH = 5
PV_ERR_CUDA = 6
PV_ERR_TIMEOUT = 7
PV_STEP_SINK = -1
PV_MAX_RING = 64
PV_MAX_STREAMS = 64
PV_PHASE_NEW, PV_PHASE_FIRST, PV_PHASE_BOOT, PV_PHASE_STEADY = 0, 1, 2, 3


class pv_kv_config(ctypes.Structure):
    _fields_ = [("layers", ctypes.c_int), ("heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("frame_w", ctypes.c_int), ("frame_h", ctypes.c_int),
                ("first_frames", ctypes.c_int), ("ring_slots", ctypes.c_int),
                ("steps", ctypes.c_int), ("max_streams", ctypes.c_int),
                ("rope_pairs_t", ctypes.c_int), ("rope_pairs_h", ctypes.c_int),
                ("rope_pairs_w", ctypes.c_int), ("max_frames", ctypes.c_int),
                ("rope_theta", ctypes.c_double)]


class pv_kv_state(ctypes.Structure):
    _fields_ = [("phase", ctypes.c_int), ("chunk", ctypes.c_int), ("fill", ctypes.c_int),
                ("slot", ctypes.c_int), ("frame0", ctypes.c_int), ("nframes", ctypes.c_int),
                ("n_queries", ctypes.c_int), ("n_keys", ctypes.c_int),
                ("slot_frame", ctypes.c_int * PV_MAX_RING)]


class PVError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"pv status {status}: {message}")
        self.status = status


_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t
_SIGS = {
    "pv_version": ([], ctypes.c_char_p),
    "pv_last_error": ([ctypes.c_char_p, _sz], _i),
    "pv_kv_required_bytes": ([ctypes.POINTER(pv_kv_config), ctypes.POINTER(_sz),
                              ctypes.POINTER(_sz)], _i),
    "pv_kv_init": ([ctypes.POINTER(_vp), ctypes.POINTER(pv_kv_config), _vp, _sz, _vp, _sz], _i),
    "pv_kv_destroy": ([_vp], _i),
    "pv_kv_begin_chunk": ([_vp, _i, _i], _i),
    "pv_kv_begin_sink": ([_vp, _i], _i),
    "pv_kv_get_state": ([_vp, _i, ctypes.POINTER(pv_kv_state)], _i),
    "pv_kv_set_state": ([_vp, _i, ctypes.POINTER(pv_kv_state)], _i),
    "pv_kv_row_offset": ([_vp, _i, _i, _i, _i, _i, ctypes.POINTER(_sz), ctypes.POINTER(_sz)], _i),
    "pv_rope_append": ([_vp, _i, ctypes.POINTER(_i), _i, _i, _vp, _vp, _vp, _vp, _vp], _i),
    "pv_chunk_attn": ([_vp, _i, ctypes.POINTER(_i), _i, _i, _vp, _vp, _vp, _vp], _i),
    "pv_rope_dense": ([_vp, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp], _i),
    "pv_attn_dense_ws_bytes": ([_i, _i, _i, _i, ctypes.POINTER(_sz)], _i),
    "pv_attn_dense": ([_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _sz, _vp], _i),
    "pv_attn_dense_noalloc": ([_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp], _i),
    "pv_euler_step": ([_vp, _vp, _sz, ctypes.c_float, _vp], _i),
    "pv_kv_poll_device_error": ([_vp, ctypes.POINTER(_i)], _i),
    "pv_kv_selftest_wait_timeout": ([_vp, _vp], _i),
    "pv_attn_poll_device_error": ([_vp, _sz, ctypes.POINTER(_i), _vp], _i),
    "pv_attn_selftest_wait_timeout": ([_vp, _vp], _i),
    "pv_attn_varlen_ws_bytes": ([_i, _vp, _vp, _i, _i, ctypes.POINTER(_sz)], _i),
    "pv_attn_varlen": ([_vp, _vp, _vp, _i, _vp, _vp, _i, _i, _vp, _vp, _vp, _sz, _vp], _i),
    "pv_attn_plan": ([_i, _vp, _vp, _i, _i, _i, ctypes.POINTER(_i), ctypes.POINTER(_i),
                      ctypes.POINTER(ctypes.c_longlong)], _i),
    "pv_qkv_ws_bytes": ([_i, _i, ctypes.POINTER(_sz)], _i),
    "pv_qkv_rope_append": ([_vp, _i, _vp, _i, _i, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, _vp,
                            _vp, _sz, _vp], _i),
    "pv_sigma_schedule": ([_i, ctypes.c_double, ctypes.c_double, ctypes.POINTER(ctypes.c_double),
                           ctypes.POINTER(_i)], _i),
    "pv_euler_cfg_step": ([_vp, _vp, _vp, _sz, ctypes.c_float, ctypes.c_float, _vp], _i),
    "pv_x0_estimate": ([_vp, _vp, _vp, _sz, ctypes.c_float, _vp], _i),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res


def last_error() -> str:
    buf = ctypes.create_string_buffer(512)
    lib.pv_last_error(buf, 512)
    return buf.value.decode()


def _check(status: int) -> None:
    if status != PV_OK:
        raise PVError(status, last_error())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _streams(ids):
    arr = (ctypes.c_int * len(ids))(*[int(i) for i in ids])
    return len(ids), arr


# ------------------------------------------------------------------ C ABI
def pv_version() -> str:
    return lib.pv_version().decode()


def make_config(layers, heads, head_dim, frame_w, frame_h, first_frames=3, ring_slots=18,
                steps=4, max_streams=1, rope_pairs=None, max_frames=1024,
                rope_theta=10000.0) -> pv_kv_config:
    """pv_kv_config with the RoPE split d - 4*(d//6) / 2*(d//6) / 2*(d//6) dims by default."""
    if rope_pairs is None:
        s6 = head_dim // 6
        rope_pairs = ((head_dim - 4 * s6) // 2, s6, s6)
    return pv_kv_config(layers, heads, head_dim, frame_w, frame_h, first_frames, ring_slots,
                        steps, max_streams, rope_pairs[0], rope_pairs[1], rope_pairs[2],
                        max_frames, rope_theta)


def pv_kv_required_bytes(cfg: pv_kv_config) -> tuple[int, int]:
    a, b = _sz(), _sz()
    _check(lib.pv_kv_required_bytes(ctypes.byref(cfg), ctypes.byref(a), ctypes.byref(b)))
    return a.value, b.value


def pv_kv_init(cfg: pv_kv_config, kv_dev=None, kv_bytes=0, ws_dev=None, ws_bytes=0) -> int:
    h = _vp()
    _check(lib.pv_kv_init(ctypes.byref(h), ctypes.byref(cfg), _ptr(kv_dev), kv_bytes,
                          _ptr(ws_dev), ws_bytes))
    return h.value


def pv_kv_destroy(kv) -> None:
    _check(lib.pv_kv_destroy(kv))


def pv_kv_begin_chunk(kv, stream: int, nframes: int) -> None:
    _check(lib.pv_kv_begin_chunk(kv, stream, nframes))


def pv_kv_begin_sink(kv, stream: int) -> None:
    _check(lib.pv_kv_begin_sink(kv, stream))


def pv_kv_get_state(kv, stream: int) -> pv_kv_state:
    st = pv_kv_state()
    _check(lib.pv_kv_get_state(kv, stream, ctypes.byref(st)))
    return st


def pv_kv_set_state(kv, stream: int, st: pv_kv_state) -> None:
    _check(lib.pv_kv_set_state(kv, stream, ctypes.byref(st)))


def pv_kv_row_offset(kv, layer, step, stream, head, key) -> tuple[int, int]:
    a, b = _sz(), _sz()
    _check(lib.pv_kv_row_offset(kv, layer, step, stream, head, key, ctypes.byref(a),
                                ctypes.byref(b)))
    return a.value, b.value


def pv_rope_append(kv, streams, layer, step, q, k, v, q_rot, cuda_stream=None) -> None:
    n, arr = _streams(streams)
    _check(lib.pv_rope_append(kv, n, arr, layer, step, _ptr(q), _ptr(k), _ptr(v), _ptr(q_rot),
                              _stream(cuda_stream)))


def pv_chunk_attn(kv, streams, layer, step, q_rot, out, lse=None, cuda_stream=None) -> None:
    n, arr = _streams(streams)
    _check(lib.pv_chunk_attn(kv, n, arr, layer, step, _ptr(q_rot), _ptr(out), _ptr(lse),
                             _stream(cuda_stream)))


def pv_rope_dense(kv, n_tokens, frame0, q, k, v, q_rot, k_rot, v_hm, cuda_stream=None) -> None:
    _check(lib.pv_rope_dense(kv, n_tokens, frame0, _ptr(q), _ptr(k), _ptr(v), _ptr(q_rot),
                             _ptr(k_rot), _ptr(v_hm), _stream(cuda_stream)))


def pv_attn_dense_ws_bytes(n_q, n_k, heads, head_dim) -> int:
    a = _sz()
    _check(lib.pv_attn_dense_ws_bytes(n_q, n_k, heads, head_dim, ctypes.byref(a)))
    return a.value


def pv_attn_dense(q, k, v, n_q, n_k, heads, head_dim, out, lse, ws, ws_bytes,
                  cuda_stream=None) -> None:
    _check(lib.pv_attn_dense(_ptr(q), _ptr(k), _ptr(v), n_q, n_k, heads, head_dim, _ptr(out),
                             _ptr(lse), _ptr(ws), ws_bytes, _stream(cuda_stream)))


def _lengths(xs):
    arr = (ctypes.c_int * len(xs))(*[int(x) for x in xs])
    return arr


def pv_attn_varlen_ws_bytes(n_q, n_k, heads, head_dim) -> int:
    """n_q, n_k: per-sequence lengths (host sequences of equal size)."""
    if len(n_q) != len(n_k):
        raise ValueError("n_q and n_k differ in length")
    a = _sz()
    _check(lib.pv_attn_varlen_ws_bytes(len(n_q), _lengths(n_q), _lengths(n_k), heads, head_dim,
                                       ctypes.byref(a)))
    return a.value


def pv_attn_varlen(q, k, v, n_q, n_k, heads, head_dim, out, lse, ws, ws_bytes,
                   cuda_stream=None) -> None:
    if len(n_q) != len(n_k):
        raise ValueError("n_q and n_k differ in length")
    _check(lib.pv_attn_varlen(_ptr(q), _ptr(k), _ptr(v), len(n_q), _lengths(n_q), _lengths(n_k),
                              heads, head_dim, _ptr(out), _ptr(lse), _ptr(ws), ws_bytes,
                              _stream(cuda_stream)))


def pv_qkv_ws_bytes(tokens, dim) -> int:
    a = _sz()
    _check(lib.pv_qkv_ws_bytes(tokens, dim, ctypes.byref(a)))
    return a.value


def pv_qkv_rope_append(kv, streams, layer, step, x, w, bias, g_q, g_k, eps, q_rot, ws, ws_bytes,
                       cuda_stream=None) -> None:
    n, arr = _streams(streams)
    _check(lib.pv_qkv_rope_append(kv, n, arr, layer, step, _ptr(x), _ptr(w), _ptr(bias),
                                  _ptr(g_q), _ptr(g_k), ctypes.c_float(eps), _ptr(q_rot), _ptr(ws),
                                  ws_bytes, _stream(cuda_stream)))


def pv_attn_plan(n_q, n_k, heads, n_sm=148, partial_slots=None):
    """(grid, mode, ranges) of the attention plan for these lengths (host only)."""
    if len(n_q) != len(n_k):
        raise ValueError("n_q and n_k differ in length")
    if partial_slots is None:
        partial_slots = 4 * 160
    grid, mode = _i(), _i()
    ranges = (ctypes.c_longlong * 161)()
    _check(lib.pv_attn_plan(len(n_q), _lengths(n_q), _lengths(n_k), heads, n_sm, partial_slots,
                            ctypes.byref(grid), ctypes.byref(mode), ranges))
    return grid.value, mode.value, list(ranges[:grid.value + 1])


def pv_attn_dense_noalloc(q, k, v, n_q, n_k, heads, head_dim, out, lse=None,
                          cuda_stream=None) -> None:
    _check(lib.pv_attn_dense_noalloc(_ptr(q), _ptr(k), _ptr(v), n_q, n_k, heads, head_dim,
                                     _ptr(out), _ptr(lse), _stream(cuda_stream)))


def pv_euler_step(x, v, n, dsigma, cuda_stream=None) -> None:
    _check(lib.pv_euler_step(_ptr(x), _ptr(v), n, ctypes.c_float(dsigma), _stream(cuda_stream)))


def pv_kv_poll_device_error(kv) -> int:
    c = _i()
    _check(lib.pv_kv_poll_device_error(kv, ctypes.byref(c)))
    return c.value


def pv_sigma_schedule(n_steps, shift, sigma_max=0.0):
    """(sigmas: list of n_steps + 1 floats, timesteps: list of n_steps ints)."""
    sig = (ctypes.c_double * (n_steps + 1))()
    ts = (ctypes.c_int * n_steps)()
    _check(lib.pv_sigma_schedule(n_steps, shift, sigma_max, sig, ts))
    return list(sig), list(ts)


def pv_euler_cfg_step(x, v_cond, v_uncond, n, guide_scale, dsigma, cuda_stream=None) -> None:
    _check(lib.pv_euler_cfg_step(_ptr(x), _ptr(v_cond), _ptr(v_uncond), n,
                                 ctypes.c_float(guide_scale), ctypes.c_float(dsigma),
                                 _stream(cuda_stream)))


def pv_x0_estimate(x0, x, v, n, sigma, cuda_stream=None) -> None:
    _check(lib.pv_x0_estimate(_ptr(x0), _ptr(x), _ptr(v), n, ctypes.c_float(sigma),
                              _stream(cuda_stream)))


def pv_kv_selftest_wait_timeout(kv, cuda_stream=None) -> None:
    _check(lib.pv_kv_selftest_wait_timeout(kv, _stream(cuda_stream)))


def pv_attn_poll_device_error(ws=None, ws_bytes=0, cuda_stream=None) -> int:
    """ws=None: the fixed scratch of pv_attn_dense_noalloc."""
    c = _i()
    _check(lib.pv_attn_poll_device_error(_ptr(ws), ws_bytes, ctypes.byref(c),
                                         _stream(cuda_stream)))
    return c.value


def pv_attn_selftest_wait_timeout(ws=None, cuda_stream=None) -> None:
    _check(lib.pv_attn_selftest_wait_timeout(_ptr(ws), _stream(cuda_stream)))


# ------------------------------------------------------------------ helpers
class KVStore:
    """Owns the caller-side device buffers (torch) of one pv_kv handle."""

    def __init__(self, cfg: pv_kv_config, device="cuda"):
        import torch
        self.cfg = cfg
        self.kv_bytes, self.ws_bytes = pv_kv_required_bytes(cfg)
        self.kv_buf = torch.empty(self.kv_bytes, dtype=torch.uint8, device=device)
        self.ws_buf = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)
        self.handle = pv_kv_init(cfg, self.kv_buf, self.kv_bytes, self.ws_buf, self.ws_bytes)
        self.T = cfg.frame_w * cfg.frame_h
        self.ltot = (cfg.first_frames + cfg.ring_slots) * self.T

    def k_region(self):
        """The K region as bf16 [layers][steps][streams][heads][Ltot][D] (a view)."""
        import torch
        c = self.cfg
        n = c.layers * c.steps * c.max_streams * c.heads * self.ltot * c.head_dim
        flat = self.kv_buf.view(torch.bfloat16)
        return flat[:n].view(c.layers, c.steps, c.max_streams, c.heads, self.ltot, c.head_dim)

    def v_region(self):
        import torch
        c = self.cfg
        n = c.layers * c.steps * c.max_streams * c.heads * self.ltot * c.head_dim
        flat = self.kv_buf.view(torch.bfloat16)
        return flat[n:2 * n].view(c.layers, c.steps, c.max_streams, c.heads, self.ltot, c.head_dim)

    def close(self):
        if self.handle:
            pv_kv_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
