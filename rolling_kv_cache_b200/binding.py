"""ctypes binding of librc.so: the C ABI in include/rc.h, same names.

Argument marshalling only. Device tensors are torch CUDA tensors whose data
pointers are passed through; every step of the path runs in the library's
kernels. There is no fallback: if librc.so is missing or fails to load, every
call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "librc.so")

RC_OK, RC_EINVAL, RC_ESTATE, RC_ECUDA, RC_ERANGE, RC_ETIMEOUT, RC_ENOMEM = range(7)
RC_NONE, RC_SLIDING, RC_ROLLING_SINK, RC_INFINITY_ROPE, RC_DEEP_FORCING, RC_RELAX_FORCING, RC_MEMROPE = range(7)
RC_REINDEX_FLUSH, RC_REINDEX_CUT, RC_REINDEX_SINK = 1, 2, 4
RC_MAX_SLOTS = 256
RC_MAX_CHUNK_FRAMES = 16


class RcError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"rc status {status}: {message}")
        self.status = status


class rc_config(ctypes.Structure):
    _fields_ = [
        ("layers", ctypes.c_int), ("heads", ctypes.c_int), ("head_dim", ctypes.c_int),
        ("frame_seqlen", ctypes.c_int), ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int),
        ("sink_frames", ctypes.c_int), ("window_frames", ctypes.c_int),
        ("chunk_frames", ctypes.c_int), ("mask_block_frames", ctypes.c_int),
        ("rope_t_pairs", ctypes.c_int), ("rope_h_pairs", ctypes.c_int), ("rope_w_pairs", ctypes.c_int),
        ("theta", ctypes.c_double), ("t_max", ctypes.c_int), ("policy", ctypes.c_int),
        ("rs_bank_blocks", ctypes.c_int), ("rs_sink_blocks", ctypes.c_int),
        ("rs_static_semantics", ctypes.c_int), ("ir_f_limit", ctypes.c_int),
        ("ir_sink_blocks", ctypes.c_int), ("ir_cache_blocks", ctypes.c_int),
        ("df_budget_tokens", ctypes.c_int), ("rf_history_frames", ctypes.c_int),
        ("rf_weight", ctypes.c_double), ("mr_alpha_long", ctypes.c_double),
        ("mr_alpha_short", ctypes.c_double),
    ]


class rc_frame_state(ctypes.Structure):
    _fields_ = [("content", ctypes.c_int32), ("tau", ctypes.c_int32), ("region", ctypes.c_int32),
                ("rank", ctypes.c_int32), ("slot", ctypes.c_int32), ("stored_time", ctypes.c_int32)]


class rc_state(ctypes.Structure):
    _fields_ = [
        ("n_kept", ctypes.c_int32), ("frames_committed", ctypes.c_int32),
        ("chunk_start", ctypes.c_int32), ("chunk_frames", ctypes.c_int32),
        ("valid_tokens", ctypes.c_int32), ("shift", ctypes.c_int32),
        ("n_candidates", ctypes.c_int32), ("n_jobs", ctypes.c_int32),
        ("evicted", ctypes.c_int32 * RC_MAX_SLOTS), ("n_evicted", ctypes.c_int32),
        ("kept", rc_frame_state * RC_MAX_SLOTS),
        ("comp_tokens", ctypes.c_int32), ("comp_tau0", ctypes.c_int32), ("comp_row0", ctypes.c_int32),
    ]


class rc_layout(ctypes.Structure):
    _fields_ = [("kv_layer_stride", ctypes.c_size_t), ("k_offset", ctypes.c_size_t),
                ("v_offset", ctypes.c_size_t), ("raw_layer_stride", ctypes.c_size_t),
                ("raw_k_offset", ctypes.c_size_t), ("raw_v_offset", ctypes.c_size_t),
                ("q_offset", ctypes.c_size_t), ("capacity", ctypes.c_int32),
                ("raw_frames", ctypes.c_int32), ("total", ctypes.c_size_t)]


RC_KERNEL_NAMES = ["rerotate", "append", "attention", "scores", "topc", "combine", "compact"]
_NK = len(RC_KERNEL_NAMES)


class rc_profile(ctypes.Structure):
    _fields_ = [("launches", ctypes.c_int64 * _NK), ("timed", ctypes.c_int64 * _NK),
                ("ms", ctypes.c_double * _NK), ("flops", ctypes.c_double * _NK),
                ("bytes", ctypes.c_double * _NK)]


EXPORTS = ["rc_config_init", "rc_cache_bytes", "rc_cache_create", "rc_step", "rc_step_noalloc",
           "rc_select_topc", "rc_reindex", "rc_comp_tokens", "rc_pool_scores",
           "rc_get_state", "rc_device_status", "rc_rope_table", "rc_cache_layout",
           "rc_watchdog_selftest", "rc_profile_begin", "rc_profile_end", "rc_cache_destroy",
           "rc_last_error"]

_lib = None


def lib() -> ctypes.CDLL:
    """Load librc.so (once). Raises if it is missing: there is no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with python -m rolling_kv_cache_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.rc_config_init.argtypes = [ctypes.POINTER(rc_config), i, i, i, i, i, i]
        L.rc_cache_bytes.argtypes = [ctypes.POINTER(rc_config), ctypes.POINTER(sz)]
        L.rc_cache_create.argtypes = [ctypes.POINTER(rc_config), vp, sz, ctypes.POINTER(vp)]
        L.rc_step.argtypes = [vp, i, vp, vp, vp, i, i, i, vp, vp, vp, vp, i, vp]
        L.rc_step_noalloc.argtypes = L.rc_step.argtypes
        L.rc_select_topc.argtypes = [vp, i, vp, i, vp, vp]
        L.rc_comp_tokens.argtypes = [vp, i, vp, vp, vp]
        L.rc_pool_scores.argtypes = [vp, i, vp, vp, vp]
        L.rc_reindex.argtypes = [vp, i, i, ctypes.c_uint, vp]
        L.rc_get_state.argtypes = [vp, i, ctypes.POINTER(rc_state)]
        L.rc_device_status.argtypes = [vp, vp]
        L.rc_rope_table.argtypes = [vp, i, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(sz)]
        L.rc_cache_layout.argtypes = [vp, ctypes.POINTER(rc_layout)]
        L.rc_watchdog_selftest.argtypes = [vp, ctypes.c_uint, vp]
        L.rc_profile_begin.argtypes = [vp, i]
        L.rc_profile_end.argtypes = [vp, ctypes.POINTER(rc_profile)]
        L.rc_cache_destroy.argtypes = [vp]
        L.rc_last_error.argtypes = []
        L.rc_last_error.restype = ctypes.c_char_p
        for name in EXPORTS[:-1]:
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def check(status: int) -> None:
    if status != RC_OK:
        raise RcError(status, lib().rc_last_error().decode())


def rc_config_init(layers, heads, head_dim, frame_seqlen, sink_frames, window_frames) -> rc_config:
    cfg = rc_config()
    check(lib().rc_config_init(ctypes.byref(cfg), layers, heads, head_dim, frame_seqlen,
                               sink_frames, window_frames))
    return cfg


def rc_cache_bytes(cfg: rc_config) -> int:
    n = ctypes.c_size_t()
    check(lib().rc_cache_bytes(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def rc_cache_create(cfg: rc_config, dev_mem: int, nbytes: int) -> int:
    h = ctypes.c_void_p()
    check(lib().rc_cache_create(ctypes.byref(cfg), dev_mem or None, nbytes, ctypes.byref(h)))
    return h.value


def rc_step(handle, layer, q, k_new, v_new, frame_start, n_frames, policy, out, lse=0,
            scores=0, topc=0, C=0, stream=0) -> None:
    check(lib().rc_step(handle, layer, q or None, k_new or None, v_new or None, frame_start,
                        n_frames, policy, out or None, lse or None, scores or None, topc or None,
                        C, stream or None))


def rc_step_noalloc(handle, layer, q, k_new, v_new, frame_start, n_frames, policy, out, lse=0,
                    scores=0, topc=0, C=0, stream=0) -> None:
    """rc_step with its per-call scratch in the library's static device array."""
    check(lib().rc_step_noalloc(handle, layer, q or None, k_new or None, v_new or None,
                                frame_start, n_frames, policy, out or None, lse or None,
                                scores or None, topc or None, C, stream or None))


def rc_select_topc(handle, layer, scores, C, topc, stream=0) -> None:
    """Top-C over a caller-supplied (e.g. rank-summed) score vector in layer's candidate order."""
    check(lib().rc_select_topc(handle, layer, scores or None, C, topc or None, stream or None))


def rc_comp_tokens(handle, layer, n, stream=0):
    """Deep Forcing: (frames, tokens) int32 arrays of the layer's compressed region."""
    frame = (ctypes.c_int32 * max(1, n))()
    tok = (ctypes.c_int32 * max(1, n))()
    check(lib().rc_comp_tokens(handle, layer, frame, tok, stream or None))
    return list(frame)[:n], list(tok)[:n]


def rc_pool_scores(handle, layer, stream=0):
    """Relax Forcing: the pool scores of the layer's last frame selection."""
    buf = (ctypes.c_float * RC_MAX_SLOTS)()
    n = ctypes.c_int32()
    check(lib().rc_pool_scores(handle, layer, buf, ctypes.byref(n), stream or None))
    return list(buf)[:n.value]


def rc_reindex(handle, policy, t_delta, flags, stream=0) -> None:
    check(lib().rc_reindex(handle, policy, t_delta, flags, stream or None))


def rc_get_state(handle, layer) -> rc_state:
    st = rc_state()
    check(lib().rc_get_state(handle, layer, ctypes.byref(st)))
    return st


def rc_device_status(handle, stream=0) -> None:
    check(lib().rc_device_status(handle, stream or None))


def rc_rope_table(handle, axis):
    import numpy as np
    n = ctypes.c_size_t()
    check(lib().rc_rope_table(handle, axis, None, ctypes.byref(n)))
    out = np.empty(n.value, dtype=np.float32)
    check(lib().rc_rope_table(handle, axis, out.ctypes.data_as(ctypes.POINTER(ctypes.c_float)),
                              ctypes.byref(n)))
    return out


def rc_cache_layout(handle) -> rc_layout:
    lay = rc_layout()
    check(lib().rc_cache_layout(handle, ctypes.byref(lay)))
    return lay


def rc_watchdog_selftest(handle, limit_us, stream=0) -> None:
    check(lib().rc_watchdog_selftest(handle, limit_us, stream or None))


def rc_profile_begin(handle, max_launches) -> None:
    check(lib().rc_profile_begin(handle, max_launches))


def rc_profile_end(handle) -> dict:
    p = rc_profile()
    check(lib().rc_profile_end(handle, ctypes.byref(p)))
    return {n: dict(launches=p.launches[i], timed=p.timed[i], ms=p.ms[i], flops=p.flops[i],
                    bytes=p.bytes[i]) for i, n in enumerate(RC_KERNEL_NAMES)}


def rc_cache_destroy(handle) -> None:
    if handle:
        check(lib().rc_cache_destroy(handle))
