"""The C ABI library loads without a GPU and exports what include/rc.h declares."""
import ctypes
import os
import re

import pytest

from rolling_kv_cache_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "rc.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rc_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = B.lib()
    names = declared_functions()
    assert "rc_step" in names and "rc_cache_create" in names and "rc_reindex" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(B.EXPORTS) <= set(names)


def _header_layout(structs):
    """sizeof and offsetof of every field, as gcc lays the header's structs out."""
    import shutil
    import subprocess
    import tempfile
    if not shutil.which("gcc"):
        pytest.skip("gcc not available")
    lines = ['#include <stdio.h>', '#include "rc.h"', "int main(void) {"]
    for st in structs:
        name = st.__name__
        lines.append(f'  printf("{name} %zu\\n", sizeof({name}));')
        for f, _ in st._fields_:
            lines.append(f'  printf("{name}.{f} %zu\\n", offsetof({name}, {f}));')
    lines += ["  return 0;", "}"]
    with tempfile.TemporaryDirectory() as d:
        src, exe = os.path.join(d, "lay.c"), os.path.join(d, "lay")
        open(src, "w").write("\n".join(lines))
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), src, "-o", exe], check=True)
        out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    return dict((k, int(v)) for k, v in (ln.split() for ln in out.splitlines()))


def test_struct_layouts_match_header():
    structs = [B.rc_config, B.rc_frame_state, B.rc_state, B.rc_layout, B.rc_profile]
    lay = _header_layout(structs)
    for st in structs:
        assert ctypes.sizeof(st) == lay[st.__name__], st.__name__
        for f, _ in st._fields_:
            assert getattr(st, f).offset == lay[f"{st.__name__}.{f}"], (st.__name__, f)


def test_config_init_and_bytes():
    cfg = B.rc_config_init(1, 12, 128, 1560, 1, 18)
    assert (cfg.chunk_frames, cfg.mask_block_frames, cfg.t_max, cfg.policy) == (3, 1, 4096, B.RC_SLIDING)
    assert cfg.grid_h * cfg.grid_w == 1560
    n = B.rc_cache_bytes(cfg)
    kv = 2 * 12 * 19 * 1560 * 128 * 2
    assert kv <= n < kv + 64 * 2 ** 20


@pytest.mark.parametrize("field,value", [("head_dim", 96), ("frame_seqlen", 17), ("chunk_frames", 0),
                                         ("window_frames", 2), ("t_max", 0), ("heads", 0)])
def test_invalid_configs_rejected(field, value):
    cfg = B.rc_config_init(1, 12, 128, 1560, 1, 18)
    setattr(cfg, field, value)
    with pytest.raises(B.RcError) as e:
        B.rc_cache_bytes(cfg)
    assert e.value.status == B.RC_EINVAL
    assert B.lib().rc_last_error()


def test_host_handle_rejects_tensors_and_policy_mismatch():
    cfg = B.rc_config_init(1, 2, 64, 16, 1, 6)
    h = B.rc_cache_create(cfg, 0, 0)
    try:
        with pytest.raises(B.RcError):
            B.rc_step(h, 0, 1234, 0, 0, 0, 3, B.RC_SLIDING, 0)
        with pytest.raises(B.RcError):
            B.rc_step(h, 0, 0, 0, 0, 0, 3, B.RC_ROLLING_SINK, 0)
        B.rc_step(h, 0, 0, 0, 0, 0, 3, B.RC_SLIDING, 0)
        with pytest.raises(B.RcError) as e:
            B.rc_step(h, 0, 0, 0, 0, 6, 3, B.RC_SLIDING, 0)
        assert e.value.status == B.RC_ESTATE
        with pytest.raises(B.RcError):
            B.rc_step(h, 1, 0, 0, 0, 3, 3, B.RC_SLIDING, 0)   # layer out of range
        st = B.rc_get_state(h, 0)
        assert st.frames_committed == 3 and st.n_kept == 3
    finally:
        B.rc_cache_destroy(h)


def test_rope_tables_are_fp32_roundings_of_fp64():
    import numpy as np
    cfg = B.rc_config_init(1, 2, 128, 1560, 1, 6)
    cfg.grid_h, cfg.grid_w, cfg.t_max = 30, 52, 400
    h = B.rc_cache_create(cfg, 0, 0)
    try:
        for axis, (n, P) in enumerate(((400, 22), (30, 21), (52, 21))):
            t = B.rc_rope_table(h, axis).reshape(n, P, 2)
            pos = np.arange(n)[:, None]
            om = 10000.0 ** (-np.arange(P) / P)
            a = pos * om[None, :]
            assert np.max(np.abs(t[..., 0] - np.cos(a))) < 6e-8
            assert np.max(np.abs(t[..., 1] - np.sin(a))) < 6e-8
    finally:
        B.rc_cache_destroy(h)


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    """No CPU fallback: without librc.so the binding raises instead of
    computing anything another way."""
    import importlib
    import rolling_kv_cache_b200.binding as binding
    fresh = importlib.reload(binding)
    try:
        monkeypatch.setattr(fresh, "LIB_PATH", str(tmp_path / "librc.so"))
        monkeypatch.setattr(fresh, "_lib", None)
        with pytest.raises(RuntimeError, match="missing"):
            fresh.lib()
        with pytest.raises(RuntimeError):
            fresh.rc_config_init(1, 2, 64, 16, 1, 6)
    finally:
        importlib.reload(binding)


def _limit_cfg(policy, sink, window, chunk=3, **over):
    cfg = B.rc_config_init(1, 2, 64, 16, sink, window)
    cfg.chunk_frames = chunk
    cfg.policy = policy
    for k, v in over.items():
        setattr(cfg, k, v)
    return cfg


@pytest.mark.parametrize("policy,sink,window,chunk,over,ok", [
    # the slot table holds RC_MAX_SLOTS (256) frames
    (B.RC_SLIDING, 1, 255, 3, {}, True),
    (B.RC_SLIDING, 1, 256, 3, {}, False),
    # chunks of up to RC_MAX_CHUNK_FRAMES (16) frames
    (B.RC_SLIDING, 0, 16, 16, {}, True),
    (B.RC_SLIDING, 0, 17, 17, {}, False),
    # Deep Forcing: sink + tail + budget frames within 256
    (B.RC_DEEP_FORCING, 1, 245, 3, {"df_budget_tokens": 10 * 16}, True),
    (B.RC_DEEP_FORCING, 1, 245, 3, {"df_budget_tokens": 11 * 16}, False),
    # MemRoPE: two memory frames beside sink + window
    (B.RC_MEMROPE, 1, 253, 3, {"mr_alpha_long": 0.9, "mr_alpha_short": 0.5}, True),
    (B.RC_MEMROPE, 1, 254, 3, {"mr_alpha_long": 0.9, "mr_alpha_short": 0.5}, False),
    # Relax Forcing: history + chunk frames within one selection CTA's 64
    (B.RC_RELAX_FORCING, 1, 6, 3, {"rf_history_frames": 61, "rf_weight": 0.5}, True),
    (B.RC_RELAX_FORCING, 1, 6, 3, {"rf_history_frames": 62, "rf_weight": 0.5}, False),
])
def test_config_limits(policy, sink, window, chunk, over, ok):
    """Each documented size limit: the largest accepted value passes, one more
    is rejected with RC_EINVAL before anything is allocated."""
    cfg = _limit_cfg(policy, sink, window, chunk, **over)
    if ok:
        assert B.rc_cache_bytes(cfg) > 0
        h = B.rc_cache_create(cfg, 0, 0)   # host-only handle: the engine accepts it too
        B.rc_cache_destroy(h)
    else:
        with pytest.raises(B.RcError) as e:
            B.rc_cache_bytes(cfg)
        assert e.value.status == B.RC_EINVAL
