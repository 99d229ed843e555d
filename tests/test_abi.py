"""The C ABI library loads, exports every symbol include/rtp.h declares, and rejects bad
arguments on the host before touching a device (CPU only, no compute calls)."""
import ctypes
import os
import re

import numpy as np
import pytest

from long_context_sparse_rtpurbo_b200 import _lib
from long_context_sparse_rtpurbo_b200 import rtp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "rtp.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(rtp_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    declared = _declared_functions()
    assert len(declared) >= 8
    for name in declared:
        assert hasattr(lib, name), name
    assert set(_lib.EXPORTS) <= set(declared)


def test_struct_layouts_match_header_sizes():
    # int32 x 8, double, int64, pointer
    assert ctypes.sizeof(_lib.RtpLayerDesc) == 8 * 4 + 8 + 8 + 8
    assert ctypes.sizeof(_lib.RtpCache) == 7 * 8 + 8


def test_status_strings():
    for c in (0, -1, -2, -3, -4, -5, -6):
        assert rtp.rtp_status_str(c)
    assert rtp.rtp_status_str(-99) == "unknown status"


def test_slot_map():
    slots, nr, nl = rtp.rtp_build_slot_map([0, 1, 1, 0, 0, 1, 0, 0])
    assert list(slots) == [-1, 0, 1, -2, -3, 2, -4, -5]
    assert (nr, nl) == (3, 5)


def _desc(**kw):
    a = dict(B=2, Hq=32, Hkv=8, sinks=4, window=2048, max_seq_len=32768,
             slot_of_kv=rtp.rtp_build_slot_map([1, 0, 0, 0, 0, 1, 0, 0])[0])
    a.update(kw)
    return rtp.LayerDesc(**a)


def test_workspace_bytes_scales_and_rejects_bad_shapes():
    small = rtp.rtp_workspace_bytes(_desc(max_seq_len=4096))
    big = rtp.rtp_workspace_bytes(_desc(max_seq_len=1 << 20))
    assert 0 < small < big
    assert rtp.rtp_workspace_bytes(_desc(Hq=30)) == 0           # Hq % Hkv
    assert rtp.rtp_workspace_bytes(_desc(Hq=24, Hkv=8)) == 0    # G = 3
    assert rtp.rtp_workspace_bytes(_desc(head_dim=64)) == 0
    assert rtp.rtp_workspace_bytes(_desc(idx_dim=8)) == 0
    assert rtp.rtp_workspace_bytes(_desc(window=0)) == 0
    assert rtp.rtp_workspace_bytes(_desc(max_seq_len=0)) == 0
    assert rtp.rtp_workspace_bytes(_desc(max_seq_len=1 << 25)) == 0
    bad = _desc(slot_of_kv=np.array([0, 0, -1, -2, -3, -4, -5, -6], np.int32))  # duplicate slot
    assert rtp.rtp_workspace_bytes(bad) == 0
    gap = _desc(slot_of_kv=np.array([1, -1, -2, -3, -4, -5, -6, -7], np.int32))  # slot 0 missing
    assert rtp.rtp_workspace_bytes(gap) == 0


def test_decode_rejects_bad_arguments_before_any_launch():
    d = _desc()
    lib = _lib.load()
    cache = _lib.RtpCache()
    dummy = 0x1000
    # null q_pre
    rc = lib.rtp_decode_step(d.ref, ctypes.byref(cache), None, dummy, dummy, 0.9, dummy, dummy,
                             None, 0, dummy, 1 << 30, None)
    assert rc == _lib.RTP_EINVAL
    cache = rtp.make_cache(dummy, dummy, dummy, dummy, dummy, dummy, dummy, 65536)
    for p in (0.0, -0.5, float("nan")):
        rc = lib.rtp_decode_step(d.ref, ctypes.byref(cache), dummy, dummy, dummy, p, dummy,
                                 dummy, None, 0, dummy, 1 << 30, None)
        assert rc == _lib.RTP_EINVAL, p
    # workspace too small / missing / misaligned
    need = rtp.rtp_workspace_bytes(d)
    rc = lib.rtp_decode_step(d.ref, ctypes.byref(cache), dummy, dummy, dummy, 0.9, dummy, dummy,
                             None, 0, dummy, need - 1, None)
    assert rc == _lib.RTP_EWORKSPACE
    rc = lib.rtp_decode_step(d.ref, ctypes.byref(cache), dummy, dummy, dummy, 0.9, dummy, dummy,
                             None, 0, None, need, None)
    assert rc == _lib.RTP_EWORKSPACE
    rc = lib.rtp_decode_step(d.ref, ctypes.byref(cache), dummy, dummy, dummy, 0.9, dummy, dummy,
                             None, 0, dummy + 8, need, None)
    assert rc == _lib.RTP_EWORKSPACE
    # sel_idx stride shorter than max_seq_len
    rc = lib.rtp_decode_step(d.ref, ctypes.byref(cache), dummy, dummy, dummy, 0.9, dummy, dummy,
                             dummy, 100, dummy, need, None)
    assert rc == _lib.RTP_EINVAL


def test_fused_decode_rejects_bad_arguments_before_any_launch():
    d = _desc()                      # has retrieval heads
    lib = _lib.load()
    dummy = 0x1000
    cache = rtp.make_cache(dummy, dummy, dummy, dummy, dummy, dummy, dummy, 65536)
    need = rtp.rtp_workspace_bytes(d)
    args = lambda k, v, wk, ws_bytes: (d.ref, ctypes.byref(cache), k, v, wk, dummy, dummy, dummy,
                                       0.9, dummy, dummy, None, 0, dummy, ws_bytes, None)
    assert lib.rtp_decode_step_append(*args(None, dummy, dummy, need)) == _lib.RTP_EINVAL
    assert lib.rtp_decode_step_append(*args(dummy, None, dummy, need)) == _lib.RTP_EINVAL
    assert lib.rtp_decode_step_append(*args(dummy, dummy, None, need)) == _lib.RTP_EINVAL
    # the decode step's own checks follow
    assert lib.rtp_decode_step_append(*args(dummy, dummy, dummy, need - 1)) == _lib.RTP_EWORKSPACE


def test_append_rejects_bad_arguments():
    d = _desc()
    lib = _lib.load()
    cache = rtp.make_cache(None, None, None, None, None, 0x1000, 0x1000, 65536)
    # retrieval caches missing while the layer has retrieval heads
    rc = lib.rtp_append_kv(d.ref, ctypes.byref(cache), 0x1000, 0x1000, 0x1000, 0x1000, None, 4,
                           None, None)
    assert rc == _lib.RTP_EINVAL
    cache = rtp.make_cache(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 65536)
    rc = lib.rtp_append_kv(d.ref, ctypes.byref(cache), 0x1000, 0x1000, 0x1000, 0x1000, None, -1,
                           None, None)
    assert rc == _lib.RTP_EINVAL
    rc = lib.rtp_append_kv(d.ref, ctypes.byref(cache), 0x1000, 0x1000, 0x1000, 0x1000, None, 0,
                           None, None)
    assert rc == _lib.RTP_OK                                        # nothing to do


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError):
        _lib._lib = None
        try:
            _lib.load(str(tmp_path / "nope.so"))
        finally:
            _lib._lib = None


def test_injected_failure_returns_before_any_launch():
    """rtp_debug_fail_next_call: the next entry-point call returns the injected status before
    looking at its arguments (so nothing reaches a device), once; then calls behave again."""
    d = _desc()
    lib = _lib.load()
    cache = rtp.make_cache(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 65536)
    append = lambda: lib.rtp_append_kv(d.ref, ctypes.byref(cache), 0x1000, 0x1000, 0x1000, 0x1000,
                                       None, 0, None, None)
    assert append() == _lib.RTP_OK                                  # n_new = 0: nothing to do
    rtp.rtp_debug_fail_next_call(_lib.RTP_ECUDA)
    assert append() == _lib.RTP_ECUDA
    assert append() == _lib.RTP_OK                                  # consumed by one call
    # decode: the injected code comes before the argument checks (null q_pre would be EINVAL)
    rtp.rtp_debug_fail_next_call(_lib.RTP_ETIMEOUT)
    rc = lib.rtp_decode_step(d.ref, ctypes.byref(cache), None, 0x1000, 0x1000, 0.9, 0x1000,
                             0x1000, None, 0, 0x1000, 1 << 30, None)
    assert rc == _lib.RTP_ETIMEOUT
    rc = lib.rtp_decode_step(d.ref, ctypes.byref(cache), None, 0x1000, 0x1000, 0.9, 0x1000,
                             0x1000, None, 0, 0x1000, 1 << 30, None)
    assert rc == _lib.RTP_EINVAL
    rtp.rtp_debug_fail_next_call(_lib.RTP_EDEVICE)
    rc = lib.rtp_decode_step_static(d.ref, ctypes.byref(cache), 0x1000, 0x1000, 0x1000, 0.9,
                                    0x1000, 0x1000, None)
    assert rc == _lib.RTP_EDEVICE
    rtp.rtp_debug_fail_next_call(_lib.RTP_EWORKSPACE)
    rtp.rtp_debug_fail_next_call(0)                                 # cancelled
    assert append() == _lib.RTP_OK
    for bad in (1, -7):
        assert lib.rtp_debug_fail_next_call(bad) == _lib.RTP_EINVAL


def test_wait_limit_hook_validates():
    lib = _lib.load()
    assert lib.rtp_debug_set_wait_limit(-1) == _lib.RTP_EINVAL
    assert lib.rtp_debug_set_wait_limit(5000) == _lib.RTP_OK
    assert lib.rtp_debug_set_wait_limit(0) == _lib.RTP_OK            # default restored


def test_prefill_workspace_and_argument_checks():
    """rtp_prefill_workspace_bytes: the status header plus the rotated keys [B][Hkv][n][128];
    rtp_prefill rejects bad arguments before any device call (n_max = 0 does nothing)."""
    d = _desc(max_seq_len=4096)
    lib = _lib.load()
    need = rtp.rtp_prefill_workspace_bytes(d, 1000)
    assert need == 256 + 2 * 8 * 1000 * 256                         # B = 2, Hkv = 8
    assert rtp.rtp_prefill_workspace_bytes(d, 0) == 0
    assert rtp.rtp_prefill_workspace_bytes(d, 4097) == 0
    assert rtp.rtp_prefill_workspace_bytes(_desc(Hq=30), 100) == 0
    x = 0x1000
    call = lambda q, n, ws, wsb: lib.rtp_prefill(d.ref, q, x, x, x, n, x, ws, wsb, None)
    assert call(None, 1000, x, need) == _lib.RTP_EINVAL
    assert call(x, -1, x, need) == _lib.RTP_EINVAL
    assert call(x, 4097, x, 1 << 30) == _lib.RTP_ESHAPE
    assert call(x, 0, None, 0) == _lib.RTP_OK                       # nothing to do
    assert call(x, 1000, x, need - 1) == _lib.RTP_EWORKSPACE
    assert call(x, 1000, None, need) == _lib.RTP_EWORKSPACE
    assert call(x, 1000, x + 16, need) == _lib.RTP_EWORKSPACE       # not 256-byte aligned
    rtp.rtp_debug_fail_next_call(_lib.RTP_ECUDA)
    assert call(None, 1000, x, need) == _lib.RTP_ECUDA               # before the checks
    assert call(None, 1000, x, need) == _lib.RTP_EINVAL


def test_misaligned_row_arrays_are_rejected_before_any_launch():
    """Row arrays are moved in 16-byte pieces: a pointer off a 16-byte boundary is RTP_EINVAL
    for the append, the decode step and the prefill (nothing reaches a device)."""
    d = _desc()
    lib = _lib.load()
    x, bad = 0x1000, 0x1002
    cache = rtp.make_cache(x, x, x, x, x, x, x, 65536)
    rc = lib.rtp_append_kv(d.ref, ctypes.byref(cache), bad, x, x, x, None, 4, None, None)
    assert rc == _lib.RTP_EINVAL
    need = rtp.rtp_workspace_bytes(d)
    for q, out, c in ((bad, x, cache), (x, bad, cache),
                      (x, x, rtp.make_cache(x, bad, x, x, x, x, x, 65536))):
        rc = lib.rtp_decode_step(d.ref, ctypes.byref(c), q, x, x, 0.9, out, x, None, 0, x,
                                 need, None)
        assert rc == _lib.RTP_EINVAL
    pf = rtp.rtp_prefill_workspace_bytes(d, 100)
    for args in ((bad, x, x, x), (x, bad, x, x), (x, x, bad, x), (x, x, x, bad)):
        q, k, v, out = args
        assert lib.rtp_prefill(d.ref, q, k, v, x, 100, out, x, pf, None) == _lib.RTP_EINVAL
