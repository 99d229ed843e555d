"""Thin Python binding of librtp's C ABI (include/rtp.h).

The functions keep the C names and only marshal arguments: torch tensors become device
pointers, the current CUDA stream becomes the stream argument. Every step of the decode path
runs in librtp's kernels; there is no CPU fallback, and a missing library raises.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import _lib
from ._lib import RtpCache, RtpLayerDesc, RTP_OK


class RtpError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {code} ({rtp_status_str(code)})")
        self.code = code


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        if t.numel() and not t.is_contiguous():
            raise ValueError("tensors passed to librtp must be contiguous")
        return t.data_ptr() if t.numel() else None
    return int(t)


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(fn: str, rc: int):
    if rc != RTP_OK:
        raise RtpError(fn, rc)
    return rc


def rtp_status_str(code: int) -> str:
    return _lib.load().rtp_status_str(code).decode()


def rtp_build_slot_map(ret_mask) -> tuple[np.ndarray, int, int]:
    """Host retrieval mask [Hkv] -> (slot_of_kv int32 [Hkv], n_ret, n_loc)."""
    m = np.ascontiguousarray(np.asarray(ret_mask, dtype=np.uint8))
    slots = np.zeros(m.shape[0], dtype=np.int32)
    nr, nl = ctypes.c_int32(), ctypes.c_int32()
    _check("rtp_build_slot_map", _lib.load().rtp_build_slot_map(
        m.ctypes.data, m.shape[0], slots.ctypes.data, ctypes.byref(nr), ctypes.byref(nl)))
    return slots, nr.value, nl.value


class LayerDesc:
    """Owns the host slot array that an RtpLayerDesc points to."""

    def __init__(self, B, Hq, Hkv, sinks, window, max_seq_len, slot_of_kv, rope_base=1e6,
                 head_dim=128, idx_dim=16):
        self.slots = np.ascontiguousarray(np.asarray(slot_of_kv, dtype=np.int32))
        self.c = RtpLayerDesc(B, Hq, Hkv, head_dim, idx_dim, sinks, window, 0, float(rope_base),
                              int(max_seq_len),
                              self.slots.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
        self.n_ret = int((self.slots >= 0).sum())
        self.n_loc = int((self.slots < 0).sum())

    @property
    def ref(self):
        return ctypes.byref(self.c)


def make_cache(k_ret, v_ret, idx, k_loc, v_loc, seq_off, seq_cap, T_total) -> RtpCache:
    return RtpCache(_ptr(k_ret), _ptr(v_ret), _ptr(idx), _ptr(k_loc), _ptr(v_loc), _ptr(seq_off),
                    _ptr(seq_cap), int(T_total))


def rtp_workspace_bytes(desc: LayerDesc) -> int:
    return int(_lib.load().rtp_workspace_bytes(desc.ref))


def rtp_workspace_init(ws: torch.Tensor, stream=None):
    _check("rtp_workspace_init",
           _lib.load().rtp_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def rtp_append_kv(desc: LayerDesc, cache: RtpCache, k_pre, v, w_kidx, start_pos, n_new_b, n_new,
                  ws=None, stream=None):
    return _check("rtp_append_kv", _lib.load().rtp_append_kv(
        desc.ref, ctypes.byref(cache), _ptr(k_pre), _ptr(v), _ptr(w_kidx), _ptr(start_pos),
        _ptr(n_new_b), int(n_new), _ptr(ws), _stream(stream)))


def rtp_decode_step(desc: LayerDesc, cache: RtpCache, q_pre, w_qidx, seq_lens, p, out, sel_counts,
                    sel_idx=None, sel_stride=0, ws=None, ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    return _check("rtp_decode_step", _lib.load().rtp_decode_step(
        desc.ref, ctypes.byref(cache), _ptr(q_pre), _ptr(w_qidx), _ptr(seq_lens), float(p),
        _ptr(out), _ptr(sel_counts), _ptr(sel_idx), int(sel_stride), _ptr(ws), int(ws_bytes),
        _stream(stream)))


def rtp_decode_step_append(desc: LayerDesc, cache: RtpCache, k_new, v_new, w_kidx, q_pre, w_qidx,
                           seq_lens, p, out, sel_counts, sel_idx=None, sel_stride=0, ws=None,
                           ws_bytes=None, stream=None):
    """rtp_append_kv of the decode token and rtp_decode_step in one launch (see include/rtp.h)."""
    if ws_bytes is None:
        ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    return _check("rtp_decode_step_append", _lib.load().rtp_decode_step_append(
        desc.ref, ctypes.byref(cache), _ptr(k_new), _ptr(v_new), _ptr(w_kidx), _ptr(q_pre),
        _ptr(w_qidx), _ptr(seq_lens), float(p), _ptr(out), _ptr(sel_counts), _ptr(sel_idx),
        int(sel_stride), _ptr(ws), int(ws_bytes), _stream(stream)))


def rtp_decode_step_topk(desc: LayerDesc, cache: RtpCache, q_pre, w_qidx, seq_lens, k, out,
                         sel_counts, sel_idx=None, sel_stride=0, ws=None, ws_bytes=None,
                         stream=None):
    """Decode step with the fixed-budget top-k selector (see include/rtp.h)."""
    if ws_bytes is None:
        ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    return _check("rtp_decode_step_topk", _lib.load().rtp_decode_step_topk(
        desc.ref, ctypes.byref(cache), _ptr(q_pre), _ptr(w_qidx), _ptr(seq_lens), int(k),
        _ptr(out), _ptr(sel_counts), _ptr(sel_idx), int(sel_stride), _ptr(ws), int(ws_bytes),
        _stream(stream)))


def rtp_prefill_workspace_bytes(desc: LayerDesc, n_max: int) -> int:
    return int(_lib.load().rtp_prefill_workspace_bytes(desc.ref, int(n_max)))


def rtp_prefill(desc: LayerDesc, q_pre, k_pre, v, n_b, n_max, out, ws=None, ws_bytes=None,
                stream=None):
    """Causal prefill attention of one layer over a prompt (see include/rtp.h)."""
    if ws_bytes is None:
        ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    return _check("rtp_prefill", _lib.load().rtp_prefill(
        desc.ref, _ptr(q_pre), _ptr(k_pre), _ptr(v), _ptr(n_b), int(n_max), _ptr(out), _ptr(ws),
        int(ws_bytes), _stream(stream)))


def rtp_decode_step_static(desc: LayerDesc, cache: RtpCache, q_pre, w_qidx, seq_lens, p, out,
                           sel_counts, stream=None):
    """rtp_decode_step on the library's own fixed scratch (no workspace argument): for callers
    that cannot allocate device memory. See include/rtp.h for its limits and sharing rules."""
    return _check("rtp_decode_step_static", _lib.load().rtp_decode_step_static(
        desc.ref, ctypes.byref(cache), _ptr(q_pre), _ptr(w_qidx), _ptr(seq_lens), float(p),
        _ptr(out), _ptr(sel_counts), _stream(stream)))


def rtp_read_device_status(ws, stream=None) -> int:
    return int(_lib.load().rtp_read_device_status(_ptr(ws), _stream(stream)))


def rtp_last_launch_count() -> int:
    return int(_lib.load().rtp_last_launch_count())


def rtp_debug_set_wait_limit(cycles: int):
    """Test hook: limit (SM cycles) of every device-side wait of later decode launches;
    0 restores the default (about one second)."""
    return _check("rtp_debug_set_wait_limit", _lib.load().rtp_debug_set_wait_limit(int(cycles)))


def rtp_debug_fail_next_call(status: int):
    """Test hook: the next append / decode entry-point call returns ``status`` (a negative
    RTP_E* code) without enqueueing anything; 0 cancels."""
    return _check("rtp_debug_fail_next_call", _lib.load().rtp_debug_fail_next_call(int(status)))
