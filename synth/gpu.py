"""GPU bulk fill of the synthetic k_pre / v streams (libsynth.so), bit-identical to gen.py."""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from . import gen

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lib = None


def load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libsynth.so not found at {LIB_PATH}; run the build first")
        lib = ctypes.CDLL(LIB_PATH)
        vp = ctypes.c_void_p
        lib.synth_fill_rows.restype = ctypes.c_int
        lib.synth_fill_rows.argtypes = [vp, ctypes.c_int, ctypes.c_int, vp, ctypes.c_int, vp, vp,
                                        vp, vp, vp, ctypes.c_float, vp, vp]
        _lib = lib
    return _lib


class LayerFiller:
    """Device tables (stream keys, planted runs) of one layer of a workload."""

    def __init__(self, w, layer: int, device="cuda"):
        self.w, self.layer, self.device = w, layer, device
        B, H = w.B, w.Hkv
        kk = np.array([[gen.stream_key(w.seed, gen.T_KPRE, layer, b, h) for h in range(H)]
                       for b in range(B)], dtype=np.uint64)
        kv = np.array([[gen.stream_key(w.seed, gen.T_V, layer, b, h) for h in range(H)]
                       for b in range(B)], dtype=np.uint64)
        self.keys_k = torch.from_numpy(kk.view(np.int64)).to(device)
        self.keys_v = torch.from_numpy(kv.view(np.int64)).to(device)
        off, st, ln, dl = [0], [], [], []
        for b in range(B):
            for h in range(H):
                for (s, n, d) in w.shifts(layer, b, h):
                    st.append(s)
                    ln.append(n)
                    dl.append(np.asarray(d, np.float32))
                off.append(len(st))
        self.cl_off = torch.tensor(off, dtype=torch.int32, device=device)
        self.cl_start = torch.tensor(st + [0], dtype=torch.int32, device=device)
        self.cl_len = torch.tensor(ln + [0], dtype=torch.int32, device=device)
        self.cl_delta = torch.from_numpy(
            np.stack(dl + [np.zeros(128, np.float32)])).to(device).contiguous()

    def fill(self, t0, n: int, n_valid=None, stream=None):
        """k_pre, v bf16 [B][n][Hkv][128] for positions t0[b] + j, j < n (or n_valid[b])."""
        lib = load()
        w = self.w
        t0 = torch.as_tensor(t0, dtype=torch.int64, device=self.device)
        nv = None if n_valid is None else torch.as_tensor(n_valid, dtype=torch.int32,
                                                          device=self.device)
        k = torch.zeros((w.B, n, w.Hkv, 128), dtype=torch.bfloat16, device=self.device)
        v = torch.zeros_like(k)
        st = (stream or torch.cuda.current_stream()).cuda_stream
        nvp = None if nv is None else nv.data_ptr()
        rc = lib.synth_fill_rows(self.keys_k.data_ptr(), w.B, w.Hkv, t0.data_ptr(), n, nvp,
                                 self.cl_off.data_ptr(), self.cl_start.data_ptr(),
                                 self.cl_len.data_ptr(), self.cl_delta.data_ptr(),
                                 float(gen.INV_STD), k.data_ptr(), st)
        rc |= lib.synth_fill_rows(self.keys_v.data_ptr(), w.B, w.Hkv, t0.data_ptr(), n, nvp,
                                  None, None, None, None, float(gen.INV_STD), v.data_ptr(), st)
        if rc != 0:
            raise RuntimeError(f"synth_fill_rows failed ({rc})")
        return k, v
