"""One decode layer's device memory (caches, workspace) allocated with PyTorch, driving
librtp through the C ABI. Allocation and stream plumbing only; no arithmetic of the method."""
from __future__ import annotations

import numpy as np
import torch

from . import rtp


class DecodeLayer:
    def __init__(self, B, Hq, Hkv, sinks, window, max_seq_len, ret_mask, seq_caps,
                 device="cuda", rope_base=1e6):
        slots, n_ret, n_loc = rtp.rtp_build_slot_map(ret_mask)
        self.B, self.Hq, self.Hkv = B, Hq, Hkv
        self.sinks, self.window = sinks, window
        self.n_ret, self.n_loc = n_ret, n_loc
        self.slots = slots
        self.desc = rtp.LayerDesc(B, Hq, Hkv, sinks, window, max_seq_len, slots, rope_base)
        caps = np.asarray(seq_caps, dtype=np.int64)
        offs = np.concatenate([[0], np.cumsum(caps)[:-1]]).astype(np.int64)
        self.seq_caps_host, self.seq_offs_host = caps, offs
        self.T_total = int(caps.sum())
        bf = torch.bfloat16
        ring = sinks + window
        self.k_ret = torch.empty((n_ret, self.T_total, 128), dtype=bf, device=device)
        self.v_ret = torch.empty((n_ret, self.T_total, 128), dtype=bf, device=device)
        self.idx = torch.empty((n_ret, self.T_total, 16), dtype=bf, device=device)
        self.k_loc = torch.empty((n_loc, B, ring, 128), dtype=bf, device=device)
        self.v_loc = torch.empty((n_loc, B, ring, 128), dtype=bf, device=device)
        self.seq_off = torch.tensor(offs, dtype=torch.int64, device=device)
        self.seq_cap = torch.tensor(caps.astype(np.int32), dtype=torch.int32, device=device)
        self.cache = rtp.make_cache(self.k_ret, self.v_ret, self.idx, self.k_loc, self.v_loc,
                                    self.seq_off, self.seq_cap, self.T_total)
        self.ws_bytes = rtp.rtp_workspace_bytes(self.desc)
        if self.ws_bytes == 0:
            raise ValueError("librtp rejected the layer description")
        self.ws = torch.empty(self.ws_bytes + 256, dtype=torch.uint8, device=device)
        off = (-self.ws.data_ptr()) % 256
        self.ws = self.ws[off:off + self.ws_bytes]
        rtp.rtp_workspace_init(self.ws)

    def append(self, k_pre, v, w_kidx, start_pos, n_new_b=None, stream=None):
        """k_pre, v: bf16 [B][n_new][Hkv][128]."""
        return rtp.rtp_append_kv(self.desc, self.cache, k_pre, v, w_kidx, start_pos, n_new_b,
                                 k_pre.shape[1], self.ws, stream)

    def decode(self, q_pre, w_qidx, seq_lens, p, out, sel_counts, sel_idx=None, stream=None):
        stride = 0 if sel_idx is None else sel_idx.shape[-1]
        return rtp.rtp_decode_step(self.desc, self.cache, q_pre, w_qidx, seq_lens, p, out,
                                   sel_counts, sel_idx, stride, self.ws, self.ws_bytes, stream)

    def decode_topk(self, q_pre, w_qidx, seq_lens, k, out, sel_counts, sel_idx=None, stream=None):
        """Decode step with the fixed-budget top-k selector."""
        stride = 0 if sel_idx is None else sel_idx.shape[-1]
        return rtp.rtp_decode_step_topk(self.desc, self.cache, q_pre, w_qidx, seq_lens, k, out,
                                        sel_counts, sel_idx, stride, self.ws, self.ws_bytes,
                                        stream)

    def decode_append(self, k_new, v_new, w_kidx, q_pre, w_qidx, seq_lens, p, out, sel_counts,
                      sel_idx=None, stream=None):
        """Append of the decode token (k_new, v_new: bf16 [B][Hkv][128] at seq_lens - 1) and
        the decode step in one launch."""
        stride = 0 if sel_idx is None else sel_idx.shape[-1]
        return rtp.rtp_decode_step_append(self.desc, self.cache, k_new, v_new, w_kidx, q_pre,
                                          w_qidx, seq_lens, p, out, sel_counts, sel_idx, stride,
                                          self.ws, self.ws_bytes, stream)

    def prefill(self, q_pre, k_pre, v, w_kidx, n_b, out, stream=None):
        """Prompt of n_b[b] tokens at positions 0..n_b[b]-1 (q_pre: bf16 [B][n_max][Hq][128];
        k_pre, v: bf16 [B][n_max][Hkv][128]; n_b: device int32 [B]): appends its K/V and index
        keys to the caches, then writes the causal prefill attention to out
        ([B][n_max][Hq][128]). The prefill scratch is allocated on first use and grown with
        the prompt."""
        n_max = q_pre.shape[1]
        start = torch.zeros(self.B, dtype=torch.int32, device=n_b.device)
        rtp.rtp_append_kv(self.desc, self.cache, k_pre, v, w_kidx, start, n_b, n_max, self.ws,
                          stream)
        need = rtp.rtp_prefill_workspace_bytes(self.desc, n_max)
        if need == 0:
            raise ValueError("librtp rejected the prompt length")
        if getattr(self, "pf_ws", None) is None or self.pf_ws.numel() < need:
            buf = torch.empty(need + 256, dtype=torch.uint8, device=q_pre.device)
            off = (-buf.data_ptr()) % 256
            self.pf_ws = buf[off:off + need]
        return rtp.rtp_prefill(self.desc, q_pre, k_pre, v, n_b, n_max, out, self.pf_ws,
                               self.pf_ws.numel(), stream)

    def status(self, stream=None) -> int:
        return rtp.rtp_read_device_status(self.ws, stream)
