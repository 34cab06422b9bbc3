"""Move a synthetic workload to the GPU and run it through the C ABI.

Used by the GPU tests, the benchmark and ``__graft_entry__.smoke``.  It only
copies arrays and calls ``sparse_attention_decode_rtpurbo_b200``; it holds no
part of the method.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

import sparse_attention_decode_rtpurbo_b200 as rtp


def bf16_tensor(a: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def bf16_to_f32(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


class DeviceCase:
    """Device copies of one workload plus a ready decode step with debug outputs."""

    def __init__(self, case, device="cuda", debug: bool = True):
        self.case = case
        self.device = device
        c = case
        self.q_pre = bf16_tensor(c.q_pre, device)
        self.q_rope = bf16_tensor(c.q_rope, device)
        self.Wq = bf16_tensor(c.Wq_idx, device)
        self.k_idx = bf16_tensor(c.k_idx, device)
        self.k_cache = bf16_tensor(c.k_cache, device)
        self.v_cache = bf16_tensor(c.v_cache, device)
        self.seq_lens = torch.from_numpy(np.ascontiguousarray(c.seq_lens, dtype=np.int32)).to(device)
        self.p = torch.from_numpy(np.ascontiguousarray(c.p, dtype=np.float32)).to(device)
        self.block_table = None if c.block_table is None else torch.from_numpy(
            np.ascontiguousarray(c.block_table, dtype=np.int32)).to(device)
        self.out = torch.zeros((c.B, c.Hq, 128), dtype=torch.bfloat16, device=device)
        BH = c.B * c.Hq
        self.words = (c.Ncap // 64 + 31) // 32
        self.dbg = None
        self.dbg_struct = None
        if debug:
            self.dbg = {
                "tau": torch.full((BH,), float("nan"), dtype=torch.float32, device=device),
                "kstar": torch.full((BH,), -1, dtype=torch.int32, device=device),
                "kept_blocks": torch.full((BH,), -1, dtype=torch.int32, device=device),
                "smax": torch.full((BH,), float("nan"), dtype=torch.float32, device=device),
                "Z": torch.full((BH,), float("nan"), dtype=torch.float64, device=device),
                "block_bitmap": torch.zeros((BH * self.words,), dtype=torch.int32, device=device),
                "trace": torch.zeros((rtp.TRACE_WORDS,), dtype=torch.int64, device=device),
            }
            self.dbg_struct = rtp.RtpDebug(*(self.dbg[k].data_ptr() for k in
                                             ("tau", "kstar", "kept_blocks", "smax", "Z", "block_bitmap", "trace")))
        self.topk = 0   # > 0: run() takes the static top-k variant with this k
        self.ring_W = 0  # > 0: run() reads the local-only KV heads from k_ring / v_ring (attach_ring)
        self.k_ring = self.v_ring = None
        self.step = rtp.Step(c.B, c.Hq, c.Hkv, c.Ncap, c.head_kind, block_table=self.block_table,
                             num_pages=c.num_pages, device=device, debug=self.dbg_struct)

    def attach_ring(self, k_ring: np.ndarray, v_ring: np.ndarray, ring_W: int):
        """Rings [B, Hkv, 64 + ring_W, 128] (uint16 bf16) for the local-only KV heads."""
        self.k_ring = bf16_tensor(k_ring, self.device)
        self.v_ring = bf16_tensor(v_ring, self.device)
        self.ring_W = int(ring_W)

    def run(self, stream=None):
        c = self.case
        if self.topk > 0:
            return self.run_topk(self.topk, stream)
        if self.ring_W > 0:
            if stream is None:
                stream = torch.cuda.current_stream(self.out.device)
            return self.step.ring(self.q_pre, self.q_rope, self.k_idx, self.k_cache, self.v_cache, self.k_ring,
                                  self.v_ring, self.ring_W, self.Wq, self.seq_lens, self.p, c.window, c.sink,
                                  self.out, stream)
        if stream is None:
            stream = torch.cuda.current_stream(self.out.device)
        self.step(self.q_pre, self.q_rope, self.k_idx, self.k_cache, self.v_cache, self.Wq, self.seq_lens, self.p,
                  c.window, c.sink, self.out, stream)

    def run_topk(self, k: int, stream=None):
        """The static top-k variant of the step (every retrieval head keeps k tokens)."""
        c = self.case
        if stream is None:
            stream = torch.cuda.current_stream(self.out.device)
        self.step.topk(self.q_pre, self.q_rope, self.k_idx, self.k_cache, self.v_cache, self.Wq, self.seq_lens, k,
                       c.window, c.sink, self.out, stream)

    def results(self) -> Dict[str, np.ndarray]:
        torch.cuda.synchronize()
        c = self.case
        r = {"out": self.out.float().cpu().numpy()}
        if self.dbg is not None:
            for k in ("tau", "kstar", "kept_blocks", "smax", "Z"):
                r[k] = self.dbg[k].cpu().numpy().reshape(c.B, c.Hq)
            bm = self.dbg["block_bitmap"].cpu().numpy().view(np.uint32).reshape(c.B, c.Hq, self.words)
            bits = np.unpackbits(bm.view(np.uint8).reshape(c.B, c.Hq, self.words, 4), axis=-1, bitorder="little")
            r["kept"] = bits.reshape(c.B, c.Hq, self.words * 32)[:, :, :c.Ncap // 64]
        r["status"] = self.step.status()
        return r
