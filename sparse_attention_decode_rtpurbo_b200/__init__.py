"""RTPurbo decode-step sparse attention on B200 (sm_100a).

Thin ctypes binding of ``librtp.so`` (C ABI declared in
``include/rtp_decode.h``).  This module only marshals arguments: every step of
the decode path runs in the library's CUDA kernels.  PyTorch supplies device
memory and streams.  There is no CPU fallback: if the library cannot be
loaded, importing this package raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

from .build import LIB as _BUILT_LIB

# RTP_LIBRARY=<path>: load another build of the library (a comparison build,
# e.g. the one whose attention tiles run on the FMA pipe); default: the
# package's librtp.so
_LIB_PATH = os.environ.get("RTP_LIBRARY") or _BUILT_LIB

__all__ = ["RTP_OK", "RtpError", "RtpDims", "RtpDebug", "lib", "status_string", "workspace_size", "decode_step",
           "get_status", "Step", "PHASES", "TIMING_EVENTS", "decode_step_noalloc", "NOALLOC_SCRATCH_BYTES",
           "prefill"]

RTP_OK = 0
_STATUS_NAMES = {0: "RTP_OK", 1: "RTP_ERR_NULL", 2: "RTP_ERR_SHAPE", 3: "RTP_ERR_UNSUPPORTED", 4: "RTP_ERR_WORKSPACE",
                 5: "RTP_ERR_CUDA", 6: "RTP_ERR_DEVICE_INPUT", 7: "RTP_ERR_TIMEOUT",
                 8: "RTP_ERR_SCRATCH_LIMIT"}


class RtpError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{_STATUS_NAMES.get(code, code)}: {status_string(code)}{' (' + what + ')' if what else ''}")


class RtpDebug(ctypes.Structure):
    _fields_ = [("tau", ctypes.c_void_p), ("kstar", ctypes.c_void_p), ("kept_blocks", ctypes.c_void_p),
                ("smax", ctypes.c_void_p), ("Z", ctypes.c_void_p), ("block_bitmap", ctypes.c_void_p),
                ("trace", ctypes.c_void_p)]


TRACE_EVENTS = ["start", "select_done", "local_done", "lists_ready", "retrieval_done", "end", "select_start",
                "stream_work_start", "unused_8", "unused_9", "unused_10", "unused_11", "select_units_done",
                "ret_kernel_start", "select_bins_done", "attn_start"]
# debug sums (slots 16..): SM cycles of one thread per CTA by category, counts,
# and the latest %globaltimer of two events
TRACE_SUMS = ["a_cyc_wait", "a_cyc_score", "a_cyc_attn", "a_n_score", "a_n_attn", "a_cyc_score_begin",
              "a_first_data", "a_consumers_done", "unused_24", "unused_25", "unused_26",
              "unused_27", "a_cyc_score_end", "a_cyc_local_begin", "a_cyc_local_end", "b_cyc_grid_sync",
              "b_attn_wait", "b_attn_tile", "b_attn_end", "b_n_attn", "b_prod_wait", "b_cyc_sel_bins",
              "b_cyc_sel_units", "b_cyc_sel_finish", "unused_40", "t_unused_41", "t_unused_42", "t_decide_reduced",
              "t_decide_modes", "t_unused_45", "t_split_ticketed", "t_split_reduced"]
# TRACE_SUMS entries that are %globaltimer maxima (events), not cycle sums
TRACE_SUM_EVENTS = ("a_first_data", "a_consumers_done") + tuple(n for n in TRACE_SUMS if n.startswith("t_"))
TRACE_WORDS = 48


class RtpDims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("idx_dim", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("max_seq_len", ctypes.c_int32), ("block_table", ctypes.c_void_p),
                ("max_blocks_per_seq", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("debug", ctypes.POINTER(RtpDebug)), ("timing_events", ctypes.c_void_p),
                ("n_timing_events", ctypes.c_int32)]


PHASES = ["stream", "retrieve"]
TIMING_EVENTS = len(PHASES) + 1


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"librtp.so not built ({_LIB_PATH}); run `python -m sparse_attention_decode_rtpurbo_b200.build`")
    L = ctypes.CDLL(_LIB_PATH)
    vp, i32 = ctypes.c_void_p, ctypes.c_int32
    L.rtp_workspace_size.argtypes = [ctypes.POINTER(RtpDims), vp]
    L.rtp_workspace_size.restype = ctypes.c_size_t
    L.rtp_decode_step.argtypes = [ctypes.POINTER(RtpDims), vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, vp, vp]
    L.rtp_decode_step.restype = ctypes.c_int
    L.rtp_decode_step_topk.argtypes = [ctypes.POINTER(RtpDims), vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, vp, vp]
    L.rtp_decode_step_topk.restype = ctypes.c_int
    L.rtp_decode_step_ring.argtypes = [ctypes.POINTER(RtpDims), vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, i32,
                                       i32, vp, vp]
    L.rtp_decode_step_ring.restype = ctypes.c_int
    L.rtp_ring_write.argtypes = [ctypes.POINTER(RtpDims), vp, vp, vp, i32, i32, vp, vp, vp, vp]
    L.rtp_ring_write.restype = ctypes.c_int
    L.rtp_decode_step_noalloc.argtypes = [ctypes.POINTER(RtpDims), vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, vp,
                                          vp, vp]
    L.rtp_decode_step_noalloc.restype = ctypes.c_int
    L.rtp_get_status.argtypes = [ctypes.POINTER(RtpDims), vp]
    L.rtp_index_append.argtypes = [ctypes.POINTER(RtpDims), vp, vp, vp, i32, vp, vp, vp]
    L.rtp_index_append.restype = ctypes.c_int
    L.rtp_kv_append.argtypes = [ctypes.POINTER(RtpDims), vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp]
    L.rtp_kv_append.restype = ctypes.c_int
    L.rtp_get_status.restype = ctypes.c_int
    L.rtp_prefill.argtypes = [ctypes.POINTER(RtpDims), vp, vp, vp, vp, vp, i32, i32, i32, vp, vp, vp]
    L.rtp_prefill.restype = ctypes.c_int
    L.rtp_status_string.argtypes = [ctypes.c_int]
    L.rtp_status_string.restype = ctypes.c_char_p
    return L


lib = _load()


def status_string(code: int) -> str:
    return lib.rtp_status_string(int(code)).decode()


def _ptr(x) -> Optional[int]:
    """The device address of an argument: None, a raw address (int), or a
    tensor, which must be contiguous and in device memory (the library reads
    it as a dense array at that address)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "is_contiguous"):
        if not x.is_contiguous():
            raise ValueError("rtp: tensor arguments must be contiguous")
        if not getattr(x, "is_cuda", False):
            raise ValueError("rtp: tensor arguments must be in device memory")
    return x.data_ptr()


def make_dims(batch: int, num_q_heads: int, num_kv_heads: int, max_seq_len: int, *, block_table=None,
              max_blocks_per_seq: int = 0, num_pages: int = 0, workspace=None, workspace_bytes: int = 0,
              debug: Optional[RtpDebug] = None) -> RtpDims:
    d = RtpDims(batch, num_q_heads, num_kv_heads, 128, 16, 64, max_seq_len, _ptr(block_table), max_blocks_per_seq,
                num_pages, _ptr(workspace), workspace_bytes, None)
    if debug is not None:
        d.debug = ctypes.pointer(debug)
    return d


def _head_kind_buf(head_kind) -> ctypes.Array:
    hk = bytes(int(x) for x in head_kind)
    return (ctypes.c_uint8 * len(hk)).from_buffer_copy(hk)


def workspace_size(dims: RtpDims, head_kind) -> int:
    return int(lib.rtp_workspace_size(ctypes.byref(dims), _head_kind_buf(head_kind)))


def decode_step(dims: RtpDims, q_pre, q_rope, k_idx, k_cache, v_cache, Wq_idx, seq_lens, head_kind, p,
                window: int, sink: int, out, stream=None) -> None:
    """rtp_decode_step: tensors are device tensors (bf16 / int32 / fp32), or
    raw device pointers as ints; head_kind is a host sequence of 0/1."""
    st = 0 if stream is None else (stream if isinstance(stream, int) else stream.cuda_stream)
    rc = lib.rtp_decode_step(ctypes.byref(dims), _ptr(q_pre), _ptr(q_rope), _ptr(k_idx), _ptr(k_cache),
                             _ptr(v_cache), _ptr(Wq_idx), _ptr(seq_lens), _head_kind_buf(head_kind), _ptr(p),
                             int(window), int(sink), _ptr(out), st)
    if rc != RTP_OK:
        raise RtpError(rc, "rtp_decode_step")


def decode_step_ring(dims: RtpDims, q_pre, q_rope, k_idx, k_cache, v_cache, k_ring, v_ring, ring_W: int, Wq_idx,
                     seq_lens, head_kind, p, window: int, sink: int, out, stream=None) -> None:
    """rtp_decode_step_ring: the decode step with the local-only KV heads'
    keys and values read from rings [B, Hkv, 64 + ring_W, 128] (block 0 in
    rows 0..63, position n >= 64 in row 64 + n % ring_W)."""
    st = 0 if stream is None else (stream if isinstance(stream, int) else stream.cuda_stream)
    rc = lib.rtp_decode_step_ring(ctypes.byref(dims), _ptr(q_pre), _ptr(q_rope), _ptr(k_idx), _ptr(k_cache),
                                  _ptr(v_cache), _ptr(k_ring), _ptr(v_ring), int(ring_W), _ptr(Wq_idx), _ptr(seq_lens),
                                  _head_kind_buf(head_kind), _ptr(p), int(window), int(sink), _ptr(out), st)
    if rc != RTP_OK:
        raise RtpError(rc, "rtp_decode_step_ring")


def ring_write(dims: RtpDims, k_new, v_new, pos, num_new: int, ring_W: int, k_ring, v_ring, device_status=None,
               stream=None) -> None:
    """rtp_ring_write: the new key and value rows of every sequence into the
    local heads' rings [B, Hkv, 64 + ring_W, 128], as if written in order."""
    st = 0 if stream is None else (stream if isinstance(stream, int) else stream.cuda_stream)
    rc = lib.rtp_ring_write(ctypes.byref(dims), _ptr(k_new), _ptr(v_new), _ptr(pos), int(num_new), int(ring_W),
                            _ptr(k_ring), _ptr(v_ring), _ptr(device_status), st)
    if rc != RTP_OK:
        raise RtpError(rc, "rtp_ring_write")


def decode_step_topk(dims: RtpDims, q_pre, q_rope, k_idx, k_cache, v_cache, Wq_idx, seq_lens, head_kind, topk: int,
                     window: int, sink: int, out, stream=None) -> None:
    """rtp_decode_step_topk: the decode step with every retrieval head keeping
    its static top-k tokens (topk >= 1) instead of the dynamic top-p set."""
    st = 0 if stream is None else (stream if isinstance(stream, int) else stream.cuda_stream)
    rc = lib.rtp_decode_step_topk(ctypes.byref(dims), _ptr(q_pre), _ptr(q_rope), _ptr(k_idx), _ptr(k_cache),
                                  _ptr(v_cache), _ptr(Wq_idx), _ptr(seq_lens), _head_kind_buf(head_kind), int(topk),
                                  int(window), int(sink), _ptr(out), st)
    if rc != RTP_OK:
        raise RtpError(rc, "rtp_decode_step_topk")


# RTP_NOALLOC_SCRATCH_BYTES of the C header: the static scratch of rtp_decode_step_noalloc
NOALLOC_SCRATCH_BYTES = 64 << 20


def decode_step_noalloc(dims: RtpDims, q_pre, q_rope, k_idx, k_cache, v_cache, Wq_idx, seq_lens, head_kind, p,
                        window: int, sink: int, out, device_status=None, stream=None) -> None:
    """rtp_decode_step_noalloc: the decode step for callers that must not
    allocate device memory (an engine plugin whose pool owns the GPU's memory,
    a loop that cannot take cudaMalloc's synchronisation).  The library uses
    its own static scratch array; dims.workspace is ignored.  device_status is
    an optional device uint32 tensor that receives the call's device-side
    status.  Calls that overlap on the GPU race on the shared scratch."""
    st = 0 if stream is None else (stream if isinstance(stream, int) else stream.cuda_stream)
    rc = lib.rtp_decode_step_noalloc(ctypes.byref(dims), _ptr(q_pre), _ptr(q_rope), _ptr(k_idx), _ptr(k_cache),
                                     _ptr(v_cache), _ptr(Wq_idx), _ptr(seq_lens), _head_kind_buf(head_kind), _ptr(p),
                                     int(window), int(sink), _ptr(out), _ptr(device_status), st)
    if rc != RTP_OK:
        raise RtpError(rc, "rtp_decode_step_noalloc")


def index_append(dims: RtpDims, k_pre, Wk_idx, pos, num_new: int, k_idx, device_status=None, stream=None) -> None:
    """rtp_index_append: rows pos[b] + t of the index cache k_idx receive
    bf16(W^K[g] . k_pre[b, g, t]) for the num_new new tokens of every sequence
    (dims gives the cache geometry).  device_status: optional device uint32
    tensor set to RTP_ERR_DEVICE_INPUT by a row or page id out of range."""
    st = 0 if stream is None else (stream if isinstance(stream, int) else stream.cuda_stream)
    rc = lib.rtp_index_append(ctypes.byref(dims), _ptr(k_pre), _ptr(Wk_idx), _ptr(pos), int(num_new), _ptr(k_idx),
                              _ptr(device_status), st)
    if rc != RTP_OK:
        raise RtpError(rc, "rtp_index_append")


def kv_append(dims: RtpDims, k_pre, v_new, Wk_idx, rope_cos, rope_sin, pos, num_new: int, k_idx, k_cache, v_cache,
              device_status=None, stream=None) -> None:
    """rtp_kv_append: for the num_new new tokens of every sequence, cache rows
    n = pos[b] + t receive k_idx = bf16(W^K[g] . k_pre), k_cache =
    bf16(RoPE_n(k_pre)) with the angle table rows rope_cos[n], rope_sin[n]
    (fp32 [max_seq_len, 64]), and v_cache = v_new."""
    st = 0 if stream is None else (stream if isinstance(stream, int) else stream.cuda_stream)
    rc = lib.rtp_kv_append(ctypes.byref(dims), _ptr(k_pre), _ptr(v_new), _ptr(Wk_idx), _ptr(rope_cos), _ptr(rope_sin),
                           _ptr(pos), int(num_new), _ptr(k_idx), _ptr(k_cache), _ptr(v_cache), _ptr(device_status), st)
    if rc != RTP_OK:
        raise RtpError(rc, "rtp_kv_append")


def prefill(dims: RtpDims, q, k_cache, v_cache, head_kind, pos, num_q: int, window: int, sink: int, out,
            device_status=None, stream=None) -> None:
    """rtp_prefill: causal attention of num_q queries per sequence (q [B, Hq,
    num_q, 128] bf16, RoPE'd) at positions pos[b] + t over the caches:
    retrieval heads densely, local heads over their sink and window; out [B,
    Hq, num_q, 128] bf16.  head_kind is a host sequence of 0/1."""
    st = 0 if stream is None else (stream if isinstance(stream, int) else stream.cuda_stream)
    rc = lib.rtp_prefill(ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(v_cache), _head_kind_buf(head_kind),
                         _ptr(pos), int(num_q), int(window), int(sink), _ptr(out), _ptr(device_status), st)
    if rc != RTP_OK:
        raise RtpError(rc, "rtp_prefill")


def get_status(dims: RtpDims, stream=None) -> int:
    st = 0 if stream is None else (stream if isinstance(stream, int) else stream.cuda_stream)
    return int(lib.rtp_get_status(ctypes.byref(dims), st))


class Step:
    """Convenience holder for one layer's decode-step configuration: owns the
    workspace (a torch uint8 device tensor, zero-filled once) and the dims."""

    def __init__(self, batch: int, num_q_heads: int, num_kv_heads: int, max_seq_len: int, head_kind, *,
                 block_table=None, num_pages: int = 0, device="cuda", debug: Optional[RtpDebug] = None):
        import torch

        self.head_kind = [int(x) for x in head_kind]
        mbps = 0 if block_table is None else int(block_table.shape[1])
        self.block_table = block_table
        probe = make_dims(batch, num_q_heads, num_kv_heads, max_seq_len, block_table=block_table,
                          max_blocks_per_seq=mbps, num_pages=num_pages)
        nbytes = workspace_size(probe, self.head_kind)
        if nbytes == 0:
            raise RtpError(2, "rtp_workspace_size returned 0 (invalid or unsupported sizes)")
        self.workspace = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        self.debug = debug
        self.dims = make_dims(batch, num_q_heads, num_kv_heads, max_seq_len, block_table=block_table,
                              max_blocks_per_seq=mbps, num_pages=num_pages, workspace=self.workspace,
                              workspace_bytes=nbytes, debug=debug)

    def __call__(self, q_pre, q_rope, k_idx, k_cache, v_cache, Wq_idx, seq_lens, p, window, sink, out, stream=None):
        decode_step(self.dims, q_pre, q_rope, k_idx, k_cache, v_cache, Wq_idx, seq_lens, self.head_kind, p, window,
                    sink, out, stream)

    def ring(self, q_pre, q_rope, k_idx, k_cache, v_cache, k_ring, v_ring, ring_W, Wq_idx, seq_lens, p, window, sink,
             out, stream=None):
        decode_step_ring(self.dims, q_pre, q_rope, k_idx, k_cache, v_cache, k_ring, v_ring, ring_W, Wq_idx, seq_lens,
                         self.head_kind, p, window, sink, out, stream)

    def topk(self, q_pre, q_rope, k_idx, k_cache, v_cache, Wq_idx, seq_lens, topk, window, sink, out, stream=None):
        decode_step_topk(self.dims, q_pre, q_rope, k_idx, k_cache, v_cache, Wq_idx, seq_lens, self.head_kind, topk,
                         window, sink, out, stream)

    def status(self, stream=None) -> int:
        return get_status(self.dims, stream)

    def set_timing_events(self, events) -> None:
        """Record the given torch.cuda.Event objects (TIMING_EVENTS of them,
        created with enable_timing=True) at the phase boundaries of every
        following call; None switches it off."""
        if events is None:
            self._ev_arr = None
            self.dims.timing_events = None
            self.dims.n_timing_events = 0
            return
        assert len(events) >= TIMING_EVENTS
        for e in events:
            if not e.cuda_event:
                e.record()      # materialise the underlying cudaEvent_t
        torch_handles = [e.cuda_event for e in events]
        self._ev_arr = (ctypes.c_void_p * len(torch_handles))(*torch_handles)
        self.dims.timing_events = ctypes.cast(self._ev_arr, ctypes.c_void_p)
        self.dims.n_timing_events = len(torch_handles)
