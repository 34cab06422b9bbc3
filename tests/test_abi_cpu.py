"""The C-ABI library loads, exports what include/rtp_decode.h declares, and
rejects bad arguments on the host before touching the GPU.  CPU only."""
import ctypes
import os
import re

import pytest

import sparse_attention_decode_rtpurbo_b200 as rtp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rtp_decode.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rtp_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol():
    names = declared_functions()
    assert {"rtp_decode_step", "rtp_workspace_size", "rtp_get_status", "rtp_status_string"} <= set(names)
    for n in names:
        assert hasattr(rtp.lib, n), n


def dims(**kw):
    base = dict(batch=1, num_q_heads=8, num_kv_heads=2, max_seq_len=4096)
    base.update(kw)
    return rtp.make_dims(**base)


HK = [1, 1, 1, 1, 0, 0, 0, 0]


def test_workspace_size_valid_and_invalid():
    n = rtp.workspace_size(dims(), HK)
    assert n > 0 and n % 256 == 0
    assert rtp.workspace_size(dims(max_seq_len=8192), HK) > n          # grows with capacity
    assert rtp.workspace_size(dims(), [0] * 8) < n                     # no retrieval heads: no score scratch
    bad = dims()
    bad.head_dim = 64
    assert rtp.workspace_size(bad, HK) == 0
    assert rtp.workspace_size(dims(num_q_heads=6, num_kv_heads=2), [1] * 6) == 0    # GQA group 3 unsupported
    assert rtp.workspace_size(dims(num_q_heads=9, num_kv_heads=2), [1] * 9) == 0
    assert rtp.workspace_size(dims(max_seq_len=100), HK) == 0                       # not a multiple of 64
    assert rtp.workspace_size(dims(), [2] + HK[1:]) == 0                            # head_kind must be 0/1


def _call(d, window=64, sink=4, ptr=256, **nulls):
    args = {k: ptr for k in ("q_pre", "q_rope", "k_idx", "k_cache", "v_cache", "Wq", "seq_lens", "p", "out")}
    args.update(nulls)
    return rtp.lib.rtp_decode_step(ctypes.byref(d), args["q_pre"], args["q_rope"], args["k_idx"], args["k_cache"],
                                   args["v_cache"], args["Wq"], args["seq_lens"], rtp._head_kind_buf(HK), args["p"],
                                   window, sink, args["out"], None)


def test_host_side_errors_launch_nothing():
    d = dims()
    assert _call(d, q_pre=None) == 1                  # RTP_ERR_NULL
    assert _call(d, out=None) == 1
    assert _call(d, window=0, sink=0) == 2            # RTP_ERR_SHAPE: empty local set
    assert _call(d, window=-1) == 2
    assert _call(d) == 4                              # RTP_ERR_WORKSPACE: none given
    d2 = dims()
    d2.workspace = 4096
    d2.workspace_bytes = 16                           # too small
    assert _call(d2) == 4
    d3 = dims()
    d3.workspace = 4096 + 8                           # misaligned
    d3.workspace_bytes = 1 << 30
    assert _call(d3) == 4
    d4 = dims()
    d4.idx_dim = 32
    assert _call(d4) == 3                             # RTP_ERR_UNSUPPORTED


def _call_topk(d, topk, window=64, sink=4, ptr=256, **nulls):
    args = {k: ptr for k in ("q_pre", "q_rope", "k_idx", "k_cache", "v_cache", "Wq", "seq_lens", "out")}
    args.update(nulls)
    return rtp.lib.rtp_decode_step_topk(ctypes.byref(d), args["q_pre"], args["q_rope"], args["k_idx"],
                                        args["k_cache"], args["v_cache"], args["Wq"], args["seq_lens"],
                                        rtp._head_kind_buf(HK), topk, window, sink, args["out"], None)


def test_topk_host_side_checks():
    """rtp_decode_step_topk: k < 1 is refused; p is not an argument, so the
    remaining checks (nulls, local set, workspace) are rtp_decode_step's."""
    d = dims()
    assert _call_topk(d, 0) == 2                      # RTP_ERR_SHAPE: k must be >= 1
    assert _call_topk(d, -5) == 2
    assert _call_topk(d, 4096, q_pre=None) == 1       # RTP_ERR_NULL
    assert _call_topk(d, 4096, window=0, sink=0) == 2
    assert _call_topk(d, 4096) == 4                   # RTP_ERR_WORKSPACE: none given (the checks passed)
    assert _call_topk(d, 1 << 30) == 4                # any k >= 1 is valid (k >= L keeps every block)
    d4 = dims()
    d4.idx_dim = 32
    assert _call_topk(d4, 16) == 3
    assert _call(d, p=None) == 1                      # the top-p step still needs p


def test_paged_geometry_checks():
    d = dims(block_table=4096, max_blocks_per_seq=32, num_pages=10)   # 32*64 != 4096
    assert rtp.workspace_size(d, HK) == 0
    d = dims(block_table=4096, max_blocks_per_seq=64, num_pages=10)
    assert rtp.workspace_size(d, HK) > 0


def test_status_strings():
    for c in range(8):
        assert rtp.status_string(c)
    assert "unknown" in rtp.status_string(99)
    with pytest.raises(rtp.RtpError):
        rtp.decode_step(dims(), 1, 1, 1, 1, 1, 1, 1, HK, 1, 64, 4, 1)


def test_index_append_host_side_checks():
    """rtp_index_append: bad arguments are refused before any CUDA call."""
    fake = 4096   # never dereferenced: every call below returns first
    d = dims()
    call = lambda dd, *a: rtp.lib.rtp_index_append(ctypes.byref(dd) if dd is not None else None, *a)
    assert call(None, fake, fake, fake, 1, fake, None, None) == 1                      # NULL dims
    assert call(d, None, fake, fake, 1, fake, None, None) == 1                         # NULL k_pre
    assert call(d, fake, fake, fake, 0, fake, None, None) == 0                         # nothing to append
    assert call(d, fake, fake, fake, -1, fake, None, None) == 2                        # negative count
    assert call(d, fake, fake, fake, 4097, fake, None, None) == 2                      # more than the capacity
    assert call(dims(max_seq_len=100), fake, fake, fake, 1, fake, None, None) == 2     # capacity not a multiple of 64
    assert call(d, fake + 2, fake, fake, 1, fake, None, None) == 3                     # k_pre not 16-byte aligned
    assert call(d, fake, fake, fake, 1, fake + 4, None, None) == 3                     # k_idx not 8-byte aligned
    assert call(dims(num_kv_heads=65, num_q_heads=65), fake, fake, fake, 1, fake, None, None) == 3


def test_ring_host_side_checks():
    """rtp_decode_step_ring: ring sizes are checked before any CUDA call."""
    fake = 4096

    def call(d, W=128, window=64, sink=4, kr=fake, vr=fake, p=fake):
        return rtp.lib.rtp_decode_step_ring(ctypes.byref(d), fake, fake, fake, fake, fake, kr, vr, W, fake, fake,
                                            rtp._head_kind_buf(HK), p, window, sink, fake, None)

    d = dims()
    assert call(d, kr=None) == 1
    assert call(d, vr=None) == 1
    assert call(d, p=None) == 1
    assert call(d, W=96) == 2                        # not a multiple of 64
    assert call(d, W=64, window=65) == 2             # the window does not fit
    assert call(d, W=0, window=0) == 2
    assert call(d, sink=65) == 2                     # the sink must fit the 64 head rows
    assert call(d, kr=fake + 8) == 3
    assert call(d) == 4                              # checks passed; no workspace given


def test_ring_write_host_side_checks():
    fake = 4096

    def call(d, n=1, W=128, kn=fake, vn=fake, kr=fake, vr=fake, pos=fake):
        return rtp.lib.rtp_ring_write(ctypes.byref(d) if d is not None else None, kn, vn, pos, n, W, kr, vr, None,
                                      None)

    d = dims()
    assert call(None) == 1
    assert call(d, n=0) == 0                         # nothing to write
    assert call(d, n=-1) == 2
    assert call(d, W=96) == 2
    assert call(d, W=0) == 2
    assert call(d, kr=None) == 1
    assert call(d, pos=None) == 1
    assert call(d, vn=fake + 4) == 3


def test_kv_append_host_side_checks():
    """rtp_kv_append: bad arguments are refused before any CUDA call."""
    fake = 4096   # never dereferenced: every call below returns first
    d = dims()

    def call(dd, k_pre=fake, v_new=fake, wk=fake, cs=fake, sn=fake, pos=fake, n=1, kidx=fake, kc=fake, vc=fake):
        return rtp.lib.rtp_kv_append(ctypes.byref(dd) if dd is not None else None, k_pre, v_new, wk, cs, sn, pos, n,
                                     kidx, kc, vc, None, None)

    assert call(None) == 1                           # NULL dims
    assert call(d, kc=None) == 1                     # NULL key cache
    assert call(d, vc=None) == 1                     # NULL value cache
    assert call(d, v_new=None) == 1                  # NULL new values
    assert call(d, cs=None) == 1                     # NULL angle table
    assert call(d, n=0) == 0                         # nothing to append
    assert call(d, n=-1) == 2
    assert call(d, n=4097) == 2                      # more than the capacity
    assert call(d, v_new=fake + 8) == 3              # 16-byte alignment of every row-wise operand
    assert call(d, sn=fake + 4) == 3
    assert call(d, kc=fake + 2) == 3
    assert call(d, vc=fake + 8) == 3
    assert call(d, kidx=fake + 4) == 3               # k_idx: 8-byte aligned, as rtp_index_append
    bad = dims()
    bad.head_dim = 64
    assert call(bad) == 3


def test_prefill_host_side_checks():
    """rtp_prefill: bad arguments are refused before any CUDA call."""
    fake = 4096   # never dereferenced: every call below returns first
    d = dims()
    HK = rtp._head_kind_buf([1, 0, 0, 1, 1, 0, 0, 1][:d.num_q_heads] + [0] * max(0, d.num_q_heads - 8))

    def call(dd, q=fake, kc=fake, vc=fake, hk=HK, pos=fake, n=16, window=64, sink=4, out=fake):
        return rtp.lib.rtp_prefill(ctypes.byref(dd) if dd is not None else None, q, kc, vc, hk, pos, n, window,
                                   sink, out, None, None)

    assert call(None) == 1                           # NULL dims
    assert call(d, hk=None) == 1                     # NULL head split
    assert call(d, q=None) == 1
    assert call(d, kc=None) == 1
    assert call(d, pos=None) == 1
    assert call(d, out=None) == 1
    assert call(d, n=0) == 0                         # no queries: nothing to do
    assert call(d, n=-1) == 2
    assert call(d, n=d.max_seq_len + 1) == 2         # more queries than the capacity
    assert call(d, window=0, sink=0) == 2            # local heads would attend to nothing
    assert call(d, window=-1) == 2
    assert call(d, q=fake + 8) == 3                  # 16-byte alignment
    assert call(d, vc=fake + 2) == 3
    assert call(d, out=fake + 4) == 3
    bad = dims()
    bad.head_dim = 64
    assert call(bad) == 3
    bad = dims()
    bad.num_kv_heads = 3                             # Hq % Hkv != 0
    assert call(bad) == 2


def test_binding_refuses_host_and_strided_tensors():
    """The binding passes tensors by address: a host tensor or a strided view
    is refused before the library is called."""
    import torch

    with pytest.raises(ValueError, match="device memory"):
        rtp.decode_step(dims(), torch.zeros(8), 1, 1, 1, 1, 1, 1, HK, 1, 64, 4, 1)
    with pytest.raises(ValueError, match="contiguous"):
        rtp.decode_step(dims(), torch.zeros(8, 8).t(), 1, 1, 1, 1, 1, 1, HK, 1, 64, 4, 1)
