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


def test_binding_refuses_host_and_strided_tensors():
    """The binding passes tensors by address: a host tensor or a strided view
    is refused before the library is called."""
    import torch

    with pytest.raises(ValueError, match="device memory"):
        rtp.decode_step(dims(), torch.zeros(8), 1, 1, 1, 1, 1, 1, HK, 1, 64, 4, 1)
    with pytest.raises(ValueError, match="contiguous"):
        rtp.decode_step(dims(), torch.zeros(8, 8).t(), 1, 1, 1, 1, 1, 1, HK, 1, 64, 4, 1)
