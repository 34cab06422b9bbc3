"""The allocation-free entry point, rtp_decode_step_noalloc.

Some callers cannot allocate device memory for a workspace: a plugin running
inside an inference engine whose memory pool owns the whole GPU, or a hot loop
that cannot afford cudaMalloc's device-wide synchronisation.  For them the
library keeps the step's scratch in a static device array of
RTP_NOALLOC_SCRATCH_BYTES.  These tests check that its output matches the
workspace entry point, rtp_decode_step, within the parity tolerance on two
calls in a row (the second call finds the first one's scratch contents, and
the second case finds the first case's, laid out for other sizes), and that
sizes beyond the array are refused on the host.

The file name makes pytest collect it after every other test file.
"""
import ctypes

import numpy as np
import pytest

import synth
import sparse_attention_decode_rtpurbo_b200 as rtp
from tests.parity import ATOL, RTOL


def test_oversize_and_null_rejected_on_host():
    """Refused before any CUDA call, so this runs without a GPU too."""
    HK = [1] * 128
    fake = 4096                        # never dereferenced: the call returns first
    args = [fake] * 7 + [rtp._head_kind_buf(HK), fake, 64, 4, fake, None, None]
    big = rtp.make_dims(256, 128, 16, 8192)          # 256 x 128 retrieval heads of selection state
    assert rtp.workspace_size(big, HK) > rtp.NOALLOC_SCRATCH_BYTES
    rc = rtp.lib.rtp_decode_step_noalloc(ctypes.byref(big), *args)
    assert rc == 8, rtp.status_string(rc)             # RTP_ERR_SCRATCH_LIMIT
    assert "static array" in rtp.status_string(8)
    small = rtp.make_dims(1, 128, 16, 4096)
    assert 0 < rtp.workspace_size(small, HK) <= rtp.NOALLOC_SCRATCH_BYTES
    bad = list(args)
    bad[0] = None                                     # q_pre
    assert rtp.lib.rtp_decode_step_noalloc(ctypes.byref(small), *bad) == 1   # RTP_ERR_NULL


@pytest.mark.gpu
@pytest.mark.parametrize("w,scale", [(1, 1), (5, 32)])
def test_noalloc_matches_workspace_entry_point(w, scale):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from synth.torch_io import DeviceCase

    case = synth.workload(w, scale=scale)
    dc = DeviceCase(case, debug=False)
    dc.run()                                          # rtp_decode_step with its own workspace
    torch.cuda.synchronize()
    assert dc.step.status() == 0
    ref = dc.out.float().cpu().numpy()

    mbps = 0 if dc.block_table is None else int(dc.block_table.shape[1])
    dims = rtp.make_dims(case.B, case.Hq, case.Hkv, case.Ncap, block_table=dc.block_table,
                         max_blocks_per_seq=mbps, num_pages=case.num_pages)      # no workspace given
    stream = torch.cuda.current_stream()
    for call in range(2):
        out = torch.full_like(dc.out, float("nan"))
        status = torch.full((1,), 0xFFFF, dtype=torch.int32, device=dc.out.device)
        rtp.decode_step_noalloc(dims, dc.q_pre, dc.q_rope, dc.k_idx, dc.k_cache, dc.v_cache, dc.Wq, dc.seq_lens,
                                case.head_kind, dc.p, case.window, case.sink, out, status, stream)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}: device status {int(status.item())}"
        got = out.float().cpu().numpy()
        assert np.all(np.isfinite(got)), f"call {call}: non-finite output"
        err = np.abs(got - ref)
        lim = ATOL + RTOL * np.abs(ref)
        assert np.all(err <= lim), f"call {call}: max excess {float(np.max(err - lim)):.3g}"
