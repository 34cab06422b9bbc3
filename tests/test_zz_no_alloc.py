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


def test_misaligned_pointer_rejected_before_any_cuda_call():
    """A misaligned tensor is refused with RTP_ERR_UNSUPPORTED before the
    scratch lookup or any other CUDA call: on a machine without a GPU a CUDA
    call would return RTP_ERR_CUDA instead, so status 3 here shows that the
    refusal comes first and that nothing was enqueued."""
    HK = [1, 1, 0, 0]
    dims = rtp.make_dims(1, 4, 1, 4096)
    ok = 1 << 20
    args = [ok] * 7 + [rtp._head_kind_buf(HK), ok, 512, 4, ok, None, None]
    for i in (0, 1, 2, 3, 4, 5, 11):                 # q_pre .. Wq_idx, out
        bad = list(args)
        bad[i] = ok + 8
        assert rtp.lib.rtp_decode_step_noalloc(ctypes.byref(dims), *bad) == 3, i   # RTP_ERR_UNSUPPORTED


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


@pytest.mark.gpu
def test_noalloc_reports_device_input_error_then_recovers():
    """A length beyond the capacity is an error only the device sees: it must
    reach the caller's device_status (copied out of the shared array), and
    the next good call must find the array's status word cleared again and
    match rtp_decode_step."""
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from synth.torch_io import DeviceCase

    case = synth.make_case("noalloc-bad", B=2, Hkv=1, G=4, seq_lens=[300, 200], ret_groups=[0], p=[0.9, 0.9],
                           window=64, sink=4, seed=9, regimes=["gaussian", "gaussian"])
    dc = DeviceCase(case, debug=False)
    dc.run()
    torch.cuda.synchronize()
    assert dc.step.status() == 0
    ref = dc.out.float().cpu().numpy()
    dims = rtp.make_dims(case.B, case.Hq, case.Hkv, case.Ncap)
    stream = torch.cuda.current_stream()
    bad_lens = dc.seq_lens.clone()
    bad_lens[0] = case.Ncap + 64                      # made on the host side of the test, never read past
    for lens, want in ((bad_lens, 6), (dc.seq_lens, 0)):
        out = torch.zeros_like(dc.out)
        status = torch.full((1,), 0xFFFF, dtype=torch.int32, device=dc.out.device)
        rtp.decode_step_noalloc(dims, dc.q_pre, dc.q_rope, dc.k_idx, dc.k_cache, dc.v_cache, dc.Wq, lens,
                                case.head_kind, dc.p, case.window, case.sink, out, status, stream)
        torch.cuda.synchronize()
        assert int(status.item()) == want           # RTP_ERR_DEVICE_INPUT, then RTP_OK
    got = out.float().cpu().numpy()
    err = np.abs(got - ref)
    assert np.all(err <= ATOL + RTOL * np.abs(ref))
