"""bench.py's host-side rules that need no GPU."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_profiled_traffic_only_for_the_profiled_sources_and_workload(monkeypatch):
    """roofline.traffic is quoted from a committed ncu summary only while the
    profiled kernels' sources hash to the recorded value and the bench runs
    the profiled workload; otherwise it is null."""
    text = open(os.path.join(ROOT, bench.PROFILED["stream"][0])).read()
    rec = dict(line.split(":", 1) for line in text.splitlines()
               if line.startswith(("traffic_bytes_per_launch:", "source_sha256_16:")))
    want = int(rec["traffic_bytes_per_launch"])
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: rec["source_sha256_16"].strip())
    assert bench.profiled_traffic("stream", "w4-1m") == want
    assert bench.profiled_traffic("stream", "w3-4x128k") is None          # another workload
    assert bench.profiled_traffic("append", "w4-1m") is None              # no summary for it
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.profiled_traffic("stream", "w4-1m") is None              # sources changed since the capture


def test_kernel_source_hash_is_stable_and_short():
    h = bench.kernel_source_hash()
    assert h == bench.kernel_source_hash() and len(h) == 16 and int(h, 16) >= 0


def test_stage_inputs_views_and_one_copy():
    """The staged inputs: views with the tensors' shapes, dtypes and values at
    256-byte aligned offsets; one copy of the host buffer reproduces them."""
    import numpy as np
    import torch

    import bench

    q = np.arange(2 * 3 * 128, dtype=np.float64).reshape(2, 3, 128) / 7.0
    q_bits = np.asarray(torch.from_numpy(q).to(torch.bfloat16).view(torch.int16).numpy()).view(np.uint16)
    lens = np.array([5, 9], np.int32)
    p = np.array([0.9, 0.5], np.float32)
    tensors = [torch.from_numpy(q_bits.view(np.int16)).view(torch.bfloat16), torch.from_numpy(lens.copy()),
               torch.from_numpy(p.copy())]
    dbuf, hbuf, views = bench.stage_inputs(tensors, [q_bits, lens, p], "cpu", pin=False)
    for t, v in zip(tensors, views):
        assert v.dtype == t.dtype and v.shape == t.shape and torch.equal(v.view(torch.uint8), t.view(torch.uint8))
        assert (v.data_ptr() - dbuf.data_ptr()) % 256 == 0
    for v in views:
        v.zero_()
    dbuf.copy_(hbuf)
    for t, v in zip(tensors, views):
        assert torch.equal(v.view(torch.uint8), t.view(torch.uint8))
