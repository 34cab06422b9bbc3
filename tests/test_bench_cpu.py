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


def test_algorithmic_bytes_by_hand():
    """The roofline numerator on hand-countable cases: index rows per
    retrieval group, the union of the group's kept blocks (the last block
    partial), sink/window rows per local group, and a group with both kinds
    counting the rows it reads once."""
    import numpy as np

    import bench
    import synth

    # two KV groups of 2 heads: group 0 retrieval, group 1 local; L = 200 (4 blocks, last 8 rows)
    case = synth.make_case("bytes", B=1, Hkv=2, G=2, seq_lens=[200], ret_groups=[0], p=[0.9], window=50, sink=4,
                           seed=1, regimes=["gaussian"])
    kept = np.zeros((1, 4, case.Ncap // 64), np.uint8)
    kept[0, 0, [0, 3]] = 1                   # head 0: blocks 0 and 3 (64 + 8 rows)
    kept[0, 1, [3]] = 1                      # head 1: block 3 again (union)
    got = bench.algorithmic_bytes(case, kept)
    assert got["index"] == 200 * 32
    assert got["kept_kv"] == (64 + 8) * 512
    assert got["local"] == (4 + 50) * 512     # sink 0..3 and window 150..199
    assert got["shared"] == 0
    assert got["total"] == got["index"] + got["kept_kv"] + got["local"]

    # one KV group with both kinds: heads 0 (retrieval) and 1 (local)
    hk = np.array([1, 0], np.uint8)
    case = synth.make_case("bytes-mixed", B=1, Hkv=1, G=2, seq_lens=[200], ret_groups=[], head_kind=hk, p=[0.9],
                           window=50, sink=4, seed=2, regimes=["gaussian"])
    kept = np.zeros((1, 2, case.Ncap // 64), np.uint8)
    kept[0, 0, [0, 2]] = 1                   # blocks 0 (rows 0..63) and 2 (rows 128..191)
    got = bench.algorithmic_bytes(case, kept)
    # local rows: sink 0..3 (in block 0), window 150..191 (in block 2), 192..199 (in no kept block)
    assert got["kept_kv"] == 128 * 512
    assert got["local"] == (4 + 50) * 512
    assert got["shared"] == (4 + 42) * 512
    assert got["total"] == got["index"] + (128 + 8) * 512
