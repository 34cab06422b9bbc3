"""GPU parity of the decode step with the local heads' ring cache
(rtp_decode_step_ring) against the fp64 oracle.  The rings are written by
the oracle's ring writer from the workload's caches; on the device, every
full-cache row of the KV heads that serve no retrieval head is NaN, and so is
every ring row never written, so a read from the wrong place shows up as a
non-finite output."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

from synth.torch_io import DeviceCase  # noqa: E402
from tests.parity import compare  # noqa: E402

S0 = 64


def _rows(cache, case, b, g, n0, n1):
    """Rows n0 .. n1-1 of (b, g) from a contiguous or paged cache."""
    if case.block_table is None:
        return cache[b, g, n0:n1]
    n = np.arange(n0, n1)
    return cache[case.block_table[b, n // 64], g, n % 64]


def _rings(case, W):
    """Rings of every (b, g) after writing positions 0 .. L_b - 1 in order
    (unwritten rows: NaN)."""
    nan = synth.nan_fill((case.B, case.Hkv, S0 + W, 128))
    kr, vr = nan.copy(), nan.copy()
    for b in range(case.B):
        L = int(case.seq_lens[b])
        for start in range(0, L, 4096):
            T = min(4096, L - start)
            kn = np.stack([_rows(case.k_cache, case, b, g, start, start + T) for g in range(case.Hkv)])[None]
            vn = np.stack([_rows(case.v_cache, case, b, g, start, start + T) for g in range(case.Hkv)])[None]
            kb, vb = oracle.ring_write(kn, vn, np.array([start], np.int32), kr[b:b + 1], vr[b:b + 1], S0, W)
            kr[b], vr[b] = kb[0], vb[0]
    return kr, vr


def _local_only_groups(case):
    G = case.Hq // case.Hkv
    return [g for g in range(case.Hkv) if not any(case.head_kind[g * G:(g + 1) * G])]


def run_ring(case, W):
    dc = DeviceCase(case)
    kr, vr = _rings(case, W)
    dc.attach_ring(kr, vr, W)
    for g in _local_only_groups(case):
        dc.k_cache[:, g] = float("nan")
        dc.v_cache[:, g] = float("nan")
    dc.run()
    gpu = dc.results()
    ref = oracle.decode_step(case)
    fails, _ = compare(case, gpu, ref)
    return fails


@pytest.mark.parametrize("w,scale,W", [(2, 1, 2048), (2, 1, 4096), (2, 8, 2048), (5, 32, 2048), (3, 32, 4096),
                                       (1, 1, 512)])
def test_ring_workloads(w, scale, W):
    case = synth.workload(w, scale=scale)
    assert run_ring(case, W) == []


@pytest.mark.parametrize("L", [1, 5, 63, 64, 65, 127, 640, 641, 704, 5000])
def test_ring_lengths(L):
    """Lengths inside the head rows, at the block edges, one window past the
    head rows, and many windows long (the oldest and newest window blocks
    then share ring slots)."""
    case = synth.make_case(f"ring-{L}", B=2, Hkv=4, G=2, seq_lens=[L, max(1, L // 2 + 3)], ret_groups=[0],
                           p=[0.9, 0.9], window=576, sink=4, seed=300 + L, regimes=["gaussian", "gaussian"])
    assert run_ring(case, 576) == []


@pytest.mark.parametrize("window,sink,W", [(64, 64, 64), (1, 0, 64), (0, 4, 64), (100, 4, 128), (128, 1, 128)])
def test_ring_windows(window, sink, W):
    case = synth.make_case("ring-w", B=1, Hkv=2, G=4, seq_lens=[3333], ret_groups=[], p=[0.9], window=window,
                           sink=sink, seed=31, regimes=["gaussian"], paged=True)
    assert run_ring(case, W) == []


@pytest.mark.parametrize("B,Hkv,T,W,starts", [(2, 3, 1, 64, [0, 63]), (2, 2, 37, 128, [60, 500]),
                                              (1, 2, 300, 64, [10]), (3, 1, 700, 256, [0, 64, 1000])])
def test_ring_write_bit_exact(B, Hkv, T, W, starts):
    """rtp_ring_write against the oracle's in-order writes: chunks that cross
    the head rows, wrap the window rows several times (T > W: only each
    row's last token lands), and untouched rows."""
    import sparse_attention_decode_rtpurbo_b200 as rtp

    rng = np.random.default_rng(T + W)
    k_new = synth.to_bf16(rng.standard_normal((B, Hkv, T, 128)))
    v_new = synth.to_bf16(rng.standard_normal((B, Hkv, T, 128)))
    kr = rng.integers(0, 2 ** 16, (B, Hkv, S0 + W, 128)).astype(np.uint16)
    vr = rng.integers(0, 2 ** 16, (B, Hkv, S0 + W, 128)).astype(np.uint16)
    pos = np.array(starts, np.int32)
    ref_k, ref_v = oracle.ring_write(k_new, v_new, pos, kr, vr, S0, W)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16) if a.dtype == np.uint16 else a).cuda()
    kn_d, vn_d, kr_d, vr_d, pos_d = dev(k_new), dev(v_new), dev(kr), dev(vr), dev(pos)
    dims = rtp.make_dims(B, Hkv, Hkv, 64)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rtp.ring_write(dims, kn_d, vn_d, pos_d, T, W, kr_d, vr_d, status, torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert np.array_equal(kr_d.cpu().numpy().view(np.uint16), ref_k)
    assert np.array_equal(vr_d.cpu().numpy().view(np.uint16), ref_v)
