"""GPU parity of the KV-cache write with the index-cache append
(rtp_kv_append) against the fp64 oracle: bit-exact over the three whole
caches (written and untouched rows), contiguous and paged layouts, one token
and a ragged chunk, with random angle tables and the position table n theta_i."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import sparse_attention_decode_rtpurbo_b200 as rtp  # noqa: E402


def _case(seed, B, Hkv, T, ncap, paged, position_angles=False):
    rng = np.random.default_rng(seed)
    k_pre = synth.to_bf16(rng.standard_normal((B, Hkv, T, 128)))
    v_new = synth.to_bf16(rng.standard_normal((B, Hkv, T, 128)))
    Wk = synth.to_bf16(rng.standard_normal((Hkv, 16, 128)) / np.sqrt(128))
    pos = rng.integers(0, ncap - T + 1, B).astype(np.int32)
    if position_angles:
        ang = np.arange(ncap, dtype=np.float64)[:, None] * synth.THETA ** (-2.0 * np.arange(64) / 128.0)[None, :]
    else:
        ang = rng.uniform(-np.pi, np.pi, (ncap, 64))
    cos, sin = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
    bt = None
    if paged:
        mbps = ncap // 64
        bt = rng.permutation(B * mbps).astype(np.int32).reshape(B, mbps)
        lead = (B * mbps, Hkv, 64)
    else:
        lead = (B, Hkv, ncap)
    kidx = rng.integers(0, 2 ** 16, lead + (16,)).astype(np.uint16)
    kc = rng.integers(0, 2 ** 16, lead + (128,)).astype(np.uint16)
    vc = rng.integers(0, 2 ** 16, lead + (128,)).astype(np.uint16)
    return k_pre, v_new, Wk, cos, sin, pos, kidx, kc, vc, bt


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16) if a.dtype == np.uint16 else
                            np.ascontiguousarray(a)).cuda()


def _run(k_pre, v_new, Wk, cos, sin, pos, kidx, kc, vc, bt, ncap):
    B, Hkv, T = k_pre.shape[:3]
    bt_d = None if bt is None else _dev(bt)
    dims = rtp.make_dims(B, Hkv, Hkv, ncap, block_table=bt_d, max_blocks_per_seq=0 if bt is None else bt.shape[1],
                         num_pages=0 if bt is None else kc.shape[0])
    dev = [_dev(a) for a in (k_pre, v_new, Wk, cos, sin, pos, kidx, kc, vc)]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rtp.kv_append(dims, dev[0], dev[1], dev[2], dev[3], dev[4], dev[5], T, dev[6], dev[7], dev[8], status,
                  torch.cuda.current_stream())
    torch.cuda.synchronize()
    return tuple(t.cpu().numpy().view(np.uint16) for t in dev[6:]), int(status.item())


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("B,Hkv,T,ncap", [(3, 4, 1, 256), (2, 8, 37, 512), (1, 1, 1024, 1024)])
def test_kv_append_bit_exact(paged, B, Hkv, T, ncap):
    case = _case(21 + T, B, Hkv, T, ncap, paged)
    got, st = _run(*case, ncap)
    k_pre, v_new, Wk, cos, sin, pos, kidx, kc, vc, bt = case
    ref = oracle.kv_append(k_pre, v_new, Wk, cos, sin, pos, kidx, kc, vc, block_table=bt)
    assert st == 0
    for name, g, r in zip(("k_idx", "k_cache", "v_cache"), got, ref):
        assert np.array_equal(g, r), (name, int(np.count_nonzero(g != r)))


def test_kv_append_position_angles():
    """The angle table of positions n theta_i over a 64K cache (large angles,
    every row of the table in use somewhere)."""
    ncap = 65536
    case = _case(3, 2, 2, 64, ncap, False, position_angles=True)
    got, st = _run(*case, ncap)
    k_pre, v_new, Wk, cos, sin, pos, kidx, kc, vc, bt = case
    ref = oracle.kv_append(k_pre, v_new, Wk, cos, sin, pos, kidx, kc, vc)
    assert st == 0
    for g, r in zip(got, ref):
        assert np.array_equal(g, r)


def test_kv_append_rows_beyond_capacity_set_status():
    """Rows past the capacity are skipped in all three caches and reported;
    the rows inside it and the other sequences are written."""
    B, Hkv, T, ncap = 3, 2, 9, 128
    case = list(_case(5, B, Hkv, T, ncap, False))
    case[5][1] = ncap - 4                    # rows ncap-4 .. ncap+4: 4 inside, 5 beyond
    got, st = _run(*case, ncap)
    k_pre, v_new, Wk, cos, sin, pos, kidx, kc, vc, bt = case
    assert st == 6                           # RTP_ERR_DEVICE_INPUT
    ok = np.array([0, 2])
    ref = oracle.kv_append(k_pre[ok], v_new[ok], Wk, cos, sin, pos[ok], kidx[ok], kc[ok], vc[ok])
    for g, r in zip(got, ref):
        assert np.array_equal(g[ok], r)
    ref1 = oracle.kv_append(k_pre[1:2, :, :4], v_new[1:2, :, :4], Wk, cos, sin, pos[1:2], kidx[1:2], kc[1:2],
                            vc[1:2])
    for g, r in zip(got, ref1):
        assert np.array_equal(g[1], r[0])


def test_kv_append_feeds_the_decode_step():
    """Caches written by rtp_kv_append (one 3000-token prefill chunk, position
    angles) are the decode step's input: its output on them matches the
    oracle's decode step on the same caches."""
    from synth.torch_io import DeviceCase
    from tests.parity import compare

    case = synth.make_case("kvapp", B=1, Hkv=2, G=4, seq_lens=[3000], ret_groups=[0], p=[0.9], window=256, sink=4,
                           seed=77, regimes=["gaussian"])
    ncap, L, Hkv = case.Ncap, int(case.seq_lens[0]), case.Hkv
    rng = np.random.default_rng(77)
    k_pre = synth.to_bf16(rng.standard_normal((1, Hkv, L, 128)))
    v_new = synth.to_bf16(rng.standard_normal((1, Hkv, L, 128)))
    Wk = synth.to_bf16(rng.standard_normal((Hkv, 16, 128)) / np.sqrt(128))
    ang = np.arange(ncap, dtype=np.float64)[:, None] * synth.THETA ** (-2.0 * np.arange(64) / 128.0)[None, :]
    cos, sin = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
    zeros = [np.zeros_like(a) for a in (case.k_idx, case.k_cache, case.v_cache)]
    pos = np.zeros(1, dtype=np.int32)
    got, st = _run(k_pre, v_new, Wk, cos, sin, pos, *zeros, None, ncap)
    assert st == 0
    ref = oracle.kv_append(k_pre, v_new, Wk, cos, sin, pos, *zeros)
    for g, r in zip(got, ref):
        assert np.array_equal(g, r)
    case.k_idx, case.k_cache, case.v_cache = got
    dc = DeviceCase(case)
    dc.run()
    fails, _ = compare(case, dc.results(), oracle.decode_step(case))
    assert not fails, "\n".join(fails[:10])
