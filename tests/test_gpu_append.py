"""GPU parity of the index-cache append (rtp_index_append) against the fp64
oracle: bit-exact over the whole cache (written and untouched rows),
contiguous and paged layouts, one token and a ragged chunk."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import sparse_attention_decode_rtpurbo_b200 as rtp  # noqa: E402


def _case(seed, B, Hkv, T, ncap, paged):
    rng = np.random.default_rng(seed)
    k_pre = synth.to_bf16(rng.standard_normal((B, Hkv, T, 128)))
    Wk = synth.to_bf16(rng.standard_normal((Hkv, 16, 128)) / np.sqrt(128))
    pos = rng.integers(0, ncap - T + 1, B).astype(np.int32)
    bt = None
    if paged:
        mbps = ncap // 64
        bt = rng.permutation(B * mbps).astype(np.int32).reshape(B, mbps)
        cache = rng.integers(0, 2 ** 16, (B * mbps, Hkv, 64, 16)).astype(np.uint16)
    else:
        cache = rng.integers(0, 2 ** 16, (B, Hkv, ncap, 16)).astype(np.uint16)
    return k_pre, Wk, pos, cache, bt


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16) if a.dtype == np.uint16 else a).cuda()


def _run(k_pre, Wk, pos, cache, bt, ncap):
    B, Hkv, T = k_pre.shape[:3]
    bt_d = None if bt is None else _dev(bt)
    dims = rtp.make_dims(B, Hkv, Hkv, ncap, block_table=bt_d, max_blocks_per_seq=0 if bt is None else bt.shape[1],
                         num_pages=0 if bt is None else cache.shape[0])
    k_d, w_d, p_d, c_d = _dev(k_pre), _dev(Wk), _dev(pos), _dev(cache)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rtp.index_append(dims, k_d, w_d, p_d, T, c_d, status, torch.cuda.current_stream())
    torch.cuda.synchronize()
    return c_d.cpu().numpy().view(np.uint16), int(status.item())


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("B,Hkv,T,ncap", [(3, 4, 1, 256), (2, 8, 37, 512), (1, 1, 1024, 1024)])
def test_append_bit_exact(paged, B, Hkv, T, ncap):
    k_pre, Wk, pos, cache, bt = _case(11 + T, B, Hkv, T, ncap, paged)
    got, st = _run(k_pre, Wk, pos, cache, bt, ncap)
    ref = oracle.index_append(k_pre, Wk, pos, cache, block_table=bt)
    assert st == 0
    assert np.array_equal(got, ref), int(np.count_nonzero(got != ref))


def test_append_rows_beyond_capacity_set_status():
    """A sequence whose new rows run past the capacity: its rows inside the
    capacity are written, the others skipped and the status set; the other
    sequences are unaffected."""
    B, Hkv, T, ncap = 3, 2, 9, 128
    k_pre, Wk, pos, cache, bt = _case(5, B, Hkv, T, ncap, False)
    pos[1] = ncap - 4                        # rows ncap-4 .. ncap+4: 4 inside, 5 beyond
    got, st = _run(k_pre, Wk, pos, cache, bt, ncap)
    assert st == 6                           # RTP_ERR_DEVICE_INPUT
    ok = np.array([0, 2])
    ref = oracle.index_append(k_pre[ok], Wk, pos[ok], cache[ok])
    assert np.array_equal(got[ok], ref)
    # sequence 1: the rows inside the capacity hold the projection of tokens 0..3
    ref1 = oracle.index_append(k_pre[1:2, :, :4], Wk, pos[1:2], cache[1:2])
    assert np.array_equal(got[1], ref1[0])
