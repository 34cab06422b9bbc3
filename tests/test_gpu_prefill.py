"""GPU parity of the prefill attention (rtp_prefill, both of its kernels)
against the fp64 oracle's prefill: query t of sequence b at position pos[b] + t attends causally, densely
for retrieval heads and over the sink and window for local heads.  Outputs
within 4e-3 + 1e-2 |ref|, element by element; cache rows at or beyond each
sequence's length are NaN, so a stray read shows up as a non-finite output."""
import numpy as np
import pytest

import oracle
import synth
import sparse_attention_decode_rtpurbo_b200 as rtp
from tests.parity import ATOL, RTOL

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

from synth.torch_io import bf16_tensor  # noqa: E402


@pytest.fixture(params=["warp-mma", "tcgen05"], autouse=True)
def prefill_kernel(request, monkeypatch):
    """Every case runs on both prefill kernels: the tcgen05 one with its
    accumulators in tensor memory (the default) and the warp-level MMA one
    (RTP_PREFILL_TC=0)."""
    if request.param == "tcgen05":
        monkeypatch.delenv("RTP_PREFILL_TC", raising=False)
    else:
        monkeypatch.setenv("RTP_PREFILL_TC", "0")
    return request.param


def run_prefill(case, q, pos, expect_status=0):
    """rtp_prefill on the case's caches; returns (out as float, status)."""
    dev = "cuda"
    k = bf16_tensor(case.k_cache, dev)
    v = bf16_tensor(case.v_cache, dev)
    bt = None if case.block_table is None else torch.from_numpy(
        np.ascontiguousarray(case.block_table, dtype=np.int32)).to(dev)
    mbps = 0 if bt is None else int(bt.shape[1])
    dims = rtp.make_dims(case.B, case.Hq, case.Hkv, case.Ncap, block_table=bt, max_blocks_per_seq=mbps,
                         num_pages=case.num_pages)
    qd = bf16_tensor(q, dev)
    posd = torch.from_numpy(np.ascontiguousarray(pos, dtype=np.int32)).to(dev)
    T = q.shape[2]
    # a NaN sentinel in every output: what the kernel leaves unwritten stays NaN
    out = torch.full((case.B, case.Hq, T, 128), float("nan"), dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    rtp.prefill(dims, qd, k, v, case.head_kind, posd, T, case.window, case.sink, out, status,
                torch.cuda.current_stream())
    torch.cuda.synchronize()
    st = int(status.item())
    assert st == expect_status, f"device status {st}"
    return out.float().cpu().numpy(), st


def check(case, q, pos, batches=None):
    got, _ = run_prefill(case, q, pos)
    ref = oracle.prefill(case, q, pos)
    for b in (range(case.B) if batches is None else batches):
        g, r = got[b], ref[b]
        assert np.all(np.isfinite(g)), f"sequence {b}: non-finite output"
        err = np.abs(g - r)
        lim = ATOL + RTOL * np.abs(r)
        bad = np.argwhere(err > lim)
        assert bad.size == 0, f"sequence {b}: {len(bad)} elements out of tolerance, first (h, t, d) {bad[0].tolist()}, " \
                              f"got {g[tuple(bad[0])]:.5f} want {r[tuple(bad[0])]:.5f}"
    return got, ref


def queries(case, T, seed):
    rng = np.random.default_rng(seed)
    return synth.to_bf16(rng.standard_normal((case.B, case.Hq, T, 128)))


def mixed_case(L, window, sink, paged=False, seed=5, B=2, Hkv=2, G=4):
    # KV groups holding both kinds of heads: every cache row below L is valid
    hk = np.array(([1, 0] * G)[:G] * Hkv, np.uint8)
    lens = [L - 7 * b for b in range(B)]
    return synth.make_case("prefill", B=B, Hkv=Hkv, G=G, seq_lens=lens, ret_groups=[], head_kind=hk,
                           p=[1.0] * B, window=window, sink=sink, seed=seed, regimes=["gaussian"] * B, paged=paged)


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("T", [1, 16, 37, 50, 64, 129])
def test_chunk_at_the_end_of_the_context(paged, T):
    """The chunk's queries at the last T positions of each sequence (the
    cache holds every position up to them); rows from L on are NaN."""
    case = mixed_case(300, 40, 3, paged=paged)
    pos = (case.seq_lens - T).astype(np.int32)
    check(case, queries(case, T, T), pos)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_whole_prompt_from_position_zero(G):
    """A whole prompt (pos = 0), group sizes 1..8, retrieval and local heads
    mixed inside the groups."""
    L = 700
    case = mixed_case(L, 100, 4, B=1, Hkv=2, G=G, seed=G)
    check(case, queries(case, L, 11 * G), np.zeros(1, np.int32))


@pytest.mark.parametrize("window,sink", [(1, 0), (0, 4), (64, 0), (5000, 4), (63, 64), (130, 2)])
def test_local_window_and_sink_edges(window, sink):
    """Local-only and retrieval-only KV groups (no poisoned rows below L):
    window 1 (each query sees itself), window 0 (the sink only), windows past
    the prompt, a sink of a whole block."""
    L, T = 520, 200
    case = synth.make_case("prefill-edges", B=2, Hkv=4, G=2, seq_lens=[L, L - 33], ret_groups=[1],
                           p=[1.0, 1.0], window=window, sink=sink, seed=17, regimes=["gaussian"] * 2, poison=False)
    pos = (case.seq_lens - T).astype(np.int32)
    check(case, queries(case, T, 3), pos)


def test_long_chunk_many_tiles_paged():
    """Two thousand queries over a paged cache: every CTA walks tens of key
    tiles, the local heads' windows start mid-tile."""
    L = 2048
    case = mixed_case(L, 333, 4, paged=True, seed=23, B=1, Hkv=4, G=4)
    check(case, queries(case, L - 48, 29), np.array([48], np.int32))


def test_bad_position_sets_status_and_skips_the_sequence():
    """pos[b] + num_q beyond the capacity is an error only the device sees:
    that sequence's outputs are not written (they keep the NaN sentinel), the
    other sequence's still match."""
    case = mixed_case(300, 40, 3)
    T = 20
    pos = np.array([case.Ncap - T + 1, int(case.seq_lens[1]) - T], np.int32)
    got, st = run_prefill(case, queries(case, T, 5), pos, expect_status=6)
    assert np.all(np.isnan(got[0]))
    ref = oracle.prefill(case, queries(case, T, 5), np.array([0, pos[1]], np.int32))
    err = np.abs(got[1] - ref[1])
    assert np.all(err <= ATOL + RTOL * np.abs(ref[1]))


def test_last_query_matches_the_decode_step():
    """The chunk's last query, given the decode query's vector at position
    L - 1, sees the decode step's position sets (p = 1): the decode step's
    output within the parity tolerance."""
    L, T = 900, 33
    case = mixed_case(L, 100, 4, seed=9)
    q = queries(case, T, 3)
    q[:, :, T - 1] = case.q_rope
    pos = (case.seq_lens - T).astype(np.int32)
    got, _ = check(case, q, pos)
    dec = oracle.decode_step(case)["out"]
    assert np.all(np.abs(got[:, :, T - 1] - dec) <= ATOL + RTOL * np.abs(dec))
