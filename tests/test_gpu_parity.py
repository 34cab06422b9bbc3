"""GPU parity of the decode step against the fp64 oracle, through the C ABI."""
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


def run_both(case, exact=False, check_kstar=False, check_tau=False):
    dc = DeviceCase(case)
    dc.run()
    gpu = dc.results()
    ref = oracle.decode_step(case)
    assert ref["rc"] == 0
    fails, stats = compare(case, gpu, ref, exact_sets=exact, check_kstar=check_kstar, check_tau=check_tau)
    return fails, stats, gpu, ref


@pytest.mark.parametrize("w,scale", [(1, 1), (2, 1), (2, 8), (3, 32), (4, 64), (5, 32), (5, 8), (1, 4)])
def test_workload_parity_reduced(w, scale):
    case = synth.workload(w, scale=scale)
    fails, stats, gpu, ref = run_both(case)
    assert not fails, "\n".join(fails[:20])


def test_integer_scores_exact_block_sets():
    """Integer scores: GPU and oracle must pick identical block sets, k* and tau.
    Seeds whose cumulative mass comes within 1e-4 of p (where fp32 and fp64
    mass sums may legitimately disagree) are skipped by the oracle's own
    prefix masses."""
    done = 0
    for seed in range(40):
        for (G, paged, p, L) in [(4, False, 0.9, 700), (8, True, 0.5, 1500), (1, False, 0.95, 333),
                                 (2, True, 0.8, 2100)]:
            case = synth.integer_case(seed, G=G, paged=paged, p=p, L=L, Hkv=2, B=2)
            ref = oracle.decode_step(case)
            ret = np.nonzero(case.head_kind)[0]
            margins = np.abs(np.concatenate([ref["cum_before"][:, ret].ravel(), ref["cum_at"][:, ret].ravel()]) - p)
            if margins.min() < 1e-4:
                continue
            dc = DeviceCase(case)
            dc.run()
            gpu = dc.results()
            fails, _ = compare(case, gpu, ref, exact_sets=True, check_kstar=True, check_tau=True)
            assert not fails, f"seed {seed} G{G} paged{paged}:\n" + "\n".join(fails[:10])
            done += 1
    assert done >= 60


@pytest.mark.parametrize("L", [1, 2, 63, 64, 65, 127, 2047, 2048, 2049, 4097])
def test_edge_lengths(L):
    case = synth.make_case(f"edge-{L}", B=2, Hkv=2, G=4, seq_lens=[L, max(1, L // 2)], ret_groups=[1],
                           p=[0.9, 0.6], window=100, sink=4, seed=100 + L, regimes=["gaussian", "diffuse"])
    fails, *_ = run_both(case)
    assert not fails, "\n".join(fails[:20])


@pytest.mark.parametrize("window,sink", [(5000, 4), (1, 0), (0, 3), (64, 64), (65, 1)])
def test_local_window_edges(window, sink):
    case = synth.make_case("win", B=1, Hkv=2, G=2, seq_lens=[3000], ret_groups=[0], p=[0.9], window=window,
                           sink=sink, seed=7, regimes=["gaussian"])
    fails, *_ = run_both(case)
    assert not fails, "\n".join(fails[:20])


def test_p_one_is_dense_and_tiny_p_keeps_one():
    case = synth.make_case("p1", B=2, Hkv=1, G=4, seq_lens=[5000, 777], ret_groups=[0], p=[1.0, 1e-6],
                           window=64, sink=4, seed=8, regimes=["gaussian", "gaussian"])
    fails, stats, gpu, ref = run_both(case, check_kstar=True)
    assert not fails, "\n".join(fails[:20])
    assert np.all(gpu["kstar"][0] == 5000) and np.all(gpu["kept"][0, :, :79].all(axis=1))
    assert np.all(gpu["kstar"][1] == 1)


@pytest.mark.parametrize("G", [1, 2, 8])
def test_group_sizes_and_all_retrieval(G):
    case = synth.make_case(f"g{G}", B=2, Hkv=2, G=G, seq_lens=[6000, 4100], ret_groups=[0, 1], p=[0.9, 0.95],
                           window=256, sink=4, seed=30 + G, regimes=["needle", "diffuse"])
    fails, *_ = run_both(case)
    assert not fails, "\n".join(fails[:20])


def test_mixed_group_heads():
    """Retrieval and local heads inside one KV group (as in the 4K workload)."""
    hk = np.array([1, 0, 1, 0, 0, 0, 0, 1], np.uint8)
    case = synth.make_case("mixed", B=1, Hkv=2, G=4, seq_lens=[9000], ret_groups=[], head_kind=hk, p=[0.9],
                           window=512, sink=4, seed=41, regimes=["gaussian"])
    fails, *_ = run_both(case)
    assert not fails, "\n".join(fails[:20])


def test_deterministic():
    case = synth.workload(2, scale=4)
    dc = DeviceCase(case)
    dc.run()
    a = dc.out.clone()
    dc.run()
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), dc.out.view(torch.int16))


def test_device_input_errors_set_status():
    case = synth.make_case("bad", B=2, Hkv=1, G=4, seq_lens=[300, 200], ret_groups=[0], p=[0.9, 0.9], window=64,
                           sink=4, seed=9, regimes=["gaussian", "gaussian"])
    dc = DeviceCase(case)
    dc.p[1] = 0.0
    dc.run()
    assert dc.step.status() == 6
    dc.p[1] = 0.9
    dc.run()
    assert dc.step.status() == 0
    dc.seq_lens[0] = case.Ncap + 64
    dc.run()
    assert dc.step.status() == 6
    dc.seq_lens[0] = 300
    dc.run()
    assert dc.step.status() == 0
    ref = oracle.decode_step(case)
    for bad in (0, -7):
        # an empty or negative length is an input error too; the other
        # sequence's results still match the oracle's
        dc.seq_lens[0] = bad
        dc.run()
        res = dc.results()
        assert res["status"] == 6
        res["status"] = 0
        fails, _ = compare(case, res, ref, batches=[1])
        assert not fails, "\n".join(fails[:10])
    dc.seq_lens[0] = 300
    dc.run()
    assert dc.step.status() == 0


def test_bad_page_id_sets_status():
    case = synth.make_case("badpage", B=1, Hkv=1, G=4, seq_lens=[500], ret_groups=[0], p=[0.9], window=64, sink=4,
                           seed=10, regimes=["gaussian"], paged=True)
    dc = DeviceCase(case)
    dc.block_table[0, 3] = case.num_pages + 5
    dc.run()
    assert dc.step.status() == 6


@pytest.mark.parametrize("w", [3, 4, 5])
def test_full_size_workloads(w):
    """The benchmark's workloads at full size (4x128K, 1M, ragged paged x16)."""
    case = synth.workload(w)
    fails, stats, gpu, ref = run_both(case)
    assert not fails, "\n".join(fails[:20])


def _ties_at_tau(case, ref, b, h):
    s = oracle.index_scores(case, b, h)[: int(case.seq_lens[b])]
    return int(np.count_nonzero(s == ref["tau"][b, h]))


def test_refine_passes_many_ties():
    """Few integer score levels over 64K tokens: the threshold bin holds more
    than 4096 tokens, so the select refines the threshold over all stored
    scores (four 8-bit passes), counts threshold ties per tile and locates the
    last tie kept.  Block sets, k* and tau must be exact."""
    done = deep = 0
    for seed in range(8):
        case = synth.integer_case(seed, B=1, Hkv=2, G=4, L=65536, p=0.9, qmax=1, kmax=1)
        ref = oracle.decode_step(case)
        assert ref["rc"] == 0
        ret = np.nonzero(case.head_kind)[0]
        # where p falls inside the mass of the last kept token: the count of
        # ties kept is robust to mass rounding unless p sits at an end
        lo, hi = ref["cum_before"][0, ret], ref["cum_at"][0, ret]
        frac = (0.9 - lo) / np.maximum(hi - lo, 1e-300)
        if np.any((frac < 1e-3) | (frac > 1 - 1e-3)):
            continue
        deep += max(_ties_at_tau(case, ref, 0, h) for h in ret) > 4096
        dc = DeviceCase(case)
        dc.run()
        fails, _ = compare(case, dc.results(), ref, exact_sets=True, check_kstar=True, check_tau=True)
        assert not fails, f"seed {seed}:\n" + "\n".join(fails[:10])
        done += 1
    assert done >= 4 and deep >= 2, (done, deep)


@pytest.mark.parametrize("cap,w,scale", [(3, 5, 8), (7, 3, 1)])
def test_small_grid_long_shares(monkeypatch, cap, w, scale):
    """Both grids capped at a few CTAs (RTP_GRID_CAP): every CTA's share of
    stored score tiles exceeds the shared-memory stages, so the select passes
    read them from global memory; with 7 CTAs over 4 x 128K, shares of more
    than 64 tiles of one group flush the shared histograms mid-run.  Results
    must not change."""
    monkeypatch.setenv("RTP_GRID_CAP", str(cap))
    case = synth.workload(w, scale=scale)
    fails, stats, gpu, ref = run_both(case)
    assert not fails, "\n".join(fails[:20])


@pytest.mark.parametrize("regime", ["diffuse", "gaussian"])
def test_full_size_1m_exact_select(regime):
    """The 1M workload's shape (B=1, L=2^20, 8 KV x GQA 4, group 0 retrieval,
    p=0.9, window 4096, sink 4) with a score field that no single token
    settles: every retrieval head goes through the exact select with 2^20
    scores (the first pass's bin range, the overflow bin and the candidate
    caps at that length), then the block-list attention."""
    case = synth.make_case(f"w4-1m-{regime}", B=1, Hkv=8, G=4, seq_lens=[1 << 20], ret_groups=[0], p=[0.9],
                           window=4096, sink=4, seed=3, regimes=[regime])
    fails, stats, gpu, ref = run_both(case)
    assert not fails, "\n".join(fails[:20])
    ret = np.nonzero(case.head_kind)[0]
    assert np.all(gpu["kstar"][0, ret] > 1)          # the select ran: no head was settled by its best token
