"""GPU parity of the static top-k variant (rtp_decode_step_topk) against the
fp64 oracle's top-k decode step, through the C ABI.  The comparison rules are
those of the top-p step: exact block sets, k* and tau on integer scores; on
random scores, blocks that differ must hold a token within 1e-4 |tau| of the
oracle's k-th score; outputs within 4e-3 + 1e-2 |ref|."""
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


def run_both(case, k, **kw):
    dc = DeviceCase(case)
    dc.run_topk(k)
    gpu = dc.results()
    ref = oracle.decode_step_topk(case, k)
    assert ref["rc"] == 0
    fails, stats = compare(case, gpu, ref, **kw)
    return fails, stats, gpu, ref


@pytest.mark.parametrize("w,scale,k", [(1, 1, 64), (1, 1, 2), (2, 1, 4096), (2, 8, 300), (3, 32, 4096),
                                       (5, 32, 1000), (4, 64, 4096), (5, 8, 4096)])
def test_workload_parity_reduced(w, scale, k):
    case = synth.workload(w, scale=scale)
    fails, stats, gpu, ref = run_both(case, k)
    assert not fails, "\n".join(fails[:20])


def test_integer_scores_exact():
    """Integer scores with many ties: the k kept tokens are fixed exactly by
    (score desc, index asc), so block sets, k* and tau must match exactly."""
    for seed in range(12):
        for (G, paged, L, k) in [(4, False, 700, 37), (8, True, 1500, 300), (1, False, 333, 332),
                                 (2, True, 2100, 1024), (4, False, 4000, 2)]:
            case = synth.integer_case(seed, G=G, paged=paged, p=0.9, L=L, Hkv=2, B=2)
            fails, _, gpu, ref = run_both(case, k, exact_sets=True, check_kstar=True, check_tau=True)
            assert not fails, f"seed {seed} G{G} paged{paged} k{k}:\n" + "\n".join(fails[:10])
            ret = np.nonzero(case.head_kind)[0]
            assert np.all(gpu["kstar"][:, ret] == np.minimum(k, case.seq_lens[:, None]))


@pytest.mark.parametrize("L", [1, 2, 63, 64, 65, 2049])
@pytest.mark.parametrize("k", [1, 2, 64, 5000])
def test_edge_lengths_and_budgets(L, k):
    """k = 1 (the best token's block, settled by the streaming kernel), k >= L
    (every block), and the exact select between them."""
    case = synth.make_case(f"topk-edge-{L}", B=2, Hkv=2, G=4, seq_lens=[L, max(1, L // 2)], ret_groups=[1],
                           p=[0.9, 0.9], window=100, sink=4, seed=200 + L, regimes=["gaussian", "needle"])
    fails, stats, gpu, ref = run_both(case, k, check_kstar=True)
    assert not fails, "\n".join(fails[:20])
    ret = np.nonzero(case.head_kind)[0]
    assert np.all(gpu["kstar"][:, ret] == np.minimum(k, case.seq_lens[:, None]))


def test_refine_passes_many_ties():
    """Two integer score levels per sign over 64K tokens: the k-th score's bin
    holds far more than 4096 tokens, so the select refines over all stored
    scores, counts ties per tile and locates the last tie kept."""
    for seed in range(3):
        case = synth.integer_case(seed, B=1, Hkv=2, G=4, L=65536, p=0.9, qmax=1, kmax=1)
        fails, _, gpu, ref = run_both(case, 20000, exact_sets=True, check_kstar=True, check_tau=True)
        assert not fails, f"seed {seed}:\n" + "\n".join(fails[:10])


@pytest.mark.parametrize("cap,w,scale", [(3, 5, 8), (7, 3, 1)])
def test_small_grid_long_shares(monkeypatch, cap, w, scale):
    """Grids capped at a few CTAs: select passes over global memory and
    mid-run histogram flushes, now with unit masses."""
    monkeypatch.setenv("RTP_GRID_CAP", str(cap))
    case = synth.workload(w, scale=scale)
    fails, *_ = run_both(case, 4096)
    assert not fails, "\n".join(fails[:20])


@pytest.mark.parametrize("w", [3, 5])
def test_full_size_workloads(w):
    """k = 4096 (the pages' static budget) on the 4 x 128K and ragged paged workloads at full size."""
    case = synth.workload(w)
    fails, *_ = run_both(case, 4096)
    assert not fails, "\n".join(fails[:20])


def test_topk_and_topp_share_a_workspace():
    """The two variants alternate on one workspace without disturbing each other."""
    case = synth.workload(2, scale=8)
    dc = DeviceCase(case)
    dc.run()
    a = dc.out.clone()
    dc.run_topk(512)
    b = dc.out.clone()
    dc.run()
    torch.cuda.synchronize()
    assert dc.step.status() == 0
    assert torch.equal(a.view(torch.int16), dc.out.view(torch.int16))
    dc.run_topk(512)
    torch.cuda.synchronize()
    assert torch.equal(b.view(torch.int16), dc.out.view(torch.int16))
