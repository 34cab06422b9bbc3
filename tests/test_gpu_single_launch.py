"""GPU parity of the single-launch decode step (RTP_SINGLE_LAUNCH=1: the
streaming phase, a grid barrier, then the retrieval phase in one kernel)
against the fp64 oracle: workloads whose groups are all settled in the
streaming phase (no retrieval work), workloads with the exact select and
block-sparse attention, capped grids, and alternation with the two-launch
step on one workspace."""
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


def run_single(monkeypatch, case, **kw):
    monkeypatch.setenv("RTP_SINGLE_LAUNCH", "1")
    dc = DeviceCase(case)
    dc.run()
    gpu = dc.results()
    ref = oracle.decode_step(case)
    fails, _ = compare(case, gpu, ref, **kw)
    return fails


@pytest.mark.parametrize("w,scale", [(1, 1), (2, 1), (2, 8), (3, 32), (4, 64), (5, 32), (5, 8)])
def test_single_launch_workloads(monkeypatch, w, scale):
    assert run_single(monkeypatch, synth.workload(w, scale=scale)) == []


@pytest.mark.parametrize("w", [3, 4, 5])
def test_single_launch_full_size(monkeypatch, w):
    assert run_single(monkeypatch, synth.workload(w)) == []


def test_single_launch_integer_scores_exact(monkeypatch):
    """Integer scores (the parity suite's shapes): identical block sets, k*
    and tau.  Seeds whose prefix mass comes within 1e-4 of p are skipped by
    the oracle's own prefix masses, as in the two-launch test."""
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
            assert run_single(monkeypatch, case, exact_sets=True, check_kstar=True, check_tau=True) == []
            done += 1
        if done >= 12:
            break
    assert done >= 12


@pytest.mark.parametrize("cap,w,scale", [(3, 5, 8), (7, 3, 1)])
def test_single_launch_small_grid(monkeypatch, cap, w, scale):
    monkeypatch.setenv("RTP_GRID_CAP", str(cap))
    assert run_single(monkeypatch, synth.workload(w, scale=scale)) == []


def test_single_and_two_launches_alternate_on_one_workspace(monkeypatch):
    """The coordination words each path leaves are the other's starting state."""
    case = synth.workload(3, scale=32)
    ref = oracle.decode_step(case)
    dc = DeviceCase(case)
    for single in (True, False, True, True, False):
        if single:
            monkeypatch.setenv("RTP_SINGLE_LAUNCH", "1")
        else:
            monkeypatch.delenv("RTP_SINGLE_LAUNCH", raising=False)
        dc.run()
        fails, _ = compare(case, dc.results(), ref)
        assert fails == [], (single, fails[:5])
