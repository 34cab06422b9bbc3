"""GPU-vs-oracle comparison rules for the decode step.

Block sets: bit-exact where the scores are exactly representable (integer
scores); otherwise every block in the symmetric difference of a head's GPU
and oracle block sets must hold a token whose oracle score lies within
1e-4 * |tau| of the oracle threshold tau (the k*-th score).
Outputs: |gpu - ref| <= 4e-3 + 1e-2 * |ref| element-wise, ref = the oracle's
output on the oracle's block set when the sets agree, else the oracle's exact
attention over the GPU's block set.
"""
import numpy as np

import oracle

ATOL = 4e-3
RTOL = 1e-2
BAND = 1e-4


def blocks_to_positions(kept: np.ndarray, L: int) -> np.ndarray:
    js = np.nonzero(kept)[0]
    if js.size == 0:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate([np.arange(64 * j, min(64 * j + 64, L)) for j in js]).astype(np.int64)


def compare(case, gpu, ref, *, exact_sets: bool = False, check_kstar: bool = False, check_tau: bool = False,
            heads=None, batches=None):
    """Returns a list of failure strings (empty = pass) and a stats dict.
    heads / batches: compare only these query heads / sequences."""
    fails = []
    stats = {"set_diffs": 0, "heads": 0, "max_err": 0.0}
    assert gpu["status"] == 0, f"device status {gpu['status']}"
    for b in (range(case.B) if batches is None else batches):
        L = int(case.seq_lens[b])
        nblk = (L + 63) // 64
        for h in (range(case.Hq) if heads is None else heads):
            stats["heads"] += 1
            g_out = gpu["out"][b, h]
            r_out = ref["out"][b, h]
            if not np.all(np.isfinite(g_out)):
                fails.append(f"b{b} h{h}: non-finite output")
                continue
            if case.head_kind[h]:
                gk = gpu["kept"][b, h, :nblk].astype(bool)
                rk = ref["kept_blocks"][b, h, :nblk].astype(bool)
                if gpu["kept"][b, h, nblk:].any():
                    fails.append(f"b{b} h{h}: GPU kept a block beyond L")
                diff = np.nonzero(gk != rk)[0]
                if diff.size:
                    stats["set_diffs"] += 1
                    if exact_sets:
                        fails.append(f"b{b} h{h}: block sets differ at {diff[:8].tolist()} (exact required)")
                        continue
                    s = oracle.index_scores(case, b, h)
                    tau = float(ref["tau"][b, h])
                    band = BAND * abs(tau)
                    for j in diff:
                        blk = s[64 * j:min(64 * j + 64, L)]
                        if not np.any(np.abs(blk - tau) <= band):
                            fails.append(f"b{b} h{h}: block {j} differs (gpu {gk[j]}) with no token within "
                                         f"{band:.3g} of tau={tau:.6g}; nearest {np.min(np.abs(blk - tau)):.3g}")
                            break
                    r_out = oracle.attend(case, b, h, blocks_to_positions(gk, L))
                else:
                    if check_kstar and int(gpu["kstar"][b, h]) != int(ref["kstar"][b, h]):
                        fails.append(f"b{b} h{h}: kstar {gpu['kstar'][b, h]} != {ref['kstar'][b, h]}")
                    if check_tau and float(gpu["tau"][b, h]) != float(ref["tau"][b, h]):
                        fails.append(f"b{b} h{h}: tau {gpu['tau'][b, h]} != {ref['tau'][b, h]}")
                if int(gpu["kept_blocks"][b, h]) != int(gk.sum()):
                    fails.append(f"b{b} h{h}: kept_blocks {gpu['kept_blocks'][b, h]} != bitmap popcount {gk.sum()}")
            err = np.abs(g_out - r_out)
            lim = ATOL + RTOL * np.abs(r_out)
            stats["max_err"] = max(stats["max_err"], float(err.max()))
            if np.any(err > lim):
                i = int(np.argmax(err - lim))
                fails.append(f"b{b} h{h} ({'ret' if case.head_kind[h] else 'loc'}): out[{i}] gpu {g_out[i]:.6g} "
                             f"ref {r_out[i]:.6g} err {err[i]:.3g} > {lim[i]:.3g}")
    return fails, stats
