"""Seeded synthetic workloads for the RTPurbo decode step.

One module feeds both sides of every comparison: the CUDA path (through the
package's binding) and the fp64 oracle.  It holds none of the method's
arithmetic.  It draws Gaussian tensors from a counter-based generator
(``synth.c``), rounds them to bf16, rotates keys and queries with RoPE (the
decode step consumes them already rotated) and builds the index-key cache
k_idx = bf16(W^K k^pre).

To shape the index scores the way the workloads ask (planted needles, a
diffuse cluster, a flattened or sharpened score temperature), it also forms
the projected query W^Q q^pre of the heads it aims at and simple statistics
of k_idx (row norms).  It never scores the cache, never takes a softmax or a
top-p set and never attends: those live in the oracle and in the kernels.

Every tensor is a pure function of (seed, tensor tag, index); bf16 tensors
are returned as uint16 arrays holding the raw bits.
"""
from __future__ import annotations

import ctypes
import math
import os
import statistics
import subprocess
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")

BF16_NAN = 0x7FC0
D = 128          # head dimension
R = 16           # index (low-rank) dimension
BLK = 64         # KV block / page size in tokens
THETA = 1.0e6    # RoPE base


def build(force: bool = False) -> str:
    """Compile synth.c into libsynth.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        lib.synth_normal_f64.argtypes = [u64, u64, u64, i64, dbl, vp]
        lib.synth_normal_bf16.argtypes = [u64, u64, u64, i64, dbl, vp]
        lib.synth_uniform_f64.argtypes = [u64, u64, u64, i64, vp]
        lib.synth_f64_to_bf16.argtypes = [vp, i64, vp]
        lib.synth_bf16_to_f64.argtypes = [vp, i64, vp]
        lib.synth_fill_u16.argtypes = [vp, i64, ctypes.c_uint16]
        lib.synth_rope_rows_bf16.argtypes = [vp, i64, vp, dbl, vp]
        lib.synth_keys.argtypes = [u64, u64, vp, i64, dbl, vp, vp, vp, vp]
        lib.synth_values.argtypes = [u64, u64, vp, i64, vp]
        lib.synth_kidx_stats.argtypes = [vp, i64, vp, vp]
        lib.synth_stream_base.argtypes = [u64, u64]
        lib.synth_stream_base.restype = u64
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "array must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


# ----------------------------------------------------------------------------
# streams: every tensor gets its own counter stream
# ----------------------------------------------------------------------------
_TAGS = {"q": 1, "Wq": 2, "Wk": 3, "k": 4, "v": 5, "pos": 6, "misc": 7, "int": 8, "len": 9}


def stream_id(tag: str, *idx: int) -> int:
    s = _TAGS[tag]
    for i in idx:
        s = (s * 1000003 + int(i) + 1) & 0xFFFFFFFFFFFFFFFF
    return s


def normal_f64(seed: int, stream: int, n: int, scale: float = 1.0, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _L().synth_normal_f64(seed, stream, offset, n, scale, _p(out))
    return out


def normal_bf16(seed: int, stream: int, n: int, scale: float = 1.0, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16)
    _L().synth_normal_bf16(seed, stream, offset, n, scale, _p(out))
    return out


def uniform_f64(seed: int, stream: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _L().synth_uniform_f64(seed, stream, offset, n, _p(out))
    return out


def to_bf16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    _L().synth_f64_to_bf16(_p(x), x.size, _p(out))
    return out


def from_bf16(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    out = np.empty(b.shape, dtype=np.float64)
    _L().synth_bf16_to_f64(_p(b), b.size, _p(out))
    return out


def nan_fill(shape) -> np.ndarray:
    a = np.empty(shape, dtype=np.uint16)
    _L().synth_fill_u16(_p(a), a.size, BF16_NAN)
    return a


def rope_rows(x_bf16: np.ndarray, pos: np.ndarray, theta: float = THETA) -> np.ndarray:
    """bf16(RoPE(x, pos)) for rows of 128 (rotate-half pairing, fp64 math)."""
    x = np.ascontiguousarray(x_bf16.reshape(-1, D), dtype=np.uint16)
    pos = np.ascontiguousarray(np.broadcast_to(np.asarray(pos, dtype=np.int64), (x.shape[0],)))
    out = np.empty_like(x)
    _L().synth_rope_rows_bf16(_p(x), x.shape[0], _p(pos), theta, _p(out))
    return out.reshape(x_bf16.shape)


def keys_for(seed: int, stream: int, pos: np.ndarray, W: Optional[np.ndarray], want_kidx: bool,
             want_kpre: bool = False, theta: float = THETA):
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    n = pos.size
    kc = np.empty((n, D), dtype=np.uint16)
    ki = np.empty((n, R), dtype=np.uint16) if want_kidx else None
    kp = np.empty((n, D), dtype=np.uint16) if want_kpre else None
    Wc = np.ascontiguousarray(W, dtype=np.uint16) if W is not None else None
    _L().synth_keys(seed, stream, _p(pos), n, theta,
                    _p(Wc) if Wc is not None else None, _p(kc),
                    _p(ki) if ki is not None else None, _p(kp) if kp is not None else None)
    return kc, ki, kp


def values_for(seed: int, stream: int, pos: np.ndarray) -> np.ndarray:
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    out = np.empty((pos.size, D), dtype=np.uint16)
    _L().synth_values(seed, stream, _p(pos), pos.size, _p(out))
    return out


def kidx_stats(kidx_rows: np.ndarray) -> Tuple[float, float]:
    """(RMS of row norms, max row norm) of bf16 [rows,16] index keys."""
    k = np.ascontiguousarray(kidx_rows, dtype=np.uint16)
    ss = ctypes.c_double()
    mx = ctypes.c_double()
    _L().synth_kidx_stats(_p(k), k.shape[0], ctypes.byref(ss), ctypes.byref(mx))
    return math.sqrt(ss.value / max(1, k.shape[0])), mx.value


# ----------------------------------------------------------------------------
# workload description
# ----------------------------------------------------------------------------
@dataclass
class Case:
    """All inputs of one decode step, host-side, bf16 tensors as uint16 bits."""
    name: str
    B: int
    Hq: int
    Hkv: int
    Ncap: int                     # per-sequence capacity in tokens (multiple of 64)
    seq_lens: np.ndarray          # int32 [B]
    head_kind: np.ndarray         # uint8 [Hq], 1 = retrieval, 0 = local
    p: np.ndarray                 # float32 [B]
    window: int
    sink: int
    q_pre: np.ndarray             # [B,Hq,128]
    q_rope: np.ndarray            # [B,Hq,128]
    Wq_idx: np.ndarray            # [Hq,16,128]
    k_idx: np.ndarray             # [B,Hkv,Ncap,16] or paged [P,Hkv,64,16]
    k_cache: np.ndarray           # [B,Hkv,Ncap,128] or paged [P,Hkv,64,128]
    v_cache: np.ndarray           # same layout as k_cache
    block_table: Optional[np.ndarray] = None   # int32 [B, max_blocks_per_seq] when paged
    num_pages: int = 0
    regimes: List[str] = field(default_factory=list)
    needles: Dict[Tuple[int, int], List[int]] = field(default_factory=dict)  # (b, h) -> planted positions
    seed: int = 0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def paged(self) -> bool:
        return self.block_table is not None

    @property
    def max_blocks_per_seq(self) -> int:
        return 0 if self.block_table is None else int(self.block_table.shape[1])


def head_kind_for(Hkv: int, G: int, ret_groups: Sequence[int]) -> np.ndarray:
    hk = np.zeros(Hkv * G, dtype=np.uint8)
    for g in ret_groups:
        hk[g * G:(g + 1) * G] = 1
    return hk


def local_positions(L: int, window: int, sink: int) -> np.ndarray:
    """Cache positions a local head reads: [0, min(sink,L)) U [max(0,L-window), L)."""
    s = np.arange(min(sink, L), dtype=np.int64)
    w = np.arange(max(0, L - window), L, dtype=np.int64)
    return np.union1d(s, w)


def sigma_for_keep_fraction(p: float, keep: float) -> float:
    """Score std (in units of s/4) at which a Gaussian score field's top-p set
    holds about `keep` of the tokens: mass above threshold t (in std units) is
    1 - Phi(t - sigma) for a lognormal weight field, so t = Phi^-1(1-keep) and
    sigma = t - Phi^-1(1-p)."""
    nd = statistics.NormalDist()
    return nd.inv_cdf(1.0 - keep) - nd.inv_cdf(1.0 - p)


class _Layout:
    """Writes rows of one (b, g) into a contiguous or paged cache."""

    def __init__(self, case: Case):
        self.c = case

    def put(self, arr: np.ndarray, b: int, g: int, pos: np.ndarray, rows: np.ndarray):
        if self.c.block_table is None:
            arr[b, g, pos, :] = rows
        else:
            pages = self.c.block_table[b, pos // BLK]
            arr[pages, g, pos % BLK, :] = rows

    def get(self, arr: np.ndarray, b: int, g: int, pos: np.ndarray) -> np.ndarray:
        if self.c.block_table is None:
            return arr[b, g, pos, :]
        pages = self.c.block_table[b, pos // BLK]
        return arr[pages, g, pos % BLK, :]


def _q_idx(Wq_bf16: np.ndarray, q_bf16: np.ndarray) -> np.ndarray:
    """Projected query W^Q q^pre in fp64 (used only to aim planted tokens)."""
    return from_bf16(Wq_bf16).reshape(R, D) @ from_bf16(q_bf16).reshape(D)


def _retarget_rows(case: Case, lay: _Layout, b: int, g: int, pos: np.ndarray, targets: np.ndarray,
                   Wk: np.ndarray, seed: int):
    """Give tokens `pos` the index keys `targets` (fp64 [n,16]); their pre-RoPE
    keys get the minimal-norm change that makes W^K k^pre hit the target, and
    their RoPE'd cache rows are rebuilt from it."""
    _, _, kpre = keys_for(seed, stream_id("k", b, g), pos, None, False, want_kpre=True)
    W = from_bf16(Wk).reshape(R, D)
    kp = from_bf16(kpre)                                   # [n,128]
    resid = targets - kp @ W.T                             # [n,16]
    delta = (W.T @ np.linalg.solve(W @ W.T, resid.T)).T    # [n,128]
    kpre_new = to_bf16(kp + delta)
    lay.put(case.k_cache, b, g, pos, rope_rows(kpre_new, pos))
    lay.put(case.k_idx, b, g, pos, to_bf16(targets))


def make_case(name: str, *, B: int, Hkv: int, G: int, seq_lens: Sequence[int], ret_groups: Sequence[int],
              p: Sequence[float], window: int, sink: int, seed: int, regimes: Sequence[str],
              paged: bool = False, shared_heads: bool = False, head_kind: Optional[np.ndarray] = None,
              n_needles: int = 0, needle_mode: str = "per_head", needle_norm: float = 4.0,
              needle_range: Optional[Tuple[int, int]] = None, cluster: int = 0,
              cluster_sigma: float = 1.5, keep_fraction: float = 0.15, ncap: Optional[int] = None,
              poison: bool = True) -> Case:
    """Build one decode-step workload.

    regimes[b] in {"gaussian", "needle", "diffuse", "needles4x"}:
      gaussian  - plain N(0,1) q/k/v; scores s/4 ~ N(0, ~1)
      needle    - one token per retrieval group whose index key sits along the
                  direction equally aligned with all the group's projected
                  queries (min-norm solution of qhat_h . u = const), sized so that its
                  score beats the Cauchy-Schwarz bound of every other token's
                  score by 4 ln(99 L): it alone carries >= 0.99 of each head's
                  softmax(s/4) mass
      diffuse   - retrieval heads' q^pre scaled so the score std reaches
                  sigma_for_keep_fraction(p, keep_fraction)
      needles4x - `n_needles` planted tokens at `needle_norm` x the RMS row
                  norm of k_idx along a projected-query direction
                  (needle_mode "per_head": n_needles per retrieval head, each
                  along that head's direction; "shared": n_needles along head
                  0's), plus an optional contiguous cluster of `cluster`
                  tokens shifted by +cluster_sigma score std along the group's
                  mean direction.
    Everything the step may not read (rows >= L, local-only groups outside
    sink+window, k_idx of local-only groups) is NaN when `poison`.
    """
    Hq = Hkv * G
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    assert seq_lens.shape == (B,)
    hk = head_kind if head_kind is not None else head_kind_for(Hkv, G, ret_groups)
    hk = np.asarray(hk, dtype=np.uint8)
    ret_group_set = sorted({h // G for h in range(Hq) if hk[h]})
    pvec = np.asarray(p, dtype=np.float32)
    Lmax = int(seq_lens.max())
    if ncap is None:
        ncap = ((Lmax + BLK - 1) // BLK) * BLK

    # ---- layout ----
    block_table = None
    num_pages = 0
    if paged:
        nblk = [(int(L) + BLK - 1) // BLK for L in seq_lens]
        mbps = max(nblk)
        num_pages = int(sum(nblk))
        perm = np.argsort(uniform_f64(seed, stream_id("misc", 1), num_pages), kind="stable").astype(np.int32)
        block_table = np.full((B, mbps), -1, dtype=np.int32)
        off = 0
        for b in range(B):
            block_table[b, :nblk[b]] = perm[off:off + nblk[b]]
            off += nblk[b]
        kshape = (num_pages, Hkv, BLK, D)
        ishape = (num_pages, Hkv, BLK, R)
        ncap = mbps * BLK
    else:
        kshape = (B, Hkv, ncap, D)
        ishape = (B, Hkv, ncap, R)
    fill = nan_fill if poison else (lambda s: np.zeros(s, dtype=np.uint16))
    k_cache = fill(kshape)
    v_cache = fill(kshape)
    k_idx = fill(ishape)

    # ---- weights and queries ----
    Wq = np.empty((Hq, R, D), dtype=np.uint16)
    for h in range(Hq):
        Wq[h] = normal_bf16(seed, stream_id("Wq", 0 if shared_heads else h), R * D, 1.0 / math.sqrt(D)).reshape(R, D)
    Wk = np.empty((Hkv, R, D), dtype=np.uint16)
    for g in range(Hkv):
        Wk[g] = normal_bf16(seed, stream_id("Wk", g), R * D, 1.0 / math.sqrt(D)).reshape(R, D)
    q_pre = np.empty((B, Hq, D), dtype=np.uint16)
    for b in range(B):
        for h in range(Hq):
            q_pre[b, h] = normal_bf16(seed, stream_id("q", b, 0 if shared_heads else h), D)

    case = Case(name=name, B=B, Hq=Hq, Hkv=Hkv, Ncap=int(ncap), seq_lens=seq_lens, head_kind=hk, p=pvec,
                window=int(window), sink=int(sink), q_pre=q_pre, q_rope=q_pre.copy(), Wq_idx=Wq,
                k_idx=k_idx, k_cache=k_cache, v_cache=v_cache, block_table=block_table,
                num_pages=num_pages, regimes=list(regimes), seed=seed)
    lay = _Layout(case)

    # ---- caches ----
    for b in range(B):
        L = int(seq_lens[b])
        for g in range(Hkv):
            if g in ret_group_set:
                pos = np.arange(L, dtype=np.int64)
            else:
                pos = local_positions(L, window, sink)
            if pos.size == 0:
                continue
            kc, ki, _ = keys_for(seed, stream_id("k", b, g), pos, Wk[g] if g in ret_group_set else None,
                                 g in ret_group_set)
            lay.put(k_cache, b, g, pos, kc)
            if ki is not None:
                lay.put(k_idx, b, g, pos, ki)
            lay.put(v_cache, b, g, pos, values_for(seed, stream_id("v", b, g), pos))

    # ---- score-shaping regimes (retrieval groups only) ----
    for b in range(B):
        L = int(seq_lens[b])
        reg = regimes[b]
        lo, hi = needle_range if needle_range is not None else (min(sink, L), max(min(sink, L) + 1, L - window))
        hi = max(hi, lo + 1)
        for g in ret_group_set:
            heads = [h for h in range(g * G, (g + 1) * G) if hk[h]]
            allpos = np.arange(L, dtype=np.int64)
            kid = lay.get(k_idx, b, g, allpos)
            rms_norm, max_norm = kidx_stats(np.ascontiguousarray(kid))
            rms_comp = rms_norm / math.sqrt(R)
            qidx = {h: _q_idx(Wq[h], q_pre[b, h]) for h in heads}
            qhat = {h: qidx[h] / np.linalg.norm(qidx[h]) for h in heads}
            # direction equally aligned with every head's projected query:
            # min-norm solution of qhat_h . u' = 1 for all heads, normalised
            Qh = np.stack([qhat[h] for h in heads])
            u = np.linalg.lstsq(Qh, np.ones(len(heads)), rcond=None)[0]
            u = u / np.linalg.norm(u)
            ms = stream_id("pos", b, g)
            if reg == "needle":
                n_star = lo + int(uniform_f64(seed, ms, 1)[0] * (hi - lo))
                n_star = min(n_star, hi - 1)
                margin = 4.0 * math.log(99.0 * L)
                cs = []
                for h in heads:
                    a = float(qidx[h] @ u)
                    if a <= 1e-3 * np.linalg.norm(qidx[h]):
                        raise ValueError(f"needle direction degenerate for head {h}")
                    cs.append((margin + np.linalg.norm(qidx[h]) * max_norm) / a)
                c = 1.02 * max(cs)
                _retarget_rows(case, lay, b, g, np.array([n_star]), (c * u)[None, :], Wk[g], seed)
                for h in heads:
                    case.needles.setdefault((b, h), []).append(n_star)
            elif reg == "diffuse":
                sig = sigma_for_keep_fraction(float(pvec[b]), keep_fraction)
                for h in heads:
                    alpha = 4.0 * sig / (np.linalg.norm(qidx[h]) * rms_comp)
                    q_pre[b, h] = to_bf16(alpha * from_bf16(q_pre[b, h]))
            elif reg == "needles4x":
                if cluster > 0:
                    c0 = lo + int(uniform_f64(seed, ms, 1, offset=7)[0] * max(1, hi - lo - cluster))
                    cpos = np.arange(c0, min(c0 + cluster, L), dtype=np.int64)
                    shift = cluster_sigma * rms_comp / float(np.mean([qhat[h] @ u for h in heads]))
                    tgt = from_bf16(lay.get(k_idx, b, g, cpos)) + shift * u[None, :]
                    _retarget_rows(case, lay, b, g, cpos, tgt, Wk[g], seed)
                aims = heads if needle_mode == "per_head" else [heads[0]]
                cnt = 0
                plist, tlist = [], []
                taken = set()
                if hi - lo < len(aims) * n_needles:
                    raise ValueError(f"needle range [{lo}, {hi}) holds fewer than {len(aims) * n_needles} positions")
                for h in aims:
                    for i in range(n_needles):
                        while True:
                            r = uniform_f64(seed, ms, 1, offset=100 + cnt)[0]
                            cnt += 1
                            n = min(lo + int(r * (hi - lo)), hi - 1)
                            if n not in taken:
                                break
                        taken.add(n)
                        plist.append(n)
                        tlist.append(needle_norm * rms_norm * qhat[h])
                        owners = heads if needle_mode == "shared" else [h]
                        for hh in owners:
                            case.needles.setdefault((b, hh), []).append(n)
                _retarget_rows(case, lay, b, g, np.array(plist, dtype=np.int64), np.array(tlist), Wk[g], seed)
            elif reg == "gaussian":
                pass
            else:
                raise ValueError(f"unknown regime {reg}")

    # ---- RoPE'd queries at position L ----
    for b in range(B):
        case.q_rope[b] = rope_rows(q_pre[b], np.full(Hq, int(seq_lens[b]), dtype=np.int64))
    case.q_pre = q_pre
    return case


# ----------------------------------------------------------------------------
# The five workloads of the decode step (seeds: workload i uses seed i-1)
# ----------------------------------------------------------------------------
WORKLOADS = {
    1: "tiny 4K: B=1, L=4096, 1 KV head x GQA 4, heads 0-1 retrieval (p=0.9), 2-3 local (sink 4, window 512), shared q/Wq, 3 needles at 4x norm",
    2: "32K: B=1, L=32768, 8 KV x GQA 4, KV group 0 retrieval (p=0.9), 28 local (sink 4, window 2048), 16 needles + 2000-token cluster at +1.5 sigma",
    3: "4x128K: B=4, L=131072, 8 KV x GQA 8, KV groups 0-1 retrieval (p=0.95), 48 local (sink 4, window 4096); needle, needle, diffuse, gaussian",
    4: "1M: B=1, L=1048576, 8 KV x GQA 4, KV group 0 retrieval (p=0.9), 28 local (sink 4, window 4096), needle-peaked",
    5: "ragged paged x16: L log-uniform in [8192, 262144], 8 KV x GQA 4, 1-2 retrieval KV groups, p in {0.8,0.9,0.95}, regimes needle/diffuse/gaussian, sink 4, window 2048",
}


def ragged_lengths(seed: int, B: int, lo: int, hi: int) -> np.ndarray:
    u = uniform_f64(seed, stream_id("len", 0), B)
    return np.floor(np.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))).astype(np.int32)


def workload(i: int, scale: int = 1, poison: bool = True) -> Case:
    """Workload i (1..5).  `scale` > 1 divides every context length by it
    (same structure, smaller, for tests the oracle must finish quickly)."""
    seed = i - 1
    if i == 1:
        L = 4096 // scale
        return make_case("w1-tiny-4k", B=1, Hkv=1, G=4, seq_lens=[L], ret_groups=[0],
                         head_kind=np.array([1, 1, 0, 0], dtype=np.uint8), p=[0.9], window=512 // min(scale, 8),
                         sink=4, seed=seed, regimes=["needles4x"], shared_heads=True, n_needles=3,
                         needle_mode="shared", needle_range=(4, max(5, L - 512 // min(scale, 8))), poison=poison)
    if i == 2:
        L = 32768 // scale
        return make_case("w2-32k", B=1, Hkv=8, G=4, seq_lens=[L], ret_groups=[0], p=[0.9],
                         window=2048 // min(scale, 8), sink=4, seed=seed, regimes=["needles4x"], n_needles=4,
                         needle_mode="per_head", cluster=2000 // scale, poison=poison)
    if i == 3:
        L = 131072 // scale
        return make_case("w3-4x128k", B=4, Hkv=8, G=8, seq_lens=[L] * 4, ret_groups=[0, 1], p=[0.95] * 4,
                         window=4096 // min(scale, 8), sink=4, seed=seed,
                         regimes=["needle", "needle", "diffuse", "gaussian"], poison=poison)
    if i == 4:
        L = 1048576 // scale
        return make_case("w4-1m", B=1, Hkv=8, G=4, seq_lens=[L], ret_groups=[0], p=[0.9],
                         window=4096 // min(scale, 8), sink=4, seed=seed, regimes=["needle"], poison=poison)
    if i == 5:
        B = 16
        lens = ragged_lengths(seed, B, 8192 // scale, 262144 // scale)
        u = uniform_f64(seed, stream_id("misc", 5), 2 + 8 + 2 * B)
        n_ret = 1 + int(u[0] * 2)
        order = np.argsort(u[2:10], kind="stable")
        ret_groups = sorted(int(g) for g in order[:n_ret])
        pchoice = [0.8, 0.9, 0.95]
        rchoice = ["needle", "diffuse", "gaussian"]
        ps = [pchoice[min(2, int(x * 3))] for x in u[10:10 + B]]
        regs = [rchoice[min(2, int(x * 3))] for x in u[10 + B:10 + 2 * B]]
        return make_case("w5-ragged-paged", B=B, Hkv=8, G=4, seq_lens=lens, ret_groups=ret_groups, p=ps,
                         window=2048 // min(scale, 8), sink=4, seed=seed, regimes=regs, paged=True, poison=poison)
    raise ValueError(i)


def integer_case(seed: int, *, B: int = 2, Hkv: int = 2, G: int = 4, L: int = 700, p: float = 0.9,
                 window: int = 64, sink: int = 4, ret_groups: Sequence[int] = (0,), paged: bool = False,
                 qmax: int = 3, kmax: int = 2) -> Case:
    """Integer-valued index scores: W^Q = [I_16 | 0], the first 16 entries of
    q^pre integers in [-qmax, qmax], k_idx entries integers in [-kmax, kmax]
    (set directly).  Every score is an integer, exact in fp32 and fp64, and
    ties are plentiful."""
    case = make_case(f"int-{seed}", B=B, Hkv=Hkv, G=G, seq_lens=[L] * B, ret_groups=ret_groups, p=[p] * B,
                     window=window, sink=sink, seed=seed, regimes=["gaussian"] * B, paged=paged)
    Wq = np.zeros((case.Hq, R, D), dtype=np.float64)
    Wq[:, np.arange(R), np.arange(R)] = 1.0
    case.Wq_idx = to_bf16(Wq)
    lay = _Layout(case)
    for b in range(B):
        for h in range(case.Hq):
            u = uniform_f64(seed, stream_id("int", b, h), R)
            q = from_bf16(case.q_pre[b, h])
            q[:R] = np.floor(u * (2 * qmax + 1)) - qmax
            case.q_pre[b, h] = to_bf16(q)
        for g in sorted({h // G for h in range(case.Hq) if case.head_kind[h]}):
            u = uniform_f64(seed, stream_id("int", b, 1000 + g), L * R).reshape(L, R)
            lay.put(case.k_idx, b, g, np.arange(L, dtype=np.int64), to_bf16(np.floor(u * (2 * kmax + 1)) - kmax))
        case.q_rope[b] = rope_rows(case.q_pre[b], np.full(case.Hq, L, dtype=np.int64))
    return case
