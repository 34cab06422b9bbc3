"""fp64 CPU oracle for the RTPurbo decode step -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path (the CUDA library and its
binding) never loads it and shares no code with it.

The arithmetic lives in ``rtp_oracle.c`` (plain C, fp64), which states what
it computes and which passage of the RTPurbo pages each step follows.  This
module compiles it with gcc and marshals numpy arrays.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(brute force, closed forms, invariants and hand-derived fixtures under
``tests/golden/``); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rtp_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
D, R, BLK = 128, 16, 64


def build(force: bool = False) -> str:
    """Compile rtp_oracle.c into liboracle.so (gcc -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i32, i64, dbl, vp = ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        lib.oracle_rope.argtypes = [vp, i64, dbl, vp]
        lib.oracle_topp.argtypes = [vp, i64, dbl, vp, vp, vp, vp, vp, vp]
        lib.oracle_topp.restype = i32
        lib.oracle_index_scores.argtypes = [i32, i32, i32, i64, vp, i32, vp, vp, vp, i32, i32, i64, vp]
        lib.oracle_attend.argtypes = [i32, i32, i32, i64, vp, i32, vp, vp, vp, i32, i32, vp, i64, vp]
        lib.oracle_decode_step.argtypes = [i32, i32, i32, i64, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32,
                                           i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, i64]
        lib.oracle_decode_step.restype = i32
        lib.oracle_index_append.argtypes = [i32, i32, i64, vp, i32, vp, i32, vp, vp, vp]
        lib.oracle_kv_append.argtypes = [i32, i32, i64, vp, i32, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp]
        lib.oracle_prefill.argtypes = [i32, i32, i32, i64, vp, i32, vp, vp, vp, vp, vp, i32, i32, i32, vp]
        lib.oracle_ring_row.argtypes = [i64, i32, i32]
        lib.oracle_ring_row.restype = i64
        lib.oracle_ring_write.argtypes = [i32, i32, i32, i32, vp, vp, i32, vp, vp, vp]
        lib.oracle_attend_ring.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, i32, i32, i64, i32, i32, vp]
        lib.oracle_attend_ring.restype = i32
        lib.oracle_topk.argtypes = [vp, i64, i64, vp, vp]
        lib.oracle_topk.restype = i32
        lib.oracle_decode_step_topk.argtypes = [i32, i32, i32, i64, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, i64, i32,
                                                i32, i32, vp, vp, vp, vp, i64]
        lib.oracle_decode_step_topk.restype = i32
        lib.oracle_bf16_rne.argtypes = [dbl]
        lib.oracle_bf16_rne.restype = ctypes.c_uint16
        _lib = lib
    return _lib


def _p(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def rope(x: np.ndarray, pos: int, theta: float = 1.0e6) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64).reshape(D)
    y = np.empty(D, dtype=np.float64)
    _L().oracle_rope(_p(x), int(pos), float(theta), _p(y))
    return y


def topp(s: np.ndarray, p: float) -> Dict[str, object]:
    """Dynamic Top-P on raw index scores s (temperature 4 = sqrt(16))."""
    s = np.ascontiguousarray(s, dtype=np.float64)
    L = s.size
    order = np.empty(L, dtype=np.int64)
    k = ctypes.c_int64()
    zm, Z, cb, ca = (ctypes.c_double() for _ in range(4))
    rc = _L().oracle_topp(_p(s), L, float(p), _p(order), ctypes.byref(k), ctypes.byref(zm), ctypes.byref(Z),
                          ctypes.byref(cb), ctypes.byref(ca))
    if rc != 0:
        raise ValueError(f"oracle_topp rc={rc}")
    return {"order": order, "kstar": int(k.value), "kept": np.sort(order[:k.value]), "zmax": zm.value, "Z": Z.value,
            "cum_before": cb.value, "cum_at": ca.value}


def topk(s: np.ndarray, k: int) -> Dict[str, object]:
    """Static Top-K on raw index scores s: the first min(k, L) tokens under
    (s desc, n asc)."""
    s = np.ascontiguousarray(s, dtype=np.float64)
    L = s.size
    order = np.empty(L, dtype=np.int64)
    kk = ctypes.c_int64()
    rc = _L().oracle_topk(_p(s), L, int(k), _p(order), ctypes.byref(kk))
    if rc != 0:
        raise ValueError(f"oracle_topk rc={rc}")
    return {"order": order, "kstar": int(kk.value), "kept": np.sort(order[:kk.value])}


def _geom(case):
    bt = None if case.block_table is None else np.ascontiguousarray(case.block_table, dtype=np.int32)
    return (case.B, case.Hq, case.Hkv, int(case.Ncap), bt, case.max_blocks_per_seq)


def index_scores(case, b: int, h: int) -> np.ndarray:
    B, Hq, Hkv, Ncap, bt, mbps = _geom(case)
    L = int(case.seq_lens[b])
    s = np.empty(L, dtype=np.float64)
    _L().oracle_index_scores(B, Hq, Hkv, Ncap, _p(bt), mbps, _p(case.q_pre), _p(case.Wq_idx), _p(case.k_idx),
                             b, h, L, _p(s))
    return s


def attend(case, b: int, h: int, positions: np.ndarray) -> np.ndarray:
    """Exact softmax attention of (b, h) over an arbitrary position set."""
    B, Hq, Hkv, Ncap, bt, mbps = _geom(case)
    pos = np.ascontiguousarray(np.sort(np.asarray(positions, dtype=np.int64)))
    out = np.empty(D, dtype=np.float64)
    _L().oracle_attend(B, Hq, Hkv, Ncap, _p(bt), mbps, _p(case.q_rope), _p(case.k_cache), _p(case.v_cache), b, h,
                       _p(pos), pos.size, _p(out))
    return out


def decode_step(case, nthreads: int = 0) -> Dict[str, np.ndarray]:
    """The whole decode step in fp64.  Returns out [B,Hq,128] and, per (b,h),
    kstar, tau, zmax, Z, cum_before, cum_at, next_s and kept_blocks
    [B,Hq,nblk_cap] (uint8)."""
    B, Hq, Hkv, Ncap, bt, mbps = _geom(case)
    BH = B * Hq
    nblk = (Ncap + BLK - 1) // BLK
    res = {
        "out": np.zeros((B, Hq, D), dtype=np.float64),
        "kstar": np.zeros((B, Hq), dtype=np.int64),
        "tau": np.full((B, Hq), np.nan),
        "zmax": np.full((B, Hq), np.nan),
        "Z": np.full((B, Hq), np.nan),
        "cum_before": np.full((B, Hq), np.nan),
        "cum_at": np.full((B, Hq), np.nan),
        "next_s": np.full((B, Hq), np.nan),
        "kept_blocks": np.zeros((B, Hq, nblk), dtype=np.uint8),
    }
    hk = np.ascontiguousarray(case.head_kind, dtype=np.uint8)
    rc = _L().oracle_decode_step(B, Hq, Hkv, Ncap, _p(bt), mbps, _p(case.q_pre), _p(case.q_rope), _p(case.k_idx),
                                 _p(case.k_cache), _p(case.v_cache), _p(case.Wq_idx),
                                 _p(np.ascontiguousarray(case.seq_lens, dtype=np.int32)), _p(hk),
                                 _p(np.ascontiguousarray(case.p, dtype=np.float32)), int(case.window), int(case.sink),
                                 int(nthreads), _p(res["out"]), _p(res["kstar"]), _p(res["tau"]), _p(res["zmax"]),
                                 _p(res["Z"]), _p(res["cum_before"]), _p(res["cum_at"]), _p(res["next_s"]),
                                 _p(res["kept_blocks"]), nblk)
    res["rc"] = rc
    return res


def decode_step_topk(case, k: int, nthreads: int = 0) -> Dict[str, np.ndarray]:
    """The decode step with every retrieval head keeping its static top-k
    (case.p unused).  Returns out, kstar, tau and kept_blocks."""
    B, Hq, Hkv, Ncap, bt, mbps = _geom(case)
    nblk = (Ncap + BLK - 1) // BLK
    res = {
        "out": np.zeros((B, Hq, D), dtype=np.float64),
        "kstar": np.zeros((B, Hq), dtype=np.int64),
        "tau": np.full((B, Hq), np.nan),
        "kept_blocks": np.zeros((B, Hq, nblk), dtype=np.uint8),
    }
    hk = np.ascontiguousarray(case.head_kind, dtype=np.uint8)
    rc = _L().oracle_decode_step_topk(B, Hq, Hkv, Ncap, _p(bt), mbps, _p(case.q_pre), _p(case.q_rope),
                                      _p(case.k_idx), _p(case.k_cache), _p(case.v_cache), _p(case.Wq_idx),
                                      _p(np.ascontiguousarray(case.seq_lens, dtype=np.int32)), _p(hk), int(k),
                                      int(case.window), int(case.sink), int(nthreads), _p(res["out"]),
                                      _p(res["kstar"]), _p(res["tau"]), _p(res["kept_blocks"]), nblk)
    res["rc"] = rc
    return res


def kv_append(k_pre: np.ndarray, v_new: np.ndarray, Wk: np.ndarray, rope_cos: np.ndarray, rope_sin: np.ndarray,
              pos: np.ndarray, k_idx: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
              block_table: Optional[np.ndarray] = None):
    """The KV-cache write of new tokens with the index-cache append: rows
    n = pos[b] + t of KV head g get k_idx = bf16(W^K_g k^pre), k_cache =
    bf16(RoPE_n(k^pre)) (pairs (i, i+64) rotated by rope_cos/rope_sin row n,
    fp32 [positions, 64]) and v_cache = v_new.  k_pre, v_new: uint16 (bf16)
    [B, Hkv, T, 128]; caches contiguous [B, Hkv, Ncap, dim] or, with
    block_table, paged [pages, Hkv, 64, dim].  Returns updated copies
    (k_idx, k_cache, v_cache)."""
    k_pre = np.ascontiguousarray(k_pre, dtype=np.uint16)
    v_new = np.ascontiguousarray(v_new, dtype=np.uint16)
    Wk = np.ascontiguousarray(Wk, dtype=np.uint16)
    rc = np.ascontiguousarray(rope_cos, dtype=np.float32)
    rs = np.ascontiguousarray(rope_sin, dtype=np.float32)
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    outs = [np.array(a, dtype=np.uint16, copy=True, order="C") for a in (k_idx, k_cache, v_cache)]
    B, Hkv, T = k_pre.shape[:3]
    if block_table is None:
        ncap, bt, mbps = outs[0].shape[2], None, 0
    else:
        bt = np.ascontiguousarray(block_table, dtype=np.int32)
        mbps = bt.shape[1]
        ncap = mbps * BLK
    if int(pos.min()) < 0 or int(pos.max()) + T > ncap or rc.shape != rs.shape or rc.shape[0] < ncap:
        raise ValueError("kv_append: positions beyond the cache or the angle table")
    _L().oracle_kv_append(B, Hkv, ncap, _p(bt), mbps, _p(k_pre), _p(v_new), T, _p(Wk), _p(rc), _p(rs), _p(pos),
                          _p(outs[0]), _p(outs[1]), _p(outs[2]))
    return tuple(outs)


def prefill(case, q: np.ndarray, pos: np.ndarray) -> np.ndarray:
    """Prefill attention of T queries per sequence (q: uint16 bf16 [B, Hq, T,
    128], RoPE'd) at positions pos[b] + t, over the case's caches: retrieval
    heads attend to [0, m], local heads to the sink and the last `window`
    positions up to m.  Returns out [B, Hq, T, 128] fp64."""
    B, Hq, Hkv, Ncap, bt, mbps = _geom(case)
    q = np.ascontiguousarray(q, dtype=np.uint16)
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    T = q.shape[2]
    if q.shape[:2] != (B, Hq) or int(pos.min()) < 0 or int(pos.max()) + T > Ncap:
        raise ValueError("prefill: query shape or positions beyond the cache")
    out = np.empty((B, Hq, T, D), dtype=np.float64)
    _L().oracle_prefill(B, Hq, Hkv, Ncap, _p(bt), mbps, _p(q), _p(case.k_cache), _p(case.v_cache),
                        _p(np.ascontiguousarray(case.head_kind, dtype=np.uint8)), _p(pos), T, int(case.window),
                        int(case.sink), _p(out))
    return out


def ring_row(n: int, S0: int, W: int) -> int:
    """Row of position n in a local head's ring of S0 + W rows."""
    return int(_L().oracle_ring_row(int(n), int(S0), int(W)))


def ring_write(k_new: np.ndarray, v_new: np.ndarray, pos: np.ndarray, k_ring: np.ndarray, v_ring: np.ndarray,
               S0: int, W: int):
    """Rings [B, Hkv, S0 + W, 128] (uint16 bf16) after writing the new rows
    [B, Hkv, T, 128] of positions pos[b] + t in order.  Returns updated copies."""
    k_new = np.ascontiguousarray(k_new, dtype=np.uint16)
    v_new = np.ascontiguousarray(v_new, dtype=np.uint16)
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    kr = np.array(k_ring, dtype=np.uint16, copy=True, order="C")
    vr = np.array(v_ring, dtype=np.uint16, copy=True, order="C")
    B, Hkv, T = k_new.shape[:3]
    if kr.shape != (B, Hkv, S0 + W, D) or vr.shape != kr.shape or W < 1 or S0 < 0 or int(pos.min()) < 0:
        raise ValueError("ring_write: ring shape, W, S0 or positions")
    _L().oracle_ring_write(B, Hkv, S0, W, _p(k_new), _p(v_new), T, _p(pos), _p(kr), _p(vr))
    return kr, vr


def attend_ring(q_rope: np.ndarray, k_ring: np.ndarray, v_ring: np.ndarray, b: int, h: int, L: int, window: int,
                sink: int, S0: int, W: int) -> np.ndarray:
    """Local head h of sequence b at length L (sink <= S0, window <= W), its
    keys and values read from the rings."""
    q = np.ascontiguousarray(q_rope, dtype=np.uint16)
    kr = np.ascontiguousarray(k_ring, dtype=np.uint16)
    vr = np.ascontiguousarray(v_ring, dtype=np.uint16)
    B, Hq = q.shape[:2]
    Hkv = kr.shape[1]
    out = np.empty(D, dtype=np.float64)
    rc = _L().oracle_attend_ring(B, Hq, Hkv, S0, W, _p(q), _p(kr), _p(vr), b, h, int(L), int(window), int(sink),
                                 _p(out))
    if rc != 0:
        raise ValueError("attend_ring: sink beyond S0 or window beyond W")
    return out


def bf16_rne(x: float) -> int:
    """The bf16 bit pattern nearest to x (ties to the even significand)."""
    return int(_L().oracle_bf16_rne(float(x)))


def index_append(k_pre: np.ndarray, Wk: np.ndarray, pos: np.ndarray, k_idx: np.ndarray,
                 block_table: Optional[np.ndarray] = None) -> np.ndarray:
    """k_idx rows pos[b] + t of KV head g <- bf16(W^K_g k^pre[b, g, t]).

    k_pre: uint16 (bf16) [B, Hkv, T, 128]; Wk: uint16 [Hkv, 16, 128]; pos:
    int32 [B]; k_idx: the cache, uint16, contiguous [B, Hkv, Ncap, 16] or,
    with block_table int32 [B, max_blocks], paged [pages, Hkv, 64, 16].
    Returns an updated copy of k_idx."""
    k_pre = np.ascontiguousarray(k_pre, dtype=np.uint16)
    Wk = np.ascontiguousarray(Wk, dtype=np.uint16)
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    out = np.array(k_idx, dtype=np.uint16, copy=True, order="C")
    B, Hkv, T = k_pre.shape[:3]
    if block_table is None:
        ncap, bt, mbps = out.shape[2], None, 0
    else:
        bt = np.ascontiguousarray(block_table, dtype=np.int32)
        mbps = bt.shape[1]
        ncap = mbps * BLK
    _L().oracle_index_append(B, Hkv, ncap, _p(bt), mbps, _p(k_pre), T, _p(Wk), _p(pos), _p(out))
    return out

