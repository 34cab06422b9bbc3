"""Pins for the fp64 oracle: brute force, closed forms, invariants and
hand-derived fixtures (tests/golden/).  CPU only."""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------------------
# a hand-built case: explicit q/k/v, contiguous layout
# ----------------------------------------------------------------------------
def hand_case(L, *, Hkv=1, G=1, head_kind=None, p=0.9, window=4, sink=1, seed=0, q_rope=None, k_cache=None,
              v_cache=None, k_idx=None, q_pre=None, Wq=None):
    Hq = Hkv * G
    ncap = ((L + 63) // 64) * 64
    rng = np.random.default_rng(seed)
    hk = np.ones(Hq, np.uint8) if head_kind is None else np.asarray(head_kind, np.uint8)

    def bf(x):
        return synth.to_bf16(np.asarray(x, np.float64))

    kc = synth.nan_fill((1, Hkv, ncap, 128))
    vc = synth.nan_fill((1, Hkv, ncap, 128))
    ki = synth.nan_fill((1, Hkv, ncap, 16))
    kc[:, :, :L] = bf(rng.standard_normal((1, Hkv, L, 128)) if k_cache is None else k_cache)
    vc[:, :, :L] = bf(rng.standard_normal((1, Hkv, L, 128)) if v_cache is None else v_cache)
    ki[:, :, :L] = bf(rng.standard_normal((1, Hkv, L, 16)) if k_idx is None else k_idx)
    qp = bf(rng.standard_normal((1, Hq, 128)) if q_pre is None else q_pre)
    qr = bf(rng.standard_normal((1, Hq, 128)) if q_rope is None else q_rope)
    W = bf(rng.standard_normal((Hq, 16, 128)) / math.sqrt(128) if Wq is None else Wq)
    return synth.Case(name="hand", B=1, Hq=Hq, Hkv=Hkv, Ncap=ncap, seq_lens=np.array([L], np.int32), head_kind=hk,
                      p=np.array([p], np.float32), window=window, sink=sink, q_pre=qp, q_rope=qr, Wq_idx=W, k_idx=ki,
                      k_cache=kc, v_cache=vc)


# ----------------------------------------------------------------------------
# Top-P
# ----------------------------------------------------------------------------
def brute_force_topp(s, p):
    """Smallest cardinality of a token set whose softmax(s/4) mass reaches p,
    and among those sets the one of largest mass, ties to the lexicographically
    smallest sorted index list -- by enumerating every subset."""
    n = len(s)
    w = np.exp(np.asarray(s) / 4.0 - np.max(s) / 4.0)
    w = w / w.sum()
    for k in range(1, n + 1):
        best = None
        for sub in itertools.combinations(range(n), k):
            m = sum(w[i] for i in sub)
            if m >= p - 1e-12:
                key = (-round(m, 12), sub)
                if best is None or key < best[0]:
                    best = (key, sub)
        if best is not None:
            return k, list(best[1])
    return n, list(range(n))


@pytest.mark.parametrize("trial", range(60))
def test_topp_matches_brute_force(trial):
    rng = np.random.default_rng(1000 + trial)
    n = int(rng.integers(1, 11))
    if trial % 3 == 0:
        s = rng.integers(-3, 4, n).astype(np.float64) * 2.0          # many ties
    else:
        s = rng.standard_normal(n) * rng.uniform(0.5, 8.0)
    w = np.exp(s / 4 - s.max() / 4)
    w /= w.sum()
    cums = np.cumsum(np.sort(w)[::-1])
    while True:
        p = float(rng.uniform(0.05, 0.999))
        if np.min(np.abs(cums - p)) > 1e-6:
            break
    r = oracle.topp(s, p)
    k_bf, set_bf = brute_force_topp(s, p)
    assert r["kstar"] == k_bf
    assert sorted(r["kept"].tolist()) == set_bf


def test_topp_golden():
    for case in load("topp_hand.json")["cases"]:
        for chk in case["checks"]:
            r = oracle.topp(np.array(case["s"]), chk["p"])
            assert r["kstar"] == chk["kstar"], (case["scores"], chk)
            assert r["kept"].tolist() == chk["kept"], (case["scores"], chk)


@pytest.mark.parametrize("L,p", [(1000, 0.3337), (1000, 0.9001), (777, 0.5555), (64, 0.01)])
def test_topp_all_equal_closed_form(L, p):
    r = oracle.topp(np.full(L, 2.5), p)
    k = math.ceil(p * L)
    assert r["kstar"] == k
    assert r["kept"].tolist() == list(range(k))          # ties toward the lower index


@pytest.mark.parametrize("a,b,L,p", [(40.0, 0.0, 5000, 0.9), (20.0, 1.0, 3000, 0.8), (30.0, -2.0, 100000, 0.95),
                                     (8.0, 0.0, 100, 0.5)])
def test_topp_one_peak_closed_form(a, b, L, p):
    s = np.full(L, b)
    pos = L // 3
    s[pos] = a
    m1 = math.exp(a / 4) / (math.exp(a / 4) + (L - 1) * math.exp(b / 4))
    m0 = math.exp(b / 4) / (math.exp(a / 4) + (L - 1) * math.exp(b / 4))
    k = 1 if m1 >= p else 1 + math.ceil((p - m1) / m0)
    r = oracle.topp(s, p)
    assert r["kstar"] == k
    expect = sorted({pos} | set([i for i in range(L) if i != pos][:k - 1]))
    assert r["kept"].tolist() == expect


def test_topp_p_one_and_invalid():
    s = np.random.default_rng(3).standard_normal(500)
    r = oracle.topp(s, 1.0)
    assert r["kstar"] == 500
    assert abs(r["cum_at"] - 1.0) < 1e-12                 # softmax mass sums to 1
    r = oracle.topp(s, 1.5)
    assert r["kstar"] == 500
    for bad in (0.0, -0.1, float("nan")):
        with pytest.raises(ValueError):
            oracle.topp(s, bad)


def test_softmax_normaliser():
    rng = np.random.default_rng(5)
    s = rng.standard_normal(10000) * 9
    r = oracle.topp(s, 1.0)
    z = s / 4
    assert abs(r["zmax"] - z.max()) == 0
    # Z = sum exp(z - zmax): compare against a log-sum-exp computed in sorted order
    zs = np.sort(z - z.max())
    assert abs(r["Z"] - math.fsum(np.exp(zs))) < 1e-12 * r["Z"]
    assert abs(r["cum_at"] - 1.0) < 1e-12


# ----------------------------------------------------------------------------
# RoPE
# ----------------------------------------------------------------------------
def test_rope_golden():
    for c in load("rope_hand.json")["cases"]:
        x = np.zeros(128)
        x[c["i"]] = 1.0
        y = oracle.rope(x, c["pos"])
        assert abs(y[c["i"]] - c["y_i"]) < 1e-12
        assert abs(y[c["i"] + 64] - c["y_i64"]) < 1e-12
        rest = np.delete(y, [c["i"], c["i"] + 64])
        assert np.all(rest == 0)


def test_rope_relative_position_identity():
    rng = np.random.default_rng(7)
    for _ in range(20):
        q, k = rng.standard_normal(128), rng.standard_normal(128)
        m, n, c = (int(x) for x in rng.integers(0, 1 << 20, 3))
        lhs = oracle.rope(q, m + c) @ oracle.rope(k, n + c)
        rhs = oracle.rope(q, m) @ oracle.rope(k, n)
        assert abs(lhs - rhs) < 1e-9 * (np.abs(q).sum() * np.abs(k).sum() / 10)


def test_rope_complex_form_and_norm():
    rng = np.random.default_rng(8)
    x = rng.standard_normal(128)
    pos = 12345
    theta = 1e6 ** (-np.arange(64) * 2 / 128)
    zc = (x[:64] + 1j * x[64:]) * np.exp(1j * pos * theta)
    y = oracle.rope(x, pos)
    assert np.allclose(y[:64], zc.real, atol=1e-12) and np.allclose(y[64:], zc.imag, atol=1e-12)
    assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-12
    assert np.array_equal(oracle.rope(x, 0), x)


def test_generator_rope_matches_oracle_rope():
    """The workloads' RoPE'd keys and queries are bf16(RoPE(pre-RoPE vector))."""
    c = synth.workload(1)
    seed = c.seed
    pos = np.array([0, 1, 77, 4095])
    _, _, kpre = synth.keys_for(seed, synth.stream_id("k", 0, 0), pos, None, False, want_kpre=True)
    for i, n in enumerate(pos):
        if n in c.needles.get((0, 0), []):
            continue
        want = synth.to_bf16(oracle.rope(synth.from_bf16(kpre[i]), int(n)))
        assert np.array_equal(c.k_cache[0, 0, n], want)
    for h in range(c.Hq):
        want = synth.to_bf16(oracle.rope(synth.from_bf16(c.q_pre[0, h]), int(c.seq_lens[0])))
        assert np.array_equal(c.q_rope[0, h], want)


# ----------------------------------------------------------------------------
# index scores
# ----------------------------------------------------------------------------
def test_index_scores_hand():
    """W^Q picks the odd dims of q^pre (W[r, 2r+1] = 1), q^pre[d] = d, and
    k_idx row n is the unit vector e_(n mod 16): s_n = 2 (n mod 16) + 1.
    A transposed W or a swapped q/k index gives different numbers."""
    L = 40
    W = np.zeros((1, 16, 128))
    for r in range(16):
        W[0, r, 2 * r + 1] = 1.0
    q = np.arange(128, dtype=np.float64)[None, None, :]
    ki = np.zeros((1, 1, L, 16))
    ki[0, 0, np.arange(L), np.arange(L) % 16] = 1.0
    c = hand_case(L, Wq=W, q_pre=q, k_idx=ki)
    s = oracle.index_scores(c, 0, 0)
    assert s.tolist() == [2.0 * (n % 16) + 1.0 for n in range(L)]


def test_index_scores_linear_in_query():
    c = hand_case(300, seed=4)
    s1 = oracle.index_scores(c, 0, 0)
    c.q_pre = synth.to_bf16(2.0 * synth.from_bf16(c.q_pre))    # exact doubling in bf16
    s2 = oracle.index_scores(c, 0, 0)
    assert np.array_equal(s2, 2.0 * s1)


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------
def test_attention_uniform_when_keys_equal():
    L = 100
    rng = np.random.default_rng(9)
    kc = np.repeat(rng.standard_normal((1, 1, 1, 128)), L, axis=2)
    c = hand_case(L, k_cache=kc, seed=9)
    pos = np.array([3, 10, 50, 99])
    out = oracle.attend(c, 0, 0, pos)
    v = synth.from_bf16(c.v_cache[0, 0, pos])
    assert np.allclose(out, v.mean(0), atol=1e-12)


def test_attention_one_dominant_key():
    L = 64
    q = np.zeros((1, 1, 128))
    q[0, 0, 5] = 8.0
    kc = np.zeros((1, 1, L, 128))
    kc[0, 0, 17, 5] = 64.0          # logit 8*64/sqrt(128) = 45.25 vs 0 elsewhere
    c = hand_case(L, q_rope=q, k_cache=kc, seed=10)
    out = oracle.attend(c, 0, 0, np.arange(L))
    v = synth.from_bf16(c.v_cache[0, 0])
    w17 = 1.0 / (1.0 + (L - 1) * math.exp(-8 * 64 / math.sqrt(128)))
    want = w17 * v[17] + (1 - w17) / (L - 1) * (v.sum(0) - v[17])
    assert np.allclose(out, want, atol=1e-12)


def test_attention_permutation_invariant_and_weights_sum_to_one():
    c = hand_case(200, seed=11)
    pos = np.random.default_rng(11).choice(200, 50, replace=False)
    a = oracle.attend(c, 0, 0, pos)
    b = oracle.attend(c, 0, 0, pos[::-1])
    assert np.allclose(a, b, atol=1e-13)
    c.v_cache[:] = synth.to_bf16(np.ones(1))                     # every value vector = 1
    assert np.allclose(oracle.attend(c, 0, 0, pos), 1.0, atol=1e-13)


# ----------------------------------------------------------------------------
# the whole step
# ----------------------------------------------------------------------------
def test_local_positions_golden():
    for cs in load("local_positions_hand.json")["cases"]:
        L = cs["L"]
        c = hand_case(L, head_kind=[0], window=cs["window"], sink=cs["sink"], seed=L)
        r = oracle.decode_step(c)
        want = oracle.attend(c, 0, 0, np.array(cs["positions"]))
        assert np.array_equal(r["out"][0, 0], want), cs
        assert r["kstar"][0, 0] == len(cs["positions"])
        assert synth.local_positions(L, cs["window"], cs["sink"]).tolist() == cs["positions"]


def test_local_head_special_cases():
    L = 300
    c = hand_case(L, head_kind=[0], window=1, sink=0, seed=12)
    r = oracle.decode_step(c)
    assert np.array_equal(r["out"][0, 0], synth.from_bf16(c.v_cache[0, 0, L - 1]))
    c = hand_case(L, head_kind=[0], window=L + 5, sink=4, seed=13)
    r = oracle.decode_step(c)
    assert np.array_equal(r["out"][0, 0], oracle.attend(c, 0, 0, np.arange(L)))


def test_widening_golden():
    """Hand fixture: kept tokens -> whole blocks.  Realised with integer scores
    so that exactly the listed tokens are kept (their score 80, all others 0,
    p chosen below their joint mass)."""
    for cs in load("widening_hand.json")["cases"]:
        L = cs["L"]
        W = np.zeros((1, 16, 128))
        W[0, 0, 0] = 1.0
        q = np.zeros((1, 1, 128))
        q[0, 0, 0] = 8.0
        ki = np.zeros((1, 1, L, 16))
        ki[0, 0, cs["kept_tokens"], 0] = 10.0                  # s = 80 vs 0
        c = hand_case(L, Wq=W, q_pre=q, k_idx=ki, p=0.99, seed=L)
        r = oracle.decode_step(c)
        assert r["kstar"][0, 0] == len(cs["kept_tokens"])
        kept = np.nonzero(r["kept_blocks"][0, 0])[0].tolist()
        assert kept == cs["blocks"]
        pos = np.concatenate([np.arange(64 * j, min(64 * j + 64, L)) for j in kept])
        assert pos.size == cs["positions_count"]
        assert np.array_equal(r["out"][0, 0], oracle.attend(c, 0, 0, pos))


def test_p_one_equals_dense():
    c = synth.workload(2, scale=16)
    c.p[:] = 1.0
    r = oracle.decode_step(c)
    for h in np.nonzero(c.head_kind)[0]:
        L = int(c.seq_lens[0])
        assert r["kstar"][0, h] == L
        assert np.array_equal(r["out"][0, h], oracle.attend(c, 0, h, np.arange(L)))


def test_kept_blocks_are_topp_widened():
    c = synth.workload(3, scale=32)
    r = oracle.decode_step(c)
    for b in range(c.B):
        for h in np.nonzero(c.head_kind)[0][:3]:
            t = oracle.topp(oracle.index_scores(c, b, h), float(c.p[b]))
            blocks = np.unique(t["kept"] // 64)
            assert np.nonzero(r["kept_blocks"][b, h])[0].tolist() == blocks.tolist()
            assert r["kstar"][b, h] == t["kstar"]


@pytest.mark.parametrize("w", [1, 2])
def test_needles_always_selected(w):
    c = synth.workload(w, scale=1 if w == 1 else 4)
    for (b, h), plist in c.needles.items():
        t = oracle.topp(oracle.index_scores(c, b, h), float(c.p[b]))
        assert set(plist) <= set(t["kept"].tolist())


def test_needle_regime_keeps_one_token():
    c = synth.workload(4, scale=64)
    r = oracle.decode_step(c)
    for h in np.nonzero(c.head_kind)[0]:
        assert r["kstar"][0, h] == 1
        assert r["cum_at"][0, h] >= 0.99


def test_paged_layout_equals_contiguous():
    base = synth.make_case("pg", B=3, Hkv=2, G=2, seq_lens=[700, 64, 1000], ret_groups=[1], p=[0.9, 0.5, 0.95],
                           window=100, sink=4, seed=21, regimes=["gaussian", "needle", "diffuse"], paged=False)
    paged = synth.make_case("pg", B=3, Hkv=2, G=2, seq_lens=[700, 64, 1000], ret_groups=[1], p=[0.9, 0.5, 0.95],
                            window=100, sink=4, seed=21, regimes=["gaussian", "needle", "diffuse"], paged=True)
    ra, rb = oracle.decode_step(base), oracle.decode_step(paged)
    assert np.array_equal(ra["out"], rb["out"])
    assert np.array_equal(ra["kstar"], rb["kstar"])


def test_gqa_head_to_group_mapping():
    """Heads 2..3 read KV head 1: giving KV head 1 the contents of KV head 0
    makes them equal to heads 0..1 run on the same queries."""
    c = synth.make_case("gqa", B=1, Hkv=2, G=2, seq_lens=[500], ret_groups=[0, 1], p=[0.9], window=64, sink=4,
                        seed=22, regimes=["gaussian"])
    for arr in (c.k_cache, c.v_cache, c.k_idx):
        arr[:, 1] = arr[:, 0]
    c.q_pre[:, 2:4] = c.q_pre[:, 0:2]
    c.q_rope[:, 2:4] = c.q_rope[:, 0:2]
    c.Wq_idx[2:4] = c.Wq_idx[0:2]
    r = oracle.decode_step(c)
    assert np.array_equal(r["out"][0, 2:4], r["out"][0, 0:2])
    c.v_cache[:, 1] = synth.to_bf16(synth.from_bf16(c.v_cache[:, 1]) + 1.0)
    r2 = oracle.decode_step(c)
    assert np.array_equal(r2["out"][0, 0:2], r["out"][0, 0:2])
    assert not np.allclose(r2["out"][0, 2:4], r["out"][0, 2:4])


def test_invalid_p_is_an_error():
    c = synth.workload(1, scale=4)
    c.p[:] = 0.0
    assert oracle.decode_step(c)["rc"] == 6


# ---------------------------------------------------------------------------
# index-cache append: k_idx_n = bf16(W^K_g k^pre_n)
# ---------------------------------------------------------------------------
def _bf16_exact_rne(v):
    """Nearest bf16 bits of the exact rational v, ties to even: written from
    the format (sign, 8-bit exponent, 7 stored fraction bits), independent of
    the oracle's C rounding."""
    from fractions import Fraction

    v = Fraction(v)
    if v == 0:
        return 0
    sign = 0x8000 if v < 0 else 0
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1                                   # 2^e <= a < 2^(e+1)
    if e < -126:                                 # subnormal: multiples of 2^-133
        q, rem = divmod(a * 2 ** 133, 1)
        q = int(q) + (1 if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and int(q) % 2) else 0)
        return sign | q
    q, rem = divmod(a / Fraction(2) ** e * 128, 1)  # 128 <= q < 256
    q = int(q) + (1 if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and int(q) % 2) else 0)
    if q == 256:
        q, e = 128, e + 1
    if e + 127 >= 255:
        return sign | 0x7F80
    return sign | ((e + 127) << 7) | (q - 128)


def _bf16_value(b):
    from fractions import Fraction

    s = -1 if b & 0x8000 else 1
    ex, fr = (b >> 7) & 0xFF, b & 0x7F
    if ex == 0:
        return s * Fraction(fr) * Fraction(2) ** -133
    return s * (128 + fr) * Fraction(2) ** (ex - 127 - 7)


def test_bf16_rounding_ties_to_even_and_edges():
    assert oracle.bf16_rne(1.0) == 0x3F80
    assert oracle.bf16_rne(1 + 2 ** -8) == 0x3F80          # halfway 1 | 1+2^-7: the even one
    assert oracle.bf16_rne(1 + 3 * 2 ** -8) == 0x3F82      # halfway 1+2^-7 | 1+2^-6: the even one
    assert oracle.bf16_rne(1 + 2 ** -8 + 2 ** -30) == 0x3F81
    assert oracle.bf16_rne(-2.5) == 0xC020
    assert oracle.bf16_rne(2.0 ** -133) == 0x0001          # smallest subnormal
    assert oracle.bf16_rne(2.0 ** -126) == 0x0080          # smallest normal
    assert oracle.bf16_rne(3.5e38) == 0x7F80               # beyond the largest finite: infinity
    rng = np.random.default_rng(7)
    xs = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-40, 38, 2000),
                         rng.standard_normal(500)])
    for x in xs:
        assert oracle.bf16_rne(float(x)) == _bf16_exact_rne(float(x)), x


def _append_case(seed, B=2, Hkv=3, T=5, ncap=64, paged=False):
    rng = np.random.default_rng(seed)
    k_pre = synth.to_bf16(rng.standard_normal((B, Hkv, T, 128)))
    Wk = synth.to_bf16(rng.standard_normal((Hkv, 16, 128)) / np.sqrt(128))
    pos = rng.integers(0, ncap - T + 1, B).astype(np.int32)
    if paged:
        mbps = ncap // 64
        pages = rng.permutation(B * mbps).astype(np.int32)
        bt = pages.reshape(B, mbps)
        cache = rng.integers(0, 2 ** 16, (B * mbps, Hkv, 64, 16)).astype(np.uint16)
    else:
        bt = None
        cache = rng.integers(0, 2 ** 16, (B, Hkv, ncap, 16)).astype(np.uint16)
    return k_pre, Wk, pos, cache, bt


def _row(cache, bt, b, g, n):
    if bt is None:
        return cache[b, g, n]
    return cache[bt[b, n // 64], g, n % 64]


@pytest.mark.parametrize("paged", [False, True])
def test_index_append_exact_dot_and_untouched_rows(paged):
    """Brute force in exact rationals: every written row is the nearest bf16
    of the exact dot product; every other row keeps its old bits."""
    from fractions import Fraction

    k_pre, Wk, pos, cache, bt = _append_case(3, paged=paged, ncap=128)
    out = oracle.index_append(k_pre, Wk, pos, cache, block_table=bt)
    B, Hkv, T = k_pre.shape[:3]
    written = set()
    for b in range(B):
        for g in range(Hkv):
            for t in range(T):
                n = int(pos[b]) + t
                written.add((b, g, n))
                got = _row(out, bt, b, g, n)
                for r in range(16):
                    exact = sum(_bf16_value(int(Wk[g, r, i])) * _bf16_value(int(k_pre[b, g, t, i]))
                                for i in range(128))
                    assert int(got[r]) == _bf16_exact_rne(exact), (b, g, t, r)
    ncap = 128
    for b in range(B):
        for g in range(Hkv):
            for n in range(ncap):
                if (b, g, n) not in written:
                    assert np.array_equal(_row(out, bt, b, g, n), _row(cache, bt, b, g, n))


def test_index_append_identity_projection_copies_inputs():
    """W^K = [I_16 | 0]: the cache row is the first 16 entries of k^pre, bit
    for bit (bf16 values are exact in fp64 and round to themselves)."""
    k_pre, Wk, pos, cache, bt = _append_case(5)
    Wk = np.zeros_like(Wk)
    one = synth.to_bf16(np.ones(1))[0]
    for r in range(16):
        Wk[:, r, r] = one
    out = oracle.index_append(k_pre, Wk, pos, cache)
    for b in range(k_pre.shape[0]):
        for g in range(k_pre.shape[1]):
            for t in range(k_pre.shape[2]):
                assert np.array_equal(out[b, g, pos[b] + t], k_pre[b, g, t, :16])


# ---------------------------------------------------------------------------
# KV-cache write with the index-cache append: k_cache = bf16(RoPE_n(k^pre)),
# v_cache = v, k_idx = bf16(W^K k^pre), rows n = pos_b + t
# ---------------------------------------------------------------------------
def _kv_case(seed, B=2, Hkv=2, T=3, ncap=128, paged=False):
    k_pre, Wk, pos, kidx, bt = _append_case(seed, B=B, Hkv=Hkv, T=T, ncap=ncap, paged=paged)
    rng = np.random.default_rng(1000 + seed)
    v_new = synth.to_bf16(rng.standard_normal(k_pre.shape))
    ang = rng.uniform(-np.pi, np.pi, (ncap, 64))
    cos, sin = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
    shape = kidx.shape[:3] + (128,)
    kc = rng.integers(0, 2 ** 16, shape).astype(np.uint16)
    vc = rng.integers(0, 2 ** 16, shape).astype(np.uint16)
    return k_pre, v_new, Wk, cos, sin, pos, kidx, kc, vc, bt


@pytest.mark.parametrize("paged", [False, True])
def test_kv_append_exact_rationals_and_untouched_rows(paged):
    """Brute force in exact rationals: every written key element is the
    nearest bf16 of k_i cos - k_(i+64) sin (resp. k_(i+64) cos + k_i sin)
    with the table's fp32 values; value rows are the new values bit for bit;
    index rows are the nearest bf16 of the exact projection; every other row
    of the three caches keeps its old bits."""
    from fractions import Fraction

    k_pre, v_new, Wk, cos, sin, pos, kidx, kc, vc, bt = _kv_case(11, paged=paged)
    o_idx, o_k, o_v = oracle.kv_append(k_pre, v_new, Wk, cos, sin, pos, kidx, kc, vc, block_table=bt)
    B, Hkv, T = k_pre.shape[:3]
    written = set()
    for b in range(B):
        for g in range(Hkv):
            for t in range(T):
                n = int(pos[b]) + t
                written.add((b, g, n))
                kv = [_bf16_value(int(x)) for x in k_pre[b, g, t]]
                got = _row(o_k, bt, b, g, n)
                for i in range(64):
                    c, sn = Fraction(float(cos[n, i])), Fraction(float(sin[n, i]))
                    assert int(got[i]) == _bf16_exact_rne(kv[i] * c - kv[i + 64] * sn), (b, g, t, i)
                    assert int(got[i + 64]) == _bf16_exact_rne(kv[i + 64] * c + kv[i] * sn), (b, g, t, i + 64)
                assert np.array_equal(_row(o_v, bt, b, g, n), v_new[b, g, t])
                gi = _row(o_idx, bt, b, g, n)
                for r in (0, 7, 15):
                    exact = sum(_bf16_value(int(Wk[g, r, i])) * kv[i] for i in range(128))
                    assert int(gi[r]) == _bf16_exact_rne(exact), (b, g, t, r)
    for b in range(B):
        for g in range(Hkv):
            for n in range(128):
                if (b, g, n) not in written:
                    for new, old in ((o_idx, kidx), (o_k, kc), (o_v, vc)):
                        assert np.array_equal(_row(new, bt, b, g, n), _row(old, bt, b, g, n))


def test_kv_append_quarter_turns_permute_and_negate():
    """Angles 0, 90, 180 and 270 degrees (cos, sin in {0, 1, -1}): the key
    row is k, (-k_hi, k_lo), -k and (k_hi, -k_lo), exactly (up to the sign of
    zero), which fixes the pairing (i, i + 64) and the direction of rotation."""
    k_pre, v_new, Wk, cos, sin, pos, kidx, kc, vc, bt = _kv_case(12, B=1, Hkv=1, T=4, ncap=64)
    pos[:] = 10
    turns = [(1.0, 0.0), (0.0, 1.0), (-1.0, 0.0), (0.0, -1.0)]
    for t, (c, sn) in enumerate(turns):
        cos[10 + t, :], sin[10 + t, :] = c, sn
    _, o_k, _ = oracle.kv_append(k_pre, v_new, Wk, cos, sin, pos, kidx, kc, vc)
    for t in range(4):
        k = synth.from_bf16(k_pre[0, 0, t])
        lo, hi = k[:64], k[64:]
        want = [np.concatenate([lo, hi]), np.concatenate([-hi, lo]), np.concatenate([-lo, -hi]),
                np.concatenate([hi, -lo])][t]
        assert np.array_equal(synth.from_bf16(o_k[0, 0, 10 + t]), want), t


def test_kv_append_one_hot_keys_give_the_table():
    """k = e_i gives y_i = cos, y_(i+64) = sin; k = e_(i+64) gives
    y_i = -sin, y_(i+64) = cos; every other element is zero."""
    k_pre, v_new, Wk, cos, sin, pos, kidx, kc, vc, bt = _kv_case(13, B=1, Hkv=1, T=2, ncap=64)
    one = synth.to_bf16(np.ones(1))[0]
    for i in (0, 5, 63):
        k_pre[:] = 0
        k_pre[0, 0, 0, i] = one
        k_pre[0, 0, 1, i + 64] = one
        pos[:] = 20
        _, o_k, _ = oracle.kv_append(k_pre, v_new, Wk, cos, sin, pos, kidx, kc, vc)
        a = synth.from_bf16(o_k[0, 0, 20])
        b = synth.from_bf16(o_k[0, 0, 21])
        c, sn = float(cos[20, i]), float(sin[21, i])
        assert a[i] == synth.from_bf16(synth.to_bf16(np.array([c])))[0]
        assert a[i + 64] == synth.from_bf16(synth.to_bf16(np.array([float(sin[20, i])])))[0]
        assert b[i] == synth.from_bf16(synth.to_bf16(np.array([-sn])))[0]
        assert b[i + 64] == synth.from_bf16(synth.to_bf16(np.array([float(cos[21, i])])))[0]
        mask = np.ones(128, bool)
        mask[[i, i + 64]] = False
        assert np.all(a[mask] == 0) and np.all(b[mask] == 0)


def test_kv_append_with_position_angles_matches_the_generator():
    """With the angle table n theta_i (theta_i = 1e6^(-2i/128), rounded to
    fp32), the written keys are the generator's RoPE'd keys (exact angles,
    computed by its own code) to within one bf16 step, nearly all bit for
    bit: the table row of token t is its cache position pos_b + t."""
    k_pre, v_new, Wk, cos, sin, pos, kidx, kc, vc, bt = _kv_case(14, B=2, Hkv=2, T=6, ncap=4096)
    n = np.arange(4096, dtype=np.float64)[:, None]
    ang = n * synth.THETA ** (-2.0 * np.arange(64) / 128.0)[None, :]
    cos, sin = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
    _, o_k, _ = oracle.kv_append(k_pre, v_new, Wk, cos, sin, pos, kidx, kc, vc)
    same = total = 0
    for b in range(2):
        p = pos[b] + np.arange(6)
        for g in range(2):
            want = synth.rope_rows(k_pre[b, g], p)
            got = o_k[b, g, p]
            d = np.abs(got.astype(np.int32) - want.astype(np.int32))
            d = np.where((got ^ want) & 0x8000, 0, d)         # (compare magnitudes only when signs agree)
            assert np.all(np.abs(synth.from_bf16(got) - synth.from_bf16(want)) <=
                          2.0 ** -7 * np.maximum(np.abs(synth.from_bf16(want)), 2.0 ** -126))
            same += int(np.count_nonzero(got == want))
            total += got.size
            assert d.max() <= 1
    assert same >= 0.99 * total, (same, total)


def test_kv_append_refuses_positions_beyond_the_cache():
    k_pre, v_new, Wk, cos, sin, pos, kidx, kc, vc, bt = _kv_case(15, ncap=64)
    pos[0] = 62                                            # 62 + 3 > 64
    with pytest.raises(ValueError):
        oracle.kv_append(k_pre, v_new, Wk, cos, sin, pos, kidx, kc, vc)


# ---------------------------------------------------------------------------
# local heads' ring cache: sink + W rows per (sequence, KV head)
# ---------------------------------------------------------------------------
def _marker_rows(positions):
    """bf16 rows whose first four entries spell the position in base 16
    (small integers are exact in bf16); the rest zero."""
    rows = np.zeros((len(positions), 128))
    for i, n in enumerate(positions):
        for d in range(4):
            rows[i, d] = (n >> (4 * d)) & 15
        rows[i, 4] = 1.0                        # a written row is never all-zero
    return synth.to_bf16(rows)


def _marker_of(row_bits):
    v = synth.from_bf16(row_bits)
    if v[4] != 1.0:
        return None
    return int(sum(int(v[d]) << (4 * d) for d in range(4)))


@pytest.mark.parametrize("S0,W,L,chunk", [(4, 16, 3, 1), (4, 16, 20, 1), (4, 16, 21, 7), (4, 16, 100, 1),
                                           (4, 16, 100, 40), (0, 8, 50, 3), (3, 1, 9, 2), (64, 64, 1000, 64),
                                           (64, 128, 1000, 100), (2, 7, 300, 300)])
def test_ring_keeps_the_head_rows_and_the_last_W_positions(S0, W, L, chunk):
    """Positions 0 .. L-1 written in order (chunks of `chunk`): the ring then
    holds exactly [0, min(S0, L)) and the last W positions past S0, each in
    the row the layout gives it; unwritten rows stay unwritten."""
    B, Hkv = 1, 1
    kr = np.zeros((B, Hkv, S0 + W, 128), np.uint16)
    vr = np.zeros_like(kr)
    start = 0
    while start < L:
        T = min(chunk, L - start)
        rows = _marker_rows(range(start, start + T)).reshape(B, Hkv, T, 128)
        kr, vr = oracle.ring_write(rows, rows, np.array([start], np.int32), kr, vr, S0, W)
        start += T
    held = {}
    for r in range(S0 + W):
        m = _marker_of(kr[0, 0, r])
        assert m == _marker_of(vr[0, 0, r])
        if m is not None:
            held[m] = r
    want = set(range(min(S0, L))) | set(range(max(S0, L - W), L))
    assert set(held) == want
    for n, r in held.items():
        assert r == oracle.ring_row(n, S0, W)
        assert (r < S0) == (n < S0)


def test_ring_blocks_occupy_aligned_slots():
    """With S0 = 64 and W a multiple of 64, the 64 positions of any block
    j >= 1 lie in 64 consecutive rows starting at a multiple of 64."""
    for W in (64, 256, 4096):
        for j in (1, 2, 63, 64, 65, 1000):
            rows = [oracle.ring_row(64 * j + o, 64, W) for o in range(64)]
            assert rows[0] % 64 == 0 and rows == list(range(rows[0], rows[0] + 64))
            assert 64 <= rows[0] < 64 + W


@pytest.mark.parametrize("L,window,sink,S0,W", [(3000, 256, 4, 64, 256), (3000, 100, 4, 64, 256),
                                                (200, 256, 4, 64, 256), (3, 256, 4, 64, 256),
                                                (700, 64, 0, 0, 64), (700, 0, 4, 4, 64), (5000, 1, 0, 0, 1),
                                                (3001, 200, 4, 4, 200)])
def test_ring_attention_equals_the_local_head_output(L, window, sink, S0, W):
    """A local head that reads its keys and values from the ring gives the
    decode step's local-head output on the full cache, bit for bit (same
    positions, same order of summation)."""
    case = synth.make_case("ring", B=2, Hkv=2, G=2, seq_lens=[L, max(1, L // 3)], ret_groups=[], p=[0.9, 0.9],
                           window=window, sink=sink, seed=L + window, regimes=["gaussian", "gaussian"])
    ref = oracle.decode_step(case)
    for b in range(case.B):
        Lb = int(case.seq_lens[b])
        kr = np.zeros((case.B, case.Hkv, S0 + W, 128), np.uint16)
        vr = np.zeros_like(kr)
        for start in range(0, Lb, 512):
            T = min(512, Lb - start)
            pos = np.full(case.B, start, np.int32)
            kr, vr = oracle.ring_write(case.k_cache[:, :, start:start + T], case.v_cache[:, :, start:start + T],
                                       pos, kr, vr, S0, W)
        for h in range(case.Hq):
            got = oracle.attend_ring(case.q_rope, kr, vr, b, h, Lb, window, sink, S0, W)
            assert np.array_equal(got, ref["out"][b, h]), (b, h)


def test_ring_refuses_a_window_or_sink_it_cannot_hold():
    case = synth.make_case("ring-w", B=1, Hkv=1, G=1, seq_lens=[100], ret_groups=[], p=[0.9], window=32, sink=4,
                           seed=3, regimes=["gaussian"])
    kr = np.zeros((1, 1, 64 + 16, 128), np.uint16)
    with pytest.raises(ValueError):
        oracle.attend_ring(case.q_rope, kr, kr, 0, 0, 100, 32, 4, 64, 16)     # window 32 > W 16
    kr = np.zeros((1, 1, 2 + 64, 128), np.uint16)
    with pytest.raises(ValueError):
        oracle.attend_ring(case.q_rope, kr, kr, 0, 0, 100, 32, 4, 2, 64)      # sink 4 > S0 2


# ---------------------------------------------------------------------------
# prefill: causal attention of a chunk of queries, dense for retrieval heads,
# sink + window for local heads
# ---------------------------------------------------------------------------
def _prefill_case(L, window, sink, paged=False, seed=5):
    # mixed KV groups (retrieval and local heads in each): every cache row valid
    hk = np.array([1, 0, 0, 1, 1, 0, 0, 1], np.uint8)
    return synth.make_case("prefill", B=2, Hkv=2, G=4, seq_lens=[L, L - 7], ret_groups=[], head_kind=hk,
                           p=[1.0, 1.0], window=window, sink=sink, seed=seed, regimes=["gaussian", "gaussian"],
                           paged=paged)


@pytest.mark.parametrize("paged", [False, True])
def test_prefill_uniform_keys_give_the_mean_of_the_attended_values(paged):
    """All keys equal: every query weighs its attended positions equally, so
    its output is the mean of their values.  Values spell the position in
    base 8, so the mean fixes the position set: [0, m] for retrieval heads,
    the sink and the last `window` positions up to m for local heads."""
    L, window, sink, T = 300, 40, 3, 50
    case = _prefill_case(L, window, sink, paged=paged)
    ones = synth.to_bf16(np.full(128, 0.25))
    vals = np.zeros((case.Ncap, 128))
    n = np.arange(case.Ncap)
    vals[:, 0], vals[:, 1], vals[:, 2], vals[:, 3] = n % 8, (n // 8) % 8, (n // 64) % 8, 1.0
    vrows = synth.to_bf16(vals)
    for b in range(case.B):
        for g in range(case.Hkv):
            for m in range(int(case.seq_lens[b])):
                if case.block_table is None:
                    case.k_cache[b, g, m], case.v_cache[b, g, m] = ones, vrows[m]
                else:
                    pg = case.block_table[b, m // 64]
                    case.k_cache[pg, g, m % 64], case.v_cache[pg, g, m % 64] = ones, vrows[m]
    pos = np.array([L - T, L - 7 - T], np.int32)
    rng = np.random.default_rng(1)
    q = synth.to_bf16(rng.standard_normal((case.B, case.Hq, T, 128)))
    out = oracle.prefill(case, q, pos)
    for b in range(case.B):
        for h in range(case.Hq):
            for t in range(T):
                m = int(pos[b]) + t
                if case.head_kind[h]:
                    S = np.arange(m + 1)
                else:
                    S = np.array(sorted(set(range(min(sink, m + 1))) | set(range(max(0, m + 1 - window), m + 1))))
                want = [np.mean(S % 8), np.mean((S // 8) % 8), np.mean((S // 64) % 8), 1.0]
                assert np.allclose(out[b, h, t, :4], want, rtol=0, atol=1e-12), (b, h, t)


def test_prefill_first_position_attends_only_itself():
    case = _prefill_case(200, 16, 4)
    rng = np.random.default_rng(2)
    q = synth.to_bf16(rng.standard_normal((case.B, case.Hq, 3, 128)))
    out = oracle.prefill(case, q, np.zeros(case.B, np.int32))
    for b in range(case.B):
        for h in range(case.Hq):
            assert np.array_equal(out[b, h, 0], synth.from_bf16(case.v_cache[b, h // 4, 0]))


@pytest.mark.parametrize("paged", [False, True])
def test_prefill_last_query_is_the_decode_step(paged):
    """The chunk's last query, at position L - 1 with the decode query's
    vector, attends exactly the decode step's positions at length L (p = 1 for
    the retrieval heads): the same output, bit for bit."""
    L, T = 900, 33
    case = _prefill_case(L, 100, 4, paged=paged, seed=9)
    ref = oracle.decode_step(case)
    rng = np.random.default_rng(3)
    q = synth.to_bf16(rng.standard_normal((case.B, case.Hq, T, 128)))
    q[:, :, T - 1] = case.q_rope
    pos = (case.seq_lens - T).astype(np.int32)
    out = oracle.prefill(case, q, pos)
    assert np.array_equal(out[:, :, T - 1], ref["out"])


# ---------------------------------------------------------------------------
# static top-k (the fixed-budget variant): the k highest scores, ties low index
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("seed", range(12))
def test_topk_brute_force_dominance(seed):
    """Brute force on tiny inputs: among all subsets of size min(k, L) exactly
    one has every member beat every non-member under (s desc, n asc), and it
    is the oracle's."""
    rng = np.random.default_rng(seed)
    L = int(rng.integers(1, 11))
    s = rng.integers(-3, 4, L).astype(np.float64)       # integer scores: many ties
    k = int(rng.integers(1, L + 3))
    beats = lambda a, b: s[a] > s[b] or (s[a] == s[b] and a < b)
    m = min(k, L)
    winners = [set(c) for c in itertools.combinations(range(L), m)
               if all(beats(a, b) for a in c for b in range(L) if b not in c)]
    assert len(winners) == 1
    r = oracle.topk(s, k)
    assert r["kstar"] == m
    assert set(r["kept"].tolist()) == winners[0]


def test_topk_closed_forms():
    # all scores equal: the first k indices
    r = oracle.topk(np.zeros(1000), 300)
    assert r["kept"].tolist() == list(range(300))
    # k = 1: the maximum, lowest index among equal maxima
    s = np.array([1.0, 5.0, 2.0, 5.0, -1.0])
    assert oracle.topk(s, 1)["kept"].tolist() == [1]
    # k >= L keeps everything
    assert oracle.topk(s, 99)["kstar"] == 5
    with pytest.raises(ValueError):
        oracle.topk(s, 0)


def test_topk_step_with_k_at_least_L_is_dense():
    """k >= L keeps every token: the step equals the top-p step with p = 1."""
    case = synth.workload(1)
    dense = case.__class__(**{**case.__dict__})
    dense.p = np.ones_like(case.p)
    a = oracle.decode_step_topk(case, 1 << 20)
    b = oracle.decode_step(dense)
    assert a["rc"] == 0 and b["rc"] == 0
    ret = np.nonzero(case.head_kind)[0]
    assert np.array_equal(a["kept_blocks"][:, ret], b["kept_blocks"][:, ret])
    assert np.max(np.abs(a["out"] - b["out"])) < 1e-12


def test_topk_step_keeps_the_blocks_of_its_k_best():
    """The step's kept blocks are the blocks of the k best tokens of each
    retrieval head (scores recomputed independently by index_scores)."""
    case = synth.workload(1)
    k = 200
    r = oracle.decode_step_topk(case, k)
    assert r["rc"] == 0
    for h in np.nonzero(case.head_kind)[0]:
        s = oracle.index_scores(case, 0, h)[: int(case.seq_lens[0])]
        best = sorted(range(s.size), key=lambda n: (-s[n], n))[:k]
        blocks = sorted({n // 64 for n in best})
        assert np.nonzero(r["kept_blocks"][0, h])[0].tolist() == blocks
        assert r["kstar"][0, h] == k


def test_oracle_results_do_not_depend_on_the_thread_count():
    """The oracle parallelises over (sequence, head) only: one thread and
    many give the same bits (the benchmark times both)."""
    case = synth.workload(5, scale=64)
    a = oracle.decode_step(case, nthreads=1)
    b = oracle.decode_step(case, nthreads=8)
    for k in ("out", "kstar", "tau", "kept_blocks"):
        assert np.array_equal(a[k], b[k], equal_nan=(k == "tau")), k
    c = oracle.decode_step_topk(case, 100, nthreads=1)
    d = oracle.decode_step_topk(case, 100, nthreads=8)
    assert np.array_equal(c["out"], d["out"]) and np.array_equal(c["kept_blocks"], d["kept_blocks"])
