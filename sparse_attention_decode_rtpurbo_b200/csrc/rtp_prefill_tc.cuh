// Prefill attention on the 5th-generation tensor cores (sm_100a): the same
// operation as prefill_kernel (rtp_prefill.cuh: retrieval heads dense and
// causal, local heads sink + window; review "RTPurbo" on
// dongryeollee1.github.io, Method: "Adaptive sparse attention", the prefill
// paragraph), with the two contractions on tcgen05 and their accumulators
// in tensor memory.
//
// A CTA takes eight (head, 16-position) units of one (KV group, head kind)
// set: M = 128 query rows that all read the same KV head.  Per 64-key tile:
//   S = Q K^T       tcgen05.mma M128 N64, K = 128 in eight K16 steps, S in
//                   tensor memory (64 columns)
//   softmax         four warps, thread i owns row i: tcgen05.ld of its 64
//                   scores, mask, max, exp2, row sum in registers; P (bf16)
//                   to shared memory as the A operand of the next MMA
//   O += P V        tcgen05.mma M128 N128, K = 64 in four K16 steps, O in
//                   tensor memory (128 columns)
// (Build option RTP_PT_P_TMEM: P goes back to tensor memory and the P V MMA
// reads its A operand from there; correct, and measured slower on the 32K
// prompt, 393 against 420 TFLOP/s.)
// K and V tiles arrive by TMA, each as two 64 x 64 boxes with the 128-byte
// swizzle, and are read in place: K as the K-major B operand of Q K^T, V as
// the MN-major B operand of P V (head dimension contiguous), so V needs no
// transpose.  Q (cp.async, once per CTA) and P are unswizzled K-major core
// matrices (8 rows x 16 bytes).  Pipeline per tile k: S_{k+1} is issued
// before the softmax of tile k, and the TMA loads of K_{k+2} and V_{k+1}
// (two buffers each) run meanwhile; one thread issues the loads and the
// MMAs, and two CTAs per SM overlap the rest.
// The online softmax keeps a reference maximum per row and rescales O in
// tensor memory only when a tile's maximum exceeds it by more than 2^8
// (P <= 256 then): the normalised result does not depend on the reference.
#pragma once
#include "rtp_prefill.cuh"
#include "rtp_tc.cuh"

namespace rtp {

constexpr int PT_UNITS = 8;                  // (head, 16 positions) units per CTA: M = 128 rows
constexpr int PT_THREADS = 128;              // warp w owns rows (tensor-memory lanes) 32w .. 32w+31
constexpr float PT_RESCALE = 8.f;            // log2 of the largest P before O is rescaled
// tensor-memory columns: S, P (bf16 pairs), O
constexpr uint32_t PT_TM_S = 0, PT_TM_P = 64, PT_TM_O = 128, PT_TM_COLS = 256;

struct PtSmem {
    alignas(1024) uint8_t q[128 * 128 * 2];      // Q: chunk (row r, dims 8c..) at c*2048 + r*16
    // K / V tiles: box b (dims 64b..64b+63) at b*8192, key r at r*128, 16-byte
    // chunk c of the row at ((c ^ r) % 8)*16 (the TMA's 128-byte swizzle)
    alignas(1024) uint8_t k[2][64 * 128 * 2];
    alignas(1024) uint8_t v[2][64 * 128 * 2];
#ifndef RTP_PT_P_TMEM
    alignas(1024) uint8_t p[128 * 64 * 2];      // P: chunk (row r, keys 8c..) at c*2048 + r*16
#endif
    alignas(8) uint64_t s_bar, o_bar;            // S = Q K^T / O += P V complete
    alignas(8) uint64_t kfull[2], vfull[2];      // a K / V buffer's TMA loads have landed
    uint32_t tmem_base;
};

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
// 3-input maximum (one instruction on sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
// packed fp32 pair arithmetic (one instruction for two lanes' worth of work)
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1,%2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0,%1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// (lo, hi) -> bf16x2, round to nearest even; lo in the low half
__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// Shared-memory matrix descriptor of a 128-byte-swizzled operand: rows of 128
// bytes in 8-row atoms of 1024 bytes (`sbo` between atoms along the rows);
// `lbo` between 64-element column groups for an MN-major operand (unused,
// 16, for K-major).  Bits 61-63 = 2: the 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return smem_desc(saddr, lbo, sbo) | ((uint64_t)2 << 61);
}

// 32 consecutive 32-bit columns into this thread's tensor-memory lane, the
// store waited for inside the same asm.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
        "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
        "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

// D[tmem] (=|+=) A[tmem] . B[smem]^T, issued by one thread (A: M lanes, K
// packed two 16-bit elements per column).
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The CTA's set, units and key tiles: as pf_cta, with PT_UNITS units.
__device__ __forceinline__ PfCta pt_cta(const PrefillParams& P) {
    PfCta c;
    const int x = (int)blockIdx.x;
    c.b = x / P.cta_per_b;
    const int lc = x - c.b * P.cta_per_b;
    int lo = 0, hi = P.n_sets - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.set_cta0[mid] <= lc) lo = mid;
        else hi = mid - 1;
    }
    c.set = lo;
    c.g = P.set_g[lo];
    c.kind = P.set_kind[lo];
    c.nh = P.set_nh[lo];
    c.units = c.nh * P.nt16;
    c.u0 = (lc - P.set_cta0[lo]) * PT_UNITS;
    c.pos_b = __ldg(P.pos + c.b);
    c.ok = c.pos_b >= 0 && (long long)c.pos_b + P.T <= (long long)P.Ncap;
    const int ulast = min(c.u0 + PT_UNITS, c.units) - 1;
    const int pt_hi = P.nt16 - 1 - c.u0 / c.nh, pt_lo = P.nt16 - 1 - ulast / c.nh;
    c.m_lo = c.pos_b + 16 * pt_lo;
    c.m_hi = c.pos_b + min(16 * pt_hi + 15, P.T - 1);
    c.s_end = min(P.sink, c.m_hi + 1);
    c.w_lo = max(0, c.m_lo + 1 - P.window);
    if (c.kind == 1) {
        c.j0a = 0;
        c.j1a = c.m_hi / BLK + 1;
        c.j0b = c.j1b = c.j1a;
    } else {
        c.j0a = 0;
        c.j1a = (c.s_end + BLK - 1) / BLK;
        if (P.window > 0) {
            c.j0b = max(c.j1a, c.w_lo / BLK);
            c.j1b = max(c.j0b, c.m_hi / BLK + 1);
        } else {
            c.j0b = c.j1b = c.j1a;
        }
    }
    return c;
}

// Global address of cache row `row` (from pf_row) of the K or V cache.
__device__ __forceinline__ const uint8_t* pt_cache_row(const uint16_t* cache, int row) {
    return reinterpret_cast<const uint8_t*>(cache) + (int64_t)row * (D * 2);
}

// bits [lo, hi) of a 64-bit word, the bounds clamped to [0, 64]
__device__ __forceinline__ uint64_t pt_bits(int lo, int hi) {
    lo = max(lo, 0);
    hi = min(hi, 64);
    if (hi <= lo) return 0ull;
    const uint64_t below_hi = hi >= 64 ? ~0ull : ((1ull << hi) - 1ull);
    return below_hi & ~((1ull << lo) - 1ull);
}

struct PrefillTcK {
    CUtensorMap tmk, tmv;   // K / V caches as [rows][128] bf16, 64 x 64 boxes, 128-byte swizzle
    PrefillParams P;
};

__global__ void __launch_bounds__(PT_THREADS, 2) prefill_tc_kernel(const __grid_constant__ PrefillTcK K) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    PtSmem& S = *reinterpret_cast<PtSmem*>(smem_raw);
    const PrefillParams& P = K.P;
    const int tid = threadIdx.x, warp = tid >> 5;
    if (smem_u32(smem_raw) & 1023u) {
        if (tid == 0) pf_status(P, 5u);
        return;
    }
    const PfCta c = pt_cta(P);
    if (!c.ok) {
        if (tid == 0) pf_status(P, ST_DEVICE_INPUT);   // this sequence's outputs are not written
        return;
    }
    const uint32_t qs = smem_u32(S.q);
    const uint32_t kbuf[2] = {smem_u32(S.k[0]), smem_u32(S.k[1])};
    const uint32_t vbuf[2] = {smem_u32(S.v[0]), smem_u32(S.v[1])};
    if (tid == 0) {
        mbar_init(&S.s_bar, 1);
        mbar_init(&S.o_bar, 1);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.kfull[i], 1);
            mbar_init(&S.vfull[i], 1);
        }
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(&S.tmem_base, PT_TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = S.tmem_base;
    const uint32_t t_lane = tbase + ((uint32_t)(32 * warp) << 16);   // this warp's lanes
    const int nt = c.ntiles();

    // ---- this thread's row: unit u0 + row / 16, position t
    const int row = tid;
    const int u = c.u0 + row / 16;
    const int t = u < c.units ? 16 * (P.nt16 - 1 - u / c.nh) + (row & 15) : P.T;
    const bool valid = u < c.units && t < P.T;
    const int h = c.g * P.G + P.set_heads[c.set][valid ? u % c.nh : 0];
    const int m = c.pos_b + t;
    const bool retr = c.kind == 1;
    const int window = P.window, sink = P.sink;
    // this thread's row of a V tile to zero on an edge tile: key zr, box zb
    const int zr = tid >> 1, zb = tid & 1;

    constexpr float SCALE = 0.08838834764831845f * 1.4426950408889634f;   // log2(e)/sqrt(128)
    constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64);
    constexpr uint32_t IDESC_O = idesc_bf16_f32(128, 128) | (1u << 16);   // B (V) MN-major
    // a tile with every key visible to every row of the CTA needs no mask; an
    // edge tile holds keys no row reads
    auto interior = [&](int n0) {
        return n0 + BLK - 1 <= c.m_lo && (retr || n0 + BLK - 1 < sink || n0 > c.m_hi - window);
    };
    auto edge = [&](int n0) { return n0 + BLK - 1 > c.m_hi || (!retr && n0 + BLK > c.s_end && n0 < c.w_lo); };
    // TMA load of tile kt's K or V (two boxes) into buffer `dst` (thread 0)
    auto load_tile = [&](const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int kt) {
        const int r0 = pf_row(P, c.b, c.g, c.tile(kt));
        mbar_expect_tx(bar, 64 * 128 * 2);
        tma_load_2d(dst, map, 0, r0, bar);
        tma_load_2d(dst + 8192, map, 64, r0, bar);
    };
    // a bounded wait that gave up marks this thread; the CTA leaves the tile
    // loop together at the next barrier that ORs the marks (__syncthreads_or)
    bool bad = false;
    auto wait_or_abort = [&](uint64_t* bar, uint32_t parity) {
        if (!mbar_wait_bounded(bar, parity)) {
            pf_status(P, ST_TIMEOUT);
            bad = true;
        }
    };
    auto issue_s = [&](uint32_t kb) {   // S = Q K^T
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            umma_bf16(tbase + PT_TM_S, smem_desc(qs + kk * 4096, 2048, 128),
                      smem_desc_sw128(kb + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), IDESC_S, kk > 0);
        umma_commit(&S.s_bar);
    };

    // ---- prologue: tiles 0 and 1 and Q in flight; S_0
    if (tid == 0)
        for (int i = 0; i < 2 && i < nt; ++i) {
            load_tile(&K.tmk, S.k[i], &S.kfull[i], i);
            load_tile(&K.tmv, S.v[i], &S.vfull[i], i);
        }
    {
        const uint8_t* qrow = reinterpret_cast<const uint8_t*>(P.q + (((int64_t)c.b * P.Hq + h) * P.T + t) * D);
#pragma unroll
        for (int ch = 0; ch < 16; ++ch) {
            const uint32_t dst = qs + (uint32_t)(ch * 2048 + row * 16);
            if (valid) cp_async16(dst, qrow + ch * 16);
            else sts128(dst, 0u, 0u, 0u, 0u);
        }
    }
    cp_async_wait_all();
    fence_proxy_async();
    tc_fence_before();
    bool aborted = __syncthreads_or(bad) != 0;
    if (nt > 0 && !aborted && tid == 0) {
        wait_or_abort(&S.kfull[0], 0u);
        if (!bad) issue_s(kbuf[0]);
    }

    float m_ref = -INFINITY, l = 0.f;
    for (int k = 0; k < nt && !aborted; ++k) {
        const int n0 = c.tile(k) * BLK;
        // (1) S_k; its K buffer is free again: K_{k+2} goes there
        wait_or_abort(&S.s_bar, (uint32_t)k & 1u);
        tc_fence_after();
        float s[64];
        tmem_ld64(t_lane + PT_TM_S, s);
        if (k + 2 < nt && tid == 0) load_tile(&K.tmk, S.k[k & 1], &S.kfull[k & 1], k + 2);
        // (2) S_{k+1} on the tensor cores while this tile's softmax runs
        if (k + 1 < nt) {
            tc_fence_before();
            if ((aborted = __syncthreads_or(bad) != 0)) break;   // every S_k is in registers
            if (tid == 0) {
                wait_or_abort(&S.kfull[(k + 1) & 1], (uint32_t)((k + 1) >> 1) & 1u);
                if (!bad) issue_s(kbuf[(k + 1) & 1]);
            }
        }
        // (3) mask, row maximum (of the unscaled scores); a reference that
        // moves only in steps above 2^8
        if (!(valid && interior(n0))) {
            uint64_t keep = 0ull;
            if (valid) {
                keep = pt_bits(0, m - n0 + 1);
                if (!retr) keep &= pt_bits(0, sink - n0) | pt_bits(m - window + 1 - n0, 64);
            }
#pragma unroll
            for (int i = 0; i < 64; ++i)
                if (!((keep >> i) & 1ull)) s[i] = -INFINITY;
        }
        float mx;
        {
            float a[22];
#pragma unroll
            for (int i = 0; i < 21; ++i) a[i] = fmax3(s[3 * i], s[3 * i + 1], s[3 * i + 2]);
            a[21] = s[63];
            float b[8];
#pragma unroll
            for (int i = 0; i < 7; ++i) b[i] = fmax3(a[3 * i], a[3 * i + 1], a[3 * i + 2]);
            b[7] = a[21];
            mx = fmax3(fmax3(b[0], b[1], b[2]), fmax3(b[3], b[4], b[5]), fmaxf(b[6], b[7])) * SCALE;
        }
        float alpha = 1.f;
        if (mx > m_ref + PT_RESCALE) {
            alpha = m_ref == -INFINITY ? 1.f : ex2_approx(m_ref - mx);
            m_ref = mx;
        }
        // (4) P V of the previous tile done: P's columns and V_{k-1}'s buffer
        // are free, O is rescaled if needed; V_{k+1} on its way
        if (k > 0) {
            wait_or_abort(&S.o_bar, (uint32_t)(k - 1) & 1u);
            tc_fence_after();
            if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float o[64];
                    tmem_ld64(t_lane + PT_TM_O + 64 * half, o);
#pragma unroll
                    for (int i = 0; i < 64; ++i) o[i] *= alpha;
                    tmem_st64(t_lane + PT_TM_O + 64 * half, o);
                }
            }
            if (k + 1 < nt && tid == 0) load_tile(&K.tmv, S.v[(k + 1) & 1], &S.vfull[(k + 1) & 1], k + 1);
        }
        // (5) P = 2^(s * SCALE - m_ref) as bf16 into tensor memory, row sum
        // in fp32 (a row with nothing visible yet has m_ref = -inf: P = 0)
        {
            const float nb = m_ref == -INFINITY ? 0.f : -m_ref;
            const uint64_t sc2 = f2pack(SCALE, SCALE), nb2 = f2pack(nb, nb);
            uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
            uint32_t w[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                float x0, x1;
                f2unpack(ffma2(f2pack(s[2 * i], s[2 * i + 1]), sc2, nb2), x0, x1);
                const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                acc[i & 3] = fadd2(acc[i & 3], f2pack(p0, p1));
                w[i] = bf16x2(p0, p1);
            }
            float a0, a1, a2, a3;
            f2unpack(fadd2(acc[0], acc[1]), a0, a1);
            f2unpack(fadd2(acc[2], acc[3]), a2, a3);
            l = l * alpha + ((a0 + a2) + (a1 + a3));
#ifndef RTP_PT_P_TMEM
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
                sts128(smem_u32(S.p) + (uint32_t)(ch * 2048 + row * 16), w[4 * ch], w[4 * ch + 1], w[4 * ch + 2], w[4 * ch + 3]);
#else
            tmem_st32(t_lane + PT_TM_P, w);
#endif
        }
        // (6) O += P V once V_k has landed; on an edge tile the value rows
        // no row of the CTA may read are zeroed first (a cache row may hold
        // anything, and 0 x NaN would reach O through P = 0)
        const bool zero_rows = edge(n0);
        if (zero_rows) {
            wait_or_abort(&S.vfull[k & 1], (uint32_t)(k >> 1) & 1u);
            if (!c.needed(n0 + zr, window)) {
                const uint32_t rowa = vbuf[k & 1] + (uint32_t)(zb * 8192 + zr * 128);
#pragma unroll
                for (int i = 0; i < 8; ++i) sts128(rowa + 16 * i, 0u, 0u, 0u, 0u);
            }
        }
        fence_proxy_async();
        tc_fence_before();
        if ((aborted = __syncthreads_or(bad) != 0)) break;
        if (tid == 0) {
            if (!zero_rows) wait_or_abort(&S.vfull[k & 1], (uint32_t)(k >> 1) & 1u);
            tc_fence_after();
            const uint32_t vb = vbuf[k & 1];
#pragma unroll
            for (int kk = 0; kk < 4 && !bad; ++kk)
#ifndef RTP_PT_P_TMEM
                umma_bf16(tbase + PT_TM_O, smem_desc(smem_u32(S.p) + kk * 4096, 2048, 128),
                          smem_desc_sw128(vb + kk * 2048, 8192, 1024), IDESC_O, (k > 0 || kk > 0) ? 1u : 0u);
#else
                umma_bf16_ts(tbase + PT_TM_O, tbase + PT_TM_P + 8 * kk, smem_desc_sw128(vb + kk * 2048, 8192, 1024),
                             IDESC_O, (k > 0 || kk > 0) ? 1u : 0u);
#endif
            umma_commit(&S.o_bar);
        }
    }
    cp_async_wait_all();
    // ---- the output of this thread's row, once the last P V is done
    if (!aborted && nt > 0) {
        wait_or_abort(&S.o_bar, (uint32_t)(nt - 1) & 1u);
        tc_fence_after();
    }
    const bool ok = !__syncthreads_or(bad) && !aborted && nt > 0;
    if (ok) {
        uint4* orow = reinterpret_cast<uint4*>(P.out + (((int64_t)c.b * P.Hq + h) * P.T + t) * D);
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float o[64];
            tmem_ld64(t_lane + PT_TM_O + 64 * half, o);
            if (valid && l > 0.f) {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    orow[8 * half + i] = make_uint4(
                        bf16x2(o[8 * i] * inv, o[8 * i + 1] * inv), bf16x2(o[8 * i + 2] * inv, o[8 * i + 3] * inv),
                        bf16x2(o[8 * i + 4] * inv, o[8 * i + 5] * inv), bf16x2(o[8 * i + 6] * inv, o[8 * i + 7] * inv));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_free(tbase, PT_TM_COLS);
    }
}

}  // namespace rtp
