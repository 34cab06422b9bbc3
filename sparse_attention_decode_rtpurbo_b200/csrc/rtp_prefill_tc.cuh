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
//                   to shared memory as the next MMA's A operand
//   O += P V        tcgen05.mma M128 N128, K = 64 in four K16 steps, O in
//                   tensor memory (128 columns)
// Operands sit in shared memory as K-major core matrices (8 rows x 16 bytes,
// no swizzle).  Q, K and V arrive by cp.async; V is transposed through
// ldmatrix.trans into V^T (the B operand of P V must be K-major in keys).
// The online softmax keeps a reference maximum per row and rescales O in
// tensor memory only when a tile's maximum exceeds it by more than 2^8
// (P <= 256 then): the normalised result does not depend on the reference.
// The next tile's K and V copies are issued while the current tile's
// softmax and P V run; two CTAs per SM overlap the rest.
#pragma once
#include "rtp_prefill.cuh"
#include "rtp_tc.cuh"

namespace rtp {

constexpr int PT_UNITS = 8;                  // (head, 16 positions) units per CTA: M = 128 rows
constexpr int PT_THREADS = 128;              // warp w owns rows (tensor-memory lanes) 32w .. 32w+31
constexpr int PT_VS_STRIDE = 272;            // bytes per staged V row (256 + 16: conflict-free ldmatrix)
constexpr float PT_RESCALE = 8.f;            // log2 of the largest P before O is rescaled

struct PtSmem {
    alignas(1024) uint8_t q[128 * 128 * 2];   // Q: chunk (row r, dims 8c..) at c*2048 + r*16
    alignas(1024) uint8_t k[64 * 128 * 2];    // K tile: chunk (key r, dims 8c..) at c*1024 + r*16
    alignas(1024) uint8_t vt[64 * 128 * 2];   // V^T: core (dims 8n.., keys 8k..) at k*2048 + n*128
    alignas(1024) uint8_t p[128 * 64 * 2];    // P: chunk (row r, keys 8c..) at c*2048 + r*16
    alignas(1024) uint8_t vs[64 * PT_VS_STRIDE];   // V tile as loaded: row-major, 272-byte rows
    alignas(8) uint64_t s_bar, o_bar;
    uint32_t tmem_base;
    uint32_t abort;   // a bounded wait gave up: every thread leaves the tile loop at the next barrier
};

__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
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

// Copies of key tile j: K into its core-matrix layout, V row-major into vs.
// Thread t takes chunks t, t + 128, ... (8 of each): K chunk x is (key x % 64,
// dims 8 (x / 64) ..), so a warp writes 32 consecutive 16-byte slots; V chunk
// x is (key x / 16, dims 8 (x % 16) ..), so a warp reads two whole rows.
__device__ __forceinline__ void pt_copy_k(const PrefillParams& P, const uint16_t* kc, const PfCta& c, int j,
                                          uint32_t ks, int tid) {
    const int row = pf_row(P, c.b, c.g, j);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int x = tid + 128 * i, r = x & 63, ch = x >> 6;
        cp_async16(ks + (uint32_t)(ch * 1024 + r * 16), pt_cache_row(kc, row + r) + ch * 16);
    }
}
__device__ __forceinline__ void pt_copy_v(const PrefillParams& P, const uint16_t* vc, const PfCta& c, int j,
                                          uint32_t vs, int tid) {
    const int row = pf_row(P, c.b, c.g, j);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int x = tid + 128 * i, r = x >> 4, ch = x & 15;
        cp_async16(vs + (uint32_t)(r * PT_VS_STRIDE + ch * 16), pt_cache_row(vc, row + r) + ch * 16);
    }
}

struct PrefillTcK {
    const uint16_t* k_cache;
    const uint16_t* v_cache;
    PrefillParams P;
};

__global__ void __launch_bounds__(PT_THREADS, 2) prefill_tc_kernel(const __grid_constant__ PrefillTcK K) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    PtSmem& S = *reinterpret_cast<PtSmem*>(smem_raw);
    const PrefillParams& P = K.P;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (smem_u32(smem_raw) & 1023u) {
        if (tid == 0) pf_status(P, 5u);
        return;
    }
    const PfCta c = pt_cta(P);
    if (!c.ok) {
        if (tid == 0) pf_status(P, ST_DEVICE_INPUT);   // this sequence's outputs are not written
        return;
    }
    const uint32_t qs = smem_u32(S.q), ks = smem_u32(S.k), vts = smem_u32(S.vt), ps = smem_u32(S.p),
                   vss = smem_u32(S.vs);
    if (tid == 0) {
        mbar_init(&S.s_bar, 1);
        mbar_init(&S.o_bar, 1);
        mbar_fence_init();
        S.abort = 0u;
    }
    if (warp == 0) tmem_alloc(&S.tmem_base, 256);   // S in columns 0..63, O in 128..255
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

    // ---- Q (once) and the first tile's K and V
    {
        const uint8_t* qrow = reinterpret_cast<const uint8_t*>(P.q + (((int64_t)c.b * P.Hq + h) * P.T + t) * D);
#pragma unroll
        for (int ch = 0; ch < 16; ++ch) {
            const uint32_t dst = qs + (uint32_t)(ch * 2048 + row * 16);
            if (valid) cp_async16(dst, qrow + ch * 16);
            else sts128(dst, 0u, 0u, 0u, 0u);
        }
    }
    if (nt > 0) {
        pt_copy_k(P, K.k_cache, c, c.tile(0), ks, tid);
        pt_copy_v(P, K.v_cache, c, c.tile(0), vss, tid);
    }
    cp_async_commit();

    constexpr float SCALE = 0.08838834764831845f * 1.4426950408889634f;   // log2(e)/sqrt(128)
    constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64), IDESC_O = idesc_bf16_f32(128, 128);
    float m_ref = -INFINITY, l = 0.f;
    uint32_t ph = 0;   // phase of both MMA barriers (one completion each per tile)
    for (int k = 0; k < nt; ++k) {
        const int n0 = c.tile(k) * BLK;
        // (a) this tile's K and V have landed
        cp_async_wait_all();
        __syncthreads();
        // (b) the previous P V is done (V^T, P and O are free); V -> V^T, with
        // the keys no row of this CTA may read zeroed
        if (k > 0) {
            if (!mbar_wait_bounded(&S.o_bar, ph ^ 1u)) {
                pf_status(P, ST_TIMEOUT);
                S.abort = 1u;
            }
            tc_fence_after();
        }
        {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                // matrices q*4 .. q*4+3 of this warp: keys 16w + 8 (mm / 16) .., dims 8 (mm % 16) ..
                const int mm = q * 4 + (lane >> 3);
                const int ki = 2 * warp + (mm >> 4), ni = mm & 15;
                uint32_t r[4];
                ldsm_x4_t(vss + (uint32_t)((8 * ki + (lane & 7)) * PT_VS_STRIDE + ni * 16), r[0], r[1], r[2], r[3]);
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int mj = q * 4 + jj;
                    const int kj = 2 * warp + (mj >> 4), nj = mj & 15;
                    // this lane's word: dim 8 nj + lane / 4, keys 8 kj + 2 (lane % 4) and + 1
                    const int key0 = n0 + 8 * kj + 2 * (lane & 3);
                    uint32_t w = r[jj];
                    if (!c.needed(key0, window)) w &= 0xFFFF0000u;
                    if (!c.needed(key0 + 1, window)) w &= 0x0000FFFFu;
                    sts32(vts + (uint32_t)(kj * 2048 + nj * 128 + (lane >> 2) * 16 + (lane & 3) * 4), w);
                }
            }
        }
        // (c) S = Q K^T; the next tile's V copy may start (vs is free)
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (S.abort) break;
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                umma_bf16(tbase, smem_desc(qs + kk * 4096, 2048, 128), smem_desc(ks + kk * 2048, 1024, 128), IDESC_S,
                          kk > 0);
            umma_commit(&S.s_bar);
        }
        if (k + 1 < nt) pt_copy_v(P, K.v_cache, c, c.tile(k + 1), vss, tid);
        // (d) the scores of this thread's row
        if (!mbar_wait_bounded(&S.s_bar, ph)) {
            pf_status(P, ST_TIMEOUT);
            S.abort = 1u;
        }
        tc_fence_after();
        if (k + 1 < nt) pt_copy_k(P, K.k_cache, c, c.tile(k + 1), ks, tid);   // K is free once S is done
        cp_async_commit();
        float s[64];
        tmem_ld64(t_lane, s);
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            const int n = n0 + i;
            const bool a = valid && n <= m && (retr || n < sink || n > m - window);
            s[i] = a ? s[i] * SCALE : -INFINITY;
            mx = fmaxf(mx, s[i]);
        }
        // a reference maximum that moves only in steps of more than 2^8 in P
        float alpha = 1.f;
        if (mx > m_ref + PT_RESCALE) {
            alpha = m_ref == -INFINITY ? 1.f : ex2_approx(m_ref - mx);
            m_ref = mx;
        }
        l *= alpha;
        if (k > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
            // rescale O (complete: the previous P V is done) in tensor memory
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float o[64];
                tmem_ld64(t_lane + 128 + 64 * half, o);
#pragma unroll
                for (int i = 0; i < 64; ++i) o[i] *= alpha;
                tmem_st64(t_lane + 128 + 64 * half, o);
            }
        }
        // P = 2^(x - m_ref) as bf16, row sum in fp32
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float p0 = m_ref == -INFINITY ? 0.f : ex2_approx(s[8 * ch + 2 * e] - m_ref);
                const float p1 = m_ref == -INFINITY ? 0.f : ex2_approx(s[8 * ch + 2 * e + 1] - m_ref);
                l += p0 + p1;
                w[e] = pack_bf16(p0, p1);
            }
            sts128(ps + (uint32_t)(ch * 2048 + row * 16), w[0], w[1], w[2], w[3]);
        }
        // (e) O += P V
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (S.abort) break;
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_bf16(tbase + 128, smem_desc(ps + kk * 4096, 2048, 128), smem_desc(vts + kk * 4096, 2048, 128),
                          IDESC_O, (k > 0 || kk > 0) ? 1u : 0u);
            umma_commit(&S.o_bar);
        }
        ph ^= 1u;
    }
    cp_async_wait_all();
    // ---- the output of this thread's row
    bool ok = S.abort == 0u && nt > 0;
    if (ok) {
        if (!mbar_wait_bounded(&S.o_bar, ph ^ 1u)) {
            pf_status(P, ST_TIMEOUT);
            S.abort = 1u;
        }
        tc_fence_after();
    }
    __syncthreads();
    ok = ok && S.abort == 0u;
    if (ok) {
        uint32_t* orow = reinterpret_cast<uint32_t*>(P.out + (((int64_t)c.b * P.Hq + h) * P.T + t) * D);
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float o[64];
            tmem_ld64(t_lane + 128 + 64 * half, o);
            if (valid && l > 0.f) {
#pragma unroll
                for (int i = 0; i < 32; ++i) orow[32 * half + i] = pack_bf16(o[2 * i] * inv, o[2 * i + 1] * inv);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_free(tbase, 256);
    }
}

}  // namespace rtp
