// Prefill attention of a chunk of queries (sm_100a), the method's second
// workload: in prefill the retrieval heads attend densely and causally, the
// local heads only to their sink and sliding window (review "RTPurbo" on
// dongryeollee1.github.io, Method: "Adaptive sparse attention", the prefill
// paragraph; Experiments, efficiency: the prefill speedups over dense
// attention; aitrends.kr summary, efficiency paragraph).
//
// Query t of sequence b sits at position m = pos[b] + t and attends, itself
// included:
//   retrieval head: [0, m]
//   local head    : [0, min(sink, m + 1)) U [max(0, m + 1 - window), m + 1)
// exact softmax(q.k / sqrt(128)) . v, bf16 out (round to nearest even).
//
// Work.  Per sequence, the (KV group, head kind) sets that hold at least one
// head; a set's units are (head, 16 consecutive positions); a CTA takes four
// units of one set, one per compute warp, so all its units read the same KV
// head: each 64-key tile is staged once (two 64 x 64 TMA boxes per K and V,
// 128-byte swizzle, a 3-stage ring fed by a copy warp) and serves up to 64
// query rows.  Per warp and tile: S = Q K^T (16 x 64: 64 MMAs m16n8k16, K
// from ldmatrix), online softmax in the log2 domain, O += P V (64 MMAs, V
// from ldmatrix.trans, P straight from S's accumulators).  Units are walked
// from the last positions down, so the CTAs with the most keys start first.
#pragma once
#include "rtp_attn.cuh"

namespace rtp {

constexpr int PF_UNITS = 4;                       // compute warps per CTA, one unit each
constexpr int PF_THREADS = (PF_UNITS + 1) * 32;   // + the copy warp
constexpr int PF_NST = 3;                         // K/V ring stages (32 KB each)
constexpr int PF_MAX_SETS = 2 * MAX_HKV;

struct PrefillParams {
    int B, Hq, Hkv, G, Ncap, mbps, num_pages, T, window, sink;
    int nt16;        // 16-position tiles per head: ceil(T / 16)
    int cta_per_b;   // CTAs per sequence
    int n_sets;
    int set_cta0[PF_MAX_SETS + 1];           // first CTA of set s within a sequence; [n_sets] = cta_per_b
    uint8_t set_g[PF_MAX_SETS], set_kind[PF_MAX_SETS], set_nh[PF_MAX_SETS];
    uint8_t set_heads[PF_MAX_SETS][MAX_G];   // the set's heads, as indices within the group
    const uint16_t* q;                       // [B, Hq, T, 128]
    const int32_t* pos;                      // [B]
    const int32_t* block_table;              // [B, mbps] or null
    uint16_t* out;                           // [B, Hq, T, 128]
    uint32_t* status;                        // optional device status word
};

struct PrefillK {
    CUtensorMap tmk, tmv;
    PrefillParams P;
};

struct PfSmem {
    alignas(1024) uint8_t stage[PF_NST][STAGE_BYTES];
    alignas(8) uint64_t full[PF_NST], empty[PF_NST];
    alignas(8) uint64_t zbar;   // the compute warps have zeroed an edge tile's unread value rows
};

__device__ __forceinline__ void pf_status(const PrefillParams& P, uint32_t code) {
    if (P.status) atomicCAS(P.status, 0u, code);
}

// The CTA's set, units and key tiles (computed alike by every warp).
struct PfCta {
    int b, set, g, kind, nh, units, u0, pos_b;
    bool ok;          // pos_b >= 0 and pos_b + T <= capacity
    int m_lo, m_hi;   // smallest and largest query position of the CTA's units
    int s_end;        // sink keys any row reads: [0, s_end)
    int w_lo;         // smallest window key any row reads (local heads)
    int j0a, j1a, j0b, j1b;   // key tiles [j0a, j1a), then [j0b, j1b)
    __device__ __forceinline__ int ntiles() const { return (j1a - j0a) + (j1b - j0b); }
    __device__ __forceinline__ int tile(int i) const { return i < j1a - j0a ? j0a + i : j0b + (i - (j1a - j0a)); }
    // can any row of this CTA read key n?
    __device__ __forceinline__ bool needed(int n, int window) const {
        if (n > m_hi) return false;
        return kind == 1 || n < s_end || (window > 0 && n >= w_lo);
    }
};

__device__ __forceinline__ PfCta pf_cta(const PrefillParams& P) {
    PfCta c;
    const int x = (int)blockIdx.x;
    c.b = x / P.cta_per_b;
    const int lc = x - c.b * P.cta_per_b;
    int lo = 0, hi = P.n_sets - 1;   // last set whose first CTA is <= lc
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
    c.u0 = (lc - P.set_cta0[lo]) * PF_UNITS;
    c.pos_b = __ldg(P.pos + c.b);
    c.ok = c.pos_b >= 0 && (long long)c.pos_b + P.T <= (long long)P.Ncap;
    // unit u: head set_heads[u % nh], positions 16 * (nt16 - 1 - u / nh) ..
    const int ulast = min(c.u0 + PF_UNITS, c.units) - 1;
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

// Cache row of (sequence b, KV head g, 64-key block j); a page id out of
// range reads page 0 and reports the input error.
__device__ __forceinline__ int pf_row(const PrefillParams& P, int b, int g, int j) {
    if (!P.block_table) return (int)(((int64_t)b * P.Hkv + g) * P.Ncap + (int64_t)j * BLK);
    int pg = __ldg(P.block_table + (int64_t)b * P.mbps + j);
    if (pg < 0 || pg >= P.num_pages) {
        pf_status(P, ST_DEVICE_INPUT);
        pg = 0;
    }
    return (pg * P.Hkv + g) * BLK;
}

__global__ void __launch_bounds__(PF_THREADS, 2) prefill_kernel(const __grid_constant__ PrefillK K) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    PfSmem& S = *reinterpret_cast<PfSmem*>(smem_raw);
    const PrefillParams& P = K.P;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (smem_u32(smem_raw) & 1023u) {   // the swizzled boxes need 1024-byte aligned stages
        if (tid == 0) pf_status(P, 5u);
        return;
    }
    const PfCta c = pf_cta(P);
    if (!c.ok) {
        if (tid == 0) pf_status(P, ST_DEVICE_INPUT);   // this sequence's outputs are not written
        return;
    }
    if (tid == 0) {
        for (int i = 0; i < PF_NST; ++i) {
            mbar_init(&S.full[i], 1);
            mbar_init(&S.empty[i], PF_UNITS);
        }
        mbar_init(&S.zbar, PF_UNITS);
        mbar_fence_init();
    }
    __syncthreads();
    const int nt = c.ntiles();

    if (warp == PF_UNITS) {
        // ---- the copy warp: K and V of every key tile, in order
        if (lane == 0) {
            int k = 0;
            for (; k < nt; ++k) {
                const int st = k % PF_NST;
                if (k >= PF_NST && !mbar_wait_bounded(&S.empty[st], ((k / PF_NST) - 1) & 1)) {
                    pf_status(P, ST_TIMEOUT);
                    break;
                }
                const int row = pf_row(P, c.b, c.g, c.tile(k));
                uint8_t* dst = &S.stage[st][0];
                mbar_expect_tx(&S.full[st], STAGE_BYTES);
                tma_load_2d(dst, &K.tmk, 0, row, &S.full[st]);
                tma_load_2d(dst + 8192, &K.tmk, 64, row, &S.full[st]);
                tma_load_2d(dst + KV_TILE, &K.tmv, 0, row, &S.full[st]);
                tma_load_2d(dst + KV_TILE + 8192, &K.tmv, 64, row, &S.full[st]);
            }
            // leave no copy in flight: the last tile issued into each stage lands first
            for (int i = (k > PF_NST ? k - PF_NST : 0); i < k; ++i) mbar_wait_bounded(&S.full[i % PF_NST], (i / PF_NST) & 1);
        }
        return;
    }

    // ---- compute warps: unit u = u0 + warp
    const int u = c.u0 + warp;
    const bool active = u < c.units;
    const int hl = active ? P.set_heads[c.set][u % c.nh] : 0;
    const int h = c.g * P.G + hl;
    const int t0 = active ? 16 * (P.nt16 - 1 - u / c.nh) : 0;
    const int gq = lane >> 2, t4 = lane & 3;
    // rows gq and gq + 8 of the unit: positions m0, m1 (tokens t0 + gq, t0 + gq + 8)
    const bool v0 = active && t0 + gq < P.T, v1 = active && t0 + gq + 8 < P.T;
    const int m0 = c.pos_b + t0 + gq, m1 = m0 + 8;
    // Q fragments (A operand, row-major 16 x 128): k-step kk covers dims 16kk..16kk+15
    uint32_t qa[8][4];
    {
        const uint32_t* q0 = reinterpret_cast<const uint32_t*>(P.q + (((int64_t)c.b * P.Hq + h) * P.T + t0 + gq) * D);
        const uint32_t* q1 = q0 + 8 * (D / 2);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            qa[kk][0] = v0 ? __ldg(q0 + 8 * kk + t4) : 0u;
            qa[kk][1] = v1 ? __ldg(q1 + 8 * kk + t4) : 0u;
            qa[kk][2] = v0 ? __ldg(q0 + 8 * kk + 4 + t4) : 0u;
            qa[kk][3] = v1 ? __ldg(q1 + 8 * kk + 4 + t4) : 0u;
        }
    }
    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float mr0 = -INFINITY, mr1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    constexpr float SCALE = 0.08838834764831845f * 1.4426950408889634f;   // log2(e)/sqrt(128)
    const bool retr = c.kind == 1;
    const int window = P.window, sink = P.sink;
    uint32_t zphase = 0;

    for (int k = 0; k < nt; ++k) {
        const int st = k % PF_NST;
        if (!mbar_wait_bounded(&S.full[st], (k / PF_NST) & 1)) {
            pf_status(P, ST_TIMEOUT);
            return;
        }
        const int n0 = c.tile(k) * BLK;
        const uint32_t Kb = smem_u32(&S.stage[st][0]), Vb = Kb + KV_TILE;
        // value rows no row of this CTA may read are zeroed first (they may
        // hold anything, NaN included, and meet a zero weight in P V)
        const bool edge = n0 + BLK - 1 > c.m_hi || (!retr && (n0 + BLK > c.s_end && n0 < c.w_lo));
        if (edge) {
            // each warp its 16 rows, then every warp waits (bounded) for all four
            const int r = warp * 16 + (lane >> 1);
            if (!c.needed(n0 + r, window)) {
                const uint32_t row = Vb + (uint32_t)((lane & 1) * 8192 + r * 128);
#pragma unroll
                for (int q = 0; q < 8; ++q) sts128_zero(row + q * 16);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.zbar);
            if (!mbar_wait_bounded(&S.zbar, zphase)) {
                pf_status(P, ST_TIMEOUT);
                return;
            }
            zphase ^= 1u;
        }
        if (active) {
            // S = Q K^T: four 32-dim steps x eight 8-key n-tiles
            float s[8][4];
#pragma unroll
            for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
            for (int kp = 0; kp < 4; ++kp)
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(sw_addr(Kb, 8 * j + (lane & 7), 4 * kp + (lane >> 3)), b0, b1, b2, b3);
                    mma_bf16(s[j], qa[2 * kp][0], qa[2 * kp][1], qa[2 * kp][2], qa[2 * kp][3], b0, b1);
                    mma_bf16(s[j], qa[2 * kp + 1][0], qa[2 * kp + 1][1], qa[2 * kp + 1][2], qa[2 * kp + 1][3], b2, b3);
                }
            // mask, scale to the log2 domain, row maxima over the four lanes of a row
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int n = n0 + 8 * j + 2 * t4 + e;
                    const bool ok0 = v0 && n <= m0 && (retr || n < sink || n > m0 - window);
                    const bool ok1 = v1 && n <= m1 && (retr || n < sink || n > m1 - window);
                    s[j][e] = ok0 ? s[j][e] * SCALE : -INFINITY;
                    s[j][2 + e] = ok1 ? s[j][2 + e] * SCALE : -INFINITY;
                    mx0 = fmaxf(mx0, s[j][e]);
                    mx1 = fmaxf(mx1, s[j][2 + e]);
                }
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
            const float mn0 = fmaxf(mr0, mx0), mn1 = fmaxf(mr1, mx1);
            const float a0 = mn0 == -INFINITY ? 1.f : ex2_approx(mr0 - mn0);
            const float a1 = mn1 == -INFINITY ? 1.f : ex2_approx(mr1 - mn1);
            float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    s[j][e] = mn0 == -INFINITY ? 0.f : ex2_approx(s[j][e] - mn0);
                    s[j][2 + e] = mn1 == -INFINITY ? 0.f : ex2_approx(s[j][2 + e] - mn1);
                    ps0 += s[j][e];
                    ps1 += s[j][2 + e];
                }
            l0 = l0 * a0 + ps0;
            l1 = l1 * a1 + ps1;
            mr0 = mn0;
            mr1 = mn1;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                o[i][0] *= a0;
                o[i][1] *= a0;
                o[i][2] *= a1;
                o[i][3] *= a1;
            }
            // O += P V: four 16-key steps x eight pairs of 8-dim n-tiles
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t pa0 = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
                const uint32_t pa1 = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
                const uint32_t pa2 = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
                const uint32_t pa3 = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
                const int vrow = 16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
                for (int np = 0; np < 8; ++np) {
                    uint32_t r0, r1, r2, r3;
                    ldsm_x4_t(sw_addr(Vb, vrow, 2 * np + (lane >> 4)), r0, r1, r2, r3);
                    mma_bf16(o[2 * np], pa0, pa1, pa2, pa3, r0, r1);
                    mma_bf16(o[2 * np + 1], pa0, pa1, pa2, pa3, r2, r3);
                }
            }
        }
        // zeroed rows are generic-proxy writes: order them before the
        // stage's next bulk copy
        if (edge) fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[st]);
    }
    if (!active) return;
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    uint32_t* o0 = reinterpret_cast<uint32_t*>(P.out + (((int64_t)c.b * P.Hq + h) * P.T + t0 + gq) * D);
    uint32_t* o1 = o0 + 8 * (D / 2);
    if (v0 && l0 > 0.f) {
        const float inv = 1.f / l0;
#pragma unroll
        for (int i = 0; i < 16; ++i) o0[4 * i + t4] = pack_bf16(o[i][0] * inv, o[i][1] * inv);
    }
    if (v1 && l1 > 0.f) {
        const float inv = 1.f / l1;
#pragma unroll
        for (int i = 0; i < 16; ++i) o1[4 * i + t4] = pack_bf16(o[i][2] * inv, o[i][3] * inv);
    }
}

}  // namespace rtp
