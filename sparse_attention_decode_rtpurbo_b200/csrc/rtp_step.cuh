// The decode step as ONE persistent, warp-specialized kernel (sm_100a).
//
// Sources: "Full Attention Strikes Back" (RTPurbo) review on
// dongryeollee1.github.io, Method: "Adaptive sparse attention" (local heads:
// sink + sliding window; retrieval heads: s_h(m,n) = (W^Q_h q^pre)^T
// (W^K_h k^pre), S_h(m) = Top-P(s_h(m,.), p), exact attention in full feature
// space) and "Hardware-aware top-p decoding kernel" (sort-free top-p: a
// 256-bin histogram of softmax mass per head, the last CTA finding where the
// cumulative mass reaches p_top and writing a block mask; block-sparse
// decoding); aitrends.kr summary items 2 and 5 ("Kernel 1 (D16)" scoring +
// histogram threshold, "Kernel 2 (D128)" block-sparse attention with a
// cross-split reduce).
//
// Work is a single in-order queue of items, claimed by CTAs with one atomic
// each:  [index-score chunks] [local-head tiles] [retrieval tiles].  Every
// CTA has one producer warp, which claims items, waits for their
// dependencies and streams their data (16-32 KB tiles) into a shared-memory
// ring with the bulk-copy engine, and four consumer warps, which compute.
// The index scores of a KV group are decided by the last CTA that finishes a
// chunk of it: when the best token alone reaches p (or p >= 1) the group's
// block list is written at once; otherwise the CTAs that have run out of
// queued items run an exact MSD radix select over the scores (4 passes of
// 256 bins of count and 2^-40 fixed-point mass), mark blocks and build the
// list.  Retrieval tiles are claimed after the local tiles, so in the common
// case they overlap the tail of the local-head stream.  Splits are combined
// by the last CTA of each (sequence, KV group).
//
// Deadlock freedom: only producer warps wait on other CTAs, and only for
// items claimed earlier by running CTAs whose consumers never wait on other
// CTAs.  Every wait is bounded (2 s of %globaltimer) and reports
// RTP_ERR_TIMEOUT.
#pragma once
#include "rtp_common.cuh"

namespace rtp {

constexpr int CONSUMERS = 128;                 // 4 consumer warps
constexpr int STEP_THREADS = CONSUMERS + 32;   // + 1 producer warp
constexpr int SCORE_ROWS = 1024;               // k_idx rows per score tile (32 KB)
constexpr int MAX_BG_CACHE = 256;

enum ItemType : int32_t { IT_SCORE = 0, IT_LOCAL = 1, IT_RET = 2, IT_RADIX = 3, IT_MARK = 4, IT_BLIST = 5, IT_STOP = 6 };

// Global coordination words (in the workspace; zero between calls: the last
// CTA to exit clears them).
struct Sync {
    uint32_t queue;            // main item queue
    uint32_t groups_decided;   // (b, retrieval group) pairs whose heads have a selection mode
    uint32_t groups_ready;     // ... whose block list is final
    uint32_t n_radix_heads;    // heads that need the radix select (list in rlist)
    uint32_t n_radix_groups;   // groups with at least one such head (list in rglist)
    uint32_t pass_claim[4], pass_done[4];
    uint32_t mark_claim, mark_done, blist_claim;
    uint32_t exit_count;
    uint32_t pad[16];
};

struct Desc {
    int32_t type, b, grp, item;
    int32_t tile, ntiles, n0, nvalid;
    uint32_t hmask;
    int32_t aux0, aux1, bad;
};

template <int G>
struct StepSmem {
    // G = 8 runs one CTA per SM (register bound), so it gets a deeper ring
    static constexpr int NST = (G >= 8) ? 4 : STAGES;
    alignas(128) uint8_t stage[NST][STAGE_BYTES];
    alignas(16) float red[4][G][D];   // per-warp partial sums of the attention accumulators; combine scratch
    alignas(16) float prob[BLK][G];
    float m_run[G], l_run[G], alpha[G];
    alignas(16) float qi[G][R];
    uint32_t hcnt[256];
    uint32_t hm[3][256];   // 17-bit slices of the per-bin fixed-point mass
    unsigned long long hmass[256];
    Desc desc[NST];
    alignas(8) uint64_t full[NST], empty[NST];
    uint32_t w_key[G][4], w_arg[G][4], w_min[G][4];
    float w_m[G][4];
    double w_sum[G][4];
    uint32_t flag, word;
    int dstar;
    int qi_tag;   // (b, retrieval group) whose q_idx is in qi, + 1; 0 = none
    unsigned long long acct[10];   // debug cycle accounting (thread 0)
};

// ---------------------------------------------------------------------------
// small utilities
// ---------------------------------------------------------------------------
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Bounded spin until *p >= target.  Returns false after about two seconds.
__device__ __forceinline__ bool wait_counter(const uint32_t* p, uint32_t target) {
    if (ld_acquire(p) >= target) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        __nanosleep(64);
        if (ld_acquire(p) >= target) return true;
        if (global_ns() - t0 > 2000000000ull) return false;
    }
}

// optional timeline (debug): latest %globaltimer of event i
__device__ __forceinline__ void trace_max(const Params& P, int i) {
    if (P.dbg_trace) atomicMax(P.dbg_trace + i, (unsigned long long)global_ns());
}

// Ticket among CONSUMER threads: true in exactly one of `count` arrivals.
__device__ __forceinline__ bool consumer_last(uint32_t* ctr, uint32_t count, uint32_t* smem_flag) {
    consumer_sync();
    if (threadIdx.x == 0) {
        __threadfence();
        const uint32_t t = atomicAdd(ctr, 1u);
        const bool last = (t == count - 1);
        if (last) {
            atomicExch(ctr, 0u);
            __threadfence();
        }
        *smem_flag = last;
    }
    consumer_sync();
    return *smem_flag != 0;
}

// per-sequence geometry of the local heads' block list
struct LocalGeom {
    int s_end, w_lo, nA, bw0, nv;
};
__device__ __forceinline__ LocalGeom local_geom(const Params& P, int L) {
    LocalGeom g;
    g.s_end = min(P.sink, L);
    g.w_lo = P.window > 0 ? max(0, L - P.window) : L;
    g.nA = (g.s_end + BLK - 1) / BLK;
    g.bw0 = max(g.w_lo / BLK, g.nA);
    const int nB = P.window > 0 ? max(0, (L + BLK - 1) / BLK - g.bw0) : 0;
    g.nv = g.nA + nB;
    return g;
}

// Element offset of the first row of block j of KV head g of sequence b.
__device__ __forceinline__ int64_t tile_off(const Params& P, int b, int g, int j, int dim, int* bad) {
    if (P.block_table == nullptr) return (((int64_t)b * P.Hkv + g) * P.Ncap + (int64_t)j * BLK) * dim;
    int pg = page_of(P, b, j);
    if (pg < 0) {
        *bad = 1;
        pg = 0;
    }
    return ((int64_t)pg * P.Hkv + g) * BLK * dim;
}

// Reduce-scatter over the 16 lanes that share bits 4.. of the lane id.
template <int CNT, int S>
struct ReduceScatter16 {
    static __device__ __forceinline__ void run(float* v, int lane) {
        if constexpr (CNT >= 2) {
            constexpr int H = CNT / 2;
            const bool up = (lane & S) != 0;
#pragma unroll
            for (int i = 0; i < H; ++i) {
                const float send = up ? v[i] : v[i + H];
                const float keep = up ? v[i + H] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, S);
            }
            if constexpr (S > 1) ReduceScatter16<H, S / 2>::run(v, lane);
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], S);
            if constexpr (S > 1) ReduceScatter16<1, S / 2>::run(v, lane);
        }
    }
    static __device__ __forceinline__ int base(int lane) {
        if constexpr (CNT >= 2) {
            constexpr int H = CNT / 2;
            const int here = (lane & S) ? H : 0;
            if constexpr (S > 1) return here + ReduceScatter16<H, S / 2>::base(lane);
            return here;
        } else {
            return 0;
        }
    }
};

// ---------------------------------------------------------------------------
// Attention over one 64x128 K/V tile for the G query heads of a KV group.
// Consumer thread (tg, dc): tg = token group of 8 tokens, dc = 16-byte chunk
// of the 128 dims; each warp reads two whole 256-byte rows per load.
// ---------------------------------------------------------------------------
template <int G>
struct AttnCore {
    float acc[G][8];
    float q[G][8];
    int q_tag = -1;   // (b, KV head) whose queries are in q

    __device__ __forceinline__ void begin(const Params& P, StepSmem<G>& S, int b, int g, int tid) {
        const int dc = tid & 15;
        const int tag = b * P.Hkv + g;
        if (tag != q_tag) {
            q_tag = tag;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const uint4 u =
                    *reinterpret_cast<const uint4*>(P.q_rope + ((int64_t)b * P.Hq + g * G + h) * D + dc * 8);
                const uint32_t* w = reinterpret_cast<const uint32_t*>(&u);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    q[h][2 * j] = bf_lo(w[j]);
                    q[h][2 * j + 1] = bf_hi(w[j]);
                }
            }
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[h][j] = 0.f;
        }
        if (tid < G) {
            S.m_run[tid] = -INFINITY;
            S.l_run[tid] = 0.f;
        }
        consumer_sync();
    }

    // `hmask`: group-local heads allowed to read this tile.  Row t (token
    // n0 + t) is readable iff t < nvalid and, for local heads, n lies in
    // [0, s_end) U [w_lo, L).  Unreadable rows never enter the arithmetic.
    __device__ __forceinline__ void tile(StepSmem<G>& S, const uint8_t* kv, uint32_t hmask, int n0, int nvalid,
                                         bool local, int s_end, int w_lo, int tid) {
        const int lane = tid & 31, tg = tid >> 4, dc = tid & 15;
        const uint32_t K = smem_u32(kv), V = K + TILE_BYTES;
        constexpr int CNT = 8 * G;
        constexpr int NV = CNT >= 16 ? CNT / 16 : 1;
        float v[CNT];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const uint4 u = lds128(K + ((tg * 8 + t) * 16 + dc) * 16);
            const uint32_t* w = reinterpret_cast<const uint32_t*>(&u);
            float k8[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                k8[2 * j] = bf_lo(w[j]);
                k8[2 * j + 1] = bf_hi(w[j]);
            }
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float s = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) s = fmaf(k8[j], q[h][j], s);
                v[t * G + h] = s;
            }
        }
        ReduceScatter16<CNT, 8>::run(v, lane);
        const int base = ReduceScatter16<CNT, 8>::base(lane);
        constexpr float SCALE = 0.08838834764831845f * 1.4426950408889634f;   // log2(e)/sqrt(128)
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int idx = base + i;
            const int t = idx / G, h = idx % G;
            const int tok = tg * 8 + t;
            const int n = n0 + tok;
            bool ok = tok < nvalid && ((hmask >> h) & 1u);
            if (local) ok = ok && (n < s_end || n >= w_lo);
            S.prob[tok][h] = ok ? v[i] * SCALE : -INFINITY;
        }
        consumer_sync();
        const int warp = tid >> 5;
        for (int h = warp; h < G; h += CONSUMERS / 32) {
            const float x0 = S.prob[lane][h], x1 = S.prob[lane + 32][h];
            float bm = fmaxf(x0, x1);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
            const float m_old = S.m_run[h];
            const float m_new = fmaxf(m_old, bm);
            float p0 = 0.f, p1 = 0.f, a = 1.f;
            if (m_new != -INFINITY) {
                p0 = exp2f(x0 - m_new);
                p1 = exp2f(x1 - m_new);
                a = exp2f(m_old - m_new);
            }
            float sum = p0 + p1;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            S.prob[lane][h] = p0;
            S.prob[lane + 32][h] = p1;
            if (lane == 0) {
                S.l_run[h] = S.l_run[h] * a + sum;
                S.m_run[h] = m_new;
                S.alpha[h] = a;
            }
        }
        consumer_sync();
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float a = S.alpha[h];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[h][j] *= a;
        }
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const int tok = tg * 8 + t;
            const int n = n0 + tok;
            bool ok = tok < nvalid;
            if (local) ok = ok && (n < s_end || n >= w_lo);
            if (!ok) continue;
            const uint4 u = lds128(V + (tok * 16 + dc) * 16);
            const uint32_t* w = reinterpret_cast<const uint32_t*>(&u);
            float v8[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                v8[2 * j] = bf_lo(w[j]);
                v8[2 * j + 1] = bf_hi(w[j]);
            }
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float pr = S.prob[tok][h];
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[h][j] = fmaf(pr, v8[j], acc[h][j]);
            }
        }
        consumer_sync();
    }

    // Partial (m, l, acc[128]) of every head in `heads` -> part[h * PSTRIDE].
    __device__ __forceinline__ void flush(StepSmem<G>& S, float* part, uint32_t heads, int tid) {
        const int warp = tid >> 5, lane = tid & 31, dc = tid & 15;
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[h][j] += __shfl_xor_sync(0xffffffffu, acc[h][j], 16);
        if (lane < 16) {
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int j = 0; j < 8; ++j) S.red[warp][h][dc * 8 + j] = acc[h][j];
        }
        consumer_sync();
        for (int h = 0; h < G; ++h) {
            if (!((heads >> h) & 1u)) continue;
            const float s = S.red[0][h][tid] + S.red[1][h][tid] + S.red[2][h][tid] + S.red[3][h][tid];
            part[h * PSTRIDE + 4 + tid] = s;
            if (tid == 0) {
                part[h * PSTRIDE + 0] = S.m_run[h];
                part[h * PSTRIDE + 1] = S.l_run[h];
            }
        }
        consumer_sync();
    }
};

// Combine the partials of `nparts` splits (stride G*PSTRIDE floats) of the
// heads in `heads` into out[b, g*G + h] (bf16, round to nearest even).
template <int G>
__device__ __forceinline__ void combine_parts(const Params& P, StepSmem<G>& S, const float* parts, int nparts, uint32_t heads, int b,
                              int g, int tid) {
    float* wts = &S.red[0][0][0];   // G * nparts weights (nparts <= 4*D)
    __shared__ float s_den[G];
    for (int x = tid; x < G * nparts; x += CONSUMERS) {
        const int h = x % G, i = x / G;
        const float* pp = parts + ((int64_t)i * G + h) * PSTRIDE;
        wts[h * nparts + i] = (__ldcg(pp + 1) > 0.f) ? __ldcg(pp) : -INFINITY;
    }
    consumer_sync();
    const int warp = tid >> 5, lane = tid & 31;
    for (int h = warp; h < G; h += CONSUMERS / 32) {
        float m = -INFINITY;
        for (int i = lane; i < nparts; i += 32) m = fmaxf(m, wts[h * nparts + i]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float den = 0.f;
        for (int i = lane; i < nparts; i += 32) {
            const float mi = wts[h * nparts + i];
            const float w = (mi == -INFINITY) ? 0.f : exp2f(mi - m);
            wts[h * nparts + i] = w;
            if (w > 0.f) den += w * __ldcg(parts + ((int64_t)i * G + h) * PSTRIDE + 1);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
        if (lane == 0) s_den[h] = den;
    }
    consumer_sync();
    for (int x = tid; x < G * 32; x += CONSUMERS) {
        const int h = x / 32, q4 = x % 32;
        if (!((heads >> h) & 1u)) continue;
        const float den = s_den[h];
        if (!(den > 0.f)) continue;
        float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
        int i = 0;
        for (; i + 1 < nparts; i += 2) {
            const float w0 = wts[h * nparts + i], w1 = wts[h * nparts + i + 1];
            const float4 v0 = __ldcg(reinterpret_cast<const float4*>(parts + ((int64_t)i * G + h) * PSTRIDE + 4) + q4);
            const float4 v1 =
                __ldcg(reinterpret_cast<const float4*>(parts + ((int64_t)(i + 1) * G + h) * PSTRIDE + 4) + q4);
            a0.x = fmaf(w0, v0.x, a0.x);
            a0.y = fmaf(w0, v0.y, a0.y);
            a0.z = fmaf(w0, v0.z, a0.z);
            a0.w = fmaf(w0, v0.w, a0.w);
            a1.x = fmaf(w1, v1.x, a1.x);
            a1.y = fmaf(w1, v1.y, a1.y);
            a1.z = fmaf(w1, v1.z, a1.z);
            a1.w = fmaf(w1, v1.w, a1.w);
        }
        if (i < nparts) {
            const float w0 = wts[h * nparts + i];
            const float4 v0 = __ldcg(reinterpret_cast<const float4*>(parts + ((int64_t)i * G + h) * PSTRIDE + 4) + q4);
            a0.x = fmaf(w0, v0.x, a0.x);
            a0.y = fmaf(w0, v0.y, a0.y);
            a0.z = fmaf(w0, v0.z, a0.z);
            a0.w = fmaf(w0, v0.w, a0.w);
        }
        const float inv = 1.f / den;
        const uint32_t lo = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn((a0.x + a1.x) * inv)) |
                            ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn((a0.y + a1.y) * inv)) << 16);
        const uint32_t hi = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn((a0.z + a1.z) * inv)) |
                            ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn((a0.w + a1.w) * inv)) << 16);
        *reinterpret_cast<uint2*>(P.out + ((int64_t)b * P.Hq + g * G + h) * D + q4 * 4) = make_uint2(lo, hi);
    }
    consumer_sync();
}

}  // namespace rtp
