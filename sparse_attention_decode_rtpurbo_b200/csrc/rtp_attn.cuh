// Warp-level tensor-core cores of the decode step (sm_100a, mma.sync bf16):
// exact split-KV attention of a KV group's query heads over staged K/V
// tiles, the log-sum-exp combine of splits, and the rank-16 index scores.
//
// Sources: "Full Attention Strikes Back" (RTPurbo) review on
// dongryeollee1.github.io, Method: "Adaptive sparse attention" (exact
// softmax attention over the selected tokens in the full feature space;
// s_h(m,n) = (W^Q_h q^pre)^T k^idx_n) and "Hardware-aware top-p decoding
// kernel" (block-sparse decoding); aitrends.kr summary, item 5 (block-sparse
// attention with a cross-split reduce).
#pragma once
#include "rtp_common.cuh"

namespace rtp {

// Per-CTA scratch of the attention split epilogue.
template <int G>
struct AttnScratch {
    alignas(16) float red[4][G][D];   // per-warp unnormalised outputs
    float wm[4][G], wl[4][G];         // per-warp running max (log2 units) and sum
    float cm[G], cden[G];             // combine: max and denominator per head
#ifdef RTP_ATTN_FMA
    alignas(16) uint16_t qf[4][G][D];   // FmaAttn: each compute warp's copy of its group's queries (bf16)
#endif
};

// Address of 16-byte chunk c (0..15, 8 dims each) of row `row` of a 64 x 128
// bf16 tile staged as two 64 x 64 boxes (dims 0-63, 64-127) with the TMA
// 128-byte swizzle: chunk c of a 128-byte row sits at chunk c ^ (row % 8).
__device__ __forceinline__ uint32_t sw_addr(uint32_t base, int row, int c) {
    return base + (uint32_t)((c >> 3) * 8192 + row * 128 + (((c & 7) ^ (row & 7)) << 4));
}

// ---------------------------------------------------------------------------
// Attention of the G query heads of one KV group, one warp per 16 tokens of
// each 64-token tile.  Per warp and 16 tokens:
//   S (heads x 16 tokens)  = Q (heads padded to 16, 128) . K^T   16 MMAs, B from ldmatrix of K rows
//   O^T (128 x heads)     += V^T (128 x 16 tokens) . P^T        8 MMAs, A from ldmatrix.trans of V rows
// The C fragment of S (head = lane/4, tokens 2(lane%4), +1) is exactly the B
// fragment P^T needs, so P never leaves registers.  Every warp keeps its own
// online softmax (log2 domain); the CTA merges the four at the split's end.
// ---------------------------------------------------------------------------
template <int G>
struct MmaAttn {
    uint32_t qa[8][2];   // A fragments of Q, row = head lane/4: dims 16kk+2t.. and 16kk+8+2t..
    float o[8][4];       // O^T: m-tile i = dims 16i..16i+15; c0,c1 = (16i+g, heads 2t, 2t+1), c2,c3 = (16i+g+8, ..)
    float m, l;          // head lane/4: running max of the scaled logits, this thread's share of the sum
    int q_tag;

    __device__ __forceinline__ void init(uint32_t = 0u) { q_tag = -1; }

    // arrive: the CTA's first segment (named barrier 4 lets the copy warp
    // issue the first tile once the query loads are on their way)
    __device__ __forceinline__ void begin(const Params& P, int b, int g, int lane, bool arrive = false) {
        const int tag = b * P.Hkv + g;
        if (tag != q_tag) {
            q_tag = tag;
            const int hr = lane >> 2, t = lane & 3;
            const uint32_t* q =
                reinterpret_cast<const uint32_t*>(P.q_rope + ((int64_t)b * P.Hq + g * G + min(hr, G - 1)) * D);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                qa[kk][0] = hr < G ? __ldg(q + 8 * kk + t) : 0u;
                qa[kk][1] = hr < G ? __ldg(q + 8 * kk + 4 + t) : 0u;
            }
        }
        if (arrive) asm volatile("bar.arrive 4, 160;" ::: "memory");
        m = -INFINITY;
        l = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    }

    // This warp's 16 rows (16*warp ..) of the staged tile: row r is token
    // n0 + r, readable iff r < nvalid and, for local heads, the token lies in
    // [0, s_end) U [w_lo, L); head h attends iff bit h of hmask is set.
    // Rows no head may read never enter the arithmetic: their logits are
    // replaced by -inf and their V rows are zeroed in shared memory first
    // (returns true then: the caller orders those writes before the stage's
    // next bulk copy).
    __device__ __forceinline__ bool tile(uint32_t K, uint32_t V, int warp, int lane, int n0, int nvalid,
                                         uint32_t hmask, bool local, int s_end, int w_lo) {
        const int hr = lane >> 2, t = lane & 3;
        const int r0 = warp * 16;
        const int rl = r0 + (lane & 15), nl = n0 + rl;
        const bool rd = rl < nvalid && (!local || nl < s_end || nl >= w_lo);
        const uint32_t bad = ~__ballot_sync(0xffffffffu, rd) & 0xFFFFu;
        if (bad) {
            const int tr = lane >> 1;   // lane pair per row, one 128-byte half each
            if ((bad >> tr) & 1u) {
                const uint32_t row = V + (uint32_t)((lane & 1) * 8192 + (r0 + tr) * 128);
#pragma unroll
                for (int c = 0; c < 8; ++c) sts128_zero(row + c * 16);
            }
            __syncwarp();
        }
        // QK^T: four independent accumulator chains per 8-token n-tile (the
        // MMA latency, not its rate, bounds a warp), summed at the end
        float sa[2][4][4];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int kp = 0; kp < 4; ++kp) sa[j][kp][0] = sa[j][kp][1] = sa[j][kp][2] = sa[j][kp][3] = 0.f;
#pragma unroll
        for (int kp = 0; kp < 4; ++kp) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(sw_addr(K, r0 + 8 * j + (lane & 7), 4 * kp + (lane >> 3)), b0, b1, b2, b3);
                mma_bf16(sa[j][kp], qa[2 * kp][0], 0u, qa[2 * kp][1], 0u, b0, b1);
                mma_bf16(sa[j][kp], qa[2 * kp + 1][0], 0u, qa[2 * kp + 1][1], 0u, b2, b3);
            }
        }
        float s[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[j][e] = (sa[j][0][e] + sa[j][1][e]) + (sa[j][2][e] + sa[j][3][e]);
        constexpr float SCALE = 0.08838834764831845f * 1.4426950408889634f;   // log2(e)/sqrt(128)
        const bool hok = (hmask >> hr) & 1u;
        float x[4];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int r = r0 + 8 * j + 2 * t + e, n = n0 + r;
                const bool ok = hok && r < nvalid && (!local || n < s_end || n >= w_lo);
                x[2 * j + e] = ok ? s[j][e] * SCALE : -INFINITY;
            }
        float mt = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
        const float m_new = fmaxf(m, mt);
        float alpha = 1.f, p[4] = {0.f, 0.f, 0.f, 0.f};
        if (m_new != -INFINITY) {
            alpha = ex2_approx(m - m_new);
#pragma unroll
            for (int i = 0; i < 4; ++i) p[i] = ex2_approx(x[i] - m_new);
        }
        l = l * alpha + ((p[0] + p[1]) + (p[2] + p[3]));
        m = m_new;
        // O^T columns are heads 2t, 2t+1: their rescale factors live in lanes 8t, 8t+4
        const float a0 = __shfl_sync(0xffffffffu, alpha, 8 * t);
        const float a1 = __shfl_sync(0xffffffffu, alpha, 8 * t + 4);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            o[i][0] *= a0;
            o[i][1] *= a1;
            o[i][2] *= a0;
            o[i][3] *= a1;
        }
        const uint32_t pb0 = pack_bf16(p[0], p[1]), pb1 = pack_bf16(p[2], p[3]);
        const int mi = lane >> 3;
        const int vrow = r0 + (mi >> 1) * 8 + (lane & 7);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t a0r, a1r, a2r, a3r;
            ldsm_x4_t(sw_addr(V, vrow, 2 * i + (mi & 1)), a0r, a1r, a2r, a3r);
            mma_bf16(o[i], a0r, a1r, a2r, a3r, pb0, pb1);
        }
        return bad != 0;
    }

    // This warp's state -> scratch (rows of heads < G only).
    __device__ __forceinline__ void finish(AttnScratch<G>& X, int warp, int lane) {
        const int hr = lane >> 2, t = lane & 3;
        float lt = l + __shfl_xor_sync(0xffffffffu, l, 1);
        lt += __shfl_xor_sync(0xffffffffu, lt, 2);
        if (t == 0 && hr < G) {
            X.wm[warp][hr] = m;
            X.wl[warp][hr] = lt;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int d0 = 16 * i + hr;
            if (2 * t < G) {
                X.red[warp][2 * t][d0] = o[i][0];
                X.red[warp][2 * t][d0 + 8] = o[i][2];
            }
            if (2 * t + 1 < G) {
                X.red[warp][2 * t + 1][d0] = o[i][1];
                X.red[warp][2 * t + 1][d0 + 8] = o[i][3];
            }
        }
    }
};

#ifdef RTP_ATTN_FMA
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

// The same per-warp split attention on the FP32 FMA pipe instead of the
// tensor cores (a build with RTP_ATTN_FMA defined), kept to compare the two
// on the same kernels: scores with lane = (token lane % 16, half of the 128
// dims), then P V with lane = 4 output dims of every head.  Same inputs,
// masks, online softmax (log2 domain) and per-warp state as MmaAttn, so
// split_emit and combine_splits serve both.
template <int G>
struct FmaAttn {
    float o[G][4];   // dims 4 lane .. 4 lane + 3 of every head
    float m[G], l[G];
    int q_tag;
    uint32_t qs;     // this warp's query copy in shared memory (bf16 [G][128])

    __device__ __forceinline__ void init(uint32_t q_smem) {
        q_tag = -1;
        qs = q_smem;
    }

    __device__ __forceinline__ void begin(const Params& P, int b, int g, int lane, bool arrive = false) {
        const int tag = b * P.Hkv + g;
        if (tag != q_tag) {
            q_tag = tag;
            __syncwarp();   // (the previous segment's reads of the copy are done)
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const uint2 v = __ldg(reinterpret_cast<const uint2*>(P.q_rope + ((int64_t)b * P.Hq + g * G + h) * D) + lane);
                asm volatile("st.shared.v2.u32 [%0], {%1,%2};" ::"r"(qs + (uint32_t)(h * D + 4 * lane) * 2), "r"(v.x),
                             "r"(v.y)
                             : "memory");
            }
            __syncwarp();
        }
        if (arrive) asm volatile("bar.arrive 4, 160;" ::: "memory");
#pragma unroll
        for (int h = 0; h < G; ++h) {
            m[h] = -INFINITY;
            l[h] = 0.f;
            o[h][0] = o[h][1] = o[h][2] = o[h][3] = 0.f;
        }
    }

    __device__ __forceinline__ bool tile(uint32_t K, uint32_t V, int warp, int lane, int n0, int nvalid,
                                         uint32_t hmask, bool local, int s_end, int w_lo) {
        const int r0 = warp * 16;
        const int rl = r0 + (lane & 15), nl = n0 + rl;
        const bool rd = rl < nvalid && (!local || nl < s_end || nl >= w_lo);
        const uint32_t bad = ~__ballot_sync(0xffffffffu, rd) & 0xFFFFu;
        if (bad) {
            const int tr = lane >> 1;
            if ((bad >> tr) & 1u) {
                const uint32_t row = V + (uint32_t)((lane & 1) * 8192 + (r0 + tr) * 128);
#pragma unroll
                for (int c = 0; c < 8; ++c) sts128_zero(row + c * 16);
            }
            __syncwarp();
        }
        // partial dots over this lane's 64 dims, every head
        const int hf = lane >> 4;
        float acc[G];
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = 0.f;
#pragma unroll 2
        for (int c = 0; c < 8; ++c) {
            const uint4 kv = lds128(sw_addr(K, rl, 8 * hf + c));
            const uint32_t ku[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const uint4 qv = lds128(qs + (uint32_t)(h * D + (8 * hf + c) * 8) * 2);
                const uint32_t qu[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[h] = fmaf(bf_lo(ku[j]), bf_lo(qu[j]), acc[h]);
                    acc[h] = fmaf(bf_hi(ku[j]), bf_hi(qu[j]), acc[h]);
                }
            }
        }
        constexpr float SCALE = 0.08838834764831845f * 1.4426950408889634f;   // log2(e)/sqrt(128)
        float pr[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float sc = acc[h] + __shfl_xor_sync(0xffffffffu, acc[h], 16);
            const float x = (rd && ((hmask >> h) & 1u)) ? sc * SCALE : -INFINITY;
            float mt = x;
#pragma unroll
            for (int ofs = 8; ofs > 0; ofs >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, ofs));
            const float mn = fmaxf(m[h], mt);
            const float alpha = mn == -INFINITY ? 1.f : ex2_approx(m[h] - mn);
            const float p = mn == -INFINITY ? 0.f : ex2_approx(x - mn);
            float ps = p;
#pragma unroll
            for (int ofs = 8; ofs > 0; ofs >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, ofs);
            l[h] = l[h] * alpha + ps;
            m[h] = mn;
            pr[h] = p;
            o[h][0] *= alpha;
            o[h][1] *= alpha;
            o[h][2] *= alpha;
            o[h][3] *= alpha;
        }
        // O += P V over the warp's 16 tokens: lane holds dims 4 lane .. 4 lane + 3
#pragma unroll 4
        for (int r = 0; r < 16; ++r) {
            const uint2 vv = lds64(sw_addr(V, r0 + r, lane >> 1) + (uint32_t)(lane & 1) * 8u);
            const float v0 = bf_lo(vv.x), v1 = bf_hi(vv.x), v2 = bf_lo(vv.y), v3 = bf_hi(vv.y);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float p = __shfl_sync(0xffffffffu, pr[h], r);
                o[h][0] = fmaf(p, v0, o[h][0]);
                o[h][1] = fmaf(p, v1, o[h][1]);
                o[h][2] = fmaf(p, v2, o[h][2]);
                o[h][3] = fmaf(p, v3, o[h][3]);
            }
        }
        return bad != 0;
    }

    __device__ __forceinline__ void finish(AttnScratch<G>& X, int warp, int lane) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            if (lane == 0) {
                X.wm[warp][h] = m[h];
                X.wl[warp][h] = l[h];
            }
            *reinterpret_cast<float4*>(&X.red[warp][h][4 * lane]) = make_float4(o[h][0], o[h][1], o[h][2], o[h][3]);
        }
    }
};
template <int G>
using Attn = FmaAttn<G>;
template <int G>
__device__ __forceinline__ uint32_t attn_q_smem(AttnScratch<G>& X, int warp) { return smem_u32(&X.qf[warp][0][0]); }
#else
template <int G>
using Attn = MmaAttn<G>;
template <int G>
__device__ __forceinline__ uint32_t attn_q_smem(AttnScratch<G>&, int) { return 0u; }
#endif

// Merge the four warps of a split (after finish + consumer_sync): each
// consumer thread owns one of the 128 dims.  Writes the split's partial
// (m, l, acc[128]) per head in `heads` to part[h * PSTRIDE], or, when part is
// null (the split is the whole item), the normalised bf16 output to
// out0[h * D] (out0 = the group's first head row).
template <int G>
__device__ __forceinline__ void split_emit(const AttnScratch<G>& X, uint32_t heads, float* part, uint16_t* out0,
                                           int tid) {
#pragma unroll 1
    for (int h = 0; h < G; ++h) {
        if (!((heads >> h) & 1u)) continue;
        const float M = fmaxf(fmaxf(X.wm[0][h], X.wm[1][h]), fmaxf(X.wm[2][h], X.wm[3][h]));
        float acc = 0.f, Lh = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float e = ex2_approx(X.wm[w][h] - M);
                acc = fmaf(X.red[w][h][tid], e, acc);
                Lh = fmaf(X.wl[w][h], e, Lh);
            }
        }
        if (part) {
            part[h * PSTRIDE + 4 + tid] = acc;
            if (tid == 0) {
                part[h * PSTRIDE + 0] = M;
                part[h * PSTRIDE + 1] = Lh;
            }
        } else if (Lh > 0.f) {
            out0[h * D + tid] = __bfloat16_as_ushort(__float2bfloat16_rn(acc / Lh));
        }
    }
}

// Combine `nparts` split partials (stride G * PSTRIDE floats) of the heads in
// `heads` into the bf16 outputs out0[h * D] (round to nearest even).  The
// split weights 2^(m_i - M) go to shared memory first (X.red, free once the
// splits are emitted, as [part][head]); then thread d sums column d of every
// head with 8 parts x G heads of loads in flight at a time, so that a
// combine costs about nparts / 8 memory round trips rather than one per part.
template <int G>
__device__ __noinline__ void combine_splits(AttnScratch<G>& X, const float* parts, int nparts, uint32_t heads,
                                            uint16_t* out0, int tid) {
    const int warp = tid >> 5, lane = tid & 31;
    float* wts = &X.red[0][0][0];   // [nparts][G]
    const bool in_smem = nparts <= 4 * D;
    for (int h = warp; h < G; h += CONSUMERS / 32) {
        // (m, l) of parts lane and lane + 32 stay in registers
        float mr[2], lr[2];
        float M = -INFINITY;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int i = lane + 32 * r;
            mr[r] = -INFINITY;
            lr[r] = 0.f;
            if (i < nparts) {
                const float* pp = parts + ((int64_t)i * G + h) * PSTRIDE;
                mr[r] = __ldcg(pp);
                lr[r] = __ldcg(pp + 1);
            }
            if (lr[r] > 0.f) M = fmaxf(M, mr[r]);
        }
        for (int i = lane + 64; i < nparts; i += 32) {
            const float* pp = parts + ((int64_t)i * G + h) * PSTRIDE;
            if (__ldcg(pp + 1) > 0.f) M = fmaxf(M, __ldcg(pp));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float den = 0.f;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int i = lane + 32 * r;
            const float w = (M != -INFINITY && lr[r] > 0.f) ? ex2_approx(mr[r] - M) : 0.f;
            den = fmaf(lr[r] > 0.f ? lr[r] : 0.f, w, den);
            if (in_smem && i < nparts) wts[i * G + h] = w;
        }
        for (int i = lane + 64; i < nparts; i += 32) {
            const float* pp = parts + ((int64_t)i * G + h) * PSTRIDE;
            const float li = __ldcg(pp + 1);
            const float w = (M != -INFINITY && li > 0.f) ? ex2_approx(__ldcg(pp) - M) : 0.f;
            den = fmaf(li > 0.f ? li : 0.f, w, den);
            if (in_smem) wts[i * G + h] = w;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
        if (lane == 0) {
            X.cm[h] = M;
            X.cden[h] = den;
        }
    }
    consumer_sync();
    if (in_smem) {
        constexpr int U = G >= 8 ? 8 : 16;   // parts per batch: 64 loads in flight per thread
        float acc[G];
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = 0.f;
        const float* col = parts + 4 + tid;
        for (int i = 0; i < nparts; i += U) {
            float v[U][G];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int h = 0; h < G; ++h)
                    v[u][h] = (i + u < nparts && ((heads >> h) & 1u))
                                  ? __ldcg(col + ((int64_t)(i + u) * G + h) * PSTRIDE) : 0.f;
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int h = 0; h < G; ++h)
                    if (i + u < nparts) acc[h] = fmaf(wts[(i + u) * G + h], v[u][h], acc[h]);
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float den = X.cden[h];
            if (((heads >> h) & 1u) && den > 0.f)
                out0[h * D + tid] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[h] / den));
        }
    } else {
#pragma unroll 1
        for (int h = 0; h < G; ++h) {
            if (!((heads >> h) & 1u)) continue;
            const float den = X.cden[h], M = X.cm[h];
            if (!(den > 0.f)) continue;
            float a = 0.f;
            for (int i = 0; i < nparts; ++i) {
                const float* p0 = parts + ((int64_t)i * G + h) * PSTRIDE;
                if (__ldcg(p0 + 1) > 0.f) a = fmaf(ex2_approx(__ldcg(p0) - M), __ldcg(p0 + 4 + tid), a);
            }
            out0[h * D + tid] = __bfloat16_as_ushort(__float2bfloat16_rn(a / den));
        }
    }
    consumer_sync();
}

// ---------------------------------------------------------------------------
// Index scores on the tensor cores: per 16 staged k_idx rows, one m16n8k16
// MMA against each of three bf16 parts of q_idx (hi + mid + lo = q_idx to
// fp32 precision; every bf16 x bf16 product is exact, the sums are fp32).
// N = 8 columns = the group's retrieval heads.  Lane (g = lane/4, t = lane%4)
// gets the scores of heads 2t, 2t+1 for rows g and g+8.
// ---------------------------------------------------------------------------
struct QFrag {
    uint32_t b[3][2];
};

// q_idx[hh][r] = Wq_idx[h] . q_pre[b,h] (fp32, fixed summation order) for the
// nh retrieval heads of group rg, by the 128 consumer threads: TPP threads per
// (head, r) pair, each over D / TPP elements, with every load of a thread
// issued before its first product (one or two memory round trips, not D / 8).
template <int TPP>
__device__ __forceinline__ void qidx_pairs(const Params& P, const HeadTab& T, float (*qi)[R], int b, int rg,
                                           int tid, bool arrive) {
    constexpr int SPAN = D / TPP, NV = SPAN / 8;
    const int nh = T.rg_nh[rg], slot0 = T.rg_slot0[rg];
    const int pr = tid / TPP, part = tid % TPP;
    // threads beyond the nh x 16 pairs load pair 0's operands (valid
    // addresses, no branch around the loads) and store nothing
    const int pe = pr < nh * R ? pr : 0;
    const int hh = pe / R, r = pe % R;
    const int h = T.slot_head[slot0 + hh];
    const uint4* w = reinterpret_cast<const uint4*>(P.Wq + ((int64_t)h * R + r) * D + part * SPAN);
    const uint4* q = reinterpret_cast<const uint4*>(P.q_pre + ((int64_t)b * P.Hq + h) * D + part * SPAN);
    constexpr int NB = NV < 8 ? NV : 8;   // loads in flight per operand (register budget)
    float a = 0.f;
#pragma unroll
    for (int i0 = 0; i0 < NV; i0 += NB) {
        uint4 wv[NB], qv[NB];
#pragma unroll
        for (int i = 0; i < NB; ++i) {
            wv[i] = __ldg(w + i0 + i);
            qv[i] = __ldg(q + i0 + i);
        }
        // the CTA's first segment: its copy warp issues the first tile only
        // once these loads are on their way (named barrier 4)
        if (i0 == 0 && arrive) asm volatile("bar.arrive 4, 160;" ::: "memory");
#pragma unroll
        for (int i = 0; i < NB; ++i) {
            a = fmaf(bf_lo(wv[i].x), bf_lo(qv[i].x), a);
            a = fmaf(bf_hi(wv[i].x), bf_hi(qv[i].x), a);
            a = fmaf(bf_lo(wv[i].y), bf_lo(qv[i].y), a);
            a = fmaf(bf_hi(wv[i].y), bf_hi(qv[i].y), a);
            a = fmaf(bf_lo(wv[i].z), bf_lo(qv[i].z), a);
            a = fmaf(bf_hi(wv[i].z), bf_hi(qv[i].z), a);
            a = fmaf(bf_lo(wv[i].w), bf_lo(qv[i].w), a);
            a = fmaf(bf_hi(wv[i].w), bf_hi(qv[i].w), a);
        }
    }
#pragma unroll
    for (int o = 1; o < TPP; o <<= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (pr < nh * R && part == 0) qi[pr / R][pr % R] = a;
}

__device__ __forceinline__ void compute_qidx(const Params& P, const HeadTab& T, float (*qi)[R], int b, int rg,
                                             int tid, bool arrive = false) {
    const int npair = T.rg_nh[rg] * R;   // <= 128
    if (npair <= CONSUMERS / 8) qidx_pairs<8>(P, T, qi, b, rg, tid, arrive);
    else if (npair <= CONSUMERS / 4) qidx_pairs<4>(P, T, qi, b, rg, tid, arrive);
    else if (npair <= CONSUMERS / 2) qidx_pairs<2>(P, T, qi, b, rg, tid, arrive);
    else qidx_pairs<1>(P, T, qi, b, rg, tid, arrive);
}

// B fragment of this lane (column g = lane/4 = head g; k = 2t, 2t+1, 2t+8, 2t+9)
__device__ __forceinline__ QFrag make_qfrag(const float (*qi)[R], int nh, int lane) {
    const int g = lane >> 2, t = lane & 3;
    float qv[4] = {0.f, 0.f, 0.f, 0.f};
    if (g < nh) {
        qv[0] = qi[g][2 * t];
        qv[1] = qi[g][2 * t + 1];
        qv[2] = qi[g][2 * t + 8];
        qv[3] = qi[g][2 * t + 9];
    }
    uint16_t part[3][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat16 hi = __float2bfloat16_rn(qv[i]);
        const float r1 = qv[i] - __bfloat162float(hi);
        const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
        const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
        part[0][i] = __bfloat16_as_ushort(hi);
        part[1][i] = __bfloat16_as_ushort(mid);
        part[2][i] = __bfloat16_as_ushort(lo);
    }
    QFrag f;
#pragma unroll
    for (int p = 0; p < 3; ++p) {
        f.b[p][0] = (uint32_t)part[p][0] | ((uint32_t)part[p][1] << 16);
        f.b[p][1] = (uint32_t)part[p][2] | ((uint32_t)part[p][3] << 16);
    }
    return f;
}

// Scores of the 16-row group `grp` of a staged k_idx tile (32-byte rows):
// c[0], c[1] = rows g, heads 2t, 2t+1; c[2], c[3] = row g+8.  The three
// parts go to independent accumulators (short dependency chains) and are
// summed (hi + mid) + lo.
__device__ __forceinline__ void score16(uint32_t tile, int grp, int lane, const QFrag& q, float* c) {
    const uint32_t lrow = (uint32_t)(((lane >> 3) & 1) * 8 + (lane & 7)) * 32u + (uint32_t)((lane >> 4) * 16);
    uint32_t a0, a1, a2, a3;
    ldsm_x4(tile + (uint32_t)grp * 512u + lrow, a0, a1, a2, a3);
    float p[3][4];
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        p[k][0] = p[k][1] = p[k][2] = p[k][3] = 0.f;
        mma_bf16(p[k], a0, a1, a2, a3, q.b[k][0], q.b[k][1]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) c[e] = (p[0][e] + p[1][e]) + p[2][e];
}

}  // namespace rtp
