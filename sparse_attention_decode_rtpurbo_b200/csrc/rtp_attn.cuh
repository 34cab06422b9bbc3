// Split-KV block attention for the decode step: local heads (sink + sliding
// window) and retrieval heads (the kept 64-token blocks), with a last-CTA
// log-sum-exp combine of the splits.
//
// Sources: "Full Attention Strikes Back" (RTPurbo) review on
// dongryeollee1.github.io, Method: "Adaptive sparse attention" (local heads:
// sliding window + attention sink; retrieval heads: exact attention over the
// selected tokens in full feature space) and "Hardware-aware top-p decoding
// kernel" (block-sparse decoding); aitrends.kr summary item 2 (O_h(m), the
// softmax over S_h(m), value vectors restored) and item 5 / "Kernel 2 (D128)"
// (block-sparse attention with a cross-split reduce).
//
// Design on sm_100a: each CTA streams 64x128 bf16 K and V tiles (16 KB each,
// contiguous in both cache layouts) into a 3-stage shared-memory ring with
// the bulk-copy engine (cp.async.bulk + mbarrier transaction counts), and
// computes all G query heads of the KV group from each tile, so every tile
// crosses HBM once per step.  QK^T and PV are fp32 FMA on bf16 inputs: the
// decode tile is G (<= 8) query rows, 4-8 flop per byte.  Thread (tg, dc):
// tg = token group of 8 tokens, dc = 16-byte dim chunk, so each warp reads two
// whole 256-byte rows per load (bank-conflict free); the QK partial sums are
// reduce-scattered over the 16 dim-chunk lanes with butterfly shuffles.
#pragma once
#include "rtp_common.cuh"

namespace rtp {

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
    // index (into the original CNT values) of the value a lane holds in slot 0
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

template <int G>
struct AttnSmem {
    alignas(128) uint8_t stage[STAGES][STAGE_BYTES];   // K tile then V tile; reused for the final reduction
    alignas(16) float prob[BLK][G];                   // log2-domain logits, then probabilities
    float m_run[G], l_run[G], alpha[G];
    alignas(8) uint64_t full[STAGES];
    int blk_bad[STAGES];
    uint32_t flag;
    int ok;
};

// One CTA's running softmax state for G heads: acc[h][8] = this thread's
// 8 dims (dc) summed over its 8 tokens (tg) of every tile so far.
template <int G>
struct AttnCore {
    float acc[G][8];
    float q[G][8];

    __device__ __forceinline__ void load_q(const Params& P, int b, int g, int dc) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const uint4 u = *reinterpret_cast<const uint4*>(P.q_rope + ((int64_t)b * P.Hq + g * G + h) * D + dc * 8);
            const uint32_t* w = reinterpret_cast<const uint32_t*>(&u);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                q[h][2 * j] = bf_lo(w[j]);
                q[h][2 * j + 1] = bf_hi(w[j]);
            }
        }
    }
    __device__ __forceinline__ void reset(AttnSmem<G>& S, int tid) {
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[h][j] = 0.f;
        if (tid < G) {
            S.m_run[tid] = -INFINITY;
            S.l_run[tid] = 0.f;
        }
    }

    // Process one 64-token tile.  `hmask`: group-local heads allowed to read
    // this tile.  Token n0 + t is readable iff t < nvalid and (for local
    // heads) inside the sink/window set [0,s_end) U [w_lo, L).
    __device__ __forceinline__ void tile(AttnSmem<G>& S, const uint8_t* kv, uint32_t hmask, int n0, int nvalid,
                                         bool local, int s_end, int w_lo, int tid) {
        const int lane = tid & 31, tg = tid >> 4, dc = tid & 15;
        const uint4* K = reinterpret_cast<const uint4*>(kv);
        const uint4* V = reinterpret_cast<const uint4*>(kv + TILE_BYTES);
        constexpr int CNT = 8 * G;
        constexpr int NV = CNT >= 16 ? CNT / 16 : 1;
        float v[CNT];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const uint4 u = K[(tg * 8 + t) * 16 + dc];
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
        __syncthreads();
        // online softmax per head (warp w handles heads w, w+4)
        const int warp = tid >> 5;
        for (int h = warp; h < G; h += ATT_THREADS / 32) {
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
        __syncthreads();
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
            if (!ok) continue;   // unreadable rows may hold anything (NaN): never touch them
            const uint4 u = V[tok * 16 + dc];
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
        __syncthreads();
    }

    // Sum acc over the 8 token groups and write the partial (m, l, acc[128]) of
    // every head in `heads` to part[h * PSTRIDE].
    __device__ __forceinline__ void flush(AttnSmem<G>& S, float* part, uint32_t heads, int tid) {
        float* red = reinterpret_cast<float*>(&S.stage[0][0]);   // [8 tg][G][128]
        const int tg = tid >> 4, dc = tid & 15;
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int j = 0; j < 8; ++j) red[(tg * G + h) * D + dc * 8 + j] = acc[h][j];
        __syncthreads();
        for (int h = 0; h < G; ++h) {
            if (!((heads >> h) & 1u)) continue;
            float s = 0.f;
#pragma unroll
            for (int t = 0; t < 8; ++t) s += red[(t * G + h) * D + tid];
            part[h * PSTRIDE + 4 + tid] = s;
            if (tid == 0) {
                part[h * PSTRIDE + 0] = S.m_run[h];
                part[h * PSTRIDE + 1] = S.l_run[h];
            }
        }
        __syncthreads();
    }
};

// Combine the partials of `nparts` splits (stride G*PSTRIDE floats) for the
// heads in `heads` and write out[b, g*G + h] as bf16.  `scratch` is free
// shared memory of at least G*nparts floats (the tile ring).  Pass 1 finds
// each head's max and the split weights 2^(m_i - m*) (threads over
// (head, split) pairs); pass 2 has each thread own 4 dims of one head and
// stream the splits' float4 partials with independent loads.
template <int G>
__device__ void combine_parts(const Params& P, const float* parts, int nparts, uint32_t heads, int b, int g, int tid,
                              float* scratch) {
    __shared__ float s_den[G];
    for (int x = tid; x < G * nparts; x += ATT_THREADS) {
        const int h = x % G, i = x / G;
        const float* pp = parts + ((int64_t)i * G + h) * PSTRIDE;
        const float l = __ldcg(pp + 1), m = __ldcg(pp);
        scratch[h * nparts + i] = (l > 0.f) ? m : -INFINITY;
    }
    __syncthreads();
    // per-head max over the splits (one warp per head)
    const int warp = tid >> 5, lane = tid & 31;
    for (int h = warp; h < G; h += ATT_THREADS / 32) {
        float m = -INFINITY;
        for (int i = lane; i < nparts; i += 32) m = fmaxf(m, scratch[h * nparts + i]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float den = 0.f;
        for (int i = lane; i < nparts; i += 32) {
            const float mi = scratch[h * nparts + i];
            const float w = (mi == -INFINITY) ? 0.f : exp2f(mi - m);
            scratch[h * nparts + i] = w;
            if (w > 0.f) den += w * __ldcg(parts + ((int64_t)i * G + h) * PSTRIDE + 1);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
        if (lane == 0) s_den[h] = den;
    }
    __syncthreads();
    for (int x = tid; x < G * 32; x += ATT_THREADS) {
        const int h = x / 32, q = x % 32;
        if (!((heads >> h) & 1u)) continue;
        const float den = s_den[h];
        if (!(den > 0.f)) continue;
        float4 acc0 = make_float4(0.f, 0.f, 0.f, 0.f), acc1 = acc0;
        int i = 0;
        for (; i + 1 < nparts; i += 2) {
            const float w0 = scratch[h * nparts + i], w1 = scratch[h * nparts + i + 1];
            const float4 a0 = __ldcg(reinterpret_cast<const float4*>(parts + ((int64_t)i * G + h) * PSTRIDE + 4) + q);
            const float4 a1 =
                __ldcg(reinterpret_cast<const float4*>(parts + ((int64_t)(i + 1) * G + h) * PSTRIDE + 4) + q);
            acc0.x = fmaf(w0, a0.x, acc0.x);
            acc0.y = fmaf(w0, a0.y, acc0.y);
            acc0.z = fmaf(w0, a0.z, acc0.z);
            acc0.w = fmaf(w0, a0.w, acc0.w);
            acc1.x = fmaf(w1, a1.x, acc1.x);
            acc1.y = fmaf(w1, a1.y, acc1.y);
            acc1.z = fmaf(w1, a1.z, acc1.z);
            acc1.w = fmaf(w1, a1.w, acc1.w);
        }
        if (i < nparts) {
            const float w0 = scratch[h * nparts + i];
            const float4 a0 = __ldcg(reinterpret_cast<const float4*>(parts + ((int64_t)i * G + h) * PSTRIDE + 4) + q);
            acc0.x = fmaf(w0, a0.x, acc0.x);
            acc0.y = fmaf(w0, a0.y, acc0.y);
            acc0.z = fmaf(w0, a0.z, acc0.z);
            acc0.w = fmaf(w0, a0.w, acc0.w);
        }
        const float inv = 1.f / den;
        const float o0 = (acc0.x + acc1.x) * inv, o1 = (acc0.y + acc1.y) * inv, o2 = (acc0.z + acc1.z) * inv,
                    o3 = (acc0.w + acc1.w) * inv;
        uint16_t* dst = P.out + ((int64_t)b * P.Hq + g * G + h) * D + q * 4;
        const uint32_t lo = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(o0)) |
                            ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(o1)) << 16);
        const uint32_t hi = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(o2)) |
                            ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(o3)) << 16);
        *reinterpret_cast<uint2*>(dst) = make_uint2(lo, hi);
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// Tile producer/consumer loop shared by both attention kernels.  BlockAt(i)
// returns the element offset of tile i's first row in the K/V caches, its
// first token position, the number of readable rows and the head mask.
// ---------------------------------------------------------------------------
struct TileRef {
    int64_t off;
    int n0, nvalid;
    uint32_t hmask;
    bool bad;
};

template <int G, typename BlockAt>
__device__ __forceinline__ bool run_tiles(const Params& P, AttnSmem<G>& S, AttnCore<G>& core, int ntiles,
                                          BlockAt block_at, bool local, int s_end, int w_lo, int tid,
                                          uint32_t& phase_bits) {
    // prologue (the stages may hold generic-proxy writes of an earlier flush)
    if (tid == 0) {
        fence_proxy_async();
        for (int i = 0; i < STAGES && i < ntiles; ++i) {
            const TileRef r = block_at(i);
            S.blk_bad[i] = r.bad;
            mbar_expect_tx(&S.full[i], STAGE_BYTES);
            bulk_g2s(&S.stage[i][0], P.k_cache + r.off, TILE_BYTES, &S.full[i]);
            bulk_g2s(&S.stage[i][TILE_BYTES], P.v_cache + r.off, TILE_BYTES, &S.full[i]);
        }
    }
    for (int i = 0; i < ntiles; ++i) {
        const int st = i % STAGES;
        const uint32_t par = (phase_bits >> st) & 1u;
        if (tid == 0) S.ok = mbar_wait_bounded(&S.full[st], par) ? 1 : 0;
        __syncthreads();
        if (!S.ok) {
            // a copy never landed: record it, drain what is still in flight, give up
            if (tid == 0) {
                set_status(P, ST_TIMEOUT);
                for (int k = i + 1; k < ntiles && k < i + STAGES; ++k) {
                    const int s2 = k % STAGES;
                    mbar_wait_bounded(&S.full[s2], (phase_bits >> s2) & 1u);
                }
            }
            __syncthreads();
            return false;
        }
        if (tid != 0) mbar_try_wait(&S.full[st], par);
        phase_bits ^= 1u << st;
        const TileRef r = block_at(i);
        if (r.bad) {
            if (tid == 0) set_status(P, ST_DEVICE_INPUT);
        } else {
            core.tile(S, &S.stage[st][0], r.hmask, r.n0, r.nvalid, local, s_end, w_lo, tid);
        }
        __syncthreads();
        if (tid == 0 && i + STAGES < ntiles) {
            fence_proxy_async();
            const TileRef r2 = block_at(i + STAGES);
            mbar_expect_tx(&S.full[st], STAGE_BYTES);
            bulk_g2s(&S.stage[st][0], P.k_cache + r2.off, TILE_BYTES, &S.full[st]);
            bulk_g2s(&S.stage[st][TILE_BYTES], P.v_cache + r2.off, TILE_BYTES, &S.full[st]);
        }
    }
    return true;
}

template <int G>
__device__ __forceinline__ void init_barriers(AttnSmem<G>& S, int tid) {
    if (tid == 0) {
        for (int i = 0; i < STAGES; ++i) mbar_init(&S.full[i], 1);
        mbar_fence_init();
    }
    __syncthreads();
}

// Element offset of the first row of block j of KV head g of sequence b.
__device__ __forceinline__ int64_t tile_off(const Params& P, int b, int g, int j, bool* bad) {
    if (P.block_table == nullptr) return (((int64_t)b * P.Hkv + g) * P.Ncap + (int64_t)j * BLK) * D;
    int pg = page_of(P, b, j);
    if (pg < 0) {
        *bad = true;
        pg = 0;
    }
    return ((int64_t)pg * P.Hkv + g) * BLK * D;
}

// ---------------------------------------------------------------------------
// Kernel: local heads.  grid (local_items, n_lg, B).  Item i of (b, group)
// covers entries [i*KB, (i+1)*KB) of the group's block list
// [sink blocks] ++ [window blocks].
// ---------------------------------------------------------------------------
template <int G>
__global__ void __launch_bounds__(ATT_THREADS) local_attn_kernel(const __grid_constant__ Params P) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    AttnSmem<G>& S = *reinterpret_cast<AttnSmem<G>*>(smem_raw);
    const int b = blockIdx.z, lgi = blockIdx.y, item = blockIdx.x, tid = threadIdx.x;
    const int L = __ldg(P.seq_lens + b);
    if (!seq_ok(P, L)) return;
    const int g = P.lg_group[lgi];
    const uint32_t heads = P.lg_mask[lgi];
    const int s_end = min(P.sink, L);
    const int w_lo = P.window > 0 ? max(0, L - P.window) : L;
    const int nA = (s_end + BLK - 1) / BLK;
    const int bw0 = max(w_lo / BLK, nA);
    const int nB = P.window > 0 ? max(0, (L + BLK - 1) / BLK - bw0) : 0;
    const int nv = nA + nB;
    const int KB = P.local_kb;
    const int nitems = (nv + KB - 1) / KB;
    if (item >= nitems) return;
    const int v0 = item * KB, ntiles = min(KB, nv - v0);

    init_barriers(S, tid);
    AttnCore<G> core;
    core.load_q(P, b, g, tid & 15);
    core.reset(S, tid);
    __syncthreads();
    auto block_at = [&](int i) -> TileRef {
        const int v = v0 + i;
        const int j = v < nA ? v : bw0 + (v - nA);
        TileRef r;
        r.bad = false;
        r.off = tile_off(P, b, g, j, &r.bad);
        r.n0 = j * BLK;
        r.nvalid = min(BLK, L - j * BLK);
        r.hmask = heads;
        return r;
    };
    uint32_t phase_bits = 0;
    const bool ok = run_tiles<G>(P, S, core, ntiles, block_at, true, s_end, w_lo, tid, phase_bits);
    float* parts = P.lpart + (((int64_t)b * P.n_lg + lgi) * P.local_items) * G * PSTRIDE;
    if (ok) core.flush(S, parts + (int64_t)item * G * PSTRIDE, heads, tid);
    __syncthreads();
    if (!last_arrival(P.tick_local + b * P.n_lg + lgi, nitems, &S.flag)) return;
    __threadfence();
    combine_parts<G>(P, parts, nitems, heads, b, g, tid, reinterpret_cast<float*>(&S.stage[0][0]));
}

// ---------------------------------------------------------------------------
// Kernel: retrieval heads.  Persistent grid; the concatenated block lists of
// all (b, retrieval group) are cut into items of KB blocks, KB chosen so the
// items about fill the grid.
// ---------------------------------------------------------------------------
template <int G>
__global__ void __launch_bounds__(ATT_THREADS) ret_attn_kernel(const __grid_constant__ Params P) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    AttnSmem<G>& S = *reinterpret_cast<AttnSmem<G>*>(smem_raw);
    const int tid = threadIdx.x;
    const int nbg = P.B * P.n_rg;
    // total kept blocks -> blocks per item
    long long total = 0;
    for (int i = 0; i < nbg; ++i) {
        const int b = i / P.n_rg;
        const int L = __ldg(P.seq_lens + b);
        if (seq_ok(P, L)) total += __ldcg(P.bcount + i);
    }
    const int KB = (int)max(1ll, (total + gridDim.x - 1) / gridDim.x);
    init_barriers(S, tid);
    uint32_t phase_bits = 0;
    // walk (b, group) segments; item ids are global, contiguous per segment
    int item_base = 0;
    for (int bg = 0; bg < nbg; ++bg) {
        const int b = bg / P.n_rg, rgi = bg % P.n_rg;
        const int L = __ldg(P.seq_lens + b);
        const int cnt = seq_ok(P, L) ? (int)__ldcg(P.bcount + bg) : 0;
        const int nitems = (cnt + KB - 1) / KB;
        const int g = P.rg_group[rgi];
        const uint32_t heads = P.rg_mask[rgi];
        const uint32_t* list = P.blist + (int64_t)bg * P.nblk_cap;
        for (int it = 0; it < nitems; ++it) {
            const int item = item_base + it;
            if (item % (int)gridDim.x != (int)blockIdx.x) continue;
            const int k0 = it * KB, ntiles = min(KB, cnt - k0);
            AttnCore<G> core;
            core.load_q(P, b, g, tid & 15);
            core.reset(S, tid);
            __syncthreads();
            auto block_at = [&](int i) -> TileRef {
                const uint32_t e = __ldcg(list + k0 + i);
                const int j = (int)(e >> 8);
                TileRef r;
                r.bad = false;
                r.off = tile_off(P, b, g, j, &r.bad);
                r.n0 = j * BLK;
                r.nvalid = min(BLK, L - j * BLK);
                r.hmask = e & 0xFFu;
                return r;
            };
            const bool ok = run_tiles<G>(P, S, core, ntiles, block_at, false, 0, 0, tid, phase_bits);
            float* parts = P.rpart + (int64_t)item_base * G * PSTRIDE;
            if (ok) core.flush(S, parts + (int64_t)it * G * PSTRIDE, heads, tid);
            __syncthreads();
            if (last_arrival(P.tick_ret + bg, nitems, &S.flag)) {
                __threadfence();
                combine_parts<G>(P, parts, nitems, heads, b, g, tid, reinterpret_cast<float*>(&S.stage[0][0]));
                __syncthreads();
            }
        }
        item_base += nitems;
    }
}

}  // namespace rtp
