// Retrieval-head selection: index scoring, exact dynamic top-p, block marking
// and the per-KV-group block list.
//
// Sources: "Full Attention Strikes Back" (RTPurbo) review on
// dongryeollee1.github.io, Method: "Adaptive sparse attention" (s_h(m,n) and
// S_h(m) = Top-P(s_h(m,.), p)) and "Hardware-aware top-p decoding kernel"
// (scores accumulated into a 256-bin histogram of softmax mass, the last CTA
// scanning it for the bin where the cumulative mass reaches p_top, then a
// block mask); aitrends.kr summary item 5 and "Kernel 1 (D16)".
//
// Design on sm_100a: the 32 B/token index-key stream is read once with
// 32-byte streaming loads (one row per load); scores go to an L2-resident key array; the last
// CTA of each KV group merges per-chunk max/argmax/sum partials.  When the
// single best token already carries mass >= p the selection is decided there
// (no further pass); otherwise an exact MSD radix select over the 32-bit
// order-preserving score keys runs (4 passes of 256 bins holding a count and
// a 2^-40 fixed-point mass each, so sums are exact and order-independent),
// followed by a lowest-index tie split.
#pragma once
#include "rtp_common.cuh"

namespace rtp {

// ---------------------------------------------------------------------------
// block-wide reductions (SEL_THREADS = 256 threads, 8 warps)
// ---------------------------------------------------------------------------
template <typename T, typename Op>
__device__ __forceinline__ T warp_reduce(T v, Op op) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// ---------------------------------------------------------------------------
// Kernel: index scores of one CHUNK of tokens for every retrieval head of one
// KV group; per-chunk partials; the group's last CTA decides the selection mode.
// grid (nchunks, n_rg, B), SEL_THREADS threads
// ---------------------------------------------------------------------------
template <int G>
__global__ void __launch_bounds__(SEL_THREADS) score_kernel(const __grid_constant__ Params P) {
    const int b = blockIdx.z, rgi = blockIdx.y, chunk = blockIdx.x, tid = threadIdx.x;
    const int L = __ldg(P.seq_lens + b);
    if (!seq_ok(P, L)) {
        if (chunk == 0 && rgi == 0 && tid == 0) set_status(P, ST_DEVICE_INPUT);
        return;
    }
    const int nch = (L + CHUNK - 1) / CHUNK;
    if (chunk >= nch) return;
    const int g = P.rg_group[rgi], nh = P.rg_nh[rgi], slot0 = P.rg_slot0[rgi];

    __shared__ __align__(16) float qi[G][R];
    __shared__ uint32_t s_key[G][8], s_arg[G][8], s_min[G][8];
    __shared__ float s_m[G][8];
    __shared__ double s_sum[G][8];
    __shared__ uint32_t t_key[8], t_arg[8], t_min[8], t_best[3];
    __shared__ double t_sum[8];
    __shared__ uint32_t s_flag;

    // q_idx = Wq_idx[h] . q_pre[b,h] (fp32, one warp per (head, row))
    {
        const int warp = tid >> 5, lane = tid & 31;
        for (int pr = warp; pr < nh * R; pr += SEL_THREADS / 32) {
            const int hh = pr / R, r = pr % R;
            const int h = P.slot_head[slot0 + hh];
            const uint2 w = *reinterpret_cast<const uint2*>(P.Wq + ((int64_t)h * R + r) * D + lane * 4);
            const uint2 q = *reinterpret_cast<const uint2*>(P.q_pre + ((int64_t)b * P.Hq + h) * D + lane * 4);
            float a = bf_lo(w.x) * bf_lo(q.x);
            a = fmaf(bf_hi(w.x), bf_hi(q.x), a);
            a = fmaf(bf_lo(w.y), bf_lo(q.y), a);
            a = fmaf(bf_hi(w.y), bf_hi(q.y), a);
            a = warp_reduce(a, [](float x, float y) { return x + y; });
            if (lane == 0) qi[hh][r] = a;
        }
    }
    __syncthreads();

    uint32_t mk[G], am[G], nk[G];
    float ms[G], sm[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
        mk[hh] = 0u;
        am[hh] = 0xFFFFFFFFu;
        nk[hh] = 0xFFFFFFFFu;
        ms[hh] = -INFINITY;
        sm[hh] = 0.f;
    }

    const int n_begin = chunk * CHUNK;
    const int n_end = min(L, n_begin + CHUNK);
    bool bad = false;
    constexpr int PER = CHUNK / SEL_THREADS;   // 8 tokens per thread
    U8x32 raw[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int n = n_begin + i * SEL_THREADS + tid;
        if (n < n_end) {
            const uint16_t* src = P.k_idx + row_off(P, b, g, n, R, &bad);
            raw[i] = ld_stream32(src);
        }
    }
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int n = n_begin + i * SEL_THREADS + tid;
        if (n >= n_end) continue;
        float k[R];
        const uint32_t* u = raw[i].w;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            k[2 * j] = bf_lo(u[j]);
            k[2 * j + 1] = bf_hi(u[j]);
        }
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
            if (hh >= nh) break;
            float s = 0.f;
#pragma unroll
            for (int r = 0; r < R; ++r) s = fmaf(qi[hh][r], k[r], s);
            const uint32_t key = f2key(s);
            P.keys[((int64_t)b * P.n_ret + slot0 + hh) * P.Ncap + n] = key;
            if (key > mk[hh]) {
                mk[hh] = key;
                am[hh] = (uint32_t)n;
            }
            nk[hh] = min(nk[hh], key);
            if (s > ms[hh]) {
                sm[hh] = sm[hh] * expf((ms[hh] - s) * 0.25f) + 1.f;
                ms[hh] = s;
            } else {
                sm[hh] += expf((s - ms[hh]) * 0.25f);
            }
        }
    }
    if (bad) set_status(P, ST_DEVICE_INPUT);

    // block reduction of (max key, argmax at max, min key, sum relative to max)
    const int warp = tid >> 5, lane = tid & 31;
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
        if (hh >= nh) break;
        uint32_t k = mk[hh], a = am[hh], mn = nk[hh];
        float m = ms[hh];
        double su = (double)sm[hh];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const uint32_t k2 = __shfl_xor_sync(0xffffffffu, k, o);
            const uint32_t a2 = __shfl_xor_sync(0xffffffffu, a, o);
            const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
            const double s2 = __shfl_xor_sync(0xffffffffu, su, o);
            mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            if (k2 > k || (k2 == k && a2 < a)) {
                k = k2;
                a = a2;
            }
            const float mm = fmaxf(m, m2);
            su = (mm == -INFINITY) ? 0.0 : su * exp((double)(m - mm) * 0.25) + s2 * exp((double)(m2 - mm) * 0.25);
            m = mm;
        }
        if (lane == 0) {
            s_key[hh][warp] = k;
            s_arg[hh][warp] = a;
            s_min[hh][warp] = mn;
            s_m[hh][warp] = m;
            s_sum[hh][warp] = su;
        }
    }
    __syncthreads();
    if (tid < nh) {
        const int hh = tid;
        uint32_t k = 0, a = 0xFFFFFFFFu, mn = 0xFFFFFFFFu;
        float m = -INFINITY;
        for (int w = 0; w < SEL_THREADS / 32; ++w) {
            if (s_key[hh][w] > k || (s_key[hh][w] == k && s_arg[hh][w] < a)) {
                k = s_key[hh][w];
                a = s_arg[hh][w];
            }
            mn = min(mn, s_min[hh][w]);
            m = fmaxf(m, s_m[hh][w]);
        }
        double su = 0.0;
        for (int w = 0; w < SEL_THREADS / 32; ++w)
            if (s_m[hh][w] != -INFINITY) su += s_sum[hh][w] * exp((double)(s_m[hh][w] - m) * 0.25);
        ChunkStat cs;
        cs.maxkey = k;
        cs.argmax = a;
        cs.minkey = mn;
        cs.pad = 0;
        cs.sum = su;   // relative to m == key2f(k)
        P.cstat[((int64_t)b * P.n_ret + slot0 + hh) * P.nchunks + chunk] = cs;
    }
    __syncthreads();

    if (!last_arrival(P.tick_score + b * P.n_rg + rgi, nch, &s_flag)) return;
    __threadfence();

    // ---- last CTA of (b, group): merge chunk partials, choose the selection mode ----
    for (int hh = 0; hh < nh; ++hh) {
        const int slot = slot0 + hh;
        const ChunkStat* cs = P.cstat + ((int64_t)b * P.n_ret + slot) * P.nchunks;
        uint32_t k = 0, a = 0xFFFFFFFFu, mn = 0xFFFFFFFFu;
        for (int c = tid; c < nch; c += SEL_THREADS) {
            const ChunkStat x = cs[c];
            if (x.maxkey > k || (x.maxkey == k && x.argmax < a)) {
                k = x.maxkey;
                a = x.argmax;
            }
            mn = min(mn, x.minkey);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const uint32_t k2 = __shfl_xor_sync(0xffffffffu, k, o);
            const uint32_t a2 = __shfl_xor_sync(0xffffffffu, a, o);
            mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            if (k2 > k || (k2 == k && a2 < a)) {
                k = k2;
                a = a2;
            }
        }
        if (lane == 0) {
            t_key[warp] = k;
            t_arg[warp] = a;
            t_min[warp] = mn;
        }
        __syncthreads();
        if (tid == 0) {
            for (int w = 1; w < SEL_THREADS / 32; ++w) {
                if (t_key[w] > k || (t_key[w] == k && t_arg[w] < a)) {
                    k = t_key[w];
                    a = t_arg[w];
                }
                mn = min(mn, t_min[w]);
            }
            t_best[0] = k;
            t_best[1] = a;
            t_best[2] = mn;
        }
        __syncthreads();
        k = t_best[0];
        a = t_best[1];
        mn = t_best[2];
        const float smax = key2f(k);
        double su = 0.0;
        for (int c = tid; c < nch; c += SEL_THREADS) {
            const ChunkStat x = cs[c];
            su += x.sum * exp(((double)key2f(x.maxkey) - (double)smax) * 0.25);
        }
        su = warp_reduce(su, [](double x, double y) { return x + y; });
        if (lane == 0) t_sum[warp] = su;
        __syncthreads();
        if (tid == 0) {
            double z = 0.0;
            for (int w = 0; w < SEL_THREADS / 32; ++w) z += t_sum[w];
            const float pb = __ldg(P.p + b);
            HeadState st;
            st.smax = smax;
            st.maxkey = k;
            st.argmax = a;
            st.minkey = mn;
            st.pad0 = 0;
            st.zrel = z;
            st.target = 0;
            st.mass_above = 0;
            st.prefix = 0;
            st.count_above = 0;
            st.n_eq = 0;
            st.n_tie = 0;
            st.all_ties = 1;
            st.tau_key = 0;
            st.pad1 = 0;
            if (!(pb > 0.f)) {
                st.mode = MODE_SKIP;
                st.kstar = 0;
                set_status(P, ST_DEVICE_INPUT);
            } else if (pb >= 1.f) {
                st.mode = MODE_ALL;
                st.kstar = (uint32_t)L;
                st.tau_key = mn;
            } else if (1.0 >= (double)pb * z * (1.0 + 1e-6)) {
                st.mode = MODE_TOP1;   // the best token alone reaches p
                st.kstar = 1;
                st.tau_key = k;
            } else {
                st.mode = MODE_RADIX;
                st.kstar = 0;
            }
            P.hs[(int64_t)b * P.n_ret + slot] = st;
            const int bh = b * P.Hq + P.slot_head[slot];
            if (P.dbg_smax) P.dbg_smax[bh] = smax;
            if (P.dbg_Z) P.dbg_Z[bh] = z;
            if (st.mode != MODE_RADIX) {
                if (P.dbg_tau) P.dbg_tau[bh] = key2f(st.tau_key);
                if (P.dbg_kstar) P.dbg_kstar[bh] = (int32_t)st.kstar;
            }
        }
        // clear this head's radix histogram for the selection passes
        for (int d = tid; d < 256; d += SEL_THREADS) {
            P.hist_cnt[((int64_t)b * P.n_ret + slot) * 256 + d] = 0;
            P.hist_mass[((int64_t)b * P.n_ret + slot) * 256 + d] = 0ull;
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Kernel: one pass of the MSD radix select (8 bits per pass) for heads in
// MODE_RADIX.  grid (nchunks, n_ret, B)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(SEL_THREADS) radix_kernel(const __grid_constant__ Params P, int pass) {
    const int b = blockIdx.z, slot = blockIdx.y, chunk = blockIdx.x, tid = threadIdx.x;
    const int L = __ldg(P.seq_lens + b);
    if (!seq_ok(P, L)) return;
    const int64_t bs = (int64_t)b * P.n_ret + slot;
    HeadState* hsp = P.hs + bs;
    if (hsp->mode != MODE_RADIX) return;
    const int nch = (L + CHUNK - 1) / CHUNK;
    if (chunk >= nch) return;

    __shared__ uint32_t cnt[256];
    __shared__ unsigned long long mass[256];
    __shared__ uint32_t s_flag;
    __shared__ int s_dstar;
    for (int d = tid; d < 256; d += SEL_THREADS) {
        cnt[d] = 0;
        mass[d] = 0ull;
    }
    __syncthreads();
    const uint32_t prefix = hsp->prefix;
    const float smax = hsp->smax;
    const int shift = 24 - 8 * pass;
    const int n_begin = chunk * CHUNK, n_end = min(L, n_begin + CHUNK);
    const uint32_t* keys = P.keys + bs * P.Ncap;
    for (int n = n_begin + tid; n < n_end; n += SEL_THREADS) {
        const uint32_t key = keys[n];
        if (pass > 0 && (key >> (32 - 8 * pass)) != prefix) continue;
        const int d = (key >> shift) & 255;
        atomicAdd(&cnt[d], 1u);
        atomicAdd(&mass[d], fixmass(key, smax));
    }
    __syncthreads();
    uint32_t* gcnt = P.hist_cnt + bs * 256;
    unsigned long long* gmass = P.hist_mass + bs * 256;
    for (int d = tid; d < 256; d += SEL_THREADS) {
        if (cnt[d]) {
            atomicAdd(gcnt + d, cnt[d]);
            atomicAdd(gmass + d, mass[d]);
        }
        if (pass == 3) P.chunk_cnt[(bs * P.nchunks + chunk) * 256 + d] = cnt[d];
    }
    __syncthreads();
    if (!last_arrival(P.tick_radix + bs, nch, &s_flag)) return;
    __threadfence();

    // ---- last CTA: locate the bin where the cumulative mass reaches the target ----
    for (int d = tid; d < 256; d += SEL_THREADS) {
        cnt[d] = __ldcg(gcnt + d);
        mass[d] = __ldcg(gmass + d);
        gcnt[d] = 0;
        gmass[d] = 0ull;
    }
    __syncthreads();
    if (tid == 0) {
        HeadState st = *hsp;
        if (pass == 0) {
            unsigned long long z = 0;
            for (int d = 0; d < 256; ++d) z += mass[d];
            const double pb = (double)__ldg(P.p + b);
            unsigned long long t = (unsigned long long)ceil(pb * (double)z);
            if (t > z) t = z;
            if (t == 0) t = 1;
            st.target = t;
            st.mass_above = 0;
            st.count_above = 0;
            st.prefix = 0;
        }
        unsigned long long cum = st.mass_above;
        uint32_t cabove = st.count_above;
        int dstar = 0;
        for (int d = 255; d >= 0; --d) {
            if (cum + mass[d] >= st.target) {
                dstar = d;
                break;
            }
            cum += mass[d];
            cabove += cnt[d];
        }
        st.mass_above = cum;
        st.count_above = cabove;
        st.prefix = (st.prefix << 8) | (uint32_t)dstar;
        if (pass == 3) {
            st.tau_key = st.prefix;
            st.n_eq = cnt[dstar];
            const unsigned long long m_tau = st.n_eq ? mass[dstar] / st.n_eq : 0ull;
            const unsigned long long need = st.target - st.mass_above;
            uint32_t nt = st.n_eq;
            if (m_tau > 0) {
                const unsigned long long q = (need + m_tau - 1) / m_tau;
                nt = (uint32_t)min((unsigned long long)st.n_eq, max(1ull, q));
            }
            st.n_tie = nt;
            st.all_ties = (nt == st.n_eq) ? 1u : 0u;
            st.kstar = st.count_above + nt;
            const int bh = b * P.Hq + P.slot_head[slot];
            if (P.dbg_tau) P.dbg_tau[bh] = key2f(st.tau_key);
            if (P.dbg_kstar) P.dbg_kstar[bh] = (int32_t)st.kstar;
        }
        *hsp = st;
        s_dstar = dstar;
    }
    __syncthreads();
    if (pass == 3 && !hsp->all_ties && tid == 0) {
        // exclusive prefix over chunks of the tie count: rank of each chunk's first tie
        const int dstar = s_dstar;
        uint32_t run = 0;
        for (int c = 0; c < nch; ++c) {
            P.tie_off[bs * P.nchunks + c] = run;
            run += P.chunk_cnt[(bs * P.nchunks + c) * 256 + dstar];
        }
    }
}

// ---------------------------------------------------------------------------
// Kernel: block mask words of one chunk (32 blocks) for every retrieval head.
// grid (nchunks, n_ret, B)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(SEL_THREADS) mark_kernel(const __grid_constant__ Params P) {
    const int b = blockIdx.z, slot = blockIdx.y, chunk = blockIdx.x, tid = threadIdx.x;
    const int L = __ldg(P.seq_lens + b);
    if (!seq_ok(P, L)) return;
    const int nch = (L + CHUNK - 1) / CHUNK;
    if (chunk >= nch) return;
    const int64_t bs = (int64_t)b * P.n_ret + slot;
    const HeadState st = P.hs[bs];
    const int n_begin = chunk * CHUNK, n_end = min(L, n_begin + CHUNK);
    const int nblk = (L + BLK - 1) / BLK;
    uint32_t* word = P.bitmap + bs * P.words_cap + chunk;   // CHUNK = 32 blocks = one word

    if (st.mode != MODE_RADIX) {
        if (tid == 0) {
            uint32_t w = 0;
            if (st.mode == MODE_TOP1) {
                const int j = (int)(st.argmax / BLK) - chunk * 32;
                if (j >= 0 && j < 32) w = 1u << j;
            } else if (st.mode == MODE_ALL) {
                const int nb = min(32, nblk - chunk * 32);
                w = nb >= 32 ? 0xFFFFFFFFu : ((1u << nb) - 1u);
            }
            *word = w;
        }
        return;
    }

    __shared__ uint32_t s_word, s_warp[SEL_THREADS / 32], s_carry;
    if (tid == 0) {
        s_word = 0;
        s_carry = 0;
    }
    __syncthreads();
    const uint32_t* keys = P.keys + bs * P.Ncap;
    const uint32_t tau = st.tau_key;
    const uint32_t tie_base = st.all_ties ? 0u : P.tie_off[bs * P.nchunks + chunk];
    const int warp = tid >> 5, lane = tid & 31;
    uint32_t mine = 0;
    for (int base = n_begin; base < n_end; base += SEL_THREADS) {
        const int n = base + tid;
        const uint32_t key = (n < n_end) ? keys[n] : 0u;
        bool keep = (n < n_end) && key > tau;
        const bool tie = (n < n_end) && key == tau;
        if (st.all_ties) {
            keep = keep || tie;
        } else {
            const uint32_t bal = __ballot_sync(0xffffffffu, tie);
            if (lane == 0) s_warp[warp] = __popc(bal);
            __syncthreads();
            uint32_t before = s_carry;
            for (int w = 0; w < warp; ++w) before += s_warp[w];
            before += __popc(bal & ((1u << lane) - 1u));
            keep = keep || (tie && tie_base + before < st.n_tie);
            __syncthreads();
            if (tid == 0) {
                uint32_t tot = 0;
                for (int w = 0; w < SEL_THREADS / 32; ++w) tot += s_warp[w];
                s_carry += tot;
            }
            __syncthreads();
        }
        if (keep) mine |= 1u << ((n - n_begin) / BLK);
    }
    mine = warp_reduce(mine, [](uint32_t x, uint32_t y) { return x | y; });
    if (lane == 0 && mine) atomicOr(&s_word, mine);
    __syncthreads();
    if (tid == 0) *word = s_word;
}

// ---------------------------------------------------------------------------
// Kernel: union over a KV group's retrieval heads of their block masks ->
// compact block list (entry = block << 8 | mask of group-local head indices).
// grid (n_rg, B), 1024 threads
// ---------------------------------------------------------------------------
constexpr int BL_THREADS = 1024;
__global__ void __launch_bounds__(BL_THREADS) blocklist_kernel(const __grid_constant__ Params P) {
    const int b = blockIdx.y, rgi = blockIdx.x, tid = threadIdx.x;
    const int L = __ldg(P.seq_lens + b);
    if (!seq_ok(P, L)) return;
    const int g = P.rg_group[rgi], nh = P.rg_nh[rgi], slot0 = P.rg_slot0[rgi];
    const int nblk = (L + BLK - 1) / BLK;
    const int nwords = (nblk + 31) / 32;
    __shared__ uint32_t s_warp[BL_THREADS / 32];
    __shared__ uint32_t s_base;
    __shared__ int s_kept[MAX_G];
    if (tid == 0) s_base = 0;
    if (tid < MAX_G) s_kept[tid] = 0;
    __syncthreads();
    uint32_t* list = P.blist + ((int64_t)b * P.n_rg + rgi) * P.nblk_cap;
    const int warp = tid >> 5, lane = tid & 31;
    for (int w0 = 0; w0 < nwords; w0 += BL_THREADS) {
        const int w = w0 + tid;
        uint32_t uni = 0;
        uint32_t wh[MAX_G];
#pragma unroll
        for (int hh = 0; hh < MAX_G; ++hh) {
            wh[hh] = 0;
            if (hh < nh && w < nwords) {
                wh[hh] = P.bitmap[((int64_t)b * P.n_ret + slot0 + hh) * P.words_cap + w];
                if (w == nwords - 1 && (nblk & 31)) wh[hh] &= (1u << (nblk & 31)) - 1u;
                uni |= wh[hh];
                if (wh[hh]) atomicAdd(&s_kept[hh], __popc(wh[hh]));
                if (P.dbg_bitmap)
                    P.dbg_bitmap[((int64_t)b * P.Hq + P.slot_head[slot0 + hh]) * P.words_cap + w] = wh[hh];
            }
        }
        const uint32_t c = __popc(uni);
        // block-wide exclusive scan of c
        uint32_t incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        if (lane == 31) s_warp[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            uint32_t v = s_warp[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t t = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += t;
            }
            s_warp[lane] = v;   // inclusive over warps
        }
        __syncthreads();
        uint32_t pos = s_base + (warp ? s_warp[warp - 1] : 0u) + incl - c;
        while (uni) {
            const int j = __ffs(uni) - 1;
            uni &= uni - 1;
            uint32_t hm = 0;
#pragma unroll
            for (int hh = 0; hh < MAX_G; ++hh)
                if ((wh[hh] >> j) & 1u) hm |= 1u << (P.slot_head[slot0 + hh] - g * P.G);
            list[pos++] = ((uint32_t)(w * 32 + j) << 8) | hm;
        }
        __syncthreads();
        if (tid == 0) s_base += s_warp[BL_THREADS / 32 - 1];
        __syncthreads();
    }
    if (tid == 0) P.bcount[b * P.n_rg + rgi] = s_base;
    if (tid < nh && P.dbg_kept) P.dbg_kept[b * P.Hq + P.slot_head[slot0 + tid]] = s_kept[tid];
}

}  // namespace rtp
