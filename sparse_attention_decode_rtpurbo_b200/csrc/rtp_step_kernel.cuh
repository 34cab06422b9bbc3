// Item handlers and the persistent kernel of the decode step (see rtp_step.cuh).
#pragma once
#include "rtp_step.cuh"

namespace rtp {

struct StepParams {
    Params P;
    Sync* sync;
    uint32_t* rlist;    // [B*n_ret] (b << 16 | slot) of heads needing the radix select
    uint32_t* rglist;   // [B*n_rg]  (b << 16 | rg) of groups holding such heads
    int n_score_items, n_local_items;
};

// ===========================================================================
// index scores (consumers)
// ===========================================================================
// Index scoring on the tensor cores: per 16 staged rows, one m16n8k16 bf16
// MMA against each of three bf16 parts of q_idx (hi + mid + lo = q_idx to
// fp32 precision; every bf16 x bf16 product is exact and the sums are fp32),
// N = 8 columns = the group's retrieval heads.  Thread (g = lane/4, t =
// lane%4) owns heads 2t, 2t+1 of rows g and g+8 of each 16-row group.
template <int G>
struct ScoreState {
    uint32_t b[3][2];                 // B fragments of q_idx hi / mid / lo
    uint32_t mk[2], am[2], nk[2];     // per owned head: max key, its lowest index, min key
    float ms[2], sm[2];               // max score, sum of exp((s - ms)/4)
};

template <int G>
__device__ __forceinline__ void score_begin(const Params& P, StepSmem<G>& S, ScoreState<G>& st, int b, int rgi, int tid) {
    const int nh = P.rg_nh[rgi], slot0 = P.rg_slot0[rgi];
    const int tag = b * MAX_HKV + rgi + 1;
    if (S.qi_tag != tag) {
        // q_idx = Wq_idx[h] . q_pre[b,h] (fp32) for the group's retrieval heads,
        // all (head, row) dots at once: TPP threads per dot, one round of loads
        const int npair = nh * R;                    // <= 128
        const int tpp = CONSUMERS / npair >= 8 ? 8 : (CONSUMERS / npair >= 4 ? 4 : (CONSUMERS / npair >= 2 ? 2 : 1));
        const int pr = tid / tpp, part = tid % tpp;
        float a = 0.f;
        if (pr < npair) {
            const int hh = pr / R, r = pr % R;
            const int h = P.slot_head[slot0 + hh];
            const int span = D / tpp;                // dims per thread: 16..128
            const uint4* w = reinterpret_cast<const uint4*>(P.Wq + ((int64_t)h * R + r) * D + part * span);
            const uint4* q = reinterpret_cast<const uint4*>(P.q_pre + ((int64_t)b * P.Hq + h) * D + part * span);
            for (int i = 0; i < span / 8; ++i) {
                const uint4 wv = w[i], qv = q[i];
                a = fmaf(bf_lo(wv.x), bf_lo(qv.x), a);
                a = fmaf(bf_hi(wv.x), bf_hi(qv.x), a);
                a = fmaf(bf_lo(wv.y), bf_lo(qv.y), a);
                a = fmaf(bf_hi(wv.y), bf_hi(qv.y), a);
                a = fmaf(bf_lo(wv.z), bf_lo(qv.z), a);
                a = fmaf(bf_hi(wv.z), bf_hi(qv.z), a);
                a = fmaf(bf_lo(wv.w), bf_lo(qv.w), a);
                a = fmaf(bf_hi(wv.w), bf_hi(qv.w), a);
            }
        }
        for (int o = 1; o < tpp; o <<= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (pr < npair && part == 0) S.qi[pr / R][pr % R] = a;
        consumer_sync();
        if (tid == 0) S.qi_tag = tag;
    }
    // B fragment of column g (head g): k = 2t, 2t+1 and 2t+8, 2t+9
    {
        const int lane = tid & 31, g = lane >> 2, t = lane & 3;
        float qv[4] = {0.f, 0.f, 0.f, 0.f};
        if (g < nh) {
            qv[0] = S.qi[g][2 * t];
            qv[1] = S.qi[g][2 * t + 1];
            qv[2] = S.qi[g][2 * t + 8];
            qv[3] = S.qi[g][2 * t + 9];
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
#pragma unroll
        for (int p = 0; p < 3; ++p) {
            st.b[p][0] = (uint32_t)part[p][0] | ((uint32_t)part[p][1] << 16);
            st.b[p][1] = (uint32_t)part[p][2] | ((uint32_t)part[p][3] << 16);
        }
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        st.mk[j] = 0u;
        st.am[j] = 0xFFFFFFFFu;
        st.nk[j] = 0xFFFFFFFFu;
        st.ms[j] = -INFINITY;
        st.sm[j] = 0.f;
    }
    consumer_sync();
}

// rows [0, nvalid) of the staged k_idx tile are tokens n0 + row; warp w
// takes the 16-row groups w, w+4, ...  Rows past nvalid may hold anything:
// each MMA row depends only on its own k_idx row and is dropped.
template <int G>
__device__ __forceinline__ void score_tile(const Params& P, StepSmem<G>& S, ScoreState<G>& st, const uint8_t* data, int b,
                                           int rgi, int n0, int nvalid, int tid) {
    const int nh = P.rg_nh[rgi], slot0 = P.rg_slot0[rgi];
    const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const uint32_t rows = smem_u32(data);
    constexpr float C = 0.25f * 1.4426950408889634f;   // (1/4) log2(e)
    const int h0 = 2 * t;                               // owned heads h0, h0 + 1
    uint32_t* keys0 = P.keys + ((int64_t)b * P.n_ret + slot0 + min(h0, nh - 1)) * P.Ncap + n0;
    uint32_t* keys1 = P.keys + ((int64_t)b * P.n_ret + slot0 + min(h0 + 1, nh - 1)) * P.Ncap + n0;
    const bool own0 = h0 < nh, own1 = h0 + 1 < nh;
    // ldmatrix row address of this lane: matrix m = lane/8 (rows +8 if m odd, bytes +16 if m >= 2)
    const uint32_t lrow = (uint32_t)(((lane >> 3) & 1) * 8 + (lane & 7)) * 32u + (uint32_t)((lane >> 4) * 16);
    const int ngroups = (nvalid + 15) / 16;
    constexpr int NW = CONSUMERS / 32;
    // four 16-row groups per warp at a time: their MMA chains are independent
#pragma unroll 1
    for (int base = warp; base < ngroups; base += 4 * NW) {
        uint32_t a[4][4];
        float c[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int grp = min(base + q * NW, ngroups - 1);
            asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                         : "=r"(a[q][0]), "=r"(a[q][1]), "=r"(a[q][2]), "=r"(a[q][3])
                         : "r"(rows + (uint32_t)grp * 512u + lrow));
            c[q][0] = c[q][1] = c[q][2] = c[q][3] = 0.f;
        }
#pragma unroll
        for (int p = 0; p < 3; ++p)
#pragma unroll
            for (int q = 0; q < 4; ++q)
                asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                    "{%0,%1,%2,%3};"
                    : "+f"(c[q][0]), "+f"(c[q][1]), "+f"(c[q][2]), "+f"(c[q][3])
                    : "r"(a[q][0]), "r"(a[q][1]), "r"(a[q][2]), "r"(a[q][3]), "r"(st.b[p][0]), "r"(st.b[p][1]));
        // per owned head: 8 values (rows g and g+8 of 4 groups, in row order)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            if (!(j ? own1 : own0)) continue;
            uint32_t* kp = j ? keys1 : keys0;
            uint32_t kb = 0u, rb = 0u, kmin = 0xFFFFFFFFu;
            float mb = -INFINITY;
            float v[8];
            bool ok[8];
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int e = q * 2 + h;
                    const int r = (base + q * NW) * 16 + g + 8 * h;
                    ok[e] = r < nvalid;
                    v[e] = ok[e] ? c[q][j + 2 * h] : -INFINITY;
                    const uint32_t key = f2key(v[e]);
                    if (ok[e]) {
                        kp[r] = key;
                        if (key > kb) {
                            kb = key;
                            rb = (uint32_t)(n0 + r);
                        }
                        kmin = min(kmin, key);
                    }
                    mb = fmaxf(mb, v[e]);
                }
            if (kb > st.mk[j]) {
                st.mk[j] = kb;
                st.am[j] = rb;
            }
            st.nk[j] = min(st.nk[j], kmin);
            if (mb > st.ms[j]) {
                st.sm[j] *= ex2_approx((st.ms[j] - mb) * C);
                st.ms[j] = mb;
            }
            float add = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) add += ok[e] ? ex2_approx((v[e] - st.ms[j]) * C) : 0.f;
            st.sm[j] += add;
        }
    }
}

// fold (max key a, running sum sa relative to score key ka) with (b, sb, kb):
// keys order-preserving; key 0 marks an empty accumulator
__device__ __forceinline__ void fold_ms(uint32_t& ka, float& sa, uint32_t kb, float sb) {
    if (kb == 0u) return;
    if (ka == 0u) {
        ka = kb;
        sa = sb;
        return;
    }
    constexpr float C = 0.25f * 1.4426950408889634f;   // (1/4) log2(e)
    const float ma = key2f(ka), mb = key2f(kb);
    if (mb > ma) {
        sa = sa * exp2f((ma - mb) * C) + sb;
        ka = kb;
    } else {
        sa += sb * exp2f((mb - ma) * C);
    }
}

// Selection of the heads of group (b, rgi) from its chunk partials.  Heads
// whose best token alone reaches p, or whose p >= 1, are final; if all heads
// of the group are final its block list is written here.
template <int G>
__device__ __forceinline__ void score_decide(const StepParams& SP, StepSmem<G>& S, int b, int rgi, int L, int nch, int tid) {
    const Params& P = SP.P;
    const int nh = P.rg_nh[rgi], slot0 = P.rg_slot0[rgi], g = P.rg_group[rgi];
    const int nblk = (L + BLK - 1) / BLK;
    const int nwords = (nblk + 31) / 32;
    __shared__ int s_mode[MAX_G];
    __shared__ uint32_t s_arg[MAX_G];
    // every chunk of the group has folded its partials into its heads'
    // buckets (score_end): one warp per head reduces the 32 buckets and
    // re-arms them for the next call
    __shared__ unsigned long long s_best[MAX_G];
    __shared__ uint32_t s_nmin[MAX_G], s_flags[MAX_G];
    __shared__ double s_zabs[MAX_G];
    {
        const int warp = tid >> 5, lane = tid & 31;
        for (int hh = warp; hh < nh; hh += CONSUMERS / 32) {
            HeadAgg* ag = P.agg + ((int64_t)b * P.n_ret + slot0 + hh) * AGG_BUCKETS + lane;
            unsigned long long best = __ldcg(&ag->best);
            uint32_t nmin = __ldcg(&ag->nmin), flags = __ldcg(&ag->flags);
            double zabs = __ldcg(&ag->zabs);
            ag->best = 0ull;
            ag->nmin = 0u;
            ag->flags = 0u;
            ag->zabs = 0.0;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
                nmin = max(nmin, __shfl_xor_sync(0xffffffffu, nmin, o));
                flags |= __shfl_xor_sync(0xffffffffu, flags, o);
                zabs += __shfl_xor_sync(0xffffffffu, zabs, o);
            }
            if (lane == 0) {
                s_best[hh] = best;
                s_nmin[hh] = nmin;
                s_flags[hh] = flags;
                s_zabs[hh] = zabs;
            }
        }
    }
    consumer_sync();
    if (tid < nh) {
        const int hh = tid;
        const int slot = slot0 + hh;
        const unsigned long long best = s_best[hh];
        const uint32_t k = (uint32_t)(best >> 32);
        const uint32_t a = 0xFFFFFFFFu - (uint32_t)(best & 0xFFFFFFFFull);
        const uint32_t mn = ~s_nmin[hh];
        const float smax = key2f(k);
        // z = sum over tokens of exp((s - smax)/4); NaN when the fp64 sum was unusable
        const double sm4 = (double)smax * 0.25;
        const double z = (s_flags[hh] || sm4 > 600.0 || sm4 < -600.0) ? NAN : s_zabs[hh] * exp(-sm4);
        {
            const float pb = __ldg(P.p + b);
            HeadState h;
            h.smax = smax;
            h.maxkey = k;
            h.argmax = a;
            h.minkey = mn;
            h.pad0 = 0;
            h.zrel = z;
            h.target = 0;
            h.mass_above = 0;
            h.prefix = 0;
            h.count_above = 0;
            h.n_eq = 0;
            h.n_tie = 0;
            h.all_ties = 1;
            h.tau_key = 0;
            h.pad1 = 0;
            if (!(pb > 0.f)) {
                h.mode = MODE_SKIP;
                h.kstar = 0;
                set_status(P, ST_DEVICE_INPUT);
            } else if (pb >= 1.f) {
                h.mode = MODE_ALL;
                h.kstar = (uint32_t)L;
                h.tau_key = mn;
            } else if (z == z && 1.0 >= (double)pb * z * (1.0 + 1e-3)) {
                h.mode = MODE_TOP1;   // the best token alone reaches p
                h.kstar = 1;
                h.tau_key = k;
            } else {
                h.mode = MODE_RADIX;
                h.kstar = 0;
            }
            P.hs[(int64_t)b * P.n_ret + slot] = h;
            const int bh = b * P.Hq + P.slot_head[slot];
            if (P.dbg_smax) P.dbg_smax[bh] = smax;
            if (P.dbg_Z) P.dbg_Z[bh] = z;
            if (h.mode != MODE_RADIX) {
                if (P.dbg_tau) P.dbg_tau[bh] = key2f(h.tau_key);
                if (P.dbg_kstar) P.dbg_kstar[bh] = (int32_t)h.kstar;
                if (P.dbg_kept)
                    P.dbg_kept[bh] = h.mode == MODE_TOP1 ? 1 : (h.mode == MODE_ALL ? nblk : 0);
            }
            s_mode[hh] = h.mode;
            s_arg[hh] = a;
        }
    }
    // the radix histograms of these heads start at zero
    for (int x = tid; x < nh * 256; x += CONSUMERS) {
        P.hist_cnt[((int64_t)b * P.n_ret + slot0) * 256 + x] = 0;
        P.hist_mass[((int64_t)b * P.n_ret + slot0) * 256 + x] = 0ull;
    }
    consumer_sync();

    bool any_radix = false, any_all = false;
    uint32_t all_mask = 0;
    for (int hh = 0; hh < nh; ++hh) {
        any_radix |= s_mode[hh] == MODE_RADIX;
        if (s_mode[hh] == MODE_ALL) {
            any_all = true;
            all_mask |= 1u << (P.slot_head[slot0 + hh] - g * P.G);
        }
    }
    // bitmap words of the heads that are final (read by the block-list
    // builder of a group that also has radix heads, and by the debug sink)
    const bool want_words = any_radix || P.dbg_bitmap != nullptr;
    if (want_words) {
        for (int hh = 0; hh < nh; ++hh) {
            const int mode = s_mode[hh];
            if (mode == MODE_RADIX) continue;
            const int slot = slot0 + hh;
            for (int w = tid; w < nwords; w += CONSUMERS) {
                uint32_t word = 0;
                if (mode == MODE_ALL) {
                    const int nb = min(32, nblk - w * 32);
                    word = nb >= 32 ? 0xFFFFFFFFu : ((1u << nb) - 1u);
                } else if (mode == MODE_TOP1) {
                    const int j = (int)(s_arg[hh] / BLK) - w * 32;
                    if (j >= 0 && j < 32) word = 1u << j;
                }
                if (any_radix) P.bitmap[((int64_t)b * P.n_ret + slot) * P.words_cap + w] = word;
                if (P.dbg_bitmap) P.dbg_bitmap[((int64_t)b * P.Hq + P.slot_head[slot]) * P.words_cap + w] = word;
            }
        }
    }
    const int bg = b * P.n_rg + rgi;
    if (any_radix) {
        consumer_sync();
        if (tid == 0) {
            for (int hh = 0; hh < nh; ++hh)
                if (s_mode[hh] == MODE_RADIX) {
                    const uint32_t k = atomicAdd(&SP.sync->n_radix_heads, 1u);
                    SP.rlist[k] = ((uint32_t)b << 16) | (uint32_t)(slot0 + hh);
                }
            const uint32_t gi = atomicAdd(&SP.sync->n_radix_groups, 1u);
            SP.rglist[gi] = ((uint32_t)b << 16) | (uint32_t)rgi;
            __threadfence();
            atomicAdd(&SP.sync->groups_decided, 1u);
        }
        return;
    }
    // every head final: write the group's block list now
    uint32_t* list = P.blist + (int64_t)bg * P.nblk_cap;
    if (any_all) {
        for (int j = tid; j < nblk; j += CONSUMERS) {
            uint32_t hm = all_mask;
            for (int hh = 0; hh < nh; ++hh)
                if (s_mode[hh] == MODE_TOP1 && (int)(s_arg[hh] / BLK) == j) hm |= 1u << (P.slot_head[slot0 + hh] - g * P.G);
            list[j] = ((uint32_t)j << 8) | hm;
        }
        if (tid == 0) P.bcount[bg] = (uint32_t)nblk;
    } else if (tid == 0) {
        // distinct argmax blocks of the TOP1 heads, ascending
        uint32_t cnt = 0;
        int last = -1;
        while (true) {
            int best = INT_MAX;
            for (int hh = 0; hh < nh; ++hh)
                if (s_mode[hh] == MODE_TOP1) {
                    const int j = (int)(s_arg[hh] / BLK);
                    if (j > last && j < best) best = j;
                }
            if (best == INT_MAX) break;
            uint32_t hm = 0;
            for (int hh = 0; hh < nh; ++hh)
                if (s_mode[hh] == MODE_TOP1 && (int)(s_arg[hh] / BLK) == best)
                    hm |= 1u << (P.slot_head[slot0 + hh] - g * P.G);
            list[cnt++] = ((uint32_t)best << 8) | hm;
            last = best;
        }
        P.bcount[bg] = cnt;
    }
    consumer_sync();
    if (tid == 0) {
        __threadfence();
        atomicAdd(&SP.sync->groups_decided, 1u);
        atomicAdd(&SP.sync->groups_ready, 1u);
        trace_max(P, 3);
    }
}

template <int G>
__device__ __forceinline__ void score_end(const StepParams& SP, StepSmem<G>& S, ScoreState<G>& st, int b, int rgi, int chunk,
                                          int L, int nch, int tid) {
    const Params& P = SP.P;
    const int nh = P.rg_nh[rgi], slot0 = P.rg_slot0[rgi];
    const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        uint32_t k = st.mk[j], a = st.am[j], mn = st.nk[j];
        uint32_t km = st.mk[j];   // the running sum is relative to the max score, whose key is mk
        float su = st.sm[j];
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            const uint32_t k2 = __shfl_xor_sync(0xffffffffu, k, o);
            const uint32_t a2 = __shfl_xor_sync(0xffffffffu, a, o);
            const uint32_t km2 = __shfl_xor_sync(0xffffffffu, km, o);
            const float s2 = __shfl_xor_sync(0xffffffffu, su, o);
            mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            if (k2 > k || (k2 == k && a2 < a)) {
                k = k2;
                a = a2;
            }
            fold_ms(km, su, km2, s2);
        }
        const int hh = 2 * t + j;
        if (g == 0 && hh < nh) {
            S.w_key[hh][warp] = k;
            S.w_arg[hh][warp] = a;
            S.w_min[hh][warp] = mn;
            S.w_m[hh][warp] = __uint_as_float(km);
            S.w_sum[hh][warp] = (double)su;
        }
    }
    consumer_sync();
    if (tid < nh) {
        const int hh = tid;
        uint32_t k = 0, a = 0xFFFFFFFFu, mn = 0xFFFFFFFFu, km = 0;
        float su = 0.f;
        for (int w = 0; w < 4; ++w) {
            if (S.w_key[hh][w] > k || (S.w_key[hh][w] == k && S.w_arg[hh][w] < a)) {
                k = S.w_key[hh][w];
                a = S.w_arg[hh][w];
            }
            mn = min(mn, S.w_min[hh][w]);
            fold_ms(km, su, __float_as_uint(S.w_m[hh][w]), (float)S.w_sum[hh][w]);
        }
        // fold this chunk into its bucket of the head's aggregate: fire-and-forget
        // atomics, the exp-sum as the fp64 sum of exp(s/4) (out of fp64's safe
        // range the head takes the exact radix path instead)
        HeadAgg* ag = P.agg + ((int64_t)b * P.n_ret + slot0 + hh) * AGG_BUCKETS + (chunk % AGG_BUCKETS);
        atomicMax(&ag->best, ((unsigned long long)k << 32) | (0xFFFFFFFFu - a));
        atomicMax(&ag->nmin, ~mn);
        if (km != 0u) {
            const double m4 = (double)key2f(km) * 0.25;
            if (m4 > 600.0 || m4 < -600.0) atomicOr(&ag->flags, 1u);
            else atomicAdd(&ag->zabs, (double)su * exp(m4));
        }
    }
    if (!consumer_last(P.tick_score + b * P.n_rg + rgi, nch, &S.flag)) return;
    __threadfence();
    if (tid == 0) trace_max(P, 6);
    score_decide<G>(SP, S, b, rgi, L, nch, tid);
    if (tid == 0) trace_max(P, 1);
}

// ===========================================================================
// exact radix select, block marking, block lists (consumers, L2-resident)
// ===========================================================================
template <int G>
__device__ __forceinline__ void radix_item(const StepParams& SP, StepSmem<G>& S, int b, int slot, int chunk, int L, int pass, int tid) {
    const Params& P = SP.P;
    const int nch = (L + CHUNK - 1) / CHUNK;
    const int64_t bs = (int64_t)b * P.n_ret + slot;
    HeadState* hsp = P.hs + bs;
    for (int d = tid; d < 256; d += CONSUMERS) {
        S.hcnt[d] = 0;
        S.hm[0][d] = 0;
        S.hm[1][d] = 0;
        S.hm[2][d] = 0;
    }
    const int n_begin = chunk * CHUNK, n_end = min(L, n_begin + CHUNK);
    const uint32_t* keys = P.keys + bs * P.Ncap;
    constexpr int PER = CHUNK / CONSUMERS;
    uint32_t kk[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int n = n_begin + tid + i * CONSUMERS;
        kk[i] = (n < n_end) ? __ldcg(keys + n) : 0u;
    }
    const uint32_t prefix = __ldcg(&hsp->prefix);
    const float smax = __ldcg(&hsp->smax);
    const int shift = 24 - 8 * pass;
    consumer_sync();
    // Lanes holding the same digit are summed in the warp (match + redux):
    // the 2^-40 fixed-point mass (< 2^41) is split into 17-bit slices so the
    // 32-bit warp and shared sums stay exact; one leader per digit updates
    // the shared histogram.
    const int lane = tid & 31;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int n = n_begin + tid + i * CONSUMERS;
        const uint32_t key = kk[i];
        const bool valid = n < n_end && (pass == 0 || (key >> (32 - 8 * pass)) == prefix);
        const uint32_t d = valid ? ((key >> shift) & 255u) : 0xFFFFFFFFu;
        const uint32_t peers = __match_any_sync(0xffffffffu, d);
        if (valid) {
            const unsigned long long ms = fixmass(key, smax);
            const uint32_t s0 = __reduce_add_sync(peers, (uint32_t)(ms & 0x1FFFFull));
            const uint32_t s1 = __reduce_add_sync(peers, (uint32_t)((ms >> 17) & 0x1FFFFull));
            const uint32_t s2 = __reduce_add_sync(peers, (uint32_t)(ms >> 34));
            if (lane == __ffs(peers) - 1) {
                atomicAdd(&S.hcnt[d], (uint32_t)__popc(peers));
                atomicAdd(&S.hm[0][d], s0);
                atomicAdd(&S.hm[1][d], s1);
                atomicAdd(&S.hm[2][d], s2);
            }
        }
    }
    consumer_sync();
    for (int d = tid; d < 256; d += CONSUMERS)
        S.hmass[d] = (unsigned long long)S.hm[0][d] + ((unsigned long long)S.hm[1][d] << 17) +
                     ((unsigned long long)S.hm[2][d] << 34);
    consumer_sync();
    uint32_t* gcnt = P.hist_cnt + bs * 256;
    unsigned long long* gmass = P.hist_mass + bs * 256;
    for (int d = tid; d < 256; d += CONSUMERS) {
        if (S.hcnt[d]) {
            atomicAdd(gcnt + d, S.hcnt[d]);
            atomicAdd(gmass + d, S.hmass[d]);
        }
        if (pass == 3) P.chunk_cnt[(bs * P.nchunks + chunk) * 256 + d] = S.hcnt[d];
    }
    if (!consumer_last(P.tick_radix + bs, nch, &S.flag)) return;
    __threadfence();
    for (int d = tid; d < 256; d += CONSUMERS) {
        S.hcnt[d] = __ldcg(gcnt + d);
        S.hmass[d] = __ldcg(gmass + d);
        gcnt[d] = 0;
        gmass[d] = 0ull;
    }
    consumer_sync();
    if (tid == 0) {
        HeadState st = *hsp;
        if (pass == 0) {
            unsigned long long z = 0;
            for (int d = 0; d < 256; ++d) z += S.hmass[d];
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
            if (cum + S.hmass[d] >= st.target) {
                dstar = d;
                break;
            }
            cum += S.hmass[d];
            cabove += S.hcnt[d];
        }
        st.mass_above = cum;
        st.count_above = cabove;
        st.prefix = (st.prefix << 8) | (uint32_t)dstar;
        if (pass == 3) {
            st.tau_key = st.prefix;
            st.n_eq = S.hcnt[dstar];
            const unsigned long long m_tau = st.n_eq ? S.hmass[dstar] / st.n_eq : 0ull;
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
            if (!st.all_ties) {
                uint32_t run = 0;
                for (int c = 0; c < nch; ++c) {
                    P.tie_off[bs * P.nchunks + c] = run;
                    run += P.chunk_cnt[(bs * P.nchunks + c) * 256 + dstar];
                }
            }
        }
        *hsp = st;
        __threadfence();
        atomicAdd(&SP.sync->pass_done[pass], 1u);
        trace_max(P, 8 + pass);
    }
}

template <int G>
__device__ __forceinline__ void mark_item(const StepParams& SP, StepSmem<G>& S, int b, int slot, int chunk, int L, int tid) {
    const Params& P = SP.P;
    const int nch = (L + CHUNK - 1) / CHUNK;
    const int64_t bs = (int64_t)b * P.n_ret + slot;
    HeadState st;
    {
        const HeadState* hsp = P.hs + bs;
        st.tau_key = __ldcg(&hsp->tau_key);
        st.all_ties = __ldcg(&hsp->all_ties);
        st.n_tie = __ldcg(&hsp->n_tie);
    }
    const int n_begin = chunk * CHUNK, n_end = min(L, n_begin + CHUNK);
    const uint32_t* keys = P.keys + bs * P.Ncap;
    const uint32_t tau = st.tau_key;
    const uint32_t tie_base = st.all_ties ? 0u : __ldcg(P.tie_off + bs * P.nchunks + chunk);
    const int warp = tid >> 5, lane = tid & 31;
    if (tid == 0) S.word = 0;
    uint32_t carry = 0;
    uint32_t mine = 0;
    constexpr int PER = CHUNK / CONSUMERS;
    uint32_t kk[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int n = n_begin + tid + i * CONSUMERS;
        kk[i] = (n < n_end) ? __ldcg(keys + n) : 0u;
    }
    consumer_sync();
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int base = n_begin + i * CONSUMERS;
        if (base >= n_end) break;
        const int n = base + tid;
        const uint32_t key = kk[i];
        bool keep = (n < n_end) && key > tau;
        const bool tie = (n < n_end) && key == tau;
        if (st.all_ties) {
            keep = keep || tie;
        } else {
            const uint32_t bal = __ballot_sync(0xffffffffu, tie);
            if (lane == 0) S.w_key[0][warp] = __popc(bal);
            consumer_sync();
            uint32_t before = carry;
            for (int w = 0; w < warp; ++w) before += S.w_key[0][w];
            before += __popc(bal & ((1u << lane) - 1u));
            keep = keep || (tie && tie_base + before < st.n_tie);
            carry += S.w_key[0][0] + S.w_key[0][1] + S.w_key[0][2] + S.w_key[0][3];
            consumer_sync();
        }
        if (keep) mine |= 1u << ((n - n_begin) / BLK);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mine |= __shfl_xor_sync(0xffffffffu, mine, o);
    if (lane == 0 && mine) atomicOr(&S.word, mine);
    consumer_sync();
    if (tid == 0) P.bitmap[bs * P.words_cap + chunk] = S.word;
    if (!consumer_last(P.tick_radix + bs, nch, &S.flag)) return;
    if (tid == 0) {
        __threadfence();
        atomicAdd(&SP.sync->mark_done, 1u);
        trace_max(P, 12);
    }
}

template <int G>
__device__ __forceinline__ void blist_item(const StepParams& SP, StepSmem<G>& S, int gi, int tid) {
    const Params& P = SP.P;
    const uint32_t e = __ldcg(SP.rglist + gi);
    const int b = (int)(e >> 16), rgi = (int)(e & 0xFFFFu);
    const int L = __ldg(P.seq_lens + b);
    const int g = P.rg_group[rgi], nh = P.rg_nh[rgi], slot0 = P.rg_slot0[rgi];
    const int nblk = (L + BLK - 1) / BLK;
    const int nwords = (nblk + 31) / 32;
    const int bg = b * P.n_rg + rgi;
    uint32_t* list = P.blist + (int64_t)bg * P.nblk_cap;
    const int warp = tid >> 5, lane = tid & 31;
    __shared__ int s_kept[MAX_G];
    __shared__ uint32_t s_base;
    if (tid < MAX_G) s_kept[tid] = 0;
    if (tid == 0) s_base = 0;
    consumer_sync();
    for (int w0 = 0; w0 < nwords; w0 += CONSUMERS) {
        const int w = w0 + tid;
        uint32_t uni = 0;
        uint32_t wh[MAX_G];
#pragma unroll
        for (int hh = 0; hh < MAX_G; ++hh) {
            wh[hh] = 0;
            if (hh < nh && w < nwords) {
                wh[hh] = __ldcg(P.bitmap + ((int64_t)b * P.n_ret + slot0 + hh) * P.words_cap + w);
                if (w == nwords - 1 && (nblk & 31)) wh[hh] &= (1u << (nblk & 31)) - 1u;
                uni |= wh[hh];
                if (wh[hh]) atomicAdd(&s_kept[hh], __popc(wh[hh]));
                if (P.dbg_bitmap)
                    P.dbg_bitmap[((int64_t)b * P.Hq + P.slot_head[slot0 + hh]) * P.words_cap + w] = wh[hh];
            }
        }
        const uint32_t c = __popc(uni);
        uint32_t incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        if (lane == 31) S.w_key[0][warp] = incl;
        consumer_sync();
        uint32_t off = s_base;
        for (int ww = 0; ww < warp; ++ww) off += S.w_key[0][ww];
        uint32_t pos = off + incl - c;
        while (uni) {
            const int jb = __ffs(uni) - 1;
            uni &= uni - 1;
            uint32_t hm = 0;
#pragma unroll
            for (int hh = 0; hh < MAX_G; ++hh)
                if ((wh[hh] >> jb) & 1u) hm |= 1u << (P.slot_head[slot0 + hh] - g * P.G);
            list[pos++] = ((uint32_t)(w * 32 + jb) << 8) | hm;
        }
        consumer_sync();
        if (tid == 0) s_base += S.w_key[0][0] + S.w_key[0][1] + S.w_key[0][2] + S.w_key[0][3];
        consumer_sync();
    }
    if (tid < nh && P.dbg_kept) P.dbg_kept[b * P.Hq + P.slot_head[slot0 + tid]] = s_kept[tid];
    if (tid == 0) {
        P.bcount[bg] = s_base;
        __threadfence();
        atomicAdd(&SP.sync->groups_ready, 1u);
        trace_max(P, 3);
    }
    consumer_sync();
}

// ===========================================================================
// the persistent kernel
// ===========================================================================
// radix / mark item j -> (b, slot, chunk, L) in d; false when the chunk is
// past the head's sequence length
__device__ __forceinline__ bool resolve_chunk(const StepParams& SP, int j, Desc& d) {
    const Params& P = SP.P;
    const int k = j / P.nchunks, chunk = j % P.nchunks;
    const uint32_t e = __ldcg(SP.rlist + k);
    const int b = (int)(e >> 16), slot = (int)(e & 0xFFFFu);
    const int L = __ldg(P.seq_lens + b);
    if (chunk >= (L + CHUNK - 1) / CHUNK) return false;
    d.b = b;
    d.grp = slot;
    d.item = chunk;
    d.aux1 = L;
    return true;
}

template <int G>
__device__ __forceinline__ void producer(const StepParams& SP, StepSmem<G>& S) {
    constexpr int NST = StepSmem<G>::NST;
    const Params& P = SP.P;
    Sync* sy = SP.sync;
    uint32_t t = 0;   // tiles published so far (same sequence the consumers follow)
    bool alive = true;
    const bool acct = P.dbg_trace != nullptr;
    unsigned long long a_slot = 0, a_dep = 0, a_claim = 0;

    auto acquire = [&]() -> int {
        const int st = (int)(t % NST);
        const uint32_t round = t / NST;
        const uint64_t t0 = acct ? global_ns() : 0;
        if (round > 0 && !mbar_wait_bounded(&S.empty[st], (round - 1) & 1u)) {
            set_status(P, ST_TIMEOUT);
            alive = false;
        }
        if (acct) a_slot += global_ns() - t0;
        return st;
    };
    auto publish_nodata = [&](const Desc& d) {
        const int st = acquire();
        if (!alive) return;
        S.desc[st] = d;
        mbar_arrive(&S.full[st]);
        ++t;
    };
    auto wait_for = [&](const uint32_t* ctr, uint32_t target) {
        const uint64_t t0 = acct ? global_ns() : 0;
        if (alive && !wait_counter(ctr, target)) {
            set_status(P, ST_TIMEOUT);
            alive = false;
        }
        if (acct) a_dep += global_ns() - t0;
    };
    auto claim = [&]() -> uint32_t {
        const uint64_t t0 = acct ? global_ns() : 0;
        const uint32_t v = atomicAdd(&sy->queue, 1u);
        if (acct) a_claim += global_ns() - t0;
        return v;
    };

    const int n_static = SP.n_score_items + SP.n_local_items;
    uint32_t x = claim();
    while (alive && (int)x < n_static) {
        if ((int)x < SP.n_score_items) {
            // ---- index-score chunk (b, rgi, chunk) ----
            const int per_b = P.n_rg * P.nschunks;
            const int b = (int)x / per_b, rgi = ((int)x % per_b) / P.nschunks, chunk = (int)x % P.nschunks;
            const int L = __ldg(P.seq_lens + b);
            if (!seq_ok(P, L)) {
                if (chunk == 0) {   // this sequence's groups: no selection, no blocks
                    set_status(P, ST_DEVICE_INPUT);
                    P.bcount[b * P.n_rg + rgi] = 0;
                    __threadfence();
                    atomicAdd(&sy->groups_decided, 1u);
                    atomicAdd(&sy->groups_ready, 1u);
                }
            } else {
                const int nch = (L + SCORE_CHUNK - 1) / SCORE_CHUNK;
                if (chunk < nch) {
                    const int g = P.rg_group[rgi];
                    const int n_begin = chunk * SCORE_CHUNK, n_end = min(L, n_begin + SCORE_CHUNK);
                    const int ntiles = (n_end - n_begin + SCORE_ROWS - 1) / SCORE_ROWS;
                    for (int ti = 0; ti < ntiles && alive; ++ti) {
                        const int n0 = n_begin + ti * SCORE_ROWS;
                        const int nvalid = min(SCORE_ROWS, n_end - n0);
                        const int nblocks = (nvalid + BLK - 1) / BLK;
                        const int st = acquire();
                        if (!alive) break;
                        Desc d;
                        d.type = IT_SCORE;
                        d.b = b;
                        d.grp = rgi;
                        d.item = chunk;
                        d.tile = ti;
                        d.ntiles = ntiles;
                        d.n0 = n0;
                        d.nvalid = nvalid;
                        d.hmask = 0;
                        d.aux0 = nch;
                        d.aux1 = L;
                        d.bad = 0;
                        S.desc[st] = d;
                        mbar_expect_tx(&S.full[st], (uint32_t)nblocks * BLK * R * 2);
                        if (P.block_table == nullptr) {
                            const uint16_t* src = P.k_idx + (((int64_t)b * P.Hkv + g) * P.Ncap + n0) * R;
                            bulk_g2s(&S.stage[st][0], src, (uint32_t)nblocks * BLK * R * 2, &S.full[st]);
                        } else {
                            for (int q = 0; q < nblocks; ++q) {
                                int bad = 0;
                                const int64_t off = tile_off(P, b, g, n0 / BLK + q, R, &bad);
                                if (bad) set_status(P, ST_DEVICE_INPUT);
                                bulk_g2s(&S.stage[st][q * BLK * R * 2], P.k_idx + off, BLK * R * 2, &S.full[st]);
                            }
                        }
                        ++t;
                    }
                }
            }
        } else {
            // ---- local-head item (b, lgi, item) ----
            const int y = (int)x - SP.n_score_items;
            const int per_b = P.n_lg * P.local_items;
            const int b = y / per_b, lgi = (y % per_b) / P.local_items, item = y % P.local_items;
            const int L = __ldg(P.seq_lens + b);
            if (seq_ok(P, L)) {
                const LocalGeom lg = local_geom(P, L);
                const int nitems = (lg.nv + P.local_kb - 1) / P.local_kb;
                if (item < nitems) {
                    const int g = P.lg_group[lgi];
                    const int v0 = item * P.local_kb, ntiles = min(P.local_kb, lg.nv - v0);
                    for (int i = 0; i < ntiles && alive; ++i) {
                        const int v = v0 + i;
                        const int j = v < lg.nA ? v : lg.bw0 + (v - lg.nA);
                        const int st = acquire();
                        if (!alive) break;
                        Desc d;
                        d.type = IT_LOCAL;
                        d.b = b;
                        d.grp = lgi;
                        d.item = item;
                        d.tile = i;
                        d.ntiles = ntiles;
                        d.n0 = j * BLK;
                        d.nvalid = min(BLK, L - j * BLK);
                        d.hmask = P.lg_mask[lgi];
                        d.aux0 = nitems;
                        d.aux1 = L;
                        d.bad = 0;
                        const int64_t off = tile_off(P, b, g, j, D, &d.bad);
                        S.desc[st] = d;
                        mbar_expect_tx(&S.full[st], STAGE_BYTES);
                        bulk_g2s(&S.stage[st][0], P.k_cache + off, TILE_BYTES, &S.full[st]);
                        bulk_g2s(&S.stage[st][TILE_BYTES], P.v_cache + off, TILE_BYTES, &S.full[st]);
                        ++t;
                    }
                }
            }
        }
        x = claim();
    }

    // ---- retrieval heads: finish the selection, then their tiles ----
    if (alive && P.n_rg > 0) {
        const uint32_t ngroups = (uint32_t)(P.B * P.n_rg);
        wait_for(&sy->groups_decided, ngroups);
        const uint32_t nrad = alive ? ld_acquire(&sy->n_radix_heads) : 0u;
        if (nrad > 0) {
            const uint32_t nitems = nrad * (uint32_t)P.nchunks;
            for (int pass = 0; pass < 4 && alive; ++pass) {
                for (uint32_t j = atomicAdd(&sy->pass_claim[pass], 1u); j < nitems && alive;
                     j = atomicAdd(&sy->pass_claim[pass], 1u)) {
                    Desc d{};
                    if (!resolve_chunk(SP, (int)j, d)) continue;
                    d.type = IT_RADIX;
                    d.aux0 = pass;
                    publish_nodata(d);
                }
                wait_for(&sy->pass_done[pass], nrad);
            }
            for (uint32_t j = atomicAdd(&sy->mark_claim, 1u); j < nitems && alive; j = atomicAdd(&sy->mark_claim, 1u)) {
                Desc d{};
                if (!resolve_chunk(SP, (int)j, d)) continue;
                d.type = IT_MARK;
                publish_nodata(d);
            }
            wait_for(&sy->mark_done, nrad);
            const uint32_t ngr = alive ? ld_acquire(&sy->n_radix_groups) : 0u;
            for (uint32_t j = atomicAdd(&sy->blist_claim, 1u); j < ngr && alive; j = atomicAdd(&sy->blist_claim, 1u)) {
                Desc d{};
                d.type = IT_BLIST;
                d.item = (int)j;
                publish_nodata(d);
            }
        }
        wait_for(&sy->groups_ready, ngroups);
        if (alive) {
            // blocks per retrieval item, chosen so that the items about fill the grid
            long long total = 0;
            for (int bg = 0; bg < (int)ngroups; ++bg)
                if (seq_ok(P, __ldg(P.seq_lens + bg / P.n_rg))) total += __ldcg(P.bcount + bg);
            const int KB = (int)max(1ll, (total + gridDim.x - 1) / gridDim.x);
            int r = (int)x - n_static;
            // walk the (b, group) segments in order; r only grows
            int bg = 0, seg_base = 0, seg_items = 0, cnt = 0, L = 0;
            auto load_seg = [&]() {
                const int b = bg / P.n_rg;
                L = __ldg(P.seq_lens + b);
                cnt = seq_ok(P, L) ? (int)__ldcg(P.bcount + bg) : 0;
                seg_items = (cnt + KB - 1) / KB;
            };
            load_seg();
            while (alive) {
                while (bg < (int)ngroups && r >= seg_base + seg_items) {
                    seg_base += seg_items;
                    ++bg;
                    if (bg < (int)ngroups) load_seg();
                }
                if (bg >= (int)ngroups) break;
                const int b = bg / P.n_rg, rgi = bg % P.n_rg, g = P.rg_group[rgi];
                const int it = r - seg_base;
                const int k0 = it * KB, ntiles = min(KB, cnt - k0);
                const uint32_t* list = P.blist + (int64_t)bg * P.nblk_cap;
                for (int i = 0; i < ntiles && alive; ++i) {
                    const uint32_t e = __ldcg(list + k0 + i);
                    const int j = (int)(e >> 8);
                    const int st = acquire();
                    if (!alive) break;
                    Desc d;
                    d.type = IT_RET;
                    d.b = b;
                    d.grp = rgi;
                    d.item = it;
                    d.tile = i;
                    d.ntiles = ntiles;
                    d.n0 = j * BLK;
                    d.nvalid = min(BLK, L - j * BLK);
                    d.hmask = e & 0xFFu;
                    d.aux0 = seg_base;   // partial slot of the group's first item
                    d.aux1 = seg_items;
                    d.bad = 0;
                    const int64_t off = tile_off(P, b, g, j, D, &d.bad);
                    S.desc[st] = d;
                    mbar_expect_tx(&S.full[st], STAGE_BYTES);
                    bulk_g2s(&S.stage[st][0], P.k_cache + off, TILE_BYTES, &S.full[st]);
                    bulk_g2s(&S.stage[st][TILE_BYTES], P.v_cache + off, TILE_BYTES, &S.full[st]);
                    ++t;
                }
                r = (int)claim() - n_static;
            }
        }
    }
    Desc d{};
    d.type = IT_STOP;
    publish_nodata(d);
    // never leave the CTA with copies in flight: wait (bounded) for the last
    // tile published into each stage to have landed
    for (uint32_t i = (t > (uint32_t)NST ? t - NST : 0u); i < t; ++i)
        mbar_wait_bounded(&S.full[i % NST], (i / NST) & 1u);
    if (acct) {
        atomicAdd(P.dbg_trace + 26, a_slot);
        atomicAdd(P.dbg_trace + 27, a_dep);
        atomicAdd(P.dbg_trace + 28, a_claim);
    }
}

template <int G>
__device__ __forceinline__ void consumers(const StepParams& SP, StepSmem<G>& S, int tid) {
    constexpr int NST = StepSmem<G>::NST;
    const Params& P = SP.P;
    AttnCore<G> core;
    ScoreState<G> sc;
    uint32_t t = 0;
    const int warp = tid >> 5, lane = tid & 31;
    // cycle accounting for the debug trace (thread 0), by category:
    // 0 wait for data, 1 score begin, 2 score tile, 3 score release, 4 score
    // epilogue, 5 attention begin, 6 attention tile, 7 attention epilogue,
    // 8 data-less items
    const bool acct = P.dbg_trace != nullptr && tid == 0;
    if (acct)
        for (int i = 0; i < 10; ++i) S.acct[i] = 0ull;
    long long c_mark = acct ? clock64() : 0;
    auto mark = [&](int cat) {
        if (!acct) return;
        const long long now = clock64();
        S.acct[cat] += (unsigned long long)(now - c_mark);
        c_mark = now;
    };
    while (true) {
        const int st = (int)(t % NST);
        const uint32_t par = (t / NST) & 1u;
        mark(8);   // whatever ran since the last mark and was not classified
        if (!mbar_wait_bounded(&S.full[st], par)) {
            set_status(P, ST_TIMEOUT);
            break;
        }
        mark(0);
        const Desc d = S.desc[st];
        const uint8_t* data = &S.stage[st][0];
        ++t;
        if (d.type == IT_STOP) break;
        if (d.type == IT_SCORE) {
            if (d.tile == 0) score_begin<G>(P, S, sc, d.b, d.grp, tid);
            mark(1);
            score_tile<G>(P, S, sc, data, d.b, d.grp, d.n0, d.nvalid, tid);
            mark(2);
            if (acct) S.acct[9] += 1;
            consumer_sync();
            if (lane == 0) mbar_arrive(&S.empty[st]);
            mark(3);
            if (d.tile == d.ntiles - 1) {
                score_end<G>(SP, S, sc, d.b, d.grp, d.item, d.aux1, d.aux0, tid);
                mark(4);
            }
            continue;
        }
        if (d.type == IT_LOCAL || d.type == IT_RET) {
            const bool local = d.type == IT_LOCAL;
            const int g = local ? P.lg_group[d.grp] : P.rg_group[d.grp];
            if (d.tile == 0) core.begin(P, S, d.b, g, tid);
            mark(5);
            if (d.bad) {
                if (tid == 0) set_status(P, ST_DEVICE_INPUT);
            } else {
                int s_end = 0, w_lo = 0;
                if (local) {
                    const LocalGeom lg = local_geom(P, d.aux1);
                    s_end = lg.s_end;
                    w_lo = lg.w_lo;
                }
                core.tile(S, data, d.hmask, d.n0, d.nvalid, local, s_end, w_lo, tid);
            }
            if (lane == 0) mbar_arrive(&S.empty[st]);
            mark(6);
            if (d.tile == d.ntiles - 1) {
                float* parts;
                uint32_t heads, *ctr;
                int nitems;
                if (local) {
                    parts = P.lpart + (((int64_t)d.b * P.n_lg + d.grp) * P.local_items) * G * PSTRIDE;
                    heads = P.lg_mask[d.grp];
                    ctr = P.tick_local + d.b * P.n_lg + d.grp;
                    nitems = d.aux0;
                } else {
                    parts = P.rpart + (int64_t)d.aux0 * G * PSTRIDE;
                    heads = P.rg_mask[d.grp];
                    ctr = P.tick_ret + d.b * P.n_rg + d.grp;
                    nitems = d.aux1;
                }
                core.flush(S, parts + (int64_t)d.item * G * PSTRIDE, heads, tid);
                if (consumer_last(ctr, nitems, &S.flag)) {
                    __threadfence();
                    if (tid == 0 && local) trace_max(P, 7);
                    combine_parts<G>(P, S, parts, nitems, heads, d.b, g, tid);
                    if (tid == 0) trace_max(P, local ? 2 : 4);
                }
                mark(7);
            }
            continue;
        }
        // data-less items: release the slot first
        consumer_sync();
        if (lane == 0) mbar_arrive(&S.empty[st]);
        if (d.type == IT_RADIX) radix_item<G>(SP, S, d.b, d.grp, d.item, d.aux1, d.aux0, tid);
        else if (d.type == IT_MARK) mark_item<G>(SP, S, d.b, d.grp, d.item, d.aux1, tid);
        else if (d.type == IT_BLIST) blist_item<G>(SP, S, d.item, tid);
    }
    if (acct) {
        for (int i = 0; i < 10; ++i) atomicAdd(P.dbg_trace + 16 + i, S.acct[i]);
    }
    (void)warp;
}

template <int G>
__global__ void __launch_bounds__(STEP_THREADS, (G >= 8) ? 1 : 2) step_kernel(const __grid_constant__ StepParams SP) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    StepSmem<G>& S = *reinterpret_cast<StepSmem<G>*>(smem_raw);
    constexpr int NST = StepSmem<G>::NST;
    const int tid = threadIdx.x;
    if (tid == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(&S.full[i], 1);
            mbar_init(&S.empty[i], CONSUMERS / 32);
        }
        S.qi_tag = 0;
        mbar_fence_init();
    }
    if (tid == 0 && SP.P.dbg_trace) atomicCAS(SP.P.dbg_trace, 0ull, (unsigned long long)global_ns());
    __syncthreads();
    if (tid >= CONSUMERS) {
        if (tid == CONSUMERS) producer<G>(SP, S);
        return;
    }
    consumers<G>(SP, S, tid);
    // last CTA out clears the coordination words for the next call
    consumer_sync();
    if (tid == 0) trace_max(SP.P, 5);
    if (tid == 0) {
        __threadfence();
        if (atomicAdd(&SP.sync->exit_count, 1u) == gridDim.x - 1) {
            uint32_t* w = reinterpret_cast<uint32_t*>(SP.sync);
            for (int i = 0; i < (int)(sizeof(Sync) / 4); ++i) atomicExch(w + i, 0u);
            __threadfence();
        }
    }
}

}  // namespace rtp
