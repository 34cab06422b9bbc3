// Streaming kernel of the decode step (sm_100a): every CTA streams a
// contiguous share of equal weight of the step's 32 KB tiles -- first the index-cache
// tiles of the retrieval groups (1024 tokens of k_idx each), then the K/V
// tiles of the local heads' sink + window blocks -- through a shared-memory
// ring fed by one copy warp (bulk copies for k_idx, 2-D TMA boxes with the
// 128-byte swizzle for K/V), while four compute warps score (tensor cores)
// or attend (tensor cores).  No CTA waits on another: a split's results are
// folded with fire-and-forget atomics, and tickets elect the last arrival of
// each item to finish it (select the retrieval heads' blocks; combine the
// local heads' splits).
//
// Sources: "Full Attention Strikes Back" (RTPurbo) review on
// dongryeollee1.github.io, Method: "Adaptive sparse attention" (local heads:
// sink + sliding window; retrieval heads: Top-P over the low-rank scores) and
// "Hardware-aware top-p decoding kernel" (per-block scoring pass at D = 16,
// the last CTA deciding the threshold); aitrends.kr summary, architecture
// paragraph (kernel 1 at D = 16, kernel 2 at D = 128).
#pragma once
#include "rtp_attn.cuh"

namespace rtp {

template <int G>
struct ASmem {
    static constexpr int NST = (G >= 8) ? 2 : 3;
    alignas(1024) uint8_t stage[NST][STAGE_BYTES];
    AttnScratch<G> X;
    alignas(16) float qi[G][R];
    float w_m[4][G], w_s[4][G], w_bv[4][G], w_mn[4][G];
    uint32_t w_bi[4][G];
    alignas(8) uint64_t full[NST], empty[NST];
    unsigned long long d_best[MAX_G];
    uint32_t d_nmin[MAX_G], d_flags[MAX_G], d_arg[MAX_G];
    double d_zabs[MAX_G];
    int d_mode[MAX_G];
    uint32_t d_list[MAX_G], d_cnt;
    int pend_b, pend_rg, pend_L;   // best-token blocks this CTA attends after its share (d_list)
    uint32_t flag;
    unsigned long long acct[ACCT_SLOTS];   // debug cycle sums of thread 0
    int tot_s, tot_l, nact;
    int n_vgroups;   // (b, retrieval group) pairs of sequences with a valid length
    HeadTab tab;
    int pre[2];   // really [2 * (B + 1)]: tiles before sequence b (score, then local)
};

template <int G>
constexpr size_t asmem_bytes(int B) {
    return sizeof(ASmem<G>) + sizeof(int) * 2 * (size_t)(B + 1);
}

// One run of consecutive tiles of a single item inside a CTA's share.
struct Seg {
    int type;         // 0 = index scores of (b, retrieval group), 1 = local heads of (b, local group), -1 = none
    int b, grp, L;
    int item_idx;     // b * n_rg + grp, or b * n_lg + grp
    int item_t0;      // global index of the item's first tile
    int item_tiles;   // tiles of the whole item
    int first;        // index within the item of this run's first tile
    int ntiles;       // tiles in this run
};

__device__ __forceinline__ int last_le(const int* a, int n, int t) {
    // largest i in [0, n) with a[i] <= t (a ascending, a[0] = 0 <= t)
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a[mid] <= t) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// The CTA of global tile t when T tiles are shared by `nact` <= T CTAs, CTA
// c taking [c*T/nact, (c+1)*T/nact) (never empty, so every CTA between the
// first and the last of an item holds a split of it).
__device__ __forceinline__ int cta_of_tile(long long t, long long T, int nact) {
    return (int)(((t + 1) * nact + T - 1) / T) - 1;
}

// This CTA's share [t0, t1) of T tiles over the first nact CTAs: min(grid,
// T / min_per) of them (at least one when T > 0), so that a share holds at
// least min_per tiles when there are few (and is never empty).
__device__ __forceinline__ void cta_share(long long T, int& t0, int& t1, int& nact, int min_per = 1) {
    long long want = T / min_per;
    if (want < 1 && T > 0) want = 1;
    nact = (int)(want < (long long)gridDim.x ? want : (long long)gridDim.x);
    if ((int)blockIdx.x < nact) {
        t0 = (int)((long long)blockIdx.x * T / nact);
        t1 = (int)((long long)(blockIdx.x + 1) * T / nact);
    } else {
        t0 = t1 = 0;
    }
}

// The streaming kernel shares tile weight, not tiles: an index tile counts
// W_SCORE, a local tile W_LOCAL.  Index tiles cost more (MMA scores, fold,
// stored scores) and the group decision and best-token attention follow
// the last index split, so index CTAs take fewer tiles and the two paths
// end closer together.  Tile t's weight starts at tile_w0(t); a CTA's share
// is a contiguous weight range, never shorter than one tile.
constexpr int W_SCORE = 5, W_LOCAL = 4;
__device__ __forceinline__ long long tile_w0(long long t, long long Ts) {
    return t < Ts ? t * W_SCORE : Ts * W_SCORE + (t - Ts) * W_LOCAL;
}
// smallest t with tile_w0(t) >= w
__device__ __forceinline__ long long first_tile_at(long long w, long long Ts) {
    const long long ws = Ts * W_SCORE;
    return w <= ws ? (w + W_SCORE - 1) / W_SCORE : Ts + (w - ws + W_LOCAL - 1) / W_LOCAL;
}
// This CTA's tiles [t0, t1) of Ts index and Tl local tiles over the first
// nact CTAs: CTA c takes the tiles whose weight starts in
// [c W / nact, (c + 1) W / nact).
__device__ __forceinline__ void cta_wshare(long long Ts, long long Tl, int& t0, int& t1, int& nact) {
    const long long W = Ts * W_SCORE + Tl * W_LOCAL;
    const long long cap = W / W_SCORE;   // spans of at least W_SCORE: every CTA owns a tile
    nact = (int)(cap < (long long)gridDim.x ? cap : (long long)gridDim.x);
    if ((int)blockIdx.x < nact) {
        t0 = (int)first_tile_at((long long)blockIdx.x * W / nact, Ts);
        t1 = (int)first_tile_at((long long)(blockIdx.x + 1) * W / nact, Ts);
    } else {
        t0 = t1 = 0;
    }
}
// the CTA owning tile t under cta_wshare
__device__ __forceinline__ int cta_of_wtile(long long t, long long Ts, long long Tl, int nact) {
    const long long W = Ts * W_SCORE + Tl * W_LOCAL;
    return (int)(((tile_w0(t, Ts) + 1) * nact + W - 1) / W) - 1;
}

// A CTA's share: tiles [t, t1) of the sequence (index tiles, then local
// tiles from tot_s on), then optionally local tiles [tot_s + l0, tot_s + l1);
// item_t0 of a local item counts from the start of the local tiles.
struct AWalk {
    int t, t1, l0, l1;
    __device__ __forceinline__ Seg next(const Params& P, const int* pre_s, const int* pre_l, int tot_s) {
        Seg s;
        s.type = -1;
        if (t >= t1 && l0 < l1) {
            t = tot_s + l0;
            t1 = tot_s + l1;
            l0 = l1;
        }
        if (t >= t1) return s;
        if (t < tot_s) {
            const int b = last_le(pre_s, P.B + 1, t);
            const int L = __ldg(P.seq_lens + b);
            const int nt = (L + SROWS - 1) / SROWS;
            const int u = t - pre_s[b];
            s.type = 0;
            s.b = b;
            s.grp = u / nt;
            s.L = L;
            s.item_idx = b * P.n_rg + s.grp;
            s.item_t0 = pre_s[b] + s.grp * nt;
            s.item_tiles = nt;
            s.first = u % nt;
        } else {
            const int tl = t - tot_s;
            const int b = last_le(pre_l, P.B + 1, tl);
            const int L = __ldg(P.seq_lens + b);
            const int nv = local_geom(P, L).nv;
            const int u = tl - pre_l[b];
            s.type = 1;
            s.b = b;
            s.grp = u / nv;
            s.L = L;
            s.item_idx = b * P.n_lg + s.grp;
            s.item_t0 = pre_l[b] + s.grp * nv;
            s.item_tiles = nv;
            s.first = u % nv;
        }
        s.ntiles = min(s.item_tiles - s.first, t1 - t);
        t += s.ntiles;
        return s;
    }
};

// The best-token blocks a CTA selected (decide_group), as one more attention
// segment after its share: type 2, tiles = the block list in shared memory.
template <typename SM>
__device__ __forceinline__ Seg best_token_seg(const SM& S) {
    Seg s;
    s.type = 2;
    s.b = S.pend_b;
    s.grp = S.pend_rg;
    s.L = S.pend_L;
    s.item_idx = 0;
    s.item_t0 = 0;
    s.item_tiles = (int)S.d_cnt;
    s.first = 0;
    s.ntiles = (int)S.d_cnt;
    return s;
}

// Ticket among the consumer threads with a variable increment: true in the
// CTA whose addition completes `total`.  The fence before the addition
// publishes this CTA's writes; the fence after it, in the CTA that completes
// the count, orders its later reads of the other CTAs' writes (and, through
// the CTA barrier, those of its other threads).  That CTA re-arms the counter
// with a plain store: the next addition to it comes from a later launch.
__device__ __forceinline__ bool ticket_add(uint32_t* ctr, uint32_t add, uint32_t total, uint32_t* smem_flag) {
    consumer_sync();
    if (threadIdx.x == 0) {
        __threadfence();
        const uint32_t old = atomicAdd(ctr, add);
        const bool last = old + add == total;
        if (last) {
            __threadfence();
            *reinterpret_cast<volatile uint32_t*>(ctr) = 0u;
        }
        *smem_flag = last;
    }
    consumer_sync();
    return *smem_flag != 0;
}

// The group's list when its heads keep only their best tokens (thread 0):
// the distinct argmax blocks, ascending, with their head masks; the first
// such group of a CTA is attended by that CTA after its share, a later one
// goes to the retrieval kernel.
template <int G>
__device__ __forceinline__ void best_token_list(const Params& P, ASmem<G>& S, int b, int rg, int L, int nh, int slot0,
                                                int g) {
    const int bg = b * P.n_rg + rg;
    uint32_t* list = P.blist + (int64_t)bg * P.nblk_cap;
    // the distinct argmax blocks ascending, written straight to their
    // destination (short loops, not unrolled: this runs once per group, on
    // code that is rarely in the instruction cache)
    const bool defer = S.d_cnt == 0;
    uint32_t* dst = defer ? S.d_list : list;
    uint32_t cnt = 0;
    int last = -1;
#pragma unroll 1
    while (true) {
        int bj = 0x7FFFFFFF;
        uint32_t hm = 0;
#pragma unroll 1
        for (int hh = 0; hh < nh; ++hh) {
            if (S.d_mode[hh] != MODE_TOP1) continue;
            const int j = (int)(S.d_arg[hh] / BLK);
            const uint32_t bit = 1u << (S.tab.slot_head[slot0 + hh] - g * P.G);
            if (j > last && j < bj) {
                bj = j;
                hm = bit;
            } else if (j == bj) {
                hm |= bit;
            }
        }
        if (bj == 0x7FFFFFFF) break;
        dst[cnt++] = ((uint32_t)bj << 8) | hm;
        last = bj;
    }
    if (defer && cnt != 0) {
        S.d_cnt = cnt;
        S.pend_b = b;
        S.pend_rg = rg;
        S.pend_L = L;
        P.bcount[bg] = 0;
    } else {
        P.bcount[bg] = cnt;
        if (cnt) atomicAdd(&P.sync->kb_work, 1u);
    }
}

// ---------------------------------------------------------------------------
// selection of one retrieval group, by the last of its score splits
// ---------------------------------------------------------------------------
// Heads whose best token alone reaches p (TOP1) or whose p >= 1 (ALL) are
// final here; if every head of the group is final its block list is written
// at once, otherwise its radix heads are registered for the exact select.
// Under static top-k (P.topk = k >= 1) the same three outcomes are k >= L
// (ALL), k = 1 (TOP1: the argmax, lowest index among equal maxima) and any
// other k (the exact select, counting tokens instead of summing mass).
template <int G>
__device__ __forceinline__ void decide_group_body(const KParams& K, ASmem<G>& S, int b, int rg, int L, float pb,
                                                  int tid) {
    const Params& P = K.P;
    const int nh = S.tab.rg_nh[rg], slot0 = S.tab.rg_slot0[rg], g = S.tab.rg_group[rg];
    const int nblk = (L + BLK - 1) / BLK;
    const int nwords = (nblk + 31) / 32;
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
                S.d_best[hh] = best;
                S.d_nmin[hh] = nmin;
                S.d_flags[hh] = flags;
                S.d_zabs[hh] = zabs;
                // the best token's block into L2 now: if the head keeps only
                // that token, this CTA attends it right after the decision
                const uint32_t a = 0xFFFFFFFFu - (uint32_t)(best & 0xFFFFFFFFull);
                if (a < (uint32_t)L) kv_prefetch_l2(&K.tmk, &K.tmv, (int)block_row(P, b, g, (int)(a / BLK)));
            }
        }
    }
    consumer_sync();
    if (tid == 0) trace_max(P, 43);
    if (tid < nh) {
        const int hh = tid, slot = slot0 + hh;
        const unsigned long long best = S.d_best[hh];
        const uint32_t k = (uint32_t)(best >> 32);
        const uint32_t a = 0xFFFFFFFFu - (uint32_t)(best & 0xFFFFFFFFull);
        const uint32_t mn = ~S.d_nmin[hh];
        const float smax = key2f(k);
        // z = sum over tokens of exp((s - smax)/4); NaN when the fp64 sum was unusable
        const double sm4 = (double)smax * 0.25;
        const double z = (S.d_flags[hh] || sm4 > 600.0 || sm4 < -600.0) ? NAN : S.d_zabs[hh] * exp_wide(-sm4);
        int mode;
        uint32_t kstar = 0, tau_key = 0;
        const int topk = P.topk;
        if (topk > 0) {
            if (topk >= L) {
                mode = MODE_ALL;
                kstar = (uint32_t)L;
                tau_key = mn;
            } else if (topk == 1) {
                mode = MODE_TOP1;
                kstar = 1;
                tau_key = k;
            } else {
                mode = MODE_RADIX;
            }
        } else if (!(pb > 0.f)) {
            mode = MODE_SKIP;
            set_status(P, ST_DEVICE_INPUT);
        } else if (pb >= 1.f) {
            mode = MODE_ALL;
            kstar = (uint32_t)L;
            tau_key = mn;
        } else if (z == z && 1.0 >= (double)pb * z * (1.0 + 1e-3)) {
            mode = MODE_TOP1;   // the best token alone reaches p
            kstar = 1;
            tau_key = k;
        } else {
            mode = MODE_RADIX;
        }
        HeadState* hs = P.hs + (int64_t)b * P.n_ret + slot;
        if (mode == MODE_RADIX) {
            // the exact select's state; its first pass bins smax - s into 255
            // bins over [0, dr), dr large enough that the tokens beyond it
            // cannot hold the last 1 - p of the mass (otherwise the select
            // continues in the overflow bin), and no wider than the scores'
            // own spread (a little more, so the lowest score lands in bin 254
            // at most): concentrated scores then spread over all the bins
            HeadState h;
            h.mode = mode;
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
            h.tie_idx = 0xFFFFFFFFu;
            h.kstar = 0;
            float dr = 400.f;   // top-k: the k-th score may lie anywhere in the range
            if (topk == 0) {
                const float omp = fmaxf(1.f - pb, 1e-6f);
                const float zz = (z == z && z >= 1.0) ? (float)fmin(z, 1e30) : 1.f;
                dr = 4.f * (__logf((float)L) - __logf(omp) - __logf(zz)) + 8.f;
                dr = fminf(fmaxf(dr, 8.f), 400.f);
            }
            const float range = smax - key2f(mn);
            if (range >= 0.f) dr = fminf(dr, range + fmaxf(range * 0x1p-10f, 1e-6f));
            h.dr = dr;
            h.inv_w = 255.f / dr;
            h.bstar = 0;
            h.n_cand = 0;
            *hs = h;
        } else {
            hs->mode = mode;   // (read by the select of a group that has radix heads too)
        }
        const int bh = b * P.Hq + S.tab.slot_head[slot];
        if (P.dbg_smax) P.dbg_smax[bh] = smax;
        if (P.dbg_Z) P.dbg_Z[bh] = z;
        if (mode != MODE_RADIX) {
            if (P.dbg_tau) P.dbg_tau[bh] = key2f(tau_key);
            if (P.dbg_kstar) P.dbg_kstar[bh] = (int32_t)kstar;
            if (P.dbg_kept) P.dbg_kept[bh] = mode == MODE_TOP1 ? 1 : (mode == MODE_ALL ? nblk : 0);
        }
        S.d_mode[hh] = mode;
        S.d_arg[hh] = a;
    }
    consumer_sync();
    if (tid == 0) trace_max(P, 44);
    {
        // the common case first: every head keeps its best token only
        bool top1 = true;
        for (int hh = 0; hh < nh; ++hh) top1 = top1 && S.d_mode[hh] == MODE_TOP1;
        top1 = top1 && P.dbg_bitmap == nullptr;
        if (top1) {
            if (tid == 0) best_token_list<G>(P, S, b, rg, L, nh, slot0, g);
            return;
        }
    }
    bool any_radix = false, any_all = false;
    uint32_t all_mask = 0;
    for (int hh = 0; hh < nh; ++hh) {
        any_radix |= S.d_mode[hh] == MODE_RADIX;
        if (S.d_mode[hh] == MODE_ALL) {
            any_all = true;
            all_mask |= 1u << (S.tab.slot_head[slot0 + hh] - g * P.G);
        }
    }
    const int bg = b * P.n_rg + rg;
    // bitmap words of the heads (read by the block-list builder of a group
    // with radix heads, and by the debug sink)
    if (any_radix || P.dbg_bitmap != nullptr) {
        for (int hh = 0; hh < nh; ++hh) {
            const int mode = S.d_mode[hh];
            const int slot = slot0 + hh;
            for (int w = tid; w < nwords; w += CONSUMERS) {
                uint32_t word = 0;
                if (mode == MODE_ALL) {
                    const int nb = min(32, nblk - w * 32);
                    word = nb >= 32 ? 0xFFFFFFFFu : ((1u << nb) - 1u);
                } else if (mode == MODE_TOP1) {
                    const int j = (int)(S.d_arg[hh] / BLK) - w * 32;
                    if (j >= 0 && j < 32) word = 1u << j;
                }
                if (any_radix) P.bitmap[((int64_t)b * P.n_ret + slot) * P.words_cap + w] = word;
                if (P.dbg_bitmap && mode != MODE_RADIX)
                    P.dbg_bitmap[((int64_t)b * P.Hq + S.tab.slot_head[slot]) * P.words_cap + w] = word;
            }
        }
    }
    if (any_radix) {
        consumer_sync();
        if (tid == 0) {
            P.bcount[bg] = 0;
            for (int hh = 0; hh < nh; ++hh)
                if (S.d_mode[hh] == MODE_RADIX) {
                    const uint32_t kx = atomicAdd(&P.sync->n_radix_heads, 1u);
                    P.rlist[kx] = ((uint32_t)b << 16) | (uint32_t)(slot0 + hh);
                }
            atomicAdd(&P.sync->kb_work, 1u);
        }
        return;
    }
    // every head final: the group's block list (ascending block ids, head masks)
    uint32_t* list = P.blist + (int64_t)bg * P.nblk_cap;
    if (any_all) {
        for (int j = tid; j < nblk; j += CONSUMERS) {
            uint32_t hm = all_mask;
            for (int hh = 0; hh < nh; ++hh)
                if (S.d_mode[hh] == MODE_TOP1 && (int)(S.d_arg[hh] / BLK) == j)
                    hm |= 1u << (S.tab.slot_head[slot0 + hh] - g * P.G);
            list[j] = ((uint32_t)j << 8) | hm;
        }
        if (tid == 0) {
            P.bcount[bg] = (uint32_t)nblk;
            atomicAdd(&P.sync->kb_work, 1u);
        }
    } else {
        // only best-token blocks: the distinct argmax blocks, ascending, are
        // attended by this CTA after its share (the first such group of the
        // CTA; a later one goes to the retrieval kernel)
        if (tid == 0) best_token_list<G>(P, S, b, rg, L, nh, slot0, g);
    }
}

// The decision of one group, then the count of decided groups (the single
// launch waits for all of them before it either leaves or goes on to the
// retrieval phase).
template <int G>
__device__ __forceinline__ void decide_group(const KParams& K, ASmem<G>& S, int b, int rg, int L, float pb, int tid) {
    decide_group_body<G>(K, S, b, rg, L, pb, tid);
    consumer_sync();
    if (tid == 0) {
        __threadfence();
        atomicAdd(&K.P.sync->n_decided, 1u);
    }
}

// ---------------------------------------------------------------------------
// index-score splits (consumers)
// ---------------------------------------------------------------------------
// Running statistics of the two heads a lane owns: max score m, sum of
// exp((s - m)/4), best score and its lowest index, min score (only when the
// sequence keeps every token, p >= 1, where it is the threshold).
struct ScoreFold {
    float m[2], s[2], bv[2], mn[2];
    uint32_t bi[2];
    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            m[j] = -INFINITY;
            s[j] = 0.f;
            bv[j] = -INFINITY;
            mn[j] = INFINITY;
            bi[j] = 0xFFFFFFFFu;
        }
    }
};

// Which scores a lane folds.  The MMA leaves lane (g, t) rows g and g+8 of
// heads 2t, 2t+1.  With at most four heads (NH4) lanes t = 2, 3 would idle,
// so they take over row g+8 of lanes t-2: then lane (g, t) folds row
// g + 8*(t/2) of heads 2*(t%2), +1 and every lane folds one row per group.
template <bool NH4>
__device__ __forceinline__ int fold_head(int t, int j) {
    return NH4 ? 2 * (t & 1) + j : 2 * t + j;
}

// Fold one staged tile of k_idx rows (tokens n0 ..; rows >= nvalid are not
// tokens unless FULL) into f.  Warp w takes the 16-row groups w, w+4, ...,
// four at a time (independent MMA chains).
template <bool NH4, bool FULL>
__device__ __forceinline__ void score_tile(uint32_t tile, int n0, int nvalid, int nh, bool track_min, const QFrag& q,
                                           ScoreFold& f, float* sbase, int ncap, int warp, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const int ng = FULL ? SROWS / 16 : (nvalid + 15) / 16;
    constexpr float C = 0.25f * 1.4426950408889634f;   // (1/4) log2(e)
    constexpr int NV = NH4 ? 4 : 8;                     // values per head and iteration
#pragma unroll 1
    for (int base = warp; base < ng; base += 16) {
        float c[4][4];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) score16(tile, FULL ? base + 4 * q4 : min(base + 4 * q4, ng - 1), lane, q, c[q4]);
        if (NH4) {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const float x0 = __shfl_xor_sync(0xffffffffu, c[q4][2], 2);
                const float x1 = __shfl_xor_sync(0xffffffffu, c[q4][3], 2);
                if (t >= 2) {
                    c[q4][0] = x0;
                    c[q4][1] = x1;
                }
            }
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            if (fold_head<NH4>(t, j) >= nh) continue;
            float v[NV];
            uint32_t rr[NV];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
                for (int h = 0; h < NV / 4; ++h) {
                    const int e = q4 * (NV / 4) + h;
                    const int r = (base + 4 * q4) * 16 + g + 8 * (NH4 ? (t >> 1) : h);
                    rr[e] = (uint32_t)r;
                    const float x = NH4 ? c[q4][j] : c[q4][j + 2 * h];
                    v[e] = (FULL || r < nvalid) ? x : -INFINITY;
                    // kept for the exact select (L2-resident until it is read or dropped)
                    if (FULL || r < nvalid) sbase[(int64_t)fold_head<NH4>(t, j) * ncap + n0 + r] = x;
                }
            float mb = v[0];
#pragma unroll
            for (int e = 1; e < NV; ++e) mb = fmaxf(mb, v[e]);
#pragma unroll
            for (int e = 0; e < NV; ++e) {
                const bool gt = v[e] > f.bv[j];
                f.bv[j] = gt ? v[e] : f.bv[j];
                f.bi[j] = gt ? (uint32_t)n0 + rr[e] : f.bi[j];
            }
            if (track_min) {
                float vm = INFINITY;
#pragma unroll
                for (int e = 0; e < NV; ++e) vm = fminf(vm, v[e] == -INFINITY ? INFINITY : v[e]);
                f.mn[j] = fminf(f.mn[j], vm);
            }
            // rescale and add in one step (branch-free; 2^0 = 1 when the max holds)
            const float mn_ = fmaxf(f.m[j], mb);
            const float mc = (mn_ == -INFINITY) ? 0.f : mn_ * C;
            float add = f.s[j] * ex2_approx(fmaf(f.m[j], C, -mc));
#pragma unroll
            for (int e = 0; e < NV; ++e) add += ex2_approx(fmaf(v[e], C, -mc));
            f.s[j] = add;
            f.m[j] = mn_;
        }
    }
}

// (m, s) pairs: s relative to exp(m/4); m = -inf marks an empty pair
__device__ __forceinline__ void fold_pair(float& m, float& s, float m2, float s2) {
    constexpr float C = 0.25f * 1.4426950408889634f;
    if (m2 == -INFINITY) return;
    if (m == -INFINITY) {
        m = m2;
        s = s2;
        return;
    }
    const float M = fmaxf(m, m2);
    s = s * ex2_approx((m - M) * C) + s2 * ex2_approx((m2 - M) * C);
    m = M;
}

// End of a score split: reduce over the CTA, fold into the heads' buckets.
template <int G, bool NH4>
__device__ __forceinline__ void score_split_end(const Params& P, ASmem<G>& S, const ScoreFold& f0, int b, int rg,
                                                int bucket, int tid) {
    const int nh = S.tab.rg_nh[rg], slot0 = S.tab.rg_slot0[rg];
    const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    ScoreFold f = f0;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        // lanes folding the same heads: equal t (equal t % 2 with NH4)
#pragma unroll
        for (int o = NH4 ? 2 : 4; o < 32; o <<= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, f.m[j], o);
            const float s2 = __shfl_xor_sync(0xffffffffu, f.s[j], o);
            const float bv2 = __shfl_xor_sync(0xffffffffu, f.bv[j], o);
            const uint32_t bi2 = __shfl_xor_sync(0xffffffffu, f.bi[j], o);
            f.mn[j] = fminf(f.mn[j], __shfl_xor_sync(0xffffffffu, f.mn[j], o));
            fold_pair(f.m[j], f.s[j], m2, s2);
            if (bv2 > f.bv[j] || (bv2 == f.bv[j] && bi2 < f.bi[j])) {
                f.bv[j] = bv2;
                f.bi[j] = bi2;
            }
        }
        const int hh = fold_head<NH4>(t, j);
        if (g == 0 && (!NH4 || t < 2) && hh < nh) {
            S.w_m[warp][hh] = f.m[j];
            S.w_s[warp][hh] = f.s[j];
            S.w_bv[warp][hh] = f.bv[j];
            S.w_bi[warp][hh] = f.bi[j];
            S.w_mn[warp][hh] = f.mn[j];
        }
    }
    consumer_sync();
    if (tid < nh) {
        const int hh = tid;
        float m = -INFINITY, s = 0.f, bv = -INFINITY, mn = INFINITY;
        uint32_t bi = 0xFFFFFFFFu;
        for (int w = 0; w < 4; ++w) {
            fold_pair(m, s, S.w_m[w][hh], S.w_s[w][hh]);
            if (S.w_bv[w][hh] > bv || (S.w_bv[w][hh] == bv && S.w_bi[w][hh] < bi)) {
                bv = S.w_bv[w][hh];
                bi = S.w_bi[w][hh];
            }
            mn = fminf(mn, S.w_mn[w][hh]);
        }
        // fire-and-forget fold into the bucket; the exp-sum as the fp64 sum of
        // exp(s/4) (outside fp64's safe range the head takes the exact select)
        HeadAgg* ag = P.agg + ((int64_t)b * P.n_ret + slot0 + hh) * AGG_BUCKETS + (bucket % AGG_BUCKETS);
        if (bi != 0xFFFFFFFFu) {
            atomicMax(&ag->best, ((unsigned long long)f2key(bv) << 32) | (0xFFFFFFFFu - bi));
            atomicMax(&ag->nmin, ~f2key(mn));
        }
        if (m != -INFINITY) {
            const double m4 = (double)m * 0.25;
            if (m4 > 600.0 || m4 < -600.0) atomicOr(&ag->flags, 1u);
            else atomicAdd(&ag->zabs, (double)s * exp_wide(m4));
        }
    }
}

// ---------------------------------------------------------------------------
// the copy warp
// ---------------------------------------------------------------------------
template <int G>
__device__ __forceinline__ void a_producer(const KParams& K, ASmem<G>& S, AWalk wk, const int* pre_s, const int* pre_l,
                                           int lane) {
    constexpr int NST = ASmem<G>::NST;
    const Params& P = K.P;
    uint32_t k = 0;
    bool alive = true;
    bool extra = false;
    for (Seg sg = wk.next(P, pre_s, pre_l, S.tot_s);; sg = extra ? Seg{-1} : wk.next(P, pre_s, pre_l, S.tot_s)) {
        if (sg.type < 0 || !alive) {
            // share (or one more round) issued: meet the compute warps, then
            // issue the best-token blocks their group decision left in d_list,
            // until a round leaves none
            extra = true;
            asm volatile("bar.sync 3, 160;" ::: "memory");
            if (!alive || S.d_cnt == 0) break;
            sg = best_token_seg(S);
        }
        const int g = sg.type == 0 ? S.tab.rg_group[sg.grp] : (sg.type == 1 ? S.tab.lg_group[sg.grp] : S.tab.rg_group[sg.grp]);
        const LocalGeom lg = local_geom(P, sg.L);
        // the first tile of the share waits until the compute warps' query
        // loads are issued: those few lines then reach this SM ahead of the
        // 32 KB tile, not behind the whole grid's first burst
        if (k == 0 && sg.type != 2) asm volatile("bar.sync 4, 160;" ::: "memory");
        for (int i = 0; i < sg.ntiles; ++i, ++k) {
            const int st = (int)(k % NST);
            const uint32_t round = k / NST;
            if (lane == 0 && round > 0 && !mbar_wait_bounded(&S.empty[st], (round - 1) & 1u)) {
                set_status(P, ST_TIMEOUT);
                alive = false;
            }
            // the second tile waits for the first to land: every CTA's first
            // tile then arrives within ~10 MB of requests, not ~30 MB
            if (lane == 0 && k == 1 && alive && !mbar_wait_bounded(&S.full[0], 0u)) {
                set_status(P, ST_TIMEOUT);
                alive = false;
            }
            alive = __shfl_sync(0xffffffffu, alive ? 1 : 0, 0) != 0;
            if (!alive) break;
            uint8_t* dst = &S.stage[st][0];
            const int ti = sg.first + i;
            if (sg.type == 0) {
                const int n0 = ti * SROWS, nvalid = min(SROWS, sg.L - n0);
                if (P.block_table == nullptr) {
                    if (lane == 0) {
                        mbar_expect_tx(&S.full[st], (uint32_t)nvalid * R * 2);
                        bulk_g2s(dst, P.k_idx + (((int64_t)sg.b * P.Hkv + g) * P.Ncap + n0) * R, (uint32_t)nvalid * R * 2,
                                 &S.full[st]);
                    }
                } else {
                    const int np = (nvalid + BLK - 1) / BLK;
                    if (lane == 0) mbar_expect_tx(&S.full[st], (uint32_t)np * BLK * R * 2);
                    __syncwarp();
                    for (int q = lane; q < np; q += 32)
                        bulk_g2s(dst + q * BLK * R * 2, P.k_idx + block_row(P, sg.b, g, n0 / BLK + q) * R, BLK * R * 2,
                                 &S.full[st]);
                }
            } else if (lane == 0) {
                const int j = sg.type == 1 ? (ti < lg.nA ? ti : lg.bw0 + (ti - lg.nA)) : (int)(S.d_list[ti] >> 8);
                // local groups without retrieval heads may keep only a ring of
                // their sink and window (the tiles' position masks stay as they are)
                const bool ring = sg.type == 1 && ((P.ring_lg_mask >> sg.grp) & 1ull);
                const int row = ring ? (int)ring_block_row(P, sg.b, g, j) : (int)block_row(P, sg.b, g, j);
                const CUtensorMap* mk = ring ? &K.tmk_r : &K.tmk;
                const CUtensorMap* mv = ring ? &K.tmv_r : &K.tmv;
                mbar_expect_tx(&S.full[st], STAGE_BYTES);
                tma_load_2d(dst, mk, 0, row, &S.full[st]);
                tma_load_2d(dst + 8192, mk, 64, row, &S.full[st]);
                tma_load_2d(dst + KV_TILE, mv, 0, row, &S.full[st]);
                tma_load_2d(dst + KV_TILE + 8192, mv, 64, row, &S.full[st]);
            }
            __syncwarp();
        }
    }
    // never leave the CTA with copies in flight: wait (bounded) for the last
    // tile issued into each stage to land, then tell the compute warps
    if (lane == 0)
        for (uint32_t i = (k > (uint32_t)NST ? k - NST : 0u); i < k; ++i)
            mbar_wait_bounded(&S.full[i % NST], (i / NST) & 1u);
}

// ---------------------------------------------------------------------------
// the compute warps
// ---------------------------------------------------------------------------
template <int G>
__device__ __forceinline__ void a_consumers(const KParams& K, ASmem<G>& S, AWalk wk, const int* pre_s,
                                            const int* pre_l, int tid) {
    constexpr int NST = ASmem<G>::NST;
    const Params& P = K.P;
    const int warp = tid >> 5, lane = tid & 31;
    uint32_t k = 0;
    int q_tag = -1;
    QFrag qf;
    Attn<G> attn;
    attn.init(attn_q_smem<G>(S.X, warp));
    Acct ac;
    ac.init(P, S.acct, tid == 0);
    bool first_data = true;
    bool first_seg = true;   // its query loads release the copy warp's first tile (barrier 4)
    bool extra = false;
    for (Seg sg = wk.next(P, pre_s, pre_l, S.tot_s);; sg = extra ? Seg{-1} : wk.next(P, pre_s, pre_l, S.tot_s)) {
        if (sg.type < 0) {
            // share done (or one more round of it): meet the copy warp; the
            // best-token blocks of a group this CTA decided (left in d_list)
            // follow through the ring as one more segment, and the rounds
            // end when none are left
            extra = true;
            asm volatile("bar.sync 3, 160;" ::: "memory");
            if (S.d_cnt == 0) break;
            sg = best_token_seg(S);
        }
        if (sg.type == 0) {
            // ---- index scores of (b, retrieval group): q_idx while the first tile is in flight
            const int nh = S.tab.rg_nh[sg.grp];
            const int tag = sg.item_idx;
            if (tag != q_tag) {
                q_tag = tag;
                compute_qidx(P, S.tab, S.qi, sg.b, sg.grp, tid, first_seg);
                first_seg = false;
                consumer_sync();
                qf = make_qfrag(S.qi, nh, lane);
                consumer_sync();
            }
            ScoreFold f;
            f.reset();
            const bool nh4 = nh <= 4;
            const float pb = P.p ? __ldg(P.p + sg.b) : 1.f;   // (no p under static top-k)
            const bool track_min = true;   // (the threshold when p >= 1; the select's bin range otherwise)
            ac.mark(21);
            for (int i = 0; i < sg.ntiles; ++i, ++k) {
                const int st = (int)(k % NST);
                if (!mbar_wait_bounded(&S.full[st], (k / NST) & 1u)) {
                    // release the copy warp's next round barrier with no
                    // blocks left, so that it stops too
                    set_status(P, ST_TIMEOUT);
                    S.d_cnt = 0;
                    asm volatile("bar.arrive 3, 160;" ::: "memory");
                    return;
                }
                ac.mark(16);
                if (first_data && tid == 0) trace_max(P, 22);
                first_data = false;
                const int n0 = (sg.first + i) * SROWS, nvalid = min(SROWS, sg.L - n0);
                const uint32_t tile = smem_u32(&S.stage[st][0]);
                float* sbase = P.scores + ((int64_t)sg.b * P.n_ret + S.tab.rg_slot0[sg.grp]) * P.sstride;
                if (nvalid == SROWS) {
                    if (nh4) score_tile<true, true>(tile, n0, nvalid, nh, track_min, qf, f, sbase, P.sstride, warp, lane);
                    else score_tile<false, true>(tile, n0, nvalid, nh, track_min, qf, f, sbase, P.sstride, warp, lane);
                } else {
                    if (nh4) score_tile<true, false>(tile, n0, nvalid, nh, track_min, qf, f, sbase, P.sstride, warp, lane);
                    else score_tile<false, false>(tile, n0, nvalid, nh, track_min, qf, f, sbase, P.sstride, warp, lane);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.empty[st]);
                ac.mark(17);
                ac.count(19);
            }
            if (nh4) score_split_end<G, true>(P, S, f, sg.b, sg.grp, sg.first, tid);
            else score_split_end<G, false>(P, S, f, sg.b, sg.grp, sg.first, tid);
            if (tid == 0) trace_max(P, 47);
            const bool won =
                ticket_add(P.tick_score + sg.item_idx, (uint32_t)sg.ntiles, (uint32_t)sg.item_tiles, &S.flag);
            if (tid == 0) trace_max(P, 46);
            if (won) {
                if (tid == 0) trace_max(P, 6);
                decide_group<G>(K, S, sg.b, sg.grp, sg.L, pb, tid);
                consumer_sync();
                if (tid == 0) trace_max(P, 1);
            }
            ac.mark(28);
        } else {
            // ---- attention: local heads of (b, local group) over sink + window
            // blocks (type 1), or the best-token blocks this CTA selected for
            // (b, retrieval group) (type 2), through the same code
            const bool local = sg.type == 1;
            const int g = local ? S.tab.lg_group[sg.grp] : S.tab.rg_group[sg.grp];
            const uint32_t heads = local ? S.tab.lg_mask[sg.grp] : S.tab.rg_mask[sg.grp];
            const LocalGeom lg = local_geom(P, sg.L);
            attn.begin(P, sg.b, g, lane, first_seg && sg.type == 1);
            first_seg = false;
            ac.mark(29);
            for (int i = 0; i < sg.ntiles; ++i, ++k) {
                const int st = (int)(k % NST);
                if (!mbar_wait_bounded(&S.full[st], (k / NST) & 1u)) {
                    // release the copy warp's next round barrier with no
                    // blocks left, so that it stops too
                    set_status(P, ST_TIMEOUT);
                    S.d_cnt = 0;
                    asm volatile("bar.arrive 3, 160;" ::: "memory");
                    return;
                }
                ac.mark(16);
                if (first_data && tid == 0) trace_max(P, 22);
                first_data = false;
                const int ti = sg.first + i;
                int j;
                uint32_t hm;
                if (local) {
                    j = ti < lg.nA ? ti : lg.bw0 + (ti - lg.nA);
                    hm = heads;
                } else {
                    j = (int)(S.d_list[ti] >> 8);
                    hm = S.d_list[ti] & 0xFFu;
                }
                const uint32_t base = smem_u32(&S.stage[st][0]);
                const bool zeroed = attn.tile(base, base + KV_TILE, warp, lane, j * BLK, min(BLK, sg.L - j * BLK), hm,
                                              local, lg.s_end, lg.w_lo);
                if (zeroed) fence_proxy_async();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.empty[st]);
                ac.mark(18);
                ac.count(20);
            }
            attn.finish(S.X, warp, lane);
            consumer_sync();
            uint16_t* out0 = P.out + ((int64_t)sg.b * P.Hq + g * G) * D;
            if (sg.ntiles == sg.item_tiles) {
                split_emit<G>(S.X, heads, nullptr, out0, tid);
                consumer_sync();
                if (tid == 0) {
                    if (sg.type == 2) S.d_cnt = 0;   // this round's blocks are done
                    trace_max(P, local ? 2 : 4);
                }
                consumer_sync();
            } else {
                const int c = (int)blockIdx.x;
                float* part = P.lpart + ((int64_t)c + sg.item_idx) * G * PSTRIDE;
                split_emit<G>(S.X, heads, part, nullptr, tid);
                if (ticket_add(P.tick_local + sg.item_idx, (uint32_t)sg.ntiles, (uint32_t)sg.item_tiles, &S.flag)) {
                    const int c0 = cta_of_wtile(S.tot_s + sg.item_t0, S.tot_s, S.tot_l, S.nact);
                    const int c1 = cta_of_wtile(S.tot_s + sg.item_t0 + sg.item_tiles - 1, S.tot_s, S.tot_l, S.nact);
                    combine_splits<G>(S.X, P.lpart + ((int64_t)c0 + sg.item_idx) * G * PSTRIDE, c1 - c0 + 1, heads,
                                      out0, tid);
                    if (tid == 0) trace_max(P, 2);
                }
            }
            ac.mark(30);
        }
    }
    if (tid == 0) {
        trace_max(P, 23);
        acct_flush(P, S.acct);
    }
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
// The streaming phase.  SINGLE: part of the single launch (no dependent
// grid to release; every thread returns here, the copy warp included).
template <int G, bool SINGLE>
__device__ __forceinline__ void s_body(const KParams& K) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];   // no static shared memory: the base is aligned
    ASmem<G>& S = *reinterpret_cast<ASmem<G>*>(smem_raw);
    constexpr int NST = ASmem<G>::NST;
    const Params& P = K.P;
    const int tid = threadIdx.x;
    // the 128-byte-swizzled TMA boxes need 1024-byte aligned stages: refuse
    // (status RTP_ERR_CUDA) rather than copy into a misaligned ring
    if (smem_u32(smem_raw) & 1023u) {
        if (tid == 0) set_status(P, 5u);
        return;
    }
    int* pre_s = S.pre;
    int* pre_l = S.pre + (P.B + 1);
    if (tid >= CONSUMERS) {
        // the queries and the retrieval heads' indexer projections into L2
        // first (every CTA a few 128-byte lines), ahead of the tile traffic
        const int lane = tid - CONSUMERS;
        const int nw = P.n_ret * (R * D * 2 / 128), nq = P.B * P.n_ret * 2, nr = P.B * P.Hq * 2;
        for (int x = (int)blockIdx.x * 32 + lane; x < nw + nq + nr; x += (int)gridDim.x * 32) {
            const char* a;
            if (x < nw) {
                a = reinterpret_cast<const char*>(P.Wq + (int64_t)P.tab.slot_head[x / 32] * R * D) + (x % 32) * 128;
            } else if (x < nw + nq) {
                const int y = x - nw, bs = y >> 1;
                a = reinterpret_cast<const char*>(P.q_pre + ((int64_t)(bs / P.n_ret) * P.Hq +
                                                             P.tab.slot_head[bs % P.n_ret]) * D) + (y & 1) * 128;
            } else {
                a = reinterpret_cast<const char*>(P.q_rope) + (int64_t)(x - nw - nq) * 128;
            }
            prefetch_l2(a);
        }
    }
    if (tid == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(&S.full[i], 1);
            mbar_init(&S.empty[i], CONSUMERS / 32);
        }
        mbar_fence_init();
        if (P.dbg_trace) atomicCAS(P.dbg_trace, 0ull, (unsigned long long)global_ns());
        S.d_cnt = 0;
        for (int i = 0; i < ACCT_SLOTS; ++i) S.acct[i] = 0ull;
    }
    // the retrieval kernel may be scheduled now; it waits for this grid's
    // completion before it reads anything this grid writes
    if constexpr (!SINGLE) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (tid >= 32) copy_tab(P.tab, S.tab, tid - 32, THREADS - 32);
    // tiles per sequence (score tiles of all retrieval groups, then local
    // tiles of all local groups), prefix-summed by warp 0
    if (tid < 32) {
        int run_s = 0, run_l = 0, nvalid = 0;
        for (int b0 = 0; b0 < P.B; b0 += 32) {
            const int b = b0 + tid;
            int ns = 0, nl = 0;
            bool okb = false;
            if (b < P.B) {
                const int L = __ldg(P.seq_lens + b);
                okb = seq_ok(P, L);
                if (okb) {
                    ns = P.n_rg * ((L + SROWS - 1) / SROWS);
                    nl = P.n_lg ? P.n_lg * local_geom(P, L).nv : 0;
                } else if (blockIdx.x == 0) {
                    // an invalid length: no outputs for this sequence, no blocks
                    set_status(P, ST_DEVICE_INPUT);
                    for (int rg = 0; rg < P.n_rg; ++rg) P.bcount[b * P.n_rg + rg] = 0;
                }
            }
            int is = ns, il = nl;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int a = __shfl_up_sync(0xffffffffu, is, o);
                const int c = __shfl_up_sync(0xffffffffu, il, o);
                if (tid >= o) {
                    is += a;
                    il += c;
                }
            }
            if (b < P.B) {
                pre_s[b] = run_s + is - ns;
                pre_l[b] = run_l + il - nl;
            }
            run_s += __shfl_sync(0xffffffffu, is, 31);
            run_l += __shfl_sync(0xffffffffu, il, 31);
            nvalid += __popc(__ballot_sync(0xffffffffu, okb));
        }
        if (tid == 0) {
            S.n_vgroups = nvalid * P.n_rg;
            pre_s[P.B] = run_s;
            pre_l[P.B] = run_l;
            S.tot_s = run_s;
            S.tot_l = run_l;
        }
    }
    __syncthreads();
    // every CTA takes a contiguous share of equal weight of the step's tiles
    // (index tiles of all retrieval groups first, then the local tiles)
    AWalk wk;
    int nact;
    cta_wshare(S.tot_s, S.tot_l, wk.t, wk.t1, nact);
    wk.l0 = wk.l1 = 0;
    if (tid == 0) {
        S.nact = nact;
        trace_max(P, 7);
    }
    __syncthreads();
    if (tid >= CONSUMERS) {
        a_producer<G>(K, S, wk, pre_s, pre_l, tid - CONSUMERS);
        return;
    }
    a_consumers<G>(K, S, wk, pre_s, pre_l, tid);
    if (tid == 0) trace_max(P, 5);
}

template <int G>
__global__ void __launch_bounds__(THREADS, 2) stream_kernel(const __grid_constant__ KParams K) {
    s_body<G, false>(K);
}

}  // namespace rtp
