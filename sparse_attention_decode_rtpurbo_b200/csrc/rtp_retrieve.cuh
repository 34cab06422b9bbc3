// Retrieval kernel of the decode step (sm_100a), launched after the
// streaming kernel:
//   1. (only when some head needs it) the exact top-p select: an MSD radix
//      select over the order-preserving u32 keys of the fp32 index scores,
//      four passes of 256 bins of count and 2^-40 fixed-point softmax mass,
//      scores recomputed from the index cache on the tensor cores; then the
//      threshold ties (lowest indices first), block marking and the groups'
//      block lists.  Passes are separated by grid barriers: the grid is one
//      resident wave and no CTA of it depends on work that is not already
//      running (the streaming kernel it follows never waits on it).
//   2. block-sparse attention of the retrieval heads over their groups'
//      block lists, split evenly over the CTAs (TMA-staged K/V, tensor
//      cores), and the log-sum-exp combine of the splits.
//
// Sources: "Full Attention Strikes Back" (RTPurbo) review on
// dongryeollee1.github.io, Method: "Adaptive sparse attention" (S_h(m) =
// Top-P(s_h(m,.), p); exact attention over S_h(m)) and "Hardware-aware top-p
// decoding kernel" (sort-free threshold from histograms of softmax mass,
// block mask, block-sparse decoding with a cross-split reduce); aitrends.kr
// summary, items 2 and 5.
#pragma once
#include "rtp_stream.cuh"

namespace rtp {

struct RDesc {
    int32_t type;   // 0 = K/V tile, 1 = stop
    int32_t b, rg, n0, nvalid;
    uint32_t hmask;
    int32_t flags;        // bit 0: first tile of the CTA's split of the group, bit 1: last
    int32_t seg_tiles;    // tiles of this split
    int32_t item_tiles;   // tiles (blocks) of the group
    int32_t c0, nsplits;  // first CTA holding a split of the group, number of splits
};

template <int G>
struct BSmem {
    static constexpr int NST = 2;
    alignas(1024) uint8_t stage[NST][STAGE_BYTES];
    AttnScratch<G> X;
    alignas(16) float qi[MAX_G][R];
    uint32_t hcnt[G][256];
    uint32_t hm[G][3][256];   // 17-bit slices of the per-bin fixed-point mass
    unsigned long long dmass[256];
    uint32_t dcnt[256];
    uint32_t tmask[MAX_G];
    uint32_t tcnt[MAX_G];
    uint8_t tflag[SROWS];
    RDesc desc[NST];
    alignas(8) uint64_t full[NST], empty[NST];
    uint32_t flag, gen, abort, base;
    int kept[MAX_G];
    uint32_t wsum[4];
    int pre[2];   // really [max(B * n_rg, 1) + 1]: tiles before group i (radix groups, then all groups)
};

template <int G>
constexpr size_t bsmem_bytes(int ngroups) {
    return sizeof(BSmem<G>) + sizeof(int) * (size_t)(ngroups + 1) + 1024;
}

__device__ __forceinline__ bool wait_counter(const uint32_t* p, uint32_t target) {
    if (ld_acquire(p) >= target) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        __nanosleep(64);
        if (ld_acquire(p) >= target) return true;
        if (global_ns() - t0 > 2000000000ull) return false;
    }
}

// Grid-wide barrier (all threads of every CTA).  Bounded: after about two
// seconds it records RTP_ERR_TIMEOUT and the CTA abandons the call.
template <typename SM>
__device__ __forceinline__ bool grid_sync(const Params& P, SM& S) {
    __syncthreads();
    if (threadIdx.x == 0) {
        S.gen += 1;
        __threadfence();
        atomicAdd(&P.sync->barrier, 1u);
        if (!wait_counter(&P.sync->barrier, S.gen * gridDim.x)) {
            set_status(P, ST_TIMEOUT);
            S.abort = 1;
        }
        __threadfence();
    }
    __syncthreads();
    return S.abort == 0;
}

// (b, group) of radix group i
__device__ __forceinline__ void radix_group(const Params& P, int i, int& b, int& rg) {
    const uint32_t e = __ldcg(P.rglist + i);
    b = (int)(e >> 16);
    rg = (int)(e & 0xFFFFu);
}

// ---------------------------------------------------------------------------
// index tiles of the radix groups: a walk shared by the copy warp and the
// compute warps (CTA c takes tiles [c*T/grid, (c+1)*T/grid))
// ---------------------------------------------------------------------------
struct RSeg {
    int gi, b, rg, L, first, ntiles;
};
struct RWalk {
    int t, t1, ngr;
    __device__ __forceinline__ bool next(const Params& P, const int* pre, RSeg& s) {
        if (t >= t1) return false;
        s.gi = last_le(pre, ngr + 1, t);
        radix_group(P, s.gi, s.b, s.rg);
        s.L = __ldg(P.seq_lens + s.b);
        const int nt = pre[s.gi + 1] - pre[s.gi];
        s.first = t - pre[s.gi];
        s.ntiles = min(nt - s.first, t1 - t);
        t += s.ntiles;
        return true;
    }
};

// The copy warp's part of a pass over the radix groups' index tiles.
template <int G>
__device__ __noinline__ void r_produce_index(const Params& P, BSmem<G>& S, RWalk wk, const int* pre, uint32_t& k,
                                               int lane) {
    constexpr int NST = BSmem<G>::NST;
    RSeg sg;
    while (wk.next(P, pre, sg)) {
        const int g = P.rg_group[sg.rg];
        for (int i = 0; i < sg.ntiles; ++i, ++k) {
            const int st = (int)(k % NST);
            const uint32_t round = k / NST;
            bool ok = true;
            if (lane == 0 && round > 0 && !mbar_wait_bounded(&S.empty[st], (round - 1) & 1u)) {
                set_status(P, ST_TIMEOUT);
                ok = false;
            }
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
                S.abort = 1;
                return;
            }
            uint8_t* dst = &S.stage[st][0];
            const int n0 = (sg.first + i) * SROWS, nvalid = min(SROWS, sg.L - n0);
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
            __syncwarp();
        }
    }
}

// Per-lane view of the radix state of the two heads (2t, 2t+1) a lane owns.
struct RHeads {
    bool on[2];
    uint32_t prefix[2], tau[2], tie_idx[2];
    float smax[2];
};

__device__ __forceinline__ RHeads load_rheads(const Params& P, int b, int rg, int lane) {
    const int nh = P.rg_nh[rg], slot0 = P.rg_slot0[rg], t = lane & 3;
    RHeads r;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int hh = 2 * t + j;
        r.on[j] = false;
        r.prefix[j] = r.tau[j] = 0u;
        r.tie_idx[j] = 0xFFFFFFFFu;
        r.smax[j] = 0.f;
        if (hh < nh) {
            const HeadState* h = P.hs + (int64_t)b * P.n_ret + slot0 + hh;
            r.on[j] = __ldcg(&h->mode) == MODE_RADIX;
            r.prefix[j] = __ldcg(&h->prefix);
            r.tau[j] = __ldcg(&h->tau_key);
            r.tie_idx[j] = __ldcg(&h->tie_idx);
            r.smax[j] = __ldcg(&h->smax);
        }
    }
    return r;
}

// What a compute pass does with every (row, owned head) score of a tile.
enum RPass : int { RP_HIST0 = 0, RP_HIST1, RP_HIST2, RP_HIST3, RP_TIES, RP_MARK };

// The compute warps' part of a pass over the radix groups' index tiles.
template <int G>
__device__ __noinline__ void r_consume_index(const Params& P, BSmem<G>& S, RWalk wk, const int* pre, uint32_t& k,
                                               int pass, int tid) {
    constexpr int NST = BSmem<G>::NST;
    const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    RSeg sg;
    Acct ac;
    ac.init(P, tid == 0);
    while (wk.next(P, pre, sg)) {
        const int nh = P.rg_nh[sg.rg], slot0 = P.rg_slot0[sg.rg];
        compute_qidx(P, S.qi, sg.b, sg.rg, tid);
        for (int x = tid; x < G * 256; x += CONSUMERS) {
            (&S.hcnt[0][0])[x] = 0;
            (&S.hm[0][0][0])[x] = 0;
            (&S.hm[0][0][0])[x + G * 256] = 0;
            (&S.hm[0][0][0])[x + 2 * G * 256] = 0;
        }
        if (tid < MAX_G) {
            S.tmask[tid] = 0;
            S.tcnt[tid] = 0;
        }
        consumer_sync();
        const QFrag qf = make_qfrag(S.qi, nh, lane);
        const RHeads rh = load_rheads(P, sg.b, sg.rg, lane);
        const int shift = pass <= RP_HIST3 ? 24 - 8 * pass : 0;
        for (int i = 0; i < sg.ntiles; ++i, ++k) {
            const int st = (int)(k % NST);
            ac.mark(27);
            if (!mbar_wait_bounded(&S.full[st], (k / NST) & 1u)) {
                set_status(P, ST_TIMEOUT);
                S.abort = 1;
                return;
            }
            ac.mark(26);
            const int tile = sg.first + i;
            const int n0 = tile * SROWS, nvalid = min(SROWS, sg.L - n0);
            const int ng = (nvalid + 15) / 16;
            const uint32_t base = smem_u32(&S.stage[st][0]);
            uint32_t bits[2] = {0u, 0u};
            uint32_t cnt[2] = {0u, 0u};
#pragma unroll 1
            for (int grp = warp; grp < ng; grp += 4) {
                float c[4];
                score16(base, grp, lane, qf, c);
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int r = grp * 16 + g + 8 * h;
                        const bool on = rh.on[j] && r < nvalid;
                        const uint32_t key = f2key(c[j + 2 * h]);
                        if (pass <= RP_HIST3) {
                            const bool valid = on && (pass == 0 || (key >> (32 - 8 * pass)) == rh.prefix[j]);
                            const uint32_t d = (key >> shift) & 255u;
                            const uint32_t mv = valid ? ((uint32_t)(2 * t + j) << 8 | d) : 0xFFFFFFFFu;
                            const uint32_t peers = __match_any_sync(0xffffffffu, mv);
                            if (valid) {
                                const unsigned long long ms = fixmass(key, rh.smax[j]);
                                const uint32_t s0 = __reduce_add_sync(peers, (uint32_t)(ms & 0x1FFFFull));
                                const uint32_t s1 = __reduce_add_sync(peers, (uint32_t)((ms >> 17) & 0x1FFFFull));
                                const uint32_t s2 = __reduce_add_sync(peers, (uint32_t)(ms >> 34));
                                if (lane == __ffs(peers) - 1) {
                                    const int hh = 2 * t + j;
                                    atomicAdd(&S.hcnt[hh][d], (uint32_t)__popc(peers));
                                    atomicAdd(&S.hm[hh][0][d], s0);
                                    atomicAdd(&S.hm[hh][1][d], s1);
                                    atomicAdd(&S.hm[hh][2][d], s2);
                                }
                            }
                        } else if (pass == RP_TIES) {
                            cnt[j] += (on && key == rh.tau[j]) ? 1u : 0u;
                        } else {
                            const bool keep = on && (key > rh.tau[j] ||
                                                     (key == rh.tau[j] && (uint32_t)(n0 + r) <= rh.tie_idx[j]));
                            if (keep) bits[j] |= 1u << (grp >> 2);
                        }
                    }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.empty[st]);
            ac.mark(24);
            ac.count(25);
            if (pass == RP_TIES || pass == RP_MARK) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
#pragma unroll
                    for (int o = 4; o < 32; o <<= 1) {
                        bits[j] |= __shfl_xor_sync(0xffffffffu, bits[j], o);
                        cnt[j] += __shfl_xor_sync(0xffffffffu, cnt[j], o);
                    }
                    if (g == 0 && 2 * t + j < nh) {
                        if (bits[j]) atomicOr(&S.tmask[2 * t + j], bits[j]);
                        if (cnt[j]) atomicAdd(&S.tcnt[2 * t + j], cnt[j]);
                    }
                }
                consumer_sync();
                if (tid < nh) {
                    const int64_t bs = (int64_t)sg.b * P.n_ret + slot0 + tid;
                    if (pass == RP_TIES) {
                        P.tie_cnt[bs * P.ntiles_cap + tile] = S.tcnt[tid];
                    } else if (S.tmask[tid]) {
                        atomicOr(P.bitmap + bs * P.words_cap + tile / 2, S.tmask[tid] << ((tile & 1) * 16));
                    }
                    S.tmask[tid] = 0;
                    S.tcnt[tid] = 0;
                }
                consumer_sync();
            }
        }
        if (pass <= RP_HIST3) {
            // this split's histograms -> the heads' global histograms
            consumer_sync();
            for (int x = tid; x < nh * 256; x += CONSUMERS) {
                const int hh = x >> 8, d = x & 255;
                const uint32_t c = S.hcnt[hh][d];
                if (c) {
                    const int64_t bs = (int64_t)sg.b * P.n_ret + slot0 + hh;
                    const unsigned long long ms = (unsigned long long)S.hm[hh][0][d] +
                                                  ((unsigned long long)S.hm[hh][1][d] << 17) +
                                                  ((unsigned long long)S.hm[hh][2][d] << 34);
                    atomicAdd(P.hist_cnt + bs * 256 + d, c);
                    atomicAdd(P.hist_mass + bs * 256 + d, ms);
                }
            }
            consumer_sync();
        }
    }
}

// ---------------------------------------------------------------------------
// per-head steps between the passes (one CTA per radix head)
// ---------------------------------------------------------------------------
// Pick the digit of pass `pass` for radix head `hx`: the largest digit d whose
// bins >= d hold at least the target mass (over the tokens above the prefix).
template <int G>
__device__ __noinline__ void r_digit(const Params& P, BSmem<G>& S, int hx, int pass, int tid) {
    const uint32_t e = __ldcg(P.rlist + hx);
    const int b = (int)(e >> 16), slot = (int)(e & 0xFFFFu);
    const int64_t bs = (int64_t)b * P.n_ret + slot;
    uint32_t* gcnt = P.hist_cnt + bs * 256;
    unsigned long long* gmass = P.hist_mass + bs * 256;
    for (int d = tid; d < 256; d += CONSUMERS) {
        S.dcnt[d] = __ldcg(gcnt + d);
        S.dmass[d] = __ldcg(gmass + d);
        gcnt[d] = 0;
        gmass[d] = 0ull;
    }
    consumer_sync();
    if (tid == 0) {
        HeadState st = P.hs[bs];
        if (pass == 0) {
            unsigned long long z = 0;
            for (int d = 0; d < 256; ++d) z += S.dmass[d];
            const double pb = (double)__ldg(P.p + b);
            unsigned long long tg = (unsigned long long)ceil(pb * (double)z);
            if (tg > z) tg = z;
            if (tg == 0) tg = 1;
            st.target = tg;
            st.mass_above = 0;
            st.count_above = 0;
            st.prefix = 0;
        }
        unsigned long long cum = st.mass_above;
        uint32_t cabove = st.count_above;
        int dstar = 0;
        for (int d = 255; d >= 0; --d) {
            if (cum + S.dmass[d] >= st.target) {
                dstar = d;
                break;
            }
            cum += S.dmass[d];
            cabove += S.dcnt[d];
        }
        st.mass_above = cum;
        st.count_above = cabove;
        st.prefix = (st.prefix << 8) | (uint32_t)dstar;
        if (pass == 3) {
            st.tau_key = st.prefix;
            st.n_eq = S.dcnt[dstar];
            const unsigned long long m_tau = st.n_eq ? S.dmass[dstar] / st.n_eq : 0ull;
            const unsigned long long need = st.target - st.mass_above;
            uint32_t nt = st.n_eq;
            if (m_tau > 0) {
                const unsigned long long q = (need + m_tau - 1) / m_tau;
                nt = (uint32_t)min((unsigned long long)st.n_eq, max(1ull, q));
            }
            st.n_tie = nt;
            st.all_ties = (nt == st.n_eq) ? 1u : 0u;
            st.tie_idx = 0xFFFFFFFFu;
            st.kstar = st.count_above + nt;
            const int bh = b * P.Hq + P.slot_head[slot];
            if (P.dbg_tau) P.dbg_tau[bh] = key2f(st.tau_key);
            if (P.dbg_kstar) P.dbg_kstar[bh] = (int32_t)st.kstar;
            if (!st.all_ties) atomicOr(&P.sync->any_ties, 1u);
        }
        P.hs[bs] = st;
    }
    consumer_sync();
}

// For a radix head that keeps only n_tie of its n_eq threshold ties: find the
// index of the n_tie-th tie in token order (per-tile counts, then a scan of
// the one tile that holds it, re-scored exactly as in the passes).
template <int G>
__device__ __noinline__ void r_tie_locate(const Params& P, BSmem<G>& S, int hx, int tid) {
    const uint32_t e = __ldcg(P.rlist + hx);
    const int b = (int)(e >> 16), slot = (int)(e & 0xFFFFu);
    const int64_t bs = (int64_t)b * P.n_ret + slot;
    if (__ldcg(&P.hs[bs].all_ties)) return;
    const int rg = P.slot_rg[slot], g = P.rg_group[rg], slot0 = P.rg_slot0[rg], nh = P.rg_nh[rg];
    const int hh = slot - slot0;
    const int L = __ldg(P.seq_lens + b);
    const int nt = (L + SROWS - 1) / SROWS;
    const uint32_t ntie = __ldcg(&P.hs[bs].n_tie), tau = __ldcg(&P.hs[bs].tau_key);
    if (tid == 0) {
        uint32_t cum = 0;
        int tile = nt - 1;
        for (int i = 0; i < nt; ++i) {
            const uint32_t c = __ldcg(P.tie_cnt + bs * P.ntiles_cap + i);
            if (cum + c >= ntie) {
                tile = i;
                break;
            }
            cum += c;
        }
        S.base = (uint32_t)tile;
        S.flag = ntie - cum;   // rank (1-based) of the wanted tie inside that tile
    }
    consumer_sync();
    const int tile = (int)S.base;
    const uint32_t rank = S.flag;
    const int n0 = tile * SROWS, nvalid = min(SROWS, L - n0);
    // stage the tile's rows with plain loads (no copy is in flight between passes)
    uint8_t* rows = &S.stage[0][0];
    for (int x = tid; x < nvalid * 2; x += CONSUMERS) {
        const int r = x >> 1, half = x & 1;
        const int n = n0 + r;
        const int64_t row = block_row(P, b, g, n / BLK) + (n % BLK);
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(P.k_idx + row * R) + half);
        *reinterpret_cast<uint4*>(rows + r * 32 + half * 16) = v;
    }
    compute_qidx(P, S.qi, b, rg, tid);
    consumer_sync();
    const int warp = tid >> 5, lane = tid & 31, gl = lane >> 2, t = lane & 3;
    const QFrag qf = make_qfrag(S.qi, nh, lane);
    const int ng = (nvalid + 15) / 16;
    for (int grp = warp; grp < ng; grp += 4) {
        float c[4];
        score16(smem_u32(rows), grp, lane, qf, c);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int j = 0; j < 2; ++j)
                if (2 * t + j == hh) {
                    const int r = grp * 16 + gl + 8 * h;
                    S.tflag[r] = (r < nvalid && f2key(c[j + 2 * h]) == tau) ? 1 : 0;
                }
    }
    consumer_sync();
    if (warp == 0) {
        uint32_t cum = 0;
        int found = nvalid - 1;
        for (int r0 = 0; r0 < nvalid; r0 += 32) {
            const int r = r0 + lane;
            const uint32_t bal = __ballot_sync(0xffffffffu, r < nvalid && S.tflag[r]);
            const uint32_t c = __popc(bal);
            if (cum + c >= rank) {
                // the (rank - cum)-th set bit
                uint32_t m = bal;
                for (uint32_t q = 1; q < rank - cum; ++q) m &= m - 1;
                found = r0 + __ffs(m) - 1;
                break;
            }
            cum += c;
        }
        if (lane == 0) P.hs[bs].tie_idx = (uint32_t)(n0 + found);
    }
    consumer_sync();
}

// Block list of radix group i: union of its heads' block bitmaps, in
// ascending block order, with the mask of heads that read each block.
template <int G>
__device__ __noinline__ void r_blist(const Params& P, BSmem<G>& S, int i, int tid) {
    int b, rg;
    radix_group(P, i, b, rg);
    const int L = __ldg(P.seq_lens + b);
    const int g = P.rg_group[rg], nh = P.rg_nh[rg], slot0 = P.rg_slot0[rg];
    const int nblk = (L + BLK - 1) / BLK;
    const int nwords = (nblk + 31) / 32;
    const int bg = b * P.n_rg + rg;
    uint32_t* list = P.blist + (int64_t)bg * P.nblk_cap;
    const int warp = tid >> 5, lane = tid & 31;
    if (tid < MAX_G) S.kept[tid] = 0;
    if (tid == 0) S.base = 0;
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
                if (wh[hh]) atomicAdd(&S.kept[hh], __popc(wh[hh]));
                if (P.dbg_bitmap)
                    P.dbg_bitmap[((int64_t)b * P.Hq + P.slot_head[slot0 + hh]) * P.words_cap + w] = wh[hh];
            }
        }
        const uint32_t c = __popc(uni);
        uint32_t incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += x;
        }
        if (lane == 31) S.wsum[warp] = incl;
        consumer_sync();
        uint32_t off = S.base;
        for (int ww = 0; ww < warp; ++ww) off += S.wsum[ww];
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
        if (tid == 0) S.base += S.wsum[0] + S.wsum[1] + S.wsum[2] + S.wsum[3];
        consumer_sync();
    }
    if (tid < nh && P.dbg_kept) {
        const int slot = slot0 + tid;
        if (__ldcg(&P.hs[(int64_t)b * P.n_ret + slot].mode) == MODE_RADIX)
            P.dbg_kept[b * P.Hq + P.slot_head[slot]] = S.kept[tid];
    }
    if (tid == 0) P.bcount[bg] = S.base;
    consumer_sync();
}

// ---------------------------------------------------------------------------
// block-sparse attention of the retrieval heads
// ---------------------------------------------------------------------------
// The copy warp walks this CTA's share [t, t1) of all groups' block-list
// tiles (pre[gi] = tiles before group gi), publishing one descriptor per
// tile and a stop descriptor at the end.
template <int G>
__device__ __forceinline__ void r_produce_attn(const KParams& K, BSmem<G>& S, const int* pre, int ngroups, int t,
                                              int t1, long long T, int nact, uint32_t& k, int lane) {
    constexpr int NST = BSmem<G>::NST;
    const Params& P = K.P;
    auto acquire = [&](int st, uint32_t round) -> bool {
        bool ok = true;
        if (lane == 0 && round > 0 && !mbar_wait_bounded(&S.empty[st], (round - 1) & 1u)) {
            set_status(P, ST_TIMEOUT);
            ok = false;
        }
        return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    };
    int gi = t < t1 ? last_le(pre, ngroups + 1, t) : 0;
    while (t < t1) {
        while (pre[gi + 1] <= t) ++gi;
        const int cnt = pre[gi + 1] - pre[gi];
        const int b = gi / P.n_rg, rg = gi % P.n_rg, g = P.rg_group[rg];
        const int L = __ldg(P.seq_lens + b);
        const int first = t - pre[gi];
        const int nseg = min(cnt - first, t1 - t);
        const int c0 = cta_of_tile(pre[gi], T, nact);
        const int c1 = cta_of_tile(pre[gi] + cnt - 1, T, nact);
        const uint32_t* list = P.blist + (int64_t)gi * P.nblk_cap;
        for (int i0 = 0; i0 < nseg; i0 += 32) {
            // 32 list entries per round of loads
            const uint32_t mine = (i0 + lane < nseg) ? __ldcg(list + first + i0 + lane) : 0u;
            const int nr = min(32, nseg - i0);
            for (int ii = 0; ii < nr; ++ii, ++k) {
                const uint32_t e = __shfl_sync(0xffffffffu, mine, ii);
                const int st = (int)(k % NST);
                if (!acquire(st, k / NST)) {
                    S.abort = 1;
                    return;
                }
                if (lane == 0) {
                    const int i = i0 + ii;
                    const int j = (int)(e >> 8);
                    RDesc d;
                    d.type = 0;
                    d.b = b;
                    d.rg = rg;
                    d.n0 = j * BLK;
                    d.nvalid = min(BLK, L - j * BLK);
                    d.hmask = e & 0xFFu;
                    d.flags = (i == 0 ? 1 : 0) | (i == nseg - 1 ? 2 : 0);
                    d.seg_tiles = nseg;
                    d.item_tiles = cnt;
                    d.c0 = c0;
                    d.nsplits = c1 - c0 + 1;
                    S.desc[st] = d;
                    const int row = (int)block_row(P, b, g, j);
                    uint8_t* dst = &S.stage[st][0];
                    mbar_expect_tx(&S.full[st], STAGE_BYTES);
                    tma_load_2d(dst, &K.tmk, 0, row, &S.full[st]);
                    tma_load_2d(dst + 8192, &K.tmk, 64, row, &S.full[st]);
                    tma_load_2d(dst + KV_TILE, &K.tmv, 0, row, &S.full[st]);
                    tma_load_2d(dst + KV_TILE + 8192, &K.tmv, 64, row, &S.full[st]);
                }
                __syncwarp();
            }
        }
        t += nseg;
    }
    const int st = (int)(k % NST);
    if (!acquire(st, k / NST)) {
        S.abort = 1;
        return;
    }
    if (lane == 0) {
        S.desc[st].type = 1;
        mbar_arrive(&S.full[st]);
    }
    ++k;
    // never leave the CTA with copies in flight
    if (lane == 0)
        for (uint32_t i = (k > (uint32_t)NST ? k - NST : 0u); i < k; ++i)
            mbar_wait_bounded(&S.full[i % NST], (i / NST) & 1u);
}

template <int G>
__device__ __forceinline__ void r_consume_attn(const KParams& K, BSmem<G>& S, uint32_t& k, int tid) {
    constexpr int NST = BSmem<G>::NST;
    const Params& P = K.P;
    const int warp = tid >> 5, lane = tid & 31;
    MmaAttn<G> attn;
    attn.init();
    while (true) {
        const int st = (int)(k % NST);
        if (!mbar_wait_bounded(&S.full[st], (k / NST) & 1u)) {
            set_status(P, ST_TIMEOUT);
            return;
        }
        ++k;
        const RDesc d = S.desc[st];
        if (d.type != 0) break;
        const int g = P.rg_group[d.rg];
        if (d.flags & 1) attn.begin(P, d.b, g, lane);
        const uint32_t base = smem_u32(&S.stage[st][0]);
        const bool zeroed = attn.tile(base, base + KV_TILE, warp, lane, d.n0, d.nvalid, d.hmask, false, 0, 0);
        if (zeroed) fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[st]);
        if (d.flags & 2) {
            attn.finish(S.X, warp, lane);
            consumer_sync();
            const uint32_t heads = P.rg_mask[d.rg];
            const int gi = d.b * P.n_rg + d.rg;
            uint16_t* out0 = P.out + ((int64_t)d.b * P.Hq + g * G) * D;
            if (d.seg_tiles == d.item_tiles) {
                split_emit<G>(S.X, heads, nullptr, out0, tid);
                consumer_sync();
            } else {
                float* part = P.rpart + ((int64_t)blockIdx.x + gi) * G * PSTRIDE;
                split_emit<G>(S.X, heads, part, nullptr, tid);
                if (ticket_add(P.tick_ret + gi, (uint32_t)d.seg_tiles, (uint32_t)d.item_tiles, &S.flag)) {
                    __threadfence();
                    combine_splits<G>(S.X, P.rpart + ((int64_t)d.c0 + gi) * G * PSTRIDE, d.nsplits, heads, out0, tid);
                }
            }
        }
    }
}

// Warp-0 prefix over `n` counts given by cnt(i): pre[i] = sum of cnt(0..i-1).
template <typename F>
__device__ __forceinline__ void warp_prefix(int* pre, int n, F cnt, int lane) {
    int run = 0;
    for (int i0 = 0; i0 < n; i0 += 32) {
        const int i = i0 + lane;
        const int c = i < n ? cnt(i) : 0;
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int a = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += a;
        }
        if (i < n) pre[i] = run + incl - c;
        run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) pre[n] = run;
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
template <int G>
__global__ void __launch_bounds__(THREADS, 1) retrieve_kernel(const __grid_constant__ KParams K) {
    extern __shared__ uint8_t smem_raw[];
    BSmem<G>& S = *reinterpret_cast<BSmem<G>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    constexpr int NST = BSmem<G>::NST;
    const Params& P = K.P;
    const int tid = threadIdx.x, lane = tid & 31;
    const bool copier = tid >= CONSUMERS;
    int* pre = S.pre;
    if (tid == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(&S.full[i], 1);
            mbar_init(&S.empty[i], CONSUMERS / 32);
        }
        mbar_fence_init();
        S.gen = 0;
        S.abort = 0;
    }
    // everything below reads the selection results of the streaming kernel,
    // which may still be streaming local heads: wait for every group's
    // decision (written before the count, with a fence)
    if (tid == 0 && !wait_counter(&P.sync->groups_decided, (uint32_t)(P.B * P.n_rg))) {
        set_status(P, ST_TIMEOUT);
        S.abort = 1;
    }
    __syncthreads();
    if (tid == 0) trace_max(P, 13);
    uint32_t k = 0;
    bool ok = S.abort == 0;
    const uint32_t nrad = ok ? __ldcg(&P.sync->n_radix_heads) : 0u;
    if (nrad > 0) {
        // ---- exact select of the radix heads
        const int ngr = (int)__ldcg(&P.sync->n_radix_groups);
        if (tid < 32)
            warp_prefix(pre, ngr, [&](int i) {
                int b, rg;
                radix_group(P, i, b, rg);
                return (__ldg(P.seq_lens + b) + SROWS - 1) / SROWS;
            }, lane);
        __syncthreads();
        const long long T = pre[ngr];
        RWalk wk;
        wk.t = (int)((long long)blockIdx.x * T / gridDim.x);
        wk.t1 = (int)((long long)(blockIdx.x + 1) * T / gridDim.x);
        wk.ngr = ngr;
        for (int pass = 0; pass < 4 && ok; ++pass) {
            if (copier) {
                r_produce_index<G>(P, S, wk, pre, k, lane);
            } else {
                r_consume_index<G>(P, S, wk, pre, k, pass, tid);
            }
            ok = grid_sync(P, S);
            if (!ok) break;
            if (tid == 0 && pass == 0) trace_max(P, 14);
            if (!copier)
                for (int hx = blockIdx.x; hx < (int)nrad; hx += gridDim.x) r_digit<G>(P, S, hx, pass, tid);
            ok = grid_sync(P, S);
            if (tid == 0) trace_max(P, 8 + pass);
        }
        if (ok && __ldcg(&P.sync->any_ties)) {
            if (copier) r_produce_index<G>(P, S, wk, pre, k, lane);
            else r_consume_index<G>(P, S, wk, pre, k, RP_TIES, tid);
            ok = grid_sync(P, S);
            if (ok && !copier)
                for (int hx = blockIdx.x; hx < (int)nrad; hx += gridDim.x) r_tie_locate<G>(P, S, hx, tid);
            ok = ok && grid_sync(P, S);
        }
        if (ok) {
            if (copier) r_produce_index<G>(P, S, wk, pre, k, lane);
            else r_consume_index<G>(P, S, wk, pre, k, RP_MARK, tid);
            ok = grid_sync(P, S);
            if (tid == 0) trace_max(P, 12);
        }
        if (ok) {
            if (!copier)
                for (int i = blockIdx.x; i < ngr; i += gridDim.x) r_blist<G>(P, S, i, tid);
            ok = grid_sync(P, S);
        }
    }
    if (tid == 0) trace_max(P, 3);
    if (ok) {
        // ---- block-sparse attention over every group's block list
        const int ngroups = P.B * P.n_rg;
        if (tid < 32)
            warp_prefix(pre, ngroups, [&](int i) {
                return seq_ok(P, __ldg(P.seq_lens + i / P.n_rg)) ? (int)__ldcg(P.bcount + i) : 0;
            }, lane);
        __syncthreads();
        if (tid == 0) trace_max(P, 15);
        const long long T = pre[ngroups];
        int t0, t1, nact;
        cta_share(T, t0, t1, nact);
        if (copier) r_produce_attn<G>(K, S, pre, ngroups, t0, t1, T, nact, k, lane);
        else r_consume_attn<G>(K, S, k, tid);
        if (tid == 0) trace_max(P, 4);
    }
    // the last CTA out clears the call's coordination words
    __syncthreads();
    if (tid == 0) {
        trace_max(P, 5);
        __threadfence();
        if (atomicAdd(&P.sync->exit_count, 1u) == gridDim.x - 1) {
            P.sync->n_radix_heads = 0;
            P.sync->n_radix_groups = 0;
            P.sync->any_ties = 0;
            P.sync->barrier = 0;
            P.sync->groups_decided = 0;
            P.sync->exit_count = 0;
            __threadfence();
        }
    }
}

}  // namespace rtp
