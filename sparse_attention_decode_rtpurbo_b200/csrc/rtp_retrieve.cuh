// Retrieval kernel of the decode step (sm_100a), launched after the
// streaming kernel (programmatic dependent launch; it waits for that grid):
//   1. (only when some head needs it) the exact top-p select over the fp32
//      index scores the streaming kernel stored, one CTA per head, with no
//      grid barrier between its steps: a first pass bins smax - s (255 bins,
//      count and 2^-40 fixed-point softmax mass, in shared memory), a 256-bin
//      search picks the bin that completes ceil(p Z), a second pass marks the
//      blocks of the tokens above that bin and gathers the bin's tokens, and
//      the CTA selects inside them (8-bit MSD digits over the
//      order-preserving u32 keys, ties toward the lowest index); a bin of
//      more than 4096 tokens takes four refine passes and a mark pass
//      instead.  The scores stream through the stage buffers in 16 KB bulk
//      copies.  The last head of a group (a ticket) builds the group's block
//      list.  One grid barrier then separates the select from the attention:
//      the grid is one resident wave (cooperative launch) and no CTA of it
//      depends on work that is not already running (the streaming kernel it
//      follows never waits on it).
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

// Select state of one radix head as the passes read it.
struct RHead {
    uint32_t prefix, tau, tie_idx, bstar, n_cand;
    float smax, dr, inv_w;
};

// Per-bin histogram of a select pass in shared memory (one head at a time): a
// count and the 2^-40 fixed-point mass held as three partial sums, of bits
// 0-15, 16-31 and 32 up of every token's mass (mass = m[0] + m[1] 2^16 +
// m[2] 2^32).  All four are 32-bit atomics, which the shared-memory units
// resolve without retries even when a warp's lanes collide; a partial sum
// cannot wrap while a bin gathers at most 65536 tokens between flushes.
template <int G>
struct RHist {
    uint32_t cnt[1][256];   // (one head at a time)
    uint32_t m[3][1][256];
};
constexpr int HIST_FLUSH_TOKENS = 65536;

template <int G>
__device__ __forceinline__ void hist_add(RHist<G>& H, int h, int d, uint32_t n, unsigned long long ms) {
    atomicAdd(&H.cnt[h][d], n);
    atomicAdd(&H.m[0][h][d], (uint32_t)(ms & 0xFFFFull));
    atomicAdd(&H.m[1][h][d], (uint32_t)((ms >> 16) & 0xFFFFull));
    atomicAdd(&H.m[2][h][d], (uint32_t)(ms >> 32));
}
// The mass alone (the spread first pass: its bin counts are not needed, the
// threshold bin's size and the count above it come from the compaction).
template <int G>
__device__ __forceinline__ void hist_add_mass(RHist<G>& H, int h, int d, unsigned long long ms) {
    atomicAdd(&H.m[0][h][d], (uint32_t)(ms & 0xFFFFull));
    atomicAdd(&H.m[1][h][d], (uint32_t)((ms >> 16) & 0xFFFFull));
    atomicAdd(&H.m[2][h][d], (uint32_t)(ms >> 32));
}
template <int G>
__device__ __forceinline__ unsigned long long hist_mass(const RHist<G>& H, int h, int d) {
    return (unsigned long long)H.m[0][h][d] + ((unsigned long long)H.m[1][h][d] << 16) +
           ((unsigned long long)H.m[2][h][d] << 32);
}

template <int G>
struct BSmem {
    static constexpr int NST = 2;   // attention ring stages of 32 KB (a third measured no faster)
    alignas(1024) uint8_t stage[NST][STAGE_BYTES];
    union {
        AttnScratch<G> X;   // attention phase
        RHist<G> H;         // select phase
    };
    alignas(16) float qi[MAX_G][R];
    unsigned long long dmass[256];
    uint32_t dcnt[256];
    uint32_t tcnt[MAX_G];
    uint32_t hcand;   // candidates gathered by a compaction pass of this CTA alone (or by the warp finish)
    uint32_t lw_key[32], lw_idx[32];   // the in-bin select's last bucket, finished by one warp
    uint32_t fin_tau, fin_tie;         // the in-bin select's result: tau and the largest tie index kept
    HeadState hst;    // the head's select state as this CTA's digit step computed it
    uint32_t lsel_prefix, lsel_count, lsel_neq;
    unsigned long long lsel_mass, lsel_meq;
    uint8_t tflag[SROWS];
    RDesc desc[NST];
    alignas(8) uint64_t full[NST], empty[NST];
    alignas(8) uint64_t hfull[2 * STAGE_BYTES / (SROWS * 4)];   // select passes: a 4 KB score copy has landed
    uint32_t flag, gen, abort, base;
    unsigned long long acct[ACCT_SLOTS];   // debug cycle sums of thread 0
    unsigned long long sc_k[4], hit_k;     // bin_search: per-warp key sums, key sum before the hit
    uint32_t sc_a[4], hit_a, hit_pos;      // bin_search: per-warp aux sums, aux sum before the hit, hit position
    int kept[MAX_G];
    uint32_t wsum[4];
    HeadTab tab;
    int pre[2];   // really [max(B * n_ret, 1) + 1]: units before radix head i, then tiles before group i
};

template <int G>
constexpr size_t bsmem_bytes(int ngroups) {
    return sizeof(BSmem<G>) + sizeof(int) * (size_t)(ngroups + 1) + 1024;
}

// The CTA's BSmem, 1024-byte aligned inside the dynamic shared memory.  It is
// derived by offset arithmetic on the shared array, so the compiler keeps it
// in the shared state space (native shared loads, stores and atomics) also in
// the helpers that are not inlined.
template <int G>
__device__ __forceinline__ BSmem<G>& bsmem() {
    extern __shared__ uint8_t rtp_dyn_smem[];
    const uint32_t pad = (1024u - (smem_u32(rtp_dyn_smem) & 1023u)) & 1023u;
    return *reinterpret_cast<BSmem<G>*>(rtp_dyn_smem + pad);
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

__device__ __forceinline__ RHead load_rhead(const HeadState* h) {
    RHead r;
    r.prefix = __ldcg(&h->prefix);
    r.tau = __ldcg(&h->tau_key);
    r.tie_idx = __ldcg(&h->tie_idx);
    r.bstar = __ldcg(&h->bstar);
    r.n_cand = __ldcg(&h->n_cand);
    r.smax = __ldcg(&h->smax);
    r.dr = __ldcg(&h->dr);
    r.inv_w = __ldcg(&h->inv_w);
    return r;
}

// First-pass bin of a score: 255 bins of width dr/255 over d = smax - s in
// [0, dr) (d >= 0: smax is the maximum of the same fp32 scores), bin 255 for
// d >= dr.  Every pass computes it with the same fp32 operations.
__device__ __forceinline__ uint32_t score_bin(float s, float smax, float dr, float inv_w) {
    const float d = smax - s;
    return d < dr ? (uint32_t)min((int)(d * inv_w), 254) : 255u;
}

// What a pass does with every stored score of the head:
// RP_BINS histograms the first-pass bins; RP_COMPACT marks the blocks of the
// tokens above the threshold bin and gathers the bin's tokens (when at most
// CAND_CAP) for the select inside the CTA; otherwise RP_REF0..3 histogram
// the next 8 key bits of the scores in the threshold bin that match the key
// prefix found so far, RP_TIES counts threshold ties per 1024-token tile and
// RP_MARK marks the blocks of the kept tokens.
enum RPass : int { RP_BINS = 0, RP_REF0, RP_REF1, RP_REF2, RP_REF3, RP_TIES, RP_MARK, RP_COMPACT };

// A head's stored scores stream through the two stage buffers as 4 KB bulk
// copies of one 1024-token tile each (sixteen in flight, issued by consumer
// thread 0); every pass of the select is one sweep over them, its
// histograms in shared memory.
constexpr int HS_CHUNK = SROWS;                               // scores per copy (4 KB)
constexpr int HS_SLOTS = 2 * STAGE_BYTES / (HS_CHUNK * 4);    // copies in flight
constexpr int HS_U = HS_CHUNK / CONSUMERS;                    // scores per thread and copy
constexpr int HS_FOLD = HIST_FLUSH_TOKENS / HS_CHUNK;         // copies between folds of the 32-bit partial sums

// The histogram's 32-bit partial sums (S.H, head 0) into the 64-bit ones
// (S.dcnt, S.dmass); every bin's partials back to zero.
template <int G>
__device__ __forceinline__ void h_fold(BSmem<G>& S, int tid) {
    consumer_sync();
    for (int d = tid; d < 256; d += CONSUMERS) {
        S.dcnt[d] += S.H.cnt[0][d];
        S.dmass[d] += hist_mass(S.H, 0, d);
        S.H.cnt[0][d] = 0;
        S.H.m[0][0][d] = 0;
        S.H.m[1][0][d] = 0;
        S.H.m[2][0][d] = 0;
    }
    consumer_sync();
}

// One pass over copies [c0, c1) of the stored scores of radix head (b, slot)
// by this CTA's consumer threads (thread tid takes scores tid + 128 u of every
// copy, so a warp's 32 scores lie in one 64-token block).  `unit`: the CTA
// holds one unit of a head shared by several CTAs, so the bins go to the
// head's global histogram and the candidates are reserved in the head's
// global count; otherwise the whole head is this CTA's.  `seq` counts the
// copies this CTA has waited for (it picks the slot and the barrier phase).
// A wait that gives up sets the status and S.abort; the pass then stops
// after waiting, bounded, for the copies it has in flight.
template <int G, int pass>
__device__ __noinline__ void h_pass(const Params& P, int b, int slot, const RHead rh, int c0, int c1, bool unit_of_many,
                                    uint32_t& seq, int tid) {
    BSmem<G>& S = bsmem<G>();
    const int lane = tid & 31, warp = tid >> 5;
    const int64_t bs = (int64_t)b * P.n_ret + slot;
    const int L = __ldg(P.seq_lens + b);
    const int nch = c1 - c0;
    const float* const src = P.scores + bs * P.sstride;
    uint8_t* const ring = &S.stage[0][0];
    const bool unit = P.topk > 0;   // static top-k: every token weighs 1 (the histograms count)
    constexpr int rp = pass - RP_REF0;
    // key bits above the refine pass's digit (the prefix found so far); unused in pass RP_REF0
    constexpr int psh = (pass > RP_REF0 && pass <= RP_REF3) ? 32 - 8 * (pass - RP_REF0) : 0;
    uint32_t* const bmp = P.bitmap + bs * P.words_cap;
    unsigned long long* const cand = P.cand + bs * CAND_CAP;
    auto issue = [&](int k) {   // copy c0 + k of the pass into its slot (thread 0)
        const uint32_t q = seq + (uint32_t)k, sl = q % HS_SLOTS;
        const int c = c0 + k;
        const int nv = min(HS_CHUNK, L - c * HS_CHUNK);
        const uint32_t bytes = (uint32_t)((nv + 3) & ~3) * 4u;   // whole 16-byte units inside the row
        mbar_expect_tx(&S.hfull[sl], bytes);
        bulk_g2s(ring + (size_t)sl * HS_CHUNK * 4, src + (size_t)c * HS_CHUNK, bytes, &S.hfull[sl]);
    };
    if constexpr (pass <= RP_REF3) {
        for (int d = tid; d < 256; d += CONSUMERS) {
            S.dcnt[d] = 0;
            S.dmass[d] = 0ull;
            S.H.cnt[0][d] = 0;
            S.H.m[0][0][d] = 0;
            S.H.m[1][0][d] = 0;
            S.H.m[2][0][d] = 0;
        }
    }
    if (tid < MAX_G) S.tcnt[tid] = 0;
    if (tid == 0) S.hcand = 0;
    consumer_sync();
    if (tid == 0)
        for (int c = 0; c < HS_SLOTS && c < nch; ++c) issue(c);
    uint32_t ovf_n = 0u;
    unsigned long long ovf_m = 0ull;
    int k = 0;
    for (; k < nch; ++k) {
        const uint32_t q = seq + (uint32_t)k, sl = q % HS_SLOTS;
        if (!mbar_wait_bounded(&S.hfull[sl], (q / HS_SLOTS) & 1u)) {
            set_status(P, ST_TIMEOUT);
            S.abort = 1;
        }
        const float* x = reinterpret_cast<const float*>(ring + (size_t)sl * HS_CHUNK * 4);
        const int c = c0 + k;
        const int n0 = c * HS_CHUNK, nv = min(HS_CHUNK, L - n0);
        uint32_t w0 = 0u;        // RP_COMPACT / RP_MARK: bits of blocks n0/64 + 0..15
        uint32_t n_above = 0u;   // RP_COMPACT: the warp's tokens above the threshold bin (lane 0)
        uint32_t tcount = 0u;    // RP_TIES: threshold ties of this thread in the tile
        uint32_t in_bin[HS_U];   // RP_COMPACT: the warp's ballots of tokens in the threshold bin
        // the thread's scores of the copy into registers first: the loads then
        // overlap, where the shared-memory atomics below would keep them in order
        float xv[HS_U];
#pragma unroll
        for (int u = 0; u < HS_U; ++u) xv[u] = x[tid + u * CONSUMERS];
#pragma unroll
        for (int u = 0; u < HS_U; ++u) {
            const int r = tid + u * CONSUMERS;
            const bool ok = r < nv;
            const float v = xv[u];
            const uint32_t key = f2key(v);
            if constexpr (pass == RP_BINS) {
                if (ok) {
                    const uint32_t bn = score_bin(v, rh.smax, rh.dr, rh.inv_w);
                    const unsigned long long ms = unit ? 1ull : fixmass(key, rh.smax);
                    if (bn < 255u) {
                        if (unit_of_many) hist_add_mass(S.H, 0, (int)bn, ms);
                        else hist_add(S.H, 0, (int)bn, 1u, ms);
                    } else {
                        ovf_n += 1u;
                        ovf_m += ms;
                    }
                }
            } else if constexpr (pass <= RP_REF3) {
                if (ok && score_bin(v, rh.smax, rh.dr, rh.inv_w) == rh.bstar && (rp == 0 || (key >> psh) == rh.prefix))
                    hist_add(S.H, 0, (int)((key >> (24 - 8 * rp)) & 255u), 1u, unit ? 1ull : fixmass(key, rh.smax));
            } else if constexpr (pass == RP_TIES) {
                tcount += (ok && key == rh.tau) ? 1u : 0u;
            } else {
                bool keep;
                if constexpr (pass == RP_COMPACT) {
                    const uint32_t bn = ok ? score_bin(v, rh.smax, rh.dr, rh.inv_w) : 256u;
                    keep = bn < rh.bstar;
                    in_bin[u] = __ballot_sync(0xffffffffu, bn == rh.bstar);
                } else {
                    keep = ok && (key > rh.tau || (key == rh.tau && (uint32_t)(n0 + r) <= rh.tie_idx));
                }
                // block of the warp's 32 scores within the tile: 2 u + warp / 2
                const uint32_t kb = __ballot_sync(0xffffffffu, keep);
                if (kb) w0 |= 1u << (2 * u + (warp >> 1));
                n_above += __popc(kb);
            }
        }
        if constexpr (pass == RP_COMPACT) {
            // the bin's tokens of the copy, in ballot order behind one
            // reservation per warp (a returning global atomic per 32 tokens
            // would put its round trip on the loop's path HS_U times)
            uint32_t tot = 0u;
#pragma unroll
            for (int u = 0; u < HS_U; ++u) tot += (uint32_t)__popc(in_bin[u]);
            if (tot) {
                uint32_t base = 0;
                if (lane == 0)
                    base = unit_of_many ? atomicAdd(P.sel_ncand + bs, tot) : atomicAdd(&S.hcand, tot);
                base = __shfl_sync(0xffffffffu, base, 0);
#pragma unroll
                for (int u = 0; u < HS_U; ++u) {
                    const uint32_t pos = base + (uint32_t)__popc(in_bin[u] & ((1u << lane) - 1u));
                    if (((in_bin[u] >> lane) & 1u) && pos < (uint32_t)CAND_CAP) {
                        const int r = tid + u * CONSUMERS;
                        cand[pos] = ((unsigned long long)f2key(xv[u]) << 32) | (uint32_t)(n0 + r);
                    }
                    base += (uint32_t)__popc(in_bin[u]);
                }
            }
        }
        if constexpr (pass == RP_COMPACT || pass == RP_MARK) {
            // the blocks straight into the head's bitmap (zeroed when the
            // group was registered for the select)
            if (lane == 0 && w0) atomicOr(bmp + c / 2, w0 << ((c & 1) * 16));
            if constexpr (pass == RP_COMPACT) {
                if (unit_of_many && lane == 0 && n_above) atomicAdd(P.sel_above + bs, n_above);
            }
        } else if constexpr (pass == RP_TIES) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) tcount += __shfl_xor_sync(0xffffffffu, tcount, o);
            if (lane == 0 && tcount) atomicAdd(&S.tcnt[k & 1], tcount);
        }
        consumer_sync();   // the slot is read (and this copy's tie counts are complete)
        if constexpr (pass == RP_TIES) {
            if (tid == 0) {
                P.tie_cnt[bs * P.ntiles_cap + c] = S.tcnt[k & 1];
                S.tcnt[k & 1] = 0;
            }
        }
        if (S.abort) break;   // (set before the barrier: every thread sees it)
        if (tid == 0 && k + HS_SLOTS < nch) issue(k + HS_SLOTS);
        if constexpr (pass <= RP_REF3) {
            if ((k + 1) % HS_FOLD == 0 && k + 1 < nch) h_fold(S, tid);
        }
    }
    if (k < nch) {
        // gave up: wait, bounded, for the copies still in flight, then stop
        for (int d = k + 1; d < nch && d <= k + HS_SLOTS - 1; ++d) {
            const uint32_t q = seq + (uint32_t)d;
            mbar_wait_bounded(&S.hfull[q % HS_SLOTS], (q / HS_SLOTS) & 1u);
        }
        consumer_sync();
        return;
    }
    seq += (uint32_t)nch;
    if constexpr (pass == RP_BINS) {
        // tokens beyond the binned range: bin 255
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            ovf_n += __shfl_xor_sync(0xffffffffu, ovf_n, o);
            ovf_m += __shfl_xor_sync(0xffffffffu, ovf_m, o);
        }
        if (lane == 0 && ovf_n) {
            atomicAdd(&S.H.cnt[0][255], ovf_n);
            atomicAdd(&S.dmass[255], ovf_m);
        }
    }
    if constexpr (pass <= RP_REF3) h_fold(S, tid);
    if constexpr (pass == RP_BINS) {
        if (unit_of_many) {
            // the unit's bins into the head's global histogram
            for (int d = tid; d < 256; d += CONSUMERS) {
                const uint32_t n = S.dcnt[d];
                const unsigned long long m = S.dmass[d];
                if (n) atomicAdd(P.sel_cnt + bs * 256 + d, n);
                if (m) atomicAdd(P.sel_mass + bs * 256 + d, m);
            }
        }
    }
    if constexpr (pass == RP_COMPACT || pass == RP_MARK || pass == RP_BINS)
        __threadfence();   // bitmap bits, candidates and bins before the head's and the group's tickets
    consumer_sync();
}

// ---------------------------------------------------------------------------
// steps between the passes (inside the head's CTA)
// ---------------------------------------------------------------------------
// Pick the digit of pass `pass` for radix head `hx`: the largest digit d whose
// bins >= d hold at least the target mass (over the tokens above the prefix).
// Search over 256 bins by the 128 compute threads (two walk positions
// each, warp scans, one cross-warp step): walking the bins from 255 down
// (desc) or from 0 up, the first position i whose inclusive key sum reaches
// `need`.  Leaves in shared memory the position (255 when none does), the
// key and aux sums of the positions before it (all positions when none
// does).  The bin of position i is 255 - i (desc) or i.
template <int G, typename KF, typename AF>
__device__ __forceinline__ void bin_search(BSmem<G>& S, KF key_of, AF aux_of, bool desc, unsigned long long need,
                                           int tid) {
    const int warp = tid >> 5, lane = tid & 31;
    const int i0 = 2 * tid;
    const int d0 = desc ? 255 - i0 : i0, d1 = desc ? 254 - i0 : i0 + 1;
    const unsigned long long k0 = key_of(d0), k1 = key_of(d1);
    const uint32_t a0 = aux_of(d0), a1 = aux_of(d1);
    unsigned long long ik = k0 + k1;
    uint32_t ia = a0 + a1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long xk = __shfl_up_sync(0xffffffffu, ik, o);
        const uint32_t xa = __shfl_up_sync(0xffffffffu, ia, o);
        if (lane >= o) {
            ik += xk;
            ia += xa;
        }
    }
    if (lane == 31) {
        S.sc_k[warp] = ik;
        S.sc_a[warp] = ia;
    }
    consumer_sync();
    unsigned long long ok_ = 0;
    uint32_t oa = 0;
    for (int w = 0; w < warp; ++w) {
        ok_ += S.sc_k[w];
        oa += S.sc_a[w];
    }
    if (tid == 0) {
        S.hit_pos = 255;
        S.hit_k = S.sc_k[0] + S.sc_k[1] + S.sc_k[2] + S.sc_k[3];
        S.hit_a = S.sc_a[0] + S.sc_a[1] + S.sc_a[2] + S.sc_a[3];
    }
    consumer_sync();
    const unsigned long long e0 = ok_ + ik - (k0 + k1), e1 = e0 + k0;
    const uint32_t f0 = oa + ia - (a0 + a1), f1 = f0 + a0;
    if (e0 + k0 >= need && (i0 == 0 || e0 < need)) {
        S.hit_pos = (uint32_t)i0;
        S.hit_k = e0;
        S.hit_a = f0;
    } else if (e1 + k1 >= need && e1 < need) {
        S.hit_pos = (uint32_t)i0 + 1;
        S.hit_k = e1;
        S.hit_a = f1;
    }
    consumer_sync();
}

// The threshold step after a pass: `publish` writes the head's new select
// state to the workspace (else it is only in S.hst, for this CTA).
template <int G, int pass>
__device__ __noinline__ void r_digit(const Params& P, int b, int slot, int tid, bool publish = true) {
    BSmem<G>& S = bsmem<G>();
    const int64_t bs = (int64_t)b * P.n_ret + slot;
    // (the pass's histogram is in S.dcnt / S.dmass)
    auto mass_of = [&](int d) { return S.dmass[d]; };
    auto cnt_of = [&](int d) { return S.dcnt[d]; };
    if constexpr (pass == RP_BINS) {
        // z = the total mass; bins ascend in smax - s: the first bin that
        // completes the target ceil(p z) (top-k: masses are counts, z = L,
        // and the target is k)
        bin_search(S, mass_of, cnt_of, false, ~0ull, tid);
        const unsigned long long z = S.hit_k;
        unsigned long long tg;
        if (P.topk > 0) {
            tg = (unsigned long long)P.topk;
        } else {
            const double pb = (double)__ldg(P.p + b);
            tg = (unsigned long long)ceil(pb * (double)z);
        }
        if (tg > z) tg = z;
        if (tg == 0) tg = 1;
        bin_search(S, mass_of, cnt_of, false, tg, tid);
        if (tid == 0) {
            HeadState st = P.hs[bs];
            st.target = tg;
            const uint32_t bstar = S.hit_pos;
            st.bstar = bstar;
            st.n_cand = S.dcnt[bstar];
            st.mass_above = S.hit_k;
            st.count_above = S.hit_a;
            st.prefix = 0;
            S.hst = st;
            if (publish) P.hs[bs] = st;
        }
        consumer_sync();
        return;
    }
    const unsigned long long tgt = __ldcg(&P.hs[bs].target), above = __ldcg(&P.hs[bs].mass_above);
    bin_search(S, mass_of, cnt_of, true, tgt > above ? tgt - above : 0ull, tid);
    if (tid == 0) {
        HeadState st = P.hs[bs];
        {
            const int rp = pass - RP_REF0;
            const int dstar = 255 - (int)S.hit_pos;
            const unsigned long long cum = st.mass_above + S.hit_k;
            const uint32_t cabove = st.count_above + S.hit_a;
            st.mass_above = cum;
            st.count_above = cabove;
            st.prefix = (st.prefix << 8) | (uint32_t)dstar;
            if (rp == 3) {
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
                const int bh = b * P.Hq + S.tab.slot_head[slot];
                if (P.dbg_tau) P.dbg_tau[bh] = key2f(st.tau_key);
                if (P.dbg_kstar) P.dbg_kstar[bh] = (int32_t)st.kstar;
            }
        }
        P.hs[bs] = st;
    }
    consumer_sync();
}

// Threshold of a radix head whose threshold bin holds at most CAND_CAP
// tokens, inside one CTA: the bin's (key, index) pairs, gathered by the
// compaction, are held in registers; 8-bit MSD passes over the keys (count
// and fixed-point mass per digit, cumulative from the mass above the bin)
// narrow them to the digit bucket that completes the target, one warp
// finishes a bucket of at most 32 (sorted by key desc, index asc), and only
// more than 32 exact ties take the four-pass select over the tie indices
// (ties toward the lower index).  The kept candidates' blocks then go into
// the head's bitmap.  CPT candidates per thread: an instance for at most
// 1024 candidates (8 per thread) and one for CAND_CAP; the smaller one is a
// quarter of the code, which matters for code that runs once per head and
// per step.
template <int G, int CPT>
__device__ __noinline__ void r_local_select(const Params& P, int b, int slot, int tid) {
    BSmem<G>& S = bsmem<G>();
    const int64_t bs = (int64_t)b * P.n_ret + slot;
    const uint32_t ncand = __ldcg(&P.hs[bs].n_cand);
    if (ncand > (uint32_t)(CPT * CONSUMERS)) return;
    const int n = (int)ncand;
    uint32_t keys[CPT], idx[CPT];
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
        const int i = tid + j * CONSUMERS;
        keys[j] = 0u;
        idx[j] = 0u;
        if (i < n) {
            const unsigned long long c = __ldcg(P.cand + bs * CAND_CAP + i);
            keys[j] = (uint32_t)(c >> 32);
            idx[j] = (uint32_t)(c & 0xFFFFFFFFull);
        }
    }
    // the leading digits every candidate shares (one threshold bin: often
    // one or two) need no pass
    uint32_t kand = 0xFFFFFFFFu, kor = 0u;
#pragma unroll
    for (int j = 0; j < CPT; ++j)
        if (tid + j * CONSUMERS < n) {
            kand &= keys[j];
            kor |= keys[j];
        }
    kand = __reduce_and_sync(0xffffffffu, kand);
    kor = __reduce_or_sync(0xffffffffu, kor);
    if ((tid & 31) == 0) {
        S.wsum[tid >> 5] = kand;
        S.tcnt[tid >> 5] = kor;
    }
    consumer_sync();
    kand = S.wsum[0] & S.wsum[1] & S.wsum[2] & S.wsum[3];
    kor = S.tcnt[0] | S.tcnt[1] | S.tcnt[2] | S.tcnt[3];
    const int rp0 = n > 0 ? min(__clz(kand ^ kor) / 8, 3) : 0;
    const float smax = __ldcg(&P.hs[bs].smax);
    consumer_sync();
    if (tid == 0) {
        S.lsel_prefix = rp0 > 0 ? kand >> (32 - 8 * rp0) : 0u;
        S.lsel_mass = __ldcg(&P.hs[bs].mass_above);
        S.lsel_count = __ldcg(&P.hs[bs].count_above);
    }
    const unsigned long long target = __ldcg(&P.hs[bs].target);
    const bool unit = P.topk > 0;   // static top-k: every token weighs 1
    // digits resolved when a bucket of at most 32 candidates is left: one warp
    // then finishes it (below); -1 while the digit rounds go on
    int depth = n <= 32 ? rp0 : -1;
    for (int rp = rp0; rp < 4 && depth < 0; ++rp) {
        for (int d = tid; d < 256; d += CONSUMERS) {
            S.H.cnt[0][d] = 0;
            S.H.m[0][0][d] = 0;
            S.H.m[1][0][d] = 0;
            S.H.m[2][0][d] = 0;
        }
        consumer_sync();
        const uint32_t prefix = S.lsel_prefix;
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            const uint32_t key = keys[j];
            if (tid + j * CONSUMERS >= n || (rp > 0 && (key >> (32 - 8 * rp)) != prefix)) continue;
            hist_add(S.H, 0, (int)((key >> (24 - 8 * rp)) & 255u), 1u, unit ? 1ull : fixmass(key, smax));
        }
        consumer_sync();
        // the highest digit whose mass completes the target (digits descend)
        const unsigned long long base = S.lsel_mass;
        bin_search(S, [&](int d) { return hist_mass(S.H, 0, d); }, [&](int d) { return S.H.cnt[0][d]; }, true,
                   target > base ? target - base : 0ull, tid);
        if (tid == 0) {
            const int dstar = 255 - (int)S.hit_pos;
            S.lsel_mass = base + S.hit_k;
            S.lsel_count += S.hit_a;
            S.lsel_prefix = (prefix << 8) | (uint32_t)dstar;
            S.lsel_neq = S.H.cnt[0][dstar];
            S.lsel_meq = hist_mass(S.H, 0, dstar);
        }
        consumer_sync();
        if (rp < 3 && S.lsel_neq <= 32u) depth = rp + 1;
    }
    auto publish = [&](uint32_t tau, uint32_t n_eq, uint32_t n_tie, uint32_t tie_idx, uint32_t count_above) {
        S.fin_tau = tau;
        S.fin_tie = tie_idx;
        HeadState* h = P.hs + bs;
        h->tau_key = tau;
        h->n_eq = n_eq;
        h->n_tie = n_tie;
        h->all_ties = n_tie == n_eq ? 1u : 0u;
        h->tie_idx = tie_idx;
        h->kstar = count_above + n_tie;
        const int bh = b * P.Hq + S.tab.slot_head[slot];
        if (P.dbg_tau) P.dbg_tau[bh] = key2f(tau);
        if (P.dbg_kstar) P.dbg_kstar[bh] = (int32_t)(count_above + n_tie);
    };
    // the blocks of the kept candidates (key above tau, or tau with an index up
    // to the largest tie kept) into the head's bitmap, from the registers
    auto mark_kept = [&]() {
        const uint32_t tau = S.fin_tau, tie = S.fin_tie;
        uint32_t* const bmp = P.bitmap + bs * P.words_cap;
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            if (tid + j * CONSUMERS >= n) continue;
            const uint32_t key = keys[j], x = idx[j];
            if (key > tau || (key == tau && x <= tie)) atomicOr(bmp + (x >> 11), 1u << ((x >> 6) & 31));
        }
        __threadfence();   // bitmap bits before the group ticket
        consumer_sync();
    };
    if (depth >= 0) {
        // The bucket (candidates that share the `depth` leading key bytes
        // found so far; it completes the target) in one warp: sorted by (key
        // desc, index asc), the order the select keeps tokens in, its masses
        // summed in that order; the first candidate that brings the mass above
        // the bucket to the target is the last one kept.
        const uint32_t prefix = S.lsel_prefix;
        if (tid == 0) S.hcand = 0;
        consumer_sync();
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            if (tid + j * CONSUMERS >= n || (depth > 0 && (keys[j] >> (32 - 8 * depth)) != prefix)) continue;
            const uint32_t pos = atomicAdd(&S.hcand, 1u);
            if (pos < 32u) {
                S.lw_key[pos] = keys[j];
                S.lw_idx[pos] = idx[j];
            }
        }
        consumer_sync();
        if (tid < 32) {
            const int lane = tid;
            const uint32_t m = min(S.hcand, 32u);
            bool v = (uint32_t)lane < m;
            uint32_t k = v ? S.lw_key[lane] : 0u, x = v ? S.lw_idx[lane] : 0xFFFFFFFFu;
            // bitonic sort over the 32 lanes; a valid entry precedes an empty one
#pragma unroll
            for (int kk = 2; kk <= 32; kk <<= 1) {
#pragma unroll
                for (int jj = kk >> 1; jj > 0; jj >>= 1) {
                    const uint32_t ok = __shfl_xor_sync(0xffffffffu, k, jj), ox = __shfl_xor_sync(0xffffffffu, x, jj);
                    const bool ov = __shfl_xor_sync(0xffffffffu, v ? 1 : 0, jj) != 0;
                    const bool self_first = v && (!ov || k > ok || (k == ok && x < ox));
                    const bool take_first = ((lane & jj) == 0) == ((lane & kk) == 0);
                    if (take_first ? !self_first : self_first) {
                        k = ok;
                        x = ox;
                        v = ov;
                    }
                }
            }
            unsigned long long inc = v ? (unit ? 1ull : fixmass(k, smax)) : 0ull;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned long long t = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += t;
            }
            const unsigned long long base = S.lsel_mass;
            const uint32_t hb = __ballot_sync(0xffffffffu, v && base + inc >= target);
            const int hit = hb ? __ffs(hb) - 1 : (int)m - 1;   // (the bucket completes the target)
            const uint32_t tau = __shfl_sync(0xffffffffu, k, hit), tie_x = __shfl_sync(0xffffffffu, x, hit);
            const uint32_t eq = __ballot_sync(0xffffffffu, v && k == tau);
            const uint32_t upto = hit == 31 ? 0xFFFFFFFFu : ((2u << hit) - 1u);
            const uint32_t n_eq = __popc(eq), n_tie = __popc(eq & upto);
            const uint32_t above = __popc(__ballot_sync(0xffffffffu, v && k > tau));
            if (lane == 0) publish(tau, n_eq, n_tie, n_tie == n_eq ? 0xFFFFFFFFu : tie_x, S.lsel_count + above);
        }
        consumer_sync();
        mark_kept();
        return;
    }
    const uint32_t tau = S.lsel_prefix, n_eq = S.lsel_neq, count_above = S.lsel_count;
    uint32_t n_tie = n_eq;
    {
        const unsigned long long m_tau = n_eq ? S.lsel_meq / n_eq : 0ull;
        const unsigned long long need = target - S.lsel_mass;
        if (m_tau > 0) {
            const unsigned long long q = (need + m_tau - 1) / m_tau;
            n_tie = (uint32_t)min((unsigned long long)n_eq, max(1ull, q));
        }
    }
    // the n_tie-th smallest index among the ties (only when some ties are left out)
    uint32_t tie_idx = 0xFFFFFFFFu;
    if (n_tie < n_eq) {
        if (tid == 0) {
            S.lsel_prefix = 0;
            S.lsel_count = n_tie;   // rank still wanted
        }
        for (int rp = 0; rp < 4; ++rp) {
            for (int d = tid; d < 256; d += CONSUMERS) S.H.cnt[0][d] = 0;
            consumer_sync();
            const uint32_t prefix = S.lsel_prefix;
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                if (tid + j * CONSUMERS >= n || keys[j] != tau) continue;
                const uint32_t x = idx[j];
                if (rp > 0 && (x >> (32 - 8 * rp)) != prefix) continue;
                atomicAdd(&S.H.cnt[0][(x >> (24 - 8 * rp)) & 255u], 1u);
            }
            consumer_sync();
            // the lowest index digit that reaches the wanted rank
            const uint32_t rank = S.lsel_count;
            bin_search(S, [&](int d) { return (unsigned long long)S.H.cnt[0][d]; }, [&](int d) { return 0u; }, false,
                       rank, tid);
            if (tid == 0) {
                S.lsel_count = rank - (uint32_t)S.hit_k;
                S.lsel_prefix = (prefix << 8) | S.hit_pos;
            }
            consumer_sync();
        }
        tie_idx = S.lsel_prefix;
    }
    if (tid == 0) publish(tau, n_eq, n_tie, tie_idx, count_above);
    consumer_sync();
    mark_kept();
}

// For a radix head that keeps only n_tie of its n_eq threshold ties: find the
// index of the n_tie-th tie in token order (per-tile counts, then a scan of
// the stored scores of the one tile that holds it).
template <int G>
__device__ __noinline__ void r_tie_locate(const Params& P, int b, int slot, int tid) {
    BSmem<G>& S = bsmem<G>();
    const int64_t bs = (int64_t)b * P.n_ret + slot;
    if (__ldcg(&P.hs[bs].all_ties)) return;
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
    const float* sc = P.scores + bs * P.sstride + n0;
    for (int r = tid; r < SROWS; r += CONSUMERS) S.tflag[r] = (r < nvalid && f2key(__ldcg(sc + r)) == tau) ? 1 : 0;
    consumer_sync();
    const int warp = tid >> 5, lane = tid & 31;
    if (warp == 0) {
        uint32_t cum = 0;
        int found = nvalid - 1;
        for (int r0 = 0; r0 < nvalid; r0 += 32) {
            const int r = r0 + lane;
            const uint32_t bal = __ballot_sync(0xffffffffu, r < nvalid && S.tflag[r]);
            const uint32_t c = __popc(bal);
            if (cum + c >= rank) {
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

// The end of the select of radix head (b, slot), by the CTA that finished the
// head's last unit: with at most CAND_CAP tokens in the threshold bin (all
// gathered by the units' compactions, which also marked the blocks above
// it), the select inside the CTA and the marks of the kept candidates;
// otherwise four refine passes, the tie location and a mark pass over the
// whole head, in this CTA.  Then the head's global select state goes back to
// zero for the next call.
template <int G>
__device__ __noinline__ void h_finish(const Params& P, int b, int slot, uint32_t& seq, int tid) {
    BSmem<G>& S = bsmem<G>();
    const int64_t bs = (int64_t)b * P.n_ret + slot;
    // the threshold bin's size and the tokens above it, as the ranges counted them
    const uint32_t ncand = __ldcg(P.sel_ncand + bs);
    if (tid == 0) {
        P.hs[bs].n_cand = ncand;
        P.hs[bs].count_above = __ldcg(P.sel_above + bs);
    }
    consumer_sync();
    if (ncand <= (uint32_t)CAND_CAP) {
        if (ncand <= 8u * CONSUMERS) r_local_select<G, 8>(P, b, slot, tid);
        else r_local_select<G, CAND_CAP / CONSUMERS>(P, b, slot, tid);
    } else {
        const int nch = (__ldg(P.seq_lens + b) + HS_CHUNK - 1) / HS_CHUNK;
        h_pass<G, RP_REF0>(P, b, slot, load_rhead(P.hs + bs), 0, nch, false, seq, tid);
        if (!S.abort) r_digit<G, RP_REF0>(P, b, slot, tid);
        if (!S.abort) h_pass<G, RP_REF1>(P, b, slot, load_rhead(P.hs + bs), 0, nch, false, seq, tid);
        if (!S.abort) r_digit<G, RP_REF1>(P, b, slot, tid);
        if (!S.abort) h_pass<G, RP_REF2>(P, b, slot, load_rhead(P.hs + bs), 0, nch, false, seq, tid);
        if (!S.abort) r_digit<G, RP_REF2>(P, b, slot, tid);
        if (!S.abort) h_pass<G, RP_REF3>(P, b, slot, load_rhead(P.hs + bs), 0, nch, false, seq, tid);
        if (!S.abort) r_digit<G, RP_REF3>(P, b, slot, tid);
        if (!S.abort && !__ldcg(&P.hs[bs].all_ties)) {
            h_pass<G, RP_TIES>(P, b, slot, load_rhead(P.hs + bs), 0, nch, false, seq, tid);
            if (!S.abort) r_tie_locate<G>(P, b, slot, tid);
        }
        if (!S.abort) h_pass<G, RP_MARK>(P, b, slot, load_rhead(P.hs + bs), 0, nch, false, seq, tid);
    }
    for (int d = tid; d < 256; d += CONSUMERS) {
        P.sel_cnt[bs * 256 + d] = 0;
        P.sel_mass[bs * 256 + d] = 0ull;
    }
    if (tid == 0) {
        P.sel_ncand[bs] = 0;
        P.sel_above[bs] = 0;
        P.sel_arrive[2 * bs] = 0;
        P.sel_arrive[2 * bs + 1] = 0;
    }
    consumer_sync();
}

// Block list of radix group i: union of its heads' block bitmaps, in
// ascending block order, with the mask of heads that read each block.
template <int G>
__device__ __noinline__ void r_blist(const Params& P, int b, int rg, int tid) {
    BSmem<G>& S = bsmem<G>();
    const int L = __ldg(P.seq_lens + b);
    const int g = S.tab.rg_group[rg], nh = S.tab.rg_nh[rg], slot0 = S.tab.rg_slot0[rg];
    const int nblk = (L + BLK - 1) / BLK;
    const int nwords = (nblk + 31) / 32;
    const int bg = b * P.n_rg + rg;
    uint32_t* list = P.blist + (int64_t)bg * P.nblk_cap;
    const int warp = tid >> 5, lane = tid & 31;
    if (tid < MAX_G) S.kept[tid] = 0;
    if (tid == 0) S.base = 0;
    consumer_sync();
    // thread tid takes 16 consecutive blocks (half a bitmap word) per round
    const int nhalf = (nblk + 15) / 16;
    for (int h0 = 0; h0 < nhalf; h0 += CONSUMERS) {
        const int hw = h0 + tid, w = hw >> 1;
        uint32_t uni = 0;
        uint32_t hb[G];   // a group has at most G heads
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
            hb[hh] = 0;
            if (hh < nh && hw < nhalf) {
                uint32_t word = __ldcg(P.bitmap + ((int64_t)b * P.n_ret + slot0 + hh) * P.words_cap + w);
                if (w == nwords - 1 && (nblk & 31)) word &= (1u << (nblk & 31)) - 1u;
                if (P.dbg_bitmap && (hw & 1) == 0)
                    P.dbg_bitmap[((int64_t)b * P.Hq + S.tab.slot_head[slot0 + hh]) * P.words_cap + w] = word;
                hb[hh] = (word >> ((hw & 1) * 16)) & 0xFFFFu;
                uni |= hb[hh];
                if (hb[hh]) atomicAdd(&S.kept[hh], __popc(hb[hh]));
            }
        }
        // exclusive scan of the per-thread counts over the CTA
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
            for (int hh = 0; hh < G; ++hh)
                if ((hb[hh] >> jb) & 1u) hm |= 1u << (S.tab.slot_head[slot0 + hh] - g * P.G);
            list[pos++] = ((uint32_t)(hw * 16 + jb) << 8) | hm;
        }
        consumer_sync();
        if (tid == 0) S.base += S.wsum[0] + S.wsum[1] + S.wsum[2] + S.wsum[3];
        consumer_sync();
    }
    if (tid < nh && P.dbg_kept) {
        const int slot = slot0 + tid;
        if (__ldcg(&P.hs[(int64_t)b * P.n_ret + slot].mode) == MODE_RADIX)
            P.dbg_kept[b * P.Hq + S.tab.slot_head[slot]] = S.kept[tid];
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
        const long long t0 = clock64();
        if (lane == 0 && round > 0 && !mbar_wait_bounded(&S.empty[st], (round - 1) & 1u)) {
            set_status(P, ST_TIMEOUT);
            ok = false;
        }
        if (lane == 0 && P.dbg_trace) S.acct[36 - 16] += (unsigned long long)(clock64() - t0);
        return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    };
    int gi = t < t1 ? last_le(pre, ngroups + 1, t) : 0;
    while (t < t1) {
        while (pre[gi + 1] <= t) ++gi;
        const int cnt = pre[gi + 1] - pre[gi];
        const int b = gi / P.n_rg, rg = gi % P.n_rg, g = S.tab.rg_group[rg];
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
    Attn<G> attn;
    attn.init(attn_q_smem<G>(S.X, warp));
    Acct ac;
    ac.init(P, S.acct, tid == 0);
    while (true) {
        const int st = (int)(k % NST);
        if (!mbar_wait_bounded(&S.full[st], (k / NST) & 1u)) {
            set_status(P, ST_TIMEOUT);
            return;
        }
        ac.mark(32);
        ++k;
        const RDesc d = S.desc[st];
        if (d.type != 0) break;
        const int g = S.tab.rg_group[d.rg];
        if (d.flags & 1) attn.begin(P, d.b, g, lane);
        const uint32_t base = smem_u32(&S.stage[st][0]);
        const bool zeroed = attn.tile(base, base + KV_TILE, warp, lane, d.n0, d.nvalid, d.hmask, false, 0, 0);
        if (zeroed) fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[st]);
        ac.mark(33);
        ac.count(35);
        if (d.flags & 2) {
            attn.finish(S.X, warp, lane);
            consumer_sync();
            const uint32_t heads = S.tab.rg_mask[d.rg];
            const int gi = d.b * P.n_rg + d.rg;
            uint16_t* out0 = P.out + ((int64_t)d.b * P.Hq + g * G) * D;
            if (d.seg_tiles == d.item_tiles) {
                split_emit<G>(S.X, heads, nullptr, out0, tid);
                consumer_sync();
            } else {
                float* part = P.rpart + ((int64_t)blockIdx.x + gi) * G * PSTRIDE;
                split_emit<G>(S.X, heads, part, nullptr, tid);
                if (ticket_add(P.tick_ret + gi, (uint32_t)d.seg_tiles, (uint32_t)d.item_tiles, &S.flag)) {
                    combine_splits<G>(S.X, P.rpart + ((int64_t)d.c0 + gi) * G * PSTRIDE, d.nsplits, heads, out0, tid);
                }
            }
            ac.mark(34);
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
// the retrieval phase: its shared-memory set-up, and its body once the
// streaming phase's results are visible (after the streaming grid completed,
// or, in the single launch, after a grid barrier)
// ---------------------------------------------------------------------------
template <int G>
__device__ __forceinline__ void r_setup(const Params& P, int tid) {
    BSmem<G>& S = bsmem<G>();
    constexpr int NST = BSmem<G>::NST;
    if (tid == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(&S.full[i], 1);
            mbar_init(&S.empty[i], CONSUMERS / 32);
        }
        for (int i = 0; i < HS_SLOTS; ++i) mbar_init(&S.hfull[i], 1);
        mbar_fence_init();
        S.gen = 0;
        S.abort = 0;
        for (int i = 0; i < ACCT_SLOTS; ++i) S.acct[i] = 0ull;
    }
    if (tid >= 32) copy_tab(P.tab, S.tab, tid - 32, THREADS - 32);
}

// The call's coordination words back to zero, by the last CTA out of the
// call's last kernel (after an aborted call also the group tickets of the
// select it may have left).
__device__ __noinline__ void clear_call_words(const Params& P) {
    P.sync->n_radix_heads = 0;
    P.sync->barrier = 0;
    P.sync->kb_work = 0;
    if (__ldcg(P.status) != 0) {
        for (int i = 0; i < P.B * P.n_rg; ++i) P.tick_grp[i] = 0;
        for (int64_t i = 0; i < (int64_t)P.B * P.n_ret; ++i) {
            for (int d = 0; d < 256; ++d) {
                P.sel_cnt[i * 256 + d] = 0;
                P.sel_mass[i * 256 + d] = 0ull;
            }
            P.sel_ncand[i] = 0;
            P.sel_above[i] = 0;
            P.sel_arrive[2 * i] = 0;
            P.sel_arrive[2 * i + 1] = 0;
        }
    }
    P.sync->n_decided = 0;
    P.sync->exit_count = 0;
    __threadfence();
}

// The stored scores, dead when every group was settled in the streaming
// kernel: drop their L2 lines without writing them back (each CTA a slice of
// every retrieval head's used range).
__device__ __forceinline__ void drop_scores(const Params& P, int tid) {
    for (int bs = 0; bs < P.B * P.n_ret; ++bs) {
        const int L = __ldg(P.seq_lens + bs / P.n_ret);
        if (!seq_ok(P, L)) continue;
        const char* base = reinterpret_cast<const char*>(P.scores + (int64_t)bs * P.sstride);
        const int nlines = (L * 4 + 127) / 128;
        // the CTAs in a rotated order per head, so a head shorter than the grid's
        // threads does not always fall to the same first CTAs
        const int rb = (int)(((long long)blockIdx.x + (long long)bs * 37) % gridDim.x);
        for (int x = rb * THREADS + tid; x < nlines; x += gridDim.x * THREADS)
            asm volatile("discard.global.L2 [%0], 128;" ::"l"(base + (int64_t)x * 128) : "memory");
    }
}

// single: the single launch, whose transition barrier always counts in
// P.sync->barrier, so the last CTA out always clears the coordination words
template <int G>
__device__ __forceinline__ void r_body(const KParams& K, bool single) {
    BSmem<G>& S = bsmem<G>();
    const Params& P = K.P;
    const int tid = threadIdx.x, lane = tid & 31;
    const bool copier = tid >= CONSUMERS;
    // grid barrier; thread 0's wait goes to debug sum 31
    auto gsync = [&]() {
        const long long t0 = clock64();
        const bool r = grid_sync(P, S);
        if (tid == 0 && P.dbg_trace) S.acct[15] += (unsigned long long)(clock64() - t0);
        return r;
    };
    int* pre = S.pre;
    if (tid == 0) S.base = __ldcg(&P.sync->kb_work);
    // (two launches: the streaming grid is complete, nothing else counts the
    // decisions of this call)
    if (!single && blockIdx.x == 0 && tid == 0) P.sync->n_decided = 0;
    __syncthreads();
    const bool work = S.base != 0;   // nothing left when every group was settled in the streaming kernel
    if (tid == 0) trace_max(P, 13);
    uint32_t k = 0;
    bool ok = S.abort == 0;
    const uint32_t nrad = (ok && work) ? __ldcg(&P.sync->n_radix_heads) : 0u;
    if (nrad > 0) {
        // ---- exact select.  The radix heads' 1024-token score tiles, in head
        // order, are split into contiguous ranges, one per CTA: every range's
        // bins go into its heads' global histograms (phase A); then, per head
        // of the range, the threshold bin from the merged histogram as soon as
        // all of the head's tiles have added their bins, and the range's
        // compaction (phase B).  The CTA that completes a head's last tile (a
        // ticket) selects inside the threshold bin, and the last head of a
        // group (a second ticket) builds the group's block list.  CTAs wait
        // only for tiles of the same head, all of which run on resident CTAs
        // that wait for nothing in phase A.
        auto head_tiles = [&](int hx) {
            const uint32_t e = __ldcg(P.rlist + hx);
            return (__ldg(P.seq_lens + (int)(e >> 16)) + HS_CHUNK - 1) / HS_CHUNK;
        };
        if (tid < 32) warp_prefix(pre, (int)nrad, head_tiles, lane);
        __syncthreads();
        const int NT = pre[nrad];
        const int t0 = (int)((long long)blockIdx.x * NT / gridDim.x);
        const int t1 = (int)((long long)(blockIdx.x + 1) * NT / gridDim.x);
        uint32_t seq = 0;   // score copies this CTA has waited for
        // the range's head segments: head hx, its tiles [c0, c1)
        auto segment = [&](int t, int& hx, int& b, int& slot, int& c0, int& c1, int& nch) {
            hx = last_le(pre, (int)nrad + 1, t);
            const uint32_t e = __ldcg(P.rlist + hx);
            b = (int)(e >> 16);
            slot = (int)(e & 0xFFFFu);
            nch = pre[hx + 1] - pre[hx];
            c0 = t - pre[hx];
            c1 = min(nch, t1 - pre[hx]);
        };
        if (!copier) {
            const long long ta = clock64();
            for (int t = t0; t < t1 && S.abort == 0;) {
                int hx, b, slot, c0, c1, nch;
                segment(t, hx, b, slot, c0, c1, nch);
                const int64_t bs = (int64_t)b * P.n_ret + slot;
                h_pass<G, RP_BINS>(P, b, slot, load_rhead(P.hs + bs), c0, c1, true, seq, tid);
                if (tid == 0) atomicAdd(P.sel_arrive + 2 * bs, (uint32_t)(c1 - c0));
                t = pre[hx] + c1;
            }
            if (tid == 0 && P.dbg_trace) S.acct[37 - 16] += (unsigned long long)(clock64() - ta);
            if (tid == 0) trace_max(P, 14);
            for (int t = t0; t < t1 && S.abort == 0;) {
                const long long tq = clock64();
                int hx, b, slot, c0, c1, nch;
                segment(t, hx, b, slot, c0, c1, nch);
                t = pre[hx] + c1;
                const int64_t bs = (int64_t)b * P.n_ret + slot;
                // every tile of the head has added its bins
                if (tid == 0 && !wait_counter(P.sel_arrive + 2 * bs, (uint32_t)nch)) {
                    set_status(P, ST_TIMEOUT);
                    S.abort = 1;
                }
                consumer_sync();
                if (S.abort) break;
                for (int d = tid; d < 256; d += CONSUMERS) {
                    S.dcnt[d] = __ldcg(P.sel_cnt + bs * 256 + d);
                    S.dmass[d] = __ldcg(P.sel_mass + bs * 256 + d);
                }
                consumer_sync();
                // the threshold bin (every range alike; the one holding tile 0 publishes it)
                r_digit<G, RP_BINS>(P, b, slot, tid, c0 == 0);
                {
                    // every range compacts (gathering at most CAND_CAP, counting
                    // all): the bin's size and the count above it are known only
                    // when the head's last range is done
                    RHead rh = load_rhead(P.hs + bs);
                    rh.bstar = S.hst.bstar;
                    h_pass<G, RP_COMPACT>(P, b, slot, rh, c0, c1, true, seq, tid);
                }
                if (tid == 0) {
                    __threadfence();
                    S.flag = atomicAdd(P.sel_arrive + 2 * bs + 1, (uint32_t)(c1 - c0)) + (uint32_t)(c1 - c0) ==
                                     (uint32_t)nch ? 1u : 0u;
                    if (S.flag) __threadfence();
                }
                consumer_sync();
                if (tid == 0 && P.dbg_trace) S.acct[38 - 16] += (unsigned long long)(clock64() - tq);
                if (!S.flag || S.abort) continue;
                // this CTA completed the head's last tiles
                const long long tf = clock64();
                h_finish<G>(P, b, slot, seq, tid);
                if (S.abort) break;
                const int rg = S.tab.slot_rg[slot];
                if (tid == 0) {
                    const int slot0 = S.tab.rg_slot0[rg], nh = S.tab.rg_nh[rg];
                    uint32_t nrh = 0;
                    for (int hh = 0; hh < nh; ++hh)
                        nrh += __ldcg(&P.hs[(int64_t)b * P.n_ret + slot0 + hh].mode) == MODE_RADIX ? 1u : 0u;
                    __threadfence();
                    const int bg = b * P.n_rg + rg;
                    S.flag = atomicAdd(P.tick_grp + bg, 1u) + 1 == nrh ? 1u : 0u;
                    if (S.flag) {
                        __threadfence();
                        P.tick_grp[bg] = 0;   // re-armed for the next call
                    }
                }
                consumer_sync();
                if (S.flag) r_blist<G>(P, b, rg, tid);
                if (tid == 0 && P.dbg_trace) S.acct[39 - 16] += (unsigned long long)(clock64() - tf);
            }
        }
        if (tid == 0) trace_max(P, 12);
        ok = gsync();
    }
    if (tid == 0) trace_max(P, 3);
    // The stored scores are dead from here on.  Without attention work they
    // are dropped from L2 (no write-back of lines that are still there).  With
    // attention work they are left: its K/V loads evict them anyway, and the
    // drop measured 11-18 us on the step's critical path at 4 x 128K, wherever
    // it was put (the discards block their thread), against ~5 us of
    // write-back bandwidth for those 32 MB during the attention.
    if (!work) drop_scores(P, tid);
    if (ok && work) {
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
        // at least 4 tiles per CTA: with few tiles, a CTA of one tile pays a
        // whole load latency and the group's last CTA combines one partial
        // per tile
        cta_share(T, t0, t1, nact, 4);
        if (copier) r_produce_attn<G>(K, S, pre, ngroups, t0, t1, T, nact, k, lane);
        else r_consume_attn<G>(K, S, k, tid);
        if (tid == 0) trace_max(P, 4);
    }
    if (tid == 0) acct_flush(P, S.acct);
    // the last CTA out clears the call's coordination words (none was set
    // when every group was settled in the streaming kernel: no count then,
    // except for the single launch's transition barrier)
    __syncthreads();
    if ((work || single) && tid == 0) {
        trace_max(P, 5);
        __threadfence();
        if (atomicAdd(&P.sync->exit_count, 1u) == gridDim.x - 1) clear_call_words(P);
    }
}

__device__ __forceinline__ void mbar_inval(uint64_t* bar) {
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// The whole decode step in one launch: the streaming phase, then (after a
// grid barrier that stands for the retrieval kernel's wait on the streaming
// grid) the retrieval phase in the same shared memory.  When every group was
// settled in the streaming phase, the CTAs only clear the call's words and
// drop the stored scores: no second launch.  One resident wave (the
// retrieval phase's grid barriers need it).
template <int G>
__global__ void __launch_bounds__(THREADS, 2) step_kernel(const __grid_constant__ KParams K) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const Params& P = K.P;
    const int tid = threadIdx.x;
    if (smem_u32(smem_raw) & 1023u) {   // (the same for every CTA: none waits for another)
        if (tid == 0) set_status(P, 5u);
        return;
    }
    s_body<G, true>(K);
    __syncthreads();
    // the streaming phase's ring barriers end here (no copy is in flight:
    // its copy warp waited for its last tiles); the memory becomes the
    // retrieval phase's
    ASmem<G>& A = *reinterpret_cast<ASmem<G>*>(smem_raw);
    const uint32_t ngroups = (uint32_t)A.n_vgroups;
    if (tid == 0) {
        for (int i = 0; i < ASmem<G>::NST; ++i) {
            mbar_inval(&A.full[i]);
            mbar_inval(&A.empty[i]);
        }
    }
    __syncthreads();
    r_setup<G>(P, tid);
    __syncthreads();
    // wait until every group is decided (the deciding CTAs are running: each
    // took its group's last ticket); if none was left to the retrieval
    // phase, drop the stored scores and leave without a grid barrier
    BSmem<G>& S = bsmem<G>();
    if (tid == 0) {
        if (!wait_counter(&P.sync->n_decided, ngroups)) {
            set_status(P, ST_TIMEOUT);
            S.abort = 1;
        }
        S.base = __ldcg(&P.sync->kb_work);
    }
    __syncthreads();
    if (S.base == 0u || S.abort != 0u) {
        drop_scores(P, tid);
        __syncthreads();
        if (tid == 0) {
            // the last CTA out clears the call's words
            __threadfence();
            if (atomicAdd(&P.sync->exit_count, 1u) == gridDim.x - 1) clear_call_words(P);
        }
        return;
    }
    grid_sync(P, S);   // a timeout sets S.abort: the body then skips its work
    r_body<G>(K, true);
}

template <int G>
__global__ void __launch_bounds__(THREADS, 2) retrieve_kernel(const __grid_constant__ KParams K) {
    const int tid = threadIdx.x;
    r_setup<G>(K.P, tid);
    // everything below reads the streaming kernel's results: wait for that
    // grid to complete (this launch overlaps only its tail)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    r_body<G>(K, false);
}

}  // namespace rtp
