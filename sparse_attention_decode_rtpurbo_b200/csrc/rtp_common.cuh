// Shared definitions of the RTPurbo decode-step kernels (sm_100a).
#pragma once
#include <cuda.h>   // CUtensorMap
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rtp {

constexpr int D = 128;            // head dimension
constexpr int R = 16;             // indexer rank
constexpr int BLK = 64;           // KV block (page) size in tokens
constexpr int SROWS = 1024;       // k_idx rows per index tile (32 KB)
constexpr int STAGE_BYTES = 32768;   // one ring stage: an index tile, or a 64-token K tile + V tile
constexpr int KV_TILE = 16384;       // one 64 x 128 bf16 tile (two 64 x 64 TMA boxes, 128-byte swizzle)
constexpr int CONSUMERS = 128;    // 4 compute warps
constexpr int THREADS = CONSUMERS + 32;   // + 1 copy warp
constexpr int PSTRIDE = 132;      // floats per split partial: m, l, 2 pad, acc[128]
constexpr int MAX_G = 8, MAX_HQ = 128, MAX_HKV = 64, MAX_B = 1024;
constexpr int AGG_BUCKETS = 32;
constexpr int CAND_CAP = 4096;    // threshold-bin tokens selected inside one CTA

enum SelMode : int32_t { MODE_SKIP = 0, MODE_TOP1 = 1, MODE_ALL = 2, MODE_RADIX = 3 };

// Status codes mirrored from rtp_decode.h (device side).
constexpr uint32_t ST_DEVICE_INPUT = 6;
constexpr uint32_t ST_TIMEOUT = 7;

// Per retrieval head and bucket (split mod AGG_BUCKETS), folded by the
// index-score splits with fire-and-forget atomics (all-zero = empty, so a
// zero-filled workspace is ready): best = (max key << 32) | ~argmax,
// nmin = ~(min key), zabs = fp64 sum of exp(s/4), flags bit 0 = a split's
// scores left the range where that sum is safe.
struct HeadAgg {
    unsigned long long best;
    uint32_t nmin, flags;
    double zabs;
};

struct HeadState {
    int32_t mode;
    float smax;
    uint32_t maxkey, argmax, minkey, pad0;
    double zrel;                            // sum over n < L of exp((s_n - smax)/4)
    unsigned long long target, mass_above;  // fixed-point masses (units of 2^-40)
    uint32_t prefix, count_above, n_eq, n_tie, all_ties, kstar, tau_key;
    uint32_t tie_idx;                       // largest index among the threshold ties kept
    float dr, inv_w;                        // first select pass: bins of width dr/255 over smax - s in [0, dr)
    uint32_t bstar, n_cand;                 // the bin that holds the threshold, and its token count
};

// Coordination words of one call (workspace; zero between calls).
struct Sync {
    uint32_t n_radix_heads;    // heads needing the exact select (list in rlist)
    uint32_t barrier;          // grid barrier arrivals of the retrieval kernel
    uint32_t exit_count;
    uint32_t kb_work;          // groups left to the retrieval kernel (a select, or blocks to attend)
    uint32_t n_decided;        // (b, group) pairs decided so far (a count the single launch waits for)
    uint32_t pad[18];
};

// Head split (host-derived): retrieval groups (KV heads with >= 1 retrieval
// head), local groups (KV heads with >= 1 local head), retrieval slots (one
// per retrieval query head).  The kernels read it with run-time indices, so
// each CTA copies it to shared memory once (copy_tab) instead of indexing the
// parameter block on its critical paths.
struct alignas(16) HeadTab {
    uint8_t rg_group[MAX_HKV], rg_mask[MAX_HKV], rg_slot0[MAX_HKV], rg_nh[MAX_HKV];
    uint8_t lg_group[MAX_HKV], lg_mask[MAX_HKV];
    uint8_t slot_head[MAX_HQ], slot_rg[MAX_HQ];
};
static_assert(sizeof(HeadTab) % 16 == 0, "HeadTab copies as 16-byte words");

// the table copied by `n` threads (t = 0 .. n-1) into shared memory
__device__ __forceinline__ void copy_tab(const HeadTab& src, HeadTab& dst, int t, int n) {
    const uint4* a = reinterpret_cast<const uint4*>(&src);
    uint4* d = reinterpret_cast<uint4*>(&dst);
    for (int i = t; i < (int)(sizeof(HeadTab) / 16); i += n) d[i] = a[i];
}

struct Params {
    int B, Hq, Hkv, G, Ncap, nblk_cap, words_cap, ntiles_cap, mbps, num_pages, window, sink;
    int sstride;   // row stride of the stored scores: ntiles_cap * SROWS (whole 4 KB tiles)
    int n_ret, n_rg, n_lg;
    const uint16_t *q_pre, *q_rope, *k_idx, *Wq;
    const uint16_t *k_cache_ptr, *v_cache_ptr;   // the caches as plain pointers (the kernels read them through TMA maps)
    const int32_t *seq_lens, *block_table;
    const float* p;   // top-p mass per sequence (unused, may be null, under static top-k)
    int topk;         // 0: dynamic top-p; k >= 1: every retrieval head keeps its k best tokens
    // local heads' ring cache: local groups i with bit i of ring_lg_mask read
    // their sink and window from rings of ring_rows = 64 + ring_W rows per
    // (sequence, KV head): block 0 in rows 0..63, block j >= 1 in the 64 rows
    // from 64 + (64 j mod ring_W)
    unsigned long long ring_lg_mask;
    int ring_W, ring_rows;
    uint16_t* out;
    HeadTab tab;
    // workspace
    uint32_t* status;
    Sync* sync;
    uint32_t* rlist;
    uint32_t *tick_score, *tick_local, *tick_ret;
    uint32_t* tick_grp;   // [B * n_rg] radix heads of the group done with their select (zero between calls)
    // the exact select's per-head global state (zero between calls): merged
    // first-pass histogram (2^-40 mass; counts only from a CTA that held the
    // whole head), gathered candidates, and the tiles that have added their
    // bins / finished their compaction
    uint32_t* sel_cnt;                // [B * n_ret, 256]
    unsigned long long* sel_mass;     // [B * n_ret, 256]
    uint32_t* sel_ncand;              // [B * n_ret] tokens in the threshold bin (all gathered up to CAND_CAP)
    uint32_t* sel_above;              // [B * n_ret] tokens above the threshold bin
    uint32_t* sel_arrive;             // [B * n_ret, 2]
    HeadAgg* agg;
    HeadState* hs;
    uint32_t* tie_cnt;
    float* scores;   // [B * n_ret, sstride] fp32 index scores, written by the streaming kernel, read by the select
    unsigned long long* cand;        // [B * n_ret, CAND_CAP] (key << 32 | token index)
    uint32_t* bitmap;
    uint32_t* blist;
    uint32_t* bcount;
    float* lpart;
    float* rpart;
    // optional diagnostics
    float* dbg_tau;
    int32_t* dbg_kstar;
    int32_t* dbg_kept;
    float* dbg_smax;
    double* dbg_Z;
    uint32_t* dbg_bitmap;
    unsigned long long* dbg_trace;
};

// Kernel argument block: the tensor maps of the K and V caches (2-D:
// rows x 128 bf16, 64 x 64 boxes, 128-byte swizzle) travel as grid constants.
struct KParams {
    CUtensorMap tmk, tmv;
    CUtensorMap tmk_r, tmv_r;   // the local heads' rings (encoded only when they are given)
    Params P;
};

// ---------------------------------------------------------------------------
// small helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
           ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
}

// order-preserving map fp32 -> uint32 (larger float, larger key)
__device__ __forceinline__ uint32_t f2key(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key2f(uint32_t k) {
    uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
    return __uint_as_float(u);
}

// e^x for |x| <= 700 as an fp64 value: 2^(x log2 e) split into an integer
// power (exact, ldexp) and a fractional one (fp32 special-function unit,
// about 2 ulp of fp32).  Used where only a ~1e-6 relative accuracy matters.
__device__ __forceinline__ double exp_wide(double x) {
    const double y = x * 1.4426950408889634;
    const double yi = floor(y);
    // f in [1, 2] times 2^yi, by adding yi to f's exponent field (the result
    // is a normal double for |x| <= 700: the same value ldexp would give)
    const double f = (double)exp2f((float)(y - yi));
    const unsigned long long e = (unsigned long long)(long long)(int)yi << 52;   // two's complement exponent step
    return __longlong_as_double((long long)((unsigned long long)__double_as_longlong(f) + e));
}

// softmax(s/4) weight of a score relative to the maximum score, in 2^-40 units
__device__ __forceinline__ unsigned long long fixmass(uint32_t key, float smax) {
    float e = expf((key2f(key) - smax) * 0.25f);
    return __float2ull_rn(e * 1099511627776.0f);
}

__device__ __forceinline__ void set_status(const Params& P, uint32_t code) { atomicCAS(P.status, 0u, code); }

__device__ __forceinline__ bool seq_ok(const Params& P, int L) { return L >= 1 && L <= P.Ncap; }

// Page id of block j of sequence b (paged layout); an id outside
// [0, num_pages) records an input error and reads page 0 instead.
__device__ __forceinline__ int page_or_zero(const Params& P, int b, int j) {
    const int pg = __ldg(P.block_table + (int64_t)b * P.mbps + j);
    if (pg >= 0 && pg < P.num_pages) return pg;
    set_status(P, ST_DEVICE_INPUT);
    return 0;
}

// First ring row (of the `rows x 128` ring views) of block j of KV head g of sequence b.
__device__ __forceinline__ int64_t ring_block_row(const Params& P, int b, int g, int j) {
    const int slot = j == 0 ? 0 : BLK + (int)(((int64_t)j * BLK) % P.ring_W);
    return ((int64_t)b * P.Hkv + g) * P.ring_rows + slot;
}

// First cache row (of `rows x dim` views) of block j of KV head g of sequence b.
__device__ __forceinline__ int64_t block_row(const Params& P, int b, int g, int j) {
    if (P.block_table == nullptr) return ((int64_t)b * P.Hkv + g) * P.Ncap + (int64_t)j * BLK;
    return ((int64_t)page_or_zero(P, b, j) * P.Hkv + g) * BLK;
}

// 2^x on the special-function unit (about 2 ulp; 0 for x = -inf)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// optional timeline (debug): latest %globaltimer of event i
__device__ __forceinline__ void trace_max(const Params& P, int i) {
    if (P.dbg_trace) atomicMax(P.dbg_trace + i, (unsigned long long)global_ns());
}

// optional cycle accounting (debug, one thread per CTA): the SM cycles since
// the previous mark are added to sum `slot` (16..47) of the CTA's shared
// array `sums`, which acct_flush adds to the trace once at the CTA's end (a
// global atomic per mark from every CTA would serialise in L2 and distort
// what it measures)
constexpr int ACCT_SLOTS = 32;   // debug sums 16..47
struct Acct {
    unsigned long long* sums;
    long long t;
    __device__ __forceinline__ void init(const Params& P, unsigned long long* s, bool me) {
        sums = (me && P.dbg_trace) ? s : nullptr;
        if (sums) t = clock64();
    }
    __device__ __forceinline__ void mark(int slot) {
        if (!sums) return;
        const long long now = clock64();
        sums[slot - 16] += (unsigned long long)(now - t);
        t = now;
    }
    __device__ __forceinline__ void count(int slot) {
        if (sums) sums[slot - 16] += 1ull;
    }
};
__device__ __forceinline__ void acct_flush(const Params& P, unsigned long long* sums) {
    if (!P.dbg_trace) return;
    for (int i = 0; i < ACCT_SLOTS; ++i)
        if (sums[i]) atomicAdd(P.dbg_trace + 16 + i, sums[i]);
}

// ---------------------------------------------------------------------------
// mbarrier, bulk copies and TMA tensor copies
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait: gives up after about two seconds of wall time.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0 && global_ns() - t0 > 2000000000ull) return false;
    }
}
// Plain bulk copy global -> shared (16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
// One 2-D TMA box (x = column, y = row) into shared memory (1024-byte aligned
// for the 128-byte swizzle).  x is 0 or 64 here: 128-byte aligned.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
// L2 prefetch (a hint: nothing to wait for) of one 2-D TMA box, and of the
// K and V boxes of one 64-row block (x as for the loads: 16-byte aligned)
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int x, int y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void kv_prefetch_l2(const CUtensorMap* mk, const CUtensorMap* mv, int row) {
    tma_prefetch_2d(mk, 0, row);
    tma_prefetch_2d(mk, 64, row);
    tma_prefetch_2d(mv, 0, row);
    tma_prefetch_2d(mv, 64, row);
}
// L2 prefetch of the 128-byte line at p (a hint: nothing to wait for)
__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 16-byte load from a shared-memory address
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ void sts128_zero(uint32_t addr) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};" ::"r"(addr), "r"(0u) : "memory");
}

// ---------------------------------------------------------------------------
// warp-level tensor-core primitives (bf16 in, fp32 accumulate)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
// c += A(16x16, row) * B(16x8, col)
__device__ __forceinline__ void mma_bf16(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// per-sequence geometry of the local heads' block list: sink blocks
// [0, nA), then window blocks [bw0, bw0 + nv - nA)
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

}  // namespace rtp
