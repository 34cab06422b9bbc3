// Shared definitions of the RTPurbo decode-step kernels (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rtp {

constexpr int D = 128;          // head dimension
constexpr int R = 16;           // indexer rank
constexpr int BLK = 64;         // KV block (page) size in tokens
constexpr int CHUNK = 2048;         // tokens per selection item (= 32 blocks = one bitmap word)
constexpr int SCORE_CHUNK = 2048;   // tokens per index-score item (2 staged tiles)
constexpr int SEL_THREADS = 256;
constexpr int ATT_THREADS = 128;
constexpr int STAGES = 3;                       // K/V tile ring depth of the attention kernels
constexpr int TILE_BYTES = BLK * D * 2;         // one 64x128 bf16 tile = 16 KB
constexpr int STAGE_BYTES = 2 * TILE_BYTES;     // K + V
constexpr int PSTRIDE = 132;                    // floats per partial: m, l, 2 pad, acc[128]
constexpr int MAX_G = 8, MAX_HQ = 128, MAX_HKV = 64;
constexpr double FIX_SCALE = 1099511627776.0;   // 2^40: fixed-point unit of softmax mass

enum SelMode : int32_t { MODE_SKIP = 0, MODE_TOP1 = 1, MODE_ALL = 2, MODE_RADIX = 3 };

// Status codes mirrored from rtp_decode.h (device side).
constexpr uint32_t ST_DEVICE_INPUT = 6;
constexpr uint32_t ST_TIMEOUT = 7;

// Per retrieval head and bucket (chunk mod AGG_BUCKETS), folded by score
// chunks with fire-and-forget atomics (all-zero = empty, so a zero-filled
// workspace is ready): best = (max key << 32) | ~argmax, nmin = ~(min key),
// zabs = fp64 sum of exp(s/4), flags bit 0 = a chunk's scores left the range
// where that sum is safe.  Buckets keep same-address atomics rare.
constexpr int AGG_BUCKETS = 32;
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
    uint32_t prefix, count_above, n_eq, n_tie, all_ties, kstar, tau_key, pad1;
};

struct Params {
    int B, Hq, Hkv, G, Ncap, nblk_cap, words_cap, mbps, num_pages, window, sink;
    int n_ret, n_rg, n_lg, nchunks, nschunks;
    int local_kb, local_items, ret_grid;
    const uint16_t *q_pre, *q_rope, *k_idx, *k_cache, *v_cache, *Wq;
    const int32_t *seq_lens, *block_table;
    const float* p;
    uint16_t* out;
    // head split (host-derived): retrieval groups (KV heads with >= 1 retrieval head),
    // local groups (KV heads with >= 1 local head), retrieval slots (one per retrieval query head)
    uint8_t rg_group[MAX_HKV], rg_mask[MAX_HKV], rg_slot0[MAX_HKV], rg_nh[MAX_HKV];
    uint8_t lg_group[MAX_HKV], lg_mask[MAX_HKV];
    uint8_t slot_head[MAX_HQ], slot_rg[MAX_HQ];
    // workspace
    uint32_t* status;
    uint32_t *tick_score, *tick_radix, *tick_local, *tick_ret;
    uint32_t* keys;
    HeadAgg* agg;
    HeadState* hs;
    uint32_t* hist_cnt;
    unsigned long long* hist_mass;
    uint32_t* chunk_cnt;
    uint32_t* tie_off;
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

// ---------------------------------------------------------------------------
// small helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// order-preserving map fp32 -> uint32 (larger float, larger key)
__device__ __forceinline__ uint32_t f2key(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key2f(uint32_t k) {
    uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
    return __uint_as_float(u);
}

// softmax(s/4) weight of a score relative to the maximum score, in 2^-40 units
__device__ __forceinline__ unsigned long long fixmass(uint32_t key, float smax) {
    float e = expf((key2f(key) - smax) * 0.25f);
    return __float2ull_rn(e * 1099511627776.0f);
}

__device__ __forceinline__ void set_status(const Params& P, uint32_t code) { atomicCAS(P.status, 0u, code); }

__device__ __forceinline__ bool seq_ok(const Params& P, int L) { return L >= 1 && L <= P.Ncap; }

// Page id of block j of sequence b (paged layout), or -1 when out of range.
__device__ __forceinline__ int page_of(const Params& P, int b, int j) {
    int pg = __ldg(P.block_table + (int64_t)b * P.mbps + j);
    return (pg >= 0 && pg < P.num_pages) ? pg : -1;
}

// Element offset of row n of KV head g of sequence b in a cache of row width `dim`.
__device__ __forceinline__ int64_t row_off(const Params& P, int b, int g, int n, int dim, bool* bad) {
    if (P.block_table == nullptr) return (((int64_t)b * P.Hkv + g) * P.Ncap + n) * dim;
    int pg = page_of(P, b, n / BLK);
    if (pg < 0) {
        *bad = true;
        pg = 0;
    }
    return (((int64_t)pg * P.Hkv + g) * BLK + (n % BLK)) * dim;
}

// Ticket: returns true in exactly one (the last) of `count` arrivals, and
// re-arms the counter for the next call.  Caller has done __syncthreads().
__device__ __forceinline__ bool last_arrival(uint32_t* ctr, uint32_t count, uint32_t* smem_flag) {
    if (threadIdx.x == 0) {
        __threadfence();
        uint32_t t = atomicAdd(ctr, 1u);
        bool last = (t == count - 1);
        if (last) {
            atomicExch(ctr, 0u);
            __threadfence();
        }
        *smem_flag = last;
    }
    __syncthreads();
    return *smem_flag != 0;
}

// ---------------------------------------------------------------------------
// mbarrier + bulk copy (TMA engine, non-tensor form)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// 2^x on the special-function unit (about 2 ulp; 0 for x = -inf)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 16-byte load from a shared-memory address (explicit shared state space)
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
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
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
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
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// One 32-byte row read once: 256-bit load, not kept in L1, evicted early from L2.
// The address must be 32-byte aligned.
struct U8x32 {
    uint32_t w[8];
};
__device__ __forceinline__ U8x32 ld_stream32(const void* p) {
    U8x32 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::evict_first.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]), "=r"(v.w[4]), "=r"(v.w[5]), "=r"(v.w[6]),
                   "=r"(v.w[7])
                 : "l"(p));
    return v;
}

}  // namespace rtp
