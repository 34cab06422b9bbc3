// C ABI of the RTPurbo decode step: argument checks, workspace layout, the
// TMA tensor maps of the K/V caches, and the launches of the two sm_100a
// kernels (rtp_stream.cuh: index scores + local heads; rtp_retrieve.cuh:
// exact select when needed + retrieval heads).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <stdio.h>
#include <stdlib.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "../../include/rtp_decode.h"
#include "rtp_retrieve.cuh"
#include "rtp_append.cuh"
#include "rtp_prefill.cuh"
#include "rtp_prefill_tc.cuh"

namespace rtp {

constexpr int MAX_GRID = 148 * 4;   // upper bound of either grid (split partials are sized for it)
constexpr int MAX_RET_GROUPS = 4096;   // B * (KV groups with retrieval heads) held in shared memory

struct Plan {
    int B, Hq, Hkv, G, Ncap, nblk_cap, words_cap, ntiles_cap;
    int n_ret, n_rg, n_lg;
    long long tiles_cap;   // upper bound of the streaming kernel's tiles
    uint8_t rg_group[MAX_HKV], rg_mask[MAX_HKV], rg_slot0[MAX_HKV], rg_nh[MAX_HKV];
    uint8_t lg_group[MAX_HKV], lg_mask[MAX_HKV];
    uint8_t slot_head[MAX_HQ], slot_rg[MAX_HQ];
    // workspace byte offsets; [0, zero_end) must be zero when a call starts
    size_t o_status, o_sync, o_tick_score, o_tick_local, o_tick_ret, o_tick_grp, o_agg, o_sel_cnt, o_sel_mass, o_sel_ncand, o_sel_above, o_sel_arrive, zero_end;
    size_t o_rlist, o_hs, o_tie_cnt, o_scores, o_cand, o_bitmap, o_blist, o_bcount, o_lpart, o_rpart, total;
};

static size_t align_up(size_t x) { return (x + 255) & ~(size_t)255; }

static rtp_status check_dims(const rtp_dims* d) {
    if (!d) return RTP_ERR_NULL;
    if (d->head_dim != D || d->idx_dim != R || d->block_size != BLK) return RTP_ERR_UNSUPPORTED;
    if (d->batch < 1 || d->num_q_heads < 1 || d->num_kv_heads < 1) return RTP_ERR_SHAPE;
    if (d->num_q_heads % d->num_kv_heads) return RTP_ERR_SHAPE;
    const int G = d->num_q_heads / d->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return RTP_ERR_UNSUPPORTED;
    if (d->num_q_heads > MAX_HQ || d->num_kv_heads > MAX_HKV || d->batch > MAX_B) return RTP_ERR_UNSUPPORTED;
    if (d->max_seq_len < BLK || d->max_seq_len % BLK) return RTP_ERR_SHAPE;
    if (d->max_seq_len > (1 << 28)) return RTP_ERR_UNSUPPORTED;
    if (d->block_table) {
        if (d->max_blocks_per_seq < 1 || d->num_pages < 1) return RTP_ERR_SHAPE;
        if ((int64_t)d->max_blocks_per_seq * BLK != d->max_seq_len) return RTP_ERR_SHAPE;
        if ((int64_t)d->num_pages * d->num_kv_heads * BLK >= (1ll << 31)) return RTP_ERR_UNSUPPORTED;
    } else if ((int64_t)d->batch * d->num_kv_heads * d->max_seq_len >= (1ll << 31)) {
        return RTP_ERR_UNSUPPORTED;   // TMA row coordinates are 32-bit
    }
    return RTP_OK;
}

static rtp_status make_plan(const rtp_dims* d, const uint8_t* head_kind, int window, int sink, Plan* pl) {
    rtp_status st = check_dims(d);
    if (st != RTP_OK) return st;
    if (!head_kind) return RTP_ERR_NULL;
    memset(pl, 0, sizeof(*pl));
    pl->B = d->batch;
    pl->Hq = d->num_q_heads;
    pl->Hkv = d->num_kv_heads;
    pl->G = pl->Hq / pl->Hkv;
    pl->Ncap = d->max_seq_len;
    pl->nblk_cap = pl->Ncap / BLK;
    pl->words_cap = (pl->nblk_cap + 31) / 32;
    pl->ntiles_cap = (pl->Ncap + SROWS - 1) / SROWS;
    for (int g = 0; g < pl->Hkv; ++g) {
        uint32_t rm = 0, lm = 0;
        for (int i = 0; i < pl->G; ++i) {
            const int h = g * pl->G + i;
            if (head_kind[h] > 1) return RTP_ERR_SHAPE;
            if (head_kind[h]) rm |= 1u << i;
            else lm |= 1u << i;
        }
        if (rm) {
            const int r = pl->n_rg++;
            pl->rg_group[r] = (uint8_t)g;
            pl->rg_mask[r] = (uint8_t)rm;
            pl->rg_slot0[r] = (uint8_t)pl->n_ret;
            for (int i = 0; i < pl->G; ++i)
                if ((rm >> i) & 1u) {
                    pl->slot_head[pl->n_ret] = (uint8_t)(g * pl->G + i);
                    pl->slot_rg[pl->n_ret] = (uint8_t)r;
                    pl->n_ret++;
                    pl->rg_nh[r]++;
                }
        }
        if (lm) {
            const int l = pl->n_lg++;
            pl->lg_group[l] = (uint8_t)g;
            pl->lg_mask[l] = (uint8_t)lm;
        }
    }
    if ((long long)pl->B * pl->n_rg > MAX_RET_GROUPS) return RTP_ERR_UNSUPPORTED;
    {
        const long long nv_max = std::min<long long>(
            pl->nblk_cap, (sink + BLK - 1) / BLK + (window > 0 ? (window + BLK - 1) / BLK + 1 : 0));
        pl->tiles_cap = (long long)pl->B * (pl->n_rg * (long long)pl->ntiles_cap + pl->n_lg * nv_max);
    }
    const size_t BR = (size_t)pl->B * pl->n_ret, BG = (size_t)pl->B * pl->n_rg, BL = (size_t)pl->B * pl->n_lg;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = align_up(o + bytes);
        return at;
    };
    pl->o_status = take(64);
    pl->o_sync = take(sizeof(Sync));
    pl->o_tick_score = take(BG * 4);
    pl->o_tick_local = take(BL * 4);
    pl->o_tick_ret = take(BG * 4);
    pl->o_tick_grp = take(BG * 4);
    pl->o_agg = take(BR * AGG_BUCKETS * sizeof(HeadAgg));
    pl->o_sel_cnt = take(BR * 256 * 4);
    pl->o_sel_mass = take(BR * 256 * 8);
    pl->o_sel_ncand = take(BR * 4);
    pl->o_sel_above = take(BR * 4);
    pl->o_sel_arrive = take(BR * 2 * 4);
    pl->zero_end = o;
    pl->o_rlist = take(BR * 4);
    pl->o_hs = take(BR * sizeof(HeadState));
    pl->o_tie_cnt = take(BR * pl->ntiles_cap * 4);
    pl->o_scores = take(BR * (size_t)pl->ntiles_cap * SROWS * 4);
    pl->o_cand = take(BR * (size_t)CAND_CAP * 8);
    pl->o_bitmap = take(BR * pl->words_cap * 4);
    pl->o_blist = take(BG * pl->nblk_cap * 4);
    pl->o_bcount = take(BG * 4);
    // a split partial per (CTA, item) pair: slot = CTA + item index, at most grid + items
    pl->o_lpart = take(((size_t)MAX_GRID + BL) * pl->G * PSTRIDE * 4);
    pl->o_rpart = take(((size_t)MAX_GRID + BG) * pl->G * PSTRIDE * 4);
    pl->total = o;
    return RTP_OK;
}

// cuTensorMapEncodeTiled from the driver, looked up once.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
static EncodeTiledFn encode_fn() {
    static std::atomic<EncodeTiledFn> fn{nullptr};
    EncodeTiledFn f = fn.load();
    if (!f) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !p)
            return nullptr;
        f = reinterpret_cast<EncodeTiledFn>(p);
        fn.store(f);
    }
    return f;
}

// A [rows, 128] bf16 cache as 64 x 64 boxes with the 128-byte swizzle.
static bool encode_cache_map(CUtensorMap* map, const void* base, long long rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, 64};
    const cuuint32_t estr[2] = {1, 1};
    return f(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Resident CTAs per SM of a kernel at a dynamic shared-memory size on the
// current device (cached per device: the shared-memory limit a kernel is
// given below is a per-device setting).
struct OccCache {
    std::mutex mu;
    const void* fn[16];
    size_t smem[16];
    int dev[16];
    int occ[16];
    int n = 0;
};
static int occupancy(const void* fn, size_t smem, int threads = THREADS) {
    static OccCache c;
    int dev = 0, maxs = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(c.mu);
    for (int i = 0; i < c.n; ++i)
        if (c.fn[i] == fn && c.smem[i] == smem && c.dev[i] == dev) return c.occ[i];
    // the limit is raised to the largest block allocation once (lowering it
    // again for a smaller call would break a later larger one)
    if (cudaDeviceGetAttribute(&maxs, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return 0;
    if ((size_t)maxs < smem) return 0;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, maxs) != cudaSuccess) return 0;
    cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, smem) != cudaSuccess) return 0;
    const int slot = c.n < 16 ? c.n++ : 15;
    c.fn[slot] = fn;
    c.smem[slot] = smem;
    c.dev[slot] = dev;
    c.occ[slot] = n;
    return n;
}

// RTP_VERBOSE=1 in the environment: CUDA failures behind RTP_ERR_CUDA are
// reported on stderr (what failed and the CUDA error string).
static cudaError_t report(cudaError_t e, const char* what) {
    static const bool verbose = getenv("RTP_VERBOSE") != nullptr;
    if (e != cudaSuccess && verbose) fprintf(stderr, "rtp: %s: %s\n", what, cudaGetErrorString(e));
    return e;
}

// SM count of the current device (cached per device).
static int num_sms() {
    constexpr int MAXDEV = 64;
    static std::atomic<int> n[MAXDEV];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (dev < 0 || dev >= MAXDEV) return 0;
    int v = n[dev].load();
    if (!v) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        n[dev].store(v);
    }
    return v;
}

// Test knob: RTP_GRID_CAP=n (n >= 1) caps both grids at n CTAs, so that small
// tests reach the paths that only long shares take (select passes reading
// the stored scores from global memory, histogram flushes every 64 tiles).
// Read at every call; results do not depend on the grid.
static int grid_cap() {
    const char* v = getenv("RTP_GRID_CAP");
    const int n = v ? atoi(v) : 0;
    return n >= 1 ? n : MAX_GRID;
}

// RTP_SINGLE_LAUNCH=1 in the environment (read at every call): the step
// runs as one launch (step_kernel: streaming phase, grid barrier, retrieval
// phase) instead of two.  Results do not depend on it.
static bool single_launch() {
    const char* v = getenv("RTP_SINGLE_LAUNCH");
    return v && atoi(v) == 1;
}

template <int G>
static cudaError_t launch(const KParams& K, const Plan& pl, cudaStream_t s, void* const* ev, unsigned ev_flags) {
    const int sms = num_sms();
    if (!sms) return report(cudaErrorUnknown, "SM count");
    const int cap = std::min(MAX_GRID, grid_cap());
    if (pl.n_rg > 0 && single_launch()) {
        // one resident wave with room for either phase's shared memory (the
        // retrieval phase's grid barriers need every CTA resident; surplus
        // CTAs take no share of the streaming phase)
        const size_t smem = std::max(asmem_bytes<G>(pl.B), bsmem_bytes<G>(pl.B * pl.n_ret));
        const int occ = occupancy((const void*)step_kernel<G>, smem);
        if (occ < 1) return report(cudaErrorInvalidConfiguration, "step kernel occupancy");
        const int grid = std::min(cap, occ * sms);
        cudaLaunchConfig_t cfg;
        memset(&cfg, 0, sizeof(cfg));
        cfg.gridDim = dim3((unsigned)grid);
        cfg.blockDim = dim3(THREADS);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;   // every CTA resident: the grid barrier's premise
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaError_t e = report(cudaLaunchKernelEx(&cfg, step_kernel<G>, K), "step kernel launch");
        if (ev) cudaEventRecordWithFlags((cudaEvent_t)ev[1], s, ev_flags);   // (no phase boundary to mark)
        return e;
    }
    // streaming kernel: as many resident CTAs as the tiles can use
    {
        const size_t smem = asmem_bytes<G>(pl.B);
        const int occ = occupancy((const void*)stream_kernel<G>, smem);
        if (occ < 1) return report(cudaErrorInvalidConfiguration, "stream kernel occupancy");
        const long long grid = std::max(1ll, std::min<long long>(std::min(cap, occ * sms), pl.tiles_cap));
        stream_kernel<G><<<(unsigned)grid, THREADS, smem, s>>>(K);
        cudaError_t e = report(cudaGetLastError(), "stream kernel launch");
        if (e != cudaSuccess) return e;
    }
    if (ev) cudaEventRecordWithFlags((cudaEvent_t)ev[1], s, ev_flags);
    if (pl.n_rg == 0) return cudaSuccess;
    // retrieval kernel: one resident wave (its CTAs meet at grid barriers),
    // launched as a programmatic dependent of the streaming kernel so that
    // its launch overlaps that kernel's tail
    {
        const size_t smem = bsmem_bytes<G>(pl.B * pl.n_ret);
        const int occ = occupancy((const void*)retrieve_kernel<G>, smem);
        if (occ < 1) return report(cudaErrorInvalidConfiguration, "retrieval kernel occupancy");
        const int grid = std::min(cap, occ * sms);
        cudaLaunchConfig_t cfg;
        memset(&cfg, 0, sizeof(cfg));
        cfg.gridDim = dim3((unsigned)grid);
        cfg.blockDim = dim3(THREADS);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        // cooperative: the driver places every CTA at once or refuses the
        // launch, so the grid barriers never wait on a CTA that kernels of
        // other streams keep from starting
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = ev ? 1 : 2;   // an event recorded in between orders the kernels anyway
        cudaError_t e = report(cudaLaunchKernelEx(&cfg, retrieve_kernel<G>, K), "retrieval kernel launch");
        if (e != cudaSuccess) return e;
    }
    return report(cudaGetLastError(), "retrieval kernel launch");
}

}  // namespace rtp

using namespace rtp;

extern "C" size_t rtp_workspace_size(const rtp_dims* dims, const uint8_t* head_kind) {
    Plan pl;
    if (make_plan(dims, head_kind, 0, 1, &pl) != RTP_OK) return 0;
    return pl.total;
}

static bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

// The decode step with a caller workspace: dynamic top-p (p, topk = 0) or
// static top-k (topk >= 1, p unused).
// (and, with k_ring, the local heads' rings of 64 + ring_W rows).
static rtp_status decode_step_ws(const rtp_dims* dims, const uint16_t* q_pre, const uint16_t* q_rope,
                                 const uint16_t* k_idx, const uint16_t* k_cache, const uint16_t* v_cache,
                                 const uint16_t* k_ring, const uint16_t* v_ring, int32_t ring_W,
                                 const uint16_t* Wq_idx, const int32_t* seq_lens, const uint8_t* head_kind,
                                 const float* p, int32_t topk, int32_t window, int32_t sink, uint16_t* out,
                                 void* stream, bool clear_first = false) {
    if (!dims || !q_pre || !q_rope || !k_idx || !k_cache || !v_cache || !Wq_idx || !seq_lens || !head_kind ||
        (topk == 0 && !p) || !out || (k_ring && !v_ring))
        return RTP_ERR_NULL;
    if (topk < 0) return RTP_ERR_SHAPE;
    if (window < 0 || sink < 0 || (int64_t)window + sink < 1) return RTP_ERR_SHAPE;
    if (k_ring && (ring_W < BLK || ring_W % BLK || ring_W < window || sink > BLK)) return RTP_ERR_SHAPE;
    if (!aligned16(q_pre) || !aligned16(q_rope) || !aligned16(k_idx) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned16(Wq_idx) || !aligned16(out) || (k_ring && (!aligned16(k_ring) || !aligned16(v_ring))))
        return RTP_ERR_UNSUPPORTED;
    Plan pl;
    rtp_status st = make_plan(dims, head_kind, window, sink, &pl);
    if (st != RTP_OK) return st;
    if (!dims->workspace || dims->workspace_bytes < pl.total || ((uintptr_t)dims->workspace & 255))
        return RTP_ERR_WORKSPACE;

    KParams K;
    memset(&K, 0, sizeof(K));
    const long long rows =
        dims->block_table ? (long long)dims->num_pages * pl.Hkv * BLK : (long long)pl.B * pl.Hkv * pl.Ncap;
    if (!encode_cache_map(&K.tmk, k_cache, rows) || !encode_cache_map(&K.tmv, v_cache, rows)) {
        report(cudaErrorInvalidValue, "K/V tensor map");
        return RTP_ERR_CUDA;
    }
    unsigned long long ring_mask = 0;
    if (k_ring) {
        // the rings serve the local groups whose KV head has no retrieval head
        for (int i = 0; i < pl.n_lg; ++i) {
            bool pure = true;
            for (int r = 0; r < pl.n_rg; ++r) pure = pure && pl.rg_group[r] != pl.lg_group[i];
            if (pure) ring_mask |= 1ull << i;
        }
        const long long ring_rows = (long long)pl.B * pl.Hkv * (BLK + ring_W);
        if (!encode_cache_map(&K.tmk_r, k_ring, ring_rows) || !encode_cache_map(&K.tmv_r, v_ring, ring_rows)) {
            report(cudaErrorInvalidValue, "ring tensor map");
            return RTP_ERR_CUDA;
        }
    }
    Params& P = K.P;
    P.ring_lg_mask = ring_mask;
    P.ring_W = k_ring ? ring_W : 0;
    P.ring_rows = k_ring ? BLK + ring_W : 0;
    P.B = pl.B;
    P.Hq = pl.Hq;
    P.Hkv = pl.Hkv;
    P.G = pl.G;
    P.Ncap = pl.Ncap;
    P.sstride = pl.ntiles_cap * SROWS;
    P.nblk_cap = pl.nblk_cap;
    P.words_cap = pl.words_cap;
    P.ntiles_cap = pl.ntiles_cap;
    P.mbps = dims->max_blocks_per_seq;
    P.num_pages = dims->num_pages;
    P.window = window;
    P.sink = sink;
    P.n_ret = pl.n_ret;
    P.n_rg = pl.n_rg;
    P.n_lg = pl.n_lg;
    P.q_pre = q_pre;
    P.q_rope = q_rope;
    P.k_idx = k_idx;
    P.k_cache_ptr = k_cache;
    P.v_cache_ptr = v_cache;
    P.Wq = Wq_idx;
    P.seq_lens = seq_lens;
    P.block_table = dims->block_table;
    P.p = topk > 0 ? nullptr : p;
    P.topk = topk;
    P.out = out;
    memcpy(P.tab.rg_group, pl.rg_group, sizeof(P.tab.rg_group));
    memcpy(P.tab.rg_mask, pl.rg_mask, sizeof(P.tab.rg_mask));
    memcpy(P.tab.rg_slot0, pl.rg_slot0, sizeof(P.tab.rg_slot0));
    memcpy(P.tab.rg_nh, pl.rg_nh, sizeof(P.tab.rg_nh));
    memcpy(P.tab.lg_group, pl.lg_group, sizeof(P.tab.lg_group));
    memcpy(P.tab.lg_mask, pl.lg_mask, sizeof(P.tab.lg_mask));
    memcpy(P.tab.slot_head, pl.slot_head, sizeof(P.tab.slot_head));
    memcpy(P.tab.slot_rg, pl.slot_rg, sizeof(P.tab.slot_rg));
    uint8_t* ws = (uint8_t*)dims->workspace;
    P.status = (uint32_t*)(ws + pl.o_status);
    P.sync = (Sync*)(ws + pl.o_sync);
    P.rlist = (uint32_t*)(ws + pl.o_rlist);
    P.tick_score = (uint32_t*)(ws + pl.o_tick_score);
    P.tick_local = (uint32_t*)(ws + pl.o_tick_local);
    P.tick_ret = (uint32_t*)(ws + pl.o_tick_ret);
    P.tick_grp = (uint32_t*)(ws + pl.o_tick_grp);
    P.sel_cnt = (uint32_t*)(ws + pl.o_sel_cnt);
    P.sel_mass = (unsigned long long*)(ws + pl.o_sel_mass);
    P.sel_ncand = (uint32_t*)(ws + pl.o_sel_ncand);
    P.sel_above = (uint32_t*)(ws + pl.o_sel_above);
    P.sel_arrive = (uint32_t*)(ws + pl.o_sel_arrive);
    P.agg = (HeadAgg*)(ws + pl.o_agg);
    P.hs = (HeadState*)(ws + pl.o_hs);
    P.tie_cnt = (uint32_t*)(ws + pl.o_tie_cnt);
    P.scores = (float*)(ws + pl.o_scores);
    P.cand = (unsigned long long*)(ws + pl.o_cand);
    P.bitmap = (uint32_t*)(ws + pl.o_bitmap);
    P.blist = (uint32_t*)(ws + pl.o_blist);
    P.bcount = (uint32_t*)(ws + pl.o_bcount);
    P.lpart = (float*)(ws + pl.o_lpart);
    P.rpart = (float*)(ws + pl.o_rpart);
    if (dims->debug) {
        P.dbg_tau = dims->debug->tau;
        P.dbg_kstar = dims->debug->kstar;
        P.dbg_kept = dims->debug->kept_blocks;
        P.dbg_smax = dims->debug->smax;
        P.dbg_Z = dims->debug->Z;
        P.dbg_bitmap = dims->debug->block_bitmap;
        P.dbg_trace = dims->debug->trace;
    }
    cudaStream_t s = (cudaStream_t)stream;
    // (the no-alloc entry point: the scratch's zero region is cleared only
    // now that every host-side check has passed)
    if (clear_first && cudaMemsetAsync(ws, 0, pl.zero_end, s) != cudaSuccess) return RTP_ERR_CUDA;
    void* const* ev = (dims->timing_events && dims->n_timing_events >= RTP_TIMING_EVENTS) ? dims->timing_events : nullptr;
    // under stream capture the records must become event nodes of the graph
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (ev) cudaStreamIsCapturing(s, &cap);
    const unsigned ev_flags = (cap == cudaStreamCaptureStatusActive) ? cudaEventRecordExternal : cudaEventRecordDefault;
    if (ev) cudaEventRecordWithFlags((cudaEvent_t)ev[0], s, ev_flags);
    cudaError_t e;
    switch (pl.G) {
        case 1: e = launch<1>(K, pl, s, ev, ev_flags); break;
        case 2: e = launch<2>(K, pl, s, ev, ev_flags); break;
        case 4: e = launch<4>(K, pl, s, ev, ev_flags); break;
        default: e = launch<8>(K, pl, s, ev, ev_flags); break;
    }
    if (ev) cudaEventRecordWithFlags((cudaEvent_t)ev[2], s, ev_flags);
    return e == cudaSuccess ? RTP_OK : RTP_ERR_CUDA;
}

extern "C" rtp_status rtp_decode_step(const rtp_dims* dims, const uint16_t* q_pre, const uint16_t* q_rope,
                                      const uint16_t* k_idx, const uint16_t* k_cache, const uint16_t* v_cache,
                                      const uint16_t* Wq_idx, const int32_t* seq_lens, const uint8_t* head_kind,
                                      const float* p, int32_t window, int32_t sink, uint16_t* out, void* stream) {
    if (!p) return RTP_ERR_NULL;
    return decode_step_ws(dims, q_pre, q_rope, k_idx, k_cache, v_cache, nullptr, nullptr, 0, Wq_idx, seq_lens,
                          head_kind, p, 0, window, sink, out, stream);
}

extern "C" rtp_status rtp_decode_step_ring(const rtp_dims* dims, const uint16_t* q_pre, const uint16_t* q_rope,
                                           const uint16_t* k_idx, const uint16_t* k_cache, const uint16_t* v_cache,
                                           const uint16_t* k_ring, const uint16_t* v_ring, int32_t ring_W,
                                           const uint16_t* Wq_idx, const int32_t* seq_lens,
                                           const uint8_t* head_kind, const float* p, int32_t window, int32_t sink,
                                           uint16_t* out, void* stream) {
    if (!p || !k_ring || !v_ring) return RTP_ERR_NULL;
    return decode_step_ws(dims, q_pre, q_rope, k_idx, k_cache, v_cache, k_ring, v_ring, ring_W, Wq_idx, seq_lens,
                          head_kind, p, 0, window, sink, out, stream);
}

extern "C" rtp_status rtp_decode_step_topk(const rtp_dims* dims, const uint16_t* q_pre, const uint16_t* q_rope,
                                           const uint16_t* k_idx, const uint16_t* k_cache, const uint16_t* v_cache,
                                           const uint16_t* Wq_idx, const int32_t* seq_lens,
                                           const uint8_t* head_kind, int32_t topk, int32_t window, int32_t sink,
                                           uint16_t* out, void* stream) {
    if (topk < 1) return RTP_ERR_SHAPE;
    return decode_step_ws(dims, q_pre, q_rope, k_idx, k_cache, v_cache, nullptr, nullptr, 0, Wq_idx, seq_lens,
                          head_kind, nullptr, topk, window, sink, out, stream);
}

extern "C" rtp_status rtp_get_status(const rtp_dims* dims, void* stream) {
    if (!dims || !dims->workspace) return RTP_ERR_NULL;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaStreamSynchronize(s) != cudaSuccess) return RTP_ERR_CUDA;
    uint32_t word = 0;
    // the status word sits at offset 0 of the workspace
    if (cudaMemcpy(&word, dims->workspace, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return RTP_ERR_CUDA;
    if (word != 0 && cudaMemset(dims->workspace, 0, 4) != cudaSuccess) return RTP_ERR_CUDA;
    return (rtp_status)word;
}

// ---------------------------------------------------------------------------
// Allocation-free variant.  Callers that may not allocate device memory (an
// engine plugin whose pool owns every byte of the GPU, a loop that cannot take
// cudaMalloc's device-wide synchronisation) get the same step with its scratch
// in a device array built into the library.  The array is only reachable from
// host code through the address looked up below: its host-side name is a
// stand-in, not a device pointer.
namespace rtp {

static __device__ __align__(256) uint8_t noalloc_scratch[RTP_NOALLOC_SCRATCH_BYTES];

// Device address of noalloc_scratch in the current device's context, looked
// up on every call: the address belongs to the module as loaded into that
// context, and a context that was destroyed and made again (cudaDeviceReset)
// may hold the module at another address.  The lookup loads the module into
// the context if it is not loaded yet; after that it is a table lookup.
static cudaError_t noalloc_scratch_ptr(uint8_t** out) {
    void* a = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&a, noalloc_scratch);
    if (e != cudaSuccess) return e;
    if (!a) return cudaErrorInvalidSymbol;
    *out = static_cast<uint8_t*>(a);
    return cudaSuccess;
}

}  // namespace rtp

extern "C" rtp_status rtp_decode_step_noalloc(const rtp_dims* dims, const uint16_t* q_pre, const uint16_t* q_rope,
                                              const uint16_t* k_idx, const uint16_t* k_cache,
                                              const uint16_t* v_cache, const uint16_t* Wq_idx,
                                              const int32_t* seq_lens, const uint8_t* head_kind, const float* p,
                                              int32_t window, int32_t sink, uint16_t* out, uint32_t* device_status,
                                              void* stream) {
    // every host-side check runs before anything is enqueued
    if (!dims || !q_pre || !q_rope || !k_idx || !k_cache || !v_cache || !Wq_idx || !seq_lens || !head_kind || !p ||
        !out)
        return RTP_ERR_NULL;
    if (window < 0 || sink < 0 || (int64_t)window + sink < 1) return RTP_ERR_SHAPE;
    if (!aligned16(q_pre) || !aligned16(q_rope) || !aligned16(k_idx) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned16(Wq_idx) || !aligned16(out))
        return RTP_ERR_UNSUPPORTED;
    Plan pl;
    rtp_status st = make_plan(dims, head_kind, window, sink, &pl);
    if (st != RTP_OK) return st;
    if (pl.total > RTP_NOALLOC_SCRATCH_BYTES) return RTP_ERR_SCRATCH_LIMIT;
    uint8_t* ws = nullptr;
    if (noalloc_scratch_ptr(&ws) != cudaSuccess) return RTP_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    // The array keeps the previous call's contents, possibly laid out for
    // other sizes.  The kernels expect zero in the status word, the
    // coordination and ticket words, the per-head bucket aggregates and the
    // radix histograms, which the layout puts first ([0, zero_end)); every
    // other region is written before it is read.  The step clears that
    // region itself, after its host-side checks, so that a call refused on
    // the host enqueues nothing.
    rtp_dims d = *dims;
    d.workspace = ws;
    d.workspace_bytes = RTP_NOALLOC_SCRATCH_BYTES;
    st = decode_step_ws(&d, q_pre, q_rope, k_idx, k_cache, v_cache, nullptr, nullptr, 0, Wq_idx, seq_lens, head_kind,
                        p, 0, window, sink, out, stream, true);
    if (st != RTP_OK) return st;
    if (device_status &&
        cudaMemcpyAsync(device_status, ws + pl.o_status, sizeof(uint32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return RTP_ERR_CUDA;
    return RTP_OK;
}

// ---------------------------------------------------------------------------
// local heads' ring write
// ---------------------------------------------------------------------------
extern "C" rtp_status rtp_ring_write(const rtp_dims* d, const uint16_t* k_new, const uint16_t* v_new,
                                     const int32_t* pos, int32_t num_new, int32_t ring_W, uint16_t* k_ring,
                                     uint16_t* v_ring, uint32_t* device_status, void* stream) {
    if (!d) return RTP_ERR_NULL;
    if (d->head_dim != D || d->block_size != BLK) return RTP_ERR_UNSUPPORTED;
    if (d->batch < 1 || d->num_kv_heads < 1 || num_new < 0) return RTP_ERR_SHAPE;
    if (d->batch > MAX_B || d->num_kv_heads > MAX_HKV) return RTP_ERR_UNSUPPORTED;
    if (ring_W < BLK || ring_W % BLK) return RTP_ERR_SHAPE;
    if (num_new == 0) return RTP_OK;
    if (!k_new || !v_new || !pos || !k_ring || !v_ring) return RTP_ERR_NULL;
    if (((uintptr_t)k_new | (uintptr_t)v_new | (uintptr_t)k_ring | (uintptr_t)v_ring) & 15u)
        return RTP_ERR_UNSUPPORTED;
    RingParams A;
    A.B = d->batch;
    A.Hkv = d->num_kv_heads;
    A.T = num_new;
    A.W = ring_W;
    A.k_new = k_new;
    A.v_new = v_new;
    A.pos = pos;
    A.k_ring = k_ring;
    A.v_ring = v_ring;
    A.status = device_status;
    const int64_t threads = (int64_t)A.B * A.Hkv * A.T * 32;
    const int64_t grid = (threads + 255) / 256;
    if (grid > 0x7FFFFFFF) return RTP_ERR_UNSUPPORTED;
    ring_write_kernel<<<(unsigned)grid, 256, 0, (cudaStream_t)stream>>>(A);
    return report(cudaGetLastError(), "ring write launch") == cudaSuccess ? RTP_OK : RTP_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// index-cache append
// ---------------------------------------------------------------------------
// The index-cache append, with the KV-cache write when k_cache is given.
static rtp_status append_impl(const rtp_dims* d, const uint16_t* k_pre, const uint16_t* v_new, const uint16_t* Wk_idx,
                              const float* rope_cos, const float* rope_sin, const int32_t* pos, int32_t num_new,
                              uint16_t* k_idx, uint16_t* k_cache, uint16_t* v_cache, uint32_t* device_status,
                              void* stream) {
    const bool kv = k_cache != nullptr;
    if (!d) return RTP_ERR_NULL;
    if (d->head_dim != D || d->idx_dim != R || d->block_size != BLK) return RTP_ERR_UNSUPPORTED;
    if (d->batch < 1 || d->num_kv_heads < 1 || num_new < 0) return RTP_ERR_SHAPE;
    if (d->batch > MAX_B || d->num_kv_heads > MAX_HKV) return RTP_ERR_UNSUPPORTED;
    if (d->max_seq_len < BLK || d->max_seq_len % BLK || num_new > d->max_seq_len) return RTP_ERR_SHAPE;
    if (d->block_table) {
        if (d->max_blocks_per_seq < 1 || d->num_pages < 1) return RTP_ERR_SHAPE;
        if ((int64_t)d->max_blocks_per_seq * BLK != d->max_seq_len) return RTP_ERR_SHAPE;
    }
    if (num_new == 0) return RTP_OK;
    if (!k_pre || !Wk_idx || !pos || !k_idx) return RTP_ERR_NULL;
    if (kv && (!v_new || !rope_cos || !rope_sin || !v_cache)) return RTP_ERR_NULL;
    if (((uintptr_t)k_pre | (uintptr_t)Wk_idx) & 15u) return RTP_ERR_UNSUPPORTED;   // 16-byte vector loads
    if ((uintptr_t)k_idx & 7u) return RTP_ERR_UNSUPPORTED;                            // 8-byte stores of 4 entries
    if (kv && (((uintptr_t)v_new | (uintptr_t)rope_cos | (uintptr_t)rope_sin | (uintptr_t)k_cache |
                (uintptr_t)v_cache) & 15u))
        return RTP_ERR_UNSUPPORTED;                                                    // 16-byte loads and stores
    AppendParams A;
    memset(&A, 0, sizeof(A));
    A.B = d->batch;
    A.Hkv = d->num_kv_heads;
    A.T = num_new;
    A.Ncap = d->max_seq_len;
    A.mbps = d->block_table ? d->max_blocks_per_seq : 0;
    A.num_pages = d->block_table ? d->num_pages : 0;
    A.k_pre = k_pre;
    A.Wk = Wk_idx;
    A.pos = pos;
    A.block_table = d->block_table;
    A.k_idx = k_idx;
    A.status = device_status;
    A.v_new = v_new;
    A.rope_cos = rope_cos;
    A.rope_sin = rope_sin;
    A.k_cache = k_cache;
    A.v_cache = v_cache;
    const int64_t total = (int64_t)A.B * A.Hkv * A.T * (R / APPEND_ROWS);
    const int64_t grid = (total + APPEND_THREADS - 1) / APPEND_THREADS;
    if (grid > 0x7FFFFFFF) return RTP_ERR_UNSUPPORTED;
    if (kv) append_kernel<true><<<(unsigned)grid, APPEND_THREADS, 0, (cudaStream_t)stream>>>(A);
    else append_kernel<false><<<(unsigned)grid, APPEND_THREADS, 0, (cudaStream_t)stream>>>(A);
    return report(cudaGetLastError(), "append launch") == cudaSuccess ? RTP_OK : RTP_ERR_CUDA;
}

extern "C" rtp_status rtp_index_append(const rtp_dims* d, const uint16_t* k_pre, const uint16_t* Wk_idx,
                                       const int32_t* pos, int32_t num_new, uint16_t* k_idx, uint32_t* device_status,
                                       void* stream) {
    return append_impl(d, k_pre, nullptr, Wk_idx, nullptr, nullptr, pos, num_new, k_idx, nullptr, nullptr,
                       device_status, stream);
}

extern "C" rtp_status rtp_kv_append(const rtp_dims* d, const uint16_t* k_pre, const uint16_t* v_new,
                                    const uint16_t* Wk_idx, const float* rope_cos, const float* rope_sin,
                                    const int32_t* pos, int32_t num_new, uint16_t* k_idx, uint16_t* k_cache,
                                    uint16_t* v_cache, uint32_t* device_status, void* stream) {
    if (!k_cache) return RTP_ERR_NULL;
    return append_impl(d, k_pre, v_new, Wk_idx, rope_cos, rope_sin, pos, num_new, k_idx, k_cache, v_cache,
                       device_status, stream);
}

// ---------------------------------------------------------------------------
// prefill attention of a chunk of queries
// ---------------------------------------------------------------------------
extern "C" rtp_status rtp_prefill(const rtp_dims* d, const uint16_t* q, const uint16_t* k_cache,
                                  const uint16_t* v_cache, const uint8_t* head_kind, const int32_t* pos,
                                  int32_t num_q, int32_t window, int32_t sink, uint16_t* out,
                                  uint32_t* device_status, void* stream) {
    if (!d || !head_kind) return RTP_ERR_NULL;
    if (d->head_dim != D || d->block_size != BLK) return RTP_ERR_UNSUPPORTED;
    if (d->batch < 1 || d->num_q_heads < 1 || d->num_kv_heads < 1 || num_q < 0) return RTP_ERR_SHAPE;
    if (d->num_q_heads % d->num_kv_heads) return RTP_ERR_SHAPE;
    const int G = d->num_q_heads / d->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return RTP_ERR_UNSUPPORTED;
    if (d->num_q_heads > MAX_HQ || d->num_kv_heads > MAX_HKV || d->batch > MAX_B) return RTP_ERR_UNSUPPORTED;
    if (d->max_seq_len < BLK || d->max_seq_len % BLK || num_q > d->max_seq_len) return RTP_ERR_SHAPE;
    if (window < 0 || sink < 0 || (int64_t)window + sink < 1) return RTP_ERR_SHAPE;
    if (d->block_table) {
        if (d->max_blocks_per_seq < 1 || d->num_pages < 1) return RTP_ERR_SHAPE;
        if ((int64_t)d->max_blocks_per_seq * BLK != d->max_seq_len) return RTP_ERR_SHAPE;
        if ((int64_t)d->num_pages * d->num_kv_heads * BLK >= (1ll << 31)) return RTP_ERR_UNSUPPORTED;
    } else if ((int64_t)d->batch * d->num_kv_heads * d->max_seq_len >= (1ll << 31)) {
        return RTP_ERR_UNSUPPORTED;   // TMA row coordinates are 32-bit
    }
    if (num_q == 0) return RTP_OK;
    if (!q || !k_cache || !v_cache || !pos || !out) return RTP_ERR_NULL;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out)) return RTP_ERR_UNSUPPORTED;
    PrefillK K;
    memset(&K, 0, sizeof(K));
    PrefillParams& P = K.P;
    P.B = d->batch;
    P.Hq = d->num_q_heads;
    P.Hkv = d->num_kv_heads;
    P.G = G;
    P.Ncap = d->max_seq_len;
    P.mbps = d->block_table ? d->max_blocks_per_seq : 0;
    P.num_pages = d->block_table ? d->num_pages : 0;
    P.T = num_q;
    P.window = window;
    P.sink = sink;
    P.nt16 = (num_q + 15) / 16;
    // the tcgen05 kernel, sixteen units per CTA; RTP_PREFILL_TC=0 (read at
    // every call): the warp-MMA kernel, four
    const char* tcv = getenv("RTP_PREFILL_TC");
    const bool tc = !(tcv && atoi(tcv) == 0);
    const int units = tc ? PT_UNITS : PF_UNITS;
    // the (KV group, head kind) sets: retrieval heads first, then local heads, per group
    int cta = 0;
    for (int g = 0; g < P.Hkv; ++g)
        for (int kind = 1; kind >= 0; --kind) {
            int nh = 0;
            uint8_t heads[MAX_G];
            for (int i = 0; i < G; ++i) {
                const uint8_t k = head_kind[g * G + i];
                if (k > 1) return RTP_ERR_SHAPE;
                if (k == kind) heads[nh++] = (uint8_t)i;
            }
            if (!nh) continue;
            const int s = P.n_sets++;
            P.set_g[s] = (uint8_t)g;
            P.set_kind[s] = (uint8_t)kind;
            P.set_nh[s] = (uint8_t)nh;
            memcpy(P.set_heads[s], heads, nh);
            P.set_cta0[s] = cta;
            cta += (int)(((int64_t)nh * P.nt16 + units - 1) / units);
        }
    P.set_cta0[P.n_sets] = cta;
    P.cta_per_b = cta;
    const int64_t grid = (int64_t)P.B * cta;
    if (grid > 0x7FFFFFFF) return RTP_ERR_UNSUPPORTED;
    P.q = q;
    P.pos = pos;
    P.block_table = d->block_table;
    P.out = out;
    P.status = device_status;
    const long long rows = d->block_table ? (long long)d->num_pages * P.Hkv * BLK : (long long)P.B * P.Hkv * P.Ncap;
    if (!encode_cache_map(&K.tmk, k_cache, rows) || !encode_cache_map(&K.tmv, v_cache, rows)) {
        report(cudaErrorInvalidValue, "prefill K/V tensor map");
        return RTP_ERR_CUDA;
    }
    if (tc) {
        PrefillTcK T;
        T.tmk = K.tmk;
        T.tmv = K.tmv;
        T.P = P;
        const size_t smem = sizeof(PtSmem);
        if (occupancy((const void*)prefill_tc_kernel, smem, PT_THREADS) < 1) {
            report(cudaErrorInvalidConfiguration, "prefill tcgen05 kernel occupancy");
            return RTP_ERR_CUDA;
        }
        prefill_tc_kernel<<<(unsigned)grid, PT_THREADS, smem, (cudaStream_t)stream>>>(T);
        return report(cudaGetLastError(), "prefill tcgen05 launch") == cudaSuccess ? RTP_OK : RTP_ERR_CUDA;
    }
    const size_t smem = sizeof(PfSmem);
    if (occupancy((const void*)prefill_kernel, smem, PF_THREADS) < 1) {
        report(cudaErrorInvalidConfiguration, "prefill kernel occupancy");
        return RTP_ERR_CUDA;
    }
    prefill_kernel<<<(unsigned)grid, PF_THREADS, smem, (cudaStream_t)stream>>>(K);
    return report(cudaGetLastError(), "prefill launch") == cudaSuccess ? RTP_OK : RTP_ERR_CUDA;
}

extern "C" const char* rtp_status_string(rtp_status status) {
    switch (status) {
        case RTP_OK: return "ok";
        case RTP_ERR_NULL: return "null pointer";
        case RTP_ERR_SHAPE: return "inconsistent sizes";
        case RTP_ERR_UNSUPPORTED: return "unsupported sizes";
        case RTP_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case RTP_ERR_CUDA: return "CUDA error";
        case RTP_ERR_DEVICE_INPUT: return "device-side input error (seq_len, p or page id)";
        case RTP_ERR_TIMEOUT: return "a bounded wait inside a kernel timed out";
        case RTP_ERR_SCRATCH_LIMIT: return "sizes need more scratch than the no-alloc entry point's static array";
    }
    return "unknown status";
}
