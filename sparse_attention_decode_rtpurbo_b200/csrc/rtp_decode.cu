// C ABI of the RTPurbo decode step: argument checks, workspace layout and the
// launch of the persistent sm_100a decode-step kernel (rtp_step.cuh, rtp_step_kernel.cuh).
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "../../include/rtp_decode.h"
#include "rtp_step_kernel.cuh"

namespace rtp {

constexpr int NSM_PLAN = 148;       // SMs of a B200: sizes the split counts
constexpr int MAX_GRID = 148 * 4;   // upper bound of the persistent grid (partials are sized for it)

struct Plan {
    int B, Hq, Hkv, G, Ncap, nblk_cap, words_cap, nchunks, nschunks;
    int n_ret, n_rg, n_lg;
    int local_kb, local_items, ret_grid;
    uint8_t rg_group[MAX_HKV], rg_mask[MAX_HKV], rg_slot0[MAX_HKV], rg_nh[MAX_HKV];
    uint8_t lg_group[MAX_HKV], lg_mask[MAX_HKV];
    uint8_t slot_head[MAX_HQ], slot_rg[MAX_HQ];
    // workspace byte offsets
    size_t o_status, o_sync, o_rlist, o_rglist, o_tick_score, o_tick_radix, o_tick_local, o_tick_ret, o_keys, o_agg,
        o_hs, o_hist_cnt, o_hist_mass, o_chunk_cnt, o_tie_off, o_bitmap, o_blist, o_bcount, o_lpart, o_rpart, total;
};

static size_t align_up(size_t x) { return (x + 255) & ~(size_t)255; }

static rtp_status check_dims(const rtp_dims* d) {
    if (!d) return RTP_ERR_NULL;
    if (d->head_dim != D || d->idx_dim != R || d->block_size != BLK) return RTP_ERR_UNSUPPORTED;
    if (d->batch < 1 || d->num_q_heads < 1 || d->num_kv_heads < 1) return RTP_ERR_SHAPE;
    if (d->num_q_heads % d->num_kv_heads) return RTP_ERR_SHAPE;
    const int G = d->num_q_heads / d->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return RTP_ERR_UNSUPPORTED;
    if (d->num_q_heads > MAX_HQ || d->num_kv_heads > MAX_HKV) return RTP_ERR_UNSUPPORTED;
    if (d->max_seq_len < BLK || d->max_seq_len % BLK) return RTP_ERR_SHAPE;
    if (d->max_seq_len > (1 << 28)) return RTP_ERR_UNSUPPORTED;
    if (d->block_table) {
        if (d->max_blocks_per_seq < 1 || d->num_pages < 1) return RTP_ERR_SHAPE;
        if ((int64_t)d->max_blocks_per_seq * BLK != d->max_seq_len) return RTP_ERR_SHAPE;
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
    pl->nchunks = (pl->Ncap + CHUNK - 1) / CHUNK;
    pl->nschunks = (pl->Ncap + SCORE_CHUNK - 1) / SCORE_CHUNK;
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
    // local heads: list of at most nv_max blocks per (b, group), cut into items
    if (pl->n_lg) {
        const int64_t nv_max = std::min<int64_t>(pl->nblk_cap, (sink + BLK - 1) / BLK + (window + BLK - 1) / BLK + 1);
        const int64_t total = (int64_t)pl->B * pl->n_lg * nv_max;
        pl->local_kb = (int)std::max<int64_t>(4, (total + 2 * NSM_PLAN - 1) / (2 * NSM_PLAN));
        // the split combine keeps one weight per (head, split) in 512*G floats
        pl->local_kb = (int)std::max<int64_t>(pl->local_kb, (nv_max + 511) / 512);
        pl->local_items = (int)((nv_max + pl->local_kb - 1) / pl->local_kb);
    }
    pl->ret_grid = MAX_GRID;
    // workspace layout
    const size_t BR = (size_t)pl->B * pl->n_ret, BG = (size_t)pl->B * pl->n_rg, BL = (size_t)pl->B * pl->n_lg;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = align_up(o + bytes);
        return at;
    };
    pl->o_status = take(64);
    pl->o_sync = take(sizeof(Sync));
    pl->o_rlist = take(BR * 4);
    pl->o_rglist = take(BG * 4);
    pl->o_tick_score = take(BG * 4);
    pl->o_tick_radix = take(BR * 4);
    pl->o_tick_local = take(BL * 4);
    pl->o_tick_ret = take(BG * 4);
    pl->o_keys = take(BR * pl->Ncap * 4);
    pl->o_agg = take(BR * AGG_BUCKETS * sizeof(HeadAgg));
    pl->o_hs = take(BR * sizeof(HeadState));
    pl->o_hist_cnt = take(BR * 256 * 4);
    pl->o_hist_mass = take(BR * 256 * 8);
    pl->o_chunk_cnt = take(BR * pl->nchunks * 256 * 4);
    pl->o_tie_off = take(BR * pl->nchunks * 4);
    pl->o_bitmap = take(BR * pl->words_cap * 4);
    pl->o_blist = take(BG * pl->nblk_cap * 4);
    pl->o_bcount = take(BG * 4);
    // B*n_lg*local_items <= total/local_kb + B*n_lg <= 2*NSM_PLAN + B*n_lg for any window and sink
    pl->o_lpart = take(((size_t)2 * NSM_PLAN + BL) * pl->G * PSTRIDE * 4);
    pl->o_rpart = take(((size_t)pl->ret_grid + BG) * pl->G * PSTRIDE * 4);
    pl->total = o;
    return RTP_OK;
}

template <int G>
static cudaError_t launch_step(const Params& P, const Plan& pl, uint8_t* ws, cudaStream_t s, void* const* ev) {
    const size_t smem = sizeof(StepSmem<G>);
    static std::atomic<int> ctas_per_sm{0};
    static std::atomic<int> num_sms{0};
    if (!ctas_per_sm.load()) {
        cudaError_t e = cudaFuncSetAttribute(step_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        int n = 0, dev = 0, sms = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, step_kernel<G>, STEP_THREADS, smem);
        if (e != cudaSuccess) return e;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        num_sms.store(sms);
        ctas_per_sm.store(std::max(1, n));
    }
    // under stream capture the records must become event nodes of the graph
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (ev) cudaStreamIsCapturing(s, &cap);
    const unsigned ev_flags = (cap == cudaStreamCaptureStatusActive) ? cudaEventRecordExternal : cudaEventRecordDefault;
    StepParams SP;
    SP.P = P;
    SP.sync = reinterpret_cast<Sync*>(ws + pl.o_sync);
    SP.rlist = reinterpret_cast<uint32_t*>(ws + pl.o_rlist);
    SP.rglist = reinterpret_cast<uint32_t*>(ws + pl.o_rglist);
    SP.n_score_items = pl.B * pl.n_rg * pl.nschunks;
    SP.n_local_items = pl.B * pl.n_lg * pl.local_items;
    const int grid = std::min(MAX_GRID, ctas_per_sm.load() * num_sms.load());
    if (ev) cudaEventRecordWithFlags((cudaEvent_t)ev[0], s, ev_flags);
    step_kernel<G><<<grid, STEP_THREADS, smem, s>>>(SP);
    if (ev) cudaEventRecordWithFlags((cudaEvent_t)ev[1], s, ev_flags);
    return cudaGetLastError();
}

}  // namespace rtp

using namespace rtp;

extern "C" size_t rtp_workspace_size(const rtp_dims* dims, const uint8_t* head_kind) {
    Plan pl;
    if (make_plan(dims, head_kind, 0, 1, &pl) != RTP_OK) return 0;
    return pl.total;
}

extern "C" rtp_status rtp_decode_step(const rtp_dims* dims, const uint16_t* q_pre, const uint16_t* q_rope,
                                      const uint16_t* k_idx, const uint16_t* k_cache, const uint16_t* v_cache,
                                      const uint16_t* Wq_idx, const int32_t* seq_lens, const uint8_t* head_kind,
                                      const float* p, int32_t window, int32_t sink, uint16_t* out, void* stream) {
    if (!dims || !q_pre || !q_rope || !k_idx || !k_cache || !v_cache || !Wq_idx || !seq_lens || !head_kind || !p ||
        !out)
        return RTP_ERR_NULL;
    if (window < 0 || sink < 0 || (int64_t)window + sink < 1) return RTP_ERR_SHAPE;
    Plan pl;
    rtp_status st = make_plan(dims, head_kind, window, sink, &pl);
    if (st != RTP_OK) return st;
    if (!dims->workspace || dims->workspace_bytes < pl.total || ((uintptr_t)dims->workspace & 255))
        return RTP_ERR_WORKSPACE;

    Params P;
    memset(&P, 0, sizeof(P));
    P.B = pl.B;
    P.Hq = pl.Hq;
    P.Hkv = pl.Hkv;
    P.G = pl.G;
    P.Ncap = pl.Ncap;
    P.nblk_cap = pl.nblk_cap;
    P.words_cap = pl.words_cap;
    P.mbps = dims->max_blocks_per_seq;
    P.num_pages = dims->num_pages;
    P.window = window;
    P.sink = sink;
    P.n_ret = pl.n_ret;
    P.n_rg = pl.n_rg;
    P.n_lg = pl.n_lg;
    P.nchunks = pl.nchunks;
    P.nschunks = pl.nschunks;
    P.local_kb = pl.local_kb;
    P.local_items = pl.local_items;
    P.ret_grid = pl.ret_grid;
    P.q_pre = q_pre;
    P.q_rope = q_rope;
    P.k_idx = k_idx;
    P.k_cache = k_cache;
    P.v_cache = v_cache;
    P.Wq = Wq_idx;
    P.seq_lens = seq_lens;
    P.block_table = dims->block_table;
    P.p = p;
    P.out = out;
    memcpy(P.rg_group, pl.rg_group, sizeof(P.rg_group));
    memcpy(P.rg_mask, pl.rg_mask, sizeof(P.rg_mask));
    memcpy(P.rg_slot0, pl.rg_slot0, sizeof(P.rg_slot0));
    memcpy(P.rg_nh, pl.rg_nh, sizeof(P.rg_nh));
    memcpy(P.lg_group, pl.lg_group, sizeof(P.lg_group));
    memcpy(P.lg_mask, pl.lg_mask, sizeof(P.lg_mask));
    memcpy(P.slot_head, pl.slot_head, sizeof(P.slot_head));
    memcpy(P.slot_rg, pl.slot_rg, sizeof(P.slot_rg));
    uint8_t* ws = (uint8_t*)dims->workspace;
    P.status = (uint32_t*)(ws + pl.o_status);
    P.tick_score = (uint32_t*)(ws + pl.o_tick_score);
    P.tick_radix = (uint32_t*)(ws + pl.o_tick_radix);
    P.tick_local = (uint32_t*)(ws + pl.o_tick_local);
    P.tick_ret = (uint32_t*)(ws + pl.o_tick_ret);
    P.keys = (uint32_t*)(ws + pl.o_keys);
    P.agg = (HeadAgg*)(ws + pl.o_agg);
    P.hs = (HeadState*)(ws + pl.o_hs);
    P.hist_cnt = (uint32_t*)(ws + pl.o_hist_cnt);
    P.hist_mass = (unsigned long long*)(ws + pl.o_hist_mass);
    P.chunk_cnt = (uint32_t*)(ws + pl.o_chunk_cnt);
    P.tie_off = (uint32_t*)(ws + pl.o_tie_off);
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
    void* const* ev = (dims->timing_events && dims->n_timing_events >= RTP_TIMING_EVENTS) ? dims->timing_events : nullptr;
    cudaError_t e;
    switch (pl.G) {
        case 1: e = launch_step<1>(P, pl, ws, s, ev); break;
        case 2: e = launch_step<2>(P, pl, ws, s, ev); break;
        case 4: e = launch_step<4>(P, pl, ws, s, ev); break;
        default: e = launch_step<8>(P, pl, ws, s, ev); break;
    }
    return e == cudaSuccess ? RTP_OK : RTP_ERR_CUDA;
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

constexpr int NOALLOC_MAX_DEVICES = 64;
static std::atomic<void*> noalloc_addr[NOALLOC_MAX_DEVICES];
static std::mutex noalloc_mutex;

// Device address of noalloc_scratch on the current device, looked up once per
// device (the lookup loads the module onto the device if needed).
static cudaError_t noalloc_scratch_ptr(uint8_t** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= NOALLOC_MAX_DEVICES) return cudaErrorInvalidDevice;
    void* a = noalloc_addr[dev].load(std::memory_order_acquire);
    if (!a) {
        std::lock_guard<std::mutex> lock(noalloc_mutex);
        a = noalloc_addr[dev].load(std::memory_order_acquire);
        if (!a) {
            e = cudaGetSymbolAddress(&a, noalloc_scratch);
            if (e != cudaSuccess) return e;
            if (!a) return cudaErrorInvalidSymbol;
            noalloc_addr[dev].store(a, std::memory_order_release);
        }
    }
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
    Plan pl;
    rtp_status st = make_plan(dims, head_kind, window, sink, &pl);
    if (st != RTP_OK) return st;
    if (pl.total > RTP_NOALLOC_SCRATCH_BYTES) return RTP_ERR_SCRATCH_LIMIT;
    uint8_t* ws = nullptr;
    if (noalloc_scratch_ptr(&ws) != cudaSuccess) return RTP_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    // The array keeps the previous call's contents, possibly laid out for
    // other sizes.  The kernel expects zero in the status word, the
    // cross-CTA counters and ticket words ([0, o_keys)) and in the per-head
    // bucket aggregates and radix histograms ([o_agg, o_chunk_cnt)); every
    // other region is written before it is read.
    if (cudaMemsetAsync(ws, 0, pl.o_keys, s) != cudaSuccess) return RTP_ERR_CUDA;
    if (cudaMemsetAsync(ws + pl.o_agg, 0, pl.o_chunk_cnt - pl.o_agg, s) != cudaSuccess) return RTP_ERR_CUDA;
    rtp_dims d = *dims;
    d.workspace = ws;
    d.workspace_bytes = RTP_NOALLOC_SCRATCH_BYTES;
    st = rtp_decode_step(&d, q_pre, q_rope, k_idx, k_cache, v_cache, Wq_idx, seq_lens, head_kind, p, window, sink,
                         out, stream);
    if (st != RTP_OK) return st;
    if (device_status &&
        cudaMemcpyAsync(device_status, ws + pl.o_status, sizeof(uint32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return RTP_ERR_CUDA;
    return RTP_OK;
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
