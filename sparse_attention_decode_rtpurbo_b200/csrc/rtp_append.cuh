// Index-cache append (sm_100a): the retrieval key of every new token,
//     k_idx[b, g, pos[b] + t, r] = bf16( sum_i W^K[g, r, i] k_pre[b, g, t, i] ),
// written into the 16-dim bf16 index cache the decode step reads.
//
// Source: "Full Attention Strikes Back" (RTPurbo) review on
// dongryeollee1.github.io, Method: "Adaptive sparse attention" (the
// retrieval key k^idx_n = W^K k^pre_n, a rank-16 projection kept as a bf16
// cache); aitrends.kr summary, item 2 (low-rank retrieval routing).
//
// One thread per (token, 4 output rows): the 128 products of two bf16 values
// are exact in fp64 and each row's are summed in index order, then rounded
// once to bf16 (round to nearest even) -- the same value whichever thread or
// launch computes it; the four rows' chains run side by side.  The work is
// a few KB per token: bound by reading k_pre (256 B per token and KV head)
// and the fp64 pipe, far below any tensor-core shape.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "rtp_common.cuh"

namespace rtp {

struct AppendParams {
    int B, Hkv, T, Ncap, mbps, num_pages;
    const uint16_t* k_pre;     // [B, Hkv, T, 128]
    const uint16_t* Wk;        // [Hkv, 16, 128]
    const int32_t* pos;        // [B]
    const int32_t* block_table;
    uint16_t* k_idx;           // contiguous [B, Hkv, Ncap, 16] or paged [pages, Hkv, 64, 16]
    uint32_t* status;          // optional: RTP_ERR_DEVICE_INPUT for a bad pos or page id
};

constexpr int APPEND_THREADS = 256;
constexpr int APPEND_ROWS = 4;   // output rows per thread: independent fp64 chains over shared k_pre loads

__global__ void __launch_bounds__(APPEND_THREADS) index_append_kernel(const __grid_constant__ AppendParams A) {
    constexpr int RQ = R / APPEND_ROWS;          // threads per token
    const int64_t i = (int64_t)blockIdx.x * APPEND_THREADS + threadIdx.x;
    const int64_t total = (int64_t)A.B * A.Hkv * A.T * RQ;
    if (i >= total) return;
    const int r0 = (int)(i % RQ) * APPEND_ROWS;   // rows r0 .. r0 + 3
    const int64_t tok = i / RQ;                  // (b, g, t) in row-major order
    const int t = (int)(tok % A.T);
    const int g = (int)((tok / A.T) % A.Hkv);
    const int b = (int)(tok / ((int64_t)A.T * A.Hkv));
    const int64_t n = (int64_t)__ldg(A.pos + b) + t;
    if (n < 0 || n >= A.Ncap) {
        if (A.status) atomicCAS(A.status, 0u, ST_DEVICE_INPUT);
        return;
    }
    int64_t row;
    if (A.block_table) {
        const int pg = __ldg(A.block_table + (int64_t)b * A.mbps + n / BLK);
        if (pg < 0 || pg >= A.num_pages) {
            if (A.status) atomicCAS(A.status, 0u, ST_DEVICE_INPUT);
            return;
        }
        row = ((int64_t)pg * A.Hkv + g) * BLK + n % BLK;
    } else {
        row = ((int64_t)b * A.Hkv + g) * A.Ncap + n;
    }
    const uint4* kp = reinterpret_cast<const uint4*>(A.k_pre + tok * D);
    const uint4* w = reinterpret_cast<const uint4*>(A.Wk + ((int64_t)g * R + r0) * D);
    double acc[APPEND_ROWS];
#pragma unroll
    for (int q = 0; q < APPEND_ROWS; ++q) acc[q] = 0.0;
    // every row's sum runs over i = 0 .. 127 in order (one fma per product,
    // exact products): the same bits however the rows are interleaved
#pragma unroll 2
    for (int c = 0; c < D / 8; ++c) {
        const uint4 kv = __ldg(kp + c);
        const uint32_t ku[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
        for (int q = 0; q < APPEND_ROWS; ++q) {
            const uint4 wv = __ldg(w + q * (D / 8) + c);
            const uint32_t wu[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                acc[q] = fma((double)bf_lo(wu[j]), (double)bf_lo(ku[j]), acc[q]);
                acc[q] = fma((double)bf_hi(wu[j]), (double)bf_hi(ku[j]), acc[q]);
            }
        }
    }
    uint16_t o[APPEND_ROWS];
#pragma unroll
    for (int q = 0; q < APPEND_ROWS; ++q) o[q] = __bfloat16_as_ushort(__double2bfloat16(acc[q]));
    *reinterpret_cast<uint2*>(A.k_idx + row * R + r0) =
        make_uint2((uint32_t)o[0] | ((uint32_t)o[1] << 16), (uint32_t)o[2] | ((uint32_t)o[3] << 16));
}

}  // namespace rtp

namespace rtp {

// Ring write: new key and value rows of local-only KV heads into their rings
// of 64 + W rows (position n < 64 in row n, n >= 64 in row 64 + n mod W).
// One warp per (sequence, KV head, new token): lanes 0..15 copy the key row,
// 16..31 the value row, 16 bytes each.  A token whose row a later token of
// the same call also maps to (n >= 64 and n + W <= the call's last position)
// is skipped, so the result is that of writing the tokens in order, whatever
// the order the warps run in.
struct RingParams {
    int B, Hkv, T, W;
    const uint16_t* k_new;     // [B, Hkv, T, 128]
    const uint16_t* v_new;
    const int32_t* pos;        // [B]
    uint16_t* k_ring;          // [B, Hkv, 64 + W, 128]
    uint16_t* v_ring;
    uint32_t* status;          // optional: RTP_ERR_DEVICE_INPUT for a negative position
};

__global__ void __launch_bounds__(256) ring_write_kernel(const __grid_constant__ RingParams A) {
    const int64_t w = ((int64_t)blockIdx.x * 256 + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t total = (int64_t)A.B * A.Hkv * A.T;
    if (w >= total) return;
    const int t = (int)(w % A.T);
    const int b = (int)(w / ((int64_t)A.T * A.Hkv));
    const int64_t p0 = (int64_t)__ldg(A.pos + b);
    const int64_t n = p0 + t;
    if (p0 < 0) {
        if (A.status && lane == 0) atomicCAS(A.status, 0u, ST_DEVICE_INPUT);
        return;
    }
    if (n >= BLK && n + A.W <= p0 + A.T - 1) return;   // a later token of this call takes the row
    const int64_t slot = n < BLK ? n : BLK + n % A.W;
    const int64_t ring_row = (w / A.T) * (BLK + A.W) + slot;   // (b, g) = w / T
    const int c = lane & 15;
    const uint4* src = reinterpret_cast<const uint4*>((lane < 16 ? A.k_new : A.v_new) + w * D) + c;
    uint4* dst = reinterpret_cast<uint4*>((lane < 16 ? A.k_ring : A.v_ring) + ring_row * D) + c;
    *dst = __ldg(src);
}

}  // namespace rtp
