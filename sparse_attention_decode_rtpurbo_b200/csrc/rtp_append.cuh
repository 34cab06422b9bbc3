// Index-cache append (sm_100a): the retrieval key of every new token,
//     k_idx[b, g, pos[b] + t, r] = bf16( sum_i W^K[g, r, i] k_pre[b, g, t, i] ),
// written into the 16-dim bf16 index cache the decode step reads.
//
// Source: "Full Attention Strikes Back" (RTPurbo) review on
// dongryeollee1.github.io, Method: "Adaptive sparse attention" (the
// retrieval key k^idx_n = W^K k^pre_n, a rank-16 projection kept as a bf16
// cache); aitrends.kr summary, item 2 (low-rank retrieval routing).
//
// One thread per token and KV head, all 16 output rows: the 128 products of
// two bf16 values are exact in fp64 and each row's are summed in index
// order, then rounded once to bf16 (round to nearest even) -- the same value
// whichever thread or launch computes it.  The 16 rows' chains run side by
// side (a chain of 128 dependent fp64 fused multiply-adds is the latency
// that bounds the kernel; 16 of them in flight per thread hide it).  The work
// is a few KB per token: bound by reading k_pre (256 B per token and KV
// head) and the fp64 pipe, far below any tensor-core shape.
//
// The KV-cache write (kv_append) runs in the same threads: for each quarter
// q the thread rotates the key pairs (i, i + 64) for i in [16q, 16q + 16) by
// the caller's angle table,
//     y_i = k_i cos - k_{i+64} sin,   y_{i+64} = k_{i+64} cos + k_i sin,
// each the fp64 fused multiply-add of one exact product onto the other
// (a bf16 times an fp32 value is exact in fp64), rounded to bf16, and copies
// the bytes [64q, 64q + 64) of the token's value row.  Source: the same
// review, Method: "Adaptive sparse attention" (the indexer reads pre-RoPE
// keys, the attention RoPE'd ones) and Insight 2 (RoPE as a rotation of
// frequency pairs by position-proportional angles).
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
    // KV-cache write (kv_append only)
    const uint16_t* v_new;     // [B, Hkv, T, 128]
    const float* rope_cos;     // [Ncap, 64]: row n = the angles of cache position n
    const float* rope_sin;     // [Ncap, 64]
    uint16_t* k_cache;         // contiguous [B, Hkv, Ncap, 128] or paged [pages, Hkv, 64, 128]
    uint16_t* v_cache;         // same layout as k_cache
};

constexpr int APPEND_THREADS = 256;
constexpr int APPEND_ROWS = R;   // output rows per thread: independent fp64 chains over shared k_pre loads

// KV = false: the index-cache append alone; KV = true: with the KV-cache write.
template <bool KV>
__global__ void __launch_bounds__(APPEND_THREADS) append_kernel(const __grid_constant__ AppendParams A) {
    constexpr int RQ = R / APPEND_ROWS;          // threads per token
    const int64_t i = (int64_t)blockIdx.x * APPEND_THREADS + threadIdx.x;
    const int64_t total = (int64_t)A.B * A.Hkv * A.T * RQ;
    if (i >= total) return;
    const int r0 = (int)(i % RQ) * APPEND_ROWS;   // rows r0 .. r0 + APPEND_ROWS - 1
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
#pragma unroll
    for (int q = 0; q < APPEND_ROWS; q += 4)   // 8-byte stores: the cache is only 8-byte aligned
        *reinterpret_cast<uint2*>(A.k_idx + row * R + r0 + q) =
            make_uint2((uint32_t)o[q] | ((uint32_t)o[q + 1] << 16), (uint32_t)o[q + 2] | ((uint32_t)o[q + 3] << 16));
    if constexpr (KV) {
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {                 // quarter: pairs 16q .. 16q+15, value bytes 64q .. 64q+63
        const int64_t n16 = n * (D / 2);            // the angle table's row n (64 floats)
        const float4* cs = reinterpret_cast<const float4*>(A.rope_cos + n16) + q * 4;
        const float4* sn = reinterpret_cast<const float4*>(A.rope_sin + n16) + q * 4;
        uint4* kd = reinterpret_cast<uint4*>(A.k_cache + row * D);
#pragma unroll
        for (int h = 0; h < 2; ++h) {               // 8 pairs per half: one 16-byte chunk of each half-row
            const uint4 lo4 = __ldg(kp + 2 * q + h), hi4 = __ldg(kp + 8 + 2 * q + h);
            const uint32_t lu[4] = {lo4.x, lo4.y, lo4.z, lo4.w}, hu[4] = {hi4.x, hi4.y, hi4.z, hi4.w};
            const float4 c0 = __ldg(cs + 2 * h), c1 = __ldg(cs + 2 * h + 1);
            const float4 s0 = __ldg(sn + 2 * h), s1 = __ldg(sn + 2 * h + 1);
            const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
            const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
            uint32_t ylo[4], yhi[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint16_t lo_out[2], hi_out[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const double kl = (double)(e ? bf_hi(lu[j]) : bf_lo(lu[j]));
                    const double kh = (double)(e ? bf_hi(hu[j]) : bf_lo(hu[j]));
                    const double c = (double)cv[2 * j + e], s = (double)sv[2 * j + e];
                    lo_out[e] = __bfloat16_as_ushort(__double2bfloat16(fma(kl, c, -(kh * s))));
                    hi_out[e] = __bfloat16_as_ushort(__double2bfloat16(fma(kh, c, kl * s)));
                }
                ylo[j] = (uint32_t)lo_out[0] | ((uint32_t)lo_out[1] << 16);
                yhi[j] = (uint32_t)hi_out[0] | ((uint32_t)hi_out[1] << 16);
            }
            kd[2 * q + h] = make_uint4(ylo[0], ylo[1], ylo[2], ylo[3]);
            kd[8 + 2 * q + h] = make_uint4(yhi[0], yhi[1], yhi[2], yhi[3]);
        }
        const uint4* vs = reinterpret_cast<const uint4*>(A.v_new + tok * D) + q * 4;
        uint4* vd = reinterpret_cast<uint4*>(A.v_cache + row * D) + q * 4;
#pragma unroll
        for (int c = 0; c < 4; ++c) vd[c] = __ldg(vs + c);
      }
    }
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
