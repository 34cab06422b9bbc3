// Prefill attention on the 5th-generation tensor cores (sm_100a), with
// 128-key tiles and two row groups per CTA: the same operation as
// prefill_kernel (rtp_prefill.cuh: retrieval heads dense and causal, local
// heads sink + window; review "RTPurbo" on dongryeollee1.github.io, Method:
// "Adaptive sparse attention", the prefill paragraph), with both
// contractions on tcgen05 and their accumulators in tensor memory.
//
// A CTA takes sixteen (head, 16-position) units of one (KV group, head kind)
// set: two row groups of M = 128 query rows that read the same KV head, so a
// 128-key K/V tile is loaded once for 256 rows.  One CTA per SM (192 KB of
// shared memory, all 512 tensor-memory columns).  Warp roles:
//   warps 0-7  softmax, row group rg = warp / 4, thread i of the group owns
//              row i (tensor-memory lane i)
//   warp 8     one lane issues every TMA load and every MMA
// Per tile k and row group g, in tensor memory: S_g (128 fp32 columns), then
// P_g (bf16 pairs) written over the first 64 of them, and O_g (128 columns).
//   S_g = Q_g K^T   tcgen05.mma M128 N128, eight K16 steps over the head dim
//   O_g += P_g V    tcgen05.mma M128 N128, eight K16 steps over the 128 keys,
//                   A = P_g from tensor memory, B = V (MN-major)
// The issuing lane orders, per tile: P V of tile k for group 0, S of tile
// k + 1 for group 0 (it may overwrite P_0 only after that P V, and the tensor
// cores run one lane's MMAs in order), then the same for group 1; so the
// tensor cores compute one group's products while the other group's softmax
// runs.  A group meets the issuing lane at two mbarriers per tile: S full
// (commit; it also means the group's previous P V is done, so O_g may be
// rescaled) and P full (the group's 128 threads).
// K and V tiles arrive by TMA, two 64-key blocks per tile, each as two 64 x
// 64 boxes with the 128-byte swizzle: box (head-dim half h, block b) at
// h * 16384 + b * 8192, so each half holds 128 consecutive key rows.  A block
// past the CTA's last query position is not loaded.
// Per tile a softmax thread makes two passes over its 128 scores, 64 at a
// time (the maximum, then 2^(s - m) into P), so its registers hold 64 scores.
#pragma once
#include "rtp_prefill.cuh"
#include "rtp_tc.cuh"

namespace rtp {

constexpr float PT_RESCALE = 8.f;            // log2 of the largest P before O is rescaled


__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
// 3-input maximum (one instruction on sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
// packed fp32 pair arithmetic (one instruction for two lanes' worth of work)
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1,%2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0,%1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// (lo, hi) -> bf16x2, round to nearest even; lo in the low half
__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// Shared-memory matrix descriptor of a 128-byte-swizzled operand: rows of 128
// bytes in 8-row atoms of 1024 bytes (`sbo` between atoms along the rows);
// `lbo` between 64-element column groups for an MN-major operand (unused,
// 16, for K-major).  Bits 61-63 = 2: the 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return smem_desc(saddr, lbo, sbo) | ((uint64_t)2 << 61);
}

// 32 consecutive 32-bit columns into this thread's tensor-memory lane, the
// store waited for inside the same asm.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
        "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
        "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

// D[tmem] (=|+=) A[tmem] . B[smem]^T, issued by one thread (A: M lanes, K
// packed two 16-bit elements per column).
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// bits [lo, hi) of a 64-bit word, the bounds clamped to [0, 64]
__device__ __forceinline__ uint64_t pt_bits(int lo, int hi) {
    lo = max(lo, 0);
    hi = min(hi, 64);
    if (hi <= lo) return 0ull;
    const uint64_t below_hi = hi >= 64 ? ~0ull : ((1ull << hi) - 1ull);
    return below_hi & ~((1ull << lo) - 1ull);
}

struct PrefillTcK {
    CUtensorMap tmk, tmv;   // K / V caches as [rows][128] bf16, 64 x 64 boxes, 128-byte swizzle
    PrefillParams P;
};

constexpr int PT_UNITS = 16;                 // (head, 16 positions) units per CTA: two groups of 128 rows
constexpr int PT_SOFT = 256;                 // softmax threads (warps 0-7)
constexpr int PT_THREADS = PT_SOFT + 32;     // + the TMA / MMA warp
constexpr int PT_TK = 2 * BLK;               // keys per tile
constexpr uint32_t PT_TM_COLS = 512;         // S_g / P_g at 128 g, O_g at 256 + 128 g

struct PtSmem {
    alignas(1024) uint8_t q[2][128 * 128 * 2];   // Q of group g: chunk (row r, dims 8c..) at c*2048 + r*16
    alignas(1024) uint8_t k[2][PT_TK * 128 * 2];   // K tiles (two stages), layout above
    alignas(1024) uint8_t v[2][PT_TK * 128 * 2];   // V tiles (two stages)
    alignas(8) uint64_t q_full;                  // Q copied (every softmax thread)
    uint64_t kfull[2], vfull[2];                 // TMA landed
    uint64_t kempty[2], vempty[2];               // the MMAs reading the stage are done (commit)
    uint64_t s_full[2];                          // [group] S computed, and the group's previous P V done
    uint64_t p_full[2];                          // [group] P written and O rescaled (the group's threads)
    uint64_t o_done[2];                          // [group] P V done (commit; its last phase gives the output)
    uint32_t tmem_base;
    volatile uint32_t abort;                     // a bounded wait gave up: every role leaves its loop
};

// The CTA's set, units and 128-key tiles (as pf_cta, with PT_UNITS units and
// tiles of PT_TK keys).
__device__ __forceinline__ PfCta pt_cta(const PrefillParams& P) {
    PfCta c;
    const int x = (int)blockIdx.x;
    c.b = x / P.cta_per_b;
    const int lc = x - c.b * P.cta_per_b;
    int lo = 0, hi = P.n_sets - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.set_cta0[mid] <= lc) lo = mid;
        else hi = mid - 1;
    }
    c.set = lo;
    c.g = P.set_g[lo];
    c.kind = P.set_kind[lo];
    c.nh = P.set_nh[lo];
    c.units = c.nh * P.nt16;
    c.u0 = (lc - P.set_cta0[lo]) * PT_UNITS;
    c.pos_b = __ldg(P.pos + c.b);
    c.ok = c.pos_b >= 0 && (long long)c.pos_b + P.T <= (long long)P.Ncap;
    const int ulast = min(c.u0 + PT_UNITS, c.units) - 1;
    const int pt_hi = P.nt16 - 1 - c.u0 / c.nh, pt_lo = P.nt16 - 1 - ulast / c.nh;
    c.m_lo = c.pos_b + 16 * pt_lo;
    c.m_hi = c.pos_b + min(16 * pt_hi + 15, P.T - 1);
    c.s_end = min(P.sink, c.m_hi + 1);
    c.w_lo = max(0, c.m_lo + 1 - P.window);
    if (c.kind == 1) {
        c.j0a = 0;
        c.j1a = c.m_hi / PT_TK + 1;
        c.j0b = c.j1b = c.j1a;
    } else {
        c.j0a = 0;
        c.j1a = (c.s_end + PT_TK - 1) / PT_TK;
        if (P.window > 0) {
            c.j0b = max(c.j1a, c.w_lo / PT_TK);
            c.j1b = max(c.j0b, c.m_hi / PT_TK + 1);
        } else {
            c.j0b = c.j1b = c.j1a;
        }
    }
    return c;
}

// Bounded mbarrier wait shared by all roles: false once this or another
// thread gave up (the CTA's abort flag), or after about two seconds (this
// thread then raises the flag and reports the timeout).
__device__ __forceinline__ bool pt_wait(uint64_t* bar, uint32_t parity, volatile uint32_t* abort,
                                        const PrefillParams& P) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 31u) == 0) {
            if (*abort) return false;
            if (global_ns() - t0 > 2000000000ull) {
                *abort = 1u;
                pf_status(P, ST_TIMEOUT);
                return false;
            }
        }
    }
}

__global__ void __launch_bounds__(PT_THREADS, 1) prefill_tc_kernel(const __grid_constant__ PrefillTcK K) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    PtSmem& S = *reinterpret_cast<PtSmem*>(smem_raw);
    const PrefillParams& P = K.P;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (smem_u32(smem_raw) & 1023u) {
        if (tid == 0) pf_status(P, 5u);
        return;
    }
    const PfCta c = pt_cta(P);
    if (!c.ok) {
        if (tid == 0) pf_status(P, ST_DEVICE_INPUT);   // this sequence's outputs are not written
        return;
    }
    if (tid == 0) {
        mbar_init(&S.q_full, PT_SOFT);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.kfull[i], 1);
            mbar_init(&S.vfull[i], 1);
            mbar_init(&S.kempty[i], 1);
            mbar_init(&S.vempty[i], 1);
            mbar_init(&S.s_full[i], 1);
            mbar_init(&S.p_full[i], 128);
            mbar_init(&S.o_done[i], 1);
        }
        S.abort = 0u;
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(&S.tmem_base, PT_TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = S.tmem_base;
    const int nt = c.ntiles();
    const bool retr = c.kind == 1;
    const int window = P.window, sink = P.sink;

    if (warp == 8) {
        // ================= TMA and MMA issue (lane 0; the warp zeroes unread value rows)
        constexpr uint32_t IDESC = idesc_bf16_f32(128, 128);
        constexpr uint32_t IDESC_O = IDESC | (1u << 16);   // B (V) MN-major
        const bool leader = lane == 0;
        // TMA of tile kt's K or V: its blocks up to the CTA's last query position
        auto load_tile = [&](const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int kt) {
            const int j0 = 2 * c.tile(kt);
            const int nb = (j0 + 1) * BLK <= c.m_hi ? 2 : 1;
            mbar_expect_tx(bar, (uint32_t)nb * BLK * 128 * 2);
            for (int bb = 0; bb < nb; ++bb) {
                const int r0 = pf_row(P, c.b, c.g, j0 + bb);
                tma_load_2d(dst + bb * 8192, map, 0, r0, bar);
                tma_load_2d(dst + 16384 + bb * 8192, map, 64, r0, bar);
            }
        };
        auto issue_s = [&](int g, int st) {   // S_g = Q_g K^T of the tile in K stage st
            tc_fence_after();
            const uint32_t qs = smem_u32(S.q[g]), kb = smem_u32(S.k[st]);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                umma_bf16(tbase + 128u * (uint32_t)g, smem_desc(qs + kk * 4096, 2048, 128),
                          smem_desc_sw128(kb + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024), IDESC, kk > 0);
            umma_commit(&S.s_full[g]);
        };
        bool ok = true;
        if (leader) {
            for (int j = 0; j < 2 && j < nt; ++j) {
                load_tile(&K.tmk, S.k[j], &S.kfull[j], j);
                load_tile(&K.tmv, S.v[j], &S.vfull[j], j);
            }
            ok = pt_wait(&S.q_full, 0u, &S.abort, P);
            if (ok && nt > 0) ok = pt_wait(&S.kfull[0], 0u, &S.abort, P);
            if (ok && nt > 0) {
                issue_s(0, 0);
                issue_s(1, 0);
                umma_commit(&S.kempty[0]);
            }
        }
        for (int k = 0; k < nt; ++k) {
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            const int st = k & 1, st1 = (k + 1) & 1;
            // V of tile k + 1 into the stage tile k - 1 used, once its P V are done
            if (leader && k >= 1 && k + 1 < nt) {
                ok = pt_wait(&S.vempty[st1], (uint32_t)((k - 1) >> 1) & 1u, &S.abort, P);
                if (ok) load_tile(&K.tmv, S.v[st1], &S.vfull[st1], k + 1);
            }
            // V of tile k landed; on an edge tile the value rows no row of the CTA
            // may read are zeroed (a cache row may hold anything, and 0 x NaN
            // would reach O through P = 0)
            const int n0 = c.tile(k) * PT_TK;
            const bool edge = n0 + PT_TK - 1 > c.m_hi || (!retr && n0 + PT_TK > c.s_end && n0 < c.w_lo);
            if (edge) {
                const bool landed = pt_wait(&S.vfull[st], (uint32_t)(k >> 1) & 1u, &S.abort, P);
                if (landed) {
                    const uint32_t vb = smem_u32(S.v[st]);
                    for (int x = lane; x < 2 * PT_TK; x += 32) {   // (key x / 2, head-dim half x % 2)
                        if (c.needed(n0 + (x >> 1), window)) continue;
                        const uint32_t rowa = vb + (uint32_t)((x & 1) * 16384 + (x >> 1) * 128);
#pragma unroll
                        for (int i = 0; i < 8; ++i) sts128(rowa + 16 * i, 0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async();
                }
                __syncwarp();
                if (!__all_sync(0xffffffffu, landed)) break;
            }
            if (leader) {
                if (!edge && ok) ok = pt_wait(&S.vfull[st], (uint32_t)(k >> 1) & 1u, &S.abort, P);
                // K of tile k + 1 landed
                if (ok && k + 1 < nt) ok = pt_wait(&S.kfull[st1], (uint32_t)((k + 1) >> 1) & 1u, &S.abort, P);
                const uint32_t vb = smem_u32(S.v[st]);
                for (int g = 0; g < 2 && ok; ++g) {
                    // O_g += P_g V once the group has written P_g ...
                    ok = pt_wait(&S.p_full[g], (uint32_t)k & 1u, &S.abort, P);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_bf16_ts(tbase + 256u + 128u * (uint32_t)g, tbase + 128u * (uint32_t)g + 8u * (uint32_t)kk,
                                     smem_desc_sw128(vb + kk * 2048, 16384, 1024), IDESC_O, (k > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&S.o_done[g]);
                    // ... then S_g of tile k + 1 over the same columns
                    if (k + 1 < nt) issue_s(g, st1);
                }
                if (ok) {
                    umma_commit(&S.vempty[st]);
                    if (k + 1 < nt) umma_commit(&S.kempty[st1]);
                }
                // K of tile k + 2 into the stage tile k used (its S MMAs were issued
                // one tile ago)
                if (ok && k + 2 < nt) {
                    ok = pt_wait(&S.kempty[st], (uint32_t)(k >> 1) & 1u, &S.abort, P);
                    if (ok) load_tile(&K.tmk, S.k[st], &S.kfull[st], k + 2);
                }
            }
        }
        // never leave with copies or MMAs of this CTA in flight: the softmax
        // threads wait for the last P V; the copies were all waited for
    } else {
        // ================= softmax: row group rg, row `row` (tensor-memory lane)
        const int rg = warp >> 2, row = tid & 127;
        const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
        const uint32_t t_s = tbase + lane_off + 128u * (uint32_t)rg;          // S_g; P_g in its first 64 columns
        const uint32_t t_o = tbase + lane_off + 256u + 128u * (uint32_t)rg;   // O_g
        const int u = c.u0 + 8 * rg + row / 16;
        const int t = u < c.units ? 16 * (P.nt16 - 1 - u / c.nh) + (row & 15) : P.T;
        const bool valid = u < c.units && t < P.T;
        const int h = c.g * P.G + P.set_heads[c.set][valid ? u % c.nh : 0];
        const int m = c.pos_b + t;
        // Q: this row's 16 chunks (zeros for a row past the units), made
        // visible to the tensor cores' proxy before the arrival
        {
            const uint32_t qs = smem_u32(S.q[rg]);
            if (valid) {
                const uint8_t* qrow = reinterpret_cast<const uint8_t*>(P.q + (((int64_t)c.b * P.Hq + h) * P.T + t) * D);
#pragma unroll
                for (int ch = 0; ch < 16; ++ch) cp_async16(qs + (uint32_t)(ch * 2048 + row * 16), qrow + ch * 16);
                cp_async_wait_all();
            } else {
#pragma unroll
                for (int ch = 0; ch < 16; ++ch) sts128(qs + (uint32_t)(ch * 2048 + row * 16), 0u, 0u, 0u, 0u);
            }
            fence_proxy_async();
            mbar_arrive(&S.q_full);
        }
        constexpr float SCALE = 0.08838834764831845f * 1.4426950408889634f;   // log2(e)/sqrt(128)
        // a tile with every key visible to every row of the CTA needs no mask
        auto interior = [&](int n0) {
            return n0 + PT_TK - 1 <= c.m_lo && (retr || n0 + PT_TK - 1 < sink || n0 > c.m_hi - window);
        };
        // the keys n0 + 64 half + i (i < 64) this row may read
        auto keep_bits = [&](int nh0) -> uint64_t {
            if (!valid) return 0ull;
            uint64_t keep = pt_bits(0, m - nh0 + 1);
            if (!retr) keep &= pt_bits(0, sink - nh0) | pt_bits(m - window + 1 - nh0, 64);
            return keep;
        };
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int k = 0; k < nt; ++k) {
            const int n0 = c.tile(k) * PT_TK;
            const bool full = valid && interior(n0);
            // (1) S_k (and the group's previous P V) done
            if (!(ok = pt_wait(&S.s_full[rg], (uint32_t)k & 1u, &S.abort, P))) break;
            tc_fence_after();
            // (2) the row maximum of the unscaled scores, 64 at a time
            float mx = -INFINITY;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                float s[64];
                tmem_ld64(t_s + 64u * (uint32_t)hf, s);
                if (!full) {
                    const uint64_t keep = keep_bits(n0 + 64 * hf);
#pragma unroll
                    for (int i = 0; i < 64; ++i)
                        if (!((keep >> i) & 1ull)) s[i] = -INFINITY;
                }
                float a[22];
#pragma unroll
                for (int i = 0; i < 21; ++i) a[i] = fmax3(s[3 * i], s[3 * i + 1], s[3 * i + 2]);
                a[21] = s[63];
                float b[8];
#pragma unroll
                for (int i = 0; i < 7; ++i) b[i] = fmax3(a[3 * i], a[3 * i + 1], a[3 * i + 2]);
                b[7] = a[21];
                mx = fmax3(mx, fmax3(fmax3(b[0], b[1], b[2]), fmax3(b[3], b[4], b[5]), fmaxf(b[6], b[7])), -INFINITY);
            }
            mx *= SCALE;
            float alpha = 1.f;
            if (mx > m_ref + PT_RESCALE) {
                alpha = m_ref == -INFINITY ? 1.f : ex2_approx(m_ref - mx);
                m_ref = mx;
            }
            // (3) O rescaled if the reference moved (the group's previous P V is done)
            if (k > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    float o[64];
                    tmem_ld64(t_o + 64 * half, o);
#pragma unroll
                    for (int i = 0; i < 64; ++i) o[i] *= alpha;
                    tmem_st64(t_o + 64 * half, o);
                }
            }
            // (4) P = 2^(s * SCALE - m_ref) as bf16 over the first 64 columns of S,
            // row sum in fp32 (a row with nothing visible yet has m_ref = -inf: P = 0)
            const float nb = m_ref == -INFINITY ? 0.f : -m_ref;
            const uint64_t sc2 = f2pack(SCALE, SCALE), nb2 = f2pack(nb, nb);
            uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                float s[64];
                tmem_ld64(t_s + 64u * (uint32_t)hf, s);
                if (!full) {
                    const uint64_t keep = keep_bits(n0 + 64 * hf);
#pragma unroll
                    for (int i = 0; i < 64; ++i)
                        if (!((keep >> i) & 1ull)) s[i] = -INFINITY;
                }
                uint32_t w[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    float x0, x1;
                    f2unpack(ffma2(f2pack(s[2 * i], s[2 * i + 1]), sc2, nb2), x0, x1);
                    const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                    acc[i & 3] = fadd2(acc[i & 3], f2pack(p0, p1));
                    w[i] = bf16x2(p0, p1);
                }
                tmem_st32(t_s + 32u * (uint32_t)hf, w);
            }
            float a0, a1, a2, a3;
            f2unpack(fadd2(acc[0], acc[1]), a0, a1);
            f2unpack(fadd2(acc[2], acc[3]), a2, a3);
            l = l * alpha + ((a0 + a2) + (a1 + a3));
            tc_fence_before();
            mbar_arrive(&S.p_full[rg]);
        }
        // ---- the output of this row, once the group's last P V is done
        if (ok && nt > 0) {
            ok = pt_wait(&S.o_done[rg], (uint32_t)(nt - 1) & 1u, &S.abort, P);
            tc_fence_after();
        }
        if (ok && nt > 0 && !S.abort) {
            uint4* orow = reinterpret_cast<uint4*>(P.out + (((int64_t)c.b * P.Hq + h) * P.T + t) * D);
            const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                float o[64];
                tmem_ld64(t_o + 64 * half, o);
                if (valid && l > 0.f) {
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        orow[8 * half + i] = make_uint4(
                            bf16x2(o[8 * i] * inv, o[8 * i + 1] * inv), bf16x2(o[8 * i + 2] * inv, o[8 * i + 3] * inv),
                            bf16x2(o[8 * i + 4] * inv, o[8 * i + 5] * inv), bf16x2(o[8 * i + 6] * inv, o[8 * i + 7] * inv));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_free(tbase, PT_TM_COLS);
    }
}

}  // namespace rtp
