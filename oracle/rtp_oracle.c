/*
 * fp64 CPU oracle for the RTPurbo decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path loads this file: it
 * is called by the tests, by __graft_entry__.smoke() and by the benchmark's
 * CPU-baseline leg, to check and to time the CUDA path.  It shares no code,
 * header, table or constant with the CUDA sources.
 *
 * What it computes, per sequence b and query head h (sources: "Full
 * Attention Strikes Back" / RTPurbo -- the paper review on
 * dongryeollee1.github.io, section Method: "Adaptive sparse attention"
 * (its equation for s_h(m,n) and S_h(m) = Top-P(s_h(m,.), p)) and
 * "Hardware-aware top-p decoding kernel" (block mask, cumulative mass
 * reaching p_top); and the aitrends.kr summary, items 2 "Low-rank Retrieval
 * Routing" (O_h(m) as a softmax over S_h(m)) and 5 (block-sparse attention)):
 *
 *   local head     : attend over P = [0, min(sink,L)) U [max(0,L-window), L)
 *   retrieval head : q_idx = W^Q_h q^pre                      (16-vector)
 *                    s_n   = q_idx . k_idx_n,  n < L           (index score)
 *                    z_n   = s_n / sqrt(16)                    (top-p temperature)
 *                    pi    = softmax(z)
 *                    order tokens by (s desc, n asc); k* = smallest k whose
 *                    prefix mass reaches p (>= p); p >= 1 keeps every token
 *                    T = first k* tokens; blocks K = { floor(n/64) : n in T }
 *                    P = union of [64j, min(64j+64, L)) over j in K
 *   both           : a_n = q_rope . k_n / sqrt(128), w = softmax(a over P),
 *                    out = sum_n w_n v_n
 *
 * Everything is fp64, from the exact upcast of the bf16 inputs, with no
 * blocking or reordering beyond the definitions above.  A sequence's p is
 * meant to lie in (0, 1]; p >= 1 keeps every token, p <= 0 or NaN is an
 * input error.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_D 128
#define ORC_R 16
#define ORC_BLK 64

static double bf(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* cache geometry: contiguous [B,Hkv,Ncap,dim] or paged [pages,Hkv,64,dim] */
typedef struct {
    int B, Hq, Hkv;
    int64_t Ncap;
    const int32_t* block_table; /* NULL = contiguous */
    int mbps;                   /* max blocks per sequence (paged) */
} geom;

static const uint16_t* row(const geom* g, const uint16_t* base, int dim, int b, int kv, int64_t n) {
    if (!g->block_table) return base + (((int64_t)b * g->Hkv + kv) * g->Ncap + n) * dim;
    int64_t page = g->block_table[(int64_t)b * g->mbps + n / ORC_BLK];
    return base + ((page * g->Hkv + kv) * ORC_BLK + n % ORC_BLK) * dim;
}

/* RoPE, rotate-half pairing (i, i+64), angle pos * theta^(-2i/128): the
 * relative-position form of the review's "RoPE ... low-dim subspace" insight
 * (score = sum_i a_i cos(theta_i D) + b_i sin(theta_i D), D = m - n). */
void oracle_rope(const double* x, int64_t pos, double theta, double* y) {
    double t[ORC_D];
    for (int i = 0; i < 64; ++i) {
        double a = (double)pos * pow(theta, -2.0 * (double)i / 128.0);
        double c = cos(a), s = sin(a);
        t[i] = x[i] * c - x[i + 64] * s;
        t[i + 64] = x[i + 64] * c + x[i] * s;
    }
    memcpy(y, t, sizeof t);
}

typedef struct {
    double s;
    int64_t n;
} scored;

/* (s descending, n ascending): the selection order, ties toward the lower index */
static int by_score_then_index(const void* a, const void* b) {
    const scored* x = (const scored*)a;
    const scored* y = (const scored*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->n < y->n) ? -1 : (x->n > y->n);
}

/*
 * Dynamic Top-P over raw index scores s[0..L) (the review's S_h(m) =
 * Top-P(s_h(m,.), p), temperature sqrt(16)).
 * Outputs: order[0..L) (selection order), *kstar, and for checks the max of
 * z = s/4, Z = sum exp(z - zmax), and the cumulative mass of the first k*-1
 * and first k* tokens.
 */
int oracle_topp(const double* s, int64_t L, double p, int64_t* order, int64_t* kstar_out, double* zmax_out,
                double* Z_out, double* cum_before_out, double* cum_at_out) {
    if (L <= 0) return 2;
    if (!(p > 0.0)) return 6;                 /* p <= 0 or NaN */
    double zmax = -INFINITY;
    for (int64_t n = 0; n < L; ++n) zmax = fmax(zmax, s[n] / 4.0);
    double Z = 0.0;
    for (int64_t n = 0; n < L; ++n) Z += exp(s[n] / 4.0 - zmax);
    scored* v = (scored*)malloc(sizeof(scored) * (size_t)L);
    for (int64_t n = 0; n < L; ++n) {
        v[n].s = s[n];
        v[n].n = n;
    }
    qsort(v, (size_t)L, sizeof(scored), by_score_then_index);
    int64_t k = L;
    double cum = 0.0, before = 0.0;
    if (p < 1.0) {
        for (int64_t i = 0; i < L; ++i) {
            before = cum;
            cum += exp(v[i].s / 4.0 - zmax) / Z;
            if (cum >= p) {
                k = i + 1;
                break;
            }
        }
    } else {
        for (int64_t i = 0; i < L; ++i) {
            before = cum;
            cum += exp(v[i].s / 4.0 - zmax) / Z;
        }
    }
    if (order)
        for (int64_t i = 0; i < L; ++i) order[i] = v[i].n;
    free(v);
    if (kstar_out) *kstar_out = k;
    if (zmax_out) *zmax_out = zmax;
    if (Z_out) *Z_out = Z;
    if (cum_before_out) *cum_before_out = before;
    if (cum_at_out) *cum_at_out = cum;
    return 0;
}

/*
 * Static Top-K (the pages' fixed-budget ablation, k = 4096 in the review's
 * comparison of top-k against top-p): the k highest index scores, ties
 * toward the lower index -- the first min(k, L) tokens under (s desc, n asc).
 * Outputs order[0..L) and *kstar = min(k, L).
 */
int oracle_topk(const double* s, int64_t L, int64_t K, int64_t* order, int64_t* kstar_out) {
    if (L <= 0) return 2;
    if (K < 1) return 6;
    scored* v = (scored*)malloc(sizeof(scored) * (size_t)L);
    for (int64_t n = 0; n < L; ++n) {
        v[n].s = s[n];
        v[n].n = n;
    }
    qsort(v, (size_t)L, sizeof(scored), by_score_then_index);
    if (order)
        for (int64_t i = 0; i < L; ++i) order[i] = v[i].n;
    free(v);
    if (kstar_out) *kstar_out = K < L ? K : L;
    return 0;
}

/* index scores s_n = (W^Q_h q^pre) . k_idx_n for n < L (fp64) */
static void index_scores(const geom* g, const uint16_t* q_pre, const uint16_t* Wq, const uint16_t* k_idx, int b,
                         int h, int64_t L, double* s) {
    int G = g->Hq / g->Hkv, kv = h / G;
    double qi[ORC_R];
    const uint16_t* q = q_pre + ((int64_t)b * g->Hq + h) * ORC_D;
    const uint16_t* W = Wq + (int64_t)h * ORC_R * ORC_D;
    for (int r = 0; r < ORC_R; ++r) {
        double a = 0.0;
        for (int d = 0; d < ORC_D; ++d) a += bf(W[r * ORC_D + d]) * bf(q[d]);
        qi[r] = a;
    }
    for (int64_t n = 0; n < L; ++n) {
        const uint16_t* k = row(g, k_idx, ORC_R, b, kv, n);
        double a = 0.0;
        for (int r = 0; r < ORC_R; ++r) a += qi[r] * bf(k[r]);
        s[n] = a;
    }
}

void oracle_index_scores(int B, int Hq, int Hkv, int64_t Ncap, const int32_t* block_table, int mbps,
                         const uint16_t* q_pre, const uint16_t* Wq, const uint16_t* k_idx, int b, int h, int64_t L,
                         double* s) {
    geom g = {B, Hq, Hkv, Ncap, block_table, mbps};
    index_scores(&g, q_pre, Wq, k_idx, b, h, L, s);
}

/* exact softmax attention of head h of sequence b over the positions pos[0..npos) */
static void attend_q(const geom* g, const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache, int b,
                     int kv, const int64_t* pos, int64_t npos, double* out);

static void attend(const geom* g, const uint16_t* q_rope, const uint16_t* k_cache, const uint16_t* v_cache, int b,
                   int h, const int64_t* pos, int64_t npos, double* out) {
    const int G = g->Hq / g->Hkv;
    attend_q(g, q_rope + ((int64_t)b * g->Hq + h) * ORC_D, k_cache, v_cache, b, h / G, pos, npos, out);
}

/* softmax(q . k_n / sqrt(128)) over the positions, times v_n, for one query vector q of KV head kv */
static void attend_q(const geom* g, const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache, int b,
                     int kv, const int64_t* pos, int64_t npos, double* out) {
    double qd[ORC_D];
    for (int d = 0; d < ORC_D; ++d) qd[d] = bf(q[d]);
    double* a = (double*)malloc(sizeof(double) * (size_t)(npos > 0 ? npos : 1));
    double amax = -INFINITY;
    for (int64_t i = 0; i < npos; ++i) {
        const uint16_t* k = row(g, k_cache, ORC_D, b, kv, pos[i]);
        double t = 0.0;
        for (int d = 0; d < ORC_D; ++d) t += qd[d] * bf(k[d]);
        a[i] = t / sqrt((double)ORC_D);
        amax = fmax(amax, a[i]);
    }
    double den = 0.0;
    for (int64_t i = 0; i < npos; ++i) den += exp(a[i] - amax);
    for (int d = 0; d < ORC_D; ++d) out[d] = 0.0;
    for (int64_t i = 0; i < npos; ++i) {
        double w = exp(a[i] - amax) / den;
        const uint16_t* v = row(g, v_cache, ORC_D, b, kv, pos[i]);
        for (int d = 0; d < ORC_D; ++d) out[d] += w * bf(v[d]);
    }
    free(a);
}

void oracle_attend(int B, int Hq, int Hkv, int64_t Ncap, const int32_t* block_table, int mbps,
                   const uint16_t* q_rope, const uint16_t* k_cache, const uint16_t* v_cache, int b, int h,
                   const int64_t* pos, int64_t npos, double* out) {
    geom g = {B, Hq, Hkv, Ncap, block_table, mbps};
    attend(&g, q_rope, k_cache, v_cache, b, h, pos, npos, out);
}

/* local head positions: [0, min(sink,L)) U [max(0,L-window), L), each once, ascending */
static int64_t local_positions(int64_t L, int window, int sink, int64_t* pos) {
    int64_t k = 0;
    int64_t s_end = sink < L ? sink : L;
    int64_t w_lo = L - window > 0 ? L - window : 0;
    for (int64_t n = 0; n < L; ++n)
        if (n < s_end || n >= w_lo) pos[k++] = n;
    return k;
}

/*
 * One decode step for every (b, h).  Returns 0, or 6 if some sequence has an
 * invalid p (its heads are then left untouched).
 * Optional per-(b,h) outputs (NULL to skip; retrieval heads only, local heads
 * get kstar = number of attended positions):
 *   kstar, tau (the k*-th score s), zmax (max z), Z (sum exp(z - zmax)),
 *   cum_before / cum_at (prefix mass of the first k*-1 / k* tokens),
 *   next_s (score of token k*+1 in the order, NaN when k* = L),
 *   kept_blocks [B,Hq,nblk_cap] (1 = block kept).
 */
/* the decode step; topk > 0 selects each retrieval head's static top-k
 * (p unused) instead of its dynamic top-p */
static int decode_step(int B, int Hq, int Hkv, int64_t Ncap, const int32_t* block_table, int mbps,
                       const uint16_t* q_pre, const uint16_t* q_rope, const uint16_t* k_idx, const uint16_t* k_cache,
                       const uint16_t* v_cache, const uint16_t* Wq_idx, const int32_t* seq_lens,
                       const uint8_t* head_kind, const float* p, int64_t topk, int window, int sink, int nthreads,
                       double* out, int64_t* kstar, double* tau, double* zmax, double* Z, double* cum_before,
                       double* cum_at, double* next_s, uint8_t* kept_blocks, int64_t nblk_cap) {
    geom g = {B, Hq, Hkv, Ncap, block_table, mbps};
    int bad = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t bh = 0; bh < (int64_t)B * Hq; ++bh) {
        int b = (int)(bh / Hq), h = (int)(bh % Hq);
        int64_t L = seq_lens[b];
        double* o = out + bh * ORC_D;
        int64_t* pos = (int64_t*)malloc(sizeof(int64_t) * (size_t)L);
        int64_t np = 0;
        if (!head_kind[h]) {
            np = local_positions(L, window, sink, pos);
            if (kstar) kstar[bh] = np;
        } else {
            double pb = topk > 0 ? 1.0 : (double)p[b];
            if (!(pb > 0.0)) {
                bad = 1;
                free(pos);
                continue;
            }
            double* s = (double*)malloc(sizeof(double) * (size_t)L);
            int64_t* order = (int64_t*)malloc(sizeof(int64_t) * (size_t)L);
            index_scores(&g, q_pre, Wq_idx, k_idx, b, h, L, s);
            int64_t k;
            double zm, Zs, cb, ca;
            oracle_topp(s, L, pb, order, &k, &zm, &Zs, &cb, &ca);
            if (topk > 0) oracle_topk(s, L, topk, order, &k);   /* same order, count k */
            uint8_t* keep = (uint8_t*)calloc((size_t)((L + ORC_BLK - 1) / ORC_BLK), 1);
            for (int64_t i = 0; i < k; ++i) keep[order[i] / ORC_BLK] = 1;
            for (int64_t n = 0; n < L; ++n)
                if (keep[n / ORC_BLK]) pos[np++] = n;
            if (kstar) kstar[bh] = k;
            if (tau) tau[bh] = s[order[k - 1]];
            if (zmax) zmax[bh] = zm;
            if (Z) Z[bh] = Zs;
            if (cum_before) cum_before[bh] = cb;
            if (cum_at) cum_at[bh] = ca;
            if (next_s) next_s[bh] = (k < L) ? s[order[k]] : NAN;
            if (kept_blocks) {
                uint8_t* kb = kept_blocks + bh * nblk_cap;
                memset(kb, 0, (size_t)nblk_cap);
                for (int64_t j = 0; j < (L + ORC_BLK - 1) / ORC_BLK && j < nblk_cap; ++j) kb[j] = keep[j];
            }
            free(keep);
            free(order);
            free(s);
        }
        attend(&g, q_rope, k_cache, v_cache, b, h, pos, np, o);
        free(pos);
    }
    return bad ? 6 : 0;
}

int oracle_decode_step(int B, int Hq, int Hkv, int64_t Ncap, const int32_t* block_table, int mbps,
                       const uint16_t* q_pre, const uint16_t* q_rope, const uint16_t* k_idx, const uint16_t* k_cache,
                       const uint16_t* v_cache, const uint16_t* Wq_idx, const int32_t* seq_lens,
                       const uint8_t* head_kind, const float* p, int window, int sink, int nthreads, double* out,
                       int64_t* kstar, double* tau, double* zmax, double* Z, double* cum_before, double* cum_at,
                       double* next_s, uint8_t* kept_blocks, int64_t nblk_cap) {
    return decode_step(B, Hq, Hkv, Ncap, block_table, mbps, q_pre, q_rope, k_idx, k_cache, v_cache, Wq_idx, seq_lens,
                       head_kind, p, 0, window, sink, nthreads, out, kstar, tau, zmax, Z, cum_before, cum_at, next_s,
                       kept_blocks, nblk_cap);
}

/* the same step with every retrieval head keeping its static top-k (k >= 1) */
int oracle_decode_step_topk(int B, int Hq, int Hkv, int64_t Ncap, const int32_t* block_table, int mbps,
                            const uint16_t* q_pre, const uint16_t* q_rope, const uint16_t* k_idx,
                            const uint16_t* k_cache, const uint16_t* v_cache, const uint16_t* Wq_idx,
                            const int32_t* seq_lens, const uint8_t* head_kind, int64_t topk, int window, int sink,
                            int nthreads, double* out, int64_t* kstar, double* tau, uint8_t* kept_blocks,
                            int64_t nblk_cap) {
    if (topk < 1) return 6;
    return decode_step(B, Hq, Hkv, Ncap, block_table, mbps, q_pre, q_rope, k_idx, k_cache, v_cache, Wq_idx, seq_lens,
                       head_kind, NULL, topk, window, sink, nthreads, out, kstar, tau, NULL, NULL, NULL, NULL, NULL,
                       kept_blocks, nblk_cap);
}

/*
 * Index-cache append (the step before the decode hot path): for each new
 * token t of sequence b and each KV head g,
 *     k_idx[b, g, pos_b + t] = bf16( W^K_g k^pre[b, g, t] )
 * (review, Method: "Adaptive sparse attention" -- the retrieval key
 * k^idx_n = W^K_h k^pre_n, kept as a 16-dim bf16 cache; W^K is per KV head
 * under GQA).  The dot product is taken in fp64 from the exact bf16 upcasts,
 * summed in index order, then rounded once to bf16.
 */

/* nearest bf16 to x, ties to the even significand: bf16 keeps the sign, the
 * 8 exponent bits and the top 7 fraction bits of an IEEE binary32. */
static uint16_t bf16_rne(double x) {
    if (isnan(x)) return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    int e;
    double m = frexp(a, &e);                 /* a = m 2^e, 0.5 <= m < 1 */
    int be = e - 1 + 127;                    /* biased exponent of a normal bf16 */
    if (be >= 1) {
        double q = nearbyint(ldexp(m, 8));   /* 8 significant bits: 128 .. 256 */
        if (q == 256.0) {
            q = 128.0;
            be += 1;
        }
        if (be >= 255) return (uint16_t)(sign | 0x7F80);   /* overflow: infinity */
        return (uint16_t)(sign | (be << 7) | ((int)q - 128));
    }
    /* subnormal: multiples of 2^-133 */
    double q = nearbyint(ldexp(a, 133));
    return (uint16_t)(sign | (int)q);        /* q = 128 lands on the smallest normal */
}

void oracle_index_append(int B, int Hkv, int64_t Ncap, const int32_t* block_table, int mbps, const uint16_t* k_pre,
                         int T, const uint16_t* Wk, const int32_t* pos, uint16_t* k_idx) {
    geom g = {B, Hkv, Hkv, Ncap, block_table, mbps};
    for (int b = 0; b < B; ++b)
        for (int kv = 0; kv < Hkv; ++kv)
            for (int t = 0; t < T; ++t) {
                const uint16_t* kp = k_pre + (((int64_t)b * Hkv + kv) * T + t) * ORC_D;
                uint16_t* dst = (uint16_t*)row(&g, k_idx, ORC_R, b, kv, (int64_t)pos[b] + t);
                for (int r = 0; r < ORC_R; ++r) {
                    const uint16_t* w = Wk + ((int64_t)kv * ORC_R + r) * ORC_D;
                    double acc = 0.0;
                    for (int i = 0; i < ORC_D; ++i) acc += bf(w[i]) * bf(kp[i]);
                    dst[r] = bf16_rne(acc);
                }
            }
}

/*
 * KV-cache write of new tokens, with the index-cache append in the same step:
 * for each new token t of sequence b, at cache position n = pos_b + t, and
 * each KV head g,
 *     k_idx[b, g, n]   = bf16( W^K_g k^pre )          (as oracle_index_append)
 *     k_cache[b, g, n] = bf16( RoPE_n(k^pre) )
 *     v_cache[b, g, n] = v[b, g, t]                   (bits copied)
 * The indexer reads keys before RoPE and the attention after it (review,
 * Method: "Adaptive sparse attention" -- s_h from W^Q q^pre and W^K k^pre,
 * exact attention on the RoPE'd q and k; Insight 2: RoPE rotates each
 * frequency pair by an angle proportional to the position).  RoPE_n rotates
 * the pairs (i, i + 64), i < 64, by the caller's angle table, row n:
 *     y_i      = k_i cos_{n,i} - k_{i+64} sin_{n,i}
 *     y_{i+64} = k_{i+64} cos_{n,i} + k_i sin_{n,i}
 * (cos, sin: fp32 [positions, 64]).  A product of a bf16 and an fp32 value
 * is exact in fp64; each y is the two products' sum rounded once to fp64
 * (a fused multiply-add onto the exact second product), then to bf16.
 */
void oracle_kv_append(int B, int Hkv, int64_t Ncap, const int32_t* block_table, int mbps, const uint16_t* k_pre,
                      const uint16_t* v_new, int T, const uint16_t* Wk, const float* rope_cos, const float* rope_sin,
                      const int32_t* pos, uint16_t* k_idx, uint16_t* k_cache, uint16_t* v_cache) {
    geom g = {B, Hkv, Hkv, Ncap, block_table, mbps};
    oracle_index_append(B, Hkv, Ncap, block_table, mbps, k_pre, T, Wk, pos, k_idx);
    for (int b = 0; b < B; ++b)
        for (int kv = 0; kv < Hkv; ++kv)
            for (int t = 0; t < T; ++t) {
                const int64_t n = (int64_t)pos[b] + t;
                const int64_t src = (((int64_t)b * Hkv + kv) * T + t) * ORC_D;
                const uint16_t* kp = k_pre + src;
                const float* c = rope_cos + n * 64;
                const float* sn = rope_sin + n * 64;
                uint16_t* kd = (uint16_t*)row(&g, k_cache, ORC_D, b, kv, n);
                uint16_t* vd = (uint16_t*)row(&g, v_cache, ORC_D, b, kv, n);
                for (int i = 0; i < 64; ++i) {
                    const double lo = bf(kp[i]), hi = bf(kp[i + 64]);
                    kd[i] = bf16_rne(fma(lo, (double)c[i], -(hi * (double)sn[i])));
                    kd[i + 64] = bf16_rne(fma(hi, (double)c[i], lo * (double)sn[i]));
                }
                memcpy(vd, v_new + src, ORC_D * sizeof(uint16_t));
            }
}

/*
 * Local heads' ring cache: a local head reads only the first `sink` tokens
 * and the last `window` ones (review, Method: "Adaptive sparse attention" --
 * local heads keep a sink and a sliding window; Insight 1: only a minority of
 * heads needs the long context), so its KV head can keep C = S0 + W rows per
 * sequence (S0 >= sink, W >= window) instead of the whole context.  Reading
 * of the layout (the pages give none): position n < S0 lives in row n;
 * position n >= S0 lives in row S0 + (n mod W), so each new position
 * overwrites the one W places before it.  With S0 and W multiples of 64,
 * every 64-token block of the context occupies whole aligned 64-row slots.
 * After positions 0 .. L-1 are written in order, the rows hold
 * [0, min(S0, L)) and [max(S0, L - W), L).
 */
int64_t oracle_ring_row(int64_t n, int S0, int W) { return n < S0 ? n : S0 + n % W; }

/* Write the rows of positions pos_b + t, t = 0 .. T-1, in that order (a later
 * position overwrites an earlier one of the same row): rings [B, Hkv, C, 128],
 * new rows [B, Hkv, T, 128]. */
void oracle_ring_write(int B, int Hkv, int S0, int W, const uint16_t* k_new, const uint16_t* v_new, int T,
                       const int32_t* pos, uint16_t* k_ring, uint16_t* v_ring) {
    const int64_t C = (int64_t)S0 + W;
    for (int b = 0; b < B; ++b)
        for (int kv = 0; kv < Hkv; ++kv)
            for (int t = 0; t < T; ++t) {
                const int64_t src = (((int64_t)b * Hkv + kv) * T + t) * ORC_D;
                const int64_t dst =
                    (((int64_t)b * Hkv + kv) * C + oracle_ring_row((int64_t)pos[b] + t, S0, W)) * ORC_D;
                memcpy(k_ring + dst, k_new + src, ORC_D * sizeof(uint16_t));
                memcpy(v_ring + dst, v_new + src, ORC_D * sizeof(uint16_t));
            }
}

/* Local head h of sequence b at length L: the attention over
 * [0, min(sink, L)) U [max(0, L - window), L), each key and value read from
 * its ring row.  Returns 0, or 2 if sink > S0 or window > W (positions the
 * ring does not hold). */
int oracle_attend_ring(int B, int Hq, int Hkv, int S0, int W, const uint16_t* q_rope, const uint16_t* k_ring,
                       const uint16_t* v_ring, int b, int h, int64_t L, int window, int sink, double* out) {
    if (window > W || sink > S0) return 2;
    geom g = {B, Hq, Hkv, (int64_t)S0 + W, NULL, 0};
    int64_t* pos = (int64_t*)malloc(sizeof(int64_t) * (size_t)(L > 0 ? L : 1));
    const int64_t np = local_positions(L, window, sink, pos);
    for (int64_t i = 0; i < np; ++i) pos[i] = oracle_ring_row(pos[i], S0, W);
    attend(&g, q_rope, k_ring, v_ring, b, h, pos, np, out);
    free(pos);
    return 0;
}

/*
 * Prefill attention of a chunk of T queries per sequence (the pages' second
 * workload; review, Method: "Adaptive sparse attention" -- in prefill the
 * retrieval heads attend densely and the local heads to their sink and
 * sliding window; Experiments: the prefill speedups).  Query t of sequence b
 * sits at position m = pos_b + t and attends causally, itself included:
 *   retrieval head : positions [0, m]
 *   local head     : [0, min(sink, m + 1)) U [max(0, m + 1 - window), m + 1)
 * (the decode step's sets at length L = m + 1).  The cache must already hold
 * the keys and values of positions up to pos_b + T - 1.  q: [B, Hq, T, 128]
 * bf16 (RoPE'd); out: [B, Hq, T, 128] fp64.
 */
void oracle_prefill(int B, int Hq, int Hkv, int64_t Ncap, const int32_t* block_table, int mbps, const uint16_t* q,
                    const uint16_t* k_cache, const uint16_t* v_cache, const uint8_t* head_kind, const int32_t* pos,
                    int T, int window, int sink, double* out) {
    geom g = {B, Hq, Hkv, Ncap, block_table, mbps};
    const int G = Hq / Hkv;
    int64_t* ps = (int64_t*)malloc(sizeof(int64_t) * (size_t)(Ncap > 0 ? Ncap : 1));
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h)
            for (int t = 0; t < T; ++t) {
                const int64_t L = (int64_t)pos[b] + t + 1;     /* positions 0 .. m */
                int64_t np;
                if (head_kind[h]) {
                    for (int64_t n = 0; n < L; ++n) ps[n] = n;
                    np = L;
                } else {
                    np = local_positions(L, window, sink, ps);
                }
                const int64_t qi = ((int64_t)b * Hq + h) * T + t;
                attend_q(&g, q + qi * ORC_D, k_cache, v_cache, b, h / G, ps, np, out + qi * ORC_D);
            }
    free(ps);
}

uint16_t oracle_bf16_rne(double x) { return bf16_rne(x); }
