/*
 * Seeded synthetic inputs for the RTPurbo decode step.
 *
 * This file is the one source of random data shared by the CUDA path's tests,
 * the benchmark and the fp64 oracle.  It holds no part of the method itself:
 * no indexer scores over the cache, no softmax, no top-p, no attention.  It
 * draws numbers, rounds them to bf16, rotates keys by RoPE (an input-side
 * transform the decode step consumes already applied) and forms the index-key
 * cache k_idx = W^K k^pre that the step reads.
 *
 * Random numbers: a counter-based generator built from SplitMix64's output
 * mixer (Steele, Lea & Flood, "Fast Splittable Pseudorandom Number
 * Generators", OOPSLA 2014) -- value i of a stream is mix(base + (i+1)*gamma)
 * with gamma the golden-ratio increment -- and the Box-Muller transform
 * (Box & Muller, Ann. Math. Stat. 1958) to turn pairs of uniforms into pairs
 * of standard normals.  Every element is a pure function of (seed, stream,
 * index), so any slice of any tensor can be drawn on its own, in parallel.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t stream_base(uint64_t seed, uint64_t stream) {
    return mix64(mix64(seed * GOLDEN_GAMMA + 0x632BE59BD9B4E019ULL) ^ (stream * 0xD1B54A32D192ED03ULL + 1));
}

/* uniform in (0, 1]: 53 random bits, shifted away from zero */
static inline double uniform_at(uint64_t base, uint64_t i) {
    uint64_t u = mix64(base + (i + 1) * GOLDEN_GAMMA);
    return ((double)(u >> 11) + 1.0) * (1.0 / 9007199254740992.0);
}

/* standard normal number i of the stream (pairs 2j, 2j+1 share one Box-Muller draw) */
static inline double normal_at(uint64_t base, uint64_t i) {
    uint64_t j = i >> 1;
    double u1 = uniform_at(base, 2 * j);
    double u2 = uniform_at(base, 2 * j + 1);
    double r = sqrt(-2.0 * log(u1));
    double a = 6.283185307179586476925286766559 * u2;
    return (i & 1) ? r * sin(a) : r * cos(a);
}

/* fp64 -> bf16 bits: round to fp32 (nearest-even), then to bf16 (nearest-even) */
static inline uint16_t to_bf16(double x) {
    float f = (float)x;
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u) {           /* inf / nan */
        return (uint16_t)((u >> 16) | ((u & 0xFFFFu) ? 0x40u : 0u));
    }
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

static inline double from_bf16(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

uint64_t synth_stream_base(uint64_t seed, uint64_t stream) { return stream_base(seed, stream); }

/* out[i] = scale * normal(offset + i), fp64 */
void synth_normal_f64(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double scale, double* out) {
    uint64_t base = stream_base(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = scale * normal_at(base, offset + (uint64_t)i);
}

/* out[i] = bf16(scale * normal(offset + i)) */
void synth_normal_bf16(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double scale, uint16_t* out) {
    uint64_t base = stream_base(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = to_bf16(scale * normal_at(base, offset + (uint64_t)i));
}

/* uniform (0,1] draws, fp64 */
void synth_uniform_f64(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double* out) {
    uint64_t base = stream_base(seed, stream);
    for (int64_t i = 0; i < n; ++i) out[i] = uniform_at(base, offset + (uint64_t)i);
}

void synth_f64_to_bf16(const double* in, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = to_bf16(in[i]);
}

void synth_bf16_to_f64(const uint16_t* in, int64_t n, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = from_bf16(in[i]);
}

void synth_fill_u16(uint16_t* p, int64_t n, uint16_t v) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) p[i] = v;
}

/*
 * Rotary position embedding of one 128-wide head vector at position pos,
 * rotate-half pairing: dimension i pairs with i+64, angle pos * theta^(-2i/128).
 * x and y are fp64 (may alias).
 */
static void rope128(const double* x, double pos, double theta, double* y) {
    for (int i = 0; i < 64; ++i) {
        double inv = pow(theta, -2.0 * (double)i / 128.0);
        double a = pos * inv;
        double c = cos(a), s = sin(a);
        double x0 = x[i], x1 = x[i + 64];
        y[i] = x0 * c - x1 * s;
        y[i + 64] = x1 * c + x0 * s;
    }
}

/* rows of 128 bf16 values rotated to positions pos[r] (fp64 math), output bf16 */
void synth_rope_rows_bf16(const uint16_t* x, int64_t rows, const int64_t* pos, double theta, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double v[128];
        for (int d = 0; d < 128; ++d) v[d] = from_bf16(x[r * 128 + d]);
        rope128(v, (double)pos[r], theta, v);
        for (int d = 0; d < 128; ++d) out[r * 128 + d] = to_bf16(v[d]);
    }
}

/*
 * Keys and index keys of one KV head for a list of positions.
 * For each row r (cache position pos[r]):
 *   k_pre = bf16(normal(stream, pos*128 + d))                (pre-RoPE key)
 *   kcache_out[r] = bf16(RoPE(k_pre, pos))                   (RoPE'd key, read by attention)
 *   kidx_out[r]   = bf16(W . k_pre)  (16 values, W is 16x128 bf16; skipped when W == NULL)
 *   kpre_out[r]   = k_pre            (skipped when NULL)
 */
void synth_keys(uint64_t seed, uint64_t stream, const int64_t* pos, int64_t rows, double theta,
                const uint16_t* W, uint16_t* kcache_out, uint16_t* kidx_out, uint16_t* kpre_out) {
    uint64_t base = stream_base(seed, stream);
    double Wd[16 * 128];
    if (W) for (int i = 0; i < 16 * 128; ++i) Wd[i] = from_bf16(W[i]);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double k[128], kr[128];
        uint16_t kb[128];
        uint64_t p = (uint64_t)pos[r];
        for (int d = 0; d < 128; ++d) {
            kb[d] = to_bf16(normal_at(base, p * 128 + (uint64_t)d));
            k[d] = from_bf16(kb[d]);
        }
        if (kpre_out) memcpy(kpre_out + r * 128, kb, sizeof kb);
        if (W && kidx_out) {
            for (int i = 0; i < 16; ++i) {
                double acc = 0.0;
                for (int d = 0; d < 128; ++d) acc += Wd[i * 128 + d] * k[d];
                kidx_out[r * 16 + i] = to_bf16(acc);
            }
        }
        if (kcache_out) {
            rope128(k, (double)p, theta, kr);
            for (int d = 0; d < 128; ++d) kcache_out[r * 128 + d] = to_bf16(kr[d]);
        }
    }
}

/* values of one KV head: out[r] = bf16(normal(stream, pos*128 + d)) */
void synth_values(uint64_t seed, uint64_t stream, const int64_t* pos, int64_t rows, uint16_t* out) {
    uint64_t base = stream_base(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        uint64_t p = (uint64_t)pos[r];
        for (int d = 0; d < 128; ++d) out[r * 128 + d] = to_bf16(normal_at(base, p * 128 + (uint64_t)d));
    }
}

/*
 * Row statistics of a bf16 [rows,16] index-key block: sum of squares of all
 * entries and the largest row norm.  Used to aim and size planted tokens.
 */
void synth_kidx_stats(const uint16_t* kidx, int64_t rows, double* sumsq_out, double* maxnorm_out) {
    double ss = 0.0, mx = 0.0;
#pragma omp parallel for schedule(static) reduction(+ : ss) reduction(max : mx)
    for (int64_t r = 0; r < rows; ++r) {
        double n2 = 0.0;
        for (int i = 0; i < 16; ++i) {
            double v = from_bf16(kidx[r * 16 + i]);
            n2 += v * v;
        }
        ss += n2;
        double nr = sqrt(n2);
        if (nr > mx) mx = nr;
    }
    *sumsq_out = ss;
    *maxnorm_out = mx;
}
