/*
 * Seeded synthetic attention inputs (fp16 Q, K, V).
 *
 * This module only draws random numbers; it holds none of the attention,
 * quantisation or selection arithmetic.  Both the CPU oracle and the CUDA
 * library are fed from it.
 *
 * Random numbers are counter based, so any element can be drawn on its own:
 *   - a stream is identified by (seed, tag, batch, head);
 *   - element i of a stream takes the SplitMix64 outputs number 2*(i/2) and
 *     2*(i/2)+1 of that stream (SplitMix64: Steele, Lea & Flood, "Fast
 *     splittable pseudorandom number generators", OOPSLA 2014), turns them into
 *     two uniforms in (0,1) with 53-bit resolution, and applies Box-Muller
 *     (cos branch for even i, sin branch for odd i).
 * Every sample is formed in double precision and rounded once to fp16
 * (round to nearest, ties to even).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ull

static uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* Output number i (0-based) of the SplitMix64 sequence started from `key`. */
static uint64_t splitmix_at(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * GOLDEN); }

uint64_t synth_stream(uint64_t seed, uint32_t tag, uint32_t b, uint32_t h) {
    uint64_t k = mix64(seed ^ 0x5851F42D4C957F2Dull);
    k = mix64(k ^ ((uint64_t)tag << 48) ^ ((uint64_t)b << 24) ^ (uint64_t)h);
    return k;
}

double synth_uniform(uint64_t key, uint64_t i) {
    /* 53 random bits, shifted by half a step so the result is never 0 or 1. */
    return ((double)(splitmix_at(key, i) >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

double synth_normal(uint64_t key, uint64_t i) {
    uint64_t pair = i >> 1;
    double u1 = synth_uniform(key, 2 * pair);
    double u2 = synth_uniform(key, 2 * pair + 1);
    double r = sqrt(-2.0 * log(u1));
    double th = 6.283185307179586476925286766559 * u2;
    return (i & 1) ? r * sin(th) : r * cos(th);
}

/* double -> IEEE binary16, round to nearest even, overflow to +-inf. */
uint16_t synth_f16(double v) {
    uint16_t sign = (v < 0 || (v == 0 && signbit(v))) ? 0x8000 : 0;
    double a = fabs(v);
    if (isnan(v)) return 0x7E00;
    if (a >= 65520.0) return sign | 0x7C00; /* rounds past the largest finite value */
    if (a < 0x1p-25) {                     /* below half the smallest subnormal */
        return sign;
    }
    int e;
    frexp(a, &e); /* a = f * 2^e, f in [0.5,1) */
    int exp16 = e - 1 + 15;                /* biased exponent if normal */
    double quantum = (exp16 >= 1) ? ldexp(1.0, e - 1 - 10) : 0x1p-24;
    double q = a / quantum;                /* exact: quantum is a power of two */
    double fl = floor(q);
    double rem = q - fl;
    uint64_t m = (uint64_t)fl;
    if (rem > 0.5 || (rem == 0.5 && (m & 1))) m += 1;
    /* m counts quanta; rebuild the bit pattern. */
    if (exp16 >= 1) {
        if (m == 2048) { m = 1024; exp16 += 1; }
        if (exp16 >= 31) return sign | 0x7C00;
        return sign | (uint16_t)(exp16 << 10) | (uint16_t)(m - 1024);
    }
    /* subnormal range: m in [0, 1024]; 1024 becomes the smallest normal */
    if (m >= 1024) return sign | (uint16_t)(1 << 10);
    return sign | (uint16_t)m;
}

enum { TAG_QN = 1, TAG_KN = 2, TAG_VN = 3, TAG_KOFF = 4, TAG_BASIS = 5,
       TAG_QC = 6, TAG_KC = 7, TAG_ROWS = 8 };

/* Recipe of one workload family (see the Python wrapper for the five named
 * workloads).  Shapes are free, so tests can use the same families at small
 * sizes. */
typedef struct {
    int B, Hq, Hkv, N, D;
    int kv_offset;        /* add a per-(head, channel) K offset ~ N(0, offset_sd^2) */
    double offset_sd;
    int sink;             /* scale K row 0 by sink_scale */
    double sink_scale;
    int n_heavy;          /* scale this many distinct random K rows (from 1..N-1) */
    double heavy_scale;
    int rank;             /* shared low-rank component added to Q and K (0 = none) */
    double coeff_sd;      /* sd of the per-token coefficients */
    int seed_per_batch;   /* seed_b = seed + 1000*b */
} synth_recipe;

static void pick_rows(uint64_t key, int N, int count, int* out) {
    int n = 0;
    uint64_t i = 0;
    while (n < count) {
        int r = 1 + (int)(synth_uniform(key, i++) * (double)(N - 1));
        if (r >= N) r = N - 1;
        int dup = 0;
        for (int t = 0; t < n; ++t) dup |= (out[t] == r);
        if (!dup) out[n++] = r;
    }
}

/* Fill Q [B,Hq,N,D], K and V [B,Hkv,N,D] (fp16 bit patterns). Returns 0 on success. */
int synth_generate(const synth_recipe* rc, uint64_t seed, uint16_t* Q, uint16_t* K, uint16_t* V) {
    const int B = rc->B, Hq = rc->Hq, Hkv = rc->Hkv, N = rc->N, D = rc->D;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || D <= 0 || Hq % Hkv) return 1;
    if (rc->n_heavy > 0 && rc->n_heavy > N - 1) return 1;
    if (rc->rank < 0 || rc->rank > 64) return 1;
    const int G = Hq / Hkv, R = rc->rank;

    for (int b = 0; b < B; ++b) {
        uint64_t sd = rc->seed_per_batch ? seed + 1000ull * (uint64_t)b : seed;
        for (int hk = 0; hk < Hkv; ++hk) {
            double* basis = R ? (double*)malloc(sizeof(double) * (size_t)R * D) : NULL;
            double* off = (double*)calloc((size_t)D, sizeof(double));
            double* rowscale = (double*)malloc(sizeof(double) * (size_t)N);
            if ((R && !basis) || !off || !rowscale) { free(basis); free(off); free(rowscale); return 2; }
            if (R) {
                uint64_t kb = synth_stream(sd, TAG_BASIS, b, hk);
                double s = 1.0 / sqrt((double)D);
                for (int i = 0; i < R * D; ++i) basis[i] = s * synth_normal(kb, i);
            }
            if (rc->kv_offset) {
                uint64_t ko = synth_stream(sd, TAG_KOFF, b, hk);
                for (int d = 0; d < D; ++d) off[d] = rc->offset_sd * synth_normal(ko, d);
            }
            for (int n = 0; n < N; ++n) rowscale[n] = 1.0;
            if (rc->n_heavy > 0) {
                int* rows = (int*)malloc(sizeof(int) * (size_t)rc->n_heavy);
                pick_rows(synth_stream(sd, TAG_ROWS, b, hk), N, rc->n_heavy, rows);
                for (int t = 0; t < rc->n_heavy; ++t) rowscale[rows[t]] = rc->heavy_scale;
                free(rows);
            }
            if (rc->sink) rowscale[0] = rc->sink_scale;

            uint64_t kn = synth_stream(sd, TAG_KN, b, hk), vn = synth_stream(sd, TAG_VN, b, hk);
            uint64_t kc = synth_stream(sd, TAG_KC, b, hk);
            size_t base = ((size_t)b * Hkv + hk) * (size_t)N * D;
            #pragma omp parallel for schedule(static)
            for (int n = 0; n < N; ++n) {
                double c[64];
                for (int r = 0; r < R; ++r) c[r] = rc->coeff_sd * synth_normal(kc, (uint64_t)n * R + r);
                for (int d = 0; d < D; ++d) {
                    uint64_t e = (uint64_t)n * D + d;
                    double k = synth_normal(kn, e) + off[d];
                    for (int r = 0; r < R; ++r) k += c[r] * basis[r * D + d];
                    K[base + e] = synth_f16(k * rowscale[n]);
                    V[base + e] = synth_f16(synth_normal(vn, e));
                }
            }
            for (int g = 0; g < G; ++g) {
                int hq = hk * G + g;
                uint64_t qn = synth_stream(sd, TAG_QN, b, hq), qc = synth_stream(sd, TAG_QC, b, hq);
                size_t qbase = ((size_t)b * Hq + hq) * (size_t)N * D;
                #pragma omp parallel for schedule(static)
                for (int n = 0; n < N; ++n) {
                    double c[64];
                    for (int r = 0; r < R; ++r) c[r] = rc->coeff_sd * synth_normal(qc, (uint64_t)n * R + r);
                    for (int d = 0; d < D; ++d) {
                        uint64_t e = (uint64_t)n * D + d;
                        double q = synth_normal(qn, e);
                        for (int r = 0; r < R; ++r) q += c[r] * basis[r * D + d];
                        Q[qbase + e] = synth_f16(q);
                    }
                }
            }
            free(basis); free(off); free(rowscale);
        }
    }
    return 0;
}
