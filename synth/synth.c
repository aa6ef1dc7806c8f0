/*
 * Seeded synthetic Q/K/V for latent-point attention workloads.
 *
 * This module only draws inputs.  It holds none of the attention method's
 * arithmetic (no pooling, scoring, selection or softmax); both the fp64
 * oracle and the CUDA path read the arrays it writes.
 *
 * Recipe (stands in for multi-view image sequences, which are not available):
 *   - every token t = s*N + n of S frames x N tokens may be tied to one shared
 *     3-D "point" p; the point's per-head latent z_{h,p} ~ N(0, I_d);
 *   - a tied token gets  q = a_lat*z + a_noise*eps_q,  k = a_lat*z + a_noise*eps_k;
 *   - an untied token gets q = eps_q, k = eps_k;  v = eps_v for every token;
 *   - the first n_sink tokens of every frame (camera + register tokens) are
 *     never tied and have k scaled by sink_k_scale;
 *   - with window W > 0, point p is visible in frames a_p .. a_p+W-1
 *     (a_p uniform in 0..S-W) and a token of frame s draws its point
 *     uniformly among the points visible in s; with W = 0 it draws uniformly
 *     among all P points.
 *
 * Randomness is counter based: every draw is a pure function of
 * (seed, stream, head, index, component pair), so any element can be
 * regenerated on its own.  The mixing function is the SplitMix64 output
 * function (Steele, Lea & Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014); normals use the Box-Muller transform.
 * Values are computed in double, rounded to float (round to nearest) and,
 * for bf16 output, to bfloat16 with round-to-nearest-even.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int32_t bh;           /* independent heads (batch folded in) */
    int32_t frames;       /* S */
    int32_t tokens;       /* N per frame */
    int32_t head_dim;     /* d (even) */
    int32_t n_sink;       /* special tokens at n < n_sink of every frame */
    int32_t n_points;     /* P */
    int32_t window;       /* visibility window in frames; 0 = every frame */
    double p_assign;      /* probability that a non-sink token is tied */
    double a_lat;         /* latent weight (0.8) */
    double a_noise;       /* noise weight (0.6) */
    double sink_k_scale;  /* key scale of sink tokens (4) */
    uint64_t seed;
    int32_t out_bf16;     /* 1: write bf16 bit patterns (uint16), 0: float32 */
    int32_t n_threads;    /* worker threads (>= 1) */
    int32_t head0;        /* global index of the first head drawn (a shard of a larger draw) */
} synth_cfg;

enum { ST_ASSIGN = 1, ST_START = 2, ST_LATENT = 3, ST_QN = 4, ST_KN = 5, ST_VN = 6 };

static inline uint64_t splitmix64_out(uint64_t x) {
    uint64_t z = x + 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* 62-bit counter: pair [0,6) index [6,28) head [28,36) stream [36,40) seed [40,62). */
static inline uint64_t counter(uint64_t seed, uint64_t stream, uint64_t head, uint64_t index,
                               uint64_t pair) {
    return ((seed & 0x3FFFFFull) << 40) | ((stream & 0xFull) << 36) | ((head & 0xFFull) << 28) |
           ((index & 0x3FFFFFull) << 6) | (pair & 0x3Full);
}

static inline double unit_open(uint64_t h) { return ((double)(h >> 11) + 0.5) * 0x1.0p-53; }

/* Two independent uniforms in (0,1) from one counter. */
static inline void uniforms(uint64_t ctr, double* u1, double* u2) {
    *u1 = unit_open(splitmix64_out(ctr << 1));
    *u2 = unit_open(splitmix64_out((ctr << 1) | 1ull));
}

/* Normal pair (Box-Muller) for component pair `pair`: returns component 2*pair and 2*pair+1. */
static inline void normal_pair(uint64_t ctr, double* z0, double* z1) {
    double u1, u2;
    uniforms(ctr, &u1, &u2);
    const double r = sqrt(-2.0 * log(u1));
    const double th = 6.283185307179586476925286766559 * u2;
    *z0 = r * cos(th);
    *z1 = r * sin(th);
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t b;
    memcpy(&b, &f, 4);
    if ((b & 0x7F800000u) == 0x7F800000u) return (uint16_t)((b >> 16) | ((b & 0xFFFFu) ? 0x40u : 0u));
    const uint32_t lsb = (b >> 16) & 1u;
    b += 0x7FFFu + lsb;
    return (uint16_t)(b >> 16);
}

/* ---- point assignment (shared by all heads) ---------------------------------------- */

typedef struct {
    const synth_cfg* c;
    int32_t* point_of_token; /* [L], -1 = untied */
    const int32_t* sorted;   /* points sorted by start frame (window > 0) */
    const int64_t* off;      /* off[a] = first sorted slot with start a; size S-W+2 */
    int64_t t0, t1;
} assign_job;

static void* assign_worker(void* arg) {
    assign_job* j = (assign_job*)arg;
    const synth_cfg* c = j->c;
    const int64_t N = c->tokens;
    for (int64_t t = j->t0; t < j->t1; ++t) {
        const int64_t s = t / N, n = t % N;
        int32_t p = -1;
        if (n >= c->n_sink) {
            double u_tie, u_pick;
            uniforms(counter(c->seed, ST_ASSIGN, 0, (uint64_t)t, 0), &u_tie, &u_pick);
            if (u_tie < c->p_assign) {
                if (c->window <= 0) {
                    int64_t q = (int64_t)(u_pick * c->n_points);
                    if (q >= c->n_points) q = c->n_points - 1;
                    p = (int32_t)q;
                } else {
                    const int64_t amax = c->frames - c->window;
                    int64_t lo = s - c->window + 1;
                    if (lo < 0) lo = 0;
                    int64_t hi = s < amax ? s : amax;
                    if (hi >= lo) {
                        const int64_t b = j->off[lo], e = j->off[hi + 1];
                        if (e > b) {
                            int64_t q = b + (int64_t)(u_pick * (double)(e - b));
                            if (q >= e) q = e - 1;
                            p = j->sorted[q];
                        }
                    }
                }
            }
        }
        j->point_of_token[t] = p;
    }
    return NULL;
}

/* ---- per-head values ----------------------------------------------------------------- */

typedef struct {
    const synth_cfg* c;
    int64_t h;
    float* latent; /* [P][d] for this head */
    const int32_t* point_of_token;
    void *q, *k, *v;
    int64_t i0, i1; /* range of points (phase 0) or tokens (phase 1) */
    int phase;
} head_job;

static void* head_worker(void* arg) {
    head_job* j = (head_job*)arg;
    const synth_cfg* c = j->c;
    const int64_t d = c->head_dim, N = c->tokens, L = (int64_t)c->frames * c->tokens;
    if (j->phase == 0) {
        for (int64_t p = j->i0; p < j->i1; ++p)
            for (int64_t e = 0; e < d; e += 2) {
                double z0, z1;
                normal_pair(counter(c->seed, ST_LATENT, (uint64_t)(c->head0 + j->h), (uint64_t)p, (uint64_t)(e / 2)), &z0,
                            &z1);
                j->latent[p * d + e] = (float)z0;
                j->latent[p * d + e + 1] = (float)z1;
            }
        return NULL;
    }
    for (int64_t t = j->i0; t < j->i1; ++t) {
        const int32_t p = j->point_of_token[t];
        const int is_sink = (t % N) < c->n_sink;
        const int64_t base = (j->h * L + t) * d;
        for (int64_t e = 0; e < d; e += 2) {
            double qn[2], kn[2], vn[2];
            const uint64_t pe = (uint64_t)(e / 2);
            normal_pair(counter(c->seed, ST_QN, (uint64_t)(c->head0 + j->h), (uint64_t)t, pe), &qn[0], &qn[1]);
            normal_pair(counter(c->seed, ST_KN, (uint64_t)(c->head0 + j->h), (uint64_t)t, pe), &kn[0], &kn[1]);
            normal_pair(counter(c->seed, ST_VN, (uint64_t)(c->head0 + j->h), (uint64_t)t, pe), &vn[0], &vn[1]);
            for (int r = 0; r < 2; ++r) {
                double qv, kv;
                if (p >= 0) {
                    const double z = (double)j->latent[(int64_t)p * d + e + r];
                    qv = c->a_lat * z + c->a_noise * qn[r];
                    kv = c->a_lat * z + c->a_noise * kn[r];
                } else {
                    qv = qn[r];
                    kv = kn[r];
                }
                if (is_sink) kv *= c->sink_k_scale;
                const float qf = (float)qv, kf = (float)kv, vf = (float)vn[r];
                if (c->out_bf16) {
                    ((uint16_t*)j->q)[base + e + r] = f32_to_bf16_rne(qf);
                    ((uint16_t*)j->k)[base + e + r] = f32_to_bf16_rne(kf);
                    ((uint16_t*)j->v)[base + e + r] = f32_to_bf16_rne(vf);
                } else {
                    ((float*)j->q)[base + e + r] = qf;
                    ((float*)j->k)[base + e + r] = kf;
                    ((float*)j->v)[base + e + r] = vf;
                }
            }
        }
    }
    return NULL;
}

static int run_parallel(void* (*fn)(void*), void* jobs, size_t job_size, int n) {
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)n);
    if (!th) return -1;
    int started = 0, rc = 0;
    for (int i = 0; i < n; ++i) {
        if (pthread_create(&th[i], NULL, fn, (char*)jobs + job_size * (size_t)i) != 0) {
            rc = -1;
            break;
        }
        ++started;
    }
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    return rc;
}

/* Returns 0 on success, negative on bad arguments or allocation failure.
 * q, k, v: [bh][S*N][d] (uint16 bf16 bits or float32); point_of_token: [S*N] int32 (may be NULL). */
int synth_generate(const synth_cfg* c, void* q, void* k, void* v, int32_t* point_of_token) {
    if (!c || !q || !k || !v) return -1;
    if (c->bh <= 0 || c->frames <= 0 || c->tokens <= 0 || c->head_dim <= 0 || (c->head_dim & 1)) return -2;
    if (c->head0 < 0 || c->head0 + c->bh > 256) return -2; /* the counter holds 8 bits of head */
    if (c->n_points <= 0 || c->n_sink < 0 || c->window < 0 || c->window > c->frames) return -3;
    if ((int64_t)c->frames * c->tokens >= (1ll << 22) || c->n_points >= (1 << 22) || c->bh > 255) return -4;
    const int nth = c->n_threads > 0 ? c->n_threads : 1;
    const int64_t L = (int64_t)c->frames * c->tokens, P = c->n_points, d = c->head_dim;

    int32_t* pot = point_of_token ? point_of_token : (int32_t*)malloc(sizeof(int32_t) * (size_t)L);
    int32_t* sorted = NULL;
    int64_t* off = NULL;
    float* latent = NULL;
    int rc = 0;
    if (!pot) return -5;

    if (c->window > 0) {
        const int64_t na = c->frames - c->window + 1;
        int32_t* start = (int32_t*)malloc(sizeof(int32_t) * (size_t)P);
        sorted = (int32_t*)malloc(sizeof(int32_t) * (size_t)P);
        off = (int64_t*)calloc((size_t)(na + 1), sizeof(int64_t));
        if (!start || !sorted || !off) {
            free(start);
            rc = -5;
            goto done;
        }
        for (int64_t p = 0; p < P; ++p) {
            double u1, u2;
            uniforms(counter(c->seed, ST_START, 0, (uint64_t)p, 0), &u1, &u2);
            int64_t a = (int64_t)(u1 * (double)na);
            if (a >= na) a = na - 1;
            start[p] = (int32_t)a;
            off[a + 1]++;
        }
        for (int64_t a = 0; a < na; ++a) off[a + 1] += off[a];
        int64_t* fill = (int64_t*)malloc(sizeof(int64_t) * (size_t)na);
        if (!fill) {
            free(start);
            rc = -5;
            goto done;
        }
        memcpy(fill, off, sizeof(int64_t) * (size_t)na);
        for (int64_t p = 0; p < P; ++p) sorted[fill[start[p]]++] = (int32_t)p; /* stable by p */
        free(fill);
        free(start);
    }

    {
        assign_job* aj = (assign_job*)calloc((size_t)nth, sizeof(assign_job));
        if (!aj) {
            rc = -5;
            goto done;
        }
        for (int i = 0; i < nth; ++i) {
            aj[i].c = c;
            aj[i].point_of_token = pot;
            aj[i].sorted = sorted;
            aj[i].off = off;
            aj[i].t0 = L * i / nth;
            aj[i].t1 = L * (i + 1) / nth;
        }
        rc = run_parallel(assign_worker, aj, sizeof(assign_job), nth);
        free(aj);
        if (rc) goto done;
    }

    latent = (float*)malloc(sizeof(float) * (size_t)(P * d));
    if (!latent) {
        rc = -5;
        goto done;
    }
    {
        head_job* hj = (head_job*)calloc((size_t)nth, sizeof(head_job));
        if (!hj) {
            rc = -5;
            goto done;
        }
        for (int64_t h = 0; h < c->bh && !rc; ++h) {
            for (int phase = 0; phase < 2 && !rc; ++phase) {
                const int64_t n = phase == 0 ? P : L;
                for (int i = 0; i < nth; ++i) {
                    hj[i].c = c;
                    hj[i].h = h;
                    hj[i].latent = latent;
                    hj[i].point_of_token = pot;
                    hj[i].q = q;
                    hj[i].k = k;
                    hj[i].v = v;
                    hj[i].i0 = n * i / nth;
                    hj[i].i1 = n * (i + 1) / nth;
                    hj[i].phase = phase;
                }
                rc = run_parallel(head_worker, hj, sizeof(head_job), nth);
            }
        }
        free(hj);
    }

done:
    free(latent);
    free(sorted);
    free(off);
    if (pot != point_of_token) free(pot);
    return rc;
}
