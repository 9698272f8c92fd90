/*
 * Seeded, counter-based synthetic input generator for the selective-scan
 * workloads.  It holds no arithmetic of the scan itself: it only draws
 * numbers (uniform, normal, log-uniform) and rounds them to the storage
 * dtype.  Both the fp64 oracle and the CUDA path take their inputs from
 * here, so the two sides always see bit-identical tensors.
 *
 * Generator: SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014), used as a counter-based function:
 * element i of stream s under seed k is mix64(key(k, s) + (i + 1) * GAMMA).
 * Any slice of a tensor can therefore be regenerated on its own, which is
 * what the sampled checks at full size rely on.
 *
 * Normals: Box-Muller in fp64 on the uniform pair (2*floor(i/2), 2*floor(i/2)+1);
 * even i takes the cosine branch, odd i the sine branch.
 *
 * Rounding to the storage dtype is round-to-nearest-even from the fp64 value
 * (no double rounding through fp32 on the way to bf16).
 *
 * Plain C, scalar libm calls only (no vector math), so that a value depends
 * only on its counter and never on where it falls in a buffer.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
    return mix64(mix64(seed + GAMMA) ^ (stream * 0xD1B54A32D192ED03ULL + 0x2545F4914F6CDD1DULL));
}

/* the SplitMix64 output function, exported for its published test vectors */
uint64_t ssm_gen_mix64(uint64_t z) { return mix64(z); }

uint64_t ssm_gen_raw64(uint64_t seed, uint64_t stream, uint64_t i) {
    return mix64(stream_key(seed, stream) + (i + 1) * GAMMA);
}

/* uniform in the open interval (0, 1): 53 random bits, offset by half a step */
static inline double u01(uint64_t key, uint64_t i) {
    uint64_t r = mix64(key + (i + 1) * GAMMA);
    return ((double)(r >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

/* fp64 -> bf16 bits, round to nearest, ties to even, straight from fp64 */
uint16_t ssm_f64_to_bf16(double x) {
    uint64_t b;
    memcpy(&b, &x, 8);
    uint64_t sign = b >> 63;
    int64_t e = (int64_t)((b >> 52) & 0x7FF);
    uint64_t m = b & ((1ULL << 52) - 1);
    if (e == 0 && m == 0) return (uint16_t)(sign << 15); /* signed zero */
    if (e == 0x7FF) { /* inf / nan */
        return (uint16_t)((sign << 15) | 0x7F80 | (m ? 0x40 : 0));
    }
    int64_t fe = e - 1023 + 127; /* fp32/bf16 biased exponent */
    if (fe >= 1) {
        uint64_t keep = m >> 45;           /* 7 mantissa bits */
        uint64_t rem = m & ((1ULL << 45) - 1);
        uint64_t half = 1ULL << 44;
        if (rem > half || (rem == half && (keep & 1))) keep += 1;
        if (keep == 128) { keep = 0; fe += 1; }
        if (fe >= 255) return (uint16_t)((sign << 15) | 0x7F80); /* overflow -> inf */
        return (uint16_t)((sign << 15) | ((uint64_t)fe << 7) | keep);
    }
    /* bf16 subnormal range: value = k * 2^-133, k < 128; round |x| / 2^-133 */
    double ax = fabs(x);
    double k = ax * 0x1p133;              /* exact scaling by a power of two */
    double fl = floor(k);
    double fr = k - fl;
    uint64_t ki = (uint64_t)fl;
    if (fr > 0.5 || (fr == 0.5 && (ki & 1))) ki += 1;
    /* ki == 128 is the smallest normal, whose bit pattern is the same */
    return (uint16_t)((sign << 15) | ki);
}

enum { GEN_F64 = 0, GEN_F32 = 1, GEN_BF16 = 2 };
enum { DIST_NORMAL = 0, DIST_UNIFORM = 1, DIST_LOGUNIFORM = 2, DIST_CONST = 3, DIST_SPINV_LOGUNIFORM = 4 };

typedef struct {
    uint64_t key;
    int64_t offset, begin, end;
    int dist;
    double p0, p1, p2;  /* normal: scale, shift; uniform: lo, hi; loguniform: lo, hi, floor;
                           const: value; spinv_loguniform: lo, hi, floor */
    int out_dtype;
    void* out;
} job_t;

static double draw(const job_t* j, uint64_t i) {
    switch (j->dist) {
    case DIST_NORMAL: {
        uint64_t pair = i & ~1ULL;
        double a = u01(j->key, pair), b = u01(j->key, pair + 1);
        double r = sqrt(-2.0 * log(a));
        double th = 6.283185307179586476925286766559 * b;
        double g = (i & 1) ? r * sin(th) : r * cos(th);
        return g * j->p0 + j->p1;
    }
    case DIST_UNIFORM:
        return j->p0 + (j->p1 - j->p0) * u01(j->key, i);
    case DIST_LOGUNIFORM:
    case DIST_SPINV_LOGUNIFORM: {
        /* log-uniform step size in [lo, hi], floored (the usual dt init) */
        double lo = log(j->p0), hi = log(j->p1);
        double dt = exp(lo + (hi - lo) * u01(j->key, i));
        if (dt < j->p2) dt = j->p2;
        if (j->dist == DIST_LOGUNIFORM) return dt;
        /* the bias b with log(1 + e^b) = dt, i.e. b = dt + log(1 - e^-dt) */
        return dt + log(-expm1(-dt));
    }
    default:
        return j->p0;
    }
}

static void* run_job(void* arg) {
    job_t* j = (job_t*)arg;
    for (int64_t k = j->begin; k < j->end; ++k) {
        double v = draw(j, (uint64_t)(j->offset + k));
        switch (j->out_dtype) {
        case GEN_F64: ((double*)j->out)[k] = v; break;
        case GEN_F32: ((float*)j->out)[k] = (float)v; break; /* IEEE cast: RN-even */
        default: ((uint16_t*)j->out)[k] = ssm_f64_to_bf16(v); break;
        }
    }
    return NULL;
}

/*
 * Fill out[0..count) with elements offset..offset+count of stream `stream`.
 * Returns 0 on success, -1 on a bad argument.
 */
int ssm_gen_fill(uint64_t seed, uint64_t stream, int64_t offset, int64_t count, int dist,
                 double p0, double p1, double p2, int out_dtype, void* out, int nthreads) {
    if (count < 0 || offset < 0 || (count > 0 && !out)) return -1;
    if (dist < 0 || dist > 4 || out_dtype < 0 || out_dtype > 2) return -1;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (count < 65536) nthreads = 1;
    job_t jobs[256];
    pthread_t th[256];
    int live[256] = {0};
    uint64_t key = stream_key(seed, stream);
    int64_t per = (count + nthreads - 1) / nthreads;
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].key = key;
        jobs[t].offset = offset;
        jobs[t].begin = t * per < count ? t * per : count;
        jobs[t].end = (t + 1) * per < count ? (t + 1) * per : count;
        jobs[t].dist = dist;
        jobs[t].p0 = p0;
        jobs[t].p1 = p1;
        jobs[t].p2 = p2;
        jobs[t].out_dtype = out_dtype;
        jobs[t].out = out;
    }
    for (int t = 1; t < nthreads; ++t) {
        live[t] = pthread_create(&th[t], NULL, run_job, &jobs[t]) == 0;
        if (!live[t]) run_job(&jobs[t]); /* no thread available: do it here */
    }
    run_job(&jobs[0]);
    for (int t = 1; t < nthreads; ++t)
        if (live[t]) pthread_join(th[t], NULL);
    return 0;
}
