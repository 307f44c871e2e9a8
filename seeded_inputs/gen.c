/*
 * Seeded synthetic inputs shared by the CPU oracle and the CUDA path.
 *
 * This file holds random-number generation only; none of the MoE layer's
 * arithmetic lives here.  Every value is a pure function of
 * (seed, tensor_id, element index), so any slice of any tensor can be
 * generated on its own, in any thread, and always comes out the same.
 *
 * Generator: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014).  The stream for one tensor
 * starts from the state key(seed, tensor_id); output i is the SplitMix64
 * finaliser applied to key + (i + 1) * golden_gamma, which is exactly the
 * (i+1)-th output of a SplitMix64 generator seeded with key.
 *
 * Normals: Box-Muller (G. Box, M. Muller, 1958).  Pair j draws two uniforms,
 * u1 in (0,1] from output 2j and u2 in [0,1) from output 2j+1, and gives
 * z[2j] = sqrt(-2 ln u1) cos(2 pi u2), z[2j+1] = sqrt(-2 ln u1) sin(2 pi u2).
 *
 * Storage: value = std * z in double, rounded to fp32 (round to nearest even);
 * bf16 storage rounds that fp32 value to bf16 (round to nearest even).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t sg_stream_key(uint64_t seed, uint64_t tensor_id) {
    return mix64(mix64(seed + GOLDEN_GAMMA) ^ (tensor_id * 0xD1B54A32D192ED03ULL));
}

static inline uint64_t draw(uint64_t key, uint64_t i) {
    return mix64(key + (i + 1) * GOLDEN_GAMMA);
}

/* Raw 64-bit outputs [start, start+count) of one stream. */
void sg_u64(uint64_t seed, uint64_t tensor_id, uint64_t start, uint64_t count, uint64_t* out) {
    uint64_t key = sg_stream_key(seed, tensor_id);
    for (uint64_t i = 0; i < count; ++i) out[i] = draw(key, start + i);
}

static inline double normal_at(uint64_t key, uint64_t i) {
    uint64_t j = i >> 1;
    uint64_t a = draw(key, 2 * j), b = draw(key, 2 * j + 1);
    double u1 = (double)((a >> 11) + 1) * 0x1.0p-53; /* (0, 1] */
    double u2 = (double)(b >> 11) * 0x1.0p-53;       /* [0, 1) */
    double r = sqrt(-2.0 * log(u1));
    double ang = 6.283185307179586476925286766559 * u2;
    return (i & 1) ? r * sin(ang) : r * cos(ang);
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40); /* quiet NaN */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

typedef struct {
    uint64_t key, start, lo, hi;
    double mean, std;
    int kind;   /* 0 normal, 1 lognormal */
    int dtype;  /* 0 f32, 1 bf16, 2 f64 */
    void* out;
} job_t;

static void* worker(void* arg) {
    job_t* jb = (job_t*)arg;
    for (uint64_t i = jb->lo; i < jb->hi; ++i) {
        double z = normal_at(jb->key, jb->start + i);
        double v = jb->kind == 0 ? jb->mean + jb->std * z : exp(jb->mean + jb->std * z);
        if (jb->dtype == 2) {
            ((double*)jb->out)[i] = v;
        } else if (jb->dtype == 0) {
            ((float*)jb->out)[i] = (float)v;
        } else {
            ((uint16_t*)jb->out)[i] = f32_to_bf16_rne((float)v);
        }
    }
    return 0;
}

/*
 * Fill out[0..count) with elements [start, start+count) of the stream
 * (seed, tensor_id): kind 0 gives mean + std*z, kind 1 gives exp(mean + std*z)
 * (lognormal with parameters mu = mean, sigma = std).  dtype: 0 fp32, 1 bf16
 * (uint16 bit patterns), 2 fp64.  Work is split over `threads` POSIX threads.
 */
int sg_fill(uint64_t seed, uint64_t tensor_id, uint64_t start, uint64_t count, int kind,
            double mean, double std, int dtype, void* out, int threads) {
    if (threads < 1) threads = 1;
    if (threads > 256) threads = 256;
    if (count < (uint64_t)threads * 65536) threads = (int)(count / 65536) + 1;
    uint64_t key = sg_stream_key(seed, tensor_id);
    pthread_t tid[256];
    job_t jobs[256];
    uint64_t per = (count + threads - 1) / threads;
    for (int t = 0; t < threads; ++t) {
        jobs[t].key = key;
        jobs[t].start = start;
        jobs[t].lo = per * t < count ? per * t : count;
        jobs[t].hi = per * (t + 1) < count ? per * (t + 1) : count;
        jobs[t].mean = mean;
        jobs[t].std = std;
        jobs[t].kind = kind;
        jobs[t].dtype = dtype;
        jobs[t].out = out;
    }
    if (threads == 1) {
        worker(&jobs[0]);
        return 0;
    }
    int started = 0;
    for (int t = 0; t < threads; ++t) {
        if (pthread_create(&tid[t], 0, worker, &jobs[t]) != 0) break;
        started++;
    }
    for (int t = started; t < threads; ++t) worker(&jobs[t]);
    for (int t = 0; t < started; ++t) pthread_join(tid[t], 0);
    return 0;
}
