/*
 * Seeded synthetic inputs for the DSA hot path (indexer -> top-k -> sparse
 * GQA attention).  Test and benchmark infrastructure only: this file holds
 * no arithmetic of the method itself, only random draws and the storage
 * encodings of the drawn values (FP8 e4m3 bytes, bf16 bits).
 *
 * Every element is a pure function of (seed, tensor id, element index):
 *
 *   base(seed, tensor) = mix(seed * G + mix(tensor + C))
 *   draw(seed, tensor, i) = mix(base + (i + 1) * G)
 *
 * where mix() is the splitmix64 output function (Steele, Lea and Flood,
 * "Fast splittable pseudorandom number generators", OOPSLA 2014) and G is
 * its golden-ratio increment.  Any sub-range of a tensor can therefore be
 * produced on its own, in any order, by any number of threads, and both
 * the oracle and the GPU path see exactly the same bytes.
 *
 *   uniform integer U{lo..hi}: lo + floor(draw * n / 2^64), n = hi - lo + 1
 *                              (multiply-shift; bias below n / 2^64)
 *   normal N(0, 1):            Box-Muller on the draw pair (2j, 2j+1):
 *                              element 2j takes the cosine branch, 2j+1 the
 *                              sine branch; u1 in (0,1], u2 in [0,1)
 *   bf16 storage:              fp64 -> fp32 -> bf16, each step
 *                              round-to-nearest-even
 *   e4m3 storage:              exact for the integers drawn here (|v| <= 16)
 *
 * The video-structured prefill (240 frames of 16 text + 1076 vision tokens,
 * then 64 trailing text tokens) draws a per-frame centroid from its own
 * tensor id and adds per-element noise to it for vision tokens.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>
#include <unistd.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t stream_base(uint64_t seed, uint32_t tensor) {
    return mix64(seed * GOLDEN + mix64((uint64_t)tensor + 0x632BE59BD9B4E019ULL));
}

static inline uint64_t draw(uint64_t base, uint64_t i) {
    return mix64(base + (i + 1) * GOLDEN);
}

static inline int uniform_int(uint64_t r, int lo, int hi) {
    uint64_t n = (uint64_t)(hi - lo + 1);
    return lo + (int)(((unsigned __int128)r * n) >> 64);
}

/* Standard normal for element i of a stream (Box-Muller, pair i/2). */
static inline double normal_at(uint64_t base, uint64_t i) {
    uint64_t j = i >> 1;
    uint64_t r1 = draw(base, 2 * j), r2 = draw(base, 2 * j + 1);
    double u1 = (double)((r1 >> 11) + 1) * 0x1.0p-53;  /* (0, 1] */
    double u2 = (double)(r2 >> 11) * 0x1.0p-53;        /* [0, 1) */
    double rad = sqrt(-2.0 * log(u1));
    double th = 6.283185307179586476925286766559 * u2;
    return (i & 1) ? rad * sin(th) : rad * cos(th);
}

static inline uint16_t to_bf16(double x) {
    float f = (float)x;
    uint32_t b;
    memcpy(&b, &f, 4);
    b += 0x7FFFu + ((b >> 16) & 1u);
    return (uint16_t)(b >> 16);
}

/* e4m3 (bias 7, no infinities, max 448) encoding, round-to-nearest-even,
 * saturating at +-448.  Only ever fed small integers here, which are exact. */
static uint8_t to_e4m3(double x) {
    uint8_t s = 0;
    if (x < 0) { s = 0x80; x = -x; }
    if (x == 0) return s;
    if (x >= 448.0) return s | 0x7E;
    int e;
    double m = frexp(x, &e);           /* x = m * 2^e, m in [0.5, 1) */
    int E = e - 1;                     /* x = (2m) * 2^E, 2m in [1, 2) */
    if (E < -6) {                      /* subnormal: multiples of 2^-9 */
        double q = ldexp(x, 9);
        double r = nearbyint(q);       /* default rounding mode is RNE */
        int mi = (int)r;
        if (mi >= 8) return s | 0x08;  /* rounds up to the smallest normal */
        return s | (uint8_t)mi;
    }
    double frac = (2.0 * m - 1.0) * 8.0;
    int mi = (int)nearbyint(frac);
    if (mi == 8) { mi = 0; E += 1; }
    if (E > 8 || (E == 8 && mi > 6)) return s | 0x7E;
    return s | (uint8_t)(((E + 7) << 3) | mi);
}

/* ---------------------------------------------------------------- threads */

typedef void (*range_fn)(void* arg, uint64_t lo, uint64_t hi);
typedef struct { range_fn fn; void* arg; uint64_t lo, hi; } job_t;

static void* run_job(void* p) {
    job_t* j = (job_t*)p;
    j->fn(j->arg, j->lo, j->hi);
    return NULL;
}

static void parallel_for(uint64_t count, int nthreads, range_fn fn, void* arg) {
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (count < (uint64_t)nthreads * 4096) nthreads = 1;
    if (nthreads == 1) { fn(arg, 0, count); return; }
    pthread_t th[256];
    job_t jobs[256];
    uint64_t per = (count + nthreads - 1) / nthreads;
    int started = 0;
    for (int t = 0; t < nthreads; ++t) {
        uint64_t lo = per * t, hi = lo + per;
        if (lo >= count) break;
        if (hi > count) hi = count;
        jobs[t] = (job_t){fn, arg, lo, hi};
        if (pthread_create(&th[t], NULL, run_job, &jobs[t]) != 0) {
            run_job(&jobs[t]);
            th[t] = 0;
        }
        started = t + 1;
    }
    for (int t = 0; t < started; ++t)
        if (th[t]) pthread_join(th[t], NULL);
}

/* ------------------------------------------------------------ i.i.d. draws */

typedef struct {
    uint64_t base, start;
    int lo, hi;
    double sigma;
    void* out;
} iid_arg;

static void k_int_e4m3(void* a_, uint64_t lo, uint64_t hi) {
    iid_arg* a = (iid_arg*)a_;
    uint8_t* out = (uint8_t*)a->out;
    for (uint64_t k = lo; k < hi; ++k)
        out[k] = to_e4m3((double)uniform_int(draw(a->base, a->start + k), a->lo, a->hi));
}
static void k_int_f32(void* a_, uint64_t lo, uint64_t hi) {
    iid_arg* a = (iid_arg*)a_;
    float* out = (float*)a->out;
    for (uint64_t k = lo; k < hi; ++k)
        out[k] = (float)uniform_int(draw(a->base, a->start + k), a->lo, a->hi);
}
static void k_int_i64(void* a_, uint64_t lo, uint64_t hi) {
    iid_arg* a = (iid_arg*)a_;
    int64_t* out = (int64_t*)a->out;
    for (uint64_t k = lo; k < hi; ++k)
        out[k] = uniform_int(draw(a->base, a->start + k), a->lo, a->hi);
}
static void k_normal_bf16(void* a_, uint64_t lo, uint64_t hi) {
    iid_arg* a = (iid_arg*)a_;
    uint16_t* out = (uint16_t*)a->out;
    for (uint64_t k = lo; k < hi; ++k)
        out[k] = to_bf16(a->sigma * normal_at(a->base, a->start + k));
}

void dsagen_int_e4m3(uint64_t seed, uint32_t tensor, uint64_t start, uint64_t count,
                     int lo, int hi, uint8_t* out, int nthreads) {
    iid_arg a = {stream_base(seed, tensor), start, lo, hi, 0.0, out};
    parallel_for(count, nthreads, k_int_e4m3, &a);
}
void dsagen_int_f32(uint64_t seed, uint32_t tensor, uint64_t start, uint64_t count,
                    int lo, int hi, float* out, int nthreads) {
    iid_arg a = {stream_base(seed, tensor), start, lo, hi, 0.0, out};
    parallel_for(count, nthreads, k_int_f32, &a);
}
void dsagen_int_i64(uint64_t seed, uint32_t tensor, uint64_t start, uint64_t count,
                    int lo, int hi, int64_t* out, int nthreads) {
    iid_arg a = {stream_base(seed, tensor), start, lo, hi, 0.0, out};
    parallel_for(count, nthreads, k_int_i64, &a);
}
void dsagen_normal_bf16(uint64_t seed, uint32_t tensor, uint64_t start, uint64_t count,
                        double sigma, uint16_t* out, int nthreads) {
    iid_arg a = {stream_base(seed, tensor), start, 0, 0, sigma, out};
    parallel_for(count, nthreads, k_normal_bf16, &a);
}

/* Encodes caller-given values (small integers) as e4m3 bytes; used by tests
 * that build hand-made inputs. */
void dsagen_encode_e4m3(const double* v, uint64_t count, uint8_t* out) {
    for (uint64_t k = 0; k < count; ++k) out[k] = to_e4m3(v[k]);
}
void dsagen_encode_bf16(const double* v, uint64_t count, uint16_t* out) {
    for (uint64_t k = 0; k < count; ++k) out[k] = to_bf16(v[k]);
}

/* ----------------------------------------------------- video-structured draws
 * Token p is a vision token of frame f = p / frame_tokens when
 * p < nframes * frame_tokens and p % frame_tokens >= text_tokens; every other
 * token (per-frame timestamp text, trailing prompt) is text. */

typedef struct {
    uint64_t noise_base, cent_base, start;
    uint64_t row_elems;   /* elements per token */
    uint64_t cent_elems;  /* centroid elements per frame (period of the pattern) */
    int64_t frame_tokens, text_tokens, nframes;
    int cent_lo, cent_hi, noise_lo, noise_hi, text_lo, text_hi, clamp_lo, clamp_hi;
    double sigma_noise;
    void* out;
} video_arg;

static inline int64_t vision_frame(const video_arg* a, uint64_t token) {
    if ((int64_t)token >= a->nframes * a->frame_tokens) return -1;
    int64_t f = (int64_t)token / a->frame_tokens;
    int64_t w = (int64_t)token % a->frame_tokens;
    return w >= a->text_tokens ? f : -1;
}

static void k_video_int(void* a_, uint64_t lo, uint64_t hi) {
    video_arg* a = (video_arg*)a_;
    uint8_t* out = (uint8_t*)a->out;
    for (uint64_t k = lo; k < hi; ++k) {
        uint64_t i = a->start + k;
        uint64_t token = i / a->row_elems;
        int64_t f = vision_frame(a, token);
        int v;
        if (f < 0) {
            v = uniform_int(draw(a->noise_base, i), a->text_lo, a->text_hi);
        } else {
            uint64_t c = (i % a->row_elems) % a->cent_elems;
            int cen = uniform_int(draw(a->cent_base, (uint64_t)f * a->cent_elems + c),
                                  a->cent_lo, a->cent_hi);
            v = cen + uniform_int(draw(a->noise_base, i), a->noise_lo, a->noise_hi);
            if (v < a->clamp_lo) v = a->clamp_lo;
            if (v > a->clamp_hi) v = a->clamp_hi;
        }
        out[k] = to_e4m3((double)v);
    }
}

static void k_video_normal(void* a_, uint64_t lo, uint64_t hi) {
    video_arg* a = (video_arg*)a_;
    uint16_t* out = (uint16_t*)a->out;
    for (uint64_t k = lo; k < hi; ++k) {
        uint64_t i = a->start + k;
        uint64_t token = i / a->row_elems;
        int64_t f = vision_frame(a, token);
        double v;
        if (f < 0) {
            v = normal_at(a->noise_base, i);
        } else {
            uint64_t c = (i % a->row_elems) % a->cent_elems;
            v = normal_at(a->cent_base, (uint64_t)f * a->cent_elems + c) +
                a->sigma_noise * normal_at(a->noise_base, i);
        }
        out[k] = to_bf16(v);
    }
}

/* Integer-valued e4m3 tensor of row_elems elements per token.  The centroid
 * has cent_elems entries per frame and element e of a token uses centroid
 * entry e % cent_elems (so all indexer heads of a query share the frame's
 * centroid with the keys of that frame). */
void dsagen_video_int_e4m3(uint64_t seed, uint32_t noise_tensor, uint32_t cent_tensor,
                           uint64_t start, uint64_t count, uint64_t row_elems,
                           uint64_t cent_elems, int64_t frame_tokens, int64_t text_tokens,
                           int64_t nframes, int cent_lo, int cent_hi, int noise_lo,
                           int noise_hi, int text_lo, int text_hi, int clamp_lo,
                           int clamp_hi, uint8_t* out, int nthreads) {
    video_arg a;
    memset(&a, 0, sizeof a);
    a.noise_base = stream_base(seed, noise_tensor);
    a.cent_base = stream_base(seed, cent_tensor);
    a.start = start; a.row_elems = row_elems; a.cent_elems = cent_elems;
    a.frame_tokens = frame_tokens; a.text_tokens = text_tokens; a.nframes = nframes;
    a.cent_lo = cent_lo; a.cent_hi = cent_hi; a.noise_lo = noise_lo; a.noise_hi = noise_hi;
    a.text_lo = text_lo; a.text_hi = text_hi; a.clamp_lo = clamp_lo; a.clamp_hi = clamp_hi;
    a.out = out;
    parallel_for(count, nthreads, k_video_int, &a);
}

/* bf16 tensor: vision tokens are centroid N(0,1) + sigma_noise * N(0,1),
 * text tokens N(0,1). */
void dsagen_video_normal_bf16(uint64_t seed, uint32_t noise_tensor, uint32_t cent_tensor,
                              uint64_t start, uint64_t count, uint64_t row_elems,
                              int64_t frame_tokens, int64_t text_tokens, int64_t nframes,
                              double sigma_noise, uint16_t* out, int nthreads) {
    video_arg a;
    memset(&a, 0, sizeof a);
    a.noise_base = stream_base(seed, noise_tensor);
    a.cent_base = stream_base(seed, cent_tensor);
    a.start = start; a.row_elems = row_elems; a.cent_elems = row_elems;
    a.frame_tokens = frame_tokens; a.text_tokens = text_tokens; a.nframes = nframes;
    a.sigma_noise = sigma_noise;
    a.out = out;
    parallel_for(count, nthreads, k_video_normal, &a);
}
