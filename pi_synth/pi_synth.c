/*
 * pi_synth.c -- seeded synthetic inputs for the pi-attention operator and its oracle.
 *
 * This module only draws numbers; it holds none of the operator's arithmetic.  Both the CUDA
 * path (through the tests and the bench) and the fp64 oracle read the arrays it writes, so they
 * see identical bits.
 *
 * Generator: Philox4x32-10, the counter-based generator of Salmon, Moraes, Dror and Shaw,
 * "Parallel random numbers: as easy as 1, 2, 3" (SC'11), written here from its published
 * definition (round function, multipliers and Weyl key increments of that paper).
 * Normals: Box-Muller in double precision on two 53-bit uniforms taken from one Philox block.
 *
 * Element e of a tensor (flat index) with (seed, stream) takes block counter
 *   ctr = (lo32(e/2), hi32(e/2), stream, 0), key = (lo32(seed), hi32(seed))
 * and uses the cosine branch when e is even, the sine branch when e is odd.  Any element, hence
 * any row, can therefore be regenerated on its own.
 *
 * Storage: the double value  mean + std * z * (row scale)  is rounded to fp32 (C cast, round to
 * nearest even), and for bf16 storage the fp32 value is rounded once more to bf16 (round to
 * nearest even on the bit pattern).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

static void philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int r = 0; r < 10; ++r) {
        uint64_t p0 = (uint64_t)PHILOX_M0 * c0;
        uint64_t p1 = (uint64_t)PHILOX_M1 * c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
        k0 += PHILOX_W0; k1 += PHILOX_W1;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* Exported for a known-answer test of the block function. */
void pi_synth_philox(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
    philox4x32_10(ctr, key, out);
}

/* Standard normal for flat element index e. */
static double normal_at(uint64_t seed, uint32_t stream, uint64_t e) {
    uint64_t pair = e >> 1;
    uint32_t ctr[4] = {(uint32_t)pair, (uint32_t)(pair >> 32), stream, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t x[4];
    philox4x32_10(ctr, key, x);
    uint64_t a = ((uint64_t)x[1] << 32 | x[0]) >> 11; /* 53 bits */
    uint64_t b = ((uint64_t)x[3] << 32 | x[2]) >> 11;
    const double two53 = 9007199254740992.0;
    double u1 = ((double)a + 0.5) / two53; /* in (0, 1) */
    double u2 = ((double)b + 0.5) / two53;
    double r = sqrt(-2.0 * log(u1));
    double th = 6.283185307179586476925286766559 * u2;
    return (e & 1) ? r * sin(th) : r * cos(th);
}

static uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)((u >> 16) | ((u & 0xFFFFu) ? 0x40u : 0u));
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* One fill request.  Rows (row_len elements each) whose position within their sequence
 * ((e / row_len) modulo seq_rows) is a multiple of scale_every have std multiplied by
 * scale_factor before rounding; scale_every == 0 disables this. */
typedef struct {
    void* out;
    int is_bf16;
    uint64_t seed;
    uint32_t stream;
    double mean, stdv;
    uint64_t row_len, seq_rows, scale_every;
    double scale_factor;
    /* contiguous mode */
    uint64_t e0, count;
    /* listed-rows mode */
    const int64_t* rows;
    uint64_t nrows;
    uint64_t begin, end; /* work slice for this thread */
} job_t;

static float value_at(const job_t* j, uint64_t e) {
    double z = normal_at(j->seed, j->stream, e);
    double s = j->stdv;
    if (j->scale_every && j->row_len && j->seq_rows) {
        uint64_t row_in_seq = (e / j->row_len) % j->seq_rows;
        if (row_in_seq % j->scale_every == 0) s *= j->scale_factor;
    }
    return (float)(j->mean + s * z);
}

static void* run_contig(void* arg) {
    job_t* j = (job_t*)arg;
    for (uint64_t t = j->begin; t < j->end; ++t) {
        float f = value_at(j, j->e0 + t);
        if (j->is_bf16) ((uint16_t*)j->out)[t] = f32_to_bf16_rne(f);
        else ((float*)j->out)[t] = f;
    }
    return 0;
}

static void* run_rows(void* arg) {
    job_t* j = (job_t*)arg;
    for (uint64_t t = j->begin; t < j->end; ++t) {
        uint64_t base = (uint64_t)j->rows[t] * j->row_len;
        for (uint64_t c = 0; c < j->row_len; ++c) {
            float f = value_at(j, base + c);
            uint64_t o = t * j->row_len + c;
            if (j->is_bf16) ((uint16_t*)j->out)[o] = f32_to_bf16_rne(f);
            else ((float*)j->out)[o] = f;
        }
    }
    return 0;
}

#define MAX_THREADS 256

static void run_threads(job_t* proto, uint64_t total, int nthreads, void* (*fn)(void*)) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > MAX_THREADS) nthreads = MAX_THREADS;
    if (total < (uint64_t)nthreads) nthreads = total ? (int)total : 1;
    pthread_t th[MAX_THREADS];
    int created[MAX_THREADS];
    job_t jobs[MAX_THREADS];
    uint64_t chunk = (total + nthreads - 1) / nthreads;
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = *proto;
        uint64_t b = (uint64_t)i * chunk, e = b + chunk;
        jobs[i].begin = b < total ? b : total;
        jobs[i].end = e < total ? e : total;
        created[i] = 0;
        if (i > 0 && jobs[i].begin < jobs[i].end)
            created[i] = pthread_create(&th[i], 0, fn, &jobs[i]) == 0;
    }
    fn(&jobs[0]);
    for (int i = 1; i < nthreads; ++i) {
        if (created[i]) pthread_join(th[i], 0);
        else if (jobs[i].begin < jobs[i].end) fn(&jobs[i]);
    }
}

/* Fill out[0..count) with elements e0..e0+count of the (seed, stream) tensor. */
void pi_synth_fill(void* out, int is_bf16, uint64_t e0, uint64_t count, uint64_t seed,
                   uint32_t stream, double mean, double stdv, uint64_t row_len, uint64_t seq_rows,
                   uint64_t scale_every, double scale_factor, int nthreads) {
    job_t j;
    memset(&j, 0, sizeof j);
    j.out = out; j.is_bf16 = is_bf16; j.seed = seed; j.stream = stream; j.mean = mean;
    j.stdv = stdv; j.row_len = row_len; j.seq_rows = seq_rows; j.scale_every = scale_every;
    j.scale_factor = scale_factor; j.e0 = e0; j.count = count;
    run_threads(&j, count, nthreads, run_contig);
}

/* Fill out[t*row_len .. (t+1)*row_len) with full row rows[t] (flat row index) of the tensor. */
void pi_synth_fill_rows(void* out, int is_bf16, const int64_t* rows, uint64_t nrows,
                        uint64_t row_len, uint64_t seed, uint32_t stream, double mean, double stdv,
                        uint64_t seq_rows, uint64_t scale_every, double scale_factor, int nthreads) {
    job_t j;
    memset(&j, 0, sizeof j);
    j.out = out; j.is_bf16 = is_bf16; j.seed = seed; j.stream = stream; j.mean = mean;
    j.stdv = stdv; j.row_len = row_len; j.seq_rows = seq_rows; j.scale_every = scale_every;
    j.scale_factor = scale_factor; j.rows = rows; j.nrows = nrows;
    run_threads(&j, nrows, nthreads, run_rows);
}
