/*
 * rrf_oracle_mt.c -- a row-parallel driver of the oracle, for the CPU
 * baseline's all-cores leg.
 *
 * TEST INFRASTRUCTURE ONLY, like rrf_oracle.c: only the tests and the
 * benchmark's CPU-baseline leg may call it.  It adds no arithmetic: the rows
 * of a call are split into contiguous chunks, one per POSIX thread, and each
 * chunk goes to the unchanged oracle_sum_rmsnorm_fp8_rows.  Rows are
 * independent (each row's statistics come from that row alone), so the
 * result is bit-identical to the single-threaded call whatever the thread
 * count.
 */
#define _GNU_SOURCE
#include <pthread.h>
#include <sched.h>
#include <stdint.h>
#include <stdlib.h>
#include <unistd.h>

void oracle_sum_rmsnorm_fp8_rows(const uint16_t* const* x, int R, int64_t row0,
                                 int64_t nrows, int64_t cols, const uint16_t* res_in,
                                 uint16_t* res_out, const uint16_t* gamma, float eps,
                                 float weight_offset, float scale_ub, uint8_t* q,
                                 float* scales, uint16_t* h_out, float* v_out);

/* Cores this process may run on (its CPU affinity mask), at least 1. */
int oracle_cores(void) {
    cpu_set_t set;
    if (sched_getaffinity(0, sizeof(set), &set) == 0) {
        const int n = CPU_COUNT(&set);
        if (n > 0) return n;
    }
    const long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

struct chunk {
    const uint16_t* const* x;
    int R;
    int64_t row0, nrows, cols;
    const uint16_t* res_in;
    uint16_t* res_out;
    const uint16_t* gamma;
    float eps, weight_offset, scale_ub;
    uint8_t* q;
    float* scales;
};

static void* run_chunk(void* p) {
    const struct chunk* c = (const struct chunk*)p;
    oracle_sum_rmsnorm_fp8_rows(c->x, c->R, c->row0, c->nrows, c->cols, c->res_in, c->res_out,
                                c->gamma, c->eps, c->weight_offset, c->scale_ub, c->q,
                                c->scales, NULL, NULL);
    return NULL;
}

/* oracle_sum_rmsnorm_fp8 over all rows on `threads` threads (0: one per
 * core of oracle_cores()); chunk k holds rows [k * rows / n, (k + 1) * rows
 * / n).  Returns the number of threads used, or -1 if a thread could not be
 * started (the rows it would have run are then run on the calling thread). */
int oracle_sum_rmsnorm_fp8_mt(const uint16_t* const* x, int R, int64_t rows, int64_t cols,
                              const uint16_t* res_in, uint16_t* res_out, const uint16_t* gamma,
                              float eps, float weight_offset, float scale_ub, uint8_t* q,
                              float* scales, int threads) {
    int n = threads > 0 ? threads : oracle_cores();
    if (n > rows) n = rows > 0 ? (int)rows : 1;
    struct chunk* cs = (struct chunk*)calloc((size_t)n, sizeof(struct chunk));
    pthread_t* ts = (pthread_t*)calloc((size_t)n, sizeof(pthread_t));
    int* started = (int*)calloc((size_t)n, sizeof(int));
    int status = n;
    if (cs == NULL || ts == NULL || started == NULL) {
        free(cs);
        free(ts);
        free(started);
        struct chunk all = {x, R, 0, rows, cols, res_in, res_out, gamma, eps, weight_offset,
                            scale_ub, q, scales};
        run_chunk(&all);
        return -1;
    }
    for (int k = 0; k < n; ++k) {
        const int64_t lo = rows * k / n, hi = rows * (k + 1) / n;
        struct chunk c = {x, R, lo, hi - lo, cols, res_in, res_out, gamma, eps, weight_offset,
                          scale_ub, q, scales};
        cs[k] = c;
        started[k] = pthread_create(&ts[k], NULL, run_chunk, &cs[k]) == 0;
        if (!started[k]) status = -1;
    }
    for (int k = 0; k < n; ++k) {
        if (started[k]) pthread_join(ts[k], NULL);
        else run_chunk(&cs[k]);
    }
    free(cs);
    free(ts);
    free(started);
    return status;
}
