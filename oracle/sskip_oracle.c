/*
 * CPU oracle for Skip-Softmax tiled attention (prefill and split-KV decode).
 *
 * TEST INFRASTRUCTURE ONLY: the parity tests, the smoke check and the CPU
 * baseline leg of the benchmark are its only callers.  It shares no code,
 * header, helper or constant with the CUDA library, and the CUDA library never
 * calls it.
 *
 * Plain C: one (batch, head, query tile) unit -- or one (batch, kv head) group
 * for decode -- at a time, in the order the algorithm states, on a pool of
 * POSIX threads that only hands out independent units.  See
 * sskip_oracle_impl.h for the algorithm and the readings of the pages.
 *
 * Build: gcc -O2 -fPIC -shared -pthread sskip_oracle.c -o libsskip_oracle.so -lm
 * (no -ffast-math: the oracle keeps IEEE semantics, including -inf).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 -> fp32 widening is exact: the bf16 bits are the top half of fp32. */
static float bf16_to_float(uint16_t h) {
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return f;
}

typedef void* (*worker_fn)(void*);

static void run_workers(worker_fn fn, void* job, int nthreads, int n_units) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > n_units) nthreads = n_units > 0 ? n_units : 1;
    if (nthreads > 512) nthreads = 512;
    pthread_t th[512];
    int started = 0;
    for (int t = 1; t < nthreads; ++t)
        if (pthread_create(&th[started], NULL, fn, job) == 0) ++started;
    fn(job);
    for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
}

#define REAL float
#define SUFFIX _f32
#define EXP expf
#define LOG logf
#include "sskip_oracle_impl.h"
#undef REAL
#undef SUFFIX
#undef EXP
#undef LOG

#define REAL double
#define SUFFIX _f64
#define EXP exp
#define LOG log
#include "sskip_oracle_impl.h"
#undef REAL
#undef SUFFIX
#undef EXP
#undef LOG

int sskip_oracle_version(void) { return 1; }
