/*
 * lores_oracle_omp.c -- the CPU oracle's decode step over many (sequence, head) tiles
 * on all host cores.
 *
 * TEST AND BENCHMARK INFRASTRUCTURE ONLY (the CPU baseline of the benchmark; nothing in
 * the product path links, loads or calls it).  It adds no arithmetic: every tile is one
 * call of lo_tile_step from lores_oracle.c, compiled into the same library, and the
 * tiles of a step are independent (value rows of different tiles share nothing), so an
 * OpenMP loop over them computes exactly what the single-threaded loop computes.
 *
 * Build: gcc -O2 -std=c11 -fopenmp -ffp-contract=off -frounding-math -fPIC -shared
 *        lores_oracle.c lores_oracle_omp.c
 */
#include <stddef.h>
#include <stdint.h>

#include <omp.h>

/* lores_oracle.c; its first argument is a const lo_cfg *, passed through untouched */
int lo_tile_step(const void *c, void *state, float *scales, const float *q, const float *k,
                 const float *v, const float *alpha, float beta, uint32_t tile_key,
                 double *o_out, float *x_out);

/* One decode step of n tiles.  Tile t uses cfgs[cfg_of[t]], its state states[t] and
 * scales scales[t] (updated in place), q + t*d_k, k + t*d_k, v + t*d_v, alpha + t*a_len,
 * beta[t], tile_keys[t], and writes o + t*d_v.  flags[t] receives the step's return
 * value.  threads <= 0: OpenMP's default.  Returns the number of threads used. */
int lo_batch_step(const void *const *cfgs, const int *cfg_of, int n, void **states,
                  float **scales, const float *q, const float *k, const float *v,
                  const float *alpha, const float *beta, const uint32_t *tile_keys,
                  int d_k, int d_v, int a_len, double *o, int *flags, int threads)
{
    int used = 1;
    if (threads > 0)
        omp_set_num_threads(threads);
#pragma omp parallel
    {
#pragma omp single
        used = omp_get_num_threads();
#pragma omp for schedule(dynamic, 1)
        for (int t = 0; t < n; t++) {
            flags[t] = lo_tile_step(cfgs[cfg_of[t]], states[t], scales[t],
                                    q + (size_t)t * d_k, k + (size_t)t * d_k,
                                    v + (size_t)t * d_v, alpha + (size_t)t * a_len, beta[t],
                                    tile_keys[t], o + (size_t)t * d_v, (float *)0);
        }
    }
    return used;
}
