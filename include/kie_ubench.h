/* kie_ubench.h -- micro-benchmarks that bound the batch-1 decode kernel.
 *
 * The monokernel page ("Kog Inference Engine" monokernel section) motivates
 * the persistent design with two costs of conventional decode stacks: about
 * 4.5 us of launch overhead per kernel and grid-wide synchronisation taking
 * roughly a third of each token's time.  These calls measure both on the
 * local GPU, together with the ceiling of the kernel's weight stream (the
 * same 32 KB bulk-copy ring with and without its GEMV arithmetic), so that
 * the decode kernel's roofline fraction can be read against what the copy
 * pipeline itself reaches.  They are measurements, not part of decoding.
 *
 * Conventions: calls are synchronous on the current device; every in-kernel
 * wait is bounded (about two seconds of SM cycles) and reports
 * KIE_UB_ERR_TIMEOUT instead of hanging.  Pointers named src are DEVICE
 * memory owned by the caller; outputs are HOST scalars.
 */
#ifndef KIE_UBENCH_H
#define KIE_UBENCH_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  KIE_UB_OK = 0,
  KIE_UB_ERR_INVALID = -1, /* bad argument */
  KIE_UB_ERR_CUDA = -3,    /* a CUDA call failed */
  KIE_UB_ERR_TIMEOUT = -6  /* a bounded in-kernel wait ran out */
};

/* n_launches empty kernels (1 block of 32 threads) back to back on one
 * stream after 16 warm-up launches; *us_per_launch = event time / n. */
int kie_ubench_launch_overhead(int32_t n_launches, float *us_per_launch);

/* The decode kernel's weight stream alone: n_ctas CTAs (one per SM), each
 * walking its own bytes_per_cta region of src (CTA c reads
 * src + c * bytes_per_cta) `passes` times in 32 KB tiles through a ring of
 * ring_slots (1..6) shared-memory slots filled by one producer lane with
 * 1-D bulk copies; 16 consumer warps wait on every tile and release it,
 * computing a row GEMV of the tile when consume != 0.  src must be 16-byte
 * aligned and hold n_ctas * bytes_per_cta bytes; bytes_per_cta a positive
 * multiple of 32768.  *ms_out = event time of one launch after a warm-up. */
int kie_ubench_stream(const void *src, int64_t bytes_per_cta, int32_t n_ctas, int32_t passes,
                      int32_t ring_slots, int32_t consume, float *ms_out);

/* n_rounds grid-wide dependency points back to back: in each round every
 * CTA release-adds 1 to one counter and waits (acquire loads) until all
 * n_ctas CTAs have added, the decode kernel's wait for every SM.  n_ctas
 * must not exceed the SM count (cooperative launch).  *us_per_round = best
 * of 3 launches' event time / n_rounds. */
int kie_ubench_barrier(int32_t n_ctas, int32_t n_rounds, float *us_per_round);

#ifdef __cplusplus
}
#endif

#endif
