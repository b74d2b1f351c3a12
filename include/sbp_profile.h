/*
 * sbp_profile.h -- launch accounting and GEMM timing of libsbp (instrumentation; the paper
 * has no counterpart).
 *
 * While profiling is on, every GEMM and attention call the library queues is bracketed by two
 * CUDA events on its own stream, so that a caller can read the device time of the dominant
 * kernels of a timed region.  Profiling is process-wide and off by default.
 */
#ifndef SBP_PROFILE_H_
#define SBP_PROFILE_H_

#include "sbp.h"

#ifdef __cplusplus
extern "C" {
#endif

enum {
  SBP_PROF_GEMM_TC = 0,   /* tcgen05 GEMM                               */
  SBP_PROF_GEMM_SIMT = 1, /* CUDA-core GEMM                             */
  SBP_PROF_ATTN_FWD = 2,  /* attention forward of a chunk (either path) */
  SBP_PROF_ATTN_BWD = 3,  /* attention backward of a chunk (either path) */
  SBP_PROF_KINDS = 4
};

typedef struct {
  long long launches[SBP_PROF_KINDS]; /* timed calls per kind                                  */
  double ms[SBP_PROF_KINDS];          /* summed device time per kind, milliseconds            */
  double busy_ms[SBP_PROF_KINDS];     /* device time during which at least one call of the kind
                                         ran (the union of its intervals: calls the library runs
                                         side by side on several streams are counted once)      */
} sbp_profile;

/* Number of kernels the library has launched in this process (all kinds). */
long long sbp_launch_count(void);

/* Start recording GEMM launches (clears earlier records). */
sbp_status sbp_profile_begin(void);

/* Stop recording, synchronise on the recorded events and fill `out` (may be NULL). */
sbp_status sbp_profile_end(sbp_profile* out);

#ifdef __cplusplus
}
#endif
#endif /* SBP_PROFILE_H_ */
