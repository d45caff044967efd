/*
 * ss_scan_debug.h -- test hooks of libssscan.so.  Not for production use.
 *
 * Each setting is picked up by the NEXT ss_scan_fwd (SS_DEBUG_STEP_SIMPLE:
 * ss_scan_step) call in the process and
 * then cleared (ss_scan_workspace_bytes honours a pending worker count, so a
 * test can size the workspace for it).  They exist so that tests can drive the
 * load-balanced schedule and its bounded carry waits on small problems:
 *
 *   SS_DEBUG_FORCE_WORKERS  value = number of CTAs that share the work (>= 1;
 *                           capped at the number of channel groups), so ranges
 *                           split channel groups and carries are handed over.
 *   SS_DEBUG_SKIP_PUBLISH   value = worker index whose carry is never published:
 *                           its successor's bounded wait runs out, the kernel
 *                           returns without hanging and ss_last_device_error
 *                           reports SS_ERR_TIMEOUT.  The outputs of that call
 *                           are then unspecified.
 *   SS_DEBUG_SPIN_LIMIT     value = polls (with back-off) before a carry wait
 *                           gives up, so that test finishes quickly.
 *   SS_DEBUG_STEP_SIMPLE    value != 0: the next ss_scan_step call takes the
 *                           plain-load kernel even where the bulk-copy
 *                           pipeline applies, so both are tested on one shape.
 *   SS_DEBUG_FORCE_SEGMENTS value = number of segments each channel group's
 *                           sequence is cut into (>= 1, capped at its number
 *                           of chunks; 1: none), so the carry-in correction
 *                           runs on problems small enough to check in full.
 *                           Ignored by the training forward.
 *   SS_DEBUG_CLEAR          value ignored: drop every pending setting.
 *
 * Returns SS_OK, or SS_ERR_INVALID_ARG for an unknown `what`.  Host-only,
 * thread-safe, launches nothing.
 */
#ifndef SS_SCAN_DEBUG_H_
#define SS_SCAN_DEBUG_H_

#include "ss_scan.h"

#ifdef __cplusplus
extern "C" {
#endif

enum {
  SS_DEBUG_CLEAR = 0,
  SS_DEBUG_FORCE_WORKERS = 1,
  SS_DEBUG_SKIP_PUBLISH = 2,
  SS_DEBUG_SPIN_LIMIT = 3,
  SS_DEBUG_STEP_SIMPLE = 4,
  SS_DEBUG_FORCE_SEGMENTS = 5
};

ss_status ss_debug_inject(int what, long long value);

/*
 * ss_debug_fwd_kernels -- how many kernels one ss_scan_fwd call launches for
 * this shape and input dtype on the current device: 1, or 2 when the
 * sequence is cut into segments scanned at once (the scan, then the carry-in
 * correction).  Pending debug settings are honoured, not cleared.  -1 for
 * unsupported arguments or when the device cannot be queried.  Host-only,
 * launches nothing.  (For benchmarks that count their launches.)
 */
int ss_debug_fwd_kernels(int64_t batch, int64_t dim, int64_t seqlen, int dstate, ss_dtype in_dtype);

/*
 * ss_debug_pointwise -- evaluate one of the scan kernels' pointwise functions
 * element by element on the device, so that a test can compare it with
 * float64 over its input range: y[i] = f(x[i]) for i < n.
 *
 *   fn  SS_PW_SOFTPLUS, SS_PW_SILU: softplus(x) = log(1 + e^x) and
 *       SiLU(x) = x sigmoid(x) as the forward kernel evaluates them (one
 *       special-function op for softplus, two for SiLU);
 *       SS_PW_SOFTPLUS2, SS_PW_SILU2: the packed forms, on pairs (x[2i], x[2i+1]);
 *       SS_PW_EXP2_NEG_FMA: 2^x for x <= 0 by polynomial on the FMA pipe
 *       (x is clamped at -126);
 *       SS_PW_RCP_1_2: 1/x for x in [1, 2] by Newton-Raphson on the FMA pipe;
 *       SS_PW_EX2: the special-function unit's 2^x (ex2.approx.ftz).
 *   x, y  device float arrays of n elements (4-byte aligned; may not overlap).
 *
 * Asynchronous on `stream`.  SS_ERR_INVALID_ARG for an unknown fn, n < 0 or
 * null or misaligned pointers with n > 0; SS_ERR_CUDA if the launch fails.
 */
enum {
  SS_PW_SOFTPLUS = 0,
  SS_PW_SILU = 1,
  SS_PW_SOFTPLUS2 = 2,
  SS_PW_SILU2 = 3,
  SS_PW_EXP2_NEG_FMA = 4,
  SS_PW_RCP_1_2 = 5,
  SS_PW_EX2 = 6
};
ss_status ss_debug_pointwise(int fn, const float* x, float* y, int64_t n, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SS_SCAN_DEBUG_H_ */
