/*
 * ss_scan.h -- C ABI of libssscan.so: the S6 selective-scan forward on one
 * NVIDIA B200 (sm_100a).
 *
 * The operation (pages: "从Transformer的痛点说起 ... Mamba", sec. 2.2, 3.1 and
 * the SelectiveSSM of sec. 4.2; "Mamba 选择性机制", sec. 1.1, 2.2 and 3.1;
 * "Mamba 深度解读报告", sec. 2.3-2.4).  For every batch row b and channel d,
 * with t = 0..L-1 and n = 0..N-1, starting from h = 0:
 *
 *   Delta_t = softplus(delta[b,d,t] + delta_bias[d])   (softplus_flag != 0)
 *           = delta[b,d,t] + delta_bias[d]             (softplus_flag == 0)
 *   h[n]    = exp(Delta_t * A[d,n]) * h[n] + Delta_t * B[b,n,t] * u[b,d,t]
 *   y[b,d,t]= (sum_n C[b,n,t] * h[n] + D[d] * u[b,d,t]) * SiLU(z[b,d,t])
 *   last_state[b,d,n] = h[n] after t = L-1
 *
 * B_bar is the simplified Delta*B of the first page's sec. 2.2; the readout
 * uses the state after the update that includes token t; the gate multiplies
 * the skip term too (sec. 4.2 order: add x*D, then multiply by SiLU(z)).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers, caller-owned, contiguous, with
 *    the fastest axis last as written ([B,D,L] means L fastest).
 *  - The library never allocates device memory at run time, never
 *    synchronises the stream (except ss_last_device_error) and keeps no state
 *    beyond one device-side error word per device (and the static scratch
 *    array of ss_scan_fwd_noalloc, part of the loaded module).
 *  - Calls are asynchronous on `stream` (0 = the legacy default stream), and
 *    may be captured into a CUDA graph and replayed (the captured buffers,
 *    workspace included, are reused by every replay; replays of one graph, or
 *    calls sharing a workspace, must not run concurrently).
 *  - Arguments are checked on the host before any launch; a rejected call
 *    launches nothing and touches no buffer.
 */
#ifndef SS_SCAN_H_
#define SS_SCAN_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SS_OK = 0,
  SS_ERR_INVALID_ARG = 1, /* null required pointer, bad size, bad alignment, workspace too small */
  SS_ERR_UNSUPPORTED = 2, /* dstate not in {16, 32, 64, 128}, unknown dtype, or more
                             scratch than ss_scan_fwd_noalloc holds */
  SS_ERR_CUDA = 3,        /* a CUDA launch or runtime call failed */
  SS_ERR_TIMEOUT = 4,     /* a bounded inter-block wait gave up (see ss_last_device_error) */
  SS_ERR_BOUNDS = 5       /* checked builds only: a kernel formed an index outside its
                             tensor and skipped the access (see ss_last_device_error) */
} ss_status;

typedef enum { SS_F32 = 0, SS_BF16 = 1 } ss_dtype;

/*
 * ss_scan_fwd -- the fused forward: discretise, scan, read out, gate, store.
 *
 *  u, delta, z   [batch, dim, seqlen]   in_dtype            (z nullable: no gate)
 *  A             [dim, dstate]          float32             (real diagonal, normally < 0)
 *  B, C          [batch, dstate, seqlen] in_dtype           (shared by all channels)
 *  D, delta_bias [dim]                  float32             (nullable: treated as 0)
 *  softplus_flag nonzero: Delta = softplus(delta + delta_bias)
 *  y_out         [batch, dim, seqlen]   float32 (written)
 *  last_state_out[batch, dim, dstate]   float32 (nullable: not written)
 *  batch, dim, seqlen >= 1; batch*dim*seqlen < 2^62
 *  dstate        16, 32, 64 or 128
 *  workspace     device scratch of at least ss_scan_workspace_bytes(...) bytes,
 *                caller-owned, 256-byte aligned (nullable when that is 0).
 *                Its contents on entry do not matter; the call may overwrite it.
 *                Two calls in flight at once must not share one workspace.
 *                It holds what the chosen schedule hands between CTAs: the
 *                carries of the load-balanced schedule and the counter from
 *                which its CTAs take their worker ids (the call zeroes it on
 *                the stream before its kernel), or, when the sequence
 *                is cut into segments scanned at once (few channels, long L),
 *                each segment's end state and sum of Delta, from which a
 *                second kernel adds every segment's carry-in to y and forms
 *                last_state (the associative operator of "Mamba 选择性机制",
 *                sec. 3.1).
 *
 * Alignment: every tensor pointer must be aligned to its element size.  When
 * seqlen*sizeof(in_dtype) is a multiple of 16 and u, delta, z, B, C, y_out are
 * 16-byte aligned the kernel moves 16-byte vectors; otherwise it falls back to
 * element-wise loads (correct, slower).
 *
 * Returns SS_OK after a successful launch (errors raised later inside the
 * kernel are reported by ss_last_device_error), or an error code with nothing
 * launched.
 */
ss_status ss_scan_fwd(const void* u, const void* delta, const float* A,
                      const void* B, const void* C, const float* D,
                      const void* z, const float* delta_bias,
                      int softplus_flag, float* y_out, float* last_state_out,
                      int64_t batch, int64_t dim, int64_t seqlen, int dstate,
                      ss_dtype in_dtype, void* workspace,
                      size_t workspace_bytes, cudaStream_t stream);

/*
 * ss_scan_fwd_from_state -- ss_scan_fwd started from a carried state instead
 * of zero: h[n] = initial_state[b,d,n] before t = 0.  This continues a
 * sequence across calls (a long prompt fed in pieces, or a prompt after
 * earlier turns of a dialogue); the pages keep h between calls for recurrent
 * inference ("从Transformer的痛点说起 ... Mamba", sec. 5.1 table and sec. 6.3).
 * Scanning [0, P) and then [P, L) from the first call's last_state gives the
 * outputs of one call over [0, L), up to fp32 rounding.
 *
 *  initial_state [batch, dim, dstate]  float32, nullable (then exactly
 *                ss_scan_fwd).  It may be the same buffer as last_state_out
 *                (the state is then advanced in place); any other overlap
 *                with an output is not allowed.
 *
 * Every other argument, layout, result and error is that of ss_scan_fwd; the
 * workspace size is the same ss_scan_workspace_bytes(...).
 */
ss_status ss_scan_fwd_from_state(const void* u, const void* delta, const float* A,
                                 const void* B, const void* C, const float* D,
                                 const void* z, const float* delta_bias,
                                 int softplus_flag, const float* initial_state,
                                 float* y_out, float* last_state_out,
                                 int64_t batch, int64_t dim, int64_t seqlen,
                                 int dstate, ss_dtype in_dtype, void* workspace,
                                 size_t workspace_bytes, cudaStream_t stream);

/*
 * ss_scan_fwd_zoh -- ss_scan_fwd with the exact zero-order-hold input matrix
 * instead of its simplification ("从Transformer的痛点说起 ... Mamba", sec. 2.2:
 * B_bar = (Delta A)^-1 (exp(Delta A) - I) Delta B, which implementations
 * usually simplify to Delta B).  For diagonal A:
 *
 *   h[n] = exp(Delta_t A[d,n]) h[n] + (exp(Delta_t A[d,n]) - 1) / A[d,n] B[b,n,t] u[b,d,t]
 *
 * and Delta_t B[b,n,t] u[b,d,t] where A[d,n] = 0 (the limit).  Near
 * Delta A = 0 the kernel takes (exp(x) - 1)/x from its Taylor series, so no
 * cancellation reaches the state.  Arguments, layouts, results, errors and
 * the workspace size are those of ss_scan_fwd.
 */
ss_status ss_scan_fwd_zoh(const void* u, const void* delta, const float* A,
                          const void* B, const void* C, const float* D,
                          const void* z, const float* delta_bias,
                          int softplus_flag, float* y_out, float* last_state_out,
                          int64_t batch, int64_t dim, int64_t seqlen, int dstate,
                          ss_dtype in_dtype, void* workspace,
                          size_t workspace_bytes, cudaStream_t stream);

/*
 * ss_scan_fwd_conv -- ss_scan_fwd whose input u is formed inside the kernel
 * from the block's short convolution: the causal depthwise Conv1d of width W
 * (padding W-1, cut to the first L outputs) followed by SiLU
 * ("从Transformer的痛点说起 ... Mamba", sec. 3.3 block diagram and the sec. 4.2
 * code), so the convolved activation never goes through HBM:
 *
 *   u[b,d,t] = SiLU(conv_bias[d] + sum_{k<W} conv_weight[d,k] x[b,d,t-(W-1)+k]),
 *   x[b,d,t] = 0 for t < 0 (tap W-1 meets the current token).
 *
 *  x            [batch, dim, seqlen]  in_dtype   (takes the place of u)
 *  conv_weight  [dim, conv_width]     float32    (required)
 *  conv_bias    [dim]                 float32    (nullable: 0)
 *  conv_width   1..4 (others: SS_ERR_UNSUPPORTED)
 *
 * The scan starts from h = 0 and from x = 0 before t = 0.  Every other
 * argument, layout, result and error is that of ss_scan_fwd (u there is the
 * convolution's output, here computed); D multiplies that output, as in the
 * sec. 4.2 code.  The workspace size is ss_scan_workspace_bytes(...).
 */
ss_status ss_scan_fwd_conv(const void* x, const float* conv_weight,
                           const float* conv_bias, int conv_width,
                           const void* delta, const float* A, const void* B,
                           const void* C, const float* D, const void* z,
                           const float* delta_bias, int softplus_flag,
                           float* y_out, float* last_state_out, int64_t batch,
                           int64_t dim, int64_t seqlen, int dstate,
                           ss_dtype in_dtype, void* workspace,
                           size_t workspace_bytes, cudaStream_t stream);

/*
 * ss_scan_step -- one recurrent (decode) step: the same recurrence over a
 * single token, advancing a carried state in place ("从Transformer的痛点说起
 * ... Mamba", sec. 5.1 table: O(1) work and memory per generated token;
 * sec. 6.3: the state h is kept per sample between steps).  For every b, d, n:
 *
 *   Delta      = softplus(delta[b,d] + delta_bias[d])  (or without softplus)
 *   state[b,d,n] <- exp(Delta * A[d,n]) * state[b,d,n] + Delta * B[b,n] * u[b,d]
 *   y[b,d]     = (sum_n C[b,n] * state[b,d,n] + D[d] * u[b,d]) * SiLU(z[b,d])
 *
 *  u, delta, z   [batch, dim]          in_dtype     (z nullable: no gate)
 *  A             [dim, dstate]         float32
 *  B, C          [batch, dstate]       in_dtype
 *  D, delta_bias [dim]                 float32      (nullable: 0)
 *  state         [batch, dim, dstate]  float32, read and written in place
 *  y_out         [batch, dim]          float32 (written); must not overlap state
 *  batch, dim >= 1, batch*dim*dstate <= 2^56, dim*dstate < 2^31;
 *  dstate 16, 32, 64 or 128
 *
 * Device pointers, caller-owned, contiguous, each aligned to its element
 * size; 16-byte aligned state and A and (4 * element size)-aligned B and C
 * take vector loads, anything else element-wise loads (correct, slower).
 * No workspace.  Returns SS_OK after the launch, or an error code with nothing
 * launched (SS_ERR_INVALID_ARG, SS_ERR_UNSUPPORTED, SS_ERR_CUDA).
 */
ss_status ss_scan_step(const void* u, const void* delta, const float* A,
                       const void* B, const void* C, const float* D,
                       const void* z, const float* delta_bias, int softplus_flag,
                       float* state, float* y_out, int64_t batch, int64_t dim,
                       int dstate, ss_dtype in_dtype, cudaStream_t stream);

/*
 * ss_scan_fwd_train -- ss_scan_fwd that also writes the state at the start of
 * every 16-step chunk, for ss_scan_bwd to start its recomputation from
 * instead of running its own forward pass first (the states within a chunk
 * are still recomputed, never stored).
 *
 *  checkpoints  [batch, ceil(seqlen / 16), dim, dstate] float32, 16-byte
 *               aligned, caller-owned (required): checkpoints[b, k, d, n] = h[n]
 *               of channel (b, d) before step 16 k (zero for k = 0).
 *
 * Every other argument, layout, result and error is that of ss_scan_fwd.
 */
ss_status ss_scan_fwd_train(const void* u, const void* delta, const float* A,
                            const void* B, const void* C, const float* D,
                            const void* z, const float* delta_bias,
                            int softplus_flag, float* y_out, float* last_state_out,
                            float* checkpoints, int64_t batch, int64_t dim,
                            int64_t seqlen, int dstate, ss_dtype in_dtype,
                            void* workspace, size_t workspace_bytes,
                            cudaStream_t stream);

/*
 * ss_scan_bwd -- gradients of ss_scan_fwd (simplified B_bar, zero initial
 * state) for an upstream gradient dy of y (and optionally dlast_state of the
 * final state).  The forward's states are not stored anywhere: the backward
 * recomputes them from the inputs ("Mamba 深度解读报告", sec. 3.3;
 * "Mamba 选择性机制", sec. 3.4), keeping only the state at the start of every
 * 16-step chunk in the caller's workspace.  With a_t = exp(Delta_t A),
 * q_t = C_t . h_t + D u_t, y_t = q_t SiLU(z_t) and the adjoint
 * g_t = dL/dh_t = dq_t C_t + a_{t+1} g_{t+1}:
 *
 *   dz       = dy q SiLU'(z),           dq = dy SiLU(z)   (dq = dy without z)
 *   du       = dq D + sum_n g Delta B
 *   ddelta   = (sum_n g (B u + A a h_{t-1})) * softplus'(delta + bias)
 *              (times 1 without the softplus)
 *   dA[d,n]  = sum_{b,t} g Delta a h_{t-1}
 *   dB, dC   = sum_d g Delta u,  sum_d dq h_t         [batch, dstate, seqlen]
 *   dD[d]    = sum_{b,t} dq u,   ddelta_bias[d] = sum_{b,t} ddelta
 *
 * Inputs exactly as ss_scan_fwd; dy [batch, dim, seqlen] float32 (required);
 * dlast_state [batch, dim, dstate] float32 (nullable: 0); checkpoints: those
 * ss_scan_fwd_train wrote for the same inputs (nullable: the call computes
 * them itself into the workspace, and then needs it; with checkpoints the
 * workspace may be null).  Outputs, all
 * float32 and overwritten: du, ddelta [batch, dim, seqlen] (required); dz
 * (required when z is given, ignored otherwise); dA [dim, dstate], dB, dC
 * [batch, dstate, seqlen] (required); dD (nullable; ignored without D),
 * ddelta_bias [dim] (nullable).  dA, dB, dC, dD and ddelta_bias are summed
 * with atomic adds after the call zeroes them on `stream` (so their low bits
 * may vary from call to call).  workspace (without checkpoints): at least
 * ss_scan_bwd_workspace_bytes(...) bytes, 256-byte aligned, caller-owned.
 * Any element alignment; errors as ss_scan_fwd.
 */
ss_status ss_scan_bwd(const void* u, const void* delta, const float* A,
                      const void* B, const void* C, const float* D,
                      const void* z, const float* delta_bias, int softplus_flag,
                      const float* dy, const float* dlast_state,
                      const float* checkpoints, float* du,
                      float* ddelta, float* dA, float* dB, float* dC, float* dD,
                      float* dz, float* ddelta_bias, int64_t batch, int64_t dim,
                      int64_t seqlen, int dstate, ss_dtype in_dtype,
                      void* workspace, size_t workspace_bytes,
                      cudaStream_t stream);

/* Bytes of workspace ss_scan_bwd needs without given checkpoints, which is
 * also the size of the checkpoint array: 4 x batch x ceil(seqlen / 16) x dim x
 * dstate, rounded up to 256; (size_t)-1 for sizes it would reject. */
size_t ss_scan_bwd_workspace_bytes(int64_t batch, int64_t dim, int64_t seqlen,
                                   int dstate);

/*
 * ss_scan_fwd_noalloc -- ss_scan_fwd for callers that cannot allocate device
 * memory at the point of the call: for example a plugin running inside a host
 * framework that owns every device allocation (a cudaMalloc of its own would
 * bypass that pool and its accounting), or a latency-critical path where the
 * implicit synchronisation of cudaMalloc/cudaFree is not acceptable.  The
 * method on the pages has no counterpart of this entry point; it only changes
 * where the scratch memory comes from.
 *
 * Arguments, layouts, results and errors are those of ss_scan_fwd, minus the
 * workspace.  The scratch the scan may need (the carries handed between CTAs
 * of the load-balanced schedule, or the segment states and sums of a long
 * sequence cut into segments) lives in one static device array of
 * SS_NOALLOC_SCRATCH_BYTES that the library owns; every GPU that loads the
 * library holds it until the process exits.  This entry point calls no
 * cudaMalloc, cudaFree or allocating library routine.
 *
 *  - The first call on a device (with that device current) looks the array's
 *    device address up once; make that first call before any stream capture.
 *  - Problems whose schedule needs more scratch than SS_NOALLOC_SCRATCH_BYTES
 *    (ss_scan_workspace_bytes(...) larger than it) are rejected with
 *    SS_ERR_UNSUPPORTED and nothing is launched.
 *  - Every call shares the one array and it keeps the last call's contents;
 *    nothing in it has to start at zero (hand-over flags carry a per-launch
 *    value, so stale contents are never taken as fresh).  Calls that overlap
 *    on the GPU (two streams, or two host threads) race on the array: issue
 *    them one after another on a stream, or use ss_scan_fwd with separate
 *    workspaces.
 */
#define SS_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)

ss_status ss_scan_fwd_noalloc(const void* u, const void* delta, const float* A,
                              const void* B, const void* C, const float* D,
                              const void* z, const float* delta_bias,
                              int softplus_flag, float* y_out,
                              float* last_state_out, int64_t batch,
                              int64_t dim, int64_t seqlen, int dstate,
                              ss_dtype in_dtype, cudaStream_t stream);

/* Bytes of workspace ss_scan_fwd needs for these sizes on the current device
 * (0 when the chosen kernel needs none).  Returns (size_t)-1 for sizes that
 * ss_scan_fwd would reject. */
size_t ss_scan_workspace_bytes(int64_t batch, int64_t dim, int64_t seqlen,
                               int dstate);

/* Static, NUL-terminated description of a status code. */
const char* ss_status_string(ss_status status);

/* Synchronises `stream`, then reads and clears the device error word of the
 * current device: SS_OK, SS_ERR_BOUNDS when a kernel of a checked build
 * (compiled with SS_BOUNDS_CHECK: every global index compared with its
 * tensor's extent, a miss skipped and recorded instead of trapping) met an
 * index outside its tensor, or SS_ERR_TIMEOUT when a bounded wait inside a
 * kernel gave up, since the last query.  SS_ERR_CUDA if the synchronisation
 * itself failed. */
ss_status ss_last_device_error(cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SS_SCAN_H_ */
