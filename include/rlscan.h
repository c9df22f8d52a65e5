/*
 * rlscan.h - C ABI of librlscan: RL credit assignment as one first-order
 * linear-recurrence scan, on CUDA kernels for NVIDIA B200 (sm_100a).
 *
 * What it computes.  The rl-triton paper (arXiv:2608.17641, abstract) recasts
 * seven credit-assignment estimators as instances of one first-order linear
 * recurrence x_t = a_t * x_{t+-1} + b_t, solved by an associative scan over
 * (a, b) pairs with the operator (a1, b1) o (a2, b2) = (a1 a2, a1 b2 + b1).
 * Each entry point below is one estimator of the rl-triton README's
 * "Kernels" table (compute_gae ... compute_episodic_prefix_sum); its call
 * follows the README's "Usage" example (rewards, values, terminateds, gamma,
 * lambda_) and the with-truncations paragraph under "Performance"
 * (terminations + time-limit truncations + bootstrap values).
 *
 * Common conventions (every entry point):
 *   - Layout: every [E, T] array is row-major and contiguous, T (seq_len)
 *     fastest: element (e, t) is at index e*T + t.  Retrace's per-action
 *     arrays are [E, T, A], A fastest.  E = num_envs, T = seq_len.
 *   - Memory: every pointer is DEVICE memory on the current device, owned by
 *     the caller, which keeps it alive until the stream reaches the call.
 *     Inputs are read, never written.  Outputs are written in full, must be
 *     preallocated, and must not overlap any input or each other
 *     (RLSCAN_ERR_INVALID_ARG).  16-byte-aligned pointers take the vectorised
 *     path; any other alignment is accepted and runs a scalar-load path.
 *   - Flags (terminateds, truncateds, dones) are float32; a flag is set iff it
 *     is nonzero.  terminated at t: the episode ends at t, nothing is
 *     bootstrapped and the trace is cut.  truncated at t: the episode ends at
 *     t, its value is bootstrapped from bootstrap_values[e, t] and the trace is
 *     cut.  If both are set, terminated wins.  bootstrap_values is read in
 *     full whenever truncateds is given (one streamed plane, no dependent
 *     loads); only its values at truncated steps matter.
 *   - last_values (nullable, [E]): the value after the last step of each row
 *     when that step carries no flag; NULL means 0.
 *   - Forward estimators (eligibility traces, prefix sum) reset after a done:
 *     dones[e, t-1] != 0 starts a new episode at t.
 *   - Results equal the sequential definition up to fp32 rounding (the scan
 *     re-associates); the int32 prefix sum is exact (two's-complement wrap).
 *   - Asynchrony: every compute call only enqueues work on `stream` (NULL =
 *     the legacy default stream); it never allocates, never synchronises and
 *     returns as soon as the kernel is launched.  E == 0 or T == 0 is a no-op
 *     returning RLSCAN_OK.  Calls are thread-safe.
 *   - Workspace: long rows (a row that spans several tiles) and rows that do
 *     not align with tiles need a device workspace of
 *     rlscan_workspace_bytes(E, T) bytes, 16-byte aligned, of any content
 *     (such a call runs two launches over chunks of consecutive elements, one
 *     chunk per warp: the first writes each chunk's 16-byte aggregate, the
 *     second scans each chunk with the carry it composes from the
 *     aggregates of the chunks before it; no kernel ever waits for another
 *     block or warp).  Shapes that need none
 *     accept ws = NULL.  A workspace holds one call's aggregates between its
 *     two launches: calls that share one must be ordered on one stream (or
 *     otherwise serialised).
 *   - Errors: a nonzero return is an rlscan_status; nothing was enqueued
 *     unless it is RLSCAN_ERR_CUDA from the launch itself.
 *     rlscan_last_error() gives a message for the calling thread.
 */
#ifndef RLSCAN_H
#define RLSCAN_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* 1.2.0: rlscan_gae_vtrace (GAE, TD(lambda) returns and V-Trace in one pass)
 * and its batch kind; rlscan_call holds four outputs and a vtrace_lambda
 * field at its end, so its size changed: clients built against an earlier
 * rlscan_call must be rebuilt (their rlscan_version() check fails).  Rows
 * that span tiles run the chunked two passes and need 16 bytes of workspace
 * per 1024 elements (time-major calls on few envs may need one too): size
 * workspaces with rlscan_workspace_bytes, never from a fixed formula.
 * 1.1.1: rlscan_call gained flag_dtype after dtype, which moved every later
 * field.  1.1.0: the _ex entry points (layout and done-convention options)
 * and rlscan_batch. */
#define RLSCAN_VERSION 120

/* Every entry point is exported from librlscan.so (built with hidden
 * visibility for everything else). */
#if defined(__GNUC__)
#define RLSCAN_API __attribute__((visibility("default")))
#else
#define RLSCAN_API
#endif

typedef enum rlscan_status {
    RLSCAN_OK = 0,
    RLSCAN_ERR_INVALID_ARG = 1, /* NULL required pointer, E/T/A < 0 or too large, non-finite
                                   gamma/lambda/rho_bar/c_bar, truncateds without
                                   bootstrap_values, overlapping buffers */
    RLSCAN_ERR_UNSUPPORTED = 2, /* unknown dtype, A above RLSCAN_MAX_ACTIONS */
    RLSCAN_ERR_WORKSPACE = 3,   /* the shape needs a workspace and ws is NULL, too small or
                                   not 16-byte aligned */
    RLSCAN_ERR_CUDA = 4,        /* a CUDA runtime call failed (message in rlscan_last_error) */
    RLSCAN_ERR_TIMEOUT = 5      /* reserved: returned by no call since 1.2.0, whose kernels
                                   never wait on one another */
} rlscan_status;

typedef enum rlscan_dtype {
    RLSCAN_F32 = 0,
    RLSCAN_I32 = 1,
    RLSCAN_BF16 = 2,
    RLSCAN_F16 = 3,
    RLSCAN_U8 = 4
} rlscan_dtype;

/* Largest action count accepted by rlscan_retrace. */
#define RLSCAN_MAX_ACTIONS 96

/*
 * GAE (README "Kernels": compute_gae, "backward scan over delta + gamma
 * lambda A"; Usage example for the positional arguments).
 *   delta_t = r_t + gamma * boot_t - V_t
 *   A_t = delta_t + gamma lambda A_{t+1} while the episode goes on, A_t = delta_t
 *   at a flagged step, A_T = 0; boot_t = V_{t+1} (V_T = last value), the
 *   bootstrap value at a truncation, 0 at a termination.
 * rewards, values [E,T] required; terminateds [E,T] nullable (no
 * terminations); truncateds [E,T] nullable; bootstrap_values [E,T] required
 * iff truncateds is given; last_values [E] nullable; advantages [E,T] output.
 */
RLSCAN_API int rlscan_gae(const float *rewards, const float *values, const float *terminateds,
               const float *truncateds, const float *bootstrap_values, const float *last_values,
               float *advantages, int64_t E, int64_t T, float gamma, float lambda_, void *ws,
               size_t ws_bytes, cudaStream_t stream);

/*
 * GAE and TD(lambda) returns in one pass (README "Kernels": compute_gae and
 * compute_lambda_returns over the same rewards, values and flags).  The
 * lambda-return equals the GAE advantage plus the value at every step
 * (Schulman et al. 2016, GAE section on value targets), so one scan gives
 * both: advantages_t = A_t as rlscan_gae, returns_t = A_t + V_t, which equals
 * rlscan_lambda_returns on the same inputs up to fp32 rounding.  Reads the
 * inputs once for both outputs (20 bytes per env-step instead of 32 for the
 * two calls).  Arguments as rlscan_gae plus the `returns` output [E,T]; the
 * two outputs must not overlap each other or any input.
 */
RLSCAN_API int rlscan_gae_with_returns(const float *rewards, const float *values, const float *terminateds,
                                       const float *truncateds, const float *bootstrap_values,
                                       const float *last_values, float *advantages, float *returns, int64_t E,
                                       int64_t T, float gamma, float lambda_, void *ws, size_t ws_bytes,
                                       cudaStream_t stream);

/*
 * GAE (and, when `returns` is not NULL, the TD(lambda) returns of the same
 * pass, as rlscan_gae_with_returns) from reduced-byte inputs: rewards,
 * values and bootstrap_values of `value_dtype` (RLSCAN_F32, RLSCAN_BF16 or
 * RLSCAN_F16), terminateds and truncateds of `flag_dtype` (RLSCAN_F32 or
 * RLSCAN_U8, one byte per flag, set iff nonzero; a bool tensor is RLSCAN_U8).
 * The path is memory-bound, so narrower inputs are fewer bytes: bf16 values
 * with u8 flags move 9 bytes per env-step for GAE instead of 16.  Inputs are
 * widened to fp32 in registers and all arithmetic and both outputs are fp32,
 * so results equal the fp32 entry points run on the widened inputs up to
 * fp32 rounding.  last_values stays fp32 [E].  Other arguments and errors as
 * rlscan_gae; an unsupported dtype returns RLSCAN_ERR_UNSUPPORTED.
 */
RLSCAN_API int rlscan_gae_typed(const void *rewards, const void *values, const void *terminateds,
                                const void *truncateds, const void *bootstrap_values, const float *last_values,
                                float *advantages, float *returns, int64_t E, int64_t T, float gamma,
                                float lambda_, int value_dtype, int flag_dtype, void *ws, size_t ws_bytes,
                                cudaStream_t stream);

/*
 * V-Trace (README "Kernels": compute_vtrace, "IS-weighted targets and
 * advantages"; IMPALA, Espeholt et al. 2018, section 4.1).
 *   rho_t = min(rho_bar, exp(log_rho_t)),  c_t = lambda min(c_bar, exp(log_rho_t))
 *   D_t = rho_t (r_t + gamma boot_t - V_t) + gamma c_t D_{t+1} (cut at flags), D_T = 0
 *   vs_t = V_t + D_t
 *   pg_advantages_t = rho_t (r_t + gamma boot'_t - V_t), boot'_t = vs_{t+1}
 *   while the episode goes on (vs_T = last value), the bootstrap value at a
 *   truncation, 0 at a termination.
 * lambda_ = 1 is IMPALA's v-trace.  log_rhos, rewards, values required;
 * others as rlscan_gae; vs and pg_advantages [E,T] outputs.
 */
RLSCAN_API int rlscan_vtrace(const float *log_rhos, const float *rewards, const float *values,
                  const float *terminateds, const float *truncateds,
                  const float *bootstrap_values, const float *last_values, float *vs,
                  float *pg_advantages, int64_t E, int64_t T, float gamma, float lambda_,
                  float rho_bar, float c_bar, void *ws, size_t ws_bytes, cudaStream_t stream);

/*
 * GAE advantages, TD(lambda) returns and V-Trace targets and advantages in
 * one pass (README "Kernels": compute_gae, compute_lambda_returns and
 * compute_vtrace over the same rewards, values and flags).  The two
 * recurrences, GAE's (gamma lambda, delta_t) and V-Trace's (gamma c_t,
 * rho_t delta_t) with the common delta_t = r_t + gamma boot_t - V_t, are
 * scanned together as one pair, so the inputs are read once for all four
 * outputs (32 bytes per env-step instead of 44 for rlscan_gae_with_returns
 * plus rlscan_vtrace).  advantages_t as rlscan_gae; returns_t = A_t + V_t as
 * rlscan_gae_with_returns (NULL: not written); vs_t and pg_advantages_t as
 * rlscan_vtrace with its lambda_ = vtrace_lambda (1 = IMPALA).  Each output
 * equals the separate entry point's on the same inputs up to fp32 rounding.
 * Inputs as rlscan_vtrace; outputs [E,T] (four, none overlapping another or
 * an input).  Errors as rlscan_vtrace.
 */
RLSCAN_API int rlscan_gae_vtrace(const float *log_rhos, const float *rewards, const float *values,
                                 const float *terminateds, const float *truncateds, const float *bootstrap_values,
                                 const float *last_values, float *advantages, float *returns, float *vs,
                                 float *pg_advantages, int64_t E, int64_t T, float gamma, float lambda_,
                                 float vtrace_lambda, float rho_bar, float c_bar, void *ws, size_t ws_bytes,
                                 cudaStream_t stream);

/*
 * Retrace(lambda) (README "Kernels": compute_retrace, "off-policy return
 * estimate with truncated IS ratios"; with-truncations paragraph:
 * terminated and truncated are both mandatory and there is no bootstrap
 * argument, the continuation value being folded into next_q_values_all at
 * every step; Munos et al. 2016).
 *   V'_t = sum_a next_target_probs[e,t,a] next_q_values_all[e,t,a]
 *          (A == 1: V'_t = next_q_values_all[e,t], next_target_probs NULL)
 *   delta_t = r_t + gamma (terminated_t ? 0 : V'_t) - q_t
 *   Dq_t = delta_t + gamma lambda min(c_bar, exp(log_rho_{t+1})) Dq_{t+1} while
 *   the episode goes on and t < T-1; Dq_t = delta_t otherwise
 *   q_ret_t = q_t + Dq_t
 * next_q_values_all[e,t,:] = Q(x_{t+1}, .) (the final observation's values at
 * a truncation; ignored at a termination); next_target_probs[e,t,:] =
 * pi(. | x_{t+1}); log_rhos[e,t] = log pi(a_t|x_t) - log mu(a_t|x_t);
 * q_values[e,t] = Q(x_t, a_t).  1 <= A <= RLSCAN_MAX_ACTIONS.  With A > 1
 * the call first writes V' into q_ret (one streaming launch over the
 * per-action arrays), then runs the recurrence on it as with A == 1,
 * rewriting q_ret in place.
 */
RLSCAN_API int rlscan_retrace(const float *rewards, const float *q_values, const float *next_q_values_all,
                   const float *next_target_probs, const float *log_rhos,
                   const float *terminateds, const float *truncateds, float *q_ret, int64_t E,
                   int64_t T, int64_t A, float gamma, float lambda_, float c_bar, void *ws,
                   size_t ws_bytes, cudaStream_t stream);

/*
 * TD(lambda) returns (README "Kernels": compute_lambda_returns, "lambda-return
 * targets mixing one-step TD and Monte Carlo").
 *   G_t = r_t + gamma ((1 - lambda) V_{t+1} + lambda G_{t+1}) while the episode goes on,
 *   G_t = r_t + gamma bootstrap_value_t at a truncation, G_t = r_t at a termination,
 *   V_T = G_T = last value.  Arguments as rlscan_gae; returns [E,T] output.
 */
RLSCAN_API int rlscan_lambda_returns(const float *rewards, const float *values, const float *terminateds,
                          const float *truncateds, const float *bootstrap_values,
                          const float *last_values, float *returns, int64_t E, int64_t T,
                          float gamma, float lambda_, void *ws, size_t ws_bytes,
                          cudaStream_t stream);

/*
 * Discounted returns (README "Kernels": compute_discounted_returns,
 * "discounted reward-to-go").
 *   R_t = r_t + gamma R_{t+1} while the episode goes on, r_t + gamma bootstrap_value_t
 *   at a truncation, r_t at a termination; R_T = last value.
 * rewards required; terminateds, truncateds, last_values nullable;
 * bootstrap_values required iff truncateds; returns [E,T] output.
 */
RLSCAN_API int rlscan_discounted_returns(const float *rewards, const float *terminateds,
                              const float *truncateds, const float *bootstrap_values,
                              const float *last_values, float *returns, int64_t E, int64_t T,
                              float gamma, void *ws, size_t ws_bytes, cudaStream_t stream);

/*
 * Eligibility traces (README "Kernels": compute_eligibility_traces,
 * "accumulating forward traces e[t] = x[t] + gamma lambda (1 - d) e[t-1]").
 *   e_t = x_t + gamma lambda e_{t-1} if t > 0 and dones[t-1] == 0, else x_t.
 * x required, dones nullable (no resets); traces [E,T] output.
 */
RLSCAN_API int rlscan_eligibility_traces(const float *x, const float *dones, float *traces, int64_t E,
                              int64_t T, float gamma, float lambda_, void *ws, size_t ws_bytes,
                              cudaStream_t stream);

/*
 * Episodic prefix sum (README "Kernels": compute_episodic_prefix_sum,
 * "episodic cumulative sum with done-mask resets").
 *   y_t = x_t + y_{t-1} if t > 0 and dones[t-1] == 0, else x_t.
 * x and out are [E,T] of `dtype`: RLSCAN_F32 (float) or RLSCAN_I32 (int32,
 * exact, wrapping modulo 2^32).  dones float32 [E,T], nullable.
 */
RLSCAN_API int rlscan_episodic_prefix_sum(const void *x, int dtype, const float *dones, void *out,
                               int64_t E, int64_t T, void *ws, size_t ws_bytes,
                               cudaStream_t stream);

/*
 * GAE with a fixed scratch area instead of a caller-supplied workspace.
 * No counterpart in the paper: the paper's kernels allocate their own
 * temporaries.  For callers that cannot allocate device memory: code whose
 * host application owns the whole device-memory budget and forbids
 * allocations from plugins, and latency-bound loops that must not call
 * cudaMalloc (which synchronises the device).  It computes exactly what
 * rlscan_gae computes, with the same arguments minus ws / ws_bytes.
 *
 * Scratch: one static device array of RLSCAN_NOALLOC_SCRATCH_BYTES bytes,
 * held on every GPU that loads the library until the process exits.  The
 * first call on a device looks up that array's device address (with that
 * device current) and caches it; make that first call before any stream
 * capture.  The cached address belongs to the device's context as it was
 * then: after cudaDeviceReset on that device it is stale, so a process that
 * resets a device must not call this entry point on it again.  Every call
 * clears the part of the array it uses with cudaMemsetAsync on `stream` and
 * allocates nothing.
 * Limit: shapes whose plan needs more scratch than the array holds (rows
 * that span tiles, over more than about 67 million elements in all: one
 * 16-byte slot per 1024 elements) return RLSCAN_ERR_WORKSPACE with the sizes
 * in rlscan_last_error().
 * All calls on one device share that device's array, which keeps the last
 * call's contents: two calls whose kernels may run at the same time on one
 * device (for example on two streams with no ordering between them) race on
 * it, so the caller must serialise them.  Calls on different devices use
 * different copies.
 */
#define RLSCAN_NOALLOC_SCRATCH_BYTES (1u << 20)
RLSCAN_API int rlscan_gae_noalloc(const float *rewards, const float *values, const float *terminateds,
                                  const float *truncateds, const float *bootstrap_values,
                                  const float *last_values, float *advantages, int64_t E, int64_t T,
                                  float gamma, float lambda_, cudaStream_t stream);

/*
 * Layout and episode-boundary options (the _ex entry points).
 *
 * Each estimator above has an _ex twin that takes one more argument,
 * `options`, an OR of the bits below, placed just before `ws`; all other
 * arguments mean what they mean above, and options == 0 is exactly the plain
 * call (the plain names are wrappers that pass 0).
 *
 *   RLSCAN_OPT_TIME_MAJOR: every [E, T] array (inputs and outputs) is
 *     instead [T, E], E (num_envs) fastest: element (e, t) is at index
 *     t*E + e, the rollout-buffer layout of vectorised environments that write
 *     one row of E per step.  last_values stays [E].  Rows are still scanned
 *     independently, reading and writing each element once with coalesced
 *     accesses along E.  With few envs and long rows, each row is split over
 *     several blocks (two launches: each split's map per env, then the
 *     splits with their carries) when ws holds rlscan_workspace_bytes(E, T)
 *     bytes (any content); with ws = NULL every row runs in one block.
 *     rlscan_retrace_ex takes it with A == 1 only, and E up to
 *     238,609,294 (offsets between timesteps are 32-bit); beyond either,
 *     RLSCAN_ERR_UNSUPPORTED.
 *   RLSCAN_OPT_DONE_STARTS_EPISODE (forward estimators only: eligibility
 *     traces and the episodic prefix sum; the rl-triton README's "Kernels"
 *     table writes the trace's (1-d) factor with no time index, and this is
 *     its other reading): dones[e, t] != 0 marks step t as
 *     the FIRST step of a new episode (the reset-flag convention: a "first" or
 *     "is_init" mask), instead of the default, where it marks t as the last
 *     step so that t+1 starts afresh.  With it, y_t = x_t where dones[t] != 0
 *     and the recurrence continues elsewhere.  Passing it to a backward
 *     estimator is RLSCAN_ERR_INVALID_ARG.
 * Unknown bits are RLSCAN_ERR_INVALID_ARG.
 */
#define RLSCAN_OPT_TIME_MAJOR 1u
#define RLSCAN_OPT_DONE_STARTS_EPISODE 2u

RLSCAN_API int rlscan_gae_ex(const float *rewards, const float *values, const float *terminateds,
                             const float *truncateds, const float *bootstrap_values, const float *last_values,
                             float *advantages, int64_t E, int64_t T, float gamma, float lambda_,
                             unsigned options, void *ws, size_t ws_bytes, cudaStream_t stream);
RLSCAN_API int rlscan_gae_typed_ex(const void *rewards, const void *values, const void *terminateds,
                                   const void *truncateds, const void *bootstrap_values, const float *last_values,
                                   float *advantages, float *returns, int64_t E, int64_t T, float gamma,
                                   float lambda_, int value_dtype, int flag_dtype, unsigned options, void *ws,
                                   size_t ws_bytes, cudaStream_t stream);
RLSCAN_API int rlscan_gae_with_returns_ex(const float *rewards, const float *values, const float *terminateds,
                                          const float *truncateds, const float *bootstrap_values,
                                          const float *last_values, float *advantages, float *returns, int64_t E,
                                          int64_t T, float gamma, float lambda_, unsigned options, void *ws,
                                          size_t ws_bytes, cudaStream_t stream);
RLSCAN_API int rlscan_vtrace_ex(const float *log_rhos, const float *rewards, const float *values,
                                const float *terminateds, const float *truncateds, const float *bootstrap_values,
                                const float *last_values, float *vs, float *pg_advantages, int64_t E, int64_t T,
                                float gamma, float lambda_, float rho_bar, float c_bar, unsigned options,
                                void *ws, size_t ws_bytes, cudaStream_t stream);
RLSCAN_API int rlscan_gae_vtrace_ex(const float *log_rhos, const float *rewards, const float *values,
                                    const float *terminateds, const float *truncateds,
                                    const float *bootstrap_values, const float *last_values, float *advantages,
                                    float *returns, float *vs, float *pg_advantages, int64_t E, int64_t T,
                                    float gamma, float lambda_, float vtrace_lambda, float rho_bar, float c_bar,
                                    unsigned options, void *ws, size_t ws_bytes, cudaStream_t stream);
RLSCAN_API int rlscan_retrace_ex(const float *rewards, const float *q_values, const float *next_q_values_all,
                                 const float *next_target_probs, const float *log_rhos, const float *terminateds,
                                 const float *truncateds, float *q_ret, int64_t E, int64_t T, int64_t A,
                                 float gamma, float lambda_, float c_bar, unsigned options, void *ws,
                                 size_t ws_bytes, cudaStream_t stream);
RLSCAN_API int rlscan_lambda_returns_ex(const float *rewards, const float *values, const float *terminateds,
                                        const float *truncateds, const float *bootstrap_values,
                                        const float *last_values, float *returns, int64_t E, int64_t T,
                                        float gamma, float lambda_, unsigned options, void *ws, size_t ws_bytes,
                                        cudaStream_t stream);
RLSCAN_API int rlscan_discounted_returns_ex(const float *rewards, const float *terminateds,
                                            const float *truncateds, const float *bootstrap_values,
                                            const float *last_values, float *returns, int64_t E, int64_t T,
                                            float gamma, unsigned options, void *ws, size_t ws_bytes,
                                            cudaStream_t stream);
RLSCAN_API int rlscan_eligibility_traces_ex(const float *x, const float *dones, float *traces, int64_t E,
                                            int64_t T, float gamma, float lambda_, unsigned options, void *ws,
                                            size_t ws_bytes, cudaStream_t stream);
RLSCAN_API int rlscan_episodic_prefix_sum_ex(const void *x, int dtype, const float *dones, void *out, int64_t E,
                                             int64_t T, unsigned options, void *ws, size_t ws_bytes,
                                             cudaStream_t stream);

/*
 * Several independent estimator calls in one request (no counterpart on the
 * pages, whose kernels each take one call): an RL update often needs several
 * estimators, or one estimator over several reward streams, on one batch.
 * Each rlscan_call describes one call of an entry point above; rlscan_batch
 * validates every call as that entry point would, then launches every call
 * whose rows fit whole in 1024-element tiles (row-major, 1024 a multiple of
 * T, A == 1 for Retrace; every kind below except GAE_VTRACE and typed GAE
 * with narrow inputs) as ONE fused kernel, each block running one tile of
 * one call, and each remaining call by its own launch.  Results are those
 * of the individual calls, bit for bit, except that a request whose fused
 * calls span three or more of the families {GAE, GAE + returns, TD(lambda)
 * returns, discounted returns}, {V-Trace}, {Retrace}, {eligibility traces,
 * fp32 prefix sum}, {int32 prefix sum}, with rows that all fit 512
 * elements, runs 4 elements per thread (smaller code per family), which
 * re-associates the fp32 scans: those results agree with the individual
 * calls to fp32 rounding (int32 stays exact).
 *
 * kind and argument slots (the pointer arguments of the entry point, in its
 * order; unused slots NULL):
 *   RLSCAN_KIND_GAE                 in: rewards values terminateds truncateds bootstrap_values last_values
 *                                   out: advantages
 *   RLSCAN_KIND_GAE_WITH_RETURNS    in: as GAE; out: advantages returns
 *   RLSCAN_KIND_VTRACE              in: log_rhos rewards values terminateds truncateds bootstrap_values
 *                                       last_values; out: vs pg_advantages
 *   RLSCAN_KIND_RETRACE             in: rewards q_values next_q_values_all next_target_probs log_rhos
 *                                       terminateds truncateds; out: q_ret
 *   RLSCAN_KIND_LAMBDA_RETURNS      in: as GAE; out: returns
 *   RLSCAN_KIND_DISCOUNTED_RETURNS  in: rewards terminateds truncateds bootstrap_values last_values;
 *                                   out: returns
 *   RLSCAN_KIND_ELIGIBILITY_TRACES  in: x dones; out: traces
 *   RLSCAN_KIND_EPISODIC_PREFIX_SUM in: x dones; out: out  (dtype RLSCAN_F32 or RLSCAN_I32)
 *   RLSCAN_KIND_GAE_TYPED           in: as GAE; out: advantages returns (returns nullable);
 *                                   dtype = value_dtype, flag_dtype = flag_dtype of
 *                                   rlscan_gae_typed
 *   RLSCAN_KIND_GAE_VTRACE          in: as VTRACE; out: advantages returns vs pg_advantages
 *                                   (returns nullable); lambda_ = GAE's, vtrace_lambda = V-Trace's
 * Scalars a kind does not take are ignored (lambda_ for discounted returns,
 * vtrace_lambda outside GAE_VTRACE, rho_bar and c_bar outside V-Trace and
 * Retrace, A outside Retrace, dtype outside the prefix sum and typed GAE,
 * flag_dtype outside typed GAE).
 * options: as for the _ex entry points.
 *
 * The calls run concurrently: no call's output may overlap any other
 * call's inputs or outputs (RLSCAN_ERR_INVALID_ARG).  ws / ws_bytes: one
 * workspace, at least the largest rlscan_workspace_bytes of the calls that
 * need one (they run one after another on `stream`).  ncalls == 0 is a no-op.
 * Errors: a nonzero return names the first failing call in
 * rlscan_last_error(); nothing was enqueued unless it is RLSCAN_ERR_CUDA
 * from a launch.
 */
typedef enum rlscan_kind {
    RLSCAN_KIND_GAE = 1,
    RLSCAN_KIND_GAE_WITH_RETURNS = 2,
    RLSCAN_KIND_VTRACE = 3,
    RLSCAN_KIND_RETRACE = 4,
    RLSCAN_KIND_LAMBDA_RETURNS = 5,
    RLSCAN_KIND_DISCOUNTED_RETURNS = 6,
    RLSCAN_KIND_ELIGIBILITY_TRACES = 7,
    RLSCAN_KIND_EPISODIC_PREFIX_SUM = 8,
    RLSCAN_KIND_GAE_TYPED = 9,
    RLSCAN_KIND_GAE_VTRACE = 10
} rlscan_kind;

#define RLSCAN_CALL_MAX_IN 8
#define RLSCAN_CALL_MAX_OUT 4
/* Largest number of calls in one rlscan_batch request. */
#define RLSCAN_BATCH_MAX 16

typedef struct rlscan_call {
    int kind;       /* rlscan_kind */
    int dtype;      /* prefix sum: RLSCAN_F32 or RLSCAN_I32; typed GAE: the value dtype */
    int flag_dtype; /* typed GAE: the flag dtype */
    unsigned options;
    int64_t E, T, A;
    float gamma, lambda_, rho_bar, c_bar;
    const void *in[RLSCAN_CALL_MAX_IN];
    void *out[RLSCAN_CALL_MAX_OUT];
    float vtrace_lambda; /* RLSCAN_KIND_GAE_VTRACE: V-Trace's lambda (lambda_ is GAE's) */
} rlscan_call;

RLSCAN_API int rlscan_batch(const rlscan_call *calls, int ncalls, void *ws, size_t ws_bytes, cudaStream_t stream);

/*
 * Workspace size in bytes that any entry point above needs for an [E, T]
 * problem (any A): 16 bytes per 1024 elements when rows span tiles, 0 when no call of
 * that shape needs one.  Negative or overflowing shapes return 0 and the
 * compute call then rejects them.
 */
RLSCAN_API size_t rlscan_workspace_bytes(int64_t E, int64_t T);

/* Zero-fill a workspace on `stream` (cudaMemsetAsync).  Not required: calls
 * accept a workspace of any content. */
RLSCAN_API int rlscan_workspace_init(void *ws, size_t ws_bytes, cudaStream_t stream);

/*
 * Synchronise `stream` and report any error of the work on it or of the
 * last launch: RLSCAN_OK, or RLSCAN_ERR_CUDA with the CUDA message.  For
 * debugging and tests; compute calls never synchronise.
 */
RLSCAN_API int rlscan_check(cudaStream_t stream);

/* Message for the last failing call on this thread ("" if none). */
RLSCAN_API const char *rlscan_last_error(void);

/* RLSCAN_VERSION of the built library. */
RLSCAN_API int rlscan_version(void);

/*
 * Launch plan that a call of this shape takes (for tests and tools):
 * writes tile size in elements, threads per block, whether tiles exchange
 * carries through the workspace (1) or not (0), and the tile count.  For
 * rows that span tiles (1) the call runs the chunked two passes: it writes
 * the workspace's granularity (1024 elements a slot), the passes' block size
 * and the workspace's slot count, an upper bound on the chunks.
 * actions: 1 for every estimator except rlscan_retrace with A > 1, whose
 * action count it is (1 .. RLSCAN_MAX_ACTIONS); every call scans on the same
 * plans, multi-action Retrace after a first launch that writes its expected
 * next-state values.
 */
RLSCAN_API int rlscan_plan(int64_t E, int64_t T, int64_t actions, int64_t *tile_elems, int *threads,
                int *lookback, int64_t *num_tiles);

#ifdef __cplusplus
}
#endif

#endif /* RLSCAN_H */
