// rlscan.cu - librlscan entry points for Retrace(lambda) and the library's
// service calls (workspace size and initialisation, the error check, the
// last error message, version, launch plan).
//
// Every compute entry point of the library (this file, gae.cu, vtrace.cu,
// returns.cu, forward.cu, batch.cu) validates its arguments on the host
// (nothing touches the GPU before the launch), picks a tile plan for the
// [E, T] shape (or the env-group plan of the time-major layout), and
// launches on the caller's stream with programmatic dependent launch
// allowed, so a kernel's prologue can overlap the tail of whatever ran
// before it on that stream.  No kernel waits on another block: rows that
// span tiles take two launches (aggregates, then the scan with carries).
#include "expect.cuh"


using namespace rlscan;

extern "C" {

int rlscan_retrace_ex(const float *rewards, const float *q_values, const float *next_q_values_all,
                   const float *next_target_probs, const float *log_rhos, const float *terminateds,
                   const float *truncateds, float *q_ret, int64_t E, int64_t T, int64_t A, float gamma,
                   float lambda_, float c_bar, unsigned options, void *ws, size_t ws_bytes, cudaStream_t stream) {
    RLSCAN_TRY(check_options(options, false));
    if (A < 1) return fail(RLSCAN_ERR_INVALID_ARG, "A must be >= 1 (got %lld)", (long long)A);
    if (A > RLSCAN_MAX_ACTIONS)
        return fail(RLSCAN_ERR_UNSUPPORTED, "A=%lld exceeds RLSCAN_MAX_ACTIONS=%d", (long long)A, RLSCAN_MAX_ACTIONS);
    RLSCAN_TRY(check_shape(E, T, A));
    RLSCAN_TRY(check_scalar(gamma, "gamma"));
    RLSCAN_TRY(check_scalar(lambda_, "lambda_"));
    RLSCAN_TRY(check_scalar(c_bar, "c_bar"));
    if (E == 0 || T == 0) return ok();
    RLSCAN_TRY(require(rewards, "rewards"));
    RLSCAN_TRY(require(q_values, "q_values"));
    RLSCAN_TRY(require(next_q_values_all, "next_q_values_all"));
    RLSCAN_TRY(require(log_rhos, "log_rhos"));
    RLSCAN_TRY(require(terminateds, "terminateds"));
    RLSCAN_TRY(require(truncateds, "truncateds"));
    RLSCAN_TRY(require(q_ret, "q_ret"));
    if (A > 1 && next_target_probs == nullptr)
        return fail(RLSCAN_ERR_INVALID_ARG, "next_target_probs is required when A > 1");
    const size_t pb = plane_bytes(E, T);
    const Span ins[] = {{rewards, pb, "rewards"}, {q_values, pb, "q_values"},
                        {next_q_values_all, pb * (size_t)A, "next_q_values_all"},
                        {A > 1 ? next_target_probs : nullptr, pb * (size_t)A, "next_target_probs"},
                        {log_rhos, pb, "log_rhos"}, {terminateds, pb, "terminateds"}, {truncateds, pb, "truncateds"}};
    const Span outs[] = {{q_ret, pb, "q_ret"}};
    RLSCAN_TRY(check_aliasing(ins, 7, outs, 1));
    if (A == 1) {
        RetraceEst::Params P{rewards, q_values, next_q_values_all, log_rhos, terminateds, truncateds, q_ret, gamma,
                             lambda_, c_bar};
        if (options & RLSCAN_OPT_TIME_MAJOR) return run_time_major<RetraceEst>("rlscan_retrace", P, E, T, stream, ws, ws_bytes);
        return run<RetraceEst>("rlscan_retrace", P, E, T, ws, ws_bytes, stream,
                               aligned16({rewards, q_values, next_q_values_all, log_rhos, terminateds, truncateds,
                                          q_ret}));
    }
    if (options & RLSCAN_OPT_TIME_MAJOR)
        return fail(RLSCAN_ERR_UNSUPPORTED, "rlscan_retrace: the time-major layout takes A == 1 only");
    // Several actions: first the expected next-state values V'_t of every
    // element into q_ret (expected_value_kernel), then the single-action
    // recurrence reading V' from q_ret and writing q_ret in place (each
    // thread reads its elements of that plane before it writes them).
    RetraceEst::Params P{rewards, q_values, q_ret, log_rhos, terminateds, truncateds, q_ret, gamma, lambda_, c_bar};
    const bool vec = aligned16({rewards, q_values, log_rhos, terminateds, truncateds, q_ret});
    if (!batch_dry()) {
        // checks of the scan's own (workspace) come first: nothing is enqueued
        // if the call is rejected
        const Plan plan = make_plan(E, T);
        if (plan.lookback && (ws == nullptr || ws_bytes < workspace_for(plan, E * T) || ((uintptr_t)ws & 15u) != 0))
            return run<RetraceEst>("rlscan_retrace", P, E, T, ws, ws_bytes, stream, vec);
        const cudaError_t e = launch_expected_values(next_q_values_all, next_target_probs, q_ret, E * T, A, stream);
        if (e != cudaSuccess)
            return fail(RLSCAN_ERR_CUDA, "rlscan_retrace: expected-value launch failed: %s", cudaGetErrorString(e));
    }
    return run<RetraceEst>("rlscan_retrace", P, E, T, ws, ws_bytes, stream, vec);
}

int rlscan_retrace(const float *rewards, const float *q_values, const float *next_q_values_all,
                   const float *next_target_probs, const float *log_rhos, const float *terminateds,
                   const float *truncateds, float *q_ret, int64_t E, int64_t T, int64_t A, float gamma,
                   float lambda_, float c_bar, void *ws, size_t ws_bytes, cudaStream_t stream) {
    return rlscan_retrace_ex(rewards, q_values, next_q_values_all, next_target_probs, log_rhos, terminateds, truncateds, q_ret, E, T, A, gamma, lambda_, c_bar, 0u, ws, ws_bytes, stream);
}

size_t rlscan_workspace_bytes(int64_t E, int64_t T) {
    if (E <= 0 || T <= 0 || E > kMaxElems / T) return 0;
    return std::max(workspace_for(make_plan(E, T), E * T), tm_workspace_for(E, T));
}

int rlscan_workspace_init(void *ws, size_t ws_bytes, cudaStream_t stream) {
    if (ws_bytes == 0) return ok();
    if (ws == nullptr) return fail(RLSCAN_ERR_INVALID_ARG, "ws must not be NULL");
    cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, stream);
    if (e != cudaSuccess) return fail(RLSCAN_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
    return ok();
}

int rlscan_check(cudaStream_t stream) {
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return fail(RLSCAN_ERR_CUDA, "stream error: %s", cudaGetErrorString(e));
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(RLSCAN_ERR_CUDA, "launch error: %s", cudaGetErrorString(e));
    return ok();
}

const char *rlscan_last_error(void) { return g_last_error.c_str(); }

int rlscan_version(void) { return RLSCAN_VERSION; }

int rlscan_plan(int64_t E, int64_t T, int64_t actions, int64_t *tile_elems, int *threads, int *lookback,
                int64_t *num_tiles) {
    if (E <= 0 || T <= 0) return fail(RLSCAN_ERR_INVALID_ARG, "E and T must be > 0");
    if (actions < 1 || actions > RLSCAN_MAX_ACTIONS) return fail(RLSCAN_ERR_INVALID_ARG, "bad action count");
    RLSCAN_TRY(check_shape(E, T, actions));
    const Plan p = make_plan(E, T); // every call scans on the single-action plan
    // rows that span tiles run the chunked two passes: report the workspace's
    // granularity (one slot per 1024 elements) and its slot count, an upper
    // bound on the chunks (their number depends on the device)
    const long long slot_elems = 2LL * 32 * kChunkV;
    if (tile_elems) *tile_elems = p.lookback ? slot_elems : kCfgTile[p.cfg];
    if (threads) *threads = p.lookback ? kChunkNT : kCfgThreads[p.cfg];
    if (lookback) *lookback = p.lookback ? 1 : 0;
    if (num_tiles) *num_tiles = p.lookback ? ceil_div(E * T, slot_elems) : p.ntiles;
    return ok();
}

} // extern "C"
