// forward.cu - librlscan entry points for the forward recurrences:
// eligibility traces and the episodic prefix sum (fp32 and int32).
#include "host.cuh"

using namespace rlscan;

extern "C" {

int rlscan_eligibility_traces_ex(const float *x, const float *dones, float *traces, int64_t E, int64_t T, float gamma,
                              float lambda_, unsigned options, void *ws, size_t ws_bytes, cudaStream_t stream) {
    RLSCAN_TRY(check_options(options, true));
    RLSCAN_TRY(check_shape(E, T));
    RLSCAN_TRY(check_scalar(gamma, "gamma"));
    RLSCAN_TRY(check_scalar(lambda_, "lambda_"));
    if (E == 0 || T == 0) return ok();
    RLSCAN_TRY(require(x, "x"));
    RLSCAN_TRY(require(traces, "traces"));
    const size_t pb = plane_bytes(E, T);
    const Span ins[] = {{x, pb, "x"}, {dones, pb, "dones"}};
    const Span outs[] = {{traces, pb, "traces"}};
    RLSCAN_TRY(check_aliasing(ins, 2, outs, 1));
    TracesEst::Params P{x, dones, traces, gamma * lambda_, (options & RLSCAN_OPT_DONE_STARTS_EPISODE) ? 1 : 0};
    if (options & RLSCAN_OPT_TIME_MAJOR)
        return run_time_major<TracesEst>("rlscan_eligibility_traces", P, E, T, stream, ws, ws_bytes);
    return run<TracesEst>("rlscan_eligibility_traces", P, E, T, ws, ws_bytes, stream,
                          aligned16({x, dones, traces}));
}

int rlscan_eligibility_traces(const float *x, const float *dones, float *traces, int64_t E, int64_t T, float gamma,
                              float lambda_, void *ws, size_t ws_bytes, cudaStream_t stream) {
    return rlscan_eligibility_traces_ex(x, dones, traces, E, T, gamma, lambda_, 0u, ws, ws_bytes, stream);
}

int rlscan_episodic_prefix_sum_ex(const void *x, int dtype, const float *dones, void *out, int64_t E, int64_t T,
                               unsigned options, void *ws, size_t ws_bytes, cudaStream_t stream) {
    RLSCAN_TRY(check_options(options, true));
    if (dtype != RLSCAN_F32 && dtype != RLSCAN_I32) return fail(RLSCAN_ERR_UNSUPPORTED, "unknown dtype %d", dtype);
    RLSCAN_TRY(check_shape(E, T));
    if (E == 0 || T == 0) return ok();
    RLSCAN_TRY(require(x, "x"));
    RLSCAN_TRY(require(out, "out"));
    const size_t pb = plane_bytes(E, T);
    const Span ins[] = {{x, pb, "x"}, {dones, pb, "dones"}};
    const Span outs[] = {{out, pb, "out"}};
    RLSCAN_TRY(check_aliasing(ins, 2, outs, 1));
    if (dtype == RLSCAN_F32) {
        PrefixF32Est::Params P{static_cast<const float *>(x), dones, static_cast<float *>(out), 1.0f, (options & RLSCAN_OPT_DONE_STARTS_EPISODE) ? 1 : 0};
        if (options & RLSCAN_OPT_TIME_MAJOR)
            return run_time_major<PrefixF32Est>("rlscan_episodic_prefix_sum", P, E, T, stream, ws, ws_bytes);
        return run<PrefixF32Est>("rlscan_episodic_prefix_sum", P, E, T, ws, ws_bytes, stream,
                                 aligned16({x, dones, out}));
    }
    PrefixI32Est::Params P{static_cast<const int32_t *>(x), dones, static_cast<int32_t *>(out), (options & RLSCAN_OPT_DONE_STARTS_EPISODE) ? 1 : 0};
    if (options & RLSCAN_OPT_TIME_MAJOR)
        return run_time_major<PrefixI32Est>("rlscan_episodic_prefix_sum", P, E, T, stream, ws, ws_bytes);
    return run<PrefixI32Est>("rlscan_episodic_prefix_sum", P, E, T, ws, ws_bytes, stream,
                             aligned16({x, dones, out}));
}

int rlscan_episodic_prefix_sum(const void *x, int dtype, const float *dones, void *out, int64_t E, int64_t T,
                               void *ws, size_t ws_bytes, cudaStream_t stream) {
    return rlscan_episodic_prefix_sum_ex(x, dtype, dones, out, E, T, 0u, ws, ws_bytes, stream);
}

} // extern "C"
