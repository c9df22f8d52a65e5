// returns.cu - librlscan entry points for TD(lambda) returns and
// discounted returns.
#include "host.cuh"

using namespace rlscan;

extern "C" {

int rlscan_lambda_returns_ex(const float *rewards, const float *values, const float *terminateds,
                          const float *truncateds, const float *bootstrap_values, const float *last_values,
                          float *returns, int64_t E, int64_t T, float gamma, float lambda_, unsigned options, void *ws, size_t ws_bytes, cudaStream_t stream) {
    RLSCAN_TRY(check_options(options, false));
    RLSCAN_TRY(check_shape(E, T));
    RLSCAN_TRY(check_scalar(gamma, "gamma"));
    RLSCAN_TRY(check_scalar(lambda_, "lambda_"));
    if (E == 0 || T == 0) return ok();
    RLSCAN_TRY(require(rewards, "rewards"));
    RLSCAN_TRY(require(values, "values"));
    RLSCAN_TRY(require(returns, "returns"));
    if (truncateds && !bootstrap_values) return fail(RLSCAN_ERR_INVALID_ARG, "truncateds given without bootstrap_values");
    const size_t pb = plane_bytes(E, T);
    const Span ins[] = {{rewards, pb, "rewards"}, {values, pb, "values"}, {terminateds, pb, "terminateds"},
                        {truncateds, pb, "truncateds"}, {bootstrap_values, pb, "bootstrap_values"},
                        {last_values, (size_t)E * 4, "last_values"}};
    const Span outs[] = {{returns, pb, "returns"}};
    RLSCAN_TRY(check_aliasing(ins, 6, outs, 1));
    LambdaReturnsEst::Params P{rewards, values, terminateds, truncateds, truncateds ? bootstrap_values : nullptr,
                               last_values, returns, gamma, lambda_};
    if (options & RLSCAN_OPT_TIME_MAJOR)
        return run_time_major<LambdaReturnsEst>("rlscan_lambda_returns", P, E, T, stream, ws, ws_bytes);
    return run<LambdaReturnsEst>("rlscan_lambda_returns", P, E, T, ws, ws_bytes, stream,
                                 aligned16({rewards, values, terminateds, truncateds, bootstrap_values, returns}));
}

int rlscan_lambda_returns(const float *rewards, const float *values, const float *terminateds,
                          const float *truncateds, const float *bootstrap_values, const float *last_values,
                          float *returns, int64_t E, int64_t T, float gamma, float lambda_, void *ws,
                          size_t ws_bytes, cudaStream_t stream) {
    return rlscan_lambda_returns_ex(rewards, values, terminateds, truncateds, bootstrap_values, last_values, returns, E, T, gamma, lambda_, 0u, ws, ws_bytes, stream);
}

int rlscan_discounted_returns_ex(const float *rewards, const float *terminateds, const float *truncateds,
                              const float *bootstrap_values, const float *last_values, float *returns, int64_t E,
                              int64_t T, float gamma, unsigned options, void *ws, size_t ws_bytes, cudaStream_t stream) {
    RLSCAN_TRY(check_options(options, false));
    RLSCAN_TRY(check_shape(E, T));
    RLSCAN_TRY(check_scalar(gamma, "gamma"));
    if (E == 0 || T == 0) return ok();
    RLSCAN_TRY(require(rewards, "rewards"));
    RLSCAN_TRY(require(returns, "returns"));
    if (truncateds && !bootstrap_values) return fail(RLSCAN_ERR_INVALID_ARG, "truncateds given without bootstrap_values");
    const size_t pb = plane_bytes(E, T);
    const Span ins[] = {{rewards, pb, "rewards"}, {terminateds, pb, "terminateds"}, {truncateds, pb, "truncateds"},
                        {bootstrap_values, pb, "bootstrap_values"}, {last_values, (size_t)E * 4, "last_values"}};
    const Span outs[] = {{returns, pb, "returns"}};
    RLSCAN_TRY(check_aliasing(ins, 5, outs, 1));
    ReturnsEst::Params P{rewards, terminateds, truncateds, truncateds ? bootstrap_values : nullptr, last_values,
                         returns, gamma};
    if (options & RLSCAN_OPT_TIME_MAJOR)
        return run_time_major<ReturnsEst>("rlscan_discounted_returns", P, E, T, stream, ws, ws_bytes);
    return run<ReturnsEst>("rlscan_discounted_returns", P, E, T, ws, ws_bytes, stream,
                           aligned16({rewards, terminateds, truncateds, bootstrap_values, returns}));
}

int rlscan_discounted_returns(const float *rewards, const float *terminateds, const float *truncateds,
                              const float *bootstrap_values, const float *last_values, float *returns, int64_t E,
                              int64_t T, float gamma, void *ws, size_t ws_bytes, cudaStream_t stream) {
    return rlscan_discounted_returns_ex(rewards, terminateds, truncateds, bootstrap_values, last_values, returns, E, T, gamma, 0u, ws, ws_bytes, stream);
}

} // extern "C"
