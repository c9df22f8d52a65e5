// vtrace.cu - librlscan entry points for V-Trace and for the one-pass GAE +
// TD(lambda) returns + V-Trace (the paired recurrence).
#include "host.cuh"

using namespace rlscan;

extern "C" {

int rlscan_vtrace_ex(const float *log_rhos, const float *rewards, const float *values, const float *terminateds,
                  const float *truncateds, const float *bootstrap_values, const float *last_values, float *vs,
                  float *pg_advantages, int64_t E, int64_t T, float gamma, float lambda_, float rho_bar,
                  float c_bar, unsigned options, void *ws, size_t ws_bytes, cudaStream_t stream) {
    RLSCAN_TRY(check_options(options, false));
    RLSCAN_TRY(check_shape(E, T));
    RLSCAN_TRY(check_scalar(gamma, "gamma"));
    RLSCAN_TRY(check_scalar(lambda_, "lambda_"));
    RLSCAN_TRY(check_scalar(rho_bar, "rho_bar"));
    RLSCAN_TRY(check_scalar(c_bar, "c_bar"));
    if (E == 0 || T == 0) return ok();
    RLSCAN_TRY(require(log_rhos, "log_rhos"));
    RLSCAN_TRY(require(rewards, "rewards"));
    RLSCAN_TRY(require(values, "values"));
    RLSCAN_TRY(require(vs, "vs"));
    RLSCAN_TRY(require(pg_advantages, "pg_advantages"));
    if (truncateds && !bootstrap_values) return fail(RLSCAN_ERR_INVALID_ARG, "truncateds given without bootstrap_values");
    const size_t pb = plane_bytes(E, T);
    const Span ins[] = {{log_rhos, pb, "log_rhos"}, {rewards, pb, "rewards"}, {values, pb, "values"},
                        {terminateds, pb, "terminateds"}, {truncateds, pb, "truncateds"},
                        {bootstrap_values, pb, "bootstrap_values"}, {last_values, (size_t)E * 4, "last_values"}};
    const Span outs[] = {{vs, pb, "vs"}, {pg_advantages, pb, "pg_advantages"}};
    RLSCAN_TRY(check_aliasing(ins, 7, outs, 2));
    VtraceEst::Params P{log_rhos, rewards, values, terminateds, truncateds, truncateds ? bootstrap_values : nullptr,
                        last_values, vs, pg_advantages, gamma, lambda_, rho_bar, c_bar};
    if (options & RLSCAN_OPT_TIME_MAJOR) return run_time_major<VtraceEst>("rlscan_vtrace", P, E, T, stream, ws, ws_bytes);
    return run<VtraceEst>("rlscan_vtrace", P, E, T, ws, ws_bytes, stream,
                          aligned16({log_rhos, rewards, values, terminateds, truncateds, bootstrap_values, vs, pg_advantages}));
}

int rlscan_vtrace(const float *log_rhos, const float *rewards, const float *values, const float *terminateds,
                  const float *truncateds, const float *bootstrap_values, const float *last_values, float *vs,
                  float *pg_advantages, int64_t E, int64_t T, float gamma, float lambda_, float rho_bar,
                  float c_bar, void *ws, size_t ws_bytes, cudaStream_t stream) {
    return rlscan_vtrace_ex(log_rhos, rewards, values, terminateds, truncateds, bootstrap_values, last_values, vs, pg_advantages, E, T, gamma, lambda_, rho_bar, c_bar, 0u, ws, ws_bytes, stream);
}

int rlscan_gae_vtrace_ex(const float *log_rhos, const float *rewards, const float *values, const float *terminateds,
                         const float *truncateds, const float *bootstrap_values, const float *last_values,
                         float *advantages, float *returns, float *vs, float *pg_advantages, int64_t E, int64_t T,
                         float gamma, float lambda_, float vtrace_lambda, float rho_bar, float c_bar,
                         unsigned options, void *ws, size_t ws_bytes, cudaStream_t stream) {
    RLSCAN_TRY(check_options(options, false));
    RLSCAN_TRY(check_shape(E, T));
    RLSCAN_TRY(check_scalar(gamma, "gamma"));
    RLSCAN_TRY(check_scalar(lambda_, "lambda_"));
    RLSCAN_TRY(check_scalar(vtrace_lambda, "vtrace_lambda"));
    RLSCAN_TRY(check_scalar(rho_bar, "rho_bar"));
    RLSCAN_TRY(check_scalar(c_bar, "c_bar"));
    if (E == 0 || T == 0) return ok();
    RLSCAN_TRY(require(log_rhos, "log_rhos"));
    RLSCAN_TRY(require(rewards, "rewards"));
    RLSCAN_TRY(require(values, "values"));
    RLSCAN_TRY(require(advantages, "advantages"));
    RLSCAN_TRY(require(vs, "vs"));
    RLSCAN_TRY(require(pg_advantages, "pg_advantages"));
    if (truncateds && !bootstrap_values) return fail(RLSCAN_ERR_INVALID_ARG, "truncateds given without bootstrap_values");
    const size_t pb = plane_bytes(E, T);
    const Span ins[] = {{log_rhos, pb, "log_rhos"}, {rewards, pb, "rewards"}, {values, pb, "values"},
                        {terminateds, pb, "terminateds"}, {truncateds, pb, "truncateds"},
                        {bootstrap_values, pb, "bootstrap_values"}, {last_values, (size_t)E * 4, "last_values"}};
    const Span outs[] = {{advantages, pb, "advantages"}, {returns, pb, "returns"}, {vs, pb, "vs"},
                         {pg_advantages, pb, "pg_advantages"}};
    RLSCAN_TRY(check_aliasing(ins, 7, outs, 4));
    GaeVtraceEst::Params P{log_rhos, rewards, values, terminateds, truncateds,
                           truncateds ? bootstrap_values : nullptr, last_values, advantages, returns, vs,
                           pg_advantages, gamma, lambda_, vtrace_lambda, rho_bar, c_bar};
    if (options & RLSCAN_OPT_TIME_MAJOR) return run_time_major<GaeVtraceEst>("rlscan_gae_vtrace", P, E, T, stream, ws, ws_bytes);
    return run<GaeVtraceEst>("rlscan_gae_vtrace", P, E, T, ws, ws_bytes, stream,
                             aligned16({log_rhos, rewards, values, terminateds, truncateds, bootstrap_values, advantages,
                                        returns, vs, pg_advantages}));
}

int rlscan_gae_vtrace(const float *log_rhos, const float *rewards, const float *values, const float *terminateds,
                      const float *truncateds, const float *bootstrap_values, const float *last_values,
                      float *advantages, float *returns, float *vs, float *pg_advantages, int64_t E, int64_t T,
                      float gamma, float lambda_, float vtrace_lambda, float rho_bar, float c_bar, void *ws,
                      size_t ws_bytes, cudaStream_t stream) {
    return rlscan_gae_vtrace_ex(log_rhos, rewards, values, terminateds, truncateds, bootstrap_values, last_values,
                                advantages, returns, vs, pg_advantages, E, T, gamma, lambda_, vtrace_lambda, rho_bar,
                                c_bar, 0u, ws, ws_bytes, stream);
}

} // extern "C"
