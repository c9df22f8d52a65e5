// typed_retrace.cu - Retrace(lambda) on reduced-byte inputs (bf16 / fp16
// rewards, Q-values, per-action rows and log ratios; one-byte flags),
// reached through rlscan_batch.  With several actions the expected
// next-state values are written (fp32) into q_ret first, as for fp32 inputs.
#include "expect.cuh"
#include "typed.cuh"

namespace rlscan {

int typed_retrace(const rlscan_call &c, void *ws, size_t ws_bytes, cudaStream_t stream) {
    const char *name = "rlscan_retrace";
    RLSCAN_TRY(check_value_dtype(c.dtype, name));
    RLSCAN_TRY(check_flag_dtype(c.flag_dtype, name));
    RLSCAN_TRY(check_options(c.options, false));
    const long long A = c.A;
    if (A < 1) return fail(RLSCAN_ERR_INVALID_ARG, "A must be >= 1 (got %lld)", A);
    if (A > RLSCAN_MAX_ACTIONS)
        return fail(RLSCAN_ERR_UNSUPPORTED, "A=%lld exceeds RLSCAN_MAX_ACTIONS=%d", A, RLSCAN_MAX_ACTIONS);
    RLSCAN_TRY(check_shape(c.E, c.T, A));
    RLSCAN_TRY(check_scalar(c.gamma, "gamma"));
    RLSCAN_TRY(check_scalar(c.lambda_, "lambda_"));
    RLSCAN_TRY(check_scalar(c.c_bar, "c_bar"));
    if (c.E == 0 || c.T == 0) return ok();
    const void *const *in = c.in;
    const char *names[7] = {"rewards", "q_values", "next_q_values_all", "next_target_probs", "log_rhos",
                            "terminateds", "truncateds"};
    for (int i : {0, 1, 2, 4, 5, 6}) RLSCAN_TRY(require(in[i], names[i]));
    RLSCAN_TRY(require(c.out[0], "q_ret"));
    if (A > 1 && in[3] == nullptr) return fail(RLSCAN_ERR_INVALID_ARG, "next_target_probs is required when A > 1");
    if (A > 1 && (c.options & RLSCAN_OPT_TIME_MAJOR))
        return fail(RLSCAN_ERR_UNSUPPORTED, "rlscan_retrace: the time-major layout takes A == 1 only");
    const size_t n = (size_t)(c.E * c.T), vb = n * value_bytes(c.dtype), fb = n * flag_bytes(c.flag_dtype);
    const Span ins[] = {{in[0], vb, "rewards"},      {in[1], vb, "q_values"},
                        {in[2], vb * (size_t)A, "next_q_values_all"},
                        {A > 1 ? in[3] : nullptr, vb * (size_t)A, "next_target_probs"},
                        {in[4], vb, "log_rhos"},     {in[5], fb, "terminateds"}, {in[6], fb, "truncateds"}};
    const Span outs[] = {{c.out[0], n * 4, "q_ret"}};
    RLSCAN_TRY(check_aliasing(ins, 7, outs, 1));
    float *q_ret = static_cast<float *>(c.out[0]);
    return with_types(c.dtype, c.flag_dtype, [&](auto vt, auto ft) {
        using VT = typename decltype(vt)::type;
        using FT = typename decltype(ft)::type;
        if (A == 1) {
            using Est = RetraceEstT<VT, FT, VT>;
            typename Est::Params P{static_cast<const VT *>(in[0]), static_cast<const VT *>(in[1]),
                                   static_cast<const VT *>(in[2]), static_cast<const VT *>(in[4]),
                                   static_cast<const FT *>(in[5]), static_cast<const FT *>(in[6]), q_ret, c.gamma,
                                   c.lambda_, c.c_bar};
            if (c.options & RLSCAN_OPT_TIME_MAJOR) return run_time_major<Est>(name, P, c.E, c.T, stream, ws, ws_bytes);
            return run<Est>(name, P, c.E, c.T, ws, ws_bytes, stream,
                            aligned16({in[0], in[1], in[2], in[4], in[5], in[6], q_ret}));
        }
        // expected next-state values into q_ret, then the recurrence on them in place
        using Est = RetraceEstT<VT, FT, float>;
        typename Est::Params P{static_cast<const VT *>(in[0]), static_cast<const VT *>(in[1]), q_ret,
                               static_cast<const VT *>(in[4]), static_cast<const FT *>(in[5]),
                               static_cast<const FT *>(in[6]), q_ret, c.gamma, c.lambda_, c.c_bar};
        const bool vec = aligned16({in[0], in[1], in[4], in[5], in[6], q_ret});
        if (!batch_dry()) {
            const Plan plan = make_plan(c.E, c.T);
            if (plan.lookback && (ws == nullptr || ws_bytes < workspace_for(plan, c.E * c.T) || ((uintptr_t)ws & 15u) != 0))
                return run<Est>(name, P, c.E, c.T, ws, ws_bytes, stream, vec); // reports the workspace error
            const cudaError_t e = launch_expected_values(static_cast<const VT *>(in[2]),
                                                         static_cast<const VT *>(in[3]), q_ret, c.E * c.T, A, stream);
            if (e != cudaSuccess)
                return fail(RLSCAN_ERR_CUDA, "rlscan_retrace: expected-value launch failed: %s", cudaGetErrorString(e));
        }
        return run<Est>(name, P, c.E, c.T, ws, ws_bytes, stream, vec);
    });
}

} // namespace rlscan
