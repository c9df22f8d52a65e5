// typed_returns.cu - TD(lambda) returns and discounted returns on
// reduced-byte inputs (bf16 / fp16 values, one-byte flags), reached through
// rlscan_batch.
#include "typed.cuh"

namespace rlscan {

int typed_lambda_returns(const rlscan_call &c, void *ws, size_t ws_bytes, cudaStream_t stream) {
    const char *name = "rlscan_lambda_returns";
    RLSCAN_TRY(check_value_dtype(c.dtype, name));
    RLSCAN_TRY(check_flag_dtype(c.flag_dtype, name));
    RLSCAN_TRY(check_options(c.options, false));
    RLSCAN_TRY(check_shape(c.E, c.T));
    RLSCAN_TRY(check_scalar(c.gamma, "gamma"));
    RLSCAN_TRY(check_scalar(c.lambda_, "lambda_"));
    if (c.E == 0 || c.T == 0) return ok();
    const void *const *in = c.in;
    RLSCAN_TRY(require(in[0], "rewards"));
    RLSCAN_TRY(require(in[1], "values"));
    RLSCAN_TRY(require(c.out[0], "returns"));
    if (in[3] && !in[4]) return fail(RLSCAN_ERR_INVALID_ARG, "truncateds given without bootstrap_values");
    const size_t n = (size_t)(c.E * c.T), vb = n * value_bytes(c.dtype), fb = n * flag_bytes(c.flag_dtype);
    const Span ins[] = {{in[0], vb, "rewards"},    {in[1], vb, "values"},           {in[2], fb, "terminateds"},
                        {in[3], fb, "truncateds"}, {in[4], vb, "bootstrap_values"}, {in[5], (size_t)c.E * 4, "last_values"}};
    const Span outs[] = {{c.out[0], n * 4, "returns"}};
    RLSCAN_TRY(check_aliasing(ins, 6, outs, 1));
    const bool vec = aligned16({in[0], in[1], in[2], in[3], in[4], c.out[0]});
    return with_types(c.dtype, c.flag_dtype, [&](auto vt, auto ft) {
        using VT = typename decltype(vt)::type;
        using FT = typename decltype(ft)::type;
        using Est = LambdaReturnsEstT<VT, FT>;
        typename Est::Params P{static_cast<const VT *>(in[0]), static_cast<const VT *>(in[1]),
                               static_cast<const FT *>(in[2]), static_cast<const FT *>(in[3]),
                               in[3] ? static_cast<const VT *>(in[4]) : nullptr,
                               static_cast<const float *>(in[5]), static_cast<float *>(c.out[0]), c.gamma,
                               c.lambda_};
        if (c.options & RLSCAN_OPT_TIME_MAJOR) return run_time_major<Est>(name, P, c.E, c.T, stream, ws, ws_bytes);
        return run<Est>(name, P, c.E, c.T, ws, ws_bytes, stream, vec);
    });
}

int typed_discounted_returns(const rlscan_call &c, void *ws, size_t ws_bytes, cudaStream_t stream) {
    const char *name = "rlscan_discounted_returns";
    RLSCAN_TRY(check_value_dtype(c.dtype, name));
    RLSCAN_TRY(check_flag_dtype(c.flag_dtype, name));
    RLSCAN_TRY(check_options(c.options, false));
    RLSCAN_TRY(check_shape(c.E, c.T));
    RLSCAN_TRY(check_scalar(c.gamma, "gamma"));
    if (c.E == 0 || c.T == 0) return ok();
    const void *const *in = c.in;
    RLSCAN_TRY(require(in[0], "rewards"));
    RLSCAN_TRY(require(c.out[0], "returns"));
    if (in[2] && !in[3]) return fail(RLSCAN_ERR_INVALID_ARG, "truncateds given without bootstrap_values");
    const size_t n = (size_t)(c.E * c.T), vb = n * value_bytes(c.dtype), fb = n * flag_bytes(c.flag_dtype);
    const Span ins[] = {{in[0], vb, "rewards"}, {in[1], fb, "terminateds"}, {in[2], fb, "truncateds"},
                        {in[3], vb, "bootstrap_values"}, {in[4], (size_t)c.E * 4, "last_values"}};
    const Span outs[] = {{c.out[0], n * 4, "returns"}};
    RLSCAN_TRY(check_aliasing(ins, 5, outs, 1));
    const bool vec = aligned16({in[0], in[1], in[2], in[3], c.out[0]});
    return with_types(c.dtype, c.flag_dtype, [&](auto vt, auto ft) {
        using VT = typename decltype(vt)::type;
        using FT = typename decltype(ft)::type;
        using Est = ReturnsEstT<VT, FT>;
        typename Est::Params P{static_cast<const VT *>(in[0]), static_cast<const FT *>(in[1]),
                               static_cast<const FT *>(in[2]), in[2] ? static_cast<const VT *>(in[3]) : nullptr,
                               static_cast<const float *>(in[4]), static_cast<float *>(c.out[0]), c.gamma};
        if (c.options & RLSCAN_OPT_TIME_MAJOR) return run_time_major<Est>(name, P, c.E, c.T, stream, ws, ws_bytes);
        return run<Est>(name, P, c.E, c.T, ws, ws_bytes, stream, vec);
    });
}

} // namespace rlscan
