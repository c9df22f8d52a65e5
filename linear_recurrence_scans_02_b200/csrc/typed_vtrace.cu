// typed_vtrace.cu - V-Trace on reduced-byte inputs (bf16 / fp16 values,
// one-byte flags), reached through rlscan_batch.
#include "typed.cuh"

namespace rlscan {

int typed_vtrace(const rlscan_call &c, void *ws, size_t ws_bytes, cudaStream_t stream) {
    const char *name = "rlscan_vtrace";
    RLSCAN_TRY(check_value_dtype(c.dtype, name));
    RLSCAN_TRY(check_flag_dtype(c.flag_dtype, name));
    RLSCAN_TRY(check_options(c.options, false));
    RLSCAN_TRY(check_shape(c.E, c.T));
    RLSCAN_TRY(check_scalar(c.gamma, "gamma"));
    RLSCAN_TRY(check_scalar(c.lambda_, "lambda_"));
    RLSCAN_TRY(check_scalar(c.rho_bar, "rho_bar"));
    RLSCAN_TRY(check_scalar(c.c_bar, "c_bar"));
    if (c.E == 0 || c.T == 0) return ok();
    const void *const *in = c.in;
    RLSCAN_TRY(require(in[0], "log_rhos"));
    RLSCAN_TRY(require(in[1], "rewards"));
    RLSCAN_TRY(require(in[2], "values"));
    RLSCAN_TRY(require(c.out[0], "vs"));
    RLSCAN_TRY(require(c.out[1], "pg_advantages"));
    if (in[4] && !in[5]) return fail(RLSCAN_ERR_INVALID_ARG, "truncateds given without bootstrap_values");
    const size_t n = (size_t)(c.E * c.T), vb = n * value_bytes(c.dtype), fb = n * flag_bytes(c.flag_dtype);
    const Span ins[] = {{in[0], vb, "log_rhos"},    {in[1], vb, "rewards"},    {in[2], vb, "values"},
                        {in[3], fb, "terminateds"}, {in[4], fb, "truncateds"}, {in[5], vb, "bootstrap_values"},
                        {in[6], (size_t)c.E * 4, "last_values"}};
    const Span outs[] = {{c.out[0], n * 4, "vs"}, {c.out[1], n * 4, "pg_advantages"}};
    RLSCAN_TRY(check_aliasing(ins, 7, outs, 2));
    const bool vec = aligned16({in[0], in[1], in[2], in[3], in[4], in[5], c.out[0], c.out[1]});
    return with_types(c.dtype, c.flag_dtype, [&](auto vt, auto ft) {
        using VT = typename decltype(vt)::type;
        using FT = typename decltype(ft)::type;
        using Est = VtraceEstT<VT, FT>;
        typename Est::Params P{static_cast<const VT *>(in[0]), static_cast<const VT *>(in[1]),
                               static_cast<const VT *>(in[2]), static_cast<const FT *>(in[3]),
                               static_cast<const FT *>(in[4]),
                               in[4] ? static_cast<const VT *>(in[5]) : nullptr,
                               static_cast<const float *>(in[6]), static_cast<float *>(c.out[0]),
                               static_cast<float *>(c.out[1]), c.gamma, c.lambda_, c.rho_bar, c.c_bar};
        if (c.options & RLSCAN_OPT_TIME_MAJOR) return run_time_major<Est>(name, P, c.E, c.T, stream, ws, ws_bytes);
        return run<Est>(name, P, c.E, c.T, ws, ws_bytes, stream, vec);
    });
}

} // namespace rlscan
