// typed_forward.cu - eligibility traces and the episodic prefix sum on
// reduced-byte inputs (bf16 / fp16 x, one-byte dones; the int32 prefix sum
// with one-byte dones), reached through rlscan_batch.
#include "typed.cuh"

namespace rlscan {

namespace {
int check_forward(const rlscan_call &c, const char *name, const char *out_name) {
    RLSCAN_TRY(check_flag_dtype(c.flag_dtype, name));
    RLSCAN_TRY(check_options(c.options, true));
    RLSCAN_TRY(check_shape(c.E, c.T));
    if (c.E == 0 || c.T == 0) return RLSCAN_OK;
    RLSCAN_TRY(require(c.in[0], "x"));
    RLSCAN_TRY(require(c.out[0], out_name));
    const size_t n = (size_t)(c.E * c.T);
    const size_t xb = n * (c.dtype == RLSCAN_I32 ? 4 : value_bytes(c.dtype));
    const Span ins[] = {{c.in[0], xb, "x"}, {c.in[1], n * flag_bytes(c.flag_dtype), "dones"}};
    const Span outs[] = {{c.out[0], n * 4, out_name}};
    return check_aliasing(ins, 2, outs, 1);
}

template <class Est>
int run_forward(const char *name, const typename Est::Params &P, const rlscan_call &c, void *ws, size_t ws_bytes,
                cudaStream_t stream) {
    if (c.options & RLSCAN_OPT_TIME_MAJOR) return run_time_major<Est>(name, P, c.E, c.T, stream, ws, ws_bytes);
    return run<Est>(name, P, c.E, c.T, ws, ws_bytes, stream, aligned16({c.in[0], c.in[1], c.out[0]}));
}
} // namespace

int typed_eligibility_traces(const rlscan_call &c, void *ws, size_t ws_bytes, cudaStream_t stream) {
    const char *name = "rlscan_eligibility_traces";
    RLSCAN_TRY(check_value_dtype(c.dtype, name));
    RLSCAN_TRY(check_scalar(c.gamma, "gamma"));
    RLSCAN_TRY(check_scalar(c.lambda_, "lambda_"));
    RLSCAN_TRY(check_forward(c, name, "traces"));
    if (c.E == 0 || c.T == 0) return ok();
    const int reset = (c.options & RLSCAN_OPT_DONE_STARTS_EPISODE) ? 1 : 0;
    return with_types(c.dtype, c.flag_dtype, [&](auto vt, auto ft) {
        using VT = typename decltype(vt)::type;
        using FT = typename decltype(ft)::type;
        using Est = ForwardEstT<VT, FT>;
        typename Est::Params P{static_cast<const VT *>(c.in[0]), static_cast<const FT *>(c.in[1]),
                               static_cast<float *>(c.out[0]), c.gamma * c.lambda_, reset};
        return run_forward<Est>(name, P, c, ws, ws_bytes, stream);
    });
}

int typed_episodic_prefix_sum(const rlscan_call &c, void *ws, size_t ws_bytes, cudaStream_t stream) {
    const char *name = "rlscan_episodic_prefix_sum";
    if (c.dtype != RLSCAN_I32) RLSCAN_TRY(check_value_dtype(c.dtype, name));
    RLSCAN_TRY(check_forward(c, name, "out"));
    if (c.E == 0 || c.T == 0) return ok();
    const int reset = (c.options & RLSCAN_OPT_DONE_STARTS_EPISODE) ? 1 : 0;
    if (c.dtype == RLSCAN_I32) { // exact int32 sums; only the dones are narrow
        using Est = PrefixI32EstT<uint8_t>;
        typename Est::Params P{static_cast<const int32_t *>(c.in[0]), static_cast<const uint8_t *>(c.in[1]),
                               static_cast<int32_t *>(c.out[0]), reset};
        return run_forward<Est>(name, P, c, ws, ws_bytes, stream);
    }
    return with_types(c.dtype, c.flag_dtype, [&](auto vt, auto ft) {
        using VT = typename decltype(vt)::type;
        using FT = typename decltype(ft)::type;
        using Est = ForwardEstT<VT, FT>;
        typename Est::Params P{static_cast<const VT *>(c.in[0]), static_cast<const FT *>(c.in[1]),
                               static_cast<float *>(c.out[0]), 1.0f, reset};
        return run_forward<Est>(name, P, c, ws, ws_bytes, stream);
    });
}

} // namespace rlscan
