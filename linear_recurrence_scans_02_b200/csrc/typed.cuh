// typed.cuh - reduced-byte inputs for every estimator.
//
// A call whose value planes (rewards, values, log importance ratios,
// Q-values, bootstrap values, traces' x) are bf16 or fp16, or whose flag
// planes (terminateds, truncateds, dones) are one byte per flag, reads them
// at that width and widens them in registers; all arithmetic and every
// output stay fp32 (the int32 prefix sum stays int32).  The path is
// memory-bound, so narrower inputs are fewer bytes per env-step.  These
// calls reach the library through rlscan_batch (rlscan_call's dtype and
// flag_dtype); the functions below are their checks and launches, one
// translation unit per estimator family, and batch.cu routes to them.
#pragma once

#include "host.cuh"

namespace rlscan {

template <class T>
struct TypeTag {
    using type = T;
};

inline size_t value_bytes(int dt) { return dt == RLSCAN_BF16 || dt == RLSCAN_F16 ? 2 : 4; }
inline size_t flag_bytes(int dt) { return dt == RLSCAN_U8 ? 1 : 4; }

inline int check_value_dtype(int dt, const char *name) {
    if (dt != RLSCAN_F32 && dt != RLSCAN_BF16 && dt != RLSCAN_F16)
        return fail(RLSCAN_ERR_UNSUPPORTED, "%s: value dtype %d not supported (F32, BF16, F16)", name, dt);
    return RLSCAN_OK;
}
inline int check_flag_dtype(int dt, const char *name) {
    if (dt != RLSCAN_F32 && dt != RLSCAN_U8)
        return fail(RLSCAN_ERR_UNSUPPORTED, "%s: flag dtype %d not supported (F32, U8)", name, dt);
    return RLSCAN_OK;
}

// f(TypeTag<ValT>, TypeTag<FlagT>) for the call's element types; never with
// both fp32 (those calls take the fp32 entry points).
template <class F>
int with_types(int vdt, int fdt, F &&f) {
    if (fdt == RLSCAN_U8) {
        if (vdt == RLSCAN_BF16) return f(TypeTag<__nv_bfloat16>{}, TypeTag<uint8_t>{});
        if (vdt == RLSCAN_F16) return f(TypeTag<__half>{}, TypeTag<uint8_t>{});
        return f(TypeTag<float>{}, TypeTag<uint8_t>{});
    }
    if (vdt == RLSCAN_BF16) return f(TypeTag<__nv_bfloat16>{}, TypeTag<float>{});
    return f(TypeTag<__half>{}, TypeTag<float>{});
}

// A call of one of these kinds is typed when any of its planes is narrower
// than fp32.
inline bool call_is_typed(const rlscan_call &c) {
    if (c.kind == RLSCAN_KIND_EPISODIC_PREFIX_SUM)
        return c.dtype == RLSCAN_BF16 || c.dtype == RLSCAN_F16 || c.flag_dtype != RLSCAN_F32;
    return c.dtype != RLSCAN_F32 || c.flag_dtype != RLSCAN_F32;
}

int typed_vtrace(const rlscan_call &c, void *ws, size_t ws_bytes, cudaStream_t stream);
int typed_lambda_returns(const rlscan_call &c, void *ws, size_t ws_bytes, cudaStream_t stream);
int typed_discounted_returns(const rlscan_call &c, void *ws, size_t ws_bytes, cudaStream_t stream);
int typed_retrace(const rlscan_call &c, void *ws, size_t ws_bytes, cudaStream_t stream);
int typed_eligibility_traces(const rlscan_call &c, void *ws, size_t ws_bytes, cudaStream_t stream);
int typed_episodic_prefix_sum(const rlscan_call &c, void *ws, size_t ws_bytes, cudaStream_t stream);

} // namespace rlscan
