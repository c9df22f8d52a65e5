// gae.cu - librlscan entry points for GAE: rlscan_gae, the one-pass GAE +
// TD(lambda) returns, reduced-byte GAE, and the GAE call that allocates
// nothing (rlscan_gae_noalloc, with its fixed device scratch).
#include <mutex>

#include "host.cuh"

// Fixed scratch of rlscan_gae_noalloc: the split-row workspace for callers
// that cannot allocate one.  In host code this name is only a handle for
// cudaGetSymbolAddress, never an address to pass to a kernel.
static __device__ __align__(256) unsigned char g_noalloc_scratch[RLSCAN_NOALLOC_SCRATCH_BYTES];

namespace rlscan {
namespace {

constexpr int kMaxDevices = 256;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {};

// Device address of this device's copy of the scratch array, looked up once
// per device with that device current.
int noalloc_scratch(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(RLSCAN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(RLSCAN_ERR_UNSUPPORTED, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr)
            return fail(RLSCAN_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return RLSCAN_OK;
}

} // namespace
} // namespace rlscan

using namespace rlscan;

extern "C" {

int rlscan_gae_ex(const float *rewards, const float *values, const float *terminateds, const float *truncateds,
               const float *bootstrap_values, const float *last_values, float *advantages, int64_t E, int64_t T,
               float gamma, float lambda_, unsigned options, void *ws, size_t ws_bytes, cudaStream_t stream) {
    RLSCAN_TRY(check_options(options, false));
    RLSCAN_TRY(check_shape(E, T));
    RLSCAN_TRY(check_scalar(gamma, "gamma"));
    RLSCAN_TRY(check_scalar(lambda_, "lambda_"));
    if (E == 0 || T == 0) return ok();
    RLSCAN_TRY(require(rewards, "rewards"));
    RLSCAN_TRY(require(values, "values"));
    RLSCAN_TRY(require(advantages, "advantages"));
    if (truncateds && !bootstrap_values) return fail(RLSCAN_ERR_INVALID_ARG, "truncateds given without bootstrap_values");
    const size_t pb = plane_bytes(E, T);
    const Span ins[] = {{rewards, pb, "rewards"}, {values, pb, "values"}, {terminateds, pb, "terminateds"},
                        {truncateds, pb, "truncateds"}, {bootstrap_values, pb, "bootstrap_values"},
                        {last_values, (size_t)E * 4, "last_values"}};
    const Span outs[] = {{advantages, pb, "advantages"}};
    RLSCAN_TRY(check_aliasing(ins, 6, outs, 1));
    GaeEst::Params P{rewards, values, terminateds, truncateds, truncateds ? bootstrap_values : nullptr,
                     last_values, advantages, nullptr, gamma, lambda_};
    if (options & RLSCAN_OPT_TIME_MAJOR) return run_time_major<GaeEst>("rlscan_gae", P, E, T, stream, ws, ws_bytes);
    return run<GaeEst>("rlscan_gae", P, E, T, ws, ws_bytes, stream,
                       aligned16({rewards, values, terminateds, truncateds, bootstrap_values, advantages}));
}

int rlscan_gae(const float *rewards, const float *values, const float *terminateds, const float *truncateds,
               const float *bootstrap_values, const float *last_values, float *advantages, int64_t E, int64_t T,
               float gamma, float lambda_, void *ws, size_t ws_bytes, cudaStream_t stream) {
    return rlscan_gae_ex(rewards, values, terminateds, truncateds, bootstrap_values, last_values, advantages, E, T, gamma, lambda_, 0u, ws, ws_bytes, stream);
}

int rlscan_gae_with_returns_ex(const float *rewards, const float *values, const float *terminateds,
                            const float *truncateds, const float *bootstrap_values, const float *last_values,
                            float *advantages, float *returns, int64_t E, int64_t T, float gamma, float lambda_,
                            unsigned options, void *ws, size_t ws_bytes, cudaStream_t stream) {
    RLSCAN_TRY(check_options(options, false));
    RLSCAN_TRY(check_shape(E, T));
    RLSCAN_TRY(check_scalar(gamma, "gamma"));
    RLSCAN_TRY(check_scalar(lambda_, "lambda_"));
    if (E == 0 || T == 0) return ok();
    RLSCAN_TRY(require(rewards, "rewards"));
    RLSCAN_TRY(require(values, "values"));
    RLSCAN_TRY(require(advantages, "advantages"));
    RLSCAN_TRY(require(returns, "returns"));
    if (truncateds && !bootstrap_values) return fail(RLSCAN_ERR_INVALID_ARG, "truncateds given without bootstrap_values");
    const size_t pb = plane_bytes(E, T);
    const Span ins[] = {{rewards, pb, "rewards"}, {values, pb, "values"}, {terminateds, pb, "terminateds"},
                        {truncateds, pb, "truncateds"}, {bootstrap_values, pb, "bootstrap_values"},
                        {last_values, (size_t)E * 4, "last_values"}};
    const Span outs[] = {{advantages, pb, "advantages"}, {returns, pb, "returns"}};
    RLSCAN_TRY(check_aliasing(ins, 6, outs, 2));
    GaeReturnsEst::Params P{rewards, values, terminateds, truncateds, truncateds ? bootstrap_values : nullptr,
                            last_values, advantages, returns, gamma, lambda_};
    if (options & RLSCAN_OPT_TIME_MAJOR)
        return run_time_major<GaeReturnsEst>("rlscan_gae_with_returns", P, E, T, stream, ws, ws_bytes);
    return run<GaeReturnsEst>("rlscan_gae_with_returns", P, E, T, ws, ws_bytes, stream,
                              aligned16({rewards, values, terminateds, truncateds, bootstrap_values, advantages, returns}));
}

int rlscan_gae_with_returns(const float *rewards, const float *values, const float *terminateds,
                            const float *truncateds, const float *bootstrap_values, const float *last_values,
                            float *advantages, float *returns, int64_t E, int64_t T, float gamma, float lambda_,
                            void *ws, size_t ws_bytes, cudaStream_t stream) {
    return rlscan_gae_with_returns_ex(rewards, values, terminateds, truncateds, bootstrap_values, last_values, advantages, returns, E, T, gamma, lambda_, 0u, ws, ws_bytes, stream);
}

int rlscan_gae_typed_ex(const void *rewards, const void *values, const void *terminateds, const void *truncateds,
                        const void *bootstrap_values, const float *last_values, float *advantages, float *returns,
                        int64_t E, int64_t T, float gamma, float lambda_, int value_dtype, int flag_dtype,
                        unsigned options, void *ws, size_t ws_bytes, cudaStream_t stream) {
    RLSCAN_TRY(check_options(options, false));
    size_t vsz, fsz;
    switch (value_dtype) {
    case RLSCAN_F32: vsz = 4; break;
    case RLSCAN_BF16:
    case RLSCAN_F16: vsz = 2; break;
    default: return fail(RLSCAN_ERR_UNSUPPORTED, "value_dtype %d not supported (F32, BF16, F16)", value_dtype);
    }
    switch (flag_dtype) {
    case RLSCAN_F32: fsz = 4; break;
    case RLSCAN_U8: fsz = 1; break;
    default: return fail(RLSCAN_ERR_UNSUPPORTED, "flag_dtype %d not supported (F32, U8)", flag_dtype);
    }
    RLSCAN_TRY(check_shape(E, T));
    RLSCAN_TRY(check_scalar(gamma, "gamma"));
    RLSCAN_TRY(check_scalar(lambda_, "lambda_"));
    if (E == 0 || T == 0) return ok();
    RLSCAN_TRY(require(rewards, "rewards"));
    RLSCAN_TRY(require(values, "values"));
    RLSCAN_TRY(require(advantages, "advantages"));
    if (truncateds && !bootstrap_values) return fail(RLSCAN_ERR_INVALID_ARG, "truncateds given without bootstrap_values");
    const size_t n = (size_t)(E * T);
    const Span ins[] = {{rewards, n * vsz, "rewards"}, {values, n * vsz, "values"},
                        {terminateds, n * fsz, "terminateds"}, {truncateds, n * fsz, "truncateds"},
                        {bootstrap_values, n * vsz, "bootstrap_values"}, {last_values, (size_t)E * 4, "last_values"}};
    const Span outs[] = {{advantages, n * 4, "advantages"}, {returns, n * 4, "returns"}};
    RLSCAN_TRY(check_aliasing(ins, 6, outs, 2));
    const bool vec = aligned16({rewards, values, terminateds, truncateds, bootstrap_values, advantages, returns});
    const void *bv = truncateds ? bootstrap_values : nullptr;
#define RLSCAN_GAE_TYPED(VT, FT)                                                                                  \
    do {                                                                                                          \
        typename GaeTypedEst<VT, FT>::Params P{static_cast<const VT *>(rewards), static_cast<const VT *>(values), \
                                               static_cast<const FT *>(terminateds),                               \
                                               static_cast<const FT *>(truncateds), static_cast<const VT *>(bv),  \
                                               last_values, advantages, returns, gamma, lambda_};                  \
        if (options & RLSCAN_OPT_TIME_MAJOR)                                                                      \
            return run_time_major<GaeTypedEst<VT, FT>>("rlscan_gae_typed", P, E, T, stream, ws, ws_bytes);                     \
        return run<GaeTypedEst<VT, FT>>("rlscan_gae_typed", P, E, T, ws, ws_bytes, stream, vec);              \
    } while (0)
    if (flag_dtype == RLSCAN_U8) {
        if (value_dtype == RLSCAN_BF16) RLSCAN_GAE_TYPED(__nv_bfloat16, uint8_t);
        if (value_dtype == RLSCAN_F16) RLSCAN_GAE_TYPED(__half, uint8_t);
        RLSCAN_GAE_TYPED(float, uint8_t);
    }
    if (value_dtype == RLSCAN_BF16) RLSCAN_GAE_TYPED(__nv_bfloat16, float);
    if (value_dtype == RLSCAN_F16) RLSCAN_GAE_TYPED(__half, float);
    RLSCAN_GAE_TYPED(float, float);
#undef RLSCAN_GAE_TYPED
}

int rlscan_gae_typed(const void *rewards, const void *values, const void *terminateds, const void *truncateds,
                     const void *bootstrap_values, const float *last_values, float *advantages, float *returns,
                     int64_t E, int64_t T, float gamma, float lambda_, int value_dtype, int flag_dtype, void *ws,
                     size_t ws_bytes, cudaStream_t stream) {
    return rlscan_gae_typed_ex(rewards, values, terminateds, truncateds, bootstrap_values, last_values, advantages,
                               returns, E, T, gamma, lambda_, value_dtype, flag_dtype, 0u, ws, ws_bytes, stream);
}

int rlscan_gae_noalloc(const float *rewards, const float *values, const float *terminateds, const float *truncateds,
                       const float *bootstrap_values, const float *last_values, float *advantages, int64_t E,
                       int64_t T, float gamma, float lambda_, cudaStream_t stream) {
    // the same host checks as rlscan_gae, so a rejected call enqueues nothing
    RLSCAN_TRY(check_shape(E, T));
    RLSCAN_TRY(check_scalar(gamma, "gamma"));
    RLSCAN_TRY(check_scalar(lambda_, "lambda_"));
    if (E == 0 || T == 0) return ok();
    RLSCAN_TRY(require(rewards, "rewards"));
    RLSCAN_TRY(require(values, "values"));
    RLSCAN_TRY(require(advantages, "advantages"));
    if (truncateds && !bootstrap_values) return fail(RLSCAN_ERR_INVALID_ARG, "truncateds given without bootstrap_values");
    const size_t pb = plane_bytes(E, T);
    const Span ins[] = {{rewards, pb, "rewards"}, {values, pb, "values"}, {terminateds, pb, "terminateds"},
                        {truncateds, pb, "truncateds"}, {bootstrap_values, pb, "bootstrap_values"},
                        {last_values, (size_t)E * 4, "last_values"}};
    const Span outs[] = {{advantages, pb, "advantages"}};
    RLSCAN_TRY(check_aliasing(ins, 6, outs, 1));
    const size_t need = workspace_for(make_plan(E, T), E * T);
    if (need > RLSCAN_NOALLOC_SCRATCH_BYTES)
        return fail(RLSCAN_ERR_WORKSPACE,
                    "rlscan_gae_noalloc: shape E=%lld T=%lld needs %zu bytes of scratch; the fixed scratch holds %u",
                    (long long)E, (long long)T, need, (unsigned)RLSCAN_NOALLOC_SCRATCH_BYTES);
    void *ws = nullptr;
    if (need > 0) {
        RLSCAN_TRY(noalloc_scratch(&ws));
        // the array keeps the previous call's contents: cleared, so that
        // each call starts from the same state as with a fresh workspace
        cudaError_t e = cudaMemsetAsync(ws, 0, need, stream);
        if (e != cudaSuccess) return fail(RLSCAN_ERR_CUDA, "cudaMemsetAsync(scratch): %s", cudaGetErrorString(e));
    }
    return rlscan_gae(rewards, values, terminateds, truncateds, bootstrap_values, last_values, advantages, E, T, gamma,
                      lambda_, ws, need, stream);
}

} // extern "C"
