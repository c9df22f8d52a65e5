// batch.cu - rlscan_batch: several independent calls in one request.  The
// fusable calls run as one launch of the fused kernels (batch.cuh), whose
// blocks run one tile of one call each; the others through their own entry
// points, which this file calls.
#include "typed.cuh"

using namespace rlscan;

extern "C" {

// ---------------------------------------------------------------------------
// rlscan_batch
// ---------------------------------------------------------------------------

// Element size of a plane dtype; 0 for a value that names no dtype.  Only
// called on calls that the dry pass (step 1 of rlscan_batch) has accepted,
// so every dtype reaching it is one its kind takes.
static size_t dtype_bytes(int dtype) {
    switch (dtype) {
    case RLSCAN_F32:
    case RLSCAN_I32: return 4;
    case RLSCAN_BF16:
    case RLSCAN_F16: return 2;
    case RLSCAN_U8: return 1;
    default: return 0;
    }
}

// Byte extent of argument slot `slot` of a call (its input when in_slot,
// else its output); 0 for slots the kind does not have.

static size_t call_slot_bytes(const rlscan_call &c, bool in_slot, int slot) {
    const size_t n = (size_t)(c.E * c.T), plane = n * 4u, row = (size_t)c.E * 4u;
    if (!in_slot) {
        const int nout = c.kind == RLSCAN_KIND_GAE_VTRACE
                             ? 4
                             : ((c.kind == RLSCAN_KIND_GAE_WITH_RETURNS || c.kind == RLSCAN_KIND_VTRACE ||
                                 c.kind == RLSCAN_KIND_GAE_TYPED)
                                    ? 2
                                    : 1);
        return slot < nout ? plane : 0;
    }
    // value planes of the call's dtype, flag planes of its flag_dtype
    const size_t v = n * dtype_bytes(c.dtype), f = n * dtype_bytes(c.flag_dtype);
    switch (c.kind) {
    case RLSCAN_KIND_GAE:
    case RLSCAN_KIND_GAE_WITH_RETURNS:
    case RLSCAN_KIND_GAE_TYPED:
    case RLSCAN_KIND_LAMBDA_RETURNS: {
        const size_t by_slot[6] = {v, v, f, f, v, row};
        return slot < 6 ? by_slot[slot] : 0;
    }
    case RLSCAN_KIND_VTRACE:
    case RLSCAN_KIND_GAE_VTRACE: {
        const size_t by_slot[7] = {v, v, v, f, f, v, row};
        return slot < 7 ? by_slot[slot] : 0;
    }
    case RLSCAN_KIND_RETRACE: {
        const size_t A = (size_t)(c.A > 0 ? c.A : 1);
        const size_t by_slot[7] = {v, v, v * A, v * A, v, f, f};
        return slot < 7 ? by_slot[slot] : 0;
    }
    case RLSCAN_KIND_DISCOUNTED_RETURNS: {
        const size_t by_slot[5] = {v, f, f, v, row};
        return slot < 5 ? by_slot[slot] : 0;
    }
    case RLSCAN_KIND_ELIGIBILITY_TRACES:
    case RLSCAN_KIND_EPISODIC_PREFIX_SUM: return slot == 0 ? v : (slot == 1 ? f : 0);
    default: return 0;
    }
}

static int call_dispatch(const rlscan_call &c, void *ws, size_t ws_bytes, cudaStream_t stream) {
    const float *const *in = reinterpret_cast<const float *const *>(c.in);
    float *const *out = reinterpret_cast<float *const *>(c.out);
    if (call_is_typed(c)) { // reduced-byte inputs
        switch (c.kind) {
        case RLSCAN_KIND_GAE:
        case RLSCAN_KIND_GAE_WITH_RETURNS:
            return rlscan_gae_typed_ex(c.in[0], c.in[1], c.in[2], c.in[3], c.in[4], in[5], out[0],
                                       c.kind == RLSCAN_KIND_GAE_WITH_RETURNS ? out[1] : nullptr, c.E, c.T, c.gamma,
                                       c.lambda_, c.dtype, c.flag_dtype, c.options, ws, ws_bytes, stream);
        case RLSCAN_KIND_VTRACE: return typed_vtrace(c, ws, ws_bytes, stream);
        case RLSCAN_KIND_RETRACE: return typed_retrace(c, ws, ws_bytes, stream);
        case RLSCAN_KIND_LAMBDA_RETURNS: return typed_lambda_returns(c, ws, ws_bytes, stream);
        case RLSCAN_KIND_DISCOUNTED_RETURNS: return typed_discounted_returns(c, ws, ws_bytes, stream);
        case RLSCAN_KIND_ELIGIBILITY_TRACES: return typed_eligibility_traces(c, ws, ws_bytes, stream);
        case RLSCAN_KIND_EPISODIC_PREFIX_SUM: return typed_episodic_prefix_sum(c, ws, ws_bytes, stream);
        case RLSCAN_KIND_GAE_TYPED: break; // its own entry point reads dtype and flag_dtype
        case RLSCAN_KIND_GAE_VTRACE:
            return fail(RLSCAN_ERR_UNSUPPORTED, "GAE_VTRACE takes fp32 inputs only (dtype and flag_dtype F32)");
        default: return fail(RLSCAN_ERR_INVALID_ARG, "unknown kind %d", c.kind);
        }
    }
    switch (c.kind) {
    case RLSCAN_KIND_GAE:
        return rlscan_gae_ex(in[0], in[1], in[2], in[3], in[4], in[5], out[0], c.E, c.T, c.gamma, c.lambda_,
                             c.options, ws, ws_bytes, stream);
    case RLSCAN_KIND_GAE_WITH_RETURNS:
        return rlscan_gae_with_returns_ex(in[0], in[1], in[2], in[3], in[4], in[5], out[0], out[1], c.E, c.T,
                                          c.gamma, c.lambda_, c.options, ws, ws_bytes, stream);
    case RLSCAN_KIND_VTRACE:
        return rlscan_vtrace_ex(in[0], in[1], in[2], in[3], in[4], in[5], in[6], out[0], out[1], c.E, c.T, c.gamma,
                                c.lambda_, c.rho_bar, c.c_bar, c.options, ws, ws_bytes, stream);
    case RLSCAN_KIND_GAE_VTRACE:
        return rlscan_gae_vtrace_ex(in[0], in[1], in[2], in[3], in[4], in[5], in[6], out[0], out[1], out[2], out[3],
                                    c.E, c.T, c.gamma, c.lambda_, c.vtrace_lambda, c.rho_bar, c.c_bar, c.options, ws,
                                    ws_bytes, stream);
    case RLSCAN_KIND_RETRACE:
        return rlscan_retrace_ex(in[0], in[1], in[2], in[3], in[4], in[5], in[6], out[0], c.E, c.T, c.A, c.gamma,
                                 c.lambda_, c.c_bar, c.options, ws, ws_bytes, stream);
    case RLSCAN_KIND_LAMBDA_RETURNS:
        return rlscan_lambda_returns_ex(in[0], in[1], in[2], in[3], in[4], in[5], out[0], c.E, c.T, c.gamma,
                                        c.lambda_, c.options, ws, ws_bytes, stream);
    case RLSCAN_KIND_DISCOUNTED_RETURNS:
        return rlscan_discounted_returns_ex(in[0], in[1], in[2], in[3], in[4], out[0], c.E, c.T, c.gamma,
                                            c.options, ws, ws_bytes, stream);
    case RLSCAN_KIND_ELIGIBILITY_TRACES:
        return rlscan_eligibility_traces_ex(in[0], in[1], out[0], c.E, c.T, c.gamma, c.lambda_, c.options, ws,
                                            ws_bytes, stream);
    case RLSCAN_KIND_EPISODIC_PREFIX_SUM:
        return rlscan_episodic_prefix_sum_ex(c.in[0], c.dtype, in[1], c.out[0], c.E, c.T, c.options, ws, ws_bytes,
                                             stream);
    case RLSCAN_KIND_GAE_TYPED:
        return rlscan_gae_typed_ex(c.in[0], c.in[1], c.in[2], c.in[3], c.in[4], in[5], out[0], out[1], c.E, c.T,
                                   c.gamma, c.lambda_, c.dtype, c.flag_dtype, c.options, ws, ws_bytes, stream);
    default: return fail(RLSCAN_ERR_INVALID_ARG, "unknown kind %d", c.kind);
    }
}

// Fused calls are tiled at 128 threads x 8 elements (measured at 4096 x
// 128: the eight estimators of one step in 15.2 us, against 15.6 us with 4
// elements per thread whenever three or more bodies meet).  The items arrive
// ordered by body, heaviest tiles first (Retrace, V-Trace, the backward
// family, the forward body, the int32 prefix sum): blocks of one body then
// mostly share each SM, and the launch ends on its lightest tiles (the step
// 14.4 us in this order against 15.2 us in the bodies' enum order).
static constexpr int kFusedBodyOrder[kNumFusedBodies] = {2, 1, 0, 3, 4}; // rank of each FusedBody
constexpr int kMaxBodiesPerLaunch = kNumFusedBodies; // every fused call in one launch

static void fused_layout(FusedBatch &fb, long long *tiles) {
    constexpr int V = kFusedV;
    long long begin = 0;
    for (int i = 0; i < fb.n; ++i) {
        FusedItem &it = fb.item[i];
        const long long T = it.g.seq_len;
        it.g.ntiles = ceil_div(it.g.n, (long long)kFusedNT * V);
        it.mode = ((32LL * V) % T == 0) ? kModeWarp : kModeBlock;
        it.g.scan_lanes = it.mode == kModeWarp ? (int)std::min<long long>(32, T >= V ? T / V : 1) : 32;
        it.tile_begin = begin;
        begin += it.g.ntiles;
    }
    *tiles = begin;
}

// A launch whose calls all have whole rows in every warp (warp-local scans),
// rows a multiple of V steps long, a whole number of tiles and 16-byte
// aligned planes, and pass no truncations (except to Retrace, whose builder
// always tests them), runs the kCasePlain kernel: one builder variant per
// body and no scalar loads, so the five bodies take less of each SM's
// instruction caches (the 4096 x 128 step of eight calls:
// 12.9 against 13.4 us; eight Retrace calls alone, on inputs that stay in
// L2, 16.9 against 16.4 us).
static bool fused_plain(const FusedBatch &fb) {
    constexpr long long S = (long long)kFusedNT * kFusedV;
    for (int i = 0; i < fb.n; ++i) {
        const FusedItem &it = fb.item[i];
        if (it.truncation_code || it.mode != kModeWarp || it.g.seq_len % kFusedV != 0 || it.g.n % S != 0 ||
            it.g.vec_ok == 0)
            return false;
    }
    return true;
}

// Runs every call of the request in the given pass; the first failure is
// reported with its call index.
static int batch_pass(BatchState &st, const rlscan_call *calls, int ncalls, void *ws, size_t ws_bytes,
                      cudaStream_t stream) {
    g_batch = &st;
    for (int i = 0; i < ncalls; ++i) {
        const int rc = call_dispatch(calls[i], ws, ws_bytes, stream);
        if (rc != RLSCAN_OK) {
            g_batch = nullptr;
            const std::string msg = g_last_error;
            return fail(rc, "call %d: %s", i, msg.c_str());
        }
    }
    g_batch = nullptr;
    return RLSCAN_OK;
}

int rlscan_batch(const rlscan_call *calls, int ncalls, void *ws, size_t ws_bytes, cudaStream_t stream) {
    if (ncalls < 0 || ncalls > RLSCAN_BATCH_MAX)
        return fail(RLSCAN_ERR_INVALID_ARG, "ncalls must be in [0, %d] (got %d)", RLSCAN_BATCH_MAX, ncalls);
    if (ncalls == 0) return ok();
    if (calls == nullptr) return fail(RLSCAN_ERR_INVALID_ARG, "calls must not be NULL");
    if (g_batch != nullptr) return fail(RLSCAN_ERR_INVALID_ARG, "rlscan_batch is not reentrant");
    // 1. every call checked as its entry point would, nothing enqueued
    BatchState st{};
    st.pass = kBatchDry;
    RLSCAN_TRY(batch_pass(st, calls, ncalls, ws, ws_bytes, stream));
    // 2. calls run concurrently: no output of one may overlap anything of another
    for (int i = 0; i < ncalls; ++i) {
        for (int j = i + 1; j < ncalls; ++j) {
            Span ins[2 * RLSCAN_CALL_MAX_IN], outs[2 * RLSCAN_CALL_MAX_OUT];
            int ni = 0, no = 0;
            const rlscan_call *pair[2] = {&calls[i], &calls[j]};
            for (const rlscan_call *c : pair) {
                const bool empty = c->E == 0 || c->T == 0;
                for (int k = 0; k < RLSCAN_CALL_MAX_IN; ++k)
                    ins[ni++] = {empty ? nullptr : c->in[k], call_slot_bytes(*c, true, k), "an input"};
                for (int k = 0; k < RLSCAN_CALL_MAX_OUT; ++k)
                    outs[no++] = {empty ? nullptr : c->out[k], call_slot_bytes(*c, false, k), "an output"};
            }
            if (check_aliasing(ins, ni, outs, no) != RLSCAN_OK) {
                const std::string msg = g_last_error;
                return fail(RLSCAN_ERR_INVALID_ARG, "calls %d and %d: %s", i, j, msg.c_str());
            }
        }
    }
    // 3. launch: unfusable calls one by one, the rest recorded for one launch
    st = BatchState{};
    st.pass = kBatchRecord;
    RLSCAN_TRY(batch_pass(st, calls, ncalls, ws, ws_bytes, stream));
    if (st.fb.n == 0) return ok();
    // the recorded calls ordered by body, then cut into launches of at most
    // kMaxBodiesPerLaunch bodies each (consecutive launches overlap through
    // programmatic dependent launch)
    std::stable_sort(st.fb.item, st.fb.item + st.fb.n, [](const FusedItem &x, const FusedItem &y) {
        return kFusedBodyOrder[x.kind] < kFusedBodyOrder[y.kind];
    });
    for (int first = 0; first < st.fb.n;) {
        int last = first, bodies = 1;
        while (last + 1 < st.fb.n &&
               (st.fb.item[last + 1].kind == st.fb.item[last].kind || bodies < kMaxBodiesPerLaunch)) {
            if (st.fb.item[last + 1].kind != st.fb.item[last].kind) ++bodies;
            ++last;
        }
        FusedBatch part{};
        part.n = last - first + 1;
        std::copy(st.fb.item + first, st.fb.item + last + 1, part.item);
        long long tiles = 0;
        fused_layout(part, &tiles);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)tiles);
        cfg.blockDim = dim3(kFusedNT);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = pdl_enabled() ? 1 : 0;
        const bool plain = fused_plain(part);
        // the first wave of blocks (the instance's resident blocks on every
        // SM) prefetches its tiles into L2
        const long long pf = num_sms() * (long long)(plain ? fused_min_blocks<kCasePlain>()
                                                           : fused_min_blocks<kCaseAny>());
        for (int i = 0; i < part.n; ++i) part.item[i].g.pf_blocks = pf;
        const cudaError_t e = plain ? cudaLaunchKernelEx(&cfg, fused_tile_kernel<kFusedV, kCasePlain>, part)
                                    : cudaLaunchKernelEx(&cfg, fused_tile_kernel<kFusedV, kCaseAny>, part);
        if (e != cudaSuccess)
            return fail(RLSCAN_ERR_CUDA, "rlscan_batch: fused launch failed: %s", cudaGetErrorString(e));
        first = last + 1;
    }
    return ok();
}

} // extern "C"
