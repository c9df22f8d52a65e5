// batch.cuh - one launch for several independent estimator calls.
//
// A fused grid is the concatenation of the calls' tile grids: block b runs
// tile b - tile_begin of the call whose range holds b, through the same tile
// body (and so the same arithmetic, bit for bit) as that call's own launch.
// Only calls whose rows fit whole in one tile are fused, so every block of
// the grid has the same shape: 128 threads x 8 elements.
#pragma once

#include <utility>

#include "estimators.cuh"

namespace rlscan {

// Tile bodies of a fused launch.  Calls whose estimators are one recurrence
// with different constants share a body, so that fewer distinct bodies share
// each SM's instruction caches: GAE, GAE + returns, TD(lambda) returns and
// discounted returns run the backward family body; eligibility traces and
// the fp32 prefix sum the forward body (the prefix sum is a trace with decay
// 1).  Each call's arithmetic in its family body is its own estimator's, in
// the same order, so results equal its own kernel's bit for bit on the same
// tiles.
enum FusedBody {
    kBodyBackward = 0, // BackwardFamilyEst
    kBodyVtrace,       // VtraceEst
    kBodyRetrace1,     // RetraceEst
    kBodyForward,      // TracesEst (the fp32 prefix sum is the same estimator)
    kBodyPrefixI32,    // PrefixI32Est
    kNumFusedBodies
};

// GAE (+ returns), TD(lambda) returns and discounted returns as one
// backward recurrence x_t = a_t x_{t+1} + b_t with
//   a_t = gamma lambda  while the episode goes on inside the row, else 0
//   b_t = r_t + gamma boot_t - [V_t]
//   boot_t = w_nv V_{t+1} inside the episode, the row's last value at a row
//            end, the bootstrap value at a truncation, 0 at a termination
// GAE: w_nv = 1, V subtracted (x = A; returns x + V); TD(lambda): w_nv =
// 1 - lambda, nothing subtracted (x = G); discounted returns: lambda = 1,
// no values (w_nv = 0), nothing subtracted (x = R).  Used by fused launches.
struct BackwardFamilyEst {
    static constexpr bool kBackward = true;
    using AT = float;
    using BT = float;
    struct Params {
        const float *rewards, *values, *terminateds, *truncateds, *bootstrap_values, *last_values;
        float *out0; // x
        float *out1; // x + V (the TD(lambda) returns beside GAE), may be null
        float gamma, lambda_, w_nv;
        int sub_v;
    };
    template <int V>
    struct State {
        float r[V], v[V], te[V], tr[V], bv[V], o0[V], o1[V];
        float v_next;
    };
    static __device__ __forceinline__ void prefetch(const Params &P, const Geometry &g, long long tile0, int S) {
        prefetch_planes(g, tile0, S, P.rewards, P.values, P.terminateds, P.truncateds, P.bootstrap_values);
    }
    static constexpr int kInputPlanes = 5;
    static __host__ __device__ __forceinline__ PlaneRef input_plane(const Params &P, int i) {
        const float *p[5] = {P.rewards, P.values, P.terminateds, P.truncateds, P.bootstrap_values};
        return {i < 5 ? p[i] : nullptr, 4};
    }
    template <int NT, int V, class Pos>
    static __device__ __forceinline__ void load(const Params &P, const Geometry &g, const Pos &pos,
                                                State<V> &S, unsigned char *) {
        const float h_v_next = pos.fetch_next(P.values);
        pos.load(P.rewards, S.r);
        pos.load(P.values, S.v);
        pos.load(P.terminateds, S.te);
        pos.load(P.truncateds, S.tr);
        pos.load(P.bootstrap_values, S.bv);
        S.v_next = pos.next(S.v, h_v_next);
    }
    template <int V, bool kTrunc, bool kFast, class Pos>
    static __device__ __forceinline__ void coeffs_impl(const Params &P, const Geometry &g, const Pos &pos,
                                                  const RowMasks &rm, State<V> &S,
                                                  float (&a)[V], float (&b)[V]) {
        const float gl = P.gamma * P.lambda_;
#pragma unroll
        for (int k = 0; k < V; ++k) {
            if (elem_valid<kFast, V>(rm, k)) {
                const StepFlags f = step_flags<kTrunc>(S.te[k], S.tr[k]);
                const bool rowend = elem_row_end<kFast, V>(rm, k);
                float boot;
                if (f.cont) {
                    boot = rowend ? row_last_value(P.last_values, elem_row<kFast>(rm, k), g.rows)
                                  : P.w_nv * ((k + 1 < V) ? S.v[k + 1] : S.v_next);
                } else {
                    boot = f.trn ? S.bv[k] : 0.0f;
                }
                a[k] = (f.cont && !rowend) ? gl : 0.0f;
                float bb = fmaf(P.gamma, boot, S.r[k]);
                if (P.sub_v) bb = bb - S.v[k];
                b[k] = bb;
            } else {
                a[k] = 1.0f;
                b[k] = 0.0f;
            }
        }
    }
    template <int V, int kCase = kCaseAny, class Pos>
    static __device__ __forceinline__ void coeffs(const Params &P, const Geometry &g, const Pos &pos,
                                                  const RowMasks &rm, State<V> &S, float (&a)[V], float (&b)[V]) {
        if constexpr (kCase == kCasePlain) {
            coeffs_impl<V, false, true>(P, g, pos, rm, S, a, b);
        } else if constexpr (kCase == kCasePlainTrunc) {
            coeffs_impl<V, true, true>(P, g, pos, rm, S, a, b);
        } else if (P.truncateds != nullptr) {
            if (rm.fast) coeffs_impl<V, true, true>(P, g, pos, rm, S, a, b);
            else coeffs_impl<V, true, false>(P, g, pos, rm, S, a, b);
        } else {
            if (rm.fast) coeffs_impl<V, false, true>(P, g, pos, rm, S, a, b);
            else coeffs_impl<V, false, false>(P, g, pos, rm, S, a, b);
        }
    }
    template <int V>
    static __device__ __forceinline__ void out(const Params &, State<V> &S, int k, float x, float, float) {
        S.o0[k] = x;
        S.o1[k] = x + S.v[k];
    }
    template <int V, class Pos>
    static __device__ __forceinline__ void store(const Params &P, const Geometry &, const Pos &pos, State<V> &S) {
        pos.store(P.out0, S.o0);
        if (P.out1 != nullptr) pos.store(P.out1, S.o1);
    }
};

// Body of each fusable estimator and its parameters in that body's form.
template <class Est>
struct FusedBodyOf {
    static constexpr int value = -1;
};
template <> struct FusedBodyOf<GaeEst> { static constexpr int value = kBodyBackward; };
template <> struct FusedBodyOf<GaeReturnsEst> { static constexpr int value = kBodyBackward; };
template <> struct FusedBodyOf<LambdaReturnsEst> { static constexpr int value = kBodyBackward; };
template <> struct FusedBodyOf<ReturnsEst> { static constexpr int value = kBodyBackward; };
template <> struct FusedBodyOf<VtraceEst> { static constexpr int value = kBodyVtrace; };
template <> struct FusedBodyOf<RetraceEst> { static constexpr int value = kBodyRetrace1; };
template <> struct FusedBodyOf<TracesEst> { static constexpr int value = kBodyForward; };
template <> struct FusedBodyOf<PrefixI32Est> { static constexpr int value = kBodyPrefixI32; };

inline BackwardFamilyEst::Params family_params(const GaeEst::Params &p) {
    return {p.rewards, p.values, p.terminateds, p.truncateds, p.bootstrap_values, p.last_values,
            p.advantages, nullptr, p.gamma, p.lambda_, 1.0f, 1};
}
inline BackwardFamilyEst::Params family_params(const GaeReturnsEst::Params &p) {
    return {p.rewards, p.values, p.terminateds, p.truncateds, p.bootstrap_values, p.last_values,
            p.advantages, p.returns, p.gamma, p.lambda_, 1.0f, 1};
}
inline BackwardFamilyEst::Params family_params(const LambdaReturnsEst::Params &p) {
    return {p.rewards, p.values, p.terminateds, p.truncateds, p.bootstrap_values, p.last_values,
            p.returns, nullptr, p.gamma, p.lambda_, 1.0f - p.lambda_, 0};
}
inline BackwardFamilyEst::Params family_params(const ReturnsEst::Params &p) {
    return {p.rewards, nullptr, p.terminateds, p.truncateds, p.bootstrap_values, p.last_values,
            p.returns, nullptr, p.gamma, 1.0f, 0.0f, 0};
}
template <class P>
inline const P &family_params(const P &p) { // estimators that are their own body
    return p;
}

constexpr int kFusedNT = 128; // 128 threads x 8 elements per tile
constexpr int kFusedV = 8;
// Blocks per SM the fused kernel is compiled to fit.  General instance: 8
// (64 registers a thread; measured at 4096 x 128: the step's eight calls
// 13.9 us at 8 blocks per SM against 14.5 us at the 72 registers the bodies
// take unbounded, 7 blocks per SM, despite a few spilled registers).  Plain
// instance: 9 (56 registers; the step 12.15 against
// 12.95 us at 8 and 12.15 at 10, where eight Retrace calls on inputs that
// stay in L2 slow from 17.0 to 19.7 us).
constexpr int kFusedMinBlocks = 8;
constexpr int kFusedMinBlocksPlain = 9;
template <int kCase>
constexpr int fused_min_blocks() {
    return kCase == kCasePlain ? kFusedMinBlocksPlain : kFusedMinBlocks;
}
constexpr int kFusedParamBytes = 128;
constexpr int kFusedMax = 16;

struct FusedItem {
    alignas(16) unsigned char params[kFusedParamBytes]; // the call's parameters in its body's form
    Geometry g;
    long long tile_begin; // first block of this call in the fused grid
    int kind;             // FusedBody: the tile body that runs the call
    int mode;             // kModeWarp or kModeBlock
    int truncation_code;  // the call needs its body's truncation variants (not kCasePlain)
};

// Host side: whether a call, in its builder's parameter form P, passes
// truncations to a builder whose kCasePlain variant compiles them out.
// Retrace's builder tests its truncation flags in every variant, and
// builders without a truncation plane never take any.
template <class P, class = void>
struct HasTruncations : std::false_type {};
template <class P>
struct HasTruncations<P, std::void_t<decltype(std::declval<P>().truncateds)>> : std::true_type {};
template <class Est>
struct PlainTestsTruncations : std::false_type {};
template <class V, class F, class N>
struct PlainTestsTruncations<RetraceEstT<V, F, N>> : std::true_type {};
template <class Est, class P>
inline bool needs_truncation_code(const P &p) {
    if constexpr (PlainTestsTruncations<Est>::value || !HasTruncations<P>::value) return false;
    else return p.truncateds != nullptr;
}

struct FusedBatch {
    FusedItem item[kFusedMax];
    int n;
};

template <class Est, int V, int kMode, int kCase>
__device__ __forceinline__ void fused_tile(const FusedItem &it, long long block, unsigned char *smem) {
    const auto &P = *reinterpret_cast<const typename Est::Params *>(it.params);
    tile_scan_body<Est, kFusedNT, V, kMode, kCase>(P, it.g, block, smem);
}

// kCasePlain launches hold warp-local calls only (see fused_plain); the
// others pick the scan mode per call.
template <class Est, int V, int kCase>
__device__ __forceinline__ void fused_tile_any_mode(const FusedItem &it, long long block, unsigned char *smem) {
    if constexpr (kCase == kCasePlain) {
        fused_tile<Est, V, kModeWarp, kCasePlain>(it, block, smem);
    } else {
        if (it.mode == kModeWarp)
            fused_tile<Est, V, kModeWarp, kCase>(it, block, smem);
        else
            fused_tile<Est, V, kModeBlock, kCase>(it, block, smem);
    }
}

template <int V, int kCase>
__global__ void __launch_bounds__(kFusedNT, fused_min_blocks<kCase>())
    fused_tile_kernel(const __grid_constant__ FusedBatch b) {
    extern __shared__ __align__(128) unsigned char dyn_smem[];
    int idx = 0;
    for (int i = 1; i < b.n; ++i)
        if ((long long)blockIdx.x >= b.item[i].tile_begin) idx = i;
    const FusedItem &it = b.item[idx];
    const long long block = (long long)blockIdx.x - it.tile_begin;
    switch (it.kind) {
    case kBodyBackward: fused_tile_any_mode<BackwardFamilyEst, V, kCase>(it, block, dyn_smem); break;
    case kBodyVtrace: fused_tile_any_mode<VtraceEst, V, kCase>(it, block, dyn_smem); break;
    case kBodyRetrace1: fused_tile_any_mode<RetraceEst, V, kCase>(it, block, dyn_smem); break;
    case kBodyForward: fused_tile_any_mode<TracesEst, V, kCase>(it, block, dyn_smem); break;
    case kBodyPrefixI32: fused_tile_any_mode<PrefixI32Est, V, kCase>(it, block, dyn_smem); break;
    default: break;
    }
}

} // namespace rlscan
