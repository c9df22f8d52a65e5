// batch.cuh - one launch for several independent estimator calls.
//
// A fused grid is the concatenation of the calls' tile grids: block b runs
// tile b - tile_begin of the call whose range holds b, through the same tile
// body (and so the same arithmetic, bit for bit) as that call's own launch.
// Only calls whose rows fit whole in one tile are fused, so every block of
// the grid has the same shape: 128 threads x 8 elements, or x 4 elements
// when the request mixes several estimators (blocks of different
// estimators then share each SM, and the smaller unrolled bodies fit the
// instruction caches better).
#pragma once

#include "fused_any.cuh"

namespace rlscan {

enum FusedKind {
    kFkGae = 0,
    kFkGaeReturns,
    kFkVtrace,
    kFkRetrace1,
    kFkLambda,
    kFkReturns,
    kFkTraces,
    kFkPrefixF32,
    kFkPrefixI32,
    kNumFusedKinds
};

template <class Est>
struct FusedKindOf {
    static constexpr int value = -1;
};
template <>
struct FusedKindOf<GaeEst> {
    static constexpr int value = kFkGae;
};
template <>
struct FusedKindOf<GaeReturnsEst> {
    static constexpr int value = kFkGaeReturns;
};
template <>
struct FusedKindOf<VtraceEst> {
    static constexpr int value = kFkVtrace;
};
template <>
struct FusedKindOf<RetraceEst<false>> {
    static constexpr int value = kFkRetrace1;
};
template <>
struct FusedKindOf<LambdaReturnsEst> {
    static constexpr int value = kFkLambda;
};
template <>
struct FusedKindOf<ReturnsEst> {
    static constexpr int value = kFkReturns;
};
template <>
struct FusedKindOf<TracesEst> {
    static constexpr int value = kFkTraces;
};
template <>
struct FusedKindOf<PrefixF32Est> {
    static constexpr int value = kFkPrefixF32;
};
template <>
struct FusedKindOf<PrefixI32Est> {
    static constexpr int value = kFkPrefixI32;
};

constexpr int kFusedNT = 128; // 128 threads x 8 (or 4) elements per tile
constexpr int kFusedVMax = 8;
constexpr int kFusedParamBytes = 128;
constexpr int kFusedMax = 16;

struct FusedItem {
    alignas(16) unsigned char params[kFusedParamBytes]; // the call's Est::Params
    Geometry g;
    long long tile_begin; // first block of this call in the fused grid
    int kind;             // FusedKind
    int mode;             // kModeWarp or kModeBlock
};

struct FusedBatch {
    FusedItem item[kFusedMax];
    int n;
};

template <class Est, int V, int kMode>
__device__ __forceinline__ void fused_tile(const FusedItem &it, long long block, unsigned char *smem) {
    const auto &P = *reinterpret_cast<const typename Est::Params *>(it.params);
    const Lookback lb{nullptr, nullptr, 0u, -1}; // no look-back in a fused launch
    tile_scan_body<Est, kFusedNT, V, kMode>(P, it.g, lb, block, smem);
}

template <class Est, int V>
__device__ __forceinline__ void fused_tile_any_mode(const FusedItem &it, long long block, unsigned char *smem) {
    if (it.mode == kModeWarp)
        fused_tile<Est, V, kModeWarp>(it, block, smem);
    else
        fused_tile<Est, V, kModeBlock>(it, block, smem);
}

// ---------------------------------------------------------------------------
// The same calls on the shared fp32 body (fused_any.cuh): each fp32 call's
// parameters in AnyParams form.  Returns false for calls that body does not
// take (the int32 prefix sum).
// ---------------------------------------------------------------------------
inline AnyParams any_base() {
    AnyParams a{};
    a.lam = 1.0f;
    a.rho_bar = 1.0f;
    a.c_bar = 1.0f;
    return a;
}
inline bool to_any(const GaeEst::Params &p, AnyParams &a) {
    a = any_base();
    a.r = p.rewards; a.v = p.values; a.f = p.terminateds; a.tr = p.truncateds;
    a.bv = p.bootstrap_values; a.lv = p.last_values; a.out0 = p.advantages;
    a.gamma = p.gamma; a.lam = p.lambda_; a.w_nv = 1.0f; a.halo = kAnyHaloV;
    a.flags = kAnySubV;
    return true;
}
inline bool to_any(const GaeReturnsEst::Params &p, AnyParams &a) {
    a = any_base();
    a.r = p.rewards; a.v = p.values; a.f = p.terminateds; a.tr = p.truncateds;
    a.bv = p.bootstrap_values; a.lv = p.last_values; a.out0 = p.advantages; a.out1 = p.returns;
    a.gamma = p.gamma; a.lam = p.lambda_; a.w_nv = 1.0f; a.halo = kAnyHaloV;
    a.flags = kAnySubV | (p.returns != nullptr ? kAnyOut1PlusV : 0u);
    return true;
}
inline bool to_any(const VtraceEst::Params &p, AnyParams &a) {
    a = any_base();
    a.r = p.rewards; a.v = p.values; a.f = p.terminateds; a.tr = p.truncateds; a.lr = p.log_rhos;
    a.bv = p.bootstrap_values; a.lv = p.last_values; a.out0 = p.vs; a.out1 = p.pg_advantages;
    a.gamma = p.gamma; a.lam = p.lambda_; a.rho_bar = p.rho_bar; a.c_bar = p.c_bar; a.w_nv = 1.0f;
    a.halo = kAnyHaloV;
    a.flags = kAnyRatioOwn | kAnySubV | kAnyOut0PlusV | kAnyOut1Pg;
    return true;
}
inline bool to_any(const RetraceEst<false>::Params &p, AnyParams &a) {
    a = any_base();
    a.r = p.rewards; a.v = p.q_values; a.f = p.terminateds; a.tr = p.truncateds; a.lr = p.log_rhos;
    a.nq = p.next_q_values_all; a.out0 = p.q_ret;
    a.gamma = p.gamma; a.lam = p.lambda_; a.c_bar = p.c_bar; a.halo = kAnyHaloLogRho;
    a.flags = kAnyRatioNext | kAnySubV | kAnyRetraceBoot | kAnyOut0PlusV;
    return true;
}
inline bool to_any(const LambdaReturnsEst::Params &p, AnyParams &a) {
    a = any_base();
    a.r = p.rewards; a.v = p.values; a.f = p.terminateds; a.tr = p.truncateds;
    a.bv = p.bootstrap_values; a.lv = p.last_values; a.out0 = p.returns;
    a.gamma = p.gamma; a.lam = p.lambda_; a.w_nv = 1.0f - p.lambda_; a.halo = kAnyHaloV;
    a.flags = 0u;
    return true;
}
inline bool to_any(const ReturnsEst::Params &p, AnyParams &a) {
    a = any_base();
    a.r = p.rewards; a.f = p.terminateds; a.tr = p.truncateds;
    a.bv = p.bootstrap_values; a.lv = p.last_values; a.out0 = p.returns;
    a.gamma = p.gamma; a.w_nv = 0.0f; a.halo = kAnyHaloNone;
    a.flags = 0u;
    return true;
}
template <int kKind>
inline bool to_any(const typename ForwardF32Est<kKind>::Params &p, AnyParams &a) {
    a = any_base();
    a.r = p.x; a.f = p.dones; a.out0 = p.out;
    a.gamma = p.decay; a.halo = kAnyHaloDone;
    a.flags = kAnyFwd | (p.reset_on_flag ? kAnyResetOnFlag : 0u);
    return true;
}
inline bool to_any(const TracesEst::Params &p, AnyParams &a) { return to_any<0>(p, a); }
inline bool to_any(const PrefixF32Est::Params &p, AnyParams &a) { return to_any<1>(p, a); }
inline bool to_any(const PrefixI32Est::Params &, AnyParams &) { return false; }

template <int V>
__global__ void __launch_bounds__(kFusedNT) fused_tile_kernel(const __grid_constant__ FusedBatch b) {
    extern __shared__ __align__(128) unsigned char dyn_smem[];
    int idx = 0;
    for (int i = 1; i < b.n; ++i)
        if ((long long)blockIdx.x >= b.item[i].tile_begin) idx = i;
    const FusedItem &it = b.item[idx];
    const long long block = (long long)blockIdx.x - it.tile_begin;
    switch (it.kind) {
    case kFkGae: fused_tile_any_mode<GaeEst, V>(it, block, dyn_smem); break;
    case kFkGaeReturns: fused_tile_any_mode<GaeReturnsEst, V>(it, block, dyn_smem); break;
    case kFkVtrace: fused_tile_any_mode<VtraceEst, V>(it, block, dyn_smem); break;
    case kFkRetrace1: fused_tile_any_mode<RetraceEst<false>, V>(it, block, dyn_smem); break;
    case kFkLambda: fused_tile_any_mode<LambdaReturnsEst, V>(it, block, dyn_smem); break;
    case kFkReturns: fused_tile_any_mode<ReturnsEst, V>(it, block, dyn_smem); break;
    case kFkTraces: fused_tile_any_mode<TracesEst, V>(it, block, dyn_smem); break;
    case kFkPrefixF32: fused_tile_any_mode<PrefixF32Est, V>(it, block, dyn_smem); break;
    case kFkPrefixI32: fused_tile_any_mode<PrefixI32Est, V>(it, block, dyn_smem); break;
    default: break;
    }
}

// Fused launch on the shared body: every fp32 call runs any_tile_body, the
// int32 prefix sum its own tile body.  Items carry AnyParams for fp32 calls.
template <int V>
__global__ void __launch_bounds__(kFusedNT) fused_any_kernel(const __grid_constant__ FusedBatch b) {
    extern __shared__ __align__(128) unsigned char dyn_smem[];
    int idx = 0;
    for (int i = 1; i < b.n; ++i)
        if ((long long)blockIdx.x >= b.item[i].tile_begin) idx = i;
    const FusedItem &it = b.item[idx];
    const long long block = (long long)blockIdx.x - it.tile_begin;
    if (it.kind == kFkPrefixI32)
        fused_tile_any_mode<PrefixI32Est, V>(it, block, dyn_smem);
    else
        any_tile_body<V>(*reinterpret_cast<const AnyParams *>(it.params), it.g, block, it.mode);
}

} // namespace rlscan
