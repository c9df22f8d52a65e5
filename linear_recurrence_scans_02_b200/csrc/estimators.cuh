// estimators.cuh - coefficient builders and epilogues of the seven rlscan
// estimators, one struct each, plugged into tile_scan_kernel.
//
// Each builder turns the estimator's inputs at step t into the pair (a_t, b_t)
// of x_t = a_t x_{t-+1} + b_t (rl-triton abstract: "algorithm-specific fused
// kernels constructing their recurrence coefficients on-chip") and each
// epilogue turns the scanned x_t into the estimator's outputs.  The
// definitions follow the rl-triton README "Kernels" table (one row per
// estimator) and its with-truncations paragraph:
//   - terminated_t: episode ends at t, no bootstrap, trace cut (a_t = 0);
//   - truncated_t (and not terminated): episode ends at t, bootstrap with
//     bootstrap_values[t], trace cut;
//   - last step of a row with no flag: bootstrap with last_values[row] (0 if
//     absent) folded into b_t, and a_t = 0 so rows never mix;
//   - forward estimators reset after a done: a_t = 0 when t == 0 or
//     dones[t-1] != 0 (or, with reset_on_flag, dones[t] != 0: the flag marks
//     the first step of an episode).
#pragma once

#include "scan_core.cuh"

namespace rlscan {

struct StepFlags {
    bool term, trn, cont;
};
template <bool kTrunc = true, class F = float>
__device__ __forceinline__ StepFlags step_flags(F te, F tr) {
    StepFlags f;
    f.term = te != F(0);
    f.trn = kTrunc && (tr != F(0)) && !f.term;
    f.cont = !f.term && !f.trn;
    return f;
}

// L2 prefetch of one tile of the given input planes (each of its own
// element type), one plane per thread (threads 0, 1, ...), before the kernel
// waits for the previous grid.
template <class... Ts>
__device__ __forceinline__ void prefetch_planes(const Geometry &g, long long tile0, int S, const Ts *... planes) {
    const long long left = g.n - tile0;
    const long long cnt = left < S ? left : S;
    int i = 0;
    ((threadIdx.x == i++ ? prefetch_l2(planes, tile0, cnt, (int)sizeof(Ts)) : (void)0), ...);
}

// A flag register is set iff nonzero (fp32 flags stay floats, byte flags
// integers).
__device__ __forceinline__ bool flag_set(float f) { return f != 0.0f; }
__device__ __forceinline__ bool flag_set(uint32_t f) { return f != 0u; }

__device__ __forceinline__ float row_last_value(const float *__restrict__ lv, long long row, long long rows) {
    return load_one(lv, row, rows);
}

// ---------------------------------------------------------------------------
// GAE: x = A,  a_t = gamma lambda (episode goes on, not row end), b_t = delta_t.
// kWithReturns: also write the TD(lambda) returns G_t = A_t + V_t from the
// same pass (the lambda-return equals the GAE advantage plus the value,
// step for step, within episodes and across truncations).
// ---------------------------------------------------------------------------
template <bool kWithReturns, class ValT = float, class FlagT = float>
struct GaeEstT {
    static constexpr bool kBackward = true;
    using AT = float;
    using BT = float;
    struct Params {
        const ValT *rewards, *values;
        const FlagT *terminateds, *truncateds;
        const ValT *bootstrap_values;
        const float *last_values;
        float *advantages;
        float *returns; // kWithReturns only; may be null there
        float gamma, lambda_;
    };
    template <int V>
    struct State {
        float r[V], v[V], bv[V], out[V], ret[V];
        FlagReg<FlagT> te[V], tr[V];
        float v_next;
    };
    static __device__ __forceinline__ void prefetch(const Params &P, const Geometry &g, long long tile0, int S) {
        const long long left = g.n - tile0;
        const long long cnt = left < S ? left : S;
        switch (threadIdx.x) {
        case 0: prefetch_l2(P.rewards, tile0, cnt, sizeof(ValT)); break;
        case 1: prefetch_l2(P.values, tile0, cnt, sizeof(ValT)); break;
        case 2: prefetch_l2(P.terminateds, tile0, cnt, sizeof(FlagT)); break;
        case 3: prefetch_l2(P.truncateds, tile0, cnt, sizeof(FlagT)); break;
        case 4: prefetch_l2(P.bootstrap_values, tile0, cnt, sizeof(ValT)); break;
        default: break;
        }
    }
    // Input planes read element by element (the time-major kernel's prefetch).
    static constexpr int kInputPlanes = 5;
    static __host__ __device__ __forceinline__ PlaneRef input_plane(const Params &P, int i) {
        switch (i) {
        case 0: return {P.rewards, (int)sizeof(ValT)};
        case 1: return {P.values, (int)sizeof(ValT)};
        case 2: return {P.terminateds, (int)sizeof(FlagT)};
        case 3: return {P.truncateds, (int)sizeof(FlagT)};
        case 4: return {P.bootstrap_values, (int)sizeof(ValT)};
        default: return {nullptr, 0};
        }
    }
    template <int NT, int V, class Pos>
    static __device__ __forceinline__ void load(const Params &P, const Geometry &g, const Pos &pos,
                                                State<V> &S, unsigned char *) {
        const float h_v_next = pos.fetch_next(P.values);
        pos.load_widen(P.rewards, S.r);
        pos.load_widen(P.values, S.v);
        pos.load_flag(P.terminateds, S.te);
        pos.load_flag(P.truncateds, S.tr);
        pos.load_widen(P.bootstrap_values, S.bv); // null (no truncations): zeros, no load
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
                float nv = (k + 1 < V) ? S.v[k + 1] : S.v_next;
                if (rowend) nv = row_last_value(P.last_values, elem_row<kFast>(rm, k), g.rows);
                const float boot = f.cont ? nv : (f.trn ? S.bv[k] : 0.0f);
                a[k] = (f.cont && !rowend) ? gl : 0.0f;
                b[k] = fmaf(P.gamma, boot, S.r[k]) - S.v[k];
            } else {
                a[k] = 1.0f;
                b[k] = 0.0f;
            }
        }
    }
    // uniform branches per thread: without truncations the truncation logic
    // is compiled out of the per-element loop, and on the fast path (all V
    // elements present, V divides T) so are the per-element row tests
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
        S.out[k] = x;
        if constexpr (kWithReturns) S.ret[k] = x + S.v[k];
    }
    template <int V, class Pos>
    static __device__ __forceinline__ void store(const Params &P, const Geometry &, const Pos &pos, State<V> &S) {
        pos.store(P.advantages, S.out);
        if constexpr (kWithReturns) {
            if (P.returns != nullptr) pos.store(P.returns, S.ret);
        }
    }
};
using GaeEst = GaeEstT<false>;
using GaeReturnsEst = GaeEstT<true>;
// reduced-byte inputs (returns written when P.returns is set)
template <class ValT, class FlagT>
using GaeTypedEst = GaeEstT<true, ValT, FlagT>;

// ---------------------------------------------------------------------------
// TD(lambda): x = G,  a_t = gamma lambda, b_t = r_t + gamma (1 - lambda) V_{t+1}
// ---------------------------------------------------------------------------
template <class ValT = float, class FlagT = float>
struct LambdaReturnsEstT {
    static constexpr bool kBackward = true;
    using AT = float;
    using BT = float;
    struct Params {
        const ValT *rewards, *values;
        const FlagT *terminateds, *truncateds;
        const ValT *bootstrap_values;
        const float *last_values;
        float *returns;
        float gamma, lambda_;
    };
    template <int V>
    struct State {
        float r[V], v[V], bv[V], out[V];
        FlagReg<FlagT> te[V], tr[V];
        float v_next;
    };
    static __device__ __forceinline__ void prefetch(const Params &P, const Geometry &g, long long tile0, int S) {
        prefetch_planes(g, tile0, S, P.rewards, P.values, P.terminateds, P.truncateds, P.bootstrap_values);
    }
    static constexpr int kInputPlanes = 5;
    static __host__ __device__ __forceinline__ PlaneRef input_plane(const Params &P, int i) {
        switch (i) {
        case 0: return {P.rewards, (int)sizeof(ValT)};
        case 1: return {P.values, (int)sizeof(ValT)};
        case 2: return {P.terminateds, (int)sizeof(FlagT)};
        case 3: return {P.truncateds, (int)sizeof(FlagT)};
        case 4: return {P.bootstrap_values, (int)sizeof(ValT)};
        default: return {nullptr, 0};
        }
    }
    template <int NT, int V, class Pos>
    static __device__ __forceinline__ void load(const Params &P, const Geometry &g, const Pos &pos,
                                                State<V> &S, unsigned char *) {
        const float h_v_next = pos.fetch_next(P.values);
        pos.load_widen(P.rewards, S.r);
        pos.load_widen(P.values, S.v);
        pos.load_flag(P.terminateds, S.te);
        pos.load_flag(P.truncateds, S.tr);
        pos.load_widen(P.bootstrap_values, S.bv);
        S.v_next = pos.next(S.v, h_v_next);
    }
    template <int V, bool kTrunc, bool kFast, class Pos>
    static __device__ __forceinline__ void coeffs_impl(const Params &P, const Geometry &g, const Pos &pos,
                                                  const RowMasks &rm, State<V> &S,
                                                  float (&a)[V], float (&b)[V]) {
        const float gl = P.gamma * P.lambda_;
        const float one_minus_l = 1.0f - P.lambda_;
#pragma unroll
        for (int k = 0; k < V; ++k) {
            if (elem_valid<kFast, V>(rm, k)) {
                const StepFlags f = step_flags<kTrunc>(S.te[k], S.tr[k]);
                const bool rowend = elem_row_end<kFast, V>(rm, k);
                // G_t = r_t + gamma * boot_t + (scan) gamma lambda G_{t+1}, with
                // boot_t = (1 - lambda) V_{t+1} inside the row, the last value at a
                // row end ((1 - lambda) V_T + lambda G_T with V_T = G_T = the last
                // value), the bootstrap value at a truncation and 0 at a termination
                float boot = 0.0f;
                if (f.trn) boot = S.bv[k];
                if (f.cont) {
                    if (rowend) {
                        boot = row_last_value(P.last_values, elem_row<kFast>(rm, k), g.rows);
                    } else {
                        boot = one_minus_l * ((k + 1 < V) ? S.v[k + 1] : S.v_next);
                    }
                }
                a[k] = (f.cont && !rowend) ? gl : 0.0f;
                b[k] = fmaf(P.gamma, boot, S.r[k]);
            } else {
                a[k] = 1.0f;
                b[k] = 0.0f;
            }
        }
    }
    // uniform branches per thread: without truncations the truncation logic
    // is compiled out of the per-element loop, and on the fast path (all V
    // elements present, V divides T) so are the per-element row tests
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
        S.out[k] = x;
    }
    template <int V, class Pos>
    static __device__ __forceinline__ void store(const Params &P, const Geometry &, const Pos &pos, State<V> &S) {
        pos.store(P.returns, S.out);
    }
};
using LambdaReturnsEst = LambdaReturnsEstT<>;

// ---------------------------------------------------------------------------
// Discounted returns: x = R,  a_t = gamma, b_t = r_t
// ---------------------------------------------------------------------------
template <class ValT = float, class FlagT = float>
struct ReturnsEstT {
    static constexpr bool kBackward = true;
    using AT = float;
    using BT = float;
    struct Params {
        const ValT *rewards;
        const FlagT *terminateds, *truncateds;
        const ValT *bootstrap_values;
        const float *last_values;
        float *returns;
        float gamma;
    };
    template <int V>
    struct State {
        float r[V], bv[V], out[V];
        FlagReg<FlagT> te[V], tr[V];
    };
    static __device__ __forceinline__ void prefetch(const Params &P, const Geometry &g, long long tile0, int S) {
        prefetch_planes(g, tile0, S, P.rewards, P.terminateds, P.truncateds, P.bootstrap_values);
    }
    static constexpr int kInputPlanes = 4;
    static __host__ __device__ __forceinline__ PlaneRef input_plane(const Params &P, int i) {
        switch (i) {
        case 0: return {P.rewards, (int)sizeof(ValT)};
        case 1: return {P.terminateds, (int)sizeof(FlagT)};
        case 2: return {P.truncateds, (int)sizeof(FlagT)};
        case 3: return {P.bootstrap_values, (int)sizeof(ValT)};
        default: return {nullptr, 0};
        }
    }
    template <int NT, int V, class Pos>
    static __device__ __forceinline__ void load(const Params &P, const Geometry &g, const Pos &pos,
                                                State<V> &S, unsigned char *) {
        pos.load_widen(P.rewards, S.r);
        pos.load_flag(P.terminateds, S.te);
        pos.load_flag(P.truncateds, S.tr);
        pos.load_widen(P.bootstrap_values, S.bv);
    }
    template <int V, bool kTrunc, bool kFast, class Pos>
    static __device__ __forceinline__ void coeffs_impl(const Params &P, const Geometry &g, const Pos &pos,
                                                  const RowMasks &rm, State<V> &S,
                                                  float (&a)[V], float (&b)[V]) {
#pragma unroll
        for (int k = 0; k < V; ++k) {
            if (elem_valid<kFast, V>(rm, k)) {
                const StepFlags f = step_flags<kTrunc>(S.te[k], S.tr[k]);
                const bool rowend = elem_row_end<kFast, V>(rm, k);
                // what this step bootstraps from outside the scan: the row's
                // last value at a row end, the bootstrap value at a
                // truncation, nothing otherwise (the scan carries R_{t+1})
                float boot = 0.0f;
                if (f.trn) boot = S.bv[k];
                if (f.cont && rowend) boot = row_last_value(P.last_values, elem_row<kFast>(rm, k), g.rows);
                a[k] = (f.cont && !rowend) ? P.gamma : 0.0f;
                b[k] = fmaf(P.gamma, boot, S.r[k]);
            } else {
                a[k] = 1.0f;
                b[k] = 0.0f;
            }
        }
    }
    // uniform branches per thread: without truncations the truncation logic
    // is compiled out of the per-element loop, and on the fast path (all V
    // elements present, V divides T) so are the per-element row tests
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
        S.out[k] = x;
    }
    template <int V, class Pos>
    static __device__ __forceinline__ void store(const Params &P, const Geometry &, const Pos &pos, State<V> &S) {
        pos.store(P.returns, S.out);
    }
};
using ReturnsEst = ReturnsEstT<>;

// ---------------------------------------------------------------------------
// V-Trace: x = D = vs - V,  a_t = gamma c_t, b_t = rho_t delta_t;
// epilogue vs_t = V_t + D_t and pg_t = rho_t (r_t + gamma vs_{t+1} - V_t).
// ---------------------------------------------------------------------------
template <class ValT = float, class FlagT = float>
struct VtraceEstT {
    static constexpr bool kBackward = true;
    using AT = float;
    using BT = float;
    struct Params {
        const ValT *log_rhos, *rewards, *values;
        const FlagT *terminateds, *truncateds;
        const ValT *bootstrap_values;
        const float *last_values;
        float *vs, *pg_advantages;
        float gamma, lambda_, rho_bar, c_bar;
    };
    template <int V>
    struct State {
        float lr[V], r[V], v[V], bv[V];
        FlagReg<FlagT> te[V], tr[V];
        float rho[V];
        float vs[V], pg[V];
        float v_next;
        unsigned chained; // bit k: the trace goes on to t+1 inside the row
    };
    static __device__ __forceinline__ void prefetch(const Params &P, const Geometry &g, long long tile0, int S) {
        prefetch_planes(g, tile0, S, P.log_rhos, P.rewards, P.values, P.terminateds, P.truncateds,
                        P.bootstrap_values);
    }
    static constexpr int kInputPlanes = 6;
    static __host__ __device__ __forceinline__ PlaneRef input_plane(const Params &P, int i) {
        switch (i) {
        case 0: return {P.log_rhos, (int)sizeof(ValT)};
        case 1: return {P.rewards, (int)sizeof(ValT)};
        case 2: return {P.values, (int)sizeof(ValT)};
        case 3: return {P.terminateds, (int)sizeof(FlagT)};
        case 4: return {P.truncateds, (int)sizeof(FlagT)};
        case 5: return {P.bootstrap_values, (int)sizeof(ValT)};
        default: return {nullptr, 0};
        }
    }
    template <int NT, int V, class Pos>
    static __device__ __forceinline__ void load(const Params &P, const Geometry &g, const Pos &pos,
                                                State<V> &S, unsigned char *) {
        const float h_v_next = pos.fetch_next(P.values);
        pos.load_widen(P.log_rhos, S.lr);
        pos.load_widen(P.rewards, S.r);
        pos.load_widen(P.values, S.v);
        pos.load_flag(P.terminateds, S.te);
        pos.load_flag(P.truncateds, S.tr);
        pos.load_widen(P.bootstrap_values, S.bv);
        S.v_next = pos.next(S.v, h_v_next);
    }
    template <int V, bool kTrunc, bool kFast, class Pos>
    static __device__ __forceinline__ void coeffs_impl(const Params &P, const Geometry &g, const Pos &pos,
                                                  const RowMasks &rm, State<V> &S,
                                                  float (&a)[V], float (&b)[V]) {
        S.chained = 0u;
#pragma unroll
        for (int k = 0; k < V; ++k) {
            if (elem_valid<kFast, V>(rm, k)) {
                const StepFlags f = step_flags<kTrunc>(S.te[k], S.tr[k]);
                const bool rowend = elem_row_end<kFast, V>(rm, k);
                const float ratio = __expf(S.lr[k]);
                const float rho = fminf(P.rho_bar, ratio);
                const float c = P.lambda_ * fminf(P.c_bar, ratio);
                float boot;
                if (f.cont) {
                    boot = rowend ? row_last_value(P.last_values, elem_row<kFast>(rm, k), g.rows)
                                  : ((k + 1 < V) ? S.v[k + 1] : S.v_next);
                } else {
                    boot = f.trn ? S.bv[k] : 0.0f;
                }
                a[k] = (f.cont && !rowend) ? P.gamma * c : 0.0f;
                b[k] = rho * (fmaf(P.gamma, boot, S.r[k]) - S.v[k]);
                S.rho[k] = rho;
                if (f.cont && !rowend) S.chained |= (1u << k);
            } else {
                a[k] = 1.0f;
                b[k] = 0.0f;
                S.rho[k] = 0.0f;
            }
        }
    }
    // vs_t = V_t + D_t.  pg_t = rho_t (r_t + gamma boot'_t - V_t) differs from
    // b_t = rho_t (r_t + gamma boot_t - V_t) only where the trace goes on,
    // where boot'_t = vs_{t+1} = V_{t+1} + D_{t+1} and boot_t = V_{t+1}:
    // there pg_t = b_t + rho_t gamma D_{t+1}; elsewhere pg_t = b_t.
    // uniform branches per thread: without truncations the truncation logic
    // is compiled out of the per-element loop, and on the fast path (all V
    // elements present, V divides T) so are the per-element row tests
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
    static __device__ __forceinline__ void out(const Params &P, State<V> &S, int k, float x, float x_next,
                                               float b_k) {
        S.vs[k] = S.v[k] + x;
        S.pg[k] = ((S.chained >> k) & 1u) ? fmaf(S.rho[k] * P.gamma, x_next, b_k) : b_k;
    }
    template <int V, class Pos>
    static __device__ __forceinline__ void store(const Params &P, const Geometry &, const Pos &pos, State<V> &S) {
        pos.store(P.vs, S.vs);
        pos.store(P.pg_advantages, S.pg);
    }
};
using VtraceEst = VtraceEstT<>;

// ---------------------------------------------------------------------------
// GAE (with the TD(lambda) returns G_t = A_t + V_t) and V-Trace from one pass
// over their common inputs: the two recurrences are scanned together as one
// pair, x = (A, D) with D = vs - V.  Both share delta_t = r_t + gamma boot_t -
// V_t; GAE's a_t = gamma lambda, b_t = delta_t; V-Trace's a_t = gamma c_t,
// b_t = rho_t delta_t (rho, c from the V-Trace lambda, rho_bar, c_bar).  Each
// component's arithmetic is that of GaeEstT and VtraceEst, in the same order.
// ---------------------------------------------------------------------------
struct GaeVtraceEst {
    static constexpr bool kBackward = true;
    using AT = float2;
    using BT = float2;
    struct Params {
        const float *log_rhos, *rewards, *values, *terminateds, *truncateds, *bootstrap_values, *last_values;
        float *advantages, *returns, *vs, *pg_advantages; // returns may be null
        float gamma, lambda_, vtrace_lambda, rho_bar, c_bar;
    };
    template <int V>
    struct State {
        float lr[V], r[V], v[V], te[V], tr[V], bv[V];
        float rho[V];
        float adv[V], ret[V], vs[V], pg[V];
        float v_next;
        unsigned chained; // bit k: the traces go on to t+1 inside the row
    };
    static __device__ __forceinline__ void prefetch(const Params &P, const Geometry &g, long long tile0, int S) {
        prefetch_planes(g, tile0, S, P.log_rhos, P.rewards, P.values, P.terminateds, P.truncateds,
                        P.bootstrap_values);
    }
    static constexpr int kInputPlanes = 6;
    static __host__ __device__ __forceinline__ PlaneRef input_plane(const Params &P, int i) {
        const float *p[6] = {P.log_rhos, P.rewards, P.values, P.terminateds, P.truncateds, P.bootstrap_values};
        return {i < 6 ? p[i] : nullptr, 4};
    }
    template <int NT, int V, class Pos>
    static __device__ __forceinline__ void load(const Params &P, const Geometry &g, const Pos &pos,
                                                State<V> &S, unsigned char *) {
        const float h_v_next = pos.fetch_next(P.values);
        pos.load(P.log_rhos, S.lr);
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
                                                  float2 (&a)[V], float2 (&b)[V]) {
        const float gl = P.gamma * P.lambda_;
        S.chained = 0u;
#pragma unroll
        for (int k = 0; k < V; ++k) {
            if (elem_valid<kFast, V>(rm, k)) {
                const StepFlags f = step_flags<kTrunc>(S.te[k], S.tr[k]);
                const bool rowend = elem_row_end<kFast, V>(rm, k);
                const float ratio = __expf(S.lr[k]);
                const float rho = fminf(P.rho_bar, ratio);
                const float c = P.vtrace_lambda * fminf(P.c_bar, ratio);
                float boot;
                if (f.cont) {
                    boot = rowend ? row_last_value(P.last_values, elem_row<kFast>(rm, k), g.rows)
                                  : ((k + 1 < V) ? S.v[k + 1] : S.v_next);
                } else {
                    boot = f.trn ? S.bv[k] : 0.0f;
                }
                const bool go = f.cont && !rowend;
                const float delta = fmaf(P.gamma, boot, S.r[k]) - S.v[k];
                a[k] = make_float2(go ? gl : 0.0f, go ? P.gamma * c : 0.0f);
                b[k] = make_float2(delta, rho * delta);
                S.rho[k] = rho;
                if (go) S.chained |= (1u << k);
            } else {
                a[k] = make_float2(1.0f, 1.0f);
                b[k] = make_float2(0.0f, 0.0f);
                S.rho[k] = 0.0f;
            }
        }
    }
    template <int V, int kCase = kCaseAny, class Pos>
    static __device__ __forceinline__ void coeffs(const Params &P, const Geometry &g, const Pos &pos,
                                                  const RowMasks &rm, State<V> &S, float2 (&a)[V],
                                                  float2 (&b)[V]) {
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
    // as VtraceEst: pg_t = b_t + rho_t gamma D_{t+1} where the trace goes on
    template <int V>
    static __device__ __forceinline__ void out(const Params &P, State<V> &S, int k, float2 x, float2 x_next,
                                               float2 b_k) {
        S.adv[k] = x.x;
        S.ret[k] = x.x + S.v[k];
        S.vs[k] = S.v[k] + x.y;
        S.pg[k] = ((S.chained >> k) & 1u) ? fmaf(S.rho[k] * P.gamma, x_next.y, b_k.y) : b_k.y;
    }
    template <int V, class Pos>
    static __device__ __forceinline__ void store(const Params &P, const Geometry &, const Pos &pos, State<V> &S) {
        pos.store(P.advantages, S.adv);
        if (P.returns != nullptr) pos.store(P.returns, S.ret);
        pos.store(P.vs, S.vs);
        pos.store(P.pg_advantages, S.pg);
    }
};

// ---------------------------------------------------------------------------
// Retrace(lambda): x = Q_ret - q,  a_t = gamma c_{t+1}, b_t = delta_t, with
// the expected next-state value V'_t = next_q_values_all[t] (one action, or
// the plane expected_value_kernel writes for several).
// ---------------------------------------------------------------------------
// NqT: the element type of the V' plane (ValT for a single action; fp32 for
// the plane expected_value_kernel writes for several).
template <class ValT = float, class FlagT = float, class NqT = ValT>
struct RetraceEstT {
    static constexpr bool kBackward = true;
    using AT = float;
    using BT = float;
    struct Params {
        const ValT *rewards, *q_values;
        const NqT *next_q_values_all;
        const ValT *log_rhos;
        const FlagT *terminateds, *truncateds;
        float *q_ret;
        float gamma, lambda_, c_bar;
    };
    template <int V>
    struct State {
        float r[V], q[V], vnext[V], lr[V], out[V];
        FlagReg<FlagT> te[V], tr[V];
        float lr_next;
    };

    static __device__ __forceinline__ void prefetch(const Params &P, const Geometry &g, long long tile0, int S) {
        prefetch_planes(g, tile0, S, P.rewards, P.q_values, P.log_rhos, P.terminateds, P.truncateds,
                        P.next_q_values_all);
    }
    static constexpr int kInputPlanes = 6;
    static __host__ __device__ __forceinline__ PlaneRef input_plane(const Params &P, int i) {
        switch (i) {
        case 0: return {P.rewards, (int)sizeof(ValT)};
        case 1: return {P.q_values, (int)sizeof(ValT)};
        case 2: return {P.log_rhos, (int)sizeof(ValT)};
        case 3: return {P.terminateds, (int)sizeof(FlagT)};
        case 4: return {P.truncateds, (int)sizeof(FlagT)};
        case 5: return {P.next_q_values_all, (int)sizeof(NqT)};
        default: return {nullptr, 0};
        }
    }
    template <int NT, int V, class Pos>
    static __device__ __forceinline__ void load(const Params &P, const Geometry &g, const Pos &pos,
                                                State<V> &S, unsigned char *) {
        const float h_lr_next = pos.fetch_next(P.log_rhos);
        pos.load_widen(P.rewards, S.r);
        pos.load_widen(P.q_values, S.q);
        pos.load_widen(P.log_rhos, S.lr);
        pos.load_flag(P.terminateds, S.te);
        pos.load_flag(P.truncateds, S.tr);
        S.lr_next = pos.next(S.lr, h_lr_next);
        pos.load_widen(P.next_q_values_all, S.vnext);
    }
    template <int V, bool kFast, class Pos>
    static __device__ __forceinline__ void coeffs_impl(const Params &P, const Geometry &g, const Pos &pos,
                                                  const RowMasks &rm, State<V> &S,
                                                  float (&a)[V], float (&b)[V]) {
#pragma unroll
        for (int k = 0; k < V; ++k) {
            if (elem_valid<kFast, V>(rm, k)) {
                const StepFlags f = step_flags(S.te[k], S.tr[k]);
                const bool rowend = elem_row_end<kFast, V>(rm, k);
                const float boot = f.term ? 0.0f : S.vnext[k];
                b[k] = fmaf(P.gamma, boot, S.r[k]) - S.q[k];
                if (f.cont && !rowend) {
                    const float lr1 = (k + 1 < V) ? S.lr[k + 1] : S.lr_next;
                    a[k] = P.gamma * (P.lambda_ * fminf(P.c_bar, __expf(lr1)));
                } else {
                    a[k] = 0.0f;
                }
            } else {
                a[k] = 1.0f;
                b[k] = 0.0f;
            }
        }
    }
    template <int V, int kCase = kCaseAny, class Pos>
    static __device__ __forceinline__ void coeffs(const Params &P, const Geometry &g, const Pos &pos,
                                                  const RowMasks &rm, State<V> &S, float (&a)[V],
                                                  float (&b)[V]) {
        if constexpr (kCase != kCaseAny) coeffs_impl<V, true>(P, g, pos, rm, S, a, b);
        else if (rm.fast) coeffs_impl<V, true>(P, g, pos, rm, S, a, b);
        else coeffs_impl<V, false>(P, g, pos, rm, S, a, b);
    }
    template <int V>
    static __device__ __forceinline__ void out(const Params &, State<V> &S, int k, float x, float, float) {
        S.out[k] = S.q[k] + x;
    }
    template <int V, class Pos>
    static __device__ __forceinline__ void store(const Params &P, const Geometry &, const Pos &pos, State<V> &S) {
        pos.store(P.q_ret, S.out);
    }
};
using RetraceEst = RetraceEstT<>;

// ---------------------------------------------------------------------------
// Forward estimators.  Eligibility traces: x = e, a_t = gamma lambda,
// b_t = x_t.  fp32 prefix sum: the same with a_t = 1.  Flags are widened to
// 0 / 1 floats (the halo flag comes from the neighbouring lane).
// ---------------------------------------------------------------------------
template <class ValT = float, class FlagT = float>
struct ForwardEstT {
    static constexpr bool kBackward = false;
    using AT = float;
    using BT = float;
    struct Params {
        const ValT *x;
        const FlagT *dones;
        float *out;
        float decay;       // gamma lambda, or 1
        int reset_on_flag; // 0: dones[t-1] != 0 resets at t; 1: dones[t] != 0 resets at t
    };
    template <int V>
    struct State {
        float x[V], d[V], out[V];
        float d_prev;
    };
    static __device__ __forceinline__ void prefetch(const Params &P, const Geometry &g, long long tile0, int S) {
        prefetch_planes(g, tile0, S, P.x, P.dones);
    }
    static constexpr int kInputPlanes = 2;
    static __host__ __device__ __forceinline__ PlaneRef input_plane(const Params &P, int i) {
        switch (i) {
        case 0: return {P.x, (int)sizeof(ValT)};
        case 1: return {P.dones, (int)sizeof(FlagT)};
        default: return {nullptr, 0};
        }
    }
    template <int NT, int V, class Pos>
    static __device__ __forceinline__ void load(const Params &P, const Geometry &g, const Pos &pos,
                                                State<V> &S, unsigned char *) {
        const float h_d_prev = pos.fetch_prev(P.dones);
        pos.load_widen(P.x, S.x);
        pos.load_widen(P.dones, S.d);
        S.d_prev = pos.prev(S.d, h_d_prev);
    }
    template <int V, bool kFast, class Pos>
    static __device__ __forceinline__ void coeffs_impl(const Params &P, const Geometry &g, const Pos &pos,
                                                  const RowMasks &rm, State<V> &S,
                                                  float (&a)[V], float (&b)[V]) {
#pragma unroll
        for (int k = 0; k < V; ++k) {
            if (elem_valid<kFast, V>(rm, k)) {
                const float dp = P.reset_on_flag ? S.d[k] : ((k > 0) ? S.d[k - 1] : S.d_prev);
                a[k] = (elem_row_start<kFast, V>(rm, k) || dp != 0.0f) ? 0.0f : P.decay;
                b[k] = S.x[k];
            } else {
                a[k] = 1.0f;
                b[k] = 0.0f;
            }
        }
    }
    template <int V, int kCase = kCaseAny, class Pos>
    static __device__ __forceinline__ void coeffs(const Params &P, const Geometry &g, const Pos &pos,
                                                  const RowMasks &rm, State<V> &S, float (&a)[V],
                                                  float (&b)[V]) {
        if constexpr (kCase != kCaseAny) coeffs_impl<V, true>(P, g, pos, rm, S, a, b);
        else if (rm.fast) coeffs_impl<V, true>(P, g, pos, rm, S, a, b);
        else coeffs_impl<V, false>(P, g, pos, rm, S, a, b);
    }
    template <int V>
    static __device__ __forceinline__ void out(const Params &, State<V> &S, int k, float x, float, float) {
        S.out[k] = x;
    }
    template <int V, class Pos>
    static __device__ __forceinline__ void store(const Params &P, const Geometry &, const Pos &pos, State<V> &S) {
        pos.store(P.out, S.out);
    }
};
using TracesEst = ForwardEstT<>;
using PrefixF32Est = TracesEst; // a trace with decay 1

// int32 episodic prefix sum: a in {0, 1}, exact wrapping sums.
template <class FlagT = float>
struct PrefixI32EstT {
    static constexpr bool kBackward = false;
    using AT = uint32_t;
    using BT = int32_t;
    struct Params {
        const int32_t *x;
        const FlagT *dones;
        int32_t *out;
        int reset_on_flag; // as ForwardEstT
    };
    template <int V>
    struct State {
        int32_t x[V], out[V];
        float d[V];
        float d_prev;
    };
    static __device__ __forceinline__ void prefetch(const Params &P, const Geometry &g, long long tile0, int S) {
        prefetch_planes(g, tile0, S, P.x, P.dones);
    }
    static constexpr int kInputPlanes = 2;
    static __host__ __device__ __forceinline__ PlaneRef input_plane(const Params &P, int i) {
        switch (i) {
        case 0: return {P.x, 4};
        case 1: return {P.dones, (int)sizeof(FlagT)};
        default: return {nullptr, 0};
        }
    }
    template <int NT, int V, class Pos>
    static __device__ __forceinline__ void load(const Params &P, const Geometry &g, const Pos &pos,
                                                State<V> &S, unsigned char *) {
        const float h_d_prev = pos.fetch_prev(P.dones);
        pos.load(P.x, S.x);
        pos.load_widen(P.dones, S.d);
        S.d_prev = pos.prev(S.d, h_d_prev);
    }
    template <int V, bool kFast, class Pos>
    static __device__ __forceinline__ void coeffs_impl(const Params &P, const Geometry &g, const Pos &pos,
                                                  const RowMasks &rm, State<V> &S,
                                                  uint32_t (&a)[V], int32_t (&b)[V]) {
#pragma unroll
        for (int k = 0; k < V; ++k) {
            if (elem_valid<kFast, V>(rm, k)) {
                const float dp = P.reset_on_flag ? S.d[k] : ((k > 0) ? S.d[k - 1] : S.d_prev);
                a[k] = (elem_row_start<kFast, V>(rm, k) || dp != 0.0f) ? 0u : 1u;
                b[k] = S.x[k];
            } else {
                a[k] = 1u;
                b[k] = 0;
            }
        }
    }
    template <int V, int kCase = kCaseAny, class Pos>
    static __device__ __forceinline__ void coeffs(const Params &P, const Geometry &g, const Pos &pos,
                                                  const RowMasks &rm, State<V> &S, uint32_t (&a)[V],
                                                  int32_t (&b)[V]) {
        if constexpr (kCase != kCaseAny) coeffs_impl<V, true>(P, g, pos, rm, S, a, b);
        else if (rm.fast) coeffs_impl<V, true>(P, g, pos, rm, S, a, b);
        else coeffs_impl<V, false>(P, g, pos, rm, S, a, b);
    }
    template <int V>
    static __device__ __forceinline__ void out(const Params &, State<V> &S, int k, int32_t x, int32_t, int32_t) {
        S.out[k] = x;
    }
    template <int V, class Pos>
    static __device__ __forceinline__ void store(const Params &P, const Geometry &, const Pos &pos, State<V> &S) {
        pos.store(P.out, S.out);
    }
};
using PrefixI32Est = PrefixI32EstT<>;

} // namespace rlscan
