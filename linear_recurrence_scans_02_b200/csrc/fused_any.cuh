// fused_any.cuh - one tile body for every fp32 estimator, for batch requests
// that mix several estimators in one launch.
//
// A fused launch whose blocks run different estimators shares each SM among
// their code; with one fully unrolled body per estimator the warps then
// stall on instruction fetch.  This body computes every fp32 estimator of
// the rl-triton README "Kernels" table (GAE, GAE + TD(lambda) returns,
// V-Trace, single-action Retrace, TD(lambda) returns, discounted returns,
// eligibility traces, the fp32 episodic prefix sum) from one instruction
// stream: the coefficient builder of each estimator is an instance of
//
//   a_t = chain_t * gamma * (lambda * cf_t)
//   b_t = rho_t * (r_t + gamma * boot_t - [V_t])          (backward)
//   b_t = x_t                                             (forward)
//
// with per-call constants and uniform (per block) branches choosing the
// terms: cf_t = min(c_bar, ratio) for V-Trace (own ratio) and Retrace (the
// next step's ratio), else 1; rho_t = min(rho_bar, ratio) for V-Trace, else
// 1; boot_t = the next value weighted by w_nv inside an episode (1 for GAE
// and V-Trace, 1 - lambda for TD(lambda), 0 for discounted returns), the
// row's last value at a row end, the bootstrap value at a truncation, 0 at a
// termination; Retrace's boot is next_q_values_all unless terminated.  The
// arithmetic of each term is the estimator's own builder's (estimators.cuh),
// in the same order, so results equal that estimator's tile kernel bit for
// bit on the same tiles.
//
// Forward recurrences (traces, prefix sum) run through the same backward
// scan on mirrored positions: warp w, lane l serves the chunk (NW-1-w, 31-l)
// of the tile and holds its V elements in reverse, so "the element before
// in scan order" is always register j+1, or register 0 of lane l+1, as for
// a backward recurrence; the warp and block scans then combine exactly the
// pairs the forward scan would, in the same association.
//
// Only calls whose rows are whole multiples of V (T >= V, V | T) and fit a
// tile take this body: every thread then holds V elements of one row, of
// which only register V-1 (scan order's first) can start a row.
#pragma once

#include "estimators.cuh"

namespace rlscan {

// Per-call switches of the shared body.
enum AnyFlags : unsigned {
    kAnyFwd = 1u << 0,          // forward recurrence (mirrored positions)
    kAnyResetOnFlag = 1u << 1,  // forward: dones[t] != 0 resets at t (else dones[t-1])
    kAnyRatioOwn = 1u << 2,     // V-Trace: rho_t, c_t from exp(log_rho_t)
    kAnyRatioNext = 1u << 3,    // Retrace: c_{t+1} from exp(log_rho_{t+1})
    kAnySubV = 1u << 4,         // b_t -= V_t (GAE, V-Trace, Retrace: q_t)
    kAnyRetraceBoot = 1u << 5,  // boot_t = terminated ? 0 : next_q_values_all_t
    kAnyOut0PlusV = 1u << 6,    // out0 = x + V (V-Trace vs, Retrace q_ret)
    kAnyOut1PlusV = 1u << 7,    // out1 = x + V (the TD(lambda) returns beside GAE)
    kAnyOut1Pg = 1u << 8,       // out1 = V-Trace policy-gradient advantage
};
// Which plane gives the halo (the input of the element before in scan order).
enum AnyHalo : int { kAnyHaloNone = 0, kAnyHaloV = 1, kAnyHaloLogRho = 2, kAnyHaloDone = 3 };

struct AnyParams {
    const float *r;   // rewards (forward: x)
    const float *v;   // values (Retrace: q_values)
    const float *f;   // terminateds (forward: dones)
    const float *tr;  // truncateds (null: none)
    const float *lr;  // log importance ratios (V-Trace, Retrace)
    const float *nq;  // Retrace: next_q_values_all
    const float *bv;  // bootstrap values, read where truncated
    const float *lv;  // last values [E] (null: 0)
    float *out0, *out1;
    float gamma, lam, rho_bar, c_bar, w_nv;
    int halo;       // AnyHalo
    unsigned flags; // AnyFlags
};

constexpr int kAnyNT = 128;

template <int V>
__device__ __forceinline__ void reverse_regs(float (&o)[V]) {
#pragma unroll
    for (int j = 0; j < V / 2; ++j) {
        const float t = o[j];
        o[j] = o[V - 1 - j];
        o[V - 1 - j] = t;
    }
}

// One tile of one call.  mode: kModeWarp (every warp holds whole rows) or
// kModeBlock (rows span warps of the tile).
template <int V>
__device__ __forceinline__ void any_tile_body(const AnyParams &P, const Geometry &g, const long long block,
                                              const int mode) {
    constexpr int NT = kAnyNT;
    constexpr int NW = NT / 32;
    __shared__ float s_wa[NW], s_wb[NW], s_wx[NW];

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const unsigned fl = P.flags;
    const bool fwd = (fl & kAnyFwd) != 0;
    const long long tile0 = block * (long long)(NT * V);

    // L2 prefetch of this tile's planes before the grid wait (one plane per
    // thread of the first six)
    {
        const long long left = g.n - tile0;
        const long long cnt = left < NT * V ? left : NT * V;
        const float *pl = nullptr;
        switch (tid) {
        case 0: pl = P.r; break;
        case 1: pl = P.v; break;
        case 2: pl = P.f; break;
        case 3: pl = P.tr; break;
        case 4: pl = P.lr; break;
        case 5: pl = P.nq; break;
        default: break;
        }
        prefetch_l2(pl, tile0, cnt, 4);
    }
    griddep_wait();
    griddep_launch_dependents();

    const int slot = fwd ? ((NW - 1 - warp) * 32 + (31 - lane)) : tid;
    const long long i0 = tile0 + (long long)slot * V;
    const bool valid = i0 < g.n; // n is a multiple of V: a thread has all V elements or none
    const bool vec = valid && g.vec_ok != 0;

    float r[V], v[V], f[V], tr[V], lr[V], nq[V];
    // the halo element: memory index i0 + V (backward) or i0 - 1 (forward)
    const float *hp = P.halo == kAnyHaloV ? P.v : (P.halo == kAnyHaloLogRho ? P.lr : (P.halo == kAnyHaloDone ? P.f : nullptr));
    const float fetched = (lane == 31 && valid) ? load_one(hp, fwd ? i0 - 1 : i0 + V, g.n) : 0.0f;
    load_plane<V>(P.r, i0, g.n, vec, r);
    load_plane<V>(P.v, i0, g.n, vec, v);
    load_plane<V>(P.f, i0, g.n, vec, f);
    load_plane<V>(P.tr, i0, g.n, vec, tr);
    load_plane<V>(P.lr, i0, g.n, vec, lr);
    load_plane<V>(P.nq, i0, g.n, vec, nq);
    if (fwd) { // forward calls only read x and dones
        reverse_regs<V>(r);
        reverse_regs<V>(f);
    }
    // h[j]: the halo plane in scan space; hn(j) = h[j + 1], or the next
    // lane's h[0], or (lane 31) the fetched element
    float h0;
    if (P.halo == kAnyHaloV) h0 = v[0];
    else if (P.halo == kAnyHaloLogRho) h0 = lr[0];
    else h0 = f[0];
    const float hs = __shfl_down_sync(kFullMask, h0, 1);
    const float h_last = lane == 31 ? fetched : hs;

    // row position: only register V-1 (scan order's first) can start a row
    long long row, t0;
    if (g.t_shift >= 0) {
        row = i0 >> g.t_shift;
        t0 = i0 & (g.seq_len - 1);
    } else {
        row = i0 / g.seq_len;
        t0 = i0 - row * g.seq_len;
    }
    const bool first = valid && (fwd ? (t0 == 0) : (t0 + V == g.seq_len));

    float a[V], b[V], rho[V];
    unsigned chained = 0u;
    const bool has_tr = P.tr != nullptr;
#pragma unroll
    for (int j = 0; j < V; ++j) {
        float hn;
        if (j + 1 < V) {
            if (P.halo == kAnyHaloV) hn = v[j + 1];
            else if (P.halo == kAnyHaloLogRho) hn = lr[j + 1];
            else hn = f[j + 1];
        } else {
            hn = h_last;
        }
        if (P.halo == kAnyHaloNone) hn = 0.0f;
        const bool is_first = (j == V - 1) && first;
        bool cont, trn = false, term = false;
        if (fwd) {
            const float d = (fl & kAnyResetOnFlag) ? f[j] : hn;
            cont = d == 0.0f;
        } else {
            term = f[j] != 0.0f;
            trn = has_tr && tr[j] != 0.0f && !term;
            cont = !term && !trn;
        }
        const bool chain = valid && cont && !is_first;
        float cf = 1.0f, rh = 1.0f;
        if (fl & kAnyRatioOwn) {
            const float ratio = __expf(lr[j]);
            rh = fminf(P.rho_bar, ratio);
            cf = fminf(P.c_bar, ratio);
        }
        if ((fl & kAnyRatioNext) && chain) cf = fminf(P.c_bar, __expf(hn));
        rho[j] = rh;
        if (!valid) {
            a[j] = 1.0f;
            b[j] = 0.0f;
            continue;
        }
        a[j] = chain ? P.gamma * (P.lam * cf) : 0.0f;
        if (fwd) {
            b[j] = r[j];
        } else {
            float boot;
            if (fl & kAnyRetraceBoot) {
                boot = term ? 0.0f : nq[j];
            } else if (cont) {
                boot = is_first ? row_last_value(P.lv, row, g.rows) : P.w_nv * hn;
            } else {
                boot = trn ? load_one(P.bv, i0 + j, g.n) : 0.0f;
            }
            float bb = fmaf(P.gamma, boot, r[j]);
            if (fl & kAnySubV) bb = bb - v[j];
            if (fl & kAnyRatioOwn) bb = rh * bb;
            b[j] = bb;
        }
        if (chain) chained |= 1u << j;
    }

    // thread aggregate, composed in scan order (register V-1 first)
    float ta = a[V - 1], tb = b[V - 1];
#pragma unroll
    for (int k = V - 2; k >= 0; --k) {
        float na = a[k], nb = b[k];
        combine(na, nb, ta, tb);
        ta = na;
        tb = nb;
    }
    float ia = ta, ib = tb;
    const bool warp_local = mode == kModeWarp;
    warp_inclusive_scan<true>(ia, ib, lane, warp_local ? g.scan_lanes : 32);
    float ea, eb;
    warp_exclusive_from_inclusive<true>(ia, ib, lane, ea, eb);
    float x;
    if (warp_local) {
        x = apply_pair(ea, eb, 0.0f);
    } else {
        if (lane == 0) {
            s_wa[warp] = ia;
            s_wb[warp] = ib;
        }
        __syncthreads();
        if (warp == 0) {
            float wa = lane < NW ? s_wa[lane] : 1.0f;
            float wb = lane < NW ? s_wb[lane] : 0.0f;
            warp_inclusive_scan<true>(wa, wb, lane);
            float wea, web;
            warp_exclusive_from_inclusive<true>(wa, wb, lane, wea, web);
            if (lane < NW) s_wx[lane] = apply_pair(wea, web, 0.0f);
        }
        __syncthreads();
        x = apply_pair(ea, eb, s_wx[warp]);
    }

    // epilogue in scan order
    float o0[V], o1[V];
#pragma unroll
    for (int j = V - 1; j >= 0; --j) {
        const float prev = x;
        x = apply_pair(a[j], b[j], x);
        o0[j] = (fl & kAnyOut0PlusV) ? v[j] + x : x;
        if (fl & kAnyOut1PlusV) o1[j] = x + v[j];
        else if (fl & kAnyOut1Pg) o1[j] = ((chained >> j) & 1u) ? fmaf(rho[j] * P.gamma, prev, b[j]) : b[j];
        else o1[j] = 0.0f;
    }
    if (!valid) return;
    if (fwd) reverse_regs<V>(o0);
    store_plane<V>(P.out0, i0, g.n, vec, o0);
    if (P.out1 != nullptr) store_plane<V>(P.out1, i0, g.n, vec, o1);
}

} // namespace rlscan
