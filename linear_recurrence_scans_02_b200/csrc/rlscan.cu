// rlscan.cu - host side of librlscan: argument checks, launch planning and
// the extern "C" entry points declared in include/rlscan.h.
//
// Each entry point validates its arguments on the host (nothing touches the
// GPU before the launch), picks a tile plan for the [E, T] shape (or the
// env-group plan of the time-major layout), and launches one kernel
// instantiation on the caller's stream with programmatic dependent launch
// allowed, so the kernel's prologue can overlap the tail of whatever ran
// before it on that stream.  rlscan_batch runs the same checks for several
// calls and launches the fusable ones as one kernel.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>
#include <cstdarg>
#include <climits>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <initializer_list>
#include <string>

#include "../../include/rlscan.h"
#include "batch.cuh"

namespace rlscan {
namespace {

thread_local std::string g_last_error;

int fail(int code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

int ok() {
    g_last_error.clear();
    return RLSCAN_OK;
}

// About a second of polling (each poll sleeps up to ~1 us).
constexpr unsigned kDefaultSpinLimit = 1u << 20;
std::atomic<unsigned> g_spin_limit{kDefaultSpinLimit};
std::atomic<long long> g_withhold{-1};

bool pdl_enabled() {
    static const bool on = [] {
        const char *v = std::getenv("RLSCAN_DISABLE_PDL");
        return !(v && v[0] && v[0] != '0');
    }();
    return on;
}

// ---------------------------------------------------------------------------
// Tile plans.  A tile is S = NT * V consecutive elements of the flattened
// [E*T] array.  Tiles need the look-back only when a tile boundary can fall
// inside a row (S not a multiple of T, more than one tile).
// ---------------------------------------------------------------------------
// Eight elements per thread keeps a grid's share of each SM small, so the
// next launch on the stream can be resident (and prefetching) while this one
// runs; the 512-element tile (four per thread) is for small look-back plans.
enum Cfg { C512 = 0, C1024, C2048, C4096, R512, R256, R128, kNumCfg };
constexpr int kCfgTile[kNumCfg] = {512, 1024, 2048, 4096, 512, 256, 128};
constexpr int kCfgThreads[kNumCfg] = {128, 128, 256, 512, 128, 64, 32};

struct Plan {
    Cfg cfg;
    bool lookback;
    long long ntiles;
    int mode; // kModeBlock / kModeLookback / kModeWarp
};

// Scan mode of a plan: look-back when rows span tiles; warp-local when
// every warp's 32*V elements hold whole rows; otherwise a block scan.
Plan with_mode(Plan p, long long T) {
    const long long warp_elems = 32ll * (kCfgTile[p.cfg] / kCfgThreads[p.cfg]);
    p.mode = p.lookback ? kModeLookback : ((warp_elems % T == 0) ? kModeWarp : kModeBlock);
    return p;
}

// SM count of the current device (queried once per device; B200's 148 when
// no device can be asked, e.g. when a plan is computed on a host without a
// GPU).  Plans fill the GPU: with fewer tiles than two per SM a plan prefers
// smaller tiles.
constexpr long long kDefaultSMs = 148;
constexpr int kMaxPlanDevices = 256;
std::atomic<int> g_sm_count[kMaxPlanDevices];

long long num_sms() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxPlanDevices) {
        (void)cudaGetLastError();
        return kDefaultSMs;
    }
    int v = g_sm_count[dev].load(std::memory_order_relaxed);
    if (v <= 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
            (void)cudaGetLastError();
            return kDefaultSMs;
        }
        g_sm_count[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

long long ceil_div(long long a, long long b) { return (a + b - 1) / b; }

int pow2_shift(long long T) {
    if (T <= 0 || (T & (T - 1)) != 0) return -1;
    int s = 0;
    while ((1ll << s) < T) ++s;
    return s;
}

Plan make_plan_tiles(long long E, long long T, long long actions) {
    const long long n = E * T;
    Plan p{};
    if (actions > 1) {
        p.cfg = actions <= 24 ? R512 : (actions <= 48 ? R256 : R128);
        const long long S = kCfgTile[p.cfg];
        p.ntiles = ceil_div(n, S);
        p.lookback = p.ntiles > 1 && (S % T) != 0;
        return p;
    }
    // Small CTAs (128 threads x 8 elements) overlap best, both with each
    // other inside a launch and with the neighbouring launches; larger tiles
    // only where a row needs them to stay inside one tile.
    const long long sms = num_sms();
    const long long min_tiles = 2 * sms;
    const Cfg whole_rows[3] = {C1024, C2048, C4096};
    for (Cfg c : whole_rows) {
        const long long S = kCfgTile[c];
        if (S % T != 0) continue;
        const long long nt = ceil_div(n, S);
        const long long nt_split = ceil_div(n, kCfgTile[C1024]);
        // whole rows, unless that leaves SMs idle while split rows would not
        if (nt >= sms || nt_split <= nt) {
            p.cfg = c;
            p.ntiles = nt;
            p.lookback = false;
            return p;
        }
        break;
    }
    // rows span tiles (long or odd-length rows, or too few rows to fill the
    // GPU): look-back over 2048-element tiles (fewer tiles per row, so a
    // shorter chain of carries), 1024 or 512 when that gives too few tiles
    p.cfg = ceil_div(n, kCfgTile[C2048]) >= min_tiles
                ? C2048
                : (ceil_div(n, kCfgTile[C1024]) >= min_tiles ? C1024 : C512);
    p.ntiles = ceil_div(n, kCfgTile[p.cfg]);
    p.lookback = p.ntiles > 1 && (kCfgTile[p.cfg] % T != 0);
    return p;
}

Plan make_plan(long long E, long long T, long long actions) { return with_mode(make_plan_tiles(E, T, actions), T); }

// Warp-local mode: a row spans T / V lanes (T a power of two dividing 32 V);
// the shuffle scan needs to reach that far only.
int scan_lanes_for(const Plan &p, long long T) {
    if (p.mode != kModeWarp) return 32;
    const long long V = kCfgTile[p.cfg] / kCfgThreads[p.cfg];
    const long long lanes = T >= V ? T / V : 1;
    return (int)(lanes < 32 ? lanes : 32);
}

// True when every given pointer is NULL or 16-byte aligned.
bool aligned16(std::initializer_list<const void *> ptrs) {
    for (const void *p : ptrs)
        if (p != nullptr && ((uintptr_t)p & 15u) != 0) return false;
    return true;
}

size_t workspace_for(const Plan &p) {
    return p.lookback ? sizeof(WsHeader) + sizeof(TileSlot) * (size_t)p.ntiles : 0;
}

size_t multi_smem_bytes(Cfg cfg, long long actions) {
    const size_t S = (size_t)kCfgTile[cfg];
    return 128 + (2 * S * (size_t)actions + S) * sizeof(float);
}

// ---------------------------------------------------------------------------
// Argument checks
// ---------------------------------------------------------------------------
constexpr long long kMaxElems = 1ll << 40;

int check_shape(long long E, long long T, long long A = 1) {
    if (E < 0 || T < 0) return fail(RLSCAN_ERR_INVALID_ARG, "E and T must be >= 0 (got E=%lld, T=%lld)", E, T);
    if (E > 0 && T > 0 && (E > kMaxElems / T || E * T > kMaxElems / (A > 0 ? A : 1)))
        return fail(RLSCAN_ERR_INVALID_ARG, "E*T*A too large (E=%lld, T=%lld, A=%lld)", E, T, A);
    if (E > 0 && T > 0 && ceil_div(E * T, 128) >= (1ll << 31) - 1)
        return fail(RLSCAN_ERR_INVALID_ARG, "E*T too large for one launch");
    return RLSCAN_OK;
}

int check_scalar(float v, const char *name) {
    if (!std::isfinite(v)) return fail(RLSCAN_ERR_INVALID_ARG, "%s must be finite", name);
    return RLSCAN_OK;
}

struct Span {
    const void *p;
    size_t bytes;
    const char *name;
};

bool overlap(const Span &a, const Span &b) {
    if (!a.p || !b.p || a.bytes == 0 || b.bytes == 0) return false;
    const uintptr_t a0 = (uintptr_t)a.p, a1 = a0 + a.bytes;
    const uintptr_t b0 = (uintptr_t)b.p, b1 = b0 + b.bytes;
    return a0 < b1 && b0 < a1;
}

// Every output against every input and every other output.
int check_aliasing(const Span *ins, int nin, const Span *outs, int nout) {
    for (int o = 0; o < nout; ++o) {
        for (int i = 0; i < nin; ++i)
            if (overlap(outs[o], ins[i]))
                return fail(RLSCAN_ERR_INVALID_ARG, "output %s overlaps input %s", outs[o].name, ins[i].name);
        for (int q = o + 1; q < nout; ++q)
            if (overlap(outs[o], outs[q]))
                return fail(RLSCAN_ERR_INVALID_ARG, "outputs %s and %s overlap", outs[o].name, outs[q].name);
    }
    return RLSCAN_OK;
}

int require(const void *p, const char *name) {
    if (p == nullptr) return fail(RLSCAN_ERR_INVALID_ARG, "%s must not be NULL", name);
    return RLSCAN_OK;
}

#define RLSCAN_TRY(expr)                                                                                   \
    do {                                                                                                   \
        int rc_ = (expr);                                                                                  \
        if (rc_ != RLSCAN_OK) return rc_;                                                                  \
    } while (0)

// ---------------------------------------------------------------------------
// Batch requests (rlscan_batch).  While a request is being served on this
// thread, the launch helpers either only validate (dry pass: every call is
// checked before anything is enqueued) or record fusable calls into one
// fused launch and launch the others as usual.
// ---------------------------------------------------------------------------
enum BatchPass { kBatchDry = 1, kBatchRecord = 2 };
struct BatchState {
    int pass;
    FusedBatch fb;
    long long tiles;
    AnyParams any[kFusedMax]; // each fused fp32 call in the shared body's form
    bool has_any[kFusedMax];  // false for calls that body does not take
};
thread_local BatchState *g_batch = nullptr;

bool batch_dry() { return g_batch != nullptr && g_batch->pass == kBatchDry; }

// ---------------------------------------------------------------------------
// Launch
// ---------------------------------------------------------------------------
template <class Est, int NT, int V, int kMode>
cudaError_t launch_one(const typename Est::Params &P, const Geometry &g, const Lookback &lb, size_t smem,
                       cudaStream_t stream, long long grid = -1) {
    auto kern = tile_scan_kernel<Est, NT, V, kMode>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(grid < 0 ? g.ntiles : grid));
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, P, g, lb);
}

template <class Est, Cfg C>
cudaError_t launch_cfg(const typename Est::Params &P, const Geometry &g, const Lookback &lb, int mode,
                       size_t smem, cudaStream_t s, long long grid = -1) {
    constexpr int NT = kCfgThreads[C];
    constexpr int V = kCfgTile[C] / NT;
    // rows that span tiles: the one-pass look-back for multi-action Retrace
    // (re-reading its per-action rows would cost more than waiting), the two
    // passes for every other call (split-row plans use 512- to 2048-element
    // tiles, make_plan_tiles)
    constexpr bool kMultiAction = std::is_same<Est, RetraceEst<true>>::value;
    switch (mode) {
    case kModeLookback:
        if constexpr (kMultiAction) return launch_one<Est, NT, V, kModeLookback>(P, g, lb, smem, s);
        return cudaErrorInvalidConfiguration;
    case kModeWarp: return launch_one<Est, NT, V, kModeWarp>(P, g, lb, smem, s);
    case kModeReduce:
    case kModeCarry:
        if constexpr (!kMultiAction && (C == C512 || C == C1024 || C == C2048)) {
            if (mode == kModeReduce) return launch_one<Est, NT, V, kModeReduce>(P, g, lb, smem, s, grid);
            return launch_one<Est, NT, V, kModeCarry>(P, g, lb, smem, s, grid);
        }
        return cudaErrorInvalidConfiguration;
    default: return launch_one<Est, NT, V, kModeBlock>(P, g, lb, smem, s);
    }
}

// Input bytes per tile a two-pass wave may hold so that pass two re-reads
// them from L2: a wave's pass one streams them from HBM, pass two finds them
// in L2 (B200: 126 MB).
constexpr long long kTwoPassWaveBytes = 64ll << 20;

// Rows that span tiles, single-action calls: pass one (aggregates) and pass
// two (scan with carries) over waves of consecutive scan-order tiles.
template <class Est>
int run_two_pass(const char *name, const typename Est::Params &P, const Geometry &g, Lookback lb, Cfg cfg,
                 cudaStream_t stream) {
    const long long tile_bytes = (long long)kCfgTile[cfg] * 4 * Est::kInputPlanes;
    const long long wave = std::max<long long>(1, kTwoPassWaveBytes / tile_bytes);
    for (long long t0 = 0; t0 < g.ntiles; t0 += wave) {
        lb.tile_base = t0;
        const long long cnt = std::min<long long>(wave, g.ntiles - t0);
        for (int mode : {kModeReduce, kModeCarry}) {
            cudaError_t e;
            switch (cfg) {
            case C512: e = launch_cfg<Est, C512>(P, g, lb, mode, 0, stream, cnt); break;
            case C1024: e = launch_cfg<Est, C1024>(P, g, lb, mode, 0, stream, cnt); break;
            case C2048: e = launch_cfg<Est, C2048>(P, g, lb, mode, 0, stream, cnt); break;
            default: return fail(RLSCAN_ERR_UNSUPPORTED, "%s: internal plan error", name);
            }
            if (e != cudaSuccess) return fail(RLSCAN_ERR_CUDA, "%s: launch failed: %s", name, cudaGetErrorString(e));
        }
    }
    return ok();
}

template <class Est>
int run(const char *name, const typename Est::Params &P, long long E, long long T, long long actions, void *ws,
        size_t ws_bytes, cudaStream_t stream, bool vec_ok) {
    const Plan plan = make_plan(E, T, actions);
    Geometry g;
    g.n = E * T;
    g.seq_len = T;
    g.ntiles = plan.ntiles;
    g.rows = E;
    g.t_shift = pow2_shift(T);
    g.vec_ok = vec_ok ? 1 : 0;
    g.scan_lanes = scan_lanes_for(plan, T);
    Lookback lb{};
    lb.withhold = -1;
    lb.spin_limit = g_spin_limit.load();
    if (plan.lookback) {
        const size_t need = workspace_for(plan);
        if (ws == nullptr || ws_bytes < need)
            return fail(RLSCAN_ERR_WORKSPACE, "%s: shape E=%lld T=%lld needs a %zu-byte workspace (got %s, %zu bytes)",
                        name, E, T, need, ws ? "a buffer" : "NULL", ws_bytes);
        if (((uintptr_t)ws & 15u) != 0) return fail(RLSCAN_ERR_WORKSPACE, "%s: workspace must be 16-byte aligned", name);
        lb.hdr = static_cast<WsHeader *>(ws);
        lb.slots = reinterpret_cast<TileSlot *>(static_cast<char *>(ws) + sizeof(WsHeader));
        lb.withhold = g_withhold.load();
        lb.row_tiles = (T % kCfgTile[plan.cfg] == 0) ? T / kCfgTile[plan.cfg] : 0;
    }
    if (batch_dry()) return ok();
    if constexpr (FusedKindOf<Est>::value >= 0) {
        // fused when whole rows fit the largest fused tile; the fused launch
        // tiles the call itself (fused_layout, once the request is known)
        constexpr long long kS = (long long)kFusedNT * kFusedVMax;
        if (g_batch != nullptr && actions == 1 && kS % T == 0 && g_batch->fb.n < kFusedMax) {
            static_assert(sizeof(typename Est::Params) <= kFusedParamBytes, "params fit a fused item");
            const int slot = g_batch->fb.n++;
            FusedItem &it = g_batch->fb.item[slot];
            std::memset(it.params, 0, sizeof it.params);
            std::memcpy(it.params, &P, sizeof P);
            it.g = g;
            it.kind = FusedKindOf<Est>::value;
            g_batch->has_any[slot] = to_any(P, g_batch->any[slot]);
            return ok();
        }
    }
    if (plan.lookback && actions == 1) return run_two_pass<Est>(name, P, g, lb, plan.cfg, stream);
    const size_t smem = actions > 1 ? multi_smem_bytes(plan.cfg, actions) : 0;
    cudaError_t e;
    switch (plan.cfg) {
    case C512: e = launch_cfg<Est, C512>(P, g, lb, plan.mode, smem, stream); break;
    case C1024: e = launch_cfg<Est, C1024>(P, g, lb, plan.mode, smem, stream); break;
    case C2048: e = launch_cfg<Est, C2048>(P, g, lb, plan.mode, smem, stream); break;
    case C4096: e = launch_cfg<Est, C4096>(P, g, lb, plan.mode, smem, stream); break;
    default: return fail(RLSCAN_ERR_UNSUPPORTED, "%s: internal plan error", name);
    }
    if (e != cudaSuccess) return fail(RLSCAN_ERR_CUDA, "%s: launch failed: %s", name, cudaGetErrorString(e));
    return ok();
}

// Multi-action Retrace uses its own (smaller) tiles; the register-only
// configurations are never instantiated for it and vice versa.
template <class Est>
int run_multi(const char *name, const typename Est::Params &P, long long E, long long T, long long actions,
              void *ws, size_t ws_bytes, cudaStream_t stream, bool vec_ok) {
    const Plan plan = make_plan(E, T, actions);
    Geometry g;
    g.n = E * T;
    g.seq_len = T;
    g.ntiles = plan.ntiles;
    g.rows = E;
    g.t_shift = pow2_shift(T);
    g.vec_ok = vec_ok ? 1 : 0;
    g.scan_lanes = scan_lanes_for(plan, T);
    Lookback lb{};
    lb.withhold = -1;
    lb.spin_limit = g_spin_limit.load();
    if (plan.lookback) {
        const size_t need = workspace_for(plan);
        if (ws == nullptr || ws_bytes < need)
            return fail(RLSCAN_ERR_WORKSPACE, "%s: shape E=%lld T=%lld A=%lld needs a %zu-byte workspace", name, E, T,
                        actions, need);
        if (((uintptr_t)ws & 15u) != 0) return fail(RLSCAN_ERR_WORKSPACE, "%s: workspace must be 16-byte aligned", name);
        lb.hdr = static_cast<WsHeader *>(ws);
        lb.slots = reinterpret_cast<TileSlot *>(static_cast<char *>(ws) + sizeof(WsHeader));
        lb.withhold = g_withhold.load();
        lb.row_tiles = (T % kCfgTile[plan.cfg] == 0) ? T / kCfgTile[plan.cfg] : 0;
    }
    if (batch_dry()) return ok();
    const size_t smem = multi_smem_bytes(plan.cfg, actions);
    cudaError_t e;
    if (plan.lookback) {
        // the one-pass look-back needs zeroed progress flags; a two-pass call
        // before this one may have left its aggregates in the workspace
        e = cudaMemsetAsync(ws, 0, workspace_for(plan), stream);
        if (e != cudaSuccess) return fail(RLSCAN_ERR_CUDA, "%s: cudaMemsetAsync(workspace): %s", name, cudaGetErrorString(e));
    }
    switch (plan.cfg) {
    case R512: e = launch_cfg<Est, R512>(P, g, lb, plan.mode, smem, stream); break;
    case R256: e = launch_cfg<Est, R256>(P, g, lb, plan.mode, smem, stream); break;
    case R128: e = launch_cfg<Est, R128>(P, g, lb, plan.mode, smem, stream); break;
    default: return fail(RLSCAN_ERR_UNSUPPORTED, "%s: internal plan error", name);
    }
    if (e != cudaSuccess) return fail(RLSCAN_ERR_CUDA, "%s: launch failed: %s", name, cudaGetErrorString(e));
    return ok();
}

size_t plane_bytes(long long E, long long T) { return (size_t)(E * T) * sizeof(float); }

// Option bits of the _ex entry points; `forward` estimators also take
// RLSCAN_OPT_DONE_STARTS_EPISODE.
int check_options(unsigned options, bool forward) {
    const unsigned known = RLSCAN_OPT_TIME_MAJOR | (forward ? RLSCAN_OPT_DONE_STARTS_EPISODE : 0u);
    if (options & ~known)
        return fail(RLSCAN_ERR_INVALID_ARG, "unknown or inapplicable option bits 0x%x", options & ~known);
    return RLSCAN_OK;
}

// Time-major [T, E] launch: a block owns G envs; a warp covers 32 / G
// chunks of kTmV timesteps of each; nw warps make a segment, the block walks
// the rows segment by segment.  No workspace.
constexpr int kTmV = 8;

struct TmPlan {
    int G, nw;
};

// Wider env groups (longer contiguous runs per load) while the grid keeps
// enough blocks: 32-env groups from about four blocks per SM up, 16-env
// groups from about one, else 8; rows of several segments (T > 256) favour
// more, smaller blocks.  Measured at E x T = 1024..65536 x 128, 4096 x 1024
// and 512 x 4096.  The segment covers the row, up to 16 warps.
TmPlan tm_plan(long long E, long long T) {
    TmPlan p;
    const long long kMinBlocks = 120;
    p.G = (E / 32 >= 4 * num_sms() && T <= 256) ? 32 : (E / 16 >= kMinBlocks ? 16 : 8);
    const long long chunks = ceil_div(T, kTmV);
    const long long nw = ceil_div(chunks, 32 / p.G);
    p.nw = (int)(nw < 1 ? 1 : (nw > kTmMaxWarps ? kTmMaxWarps : nw));
    return p;
}

template <class Est>
int run_time_major(const char *name, const typename Est::Params &P, long long E, long long T, cudaStream_t stream) {
    if (E > (long long)INT_MAX / (kTmV + 1))
        return fail(RLSCAN_ERR_UNSUPPORTED, "%s: the time-major layout takes E <= %d", name, INT_MAX / (kTmV + 1));
    if (batch_dry()) return ok();
    const TmPlan tp = tm_plan(E, T);
    Geometry g;
    g.n = E * T;
    g.seq_len = T;
    g.rows = E;
    g.ntiles = ceil_div(T, (long long)tp.nw * (32 / tp.G) * kTmV); // segments per row
    g.t_shift = pow2_shift(T);
    g.vec_ok = 0;
    g.scan_lanes = 32;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ceil_div(E, tp.G));
    cfg.blockDim = dim3(tp.nw * 32);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    cudaError_t e;
    switch (tp.G) {
    case 32: e = cudaLaunchKernelEx(&cfg, time_major_scan_kernel<Est, 32, kTmV>, P, g); break;
    case 16: e = cudaLaunchKernelEx(&cfg, time_major_scan_kernel<Est, 16, kTmV>, P, g); break;
    default: e = cudaLaunchKernelEx(&cfg, time_major_scan_kernel<Est, 8, kTmV>, P, g); break;
    }
    if (e != cudaSuccess) return fail(RLSCAN_ERR_CUDA, "%s: launch failed: %s", name, cudaGetErrorString(e));
    return ok();
}

} // namespace
} // namespace rlscan

// Fixed scratch of rlscan_gae_noalloc: the look-back workspace for callers
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
    if (options & RLSCAN_OPT_TIME_MAJOR) return run_time_major<GaeEst>("rlscan_gae", P, E, T, stream);
    return run<GaeEst>("rlscan_gae", P, E, T, 1, ws, ws_bytes, stream,
                       aligned16({rewards, values, terminateds, truncateds, advantages}));
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
        return run_time_major<GaeReturnsEst>("rlscan_gae_with_returns", P, E, T, stream);
    return run<GaeReturnsEst>("rlscan_gae_with_returns", P, E, T, 1, ws, ws_bytes, stream,
                              aligned16({rewards, values, terminateds, truncateds, advantages, returns}));
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
    const bool vec = aligned16({rewards, values, terminateds, truncateds, advantages, returns});
    const void *bv = truncateds ? bootstrap_values : nullptr;
#define RLSCAN_GAE_TYPED(VT, FT)                                                                                  \
    do {                                                                                                          \
        typename GaeTypedEst<VT, FT>::Params P{static_cast<const VT *>(rewards), static_cast<const VT *>(values), \
                                               static_cast<const FT *>(terminateds),                               \
                                               static_cast<const FT *>(truncateds), static_cast<const VT *>(bv),  \
                                               last_values, advantages, returns, gamma, lambda_};                  \
        if (options & RLSCAN_OPT_TIME_MAJOR)                                                                      \
            return run_time_major<GaeTypedEst<VT, FT>>("rlscan_gae_typed", P, E, T, stream);                     \
        return run<GaeTypedEst<VT, FT>>("rlscan_gae_typed", P, E, T, 1, ws, ws_bytes, stream, vec);              \
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

int rlscan_vtrace_ex(const float *log_rhos, const float *rewards, const float *values, const float *terminateds,
                  const float *truncateds, const float *bootstrap_values, const float *last_values, float *vs,
                  float *pg_advantages, int64_t E, int64_t T, float gamma, float lambda_, float rho_bar,
                  float c_bar, unsigned options, void *ws, size_t ws_bytes, cudaStream_t stream) {
    RLSCAN_TRY(check_options(options, false));
    RLSCAN_TRY(check_shape(E, T));
    RLSCAN_TRY(check_scalar(gamma, "gamma"));
    RLSCAN_TRY(check_scalar(lambda_, "lambda_"));
    RLSCAN_TRY(check_scalar(rho_bar, "rho_bar"));
    RLSCAN_TRY(check_scalar(c_bar, "c_bar"));
    if (E == 0 || T == 0) return ok();
    RLSCAN_TRY(require(log_rhos, "log_rhos"));
    RLSCAN_TRY(require(rewards, "rewards"));
    RLSCAN_TRY(require(values, "values"));
    RLSCAN_TRY(require(vs, "vs"));
    RLSCAN_TRY(require(pg_advantages, "pg_advantages"));
    if (truncateds && !bootstrap_values) return fail(RLSCAN_ERR_INVALID_ARG, "truncateds given without bootstrap_values");
    const size_t pb = plane_bytes(E, T);
    const Span ins[] = {{log_rhos, pb, "log_rhos"}, {rewards, pb, "rewards"}, {values, pb, "values"},
                        {terminateds, pb, "terminateds"}, {truncateds, pb, "truncateds"},
                        {bootstrap_values, pb, "bootstrap_values"}, {last_values, (size_t)E * 4, "last_values"}};
    const Span outs[] = {{vs, pb, "vs"}, {pg_advantages, pb, "pg_advantages"}};
    RLSCAN_TRY(check_aliasing(ins, 7, outs, 2));
    VtraceEst::Params P{log_rhos, rewards, values, terminateds, truncateds, truncateds ? bootstrap_values : nullptr,
                        last_values, vs, pg_advantages, gamma, lambda_, rho_bar, c_bar};
    if (options & RLSCAN_OPT_TIME_MAJOR) return run_time_major<VtraceEst>("rlscan_vtrace", P, E, T, stream);
    return run<VtraceEst>("rlscan_vtrace", P, E, T, 1, ws, ws_bytes, stream,
                          aligned16({log_rhos, rewards, values, terminateds, truncateds, vs, pg_advantages}));
}

int rlscan_vtrace(const float *log_rhos, const float *rewards, const float *values, const float *terminateds,
                  const float *truncateds, const float *bootstrap_values, const float *last_values, float *vs,
                  float *pg_advantages, int64_t E, int64_t T, float gamma, float lambda_, float rho_bar,
                  float c_bar, void *ws, size_t ws_bytes, cudaStream_t stream) {
    return rlscan_vtrace_ex(log_rhos, rewards, values, terminateds, truncateds, bootstrap_values, last_values, vs, pg_advantages, E, T, gamma, lambda_, rho_bar, c_bar, 0u, ws, ws_bytes, stream);
}

int rlscan_gae_vtrace_ex(const float *log_rhos, const float *rewards, const float *values, const float *terminateds,
                         const float *truncateds, const float *bootstrap_values, const float *last_values,
                         float *advantages, float *returns, float *vs, float *pg_advantages, int64_t E, int64_t T,
                         float gamma, float lambda_, float vtrace_lambda, float rho_bar, float c_bar,
                         unsigned options, void *ws, size_t ws_bytes, cudaStream_t stream) {
    RLSCAN_TRY(check_options(options, false));
    RLSCAN_TRY(check_shape(E, T));
    RLSCAN_TRY(check_scalar(gamma, "gamma"));
    RLSCAN_TRY(check_scalar(lambda_, "lambda_"));
    RLSCAN_TRY(check_scalar(vtrace_lambda, "vtrace_lambda"));
    RLSCAN_TRY(check_scalar(rho_bar, "rho_bar"));
    RLSCAN_TRY(check_scalar(c_bar, "c_bar"));
    if (E == 0 || T == 0) return ok();
    RLSCAN_TRY(require(log_rhos, "log_rhos"));
    RLSCAN_TRY(require(rewards, "rewards"));
    RLSCAN_TRY(require(values, "values"));
    RLSCAN_TRY(require(advantages, "advantages"));
    RLSCAN_TRY(require(vs, "vs"));
    RLSCAN_TRY(require(pg_advantages, "pg_advantages"));
    if (truncateds && !bootstrap_values) return fail(RLSCAN_ERR_INVALID_ARG, "truncateds given without bootstrap_values");
    const size_t pb = plane_bytes(E, T);
    const Span ins[] = {{log_rhos, pb, "log_rhos"}, {rewards, pb, "rewards"}, {values, pb, "values"},
                        {terminateds, pb, "terminateds"}, {truncateds, pb, "truncateds"},
                        {bootstrap_values, pb, "bootstrap_values"}, {last_values, (size_t)E * 4, "last_values"}};
    const Span outs[] = {{advantages, pb, "advantages"}, {returns, pb, "returns"}, {vs, pb, "vs"},
                         {pg_advantages, pb, "pg_advantages"}};
    RLSCAN_TRY(check_aliasing(ins, 7, outs, 4));
    GaeVtraceEst::Params P{log_rhos, rewards, values, terminateds, truncateds,
                           truncateds ? bootstrap_values : nullptr, last_values, advantages, returns, vs,
                           pg_advantages, gamma, lambda_, vtrace_lambda, rho_bar, c_bar};
    if (options & RLSCAN_OPT_TIME_MAJOR) return run_time_major<GaeVtraceEst>("rlscan_gae_vtrace", P, E, T, stream);
    return run<GaeVtraceEst>("rlscan_gae_vtrace", P, E, T, 1, ws, ws_bytes, stream,
                             aligned16({log_rhos, rewards, values, terminateds, truncateds, advantages, returns, vs,
                                        pg_advantages}));
}

int rlscan_gae_vtrace(const float *log_rhos, const float *rewards, const float *values, const float *terminateds,
                      const float *truncateds, const float *bootstrap_values, const float *last_values,
                      float *advantages, float *returns, float *vs, float *pg_advantages, int64_t E, int64_t T,
                      float gamma, float lambda_, float vtrace_lambda, float rho_bar, float c_bar, void *ws,
                      size_t ws_bytes, cudaStream_t stream) {
    return rlscan_gae_vtrace_ex(log_rhos, rewards, values, terminateds, truncateds, bootstrap_values, last_values,
                                advantages, returns, vs, pg_advantages, E, T, gamma, lambda_, vtrace_lambda, rho_bar,
                                c_bar, 0u, ws, ws_bytes, stream);
}

int rlscan_retrace_ex(const float *rewards, const float *q_values, const float *next_q_values_all,
                   const float *next_target_probs, const float *log_rhos, const float *terminateds,
                   const float *truncateds, float *q_ret, int64_t E, int64_t T, int64_t A, float gamma,
                   float lambda_, float c_bar, unsigned options, void *ws, size_t ws_bytes, cudaStream_t stream) {
    RLSCAN_TRY(check_options(options, false));
    if (A < 1) return fail(RLSCAN_ERR_INVALID_ARG, "A must be >= 1 (got %lld)", (long long)A);
    if (A > RLSCAN_MAX_ACTIONS)
        return fail(RLSCAN_ERR_UNSUPPORTED, "A=%lld exceeds RLSCAN_MAX_ACTIONS=%d", (long long)A, RLSCAN_MAX_ACTIONS);
    RLSCAN_TRY(check_shape(E, T, A));
    RLSCAN_TRY(check_scalar(gamma, "gamma"));
    RLSCAN_TRY(check_scalar(lambda_, "lambda_"));
    RLSCAN_TRY(check_scalar(c_bar, "c_bar"));
    if (E == 0 || T == 0) return ok();
    RLSCAN_TRY(require(rewards, "rewards"));
    RLSCAN_TRY(require(q_values, "q_values"));
    RLSCAN_TRY(require(next_q_values_all, "next_q_values_all"));
    RLSCAN_TRY(require(log_rhos, "log_rhos"));
    RLSCAN_TRY(require(terminateds, "terminateds"));
    RLSCAN_TRY(require(truncateds, "truncateds"));
    RLSCAN_TRY(require(q_ret, "q_ret"));
    if (A > 1 && next_target_probs == nullptr)
        return fail(RLSCAN_ERR_INVALID_ARG, "next_target_probs is required when A > 1");
    const size_t pb = plane_bytes(E, T);
    const Span ins[] = {{rewards, pb, "rewards"}, {q_values, pb, "q_values"},
                        {next_q_values_all, pb * (size_t)A, "next_q_values_all"},
                        {A > 1 ? next_target_probs : nullptr, pb * (size_t)A, "next_target_probs"},
                        {log_rhos, pb, "log_rhos"}, {terminateds, pb, "terminateds"}, {truncateds, pb, "truncateds"}};
    const Span outs[] = {{q_ret, pb, "q_ret"}};
    RLSCAN_TRY(check_aliasing(ins, 7, outs, 1));
    if (A == 1) {
        RetraceEst<false>::Params P{rewards, q_values, next_q_values_all, nullptr, log_rhos, terminateds,
                                    truncateds, q_ret, 1, gamma, lambda_, c_bar, 0u};
        if (options & RLSCAN_OPT_TIME_MAJOR)
            return run_time_major<RetraceEst<false>>("rlscan_retrace", P, E, T, stream);
        return run<RetraceEst<false>>("rlscan_retrace", P, E, T, 1, ws, ws_bytes, stream,
                                      aligned16({rewards, q_values, next_q_values_all, log_rhos, terminateds,
                                                 truncateds, q_ret}));
    }
    if (options & RLSCAN_OPT_TIME_MAJOR)
        return fail(RLSCAN_ERR_UNSUPPORTED, "rlscan_retrace: the time-major layout takes A == 1 only");
    RetraceEst<true>::Params P{rewards, q_values, next_q_values_all, next_target_probs, log_rhos, terminateds,
                               truncateds, q_ret, A, gamma, lambda_, c_bar, 1u << 24};
    return run_multi<RetraceEst<true>>("rlscan_retrace", P, E, T, A, ws, ws_bytes, stream,
                                       aligned16({rewards, q_values, log_rhos, terminateds, truncateds, q_ret}));
}

int rlscan_retrace(const float *rewards, const float *q_values, const float *next_q_values_all,
                   const float *next_target_probs, const float *log_rhos, const float *terminateds,
                   const float *truncateds, float *q_ret, int64_t E, int64_t T, int64_t A, float gamma,
                   float lambda_, float c_bar, void *ws, size_t ws_bytes, cudaStream_t stream) {
    return rlscan_retrace_ex(rewards, q_values, next_q_values_all, next_target_probs, log_rhos, terminateds, truncateds, q_ret, E, T, A, gamma, lambda_, c_bar, 0u, ws, ws_bytes, stream);
}

int rlscan_lambda_returns_ex(const float *rewards, const float *values, const float *terminateds,
                          const float *truncateds, const float *bootstrap_values, const float *last_values,
                          float *returns, int64_t E, int64_t T, float gamma, float lambda_, unsigned options, void *ws, size_t ws_bytes, cudaStream_t stream) {
    RLSCAN_TRY(check_options(options, false));
    RLSCAN_TRY(check_shape(E, T));
    RLSCAN_TRY(check_scalar(gamma, "gamma"));
    RLSCAN_TRY(check_scalar(lambda_, "lambda_"));
    if (E == 0 || T == 0) return ok();
    RLSCAN_TRY(require(rewards, "rewards"));
    RLSCAN_TRY(require(values, "values"));
    RLSCAN_TRY(require(returns, "returns"));
    if (truncateds && !bootstrap_values) return fail(RLSCAN_ERR_INVALID_ARG, "truncateds given without bootstrap_values");
    const size_t pb = plane_bytes(E, T);
    const Span ins[] = {{rewards, pb, "rewards"}, {values, pb, "values"}, {terminateds, pb, "terminateds"},
                        {truncateds, pb, "truncateds"}, {bootstrap_values, pb, "bootstrap_values"},
                        {last_values, (size_t)E * 4, "last_values"}};
    const Span outs[] = {{returns, pb, "returns"}};
    RLSCAN_TRY(check_aliasing(ins, 6, outs, 1));
    LambdaReturnsEst::Params P{rewards, values, terminateds, truncateds, truncateds ? bootstrap_values : nullptr,
                               last_values, returns, gamma, lambda_};
    if (options & RLSCAN_OPT_TIME_MAJOR)
        return run_time_major<LambdaReturnsEst>("rlscan_lambda_returns", P, E, T, stream);
    return run<LambdaReturnsEst>("rlscan_lambda_returns", P, E, T, 1, ws, ws_bytes, stream,
                                 aligned16({rewards, values, terminateds, truncateds, returns}));
}

int rlscan_lambda_returns(const float *rewards, const float *values, const float *terminateds,
                          const float *truncateds, const float *bootstrap_values, const float *last_values,
                          float *returns, int64_t E, int64_t T, float gamma, float lambda_, void *ws,
                          size_t ws_bytes, cudaStream_t stream) {
    return rlscan_lambda_returns_ex(rewards, values, terminateds, truncateds, bootstrap_values, last_values, returns, E, T, gamma, lambda_, 0u, ws, ws_bytes, stream);
}

int rlscan_discounted_returns_ex(const float *rewards, const float *terminateds, const float *truncateds,
                              const float *bootstrap_values, const float *last_values, float *returns, int64_t E,
                              int64_t T, float gamma, unsigned options, void *ws, size_t ws_bytes, cudaStream_t stream) {
    RLSCAN_TRY(check_options(options, false));
    RLSCAN_TRY(check_shape(E, T));
    RLSCAN_TRY(check_scalar(gamma, "gamma"));
    if (E == 0 || T == 0) return ok();
    RLSCAN_TRY(require(rewards, "rewards"));
    RLSCAN_TRY(require(returns, "returns"));
    if (truncateds && !bootstrap_values) return fail(RLSCAN_ERR_INVALID_ARG, "truncateds given without bootstrap_values");
    const size_t pb = plane_bytes(E, T);
    const Span ins[] = {{rewards, pb, "rewards"}, {terminateds, pb, "terminateds"}, {truncateds, pb, "truncateds"},
                        {bootstrap_values, pb, "bootstrap_values"}, {last_values, (size_t)E * 4, "last_values"}};
    const Span outs[] = {{returns, pb, "returns"}};
    RLSCAN_TRY(check_aliasing(ins, 5, outs, 1));
    ReturnsEst::Params P{rewards, terminateds, truncateds, truncateds ? bootstrap_values : nullptr, last_values,
                         returns, gamma};
    if (options & RLSCAN_OPT_TIME_MAJOR)
        return run_time_major<ReturnsEst>("rlscan_discounted_returns", P, E, T, stream);
    return run<ReturnsEst>("rlscan_discounted_returns", P, E, T, 1, ws, ws_bytes, stream,
                           aligned16({rewards, terminateds, truncateds, returns}));
}

int rlscan_discounted_returns(const float *rewards, const float *terminateds, const float *truncateds,
                              const float *bootstrap_values, const float *last_values, float *returns, int64_t E,
                              int64_t T, float gamma, void *ws, size_t ws_bytes, cudaStream_t stream) {
    return rlscan_discounted_returns_ex(rewards, terminateds, truncateds, bootstrap_values, last_values, returns, E, T, gamma, 0u, ws, ws_bytes, stream);
}

int rlscan_eligibility_traces_ex(const float *x, const float *dones, float *traces, int64_t E, int64_t T, float gamma,
                              float lambda_, unsigned options, void *ws, size_t ws_bytes, cudaStream_t stream) {
    RLSCAN_TRY(check_options(options, true));
    RLSCAN_TRY(check_shape(E, T));
    RLSCAN_TRY(check_scalar(gamma, "gamma"));
    RLSCAN_TRY(check_scalar(lambda_, "lambda_"));
    if (E == 0 || T == 0) return ok();
    RLSCAN_TRY(require(x, "x"));
    RLSCAN_TRY(require(traces, "traces"));
    const size_t pb = plane_bytes(E, T);
    const Span ins[] = {{x, pb, "x"}, {dones, pb, "dones"}};
    const Span outs[] = {{traces, pb, "traces"}};
    RLSCAN_TRY(check_aliasing(ins, 2, outs, 1));
    TracesEst::Params P{x, dones, traces, gamma * lambda_, (options & RLSCAN_OPT_DONE_STARTS_EPISODE) ? 1 : 0};
    if (options & RLSCAN_OPT_TIME_MAJOR)
        return run_time_major<TracesEst>("rlscan_eligibility_traces", P, E, T, stream);
    return run<TracesEst>("rlscan_eligibility_traces", P, E, T, 1, ws, ws_bytes, stream,
                          aligned16({x, dones, traces}));
}

int rlscan_eligibility_traces(const float *x, const float *dones, float *traces, int64_t E, int64_t T, float gamma,
                              float lambda_, void *ws, size_t ws_bytes, cudaStream_t stream) {
    return rlscan_eligibility_traces_ex(x, dones, traces, E, T, gamma, lambda_, 0u, ws, ws_bytes, stream);
}

int rlscan_episodic_prefix_sum_ex(const void *x, int dtype, const float *dones, void *out, int64_t E, int64_t T,
                               unsigned options, void *ws, size_t ws_bytes, cudaStream_t stream) {
    RLSCAN_TRY(check_options(options, true));
    if (dtype != RLSCAN_F32 && dtype != RLSCAN_I32) return fail(RLSCAN_ERR_UNSUPPORTED, "unknown dtype %d", dtype);
    RLSCAN_TRY(check_shape(E, T));
    if (E == 0 || T == 0) return ok();
    RLSCAN_TRY(require(x, "x"));
    RLSCAN_TRY(require(out, "out"));
    const size_t pb = plane_bytes(E, T);
    const Span ins[] = {{x, pb, "x"}, {dones, pb, "dones"}};
    const Span outs[] = {{out, pb, "out"}};
    RLSCAN_TRY(check_aliasing(ins, 2, outs, 1));
    if (dtype == RLSCAN_F32) {
        PrefixF32Est::Params P{static_cast<const float *>(x), dones, static_cast<float *>(out), 1.0f, (options & RLSCAN_OPT_DONE_STARTS_EPISODE) ? 1 : 0};
        if (options & RLSCAN_OPT_TIME_MAJOR)
            return run_time_major<PrefixF32Est>("rlscan_episodic_prefix_sum", P, E, T, stream);
        return run<PrefixF32Est>("rlscan_episodic_prefix_sum", P, E, T, 1, ws, ws_bytes, stream,
                                 aligned16({x, dones, out}));
    }
    PrefixI32Est::Params P{static_cast<const int32_t *>(x), dones, static_cast<int32_t *>(out), (options & RLSCAN_OPT_DONE_STARTS_EPISODE) ? 1 : 0};
    if (options & RLSCAN_OPT_TIME_MAJOR)
        return run_time_major<PrefixI32Est>("rlscan_episodic_prefix_sum", P, E, T, stream);
    return run<PrefixI32Est>("rlscan_episodic_prefix_sum", P, E, T, 1, ws, ws_bytes, stream,
                             aligned16({x, dones, out}));
}

int rlscan_episodic_prefix_sum(const void *x, int dtype, const float *dones, void *out, int64_t E, int64_t T,
                               void *ws, size_t ws_bytes, cudaStream_t stream) {
    return rlscan_episodic_prefix_sum_ex(x, dtype, dones, out, E, T, 0u, ws, ws_bytes, stream);
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
    const size_t need = workspace_for(make_plan(E, T, 1));
    if (need > RLSCAN_NOALLOC_SCRATCH_BYTES)
        return fail(RLSCAN_ERR_WORKSPACE,
                    "rlscan_gae_noalloc: shape E=%lld T=%lld needs %zu bytes of scratch; the fixed scratch holds %u",
                    (long long)E, (long long)T, need, (unsigned)RLSCAN_NOALLOC_SCRATCH_BYTES);
    void *ws = nullptr;
    if (need > 0) {
        RLSCAN_TRY(noalloc_scratch(&ws));
        // the array keeps the previous call's contents: the tile counters and
        // flags this call uses must start at zero
        cudaError_t e = cudaMemsetAsync(ws, 0, need, stream);
        if (e != cudaSuccess) return fail(RLSCAN_ERR_CUDA, "cudaMemsetAsync(scratch): %s", cudaGetErrorString(e));
    }
    return rlscan_gae(rewards, values, terminateds, truncateds, bootstrap_values, last_values, advantages, E, T, gamma,
                      lambda_, ws, need, stream);
}

size_t rlscan_workspace_bytes(int64_t E, int64_t T) {
    if (E <= 0 || T <= 0 || E > kMaxElems / T) return 0;
    size_t need = 0;
    const long long probe_actions[] = {1, 2, 25, 49};
    for (long long a : probe_actions) {
        const size_t w = workspace_for(make_plan(E, T, a));
        if (w > need) need = w;
    }
    return need;
}

int rlscan_workspace_init(void *ws, size_t ws_bytes, cudaStream_t stream) {
    if (ws_bytes == 0) return ok();
    if (ws == nullptr) return fail(RLSCAN_ERR_INVALID_ARG, "ws must not be NULL");
    cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, stream);
    if (e != cudaSuccess) return fail(RLSCAN_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
    return ok();
}

int rlscan_check(cudaStream_t stream) {
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return fail(RLSCAN_ERR_CUDA, "stream error: %s", cudaGetErrorString(e));
    unsigned word = 0;
    e = cudaMemcpyFromSymbol(&word, g_device_error, sizeof word);
    if (e != cudaSuccess) return fail(RLSCAN_ERR_CUDA, "reading the error word: %s", cudaGetErrorString(e));
    if (word != 0) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero);
        if (e != cudaSuccess) return fail(RLSCAN_ERR_CUDA, "clearing the error word: %s", cudaGetErrorString(e));
        return fail(RLSCAN_ERR_TIMEOUT, "a kernel gave up a bounded wait (error word 0x%x)", word);
    }
    return ok();
}

const char *rlscan_last_error(void) { return g_last_error.c_str(); }

int rlscan_version(void) { return RLSCAN_VERSION; }

int rlscan_debug_set_lookback(uint32_t spin_limit, int64_t withhold_tile) {
    g_spin_limit.store(spin_limit == 0 ? kDefaultSpinLimit : spin_limit);
    g_withhold.store(withhold_tile < 0 ? -1 : (long long)withhold_tile);
    return ok();
}

int rlscan_plan(int64_t E, int64_t T, int64_t actions, int64_t *tile_elems, int *threads, int *lookback,
                int64_t *num_tiles) {
    if (E <= 0 || T <= 0) return fail(RLSCAN_ERR_INVALID_ARG, "E and T must be > 0");
    if (actions < 1 || actions > RLSCAN_MAX_ACTIONS) return fail(RLSCAN_ERR_INVALID_ARG, "bad action count");
    RLSCAN_TRY(check_shape(E, T, actions));
    const Plan p = make_plan(E, T, actions);
    if (tile_elems) *tile_elems = kCfgTile[p.cfg];
    if (threads) *threads = kCfgThreads[p.cfg];
    if (lookback) *lookback = p.lookback ? 1 : 0;
    if (num_tiles) *num_tiles = p.ntiles;
    return ok();
}

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
    switch (c.kind) {
    case RLSCAN_KIND_GAE_TYPED: {
        const size_t v = n * dtype_bytes(c.dtype), f = n * dtype_bytes(c.flag_dtype);
        const size_t by_slot[6] = {v, v, f, f, v, row};
        return slot < 6 ? by_slot[slot] : 0;
    }
    case RLSCAN_KIND_GAE:
    case RLSCAN_KIND_GAE_WITH_RETURNS:
    case RLSCAN_KIND_LAMBDA_RETURNS: return slot < 5 ? plane : (slot == 5 ? row : 0);
    case RLSCAN_KIND_VTRACE:
    case RLSCAN_KIND_GAE_VTRACE: return slot < 6 ? plane : (slot == 6 ? row : 0);
    case RLSCAN_KIND_RETRACE: return (slot == 2 || slot == 3) ? plane * (size_t)(c.A > 0 ? c.A : 1) : (slot < 7 ? plane : 0);
    case RLSCAN_KIND_DISCOUNTED_RETURNS: return slot < 4 ? plane : (slot == 4 ? row : 0);
    case RLSCAN_KIND_ELIGIBILITY_TRACES:
    case RLSCAN_KIND_EPISODIC_PREFIX_SUM: return slot < 2 ? plane : 0;
    default: return 0;
    }
}

static int call_dispatch(const rlscan_call &c, void *ws, size_t ws_bytes, cudaStream_t stream) {
    const float *const *in = reinterpret_cast<const float *const *>(c.in);
    float *const *out = reinterpret_cast<float *const *>(c.out);
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

// Which kernel and how many elements per thread a fused request takes.
// Requests mixing three or more estimators run every fp32 call on the shared
// body (one instruction stream for all of them, fused_any.cuh) when every
// fp32 call's rows hold whole multiples of V elements; otherwise each call
// runs its own estimator's body, 4 elements per thread when the request
// mixes three or more estimators and every row fits a 512-element tile
// (smaller code per estimator), else 8.
struct FusedChoice {
    bool shared_body;
    int V;
};
static FusedChoice choose_fused(const BatchState &st) {
    const FusedBatch &fb = st.fb;
    unsigned kinds = 0u;
    bool fit4 = true;
    for (int i = 0; i < fb.n; ++i) {
        kinds |= 1u << fb.item[i].kind;
        if ((long long)(kFusedNT * 4) % fb.item[i].g.seq_len != 0) fit4 = false;
    }
    const bool mixed = __builtin_popcount(kinds) >= 3;
    if (mixed) {
        constexpr int kSharedV = 4;
        bool shared_ok = true;
        for (int i = 0; i < fb.n; ++i) {
            const long long T = fb.item[i].g.seq_len;
            if ((long long)(kFusedNT * kSharedV) % T != 0) shared_ok = false; // rows whole in a tile
            if (st.has_any[i] && T < kSharedV) shared_ok = false;             // and whole in a thread
        }
        if (shared_ok) return {true, kSharedV};
    }
    return {false, (mixed && fit4) ? 4 : 8};
}

// Tiling of each item of a fused launch of V elements per thread; with the
// shared body, fp32 items carry their AnyParams.
static void fused_layout(BatchState &st, const FusedChoice &ch, long long *tiles) {
    FusedBatch &fb = st.fb;
    const int V = ch.V;
    if (ch.shared_body) {
        for (int i = 0; i < fb.n; ++i) {
            if (!st.has_any[i]) continue;
            static_assert(sizeof(AnyParams) <= kFusedParamBytes, "shared-body params fit a fused item");
            std::memset(fb.item[i].params, 0, sizeof fb.item[i].params);
            std::memcpy(fb.item[i].params, &st.any[i], sizeof(AnyParams));
        }
    }
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
    const FusedChoice ch = choose_fused(st);
    fused_layout(st, ch, &st.tiles);
    const int V = ch.V;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)st.tiles);
    cfg.blockDim = dim3(kFusedNT);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    cudaError_t e;
    if (ch.shared_body)
        e = V == 4 ? cudaLaunchKernelEx(&cfg, fused_any_kernel<4>, st.fb)
                   : cudaLaunchKernelEx(&cfg, fused_any_kernel<8>, st.fb);
    else
        e = V == 4 ? cudaLaunchKernelEx(&cfg, fused_tile_kernel<4>, st.fb)
                   : cudaLaunchKernelEx(&cfg, fused_tile_kernel<8>, st.fb);
    if (e != cudaSuccess) return fail(RLSCAN_ERR_CUDA, "rlscan_batch: fused launch failed: %s", cudaGetErrorString(e));
    return ok();
}

} // extern "C"
