// host.cuh - host side of librlscan shared by its translation units:
// status and message helpers, argument checks, tile plans, batch-request
// state, and the launch helpers that instantiate the kernels (each
// translation unit instantiates the kernels of the estimators it serves).
// State shared by all units (the thread's last error message, the SM
// counts, the batch request being served) is held in
// inline variables, one instance per process.
#pragma once

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <climits>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <initializer_list>
#include <string>
#include <type_traits>

#include "../../include/rlscan.h"
#include "batch.cuh"

namespace rlscan {

inline thread_local std::string g_last_error;

inline int fail(int code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

inline int ok() {
    g_last_error.clear();
    return RLSCAN_OK;
}

inline bool pdl_enabled() {
    static const bool on = [] {
        const char *v = std::getenv("RLSCAN_DISABLE_PDL");
        return !(v && v[0] && v[0] != '0');
    }();
    return on;
}

// ---------------------------------------------------------------------------
// Tile plans.  A tile is S = NT * V consecutive elements of the flattened
// [E*T] array.  Rows need carries across tiles (the chunked two passes) only
// when a tile boundary can fall inside a row (S not a multiple of T, more
// than one tile).
// ---------------------------------------------------------------------------
// Eight elements per thread keeps a grid's share of each SM small, so the
// next launch on the stream can be resident (and prefetching) while this one
// runs; the 512-element tile (four per thread) is for small plans.  Calls on
// 2-byte value planes take the same tiles (measured at 4096 x 128 and 65536
// x 128: 8 elements per thread in 128-thread blocks beat 16 elements per
// thread in half as many threads, 23.7 against 28.9 us for bf16 / uint8 GAE
// + returns at 65536 x 128).
enum Cfg { C512 = 0, C1024, C2048, C4096, kNumCfg };
constexpr int kCfgTile[kNumCfg] = {512, 1024, 2048, 4096};
constexpr int kCfgThreads[kNumCfg] = {128, 128, 256, 512};

struct Plan {
    Cfg cfg;
    bool lookback;
    long long ntiles;
    int mode; // kModeBlock / kModeWarp (whole rows per tile); rows that span
              // tiles (lookback) take the chunked two passes instead
};

// Scan mode of a whole-row plan: warp-local when every warp's 32*V elements
// hold whole rows; otherwise a block scan.
inline Plan with_mode(Plan p, long long T) {
    const long long warp_elems = 32ll * (kCfgTile[p.cfg] / kCfgThreads[p.cfg]);
    p.mode = (warp_elems % T == 0) ? kModeWarp : kModeBlock;
    return p;
}

// SM count of the current device (queried once per device; B200's 148 when
// no device can be asked, e.g. when a plan is computed on a host without a
// GPU).  Plans fill the GPU: with fewer tiles than two per SM a plan prefers
// smaller tiles.
constexpr long long kDefaultSMs = 148;
constexpr int kMaxPlanDevices = 256;
inline std::atomic<int> g_sm_count[kMaxPlanDevices];

inline long long num_sms() {
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

inline long long ceil_div(long long a, long long b) { return (a + b - 1) / b; }

inline int pow2_shift(long long T) {
    if (T <= 0 || (T & (T - 1)) != 0) return -1;
    int s = 0;
    while ((1ll << s) < T) ++s;
    return s;
}

// Every call scans on these plans; multi-action Retrace scans its expected
// values (a plane written first) like a single-action call.
inline Plan make_plan_tiles(long long E, long long T) {
    const long long n = E * T;
    Plan p{};
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
    // GPU): the chunked two passes (run_chunked), unless the whole array fits
    // one tile
    p.cfg = ceil_div(n, kCfgTile[C2048]) >= min_tiles
                ? C2048
                : (ceil_div(n, kCfgTile[C1024]) >= min_tiles ? C1024 : C512);
    p.ntiles = ceil_div(n, kCfgTile[p.cfg]);
    p.lookback = p.ntiles > 1 && (kCfgTile[p.cfg] % T != 0);
    return p;
}

inline Plan make_plan(long long E, long long T) { return with_mode(make_plan_tiles(E, T), T); }

// Warp-local mode: a row spans T / V lanes (T a power of two dividing 32 V);
// the shuffle scan needs to reach that far only.
inline int scan_lanes_for(const Plan &p, long long T) {
    if (p.mode != kModeWarp) return 32;
    const long long V = kCfgTile[p.cfg] / kCfgThreads[p.cfg];
    const long long lanes = T >= V ? T / V : 1;
    return (int)(lanes < 32 ? lanes : 32);
}

// True when every given pointer is NULL or 16-byte aligned.
inline bool aligned16(std::initializer_list<const void *> ptrs) {
    for (const void *p : ptrs)
        if (p != nullptr && ((uintptr_t)p & 15u) != 0) return false;
    return true;
}

// Rows that span tiles: one 16-byte slot per chunk of the chunked two
// passes, at most one per 1024 elements (a chunk holds at least two warp
// steps of 512); nothing otherwise.
inline size_t workspace_for(const Plan &p, long long n) {
    return p.lookback ? sizeof(TileSlot) * (size_t)ceil_div(n, 2LL * 32 * kChunkV) : 0;
}

// ---------------------------------------------------------------------------
// Argument checks
// ---------------------------------------------------------------------------
constexpr long long kMaxElems = 1ll << 40;

inline int check_shape(long long E, long long T, long long A = 1) {
    if (E < 0 || T < 0) return fail(RLSCAN_ERR_INVALID_ARG, "E and T must be >= 0 (got E=%lld, T=%lld)", E, T);
    if (E > 0 && T > 0 && (E > kMaxElems / T || E * T > kMaxElems / (A > 0 ? A : 1)))
        return fail(RLSCAN_ERR_INVALID_ARG, "E*T*A too large (E=%lld, T=%lld, A=%lld)", E, T, A);
    if (E > 0 && T > 0 && ceil_div(E * T, 128) >= (1ll << 31) - 1)
        return fail(RLSCAN_ERR_INVALID_ARG, "E*T too large for one launch");
    return RLSCAN_OK;
}

inline int check_scalar(float v, const char *name) {
    if (!std::isfinite(v)) return fail(RLSCAN_ERR_INVALID_ARG, "%s must be finite", name);
    return RLSCAN_OK;
}

struct Span {
    const void *p;
    size_t bytes;
    const char *name;
};

inline bool overlap(const Span &a, const Span &b) {
    if (!a.p || !b.p || a.bytes == 0 || b.bytes == 0) return false;
    const uintptr_t a0 = (uintptr_t)a.p, a1 = a0 + a.bytes;
    const uintptr_t b0 = (uintptr_t)b.p, b1 = b0 + b.bytes;
    return a0 < b1 && b0 < a1;
}

// Every output against every input and every other output.
inline int check_aliasing(const Span *ins, int nin, const Span *outs, int nout) {
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

inline int require(const void *p, const char *name) {
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
};
inline thread_local BatchState *g_batch = nullptr;

inline bool batch_dry() { return g_batch != nullptr && g_batch->pass == kBatchDry; }

// ---------------------------------------------------------------------------
// Launch
// ---------------------------------------------------------------------------
// Bytes per element of the input planes a call streams (its given planes).
template <class Est>
inline long long streamed_input_bytes(const typename Est::Params &P) {
    long long b = 0;
    for (int i = 0; i < Est::kInputPlanes; ++i) {
        const PlaneRef r = Est::input_plane(P, i);
        if (r.p != nullptr) b += r.bytes;
    }
    return b;
}

// Resident blocks per SM of a kernel, queried once per kernel (`unknown`
// when the query fails).
template <class K>
inline int resident_blocks(K kern, int threads, size_t smem, std::atomic<int> &cache, int unknown) {
    int r = cache.load(std::memory_order_relaxed);
    if (r == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&r, kern, threads, smem) != cudaSuccess || r < 1) {
            (void)cudaGetLastError();
            r = unknown;
        }
        cache.store(r, std::memory_order_relaxed);
    }
    return r;
}

constexpr long long kPrefetchAllBelowBytes = 8; // input bytes per element

template <class Est, int NT, int V, int kMode, int kCase>
cudaError_t launch_one(const typename Est::Params &P, const Geometry &g, size_t smem, cudaStream_t stream) {
    auto kern = tile_scan_kernel<Est, NT, V, kMode, kCase>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)g.ntiles);
    cfg.blockDim = dim3(NT);
    static std::atomic<int> resident_cache{0};
    const int resident = resident_blocks(kern, NT, smem, resident_cache, 1 << 16); // unknown: all prefetch
    // Calls that stream few bytes per element (reduced-byte planes) keep few
    // bytes in flight per thread: every block prefetches its tile there, so
    // the L2 fetches run ahead of the loads (measured: bf16 / uint8 GAE +
    // returns at 65536 x 128 in 23.7 us this way, 28.0 us with the first
    // wave alone).  Elsewhere the first wave of blocks alone prefetches.
    Geometry gl = g;
    gl.pf_blocks = streamed_input_bytes<Est>(P) < kPrefetchAllBelowBytes ? (1ll << 62) : (long long)num_sms() * resident;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, P, gl);
}

template <class Est, Cfg C>
cudaError_t launch_cfg(const typename Est::Params &P, const Geometry &g, int mode, int kcase, size_t smem,
                       cudaStream_t s) {
    constexpr int NT = kCfgThreads[C];
    constexpr int V = kCfgTile[C] / NT;
    if constexpr (HasTruncations<typename Est::Params>::value && !PlainTestsTruncations<Est>::value) {
        if (kcase == kCasePlainTrunc) {
            if (mode == kModeWarp) return launch_one<Est, NT, V, kModeWarp, kCasePlainTrunc>(P, g, smem, s);
            return launch_one<Est, NT, V, kModeBlock, kCasePlainTrunc>(P, g, smem, s);
        }
    }
    if (kcase == kCasePlain) {
        if (mode == kModeWarp) return launch_one<Est, NT, V, kModeWarp, kCasePlain>(P, g, smem, s);
        return launch_one<Est, NT, V, kModeBlock, kCasePlain>(P, g, smem, s);
    }
    if (mode == kModeWarp) return launch_one<Est, NT, V, kModeWarp, kCaseAny>(P, g, smem, s);
    return launch_one<Est, NT, V, kModeBlock, kCaseAny>(P, g, smem, s);
}

// Input bytes a two-pass wave may hold so that pass two re-reads them from
// L2: a wave's pass one streams them from HBM, pass two finds them in L2
// (B200: 126 MB).
constexpr long long kTwoPassWaveBytes = 64ll << 20;

// Rows that span tiles: the chunked two passes (chunk_scan_kernel).  One
// chunk per warp the GPU holds at once (at least two steps a chunk, so the
// chunks fit the workspace of workspace_for), over as few waves as keep each
// wave's inputs within kTwoPassWaveBytes.
template <class Est, int kCase>
int run_chunked(const char *name, const typename Est::Params &P, const Geometry &g, TileSlot *slots,
                cudaStream_t stream) {
    constexpr long long SW = 32LL * kChunkV;
    constexpr int WPB = kChunkNT / 32;
    // both passes run on the same grid, which the GPU holds at once
    static std::atomic<int> res_a{0}, res_b{0};
    const long long resident = std::min(resident_blocks(chunk_scan_kernel<Est, kChunkAggregates, kCase>, kChunkNT, 0, res_a, 1),
                                        resident_blocks(chunk_scan_kernel<Est, kChunkScan, kCase>, kChunkNT, 0, res_b, 1));
    const long long warps = (long long)num_sms() * resident * WPB;
    const long long nsteps = ceil_div(g.n, SW);
    const long long in_bytes = std::max<long long>(1, streamed_input_bytes<Est>(P)) * g.n;
    const long long nwaves = ceil_div(in_bytes, kTwoPassWaveBytes);
    const long long wave_steps = ceil_div(nsteps, nwaves);
    const long long chunk_steps = std::max<long long>(2, ceil_div(wave_steps, warps));
    const long long nchunks = ceil_div(nsteps, chunk_steps);
    const long long wave_chunks = ceil_div(wave_steps, chunk_steps);
    ChunkSplit cs{slots, nsteps, chunk_steps, 0, 0, (long long)num_sms() * resident};
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kChunkNT);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    for (long long c0 = 0; c0 < nchunks; c0 += wave_chunks) {
        cs.chunk_begin = c0;
        cs.chunk_end = std::min(nchunks, c0 + wave_chunks);
        cfg.gridDim = dim3((unsigned)ceil_div(cs.chunk_end - cs.chunk_begin, (long long)WPB));
        cudaError_t e = cudaLaunchKernelEx(&cfg, chunk_scan_kernel<Est, kChunkAggregates, kCase>, P, g, cs);
        if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, chunk_scan_kernel<Est, kChunkScan, kCase>, P, g, cs);
        if (e != cudaSuccess) return fail(RLSCAN_ERR_CUDA, "%s: launch failed: %s", name, cudaGetErrorString(e));
    }
    return ok();
}

template <class Est>
int run(const char *name, const typename Est::Params &P, long long E, long long T, void *ws, size_t ws_bytes,
        cudaStream_t stream, bool vec_ok) {
    const Plan plan = make_plan(E, T);
    Geometry g;
    g.n = E * T;
    g.seq_len = T;
    g.ntiles = plan.ntiles;
    g.rows = E;
    g.t_shift = pow2_shift(T);
    g.vec_ok = vec_ok ? 1 : 0;
    g.scan_lanes = scan_lanes_for(plan, T);
    TileSlot *slots = nullptr;
    if (plan.lookback) {
        const size_t need = workspace_for(plan, E * T);
        if (ws == nullptr || ws_bytes < need)
            return fail(RLSCAN_ERR_WORKSPACE, "%s: shape E=%lld T=%lld needs a %zu-byte workspace (got %s, %zu bytes)",
                        name, E, T, need, ws ? "a buffer" : "NULL", ws_bytes);
        if (((uintptr_t)ws & 15u) != 0) return fail(RLSCAN_ERR_WORKSPACE, "%s: workspace must be 16-byte aligned", name);
        slots = static_cast<TileSlot *>(ws);
    }
    if (batch_dry()) return ok();
    if constexpr (FusedBodyOf<Est>::value >= 0) {
        // fused when whole rows fit the largest fused tile; the fused launch
        // tiles the call itself (fused_layout, once the request is known)
        constexpr long long kS = (long long)kFusedNT * kFusedV;
        if (g_batch != nullptr && kS % T == 0 && g_batch->fb.n < kFusedMax) {
            const auto body_params = family_params(P);
            static_assert(sizeof(body_params) <= kFusedParamBytes, "params fit a fused item");
            FusedItem &it = g_batch->fb.item[g_batch->fb.n++];
            std::memset(it.params, 0, sizeof it.params);
            std::memcpy(it.params, &body_params, sizeof body_params);
            it.g = g;
            it.kind = FusedBodyOf<Est>::value;
            it.truncation_code = needs_truncation_code<Est>(body_params) ? 1 : 0;
            return ok();
        }
    }
    if (plan.lookback) {
        // the plain chunk kernel when every warp step is whole, every plane
        // 16-byte aligned and no truncation logic is needed (16 x 262144:
        // discounted returns 15.9 against 17.1 us, GAE 21.8 against 22.1)
        const bool plain = vec_ok && g.n % (32LL * kChunkV) == 0 && T % kChunkV == 0 &&
                           !needs_truncation_code<Est>(P);
        return plain ? run_chunked<Est, kCasePlain>(name, P, g, slots, stream)
                     : run_chunked<Est, kCaseAny>(name, P, g, slots, stream);
    }
    // the plain kernel (one builder variant, vector accesses only) when every
    // thread has all its elements (V divides T, whole tiles) and every plane
    // is 16-byte aligned (measured at 4096 x 128: GAE 2.34 against 2.41 us,
    // V-Trace 3.03 against 3.19, bf16 / uint8 GAE + returns 2.52 against
    // 2.99); with truncation logic when the call passes truncations (GAE
    // with truncations 2.88 against 3.01 us)
    const long long S = kCfgTile[plan.cfg], Vp = S / kCfgThreads[plan.cfg];
    const bool whole = vec_ok && T % Vp == 0 && g.n % S == 0;
    const int kcase = !whole ? kCaseAny : (needs_truncation_code<Est>(P) ? kCasePlainTrunc : kCasePlain);
    cudaError_t e;
    switch (plan.cfg) {
    case C512: e = launch_cfg<Est, C512>(P, g, plan.mode, kcase, 0, stream); break;
    case C1024: e = launch_cfg<Est, C1024>(P, g, plan.mode, kcase, 0, stream); break;
    case C2048: e = launch_cfg<Est, C2048>(P, g, plan.mode, kcase, 0, stream); break;
    case C4096: e = launch_cfg<Est, C4096>(P, g, plan.mode, kcase, 0, stream); break;
    default: return fail(RLSCAN_ERR_UNSUPPORTED, "%s: internal plan error", name);
    }
    if (e != cudaSuccess) return fail(RLSCAN_ERR_CUDA, "%s: launch failed: %s", name, cudaGetErrorString(e));
    return ok();
}

inline size_t plane_bytes(long long E, long long T) { return (size_t)(E * T) * sizeof(float); }

// Option bits of the _ex entry points; `forward` estimators also take
// RLSCAN_OPT_DONE_STARTS_EPISODE.
inline int check_options(unsigned options, bool forward) {
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
    long long nseg; // segments per row
    int nsplit;     // blocks per row (1: whole rows)
    int sps;        // segments per split
};

// Wider env groups (longer contiguous runs per load) while the grid keeps
// enough blocks: 32-env groups from about four blocks per SM up, 16-env
// groups from about one, else 8; rows of several segments (T > 256) favour
// more, smaller blocks.  Measured at E x T = 1024..65536 x 128, 4096 x 1024
// and 512 x 4096.  The segment covers the row, up to 16 warps.
inline TmPlan tm_plan(long long E, long long T) {
    TmPlan p;
    const long long kMinBlocks = 120;
    p.G = (E / 32 >= 4 * num_sms() && T <= 256) ? 32 : (E / 16 >= kMinBlocks ? 16 : 8);
    const long long chunks = ceil_div(T, kTmV);
    const long long nw = ceil_div(chunks, 32 / p.G);
    p.nw = (int)(nw < 1 ? 1 : (nw > kTmMaxWarps ? kTmMaxWarps : nw));
    p.nseg = ceil_div(T, (long long)p.nw * (32 / p.G) * kTmV);
    // rows split over blocks when the env groups alone leave the GPU short of
    // two blocks per SM and rows hold several segments
    const long long blocks = ceil_div(E, p.G), want = 2 * num_sms();
    p.nsplit = 1;
    p.sps = (int)p.nseg;
    if (blocks < want && p.nseg > 1) {
        const long long ns = std::min<long long>(p.nseg, ceil_div(want, blocks));
        p.sps = (int)ceil_div(p.nseg, ns);
        p.nsplit = (int)ceil_div(p.nseg, p.sps);
    }
    return p;
}

// Workspace of a time-major call: one 16-byte slot per env and split when
// its rows are split over blocks, else none.
inline size_t tm_workspace_for(long long E, long long T) {
    const TmPlan p = tm_plan(E, T);
    return p.nsplit > 1 ? sizeof(TileSlot) * (size_t)E * (size_t)p.nsplit : 0;
}

template <class Est>
int run_time_major(const char *name, const typename Est::Params &P, long long E, long long T, cudaStream_t stream,
                   void *ws = nullptr, size_t ws_bytes = 0) {
    if (E > (long long)INT_MAX / (kTmV + 1))
        return fail(RLSCAN_ERR_UNSUPPORTED, "%s: the time-major layout takes E <= %d", name, INT_MAX / (kTmV + 1));
    if (batch_dry()) return ok();
    const TmPlan tp = tm_plan(E, T);
    Geometry g;
    g.n = E * T;
    g.seq_len = T;
    g.rows = E;
    g.ntiles = tp.nseg; // segments per row
    g.t_shift = pow2_shift(T);
    g.vec_ok = 0;
    g.scan_lanes = 32;
    cudaLaunchConfig_t cfg = {};
    // split rows need a workspace (of any content); without one (or too
    // small) the rows run whole
    TmSplit sp{nullptr, 1, (int)tp.nseg};
    const size_t need = tp.nsplit > 1 ? sizeof(TileSlot) * (size_t)E * (size_t)tp.nsplit : 0;
    if (need > 0 && ws != nullptr && ws_bytes >= need && ((uintptr_t)ws & 15u) == 0)
        sp = TmSplit{static_cast<TileSlot *>(ws), tp.nsplit, tp.sps};
    cfg.gridDim = dim3((unsigned)ceil_div(E, tp.G), (unsigned)sp.nsplit);
    cfg.blockDim = dim3(tp.nw * 32);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    cudaError_t e = cudaSuccess;
    const int passes[2] = {sp.nsplit > 1 ? kTmMaps : kTmWhole, kTmCarry};
    for (int i = 0; i < (sp.nsplit > 1 ? 2 : 1); ++i) {
        const int pass = passes[i];
        switch (tp.G * 4 + pass) {
        case 32 * 4 + kTmWhole: e = cudaLaunchKernelEx(&cfg, time_major_scan_kernel<Est, 32, kTmV, kTmWhole>, P, g, sp); break;
        case 32 * 4 + kTmMaps: e = cudaLaunchKernelEx(&cfg, time_major_scan_kernel<Est, 32, kTmV, kTmMaps>, P, g, sp); break;
        case 32 * 4 + kTmCarry: e = cudaLaunchKernelEx(&cfg, time_major_scan_kernel<Est, 32, kTmV, kTmCarry>, P, g, sp); break;
        case 16 * 4 + kTmWhole: e = cudaLaunchKernelEx(&cfg, time_major_scan_kernel<Est, 16, kTmV, kTmWhole>, P, g, sp); break;
        case 16 * 4 + kTmMaps: e = cudaLaunchKernelEx(&cfg, time_major_scan_kernel<Est, 16, kTmV, kTmMaps>, P, g, sp); break;
        case 16 * 4 + kTmCarry: e = cudaLaunchKernelEx(&cfg, time_major_scan_kernel<Est, 16, kTmV, kTmCarry>, P, g, sp); break;
        case 8 * 4 + kTmWhole: e = cudaLaunchKernelEx(&cfg, time_major_scan_kernel<Est, 8, kTmV, kTmWhole>, P, g, sp); break;
        case 8 * 4 + kTmMaps: e = cudaLaunchKernelEx(&cfg, time_major_scan_kernel<Est, 8, kTmV, kTmMaps>, P, g, sp); break;
        default: e = cudaLaunchKernelEx(&cfg, time_major_scan_kernel<Est, 8, kTmV, kTmCarry>, P, g, sp); break;
        }
        if (e != cudaSuccess) return fail(RLSCAN_ERR_CUDA, "%s: launch failed: %s", name, cudaGetErrorString(e));
    }
    return ok();
}

} // namespace rlscan
