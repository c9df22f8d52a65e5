// scan_core.cuh - the tile scan shared by every rlscan estimator.
//
// The rl-triton paper (arXiv:2608.17641, abstract) solves every estimator as
// one first-order linear recurrence x_t = a_t x_{t-+1} + b_t with the
// associative operator (a1, b1) o (a2, b2) = (a1 a2, a1 b2 + b1), where
// (a2, b2) is the map applied first.  This file holds that operator and the
// scan over the flattened [E*T] array:
//
//   * the array is cut into tiles of S = NT*V consecutive elements, one CTA
//     per tile; each thread owns V consecutive elements (256-bit loads);
//   * rows never leak into each other because each estimator's coefficient
//     builder sets a = 0 on the first element of a row in scan order (the
//     row's last value is folded into b there), the same cut a done makes;
//   * in-thread sequential compose -> warp shuffle scan -> shared-memory scan
//     of warp aggregates -> per-thread carry -> sequential epilogue;
//   * when rows span tiles, two launches over chunks of consecutive warp
//     steps, one chunk per warp: the first writes every chunk's aggregate,
//     the second scans each chunk with the carry composed from the complete
//     aggregates of the chunks before it (no block or warp ever waits for
//     another).
//
// Scan order is memory order for forward recurrences and reversed memory
// order for backward ones.  "Earlier" below always means earlier in scan
// order.
#pragma once

#include <cstdint>
#include <type_traits>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace rlscan {

constexpr unsigned kFullMask = 0xffffffffu;

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------

// Programmatic dependent launch: wait until the preceding grid on the stream
// has completed and its memory is visible (a no-op without the launch
// attribute), and let the next grid start its prologue early.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Hint: bring [p + first, p + first + count) elements of a plane into L2.  The
// range is shrunk to 16-byte boundaries inside it, so nothing outside the
// caller's buffer is touched.  A prefetch has no effect on memory ordering,
// so it may be issued before griddep_wait(), while the previous grid on the
// stream is still running.
__device__ __forceinline__ void prefetch_l2(const void *p, long long first, long long count, int elem_bytes) {
    if (p == nullptr || count <= 0) return;
    const uintptr_t a = reinterpret_cast<uintptr_t>(p) + (uintptr_t)first * (uintptr_t)elem_bytes;
    const uintptr_t lo = (a + 15u) & ~(uintptr_t)15u;
    const uintptr_t hi = (a + (uintptr_t)count * (uintptr_t)elem_bytes) & ~(uintptr_t)15u;
    if (hi <= lo) return;
    const uintptr_t len = hi - lo;
    if (len > 0xffff0u) return; // only tile-sized ranges are prefetched
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(lo), "r"((uint32_t)len) : "memory");
}

// ---------------------------------------------------------------------------
// Scan algebra.  A pair (a, b) is the map x -> a x + b.  combine(p1, p2)
// replaces p1 with p1 o p2 (p2 applied first).  a == 0 cuts the chain: the
// earlier value is not read, so a non-finite value never crosses an episode
// or row boundary.
// ---------------------------------------------------------------------------

__device__ __forceinline__ float apply_pair(float a, float b, float x) { return a == 0.0f ? b : fmaf(a, x, b); }
__device__ __forceinline__ void combine(float &a1, float &b1, float a2, float b2) {
    b1 = apply_pair(a1, b1, b2);
    a1 = a1 * a2;
}
__device__ __forceinline__ float identity_a(float) { return 1.0f; }
__device__ __forceinline__ float identity_b(float) { return 0.0f; }
__device__ __forceinline__ unsigned to_bits(float v) { return __float_as_uint(v); }
__device__ __forceinline__ float from_bits(unsigned u, float) { return __uint_as_float(u); }

// Integer pairs with a 0/1 multiplier: exact two's-complement sums.
__device__ __forceinline__ int32_t apply_pair(uint32_t a, int32_t b, int32_t x) {
    return a ? static_cast<int32_t>(static_cast<uint32_t>(b) + static_cast<uint32_t>(x)) : b;
}
__device__ __forceinline__ void combine(uint32_t &a1, int32_t &b1, uint32_t a2, int32_t b2) {
    b1 = apply_pair(a1, b1, b2);
    a1 = a1 & a2;
}
__device__ __forceinline__ uint32_t identity_a(uint32_t) { return 1u; }
__device__ __forceinline__ int32_t identity_b(int32_t) { return 0; }
__device__ __forceinline__ unsigned to_bits(uint32_t v) { return v; }
__device__ __forceinline__ unsigned to_bits(int32_t v) { return static_cast<unsigned>(v); }
__device__ __forceinline__ uint32_t from_bits(unsigned u, uint32_t) { return u; }
__device__ __forceinline__ int32_t from_bits(unsigned u, int32_t) { return static_cast<int32_t>(u); }

// A pair of independent fp32 recurrences scanned together with the
// component-wise operator: two estimators that share one pass over their
// common inputs (the pair is cut only where both components are).
__device__ __forceinline__ float2 apply_pair(float2 a, float2 b, float2 x) {
    return make_float2(apply_pair(a.x, b.x, x.x), apply_pair(a.y, b.y, x.y));
}
__device__ __forceinline__ void combine(float2 &a1, float2 &b1, float2 a2, float2 b2) {
    b1 = apply_pair(a1, b1, b2);
    a1 = make_float2(a1.x * a2.x, a1.y * a2.y);
}
__device__ __forceinline__ float2 identity_a(float2) { return make_float2(1.0f, 1.0f); }
__device__ __forceinline__ float2 identity_b(float2) { return make_float2(0.0f, 0.0f); }

// The multiplier of a map that ignores its input (a cut chain), and the test
// for one.
__device__ __forceinline__ float cut_a(float) { return 0.0f; }
__device__ __forceinline__ uint32_t cut_a(uint32_t) { return 0u; }
__device__ __forceinline__ float2 cut_a(float2) { return make_float2(0.0f, 0.0f); }
__device__ __forceinline__ bool is_cut(float a) { return a == 0.0f; }
__device__ __forceinline__ bool is_cut(uint32_t a) { return a == 0u; }
__device__ __forceinline__ bool is_cut(float2 a) { return a.x == 0.0f && a.y == 0.0f; }

// Warp shuffles of scan values (full warp).
template <class T>
__device__ __forceinline__ T shfl_down(T v, int d) { return __shfl_down_sync(kFullMask, v, d); }
template <class T>
__device__ __forceinline__ T shfl_up(T v, int d) { return __shfl_up_sync(kFullMask, v, d); }
template <class T>
__device__ __forceinline__ T shfl_idx(T v, int l) { return __shfl_sync(kFullMask, v, l); }
__device__ __forceinline__ float2 shfl_down(float2 v, int d) {
    return make_float2(__shfl_down_sync(kFullMask, v.x, d), __shfl_down_sync(kFullMask, v.y, d));
}
__device__ __forceinline__ float2 shfl_up(float2 v, int d) {
    return make_float2(__shfl_up_sync(kFullMask, v.x, d), __shfl_up_sync(kFullMask, v.y, d));
}
__device__ __forceinline__ float2 shfl_idx(float2 v, int l) {
    return make_float2(__shfl_sync(kFullMask, v.x, l), __shfl_sync(kFullMask, v.y, l));
}

// Inclusive warp scan in scan order: forward = increasing lane, backward =
// decreasing lane.  `width` (a power of two) bounds the distance a value
// must travel: when rows start every `width` lanes, later steps would only
// combine across a row boundary, where a = 0 already cuts the chain.
template <bool kBackward, class AT, class BT>
__device__ __forceinline__ void warp_inclusive_scan(AT &a, BT &b, int lane, int width = 32) {
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        if (d >= width) break;
        if (kBackward) {
            AT ao = shfl_down(a, d);
            BT bo = shfl_down(b, d);
            if (lane + d < 32) combine(a, b, ao, bo);
        } else {
            AT ao = shfl_up(a, d);
            BT bo = shfl_up(b, d);
            if (lane >= d) combine(a, b, ao, bo);
        }
    }
}

// Exclusive value of an inclusive warp scan (identity on the first lane in
// scan order).
template <bool kBackward, class AT, class BT>
__device__ __forceinline__ void warp_exclusive_from_inclusive(AT ia, BT ib, int lane, AT &ea, BT &eb) {
    if (kBackward) {
        ea = shfl_down(ia, 1);
        eb = shfl_down(ib, 1);
        if (lane == 31) { ea = identity_a(ia); eb = identity_b(ib); }
    } else {
        ea = shfl_up(ia, 1);
        eb = shfl_up(ib, 1);
        if (lane == 0) { ea = identity_a(ia); eb = identity_b(ib); }
    }
}

// ---------------------------------------------------------------------------
// Workspace slot of a split-row call (one per chunk of the chunked two
// passes; one per env and split of a time-major call whose rows are split
// over blocks): a map's aggregate, {a, b, 0, 0} or, for a pair of
// recurrences, {a.x, a.y, b.x, b.y}.
// ---------------------------------------------------------------------------
struct TileSlot {
    unsigned w[4];
};
static_assert(sizeof(TileSlot) == 16, "slot is 16 bytes");

// Geometry of one launch over the flattened [E*T] array.
struct Geometry {
    long long n;       // E * T
    long long seq_len; // T
    long long ntiles;  // tiles (tile kernel) or segments per row (time-major kernel)
    long long rows;    // E
    int t_shift;       // log2(T) when T is a power of two, else -1
    int vec_ok;        // every plane pointer of the call is 16-byte aligned
    int scan_lanes;    // warp-local mode: lanes one row spans (a power of two <= 32)
    // Blocks with blockIdx.x below this prefetch their tile into L2 before
    // waiting for the previous grid: the first wave of resident blocks, which
    // overlaps that grid's tail.  Later blocks start once it has finished and
    // load directly (their prefetch would only add L2 requests).
    long long pf_blocks = 1ll << 62;
};

// Where a thread's V elements sit in their rows, as bit masks over k:
// end bit k = element k is the last step of its row (t == T-1), start bit
// k = element k is the first (t == 0), valid bit k = element k exists
// (i0 + k < n); row0 = row of element 0.  When V divides T (the common
// case) a thread's elements share one row, so only element V-1 can end a
// row and only element 0 can start one: one division (a shift for powers of
// two) per thread instead of per-element bookkeeping.
struct RowMasks {
    unsigned end, start, valid;
    long long row0;
    bool fast; // all V elements exist and V divides T: only element V-1 can end a row, only 0 start one
};

// What a launch knows at compile time about its calls, for the coefficient
// builders (`coeffs<V, kCase>`):
//   kCaseAny    truncations and the fast path are decided per call and
//               thread at run time (every variant is compiled in);
//   kCasePlain  no call passes truncations, every thread takes the fast
//               path (V divides T and the array is a whole number of tiles)
//               and every plane is 16-byte aligned: one variant per builder
//               and vector accesses only, a smaller kernel;
//   kCasePlainTrunc  the same with truncations: the fast builder with its
//               truncation logic, vector accesses only (tile kernels).
constexpr int kCaseAny = 0;
constexpr int kCasePlain = 1;
constexpr int kCasePlainTrunc = 2;
template <int V>
__device__ __forceinline__ RowMasks row_masks(long long i0, const Geometry &g) {
    RowMasks m;
    const long long T = g.seq_len;
    long long t0;
    if (g.t_shift >= 0) {
        m.row0 = i0 >> g.t_shift;
        t0 = i0 & (T - 1);
    } else if ((unsigned long long)i0 <= 0xffffffffull && (unsigned long long)T <= 0xffffffffull) {
        const unsigned q = (unsigned)i0 / (unsigned)T;
        m.row0 = q;
        t0 = (unsigned)i0 - q * (unsigned)T;
    } else {
        m.row0 = i0 / T;
        t0 = i0 - m.row0 * T;
    }
    const long long left = g.n - i0;
    m.valid = left >= V ? ((1u << V) - 1u) : (left > 0 ? ((1u << left) - 1u) : 0u);
    m.fast = (T % V == 0) && (left >= V);
    if (T % V == 0) {
        m.end = (t0 + V == T) ? (1u << (V - 1)) : 0u;
        m.start = (t0 == 0) ? 1u : 0u;
    } else {
        m.end = 0u;
        m.start = 0u;
        long long t = t0;
#pragma unroll
        for (int k = 0; k < V; ++k) {
            if (t == T - 1) m.end |= 1u << k;
            if (t == 0) m.start |= 1u << k;
            if (++t == T) t = 0;
        }
    }
    return m;
}
// Row of element k (only needed where element k ends a row).
__device__ __forceinline__ long long row_of(const RowMasks &m, int k) {
    return m.row0 + __popc(m.end & ((1u << k) - 1u));
}

// Per-element tests, folded at compile time on the fast path (k is a
// constant once the element loop is unrolled).
template <bool kFast, int V>
__device__ __forceinline__ bool elem_valid(const RowMasks &m, int k) {
    return kFast || ((m.valid >> k) & 1u);
}
template <bool kFast, int V>
__device__ __forceinline__ bool elem_row_end(const RowMasks &m, int k) {
    return kFast ? (k == V - 1 && ((m.end >> (V - 1)) & 1u)) : ((m.end >> k) & 1u);
}
template <bool kFast, int V>
__device__ __forceinline__ bool elem_row_start(const RowMasks &m, int k) {
    return kFast ? (k == 0 && (m.start & 1u)) : ((m.start >> k) & 1u);
}
template <bool kFast>
__device__ __forceinline__ long long elem_row(const RowMasks &m, int k) {
    return kFast ? m.row0 : row_of(m, k);
}

// Aggregate of a map into a workspace slot (all 16 bytes written).
template <class AT, class BT>
__device__ __forceinline__ void publish_aggregate(TileSlot *slot, AT a, BT b) {
    *reinterpret_cast<uint4 *>(slot) = make_uint4(to_bits(a), to_bits(b), 0u, 0u);
}
__device__ __forceinline__ void publish_aggregate(TileSlot *slot, float2 a, float2 b) {
    *reinterpret_cast<uint4 *>(slot) =
        make_uint4(__float_as_uint(a.x), __float_as_uint(a.y), __float_as_uint(b.x), __float_as_uint(b.y));
}
// The aggregate a slot holds.
template <class AT, class BT>
__device__ __forceinline__ void read_aggregate(const TileSlot *slot, AT &a, BT &b) {
    const uint4 v = *reinterpret_cast<const uint4 *>(slot);
    a = from_bits(v.x, a);
    b = from_bits(v.y, b);
}
__device__ __forceinline__ void read_aggregate(const TileSlot *slot, float2 &a, float2 &b) {
    const uint4 v = *reinterpret_cast<const uint4 *>(slot);
    a = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
    b = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
}

// Slots a lane reads per round trip when composing earlier aggregates.
constexpr int kSlotsPerLane = 4;

// ---------------------------------------------------------------------------
// Vector loads / stores of V consecutive elements (V a multiple of 4).  When
// the thread's elements all exist and every plane is 16-byte aligned (`vec`),
// a plane whose run starts on a 32-byte boundary moves in 256-bit accesses
// (one full 32-byte sector per lane and access: a warp's stores never leave
// half-written sectors for L2 to merge), any other in 128-bit ones; otherwise
// each element is loaded on its own.  Elements at or past n read as zero / are
// not written.  A null plane reads as zeros.
//
// Loads are coherent and cached in L2 only (ld.global.cg), never through the
// read-only path: with programmatic dependent launch this kernel starts while
// the previous grid may still be writing these inputs, so they are not
// read-only for the whole life of this kernel.  Every element is read once,
// so L1 would not help anyway.
// ---------------------------------------------------------------------------

// 256-bit accesses (sm_100 and later): eight 32-bit words at a 32-byte-aligned
// address.  Both are volatile so that they stay after the grid-dependency
// wait like every other memory access.
__device__ __forceinline__ void ld_cg_v8(const void *p, unsigned (&w)[8]) {
    asm volatile("ld.global.cg.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
                 : "l"(p));
}
__device__ __forceinline__ void st_cs_v8(void *p, const unsigned (&w)[8]) {
    asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]), "r"(w[1]),
                 "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
}

// `vec`: the caller's per-thread flag "all planes 16-byte aligned and this
// thread's V elements all exist" (one test per thread, not per plane).
template <int V, class T>
__device__ __forceinline__ void load_plane(const T *__restrict__ p, long long i0, long long n, bool vec,
                                           T (&o)[V]) {
    static_assert(V % 4 == 0, "V must be a multiple of 4");
    static_assert(sizeof(T) == 4, "32-bit planes only");
    if (p == nullptr) {
#pragma unroll
        for (int k = 0; k < V; ++k) o[k] = T(0);
        return;
    }
    if constexpr (V % 8 == 0) {
        if (vec && (reinterpret_cast<uintptr_t>(p + i0) & 31u) == 0) {
#pragma unroll
            for (int k = 0; k < V; k += 8) {
                unsigned w[8];
                ld_cg_v8(p + i0 + k, w);
#pragma unroll
                for (int j = 0; j < 8; ++j) o[k + j] = from_bits(w[j], T());
            }
            return;
        }
    }
    if (vec) {
#pragma unroll
        for (int k = 0; k < V; k += 4) {
            if constexpr (std::is_same<T, float>::value) {
                float4 q = __ldcg(reinterpret_cast<const float4 *>(p + i0 + k));
                o[k] = q.x; o[k + 1] = q.y; o[k + 2] = q.z; o[k + 3] = q.w;
            } else {
                int4 q = __ldcg(reinterpret_cast<const int4 *>(p + i0 + k));
                o[k] = q.x; o[k + 1] = q.y; o[k + 2] = q.z; o[k + 3] = q.w;
            }
        }
    } else {
#pragma unroll
        for (int k = 0; k < V; ++k) o[k] = (i0 + k < n && i0 + k >= 0) ? __ldcg(p + i0 + k) : T(0);
    }
}

template <int V, class T>
__device__ __forceinline__ void store_plane(T *__restrict__ p, long long i0, long long n, bool vec,
                                            const T (&o)[V]) {
    if constexpr (V % 8 == 0) {
        if (vec && (reinterpret_cast<uintptr_t>(p + i0) & 31u) == 0) {
#pragma unroll
            for (int k = 0; k < V; k += 8) {
                unsigned w[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) w[j] = to_bits(o[k + j]);
                st_cs_v8(p + i0 + k, w);
            }
            return;
        }
    }
    if (vec) {
#pragma unroll
        for (int k = 0; k < V; k += 4) {
            if constexpr (std::is_same<T, float>::value) {
                __stcs(reinterpret_cast<float4 *>(p + i0 + k), make_float4(o[k], o[k + 1], o[k + 2], o[k + 3]));
            } else {
                __stcs(reinterpret_cast<int4 *>(p + i0 + k), make_int4(o[k], o[k + 1], o[k + 2], o[k + 3]));
            }
        }
    } else {
#pragma unroll
        for (int k = 0; k < V; ++k)
            if (i0 + k < n) p[i0 + k] = o[k];
    }
}

// Scalar element of a plane (null -> 0), for halos and rare reads.
template <class T>
__device__ __forceinline__ T load_one(const T *__restrict__ p, long long i, long long n) {
    return (p != nullptr && i >= 0 && i < n) ? __ldcg(p + i) : T(0);
}

// Reduced-byte planes, widened to fp32 in registers: bf16 or fp16 values,
// uint8 flags (nonzero = set).  The vector path reads V * sizeof(T) bytes per
// thread in one load (16 bytes for eight bf16, 8 bytes for eight flags).
__device__ __forceinline__ float widen(uint16_t bits, __nv_bfloat16) { return __uint_as_float((uint32_t)bits << 16); }
__device__ __forceinline__ float widen(uint16_t bits, __half) { return __half2float(__ushort_as_half(bits)); }
__device__ __forceinline__ float widen(uint8_t byte, uint8_t) { return byte != 0 ? 1.0f : 0.0f; }

template <int V, class T>
__device__ __forceinline__ void load_plane_widen(const T *__restrict__ p, long long i0, long long n, bool vec,
                                                 float (&o)[V]) {
    if constexpr (std::is_same<T, float>::value) {
        load_plane<V>(p, i0, n, vec, o);
    } else {
        static_assert(sizeof(T) == 1 || sizeof(T) == 2, "8- or 16-bit planes");
        using Bits = typename std::conditional<sizeof(T) == 2, uint16_t, uint8_t>::type;
        const Bits *q = reinterpret_cast<const Bits *>(p);
        if (q == nullptr) {
#pragma unroll
            for (int k = 0; k < V; ++k) o[k] = 0.0f;
            return;
        }
        constexpr int kBytes = V * (int)sizeof(T);
        if (vec) {
            uint32_t w[kBytes / 4 > 0 ? kBytes / 4 : 1];
            if constexpr (kBytes == 32) {
                const uint4 v0 = __ldcg(reinterpret_cast<const uint4 *>(q + i0));
                const uint4 v1 = __ldcg(reinterpret_cast<const uint4 *>(q + i0) + 1);
                w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
                w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
            } else if constexpr (kBytes == 16) {
                const uint4 v = __ldcg(reinterpret_cast<const uint4 *>(q + i0));
                w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
            } else if constexpr (kBytes == 8) {
                const uint2 v = __ldcg(reinterpret_cast<const uint2 *>(q + i0));
                w[0] = v.x; w[1] = v.y;
            } else {
                static_assert(kBytes == 4, "V * sizeof(T) must be 4, 8, 16 or 32 bytes");
                w[0] = __ldcg(reinterpret_cast<const unsigned int *>(q + i0));
            }
#pragma unroll
            for (int k = 0; k < V; ++k) {
                const uint32_t word = w[(k * (int)sizeof(T)) / 4];
                const int shift = 8 * ((k * (int)sizeof(T)) % 4);
                if constexpr (std::is_same<T, __nv_bfloat16>::value) {
                    // a bf16 is the high half of an fp32: one shift or mask
                    o[k] = __uint_as_float(shift == 0 ? (word << 16) : (word & 0xffff0000u));
                } else {
                    o[k] = widen((Bits)(word >> shift), T());
                }
            }
        } else {
#pragma unroll
            for (int k = 0; k < V; ++k) {
                const long long i = i0 + k;
                o[k] = (i >= 0 && i < n) ? widen((Bits)__ldcg(q + i), T()) : 0.0f;
            }
        }
    }
}

// Flags as registers: fp32 flags stay floats, uint8 flags stay integers
// (the byte itself); either way a flag is set iff nonzero.
template <class FlagT>
using FlagReg = typename std::conditional<std::is_same<FlagT, float>::value, float, uint32_t>::type;

template <int V, class T>
__device__ __forceinline__ void load_flags(const T *__restrict__ p, long long i0, long long n, bool vec,
                                           FlagReg<T> (&o)[V]) {
    if constexpr (std::is_same<T, float>::value) {
        load_plane<V>(p, i0, n, vec, o);
    } else {
        static_assert(std::is_same<T, uint8_t>::value, "float or uint8 flags");
        if (p == nullptr) {
#pragma unroll
            for (int k = 0; k < V; ++k) o[k] = 0u;
            return;
        }
        if (vec) {
            uint32_t w[V / 4];
            if constexpr (V == 16) {
                const uint4 v = __ldcg(reinterpret_cast<const uint4 *>(p + i0));
                w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
            } else if constexpr (V == 8) {
                const uint2 v = __ldcg(reinterpret_cast<const uint2 *>(p + i0));
                w[0] = v.x; w[1] = v.y;
            } else {
                static_assert(V == 4, "V must be 4, 8 or 16");
                w[0] = __ldcg(reinterpret_cast<const unsigned int *>(p + i0));
            }
#pragma unroll
            for (int k = 0; k < V; ++k) o[k] = (w[k / 4] >> (8 * (k % 4))) & 0xffu;
        } else {
#pragma unroll
            for (int k = 0; k < V; ++k) {
                const long long i = i0 + k;
                o[k] = (i >= 0 && i < n) ? (uint32_t)__ldcg(p + i) : 0u;
            }
        }
    }
}

template <class T>
__device__ __forceinline__ float load_one_widen(const T *__restrict__ p, long long i, long long n) {
    if constexpr (std::is_same<T, float>::value) {
        return load_one(p, i, n);
    } else {
        using Bits = typename std::conditional<sizeof(T) == 2, uint16_t, uint8_t>::type;
        const Bits *q = reinterpret_cast<const Bits *>(p);
        return (q != nullptr && i >= 0 && i < n) ? widen((Bits)__ldcg(q + i), T()) : 0.0f;
    }
}


// ---------------------------------------------------------------------------
// Element positions.  A builder never indexes memory itself: it asks a
// position policy for "my V elements" of a plane, for the halo element after
// (or before) them, for element k of a sparse plane, and to store its V
// outputs.  Two layouts:
//   RowMajorPos   [E, T] with T contiguous: a thread owns V consecutive
//                 elements of the flattened array (256-bit vector loads; the
//                 halo comes from the neighbouring lane by a shuffle);
//   TimeMajorPos  [T, E] with E contiguous: a thread owns V consecutive
//                 timesteps of one env; lanes are consecutive envs, so each
//                 load instruction reads one contiguous 128-byte line per warp.
// ---------------------------------------------------------------------------
template <int V>
struct RowMajorPos {
    static constexpr bool kRowMajor = true;
    long long i0, n;
    bool vec;
    int lane;
    __device__ __forceinline__ long long index(int k) const { return i0 + k; }
    template <class T>
    __device__ __forceinline__ void load(const T *p, T (&o)[V]) const { load_plane<V>(p, i0, n, vec, o); }
    template <class T>
    __device__ __forceinline__ void load_widen(const T *p, float (&o)[V]) const {
        load_plane_widen<V>(p, i0, n, vec, o);
    }
    template <class T>
    __device__ __forceinline__ void load_flag(const T *p, FlagReg<T> (&o)[V]) const {
        load_flags<V>(p, i0, n, vec, o);
    }
    template <class T>
    __device__ __forceinline__ float fetch_next(const T *p) const {
        return lane == 31 ? load_one_widen(p, i0 + V, n) : 0.0f;
    }
    __device__ __forceinline__ float next(const float (&own)[V], float fetched) const {
        const float h = shfl_down(own[0], 1);
        return lane == 31 ? fetched : h;
    }
    template <class T>
    __device__ __forceinline__ float fetch_prev(const T *p) const {
        return lane == 0 ? load_one_widen(p, i0 - 1, n) : 0.0f;
    }
    __device__ __forceinline__ float prev(const float (&own)[V], float fetched) const {
        const float h = shfl_up(own[V - 1], 1);
        return lane == 0 ? fetched : h;
    }
    template <class T>
    __device__ __forceinline__ float one(const T *p, int k) const { return load_one_widen(p, i0 + k, n); }
    template <class T>
    __device__ __forceinline__ void store(T *p, const T (&o)[V]) const { store_plane<V>(p, i0, n, vec, o); }
};

template <int V>
struct TimeMajorPos {
    static constexpr bool kRowMajor = false;
    long long base; // index of element k = 0: t0 * E + e
    int stride;     // E: elements between consecutive timesteps (the host keeps (V + 1) * E < 2^31)
    long long e;    // the env (row)
    int kbeg, kend; // element k exists iff kbeg <= k < kend (clamped to [-1, V + 1])
    bool fast;      // all V elements exist and V divides T (t0 is a multiple of V)
    __device__ __forceinline__ static TimeMajorPos make(long long e, long long t0, long long E, long long T,
                                                        bool env_ok) {
        TimeMajorPos p;
        p.base = t0 * E + e;
        p.stride = (int)E;
        p.e = e;
        const long long lo = -t0, hi = T - t0;
        p.kbeg = env_ok ? (int)max(min(lo, (long long)V + 1), -1ll) : V + 1;
        p.kend = env_ok ? (int)max(min(hi, (long long)V + 1), -1ll) : V + 1;
        p.fast = env_ok && T % V == 0 && p.kbeg <= 0 && p.kend >= V;
        return p;
    }
    // Element k of plane p: one 64-bit base per plane, 32-bit offsets shared
    // by all planes.
    template <class T_>
    __device__ __forceinline__ const T_ *at(const T_ *p, int k) const { return (p + base) + k * stride; }
    template <class T_>
    __device__ __forceinline__ T_ *at(T_ *p, int k) const { return (p + base) + k * stride; }
    __device__ __forceinline__ bool ok(int k) const { return k >= kbeg && k < kend; }
    template <class T_>
    __device__ __forceinline__ float widen_at(const T_ *p, int k) const {
        if constexpr (std::is_same<T_, float>::value) {
            return __ldcg(at(p, k));
        } else {
            using Bits = typename std::conditional<sizeof(T_) == 2, uint16_t, uint8_t>::type;
            return widen((Bits)__ldcg(reinterpret_cast<const Bits *>(at(p, k))), T_());
        }
    }
    template <class T_>
    __device__ __forceinline__ void load(const T_ *p, T_ (&o)[V]) const {
#pragma unroll
        for (int k = 0; k < V; ++k) o[k] = (p != nullptr && ok(k)) ? __ldcg(at(p, k)) : T_(0);
    }
    template <class T_>
    __device__ __forceinline__ void load_widen(const T_ *p, float (&o)[V]) const {
#pragma unroll
        for (int k = 0; k < V; ++k) o[k] = (p != nullptr && ok(k)) ? widen_at(p, k) : 0.0f;
    }
    template <class T_>
    __device__ __forceinline__ void load_flag(const T_ *p, FlagReg<T_> (&o)[V]) const {
        if constexpr (std::is_same<T_, float>::value) {
            load(p, o);
        } else {
#pragma unroll
            for (int k = 0; k < V; ++k) o[k] = (p != nullptr && ok(k)) ? (uint32_t)__ldcg(at(p, k)) : 0u;
        }
    }
    template <class T_>
    __device__ __forceinline__ float one(const T_ *p, int k) const {
        return (p != nullptr && ok(k)) ? widen_at(p, k) : 0.0f;
    }
    template <class T_>
    __device__ __forceinline__ float fetch_next(const T_ *p) const { return one(p, V); }
    __device__ __forceinline__ float next(const float (&)[V], float fetched) const { return fetched; }
    template <class T_>
    __device__ __forceinline__ float fetch_prev(const T_ *p) const { return one(p, -1); }
    __device__ __forceinline__ float prev(const float (&)[V], float fetched) const { return fetched; }
    template <class T_>
    __device__ __forceinline__ void store(T_ *p, const T_ (&o)[V]) const {
#pragma unroll
        for (int k = 0; k < V; ++k)
            if (ok(k)) __stcs(at(p, k), o[k]);
    }
};

// Row masks of a time-major thread: its V timesteps t0.. of env e (row e).
// Element k is the row's first step iff t0 + k == 0 (k == kbeg >= 0) and its
// last iff t0 + k == T - 1 (k == kend - 1 < V).
template <int V>
__device__ __forceinline__ RowMasks time_major_masks(const TimeMajorPos<V> &pos) {
    RowMasks m;
    m.row0 = pos.e;
    m.valid = 0u;
#pragma unroll
    for (int k = 0; k < V; ++k)
        if (pos.ok(k)) m.valid |= 1u << k;
    m.start = (pos.kbeg >= 0 && pos.kbeg < V && pos.kbeg < pos.kend) ? (1u << pos.kbeg) : 0u;
    m.end = (pos.kend >= 1 && pos.kend <= V && pos.kbeg < pos.kend) ? (1u << (pos.kend - 1)) : 0u;
    m.fast = pos.fast;
    return m;
}

// ---------------------------------------------------------------------------
// The tile kernel.  Est supplies (see estimators.cuh):
//   kBackward, AT, BT, Params, State<V>,
//   load<NT, V>(P, g, pos, S, dyn_smem)         -- every thread, incl. past n
//   coeffs<V, kCase>(P, g, pos, rm, S, a, b)    -- (a, b) per element, identity past n
//   out<V>(P, S, k, x, x_prev, b_k)             -- record output k (x_prev = value
//                                                  of the element before it in scan order,
//                                                  b_k = its scan coefficient b)
//   store<V>(P, g, pos, S)
// where `pos` is the thread's element-position policy (RowMajorPos or
// TimeMajorPos).
// ---------------------------------------------------------------------------

// Scan modes of a tile launch (tiles always hold whole rows; rows that span
// tiles run the chunked two passes below):
//   kModeBlock     warps exchange carries in shared memory
//   kModeWarp      every warp's 32*V elements hold whole rows: no block scan at all
constexpr int kModeBlock = 0;
constexpr int kModeWarp = 2;

// The body of one tile, for a launch whose block `block` owns that tile
// (the tile kernel below, or one part of a fused launch).
template <class Est, int NT, int V, int kMode, int kCase = kCaseAny>
__device__ __forceinline__ void tile_scan_body(const typename Est::Params &P, const Geometry &g,
                                               const long long block, unsigned char *dyn_smem) {
    using AT = typename Est::AT;
    using BT = typename Est::BT;
    constexpr bool kBwd = Est::kBackward;
    constexpr bool kWarpLocal = kMode == kModeWarp;
    constexpr int NW = NT / 32;
    static_assert(NT % 32 == 0 && NW <= 32, "block must be whole warps, at most 32");

    __shared__ AT s_wa[NW];
    __shared__ BT s_wb[NW];
    __shared__ BT s_wx[NW];

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;

    // tile index in scan order
    const long long j = block;
    // Start this tile's DRAM reads before waiting for the previous grid on
    // the stream: the L2 prefetch overlaps them with that grid's tail.  Once
    // the wait returns, let the next grid launch (it waits for this one to
    // complete before touching memory).
    {
        const long long mg = kBwd ? (g.ntiles - 1 - j) : j;
        if ((long long)blockIdx.x < g.pf_blocks) Est::prefetch(P, g, mg * (long long)(NT * V), NT * V);
    }
    griddep_wait();
    griddep_launch_dependents();

    const long long m = kBwd ? (g.ntiles - 1 - j) : j; // tile index in memory
    const long long tile0 = m * (long long)(NT * V);
    const long long i0 = tile0 + (long long)tid * V;

    // the plain cases guarantee vector accesses (every plane 16-byte aligned,
    // every thread's V elements present): no scalar path compiled in
    const bool vec = kCase != kCaseAny || (g.vec_ok != 0 && i0 + V <= g.n);
    const RowMajorPos<V> pos{i0, g.n, vec, lane};
    typename Est::template State<V> S;
    Est::template load<NT, V>(P, g, pos, S, dyn_smem);

    AT a[V];
    BT b[V];
    const RowMasks rm = row_masks<V>(i0, g);
    Est::template coeffs<V, kCase>(P, g, pos, rm, S, a, b);

    // thread aggregate, composed in scan order
    AT ta;
    BT tb;
    if (kBwd) {
        ta = a[V - 1];
        tb = b[V - 1];
#pragma unroll
        for (int k = V - 2; k >= 0; --k) {
            AT na = a[k];
            BT nb = b[k];
            combine(na, nb, ta, tb);
            ta = na;
            tb = nb;
        }
    } else {
        ta = a[0];
        tb = b[0];
#pragma unroll
        for (int k = 1; k < V; ++k) {
            AT na = a[k];
            BT nb = b[k];
            combine(na, nb, ta, tb);
            ta = na;
            tb = nb;
        }
    }

    AT ia = ta;
    BT ib = tb;
    warp_inclusive_scan<kBwd>(ia, ib, lane, kWarpLocal ? g.scan_lanes : 32);
    AT ea;
    BT eb;
    warp_exclusive_from_inclusive<kBwd>(ia, ib, lane, ea, eb);
    BT x;
    if constexpr (kWarpLocal) {
        // the warp's first element in scan order starts a row: nothing flows in
        x = apply_pair(ea, eb, identity_b(tb));
    } else {
        // value flowing into this warp: block scan of warp aggregates
        if (lane == (kBwd ? 0 : 31)) {
            s_wa[warp] = ia;
            s_wb[warp] = ib;
        }
        __syncthreads();
        if (warp == 0) {
            AT wa = lane < NW ? s_wa[lane] : identity_a(ta);
            BT wb = lane < NW ? s_wb[lane] : identity_b(tb);
            warp_inclusive_scan<kBwd>(wa, wb, lane);
            AT wea;
            BT web;
            warp_exclusive_from_inclusive<kBwd>(wa, wb, lane, wea, web);
            // the tile's first warp in scan order starts a row: nothing flows in
            if (lane < NW) s_wx[lane] = apply_pair(wea, web, identity_b(tb));
        }
        __syncthreads();
        x = apply_pair(ea, eb, s_wx[warp]);
    }

    // sequential epilogue over this thread's elements in scan order
    if (kBwd) {
#pragma unroll
        for (int k = V - 1; k >= 0; --k) {
            const BT prev = x;
            x = apply_pair(a[k], b[k], x);
            Est::template out<V>(P, S, k, x, prev, b[k]);
        }
    } else {
#pragma unroll
        for (int k = 0; k < V; ++k) {
            const BT prev = x;
            x = apply_pair(a[k], b[k], x);
            Est::template out<V>(P, S, k, x, prev, b[k]);
        }
    }
    Est::template store<V>(P, g, pos, S);

}

template <class Est, int NT, int V, int kMode, int kCase>
__global__ void __launch_bounds__(NT) tile_scan_kernel(const typename Est::Params P, const Geometry g) {
    extern __shared__ __align__(128) unsigned char dyn_smem[];
    tile_scan_body<Est, NT, V, kMode, kCase>(P, g, (long long)blockIdx.x, dyn_smem);
}

// ---------------------------------------------------------------------------
// Rows that span tiles: chunked two passes.  The flattened array is cut into
// warp steps of 32 V consecutive elements (lane l owns V of them), and the
// steps, in scan order, into equal chunks of consecutive steps, one chunk per
// warp.  A warp walks its chunk step by step and carries its running value
// from one step to the next itself, so no block barrier and no other warp is
// involved inside a chunk:
//   pass one (kChunkAggregates): compose the maps of the chunk's steps into
//     the chunk's aggregate and write it to the chunk's 16-byte slot;
//   pass two (kChunkScan), the next launch on the stream: compose the
//     aggregates of the earlier chunks up to the first that cuts the chain
//     (an episode or row start, a == 0, or the array's start) into the
//     chunk's carry, then scan the steps again with that carry, writing the
//     outputs.
// Every slot pass two reads was written by pass one, which has completed
// before pass two reads it, so nothing waits and the workspace needs no
// initial content.  A launch covers the chunks [chunk_begin, chunk_end), so a
// long array runs in waves whose inputs pass two finds in L2.
// ---------------------------------------------------------------------------
constexpr int kChunkNT = 128; // 4 independent warps per block
constexpr int kChunkV = 16;   // elements per lane and step: two 256-bit loads per plane
                              // (GAE at 16 x 262144: 22.0 us, against 25.7 us with 8)
constexpr int kChunkAggregates = 0;
constexpr int kChunkScan = 1;

struct ChunkSplit {
    TileSlot *slots;       // one per chunk, in scan order
    long long nsteps;      // warp steps over the array: ceil(n / (32 V))
    long long chunk_steps; // steps per chunk (the last chunk may hold fewer)
    long long chunk_begin; // this launch's chunks
    long long chunk_end;
    long long pf_blocks;   // blocks that prefetch their chunks into L2 before the grid wait
};

// Carry into chunk c: the composition of the aggregates of chunks c-1, c-2,
// ... up to the first that cuts the chain, applied to the identity value.
// Called by all 32 lanes of one warp; each round trip reads 32 x M slots
// (lane i: chunks base - i M - m, m = 0 .. M-1, nearest first).
template <class AT, class BT>
__device__ BT chunk_carry(const TileSlot *slots, long long c, int lane, AT proto_a, BT proto_b) {
    constexpr int M = kSlotsPerLane;
    AT acc_a = identity_a(proto_a);
    BT acc_b = identity_b(proto_b);
    for (long long base = c - 1;; base -= 32 * M) {
        const long long k0 = base - (long long)lane * M;
        AT sa[M];
        BT sb[M];
#pragma unroll
        for (int m = 0; m < M; ++m) {
            sa[m] = cut_a(proto_a); // before the array's start: nothing flows in
            sb[m] = identity_b(proto_b);
            if (k0 - m >= 0) read_aggregate(slots + (k0 - m), sa[m], sb[m]);
        }
        AT la = identity_a(proto_a);
        BT lb = identity_b(proto_b);
        bool stop = false;
#pragma unroll
        for (int m = 0; m < M; ++m) {
            if (!stop) {
                combine(la, lb, sa[m], sb[m]);
                stop = is_cut(sa[m]);
            }
        }
        const unsigned stops = __ballot_sync(kFullMask, stop);
        const int last = stops ? __ffs(stops) - 1 : 31;
        if (lane > last) { // farther than the nearest stop: contributes nothing
            la = identity_a(proto_a);
            lb = identity_b(proto_b);
        }
        // ordered composition over lanes 0..last: lane 0 (nearest) applied last
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const AT oa = shfl_down(la, d);
            const BT ob = shfl_down(lb, d);
            if (lane + d < 32) combine(la, lb, oa, ob);
        }
        la = shfl_idx(la, 0);
        lb = shfl_idx(lb, 0);
        combine(acc_a, acc_b, la, lb);
        if (stops) return acc_b;
    }
}

template <class Est, int kPass, int kCase>
__global__ void __launch_bounds__(kChunkNT) chunk_scan_kernel(const typename Est::Params P, const Geometry g,
                                                              const ChunkSplit cs) {
    using AT = typename Est::AT;
    using BT = typename Est::BT;
    constexpr int V = kChunkV;
    constexpr bool kBwd = Est::kBackward;
    constexpr long long SW = 32LL * V; // elements per warp step
    constexpr int WPB = kChunkNT / 32;
    const int lane = threadIdx.x & 31;
    const long long c = cs.chunk_begin + (long long)blockIdx.x * WPB + (threadIdx.x >> 5);

    // L2 prefetch of the block's chunks (consecutive in memory) before
    // waiting for the previous grid, by the first wave of blocks
    if ((long long)blockIdx.x < cs.pf_blocks) {
        const long long cb = cs.chunk_begin + (long long)blockIdx.x * WPB;
        const long long ce = min(cs.chunk_end, cb + WPB);
        const long long sb = cb * cs.chunk_steps, se = min(cs.nsteps, ce * cs.chunk_steps);
        if (se > sb) {
            const long long m0 = kBwd ? cs.nsteps - se : sb; // first memory step of the range
            Est::prefetch(P, g, m0 * SW, (int)min((se - sb) * SW, 1LL << 18)); // at most 1 MB a plane
        }
    }
    griddep_wait();
    griddep_launch_dependents();
    if (c >= cs.chunk_end) return; // the whole warp

    const long long s0 = c * cs.chunk_steps;
    const long long s1 = min(cs.nsteps, s0 + cs.chunk_steps);
    AT agg_a = identity_a(AT{});
    BT agg_b = identity_b(BT{});
    BT carry = identity_b(BT{});
    if constexpr (kPass == kChunkScan) carry = chunk_carry<AT, BT>(cs.slots, c, lane, AT{}, BT{});

    for (long long s = s0; s < s1; ++s) {
        const long long m = kBwd ? (cs.nsteps - 1 - s) : s; // step in memory order
        const long long i0 = m * SW + (long long)lane * V;
        // kCasePlain: every plane 16-byte aligned and every step whole
        const bool vec = kCase == kCasePlain || (g.vec_ok != 0 && i0 + V <= g.n);
        const RowMajorPos<V> pos{i0, g.n, vec, lane};
        typename Est::template State<V> S;
        Est::template load<32, V>(P, g, pos, S, nullptr);
        AT a[V];
        BT b[V];
        const RowMasks rm = row_masks<V>(i0, g);
        Est::template coeffs<V, kCase>(P, g, pos, rm, S, a, b);

        // lane map, composed in scan order
        AT ta;
        BT tb;
        if (kBwd) {
            ta = a[V - 1];
            tb = b[V - 1];
#pragma unroll
            for (int k = V - 2; k >= 0; --k) {
                AT na = a[k];
                BT nb = b[k];
                combine(na, nb, ta, tb);
                ta = na;
                tb = nb;
            }
        } else {
            ta = a[0];
            tb = b[0];
#pragma unroll
            for (int k = 1; k < V; ++k) {
                AT na = a[k];
                BT nb = b[k];
                combine(na, nb, ta, tb);
                ta = na;
                tb = nb;
            }
        }
        AT ia = ta;
        BT ib = tb;
        warp_inclusive_scan<kBwd>(ia, ib, lane);
        // the step's map: the inclusive value of its last lane in scan order
        AT sa = shfl_idx(ia, kBwd ? 0 : 31);
        BT sb = shfl_idx(ib, kBwd ? 0 : 31);
        if constexpr (kPass == kChunkAggregates) {
            combine(sa, sb, agg_a, agg_b); // this step after the earlier ones
            agg_a = sa;
            agg_b = sb;
        } else {
            AT ea;
            BT eb;
            warp_exclusive_from_inclusive<kBwd>(ia, ib, lane, ea, eb);
            BT x = apply_pair(ea, eb, carry);
            if (kBwd) {
#pragma unroll
                for (int k = V - 1; k >= 0; --k) {
                    const BT prev = x;
                    x = apply_pair(a[k], b[k], x);
                    Est::template out<V>(P, S, k, x, prev, b[k]);
                }
            } else {
#pragma unroll
                for (int k = 0; k < V; ++k) {
                    const BT prev = x;
                    x = apply_pair(a[k], b[k], x);
                    Est::template out<V>(P, S, k, x, prev, b[k]);
                }
            }
            Est::template store<V>(P, g, pos, S);
            carry = apply_pair(sa, sb, carry);
        }
    }
    if constexpr (kPass == kChunkAggregates) {
        if (lane == 0) publish_aggregate(cs.slots + c, agg_a, agg_b);
    }
}

// ---------------------------------------------------------------------------
// The time-major kernel, for [T, E] arrays (E contiguous).  A block owns G
// consecutive envs and walks their rows in segments, in scan order.  Within
// a warp, lane l serves env l % G and chunk l / G: the warp covers 32 / G
// chunks of V timesteps of its G envs, so each load instruction of a warp
// reads 32 / G runs of G consecutive envs (whole 32-byte sectors for G >= 8).
// A segment is nw warps x 32 / G chunks x V timesteps.  Chunk aggregates
// are scanned across a warp's chunks with shuffles (stride G lanes), the
// warps of a segment are chained per env through shared memory, and the
// value a segment leaves is the carry into the next one.  Rows never span
// blocks unless the host splits them (below), with a workspace then.
// ---------------------------------------------------------------------------
struct PlaneRef {
    const void *p;
    int bytes; // element size
};

constexpr int kTmMaxWarps = 16;

// Rows of the time-major kernel split over several blocks (few envs with
// long rows): blockIdx.y is the split, each split a run of `sps` consecutive
// segments in scan order.  Pass kTmMaps writes, per env, the map of its
// split (the composition of its elements' (a, b) in scan order) into
// slots[e * nsplit + split]; pass kTmCarry starts each split from the value
// the maps of the splits before it carry in, and writes the outputs.
// kTmWhole runs every row in one block (nsplit = 1, no workspace).
struct TmSplit {
    TileSlot *slots;
    int nsplit;
    int sps;
};
constexpr int kTmWhole = 0;
constexpr int kTmMaps = 1;
constexpr int kTmCarry = 2;

__device__ __forceinline__ void prefetch_line_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

template <class Est, int G, int V, int kPass>
__global__ void __launch_bounds__(kTmMaxWarps * 32) time_major_scan_kernel(const typename Est::Params P,
                                                                           const Geometry g, const TmSplit sp) {
    using AT = typename Est::AT;
    using BT = typename Est::BT;
    constexpr bool kBwd = Est::kBackward;
    constexpr int CPW = 32 / G; // chunks per warp
    static_assert(G >= 1 && G <= 32 && 32 % G == 0, "G divides the warp");
    __shared__ AT s_a[kTmMaxWarps][G];
    __shared__ BT s_b[kTmMaxWarps][G];
    __shared__ BT s_x[kTmMaxWarps][G];
    __shared__ BT s_carry[G];
    __shared__ AT s_ma[G]; // kTmMaps: each env's map of the segments so far
    __shared__ BT s_mb[G];

    const int lane = threadIdx.x & 31;
    const int w = threadIdx.x >> 5;
    const int nw = blockDim.x >> 5;
    const int es = lane % G; // env within the block
    const int cs = lane / G; // chunk within the warp
    const long long E = g.rows, T = g.seq_len;
    const long long e0 = (long long)blockIdx.x * G;
    const long long e = e0 + es;
    const bool env_ok = e < E;
    const int S = nw * CPW * V;       // timesteps per segment (<= 16 * 32 * V)
    const long long nseg = g.ntiles;  // ceil(T / S), from the host
    const int split = blockIdx.y;
    const long long s_begin = (long long)split * sp.sps;            // this block's segments,
    const long long s_end = min(nseg, s_begin + (long long)sp.sps); // in scan order

    // L2 prefetch of the first segment's input rows, before waiting for the
    // previous grid (L2 is coherent, so a prefetched line is never stale)
    {
        const long long t_first = (kBwd ? nseg - 1 - s_begin : s_begin) * S;
        const int rows = (int)((T - t_first) < S ? (T - t_first) : S);
        const int envs = (int)((E - e0) < G ? (E - e0) : G);
#pragma unroll
        for (int plane = 0; plane < Est::kInputPlanes; ++plane) {
            const PlaneRef pr = Est::input_plane(P, plane);
            if (pr.p == nullptr) continue;
            for (int r = threadIdx.x; r < rows; r += blockDim.x) {
                const char *row = static_cast<const char *>(pr.p) + ((t_first + r) * E + e0) * pr.bytes;
                prefetch_line_l2(row);
                const char *last = row + (envs - 1) * pr.bytes;
                if (((uintptr_t)row >> 7) != ((uintptr_t)last >> 7)) prefetch_line_l2(last);
            }
        }
    }
    griddep_wait();
    griddep_launch_dependents();

    if (threadIdx.x < G) {
        const int ee = threadIdx.x;
        BT x = identity_b(BT());
        if constexpr (kPass == kTmCarry) { // the value the earlier splits carry in
            if (e0 + ee < E) {
                const TileSlot *row = sp.slots + (e0 + ee) * sp.nsplit;
                for (int k = 0; k < split; ++k) {
                    AT ka = AT();
                    BT kb = BT();
                    read_aggregate(row + k, ka, kb);
                    x = apply_pair(ka, kb, x);
                }
            }
        }
        s_carry[ee] = x;
        s_ma[ee] = identity_a(AT());
        s_mb[ee] = identity_b(BT());
    }

    for (long long si = s_begin; si < s_end; ++si) {
        const long long seg = kBwd ? nseg - 1 - si : si;
        const long long t0 = seg * S + (w * CPW + cs) * V;
        const TimeMajorPos<V> pos = TimeMajorPos<V>::make(e, t0, E, T, env_ok);
        typename Est::template State<V> St;
        Est::template load<kTmMaxWarps * 32, V>(P, g, pos, St, nullptr);
        AT a[V];
        BT b[V];
        const RowMasks rm = time_major_masks<V>(pos);
        Est::template coeffs<V>(P, g, pos, rm, St, a, b);

        // chunk aggregate, composed in scan order
        AT ia;
        BT ib;
        if (kBwd) {
            ia = a[V - 1];
            ib = b[V - 1];
#pragma unroll
            for (int k = V - 2; k >= 0; --k) {
                AT na = a[k];
                BT nb = b[k];
                combine(na, nb, ia, ib);
                ia = na;
                ib = nb;
            }
        } else {
            ia = a[0];
            ib = b[0];
#pragma unroll
            for (int k = 1; k < V; ++k) {
                AT na = a[k];
                BT nb = b[k];
                combine(na, nb, ia, ib);
                ia = na;
                ib = nb;
            }
        }
        const AT own_a = ia;

        // inclusive scan over the warp's chunks of each env (lanes G apart)
#pragma unroll
        for (int d = 1; d < CPW; d <<= 1) {
            if (kBwd) {
                const AT oa = shfl_down(ia, d * G);
                const BT ob = shfl_down(ib, d * G);
                if (cs + d < CPW) combine(ia, ib, oa, ob);
            } else {
                const AT oa = shfl_up(ia, d * G);
                const BT ob = shfl_up(ib, d * G);
                if (cs >= d) combine(ia, ib, oa, ob);
            }
        }
        AT ea = identity_a(own_a);
        BT eb = identity_b(ib);
        if constexpr (CPW > 1) {
            const AT xa = kBwd ? shfl_down(ia, G) : shfl_up(ia, G);
            const BT xb = kBwd ? shfl_down(ib, G) : shfl_up(ib, G);
            if (kBwd ? (cs + 1 < CPW) : (cs > 0)) {
                ea = xa;
                eb = xb;
            }
        }
        if (cs == (kBwd ? 0 : CPW - 1)) { // the warp's aggregate per env
            s_a[w][es] = ia;
            s_b[w][es] = ib;
        }
        __syncthreads();
        if (kPass == kTmMaps && threadIdx.x < G) { // compose this env's warp maps in scan order
            const int ee = threadIdx.x;
            AT ma = s_ma[ee];
            BT mb = s_mb[ee];
            for (int j = 0; j < nw; ++j) {
                const int ww = kBwd ? nw - 1 - j : j;
                AT na = s_a[ww][ee];
                BT nb = s_b[ww][ee];
                combine(na, nb, ma, mb); // the later warp applied after the map so far
                ma = na;
                mb = nb;
            }
            s_ma[ee] = ma;
            s_mb[ee] = mb;
        } else if (threadIdx.x < G) { // chain this env's warps in scan order
            const int ee = threadIdx.x;
            BT x = s_carry[ee];
            // four warps at a time: their shared loads issue together, ahead
            // of the dependent applies
            for (int j0 = 0; j0 < nw; j0 += 4) {
                AT qa[4];
                BT qb[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int ww = kBwd ? nw - 1 - (j0 + q) : j0 + q;
                    const bool in = j0 + q < nw;
                    qa[q] = in ? s_a[ww][ee] : identity_a(AT());
                    qb[q] = in ? s_b[ww][ee] : identity_b(BT());
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (j0 + q < nw) {
                        const int ww = kBwd ? nw - 1 - (j0 + q) : j0 + q;
                        s_x[ww][ee] = x;
                        x = apply_pair(qa[q], qb[q], x);
                    }
                }
            }
            s_carry[ee] = x;
        }
        __syncthreads();
        if constexpr (kPass == kTmMaps) continue; // maps only: no outputs
        // shared arrays: the next segment writes s_a / s_b before its first
        // barrier, after every read of them here (before this barrier), and
        // s_x / s_carry only after that barrier, when every thread has read
        // s_x below; so no third barrier is needed
        BT x = apply_pair(ea, eb, s_x[w][es]);
        if (kBwd) {
#pragma unroll
            for (int k = V - 1; k >= 0; --k) {
                const BT prev = x;
                x = apply_pair(a[k], b[k], x);
                Est::template out<V>(P, St, k, x, prev, b[k]);
            }
        } else {
#pragma unroll
            for (int k = 0; k < V; ++k) {
                const BT prev = x;
                x = apply_pair(a[k], b[k], x);
                Est::template out<V>(P, St, k, x, prev, b[k]);
            }
        }
        Est::template store<V>(P, g, pos, St);
    }
    if constexpr (kPass == kTmMaps) {
        if (threadIdx.x < G && e0 + threadIdx.x < E)
            publish_aggregate(sp.slots + (e0 + threadIdx.x) * sp.nsplit + split, s_ma[threadIdx.x],
                              s_mb[threadIdx.x]);
    }
}

} // namespace rlscan
