// expect.cuh - expected next-state values of multi-action Retrace.
//
// out[i] = sum over a of pi[i, a] q[i, a] (a = 0 .. A-1 in order) for the n
// elements of the flattened [E, T] array, with q = next_q_values_all and
// pi = next_target_probs, both [E, T, A] (the rl-triton README's Retrace row
// folds the continuation value into next_q_values_all; the expectation
// under the target policy is the V'_t of Retrace, Munos et al. 2016).  The
// recurrence then runs as single-action Retrace on the plane `out`.
#pragma once

#include "host.cuh"

namespace rlscan {

constexpr int kExpectNT = 256;

// A block stages its tile's rows of both planes (contiguous) in shared
// memory with 16-byte loads (scalar loads when `vec` is 0: a base not
// 16-byte aligned, or a tail not a whole number of 16-byte words), then each
// thread sums one element's products (widened to fp32) and the block writes
// its values coalesced.  Dynamic shared memory: 2 kExpectNT A elements of
// ValT.
template <class ValT>
__global__ void __launch_bounds__(kExpectNT) expected_value_kernel(const ValT *__restrict__ q,
                                                                   const ValT *__restrict__ pi,
                                                                   float *__restrict__ out, long long n, int A,
                                                                   int vec) {
    using Bits = typename std::conditional<sizeof(ValT) == 4, uint32_t, uint16_t>::type;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Bits *sq = reinterpret_cast<Bits *>(smem_raw);
    Bits *sp = sq + (size_t)kExpectNT * A;
    const long long e0 = (long long)blockIdx.x * kExpectNT;
    const int cnt = (int)((n - e0) < kExpectNT ? (n - e0) : kExpectNT);
    const int total = cnt * A; // elements of each plane in this tile
    const Bits *gq = reinterpret_cast<const Bits *>(q) + e0 * A;
    const Bits *gp = reinterpret_cast<const Bits *>(pi) + e0 * A;
    if (threadIdx.x == 0) prefetch_l2(gq, 0, total, (int)sizeof(Bits));
    if (threadIdx.x == 1) prefetch_l2(gp, 0, total, (int)sizeof(Bits));
    griddep_wait();
    griddep_launch_dependents();
    constexpr int kPerVec = 16 / (int)sizeof(Bits);
    if (vec && total % kPerVec == 0) {
        const uint4 *q4 = reinterpret_cast<const uint4 *>(gq);
        const uint4 *p4 = reinterpret_cast<const uint4 *>(gp);
#pragma unroll 4
        for (int i = threadIdx.x; i < total / kPerVec; i += kExpectNT) {
            const uint4 vq = __ldcg(q4 + i);
            const uint4 vp = __ldcg(p4 + i);
            reinterpret_cast<uint4 *>(sq)[i] = vq;
            reinterpret_cast<uint4 *>(sp)[i] = vp;
        }
    } else {
        for (int i = threadIdx.x; i < total; i += kExpectNT) {
            sq[i] = __ldcg(gq + i);
            sp[i] = __ldcg(gp + i);
        }
    }
    __syncthreads();
    if (threadIdx.x < cnt) {
        const Bits *qe = sq + (size_t)threadIdx.x * A;
        const Bits *pe = sp + (size_t)threadIdx.x * A;
        float s = 0.0f;
        for (int act = 0; act < A; ++act) {
            if constexpr (sizeof(ValT) == 4) {
                s = fmaf(__uint_as_float(pe[act]), __uint_as_float(qe[act]), s);
            } else {
                s = fmaf(widen(pe[act], ValT()), widen(qe[act], ValT()), s);
            }
        }
        out[e0 + threadIdx.x] = s;
    }
}

// Launch expected_value_kernel over n elements on `stream` (programmatic
// dependent launch allowed, as every launch of the library).
template <class ValT>
cudaError_t launch_expected_values(const ValT *q, const ValT *pi, float *out, long long n, long long A,
                                   cudaStream_t stream) {
    const size_t smem = (size_t)2 * kExpectNT * (size_t)A * sizeof(ValT);
    auto kern = expected_value_kernel<ValT>;
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ceil_div(n, kExpectNT));
    cfg.blockDim = dim3(kExpectNT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, q, pi, out, n, (int)A, aligned16({q, pi}) ? 1 : 0);
}

} // namespace rlscan
