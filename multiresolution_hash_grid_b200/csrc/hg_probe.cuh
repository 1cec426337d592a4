// hg_probe.cuh -- memory-system probes: the ceilings that the encoding's kernels are held
// against, measured on the device they run on.
//
// [Overview-HG] section 3.1: the encoding's cost is its irregular table accesses, not its
// arithmetic. The forward pass is a stream of small random gathers from a table that (at
// the default sizes) sits in L2, and the backward pass a stream of small random fp32
// reductions into one. These kernels issue exactly those accesses, and nothing else, so
// their rates are the roofline denominators:
//   gather  -- one load of W bytes (4, 8, 16 or 32) per lane and operation;
//   red     -- one red.global.add of W fp32 bytes (4, 8 or 16) per lane and operation;
//   red f16 -- one red.global.add.noftz of W bytes of packed fp16 pairs (4, 8 or 16).
// Address patterns (units are W-byte slots of the buffer, the buffer a power of two):
//   kRandom     -- every lane an independent uniformly random unit;
//   kXPair      -- lanes 2k and 2k+1 take units (v ^ K) and ((v + 1) ^ K) for one random v
//                  and K: the x-neighbour pattern of the hash, whose x prime is 1;
//   kSectorPair -- lanes 2k and 2k+1 take the two 16-byte halves of one random 32-byte sector;
//   kLinePair   -- lanes 2k and 2k+1 take two different 32-byte sectors of one random
//                  128-byte line (16-byte units);
//   kStream     -- consecutive lanes take consecutive units (a coalesced sweep).
// Every address is the buffer base plus (unit & (units - 1)) * W, so the probes never
// leave the buffer. Random units come from a stateless 32-bit integer mixer (the
// "lowbias32" finaliser published by C. Wellons), evaluated on (thread, operation).
#pragma once

#include <stdint.h>

namespace hg {
namespace probe {

enum Pattern { kRandom = 0, kXPair = 1, kSectorPair = 2, kLinePair = 3, kStream = 4 };

constexpr int kOpsPerIter = 8;  // independent operations in flight per thread
constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t mix32(uint32_t x) {
    x ^= x >> 16;
    x *= 0x7feb352du;
    x ^= x >> 15;
    x *= 0x846ca68bu;
    x ^= x >> 16;
    return x;
}

// Unit of operation j of thread t (0 <= unit <= mask).
__device__ __forceinline__ uint32_t unit_of(int pattern, uint32_t t, uint32_t nthreads, uint32_t j,
                                            uint32_t seed, uint32_t mask) {
    const uint32_t d = t & 1u;  // position inside a lane pair
    const uint32_t who = pattern == kRandom ? t : (t >> 1);
    const uint32_t h = mix32(who * 2654435761u ^ j * 0x85ebca6bu ^ seed);
    switch (pattern) {
        case kXPair: {
            const uint32_t K = mix32(h ^ 0x5bd1e995u);
            return ((h + d) ^ K) & mask;
        }
        case kSectorPair:  // 16-byte units: a sector holds units 2s and 2s + 1
            return ((h & ~1u) | d) & mask;
        case kLinePair: {  // 16-byte units: a line holds 4 sectors of 2 units
            const uint32_t s0 = h >> 30;
            const uint32_t s1 = (s0 + 1u + (mix32(h) % 3u)) & 3u;
            return ((h & ~7u) | ((d ? s1 : s0) << 1)) & mask;
        }
        case kStream:
            return (j * nthreads + t) & mask;
        default:
            return h & mask;
    }
}

template <int W> struct Gather;
template <> struct Gather<4> {
    static __device__ __forceinline__ float ld(const char* p) {
        float v;
        asm("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(p));
        return v;
    }
};
template <> struct Gather<8> {
    static __device__ __forceinline__ float ld(const char* p) {
        float a, b;
        asm("ld.global.nc.v2.f32 {%0, %1}, [%2];" : "=f"(a), "=f"(b) : "l"(p));
        return a + b;
    }
};
template <> struct Gather<16> {
    static __device__ __forceinline__ float ld(const char* p) {
        float a, b, c, e;
        asm("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(a), "=f"(b), "=f"(c), "=f"(e) : "l"(p));
        return (a + b) + (c + e);
    }
};
template <> struct Gather<32> {
    static __device__ __forceinline__ float ld(const char* p) {
        uint32_t w[8];
        asm("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                     : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
                     : "l"(p));
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) s += __uint_as_float(w[k]);
        return s;
    }
};

template <int W> struct Red;
template <> struct Red<4> {
    static __device__ __forceinline__ void add(char* p, float v) {
        asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
    }
};
template <> struct Red<8> {
    static __device__ __forceinline__ void add(char* p, float v) {
        asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(v), "f"(v) : "memory");
    }
};
template <> struct Red<16> {
    static __device__ __forceinline__ void add(char* p, float v) {
        asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v), "f"(v), "f"(v), "f"(v)
                     : "memory");
    }
};

// fp16 reductions: packed half pairs of 1.0 (0x3c00), 4, 8 or 16 bytes per lane.
template <int W> struct RedHalf;
template <> struct RedHalf<4> {
    static __device__ __forceinline__ void add(char* p) {
        asm volatile("red.global.add.noftz.f16x2 [%0], %1;" ::"l"(p), "r"(0x3c003c00u) : "memory");
    }
};
template <> struct RedHalf<8> {
    static __device__ __forceinline__ void add(char* p) {
        asm volatile("red.global.add.noftz.v2.f16x2 [%0], {%1, %1};" ::"l"(p), "r"(0x3c003c00u) : "memory");
    }
};
template <> struct RedHalf<16> {
    static __device__ __forceinline__ void add(char* p) {
        asm volatile("red.global.add.noftz.v4.f16x2 [%0], {%1, %1, %1, %1};" ::"l"(p), "r"(0x3c003c00u) : "memory");
    }
};

enum Kind { kGather = 0, kRedF32 = 1, kRedF16 = 2 };

// Each thread performs iters * kOpsPerIter operations. Gathers sum what they load and
// store the sum only if it equals a value the caller never puts in the buffer (so the
// loads cannot be dropped and nothing is written in practice).
template <int W, int kKind>
__global__ void __launch_bounds__(kThreads) probe_kernel(char* __restrict__ buf, uint32_t mask, int pattern, int iters,
                                                         uint32_t seed, float* __restrict__ sink) {
    const uint32_t t = blockIdx.x * blockDim.x + threadIdx.x;
    const uint32_t nthreads = gridDim.x * blockDim.x;
    float acc = 0.f;
    for (int it = 0; it < iters; ++it) {
        uint32_t u[kOpsPerIter];
#pragma unroll
        for (int k = 0; k < kOpsPerIter; ++k) u[k] = unit_of(pattern, t, nthreads, (uint32_t)(it * kOpsPerIter + k), seed, mask);
        if constexpr (kKind == kRedF32) {
#pragma unroll
            for (int k = 0; k < kOpsPerIter; ++k) Red<W>::add(buf + (uint64_t)u[k] * W, 1.0f);
        } else if constexpr (kKind == kRedF16) {
#pragma unroll
            for (int k = 0; k < kOpsPerIter; ++k) RedHalf<W>::add(buf + (uint64_t)u[k] * W);
        } else {
            float v[kOpsPerIter];
#pragma unroll
            for (int k = 0; k < kOpsPerIter; ++k) v[k] = Gather<W>::ld(buf + (uint64_t)u[k] * W);
#pragma unroll
            for (int k = 0; k < kOpsPerIter; ++k) acc += v[k];
        }
    }
    if constexpr (kKind == kGather) {
        if (acc == -3.0e38f) *sink = acc;
    }
}

}  // namespace probe
}  // namespace hg
