// hg_device.cuh -- device code of the multiresolution hash-grid encoding for sm_100a.
//
// Sources (cited by page and section; see include/hashgrid.h for the full list):
//   [NeRFace-HG] section 2: voxel of the scaled point, 8 corners, corner hash, trilinear
//                interpolation, concatenation of levels; end of section 2 and section 3:
//                only the sampled table entries receive gradient.
//   [Repro-HG]   section 2.2 (hash), section 3 (layer), section 5 (fp16 tables, a CUDA
//                kernel for the hash).
//   [Overview-HG] section 2.2 (hash formula), section 3.1 (table reads are irregular; the
//                cache hierarchy is what limits them).
//
// Work decomposition. One thread computes one (point, level) pair. A warp always holds 32
// consecutive points of a block tile at ONE level, so its 8 corner gathers per lane hit
// one level's table and neighbouring points share cache sectors. A block owns a tile of BP
// points: it stages the tile's x rows (and, in the backward pass, the upstream-gradient
// rows) in shared memory with coalesced loads, runs its warps over the tile's
// (32-point group, level) items, and (forward) writes the [BP, L*F] output tile back with
// contiguous vector stores. Nothing is saved between forward and backward; the backward
// pass recomputes voxel, indices and weights.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "hg_check.cuh"

namespace hg {

constexpr int kMaxLevels = 32;
constexpr uint32_t kPrimeY = 2654435761u;  // [NeRFace-HG] section 2; [Repro-HG] section 2.2
constexpr uint32_t kPrimeZ = 805459861u;   // (the x prime is 1)

// Per-call level parameters, passed by value (kernel parameter space, read with uniform
// indices by each warp).
struct LevelParams {
    float scale[kMaxLevels];  // (float)N_l
    uint32_t mask;            // T - 1
    int L;
    uint64_t T;               // entries per level table
    // Level groups of the level-major lane-pair kernels: group g is levels
    // [group_lo[g], group_lo[g + 1]), consecutive levels whose table entries that points in
    // the unit cube can reach fit in a shared L2 budget together (one pass per group).
    int ngroups;
    int group_lo[kMaxLevels + 1];
};

// Shared-memory row stride (in floats) of a staged [BP, L*F] tile. The padding keeps the
// per-lane row writes of one level conflict-free for F-wide vector stores.
__host__ __device__ constexpr int row_pad(int F) { return F < 4 ? F : 4; }

// ---------------------------------------------------------------------------------------
// Table entry loads (read-only path). F fp32 or fp16 values -> F fp32 registers.
// fp16 -> fp32 conversion is exact (binary16 values, subnormals included, are all
// representable in binary32).
// ---------------------------------------------------------------------------------------
template <int F, typename TT> struct EntryLoadRaw;

template <> struct EntryLoadRaw<1, float> {
    static __device__ __forceinline__ void load(const float* p, float* e) { e[0] = __ldg(p); }
};
template <> struct EntryLoadRaw<2, float> {
    static __device__ __forceinline__ void load(const float* p, float* e) {
        float2 v = __ldg(reinterpret_cast<const float2*>(p));
        e[0] = v.x; e[1] = v.y;
    }
};
template <> struct EntryLoadRaw<4, float> {
    static __device__ __forceinline__ void load(const float* p, float* e) {
        float4 v = __ldg(reinterpret_cast<const float4*>(p));
        e[0] = v.x; e[1] = v.y; e[2] = v.z; e[3] = v.w;
    }
};
template <> struct EntryLoadRaw<8, float> {
    static __device__ __forceinline__ void load(const float* p, float* e) {
        float4 a = __ldg(reinterpret_cast<const float4*>(p));
        float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
        e[0] = a.x; e[1] = a.y; e[2] = a.z; e[3] = a.w;
        e[4] = b.x; e[5] = b.y; e[6] = b.z; e[7] = b.w;
    }
};
template <> struct EntryLoadRaw<1, __half> {
    static __device__ __forceinline__ void load(const __half* p, float* e) {
        e[0] = __half2float(__ldg(p));
    }
};
template <> struct EntryLoadRaw<2, __half> {
    static __device__ __forceinline__ void load(const __half* p, float* e) {
        float2 v = __half22float2(__ldg(reinterpret_cast<const __half2*>(p)));
        e[0] = v.x; e[1] = v.y;
    }
};
__device__ __forceinline__ float2 h2_bits_to_f2(uint32_t bits) {
    __half2 h = *reinterpret_cast<__half2*>(&bits);
    return __half22float2(h);
}
template <> struct EntryLoadRaw<4, __half> {
    static __device__ __forceinline__ void load(const __half* p, float* e) {
        uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
        float2 a = h2_bits_to_f2(v.x), b = h2_bits_to_f2(v.y);
        e[0] = a.x; e[1] = a.y; e[2] = b.x; e[3] = b.y;
    }
};
template <> struct EntryLoadRaw<8, __half> {
    static __device__ __forceinline__ void load(const __half* p, float* e) {
        uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
        float2 a = h2_bits_to_f2(v.x), b = h2_bits_to_f2(v.y);
        float2 c = h2_bits_to_f2(v.z), d = h2_bits_to_f2(v.w);
        e[0] = a.x; e[1] = a.y; e[2] = b.x; e[3] = b.y;
        e[4] = c.x; e[5] = c.y; e[6] = d.x; e[7] = d.y;
    }
};

// Table entry load through the range check of the checked build (a load outside the table
// reads zeros there; in the regular build the check compiles away).
template <int F, typename TT> struct EntryLoad {
    static __device__ __forceinline__ void load(const TT* p, float* e) {
        if (!in_bounds<kChkTable>(p, F * sizeof(TT))) {
#pragma unroll
            for (int f = 0; f < F; ++f) e[f] = 0.f;
            return;
        }
        EntryLoadRaw<F, TT>::load(p, e);
    }
};

// Point coordinate load (streaming).
__device__ __forceinline__ float ld_x(const float* p) { return in_bounds<kChkX>(p, 4) ? __ldcs(p) : 0.f; }

// Four consecutive coordinates (streaming); p is 16-byte aligned.
__device__ __forceinline__ float4 ld_x4(const float* p) {
    return in_bounds<kChkX>(p, 16) ? __ldcs(reinterpret_cast<const float4*>(p)) : make_float4(0.f, 0.f, 0.f, 0.f);
}

// Block-wide staging of the n coordinates of a tile, src = x + p0 * D (16-byte aligned: the
// library takes x 16-byte aligned, and every tile starts at a multiple of 4 points):
// coalesced float4 loads for the whole groups of four, scalar loads for the tail. put(k, v)
// stores coordinate k of the tile.
template <class Put>
__device__ __forceinline__ void stage_x(const float* __restrict__ src, int n, Put put) {
    const int n4 = n >> 2;
    for (int q = threadIdx.x; q < n4; q += blockDim.x) {
        const float4 v = ld_x4(src + 4 * q);
        put(4 * q, v.x);
        put(4 * q + 1, v.y);
        put(4 * q + 2, v.z);
        put(4 * q + 3, v.w);
    }
    for (int k = 4 * n4 + threadIdx.x; k < n; k += blockDim.x) put(k, ld_x(src + k));
}

// The same into a contiguous, 16-byte-aligned shared-memory array.
__device__ __forceinline__ void stage_x(float* xs, const float* __restrict__ src, int n) {
    const int n4 = n >> 2;
    for (int q = threadIdx.x; q < n4; q += blockDim.x)
        *reinterpret_cast<float4*>(xs + 4 * q) = ld_x4(src + 4 * q);
    for (int k = 4 * n4 + threadIdx.x; k < n; k += blockDim.x) xs[k] = ld_x(src + k);
}

// ---------------------------------------------------------------------------------------
// Sector gathers. The x prime is 1, so the two corners that differ only in x, v0 and
// v0 + 1, hash to (v0 ^ K) and ((v0 + 1) ^ K) for the same K = hash of (y, z): their
// indices agree in every bit above the lowest carry of v0 + 1. Whenever both land in the
// same aligned 32-byte sector of the table, one 256-bit load (sm_100) fetches both entries
// and the L1 sends one sector request to L2 instead of two. The second corner is loaded
// separately only when it lies in another sector.
// ---------------------------------------------------------------------------------------
template <int F, typename TT>
struct Sector {
    static constexpr int kEntryBytes = F * (int)sizeof(TT);       // 2 .. 32
    static constexpr int kPerSector = 32 / kEntryBytes;            // entries per sector
    static constexpr int kWords = kEntryBytes >= 4 ? kEntryBytes / 4 : 1;  // words per entry
};

__device__ __forceinline__ void ld_sector(const void* p, uint32_t (&w)[8]) {
    if (!in_bounds<kChkTable>(p, 32)) {
#pragma unroll
        for (int k = 0; k < 8; ++k) w[k] = 0u;
        return;
    }
    asm("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]),
          "=r"(w[7])
        : "l"(p));
}

// Entry j (0 <= j < kPerSector) of a loaded sector as F fp32 values (select chains, no
// local-memory indexing).
template <int F, typename TT>
__device__ __forceinline__ void sector_entry(const uint32_t (&w)[8], uint32_t j, float* e) {
    using S = Sector<F, TT>;
    constexpr int WE = S::kWords;
    constexpr int G = 8 / WE;                // word groups in a sector
    uint32_t sel[WE];
    const uint32_t jw = (S::kEntryBytes >= 4) ? j : (j >> 1);
#pragma unroll
    for (int k = 0; k < WE; ++k) {
        uint32_t v = w[k];
#pragma unroll
        for (int g = 1; g < G; ++g) v = (jw == (uint32_t)g) ? w[g * WE + k] : v;
        sel[k] = v;
    }
    if constexpr (sizeof(TT) == 4) {
#pragma unroll
        for (int f = 0; f < F; ++f) e[f] = __uint_as_float(sel[f]);
    } else if constexpr (S::kEntryBytes >= 4) {
#pragma unroll
        for (int k = 0; k < WE; ++k) {
            float2 v = h2_bits_to_f2(sel[k]);
            e[2 * k] = v.x;
            e[2 * k + 1] = v.y;
        }
    } else {  // one fp16 value: low or high half of the selected word
        const uint32_t bits = (j & 1) ? (sel[0] >> 16) : (sel[0] & 0xffffu);
        e[0] = __half2float(__ushort_as_half((unsigned short)bits));
    }
}

// L2 policy that keeps lines resident (evict-last): the level-major kernels give it to the
// gathers from, and the reductions into, the level's table or gradient slice, so that the
// streamed rows (x, output, upstream gradient) do not push the slice out of L2.
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
    uint64_t pol;
    asm("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// ---------------------------------------------------------------------------------------
// fp32 vector reductions into global memory (red.global.add, vector forms are sm_90+).
// kKeep adds the evict-last L2 policy (the level-major backward: a 64 MB gradient slice
// next to the streamed rows measured 2.91 ms with it and 3.41 ms without on the 1 GiB
// grid; on L2-resident gradients it changes nothing).
// ---------------------------------------------------------------------------------------
template <int F, bool kKeep = false> struct RedAdd;
template <bool kKeep> struct RedAdd<1, kKeep> {
    static __device__ __forceinline__ void add(float* p, const float* v) {
        if (!in_bounds<kChkGrad>(p, 4)) return;
        if constexpr (kKeep) {
            asm volatile("red.global.add.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v[0]),
                         "l"(l2_evict_last_policy())
                         : "memory");
        } else {
            asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v[0]) : "memory");
        }
    }
};
template <bool kKeep> struct RedAdd<2, kKeep> {
    static __device__ __forceinline__ void add(float* p, const float* v) {
        if (!in_bounds<kChkGrad>(p, 8)) return;
        if constexpr (kKeep) {
            asm volatile("red.global.add.L2::cache_hint.v2.f32 [%0], {%1, %2}, %3;" ::"l"(p), "f"(v[0]), "f"(v[1]),
                         "l"(l2_evict_last_policy())
                         : "memory");
        } else {
            asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(v[0]), "f"(v[1])
                         : "memory");
        }
    }
};
template <bool kKeep> struct RedAdd<4, kKeep> {
    static __device__ __forceinline__ void add(float* p, const float* v) {
        if (!in_bounds<kChkGrad>(p, 16)) return;
        if constexpr (kKeep) {
            asm volatile("red.global.add.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "f"(v[0]),
                         "f"(v[1]), "f"(v[2]), "f"(v[3]), "l"(l2_evict_last_policy())
                         : "memory");
        } else {
            asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v[0]),
                         "f"(v[1]), "f"(v[2]), "f"(v[3])
                         : "memory");
        }
    }
};
template <bool kKeep> struct RedAdd<8, kKeep> {
    static __device__ __forceinline__ void add(float* p, const float* v) {
        RedAdd<4, kKeep>::add(p, v);
        RedAdd<4, kKeep>::add(p + 4, v + 4);
    }
};

// Reductions of the x-corner pair (a, b) of one (y, z) edge into level table dl, always
// as 16-byte red.v4 instructions (L2 reduction throughput is per request, not per byte,
// and uniform widths keep the warp's red instructions converged). For F <= 2 a 16-byte
// unit holds 4 / F entries: when a and b share a unit (for F = 2: v0 even), one red.v4
// carries both; otherwise each goes in its own unit, the unit's other elements receiving
// +0.0, which leaves them unchanged. ra / rb say which of the two is reduced.
template <int F>
__device__ __forceinline__ void unit_vals(uint32_t i, const float* v, float (&u)[4]) {
    constexpr uint32_t kUnit = 4 / F;
    const uint32_t o = (i & (kUnit - 1)) * F;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        float t = 0.f;
#pragma unroll
        for (int f = 0; f < F; ++f) t = (o + f == (uint32_t)k) ? v[f] : t;
        u[k] = t;
    }
}

template <int F, bool kKeep = false>
__device__ __forceinline__ void red_pair(float* dl, uint32_t a, uint32_t b, const float* va,
                                         const float* vb, bool ra = true, bool rb = true) {
    if constexpr (F <= 2) {
        constexpr uint32_t kUnit = 4 / F;
        const bool shared = ra && rb && (a ^ b) < kUnit;
        float ua[4], ub[4];
        unit_vals<F>(a, va, ua);
        unit_vals<F>(b, vb, ub);
        // first instruction: the shared unit, or a's unit, or (only b) b's unit
        float u1[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) u1[k] = shared ? ua[k] + ub[k] : (ra ? ua[k] : ub[k]);
        const uint32_t i1 = ra ? a : b;
        if (ra || rb) RedAdd<4, kKeep>::add(dl + (uint64_t)(i1 & ~(kUnit - 1)) * F, u1);
        // second instruction: b's own unit when both are reduced but do not share one
        if (ra && rb && !shared) RedAdd<4, kKeep>::add(dl + (uint64_t)(b & ~(kUnit - 1)) * F, ub);
    } else {
        if (ra) RedAdd<F, kKeep>::add(dl + (uint64_t)a * F, va);
        if (rb) RedAdd<F, kKeep>::add(dl + (uint64_t)b * F, vb);
    }
}

// fp16 gradient tables: 16-byte red.global.add.noftz.v4.f16x2 (sm_90+) on aligned units of
// 8 halves (8 / F entries). Contributions are rounded to fp16 (round to nearest, subnormals
// kept) and the L2 adds in fp16. Two x-corners share a unit more often than in fp32
// (F = 2: when v0 mod 4 != 3), so fewer reductions reach L2. kKeep: evict-last, as RedAdd.
template <bool kKeep = false>
__device__ __forceinline__ void red_half_unit(__half* p, const float (&u)[8]) {
    if (!in_bounds<kChkGrad>(p, 16)) return;
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        __half2 h = __floats2half2_rn(u[2 * k], u[2 * k + 1]);
        w[k] = *reinterpret_cast<uint32_t*>(&h);
    }
    if constexpr (kKeep) {
        asm volatile("red.global.add.L2::cache_hint.noftz.v4.f16x2 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "r"(w[0]),
                     "r"(w[1]), "r"(w[2]), "r"(w[3]), "l"(l2_evict_last_policy())
                     : "memory");
    } else {
        asm volatile("red.global.add.noftz.v4.f16x2 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]),
                     "r"(w[3])
                     : "memory");
    }
}

template <int F>
__device__ __forceinline__ void unit_vals_half(uint32_t i, const float* v, float (&u)[8]) {
    constexpr uint32_t kUnit = 8 / F;
    const uint32_t o = (i & (kUnit - 1)) * F;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        float t = 0.f;
#pragma unroll
        for (int f = 0; f < F; ++f) t = (o + f == (uint32_t)k) ? v[f] : t;
        u[k] = t;
    }
}

template <int F, bool kKeep = false>
__device__ __forceinline__ void red_pair(__half* dl, uint32_t a, uint32_t b, const float* va, const float* vb,
                                         bool ra = true, bool rb = true) {
    constexpr uint32_t kUnit = 8 / F;
    const bool shared = ra && rb && (a ^ b) < kUnit;
    float ua[8], ub[8], u1[8];
    unit_vals_half<F>(a, va, ua);
    unit_vals_half<F>(b, vb, ub);
#pragma unroll
    for (int k = 0; k < 8; ++k) u1[k] = shared ? ua[k] + ub[k] : (ra ? ua[k] : ub[k]);
    const uint32_t i1 = ra ? a : b;
    if (ra || rb) red_half_unit<kKeep>(dl + (uint64_t)(i1 & ~(kUnit - 1)) * F, u1);
    if (ra && rb && !shared) red_half_unit<kKeep>(dl + (uint64_t)(b & ~(kUnit - 1)) * F, ub);
}

// ---------------------------------------------------------------------------------------
// Voxel, corner indices and trilinear weights of one point at one level.
// [NeRFace-HG] section 2: xs = x * N_l (one fp32 multiply, never fused), v = floor(xs),
// frac = xs - v (exact in fp32). The hash of corner v + d is
//   (v0 + d0) XOR (v1 + d1) * P_y XOR (v2 + d2) * P_z   (mod 2^32),
// and (v_i + 1) * P = v_i * P + P mod 2^32, so each axis needs one multiply for both of
// its offsets. Weight of corner c: product over axes of frac_i (offset 1) or 1 - frac_i.
// ---------------------------------------------------------------------------------------
struct Corners {
    uint32_t idx[8];
    float w[8];
    int v[3];  // the voxel (lower corner)
    float f[3];  // position inside the voxel
};

__device__ __forceinline__ void locate_corners(float x0, float x1, float x2, float scale,
                                               uint32_t mask, Corners& cr) {
    const float xs0 = __fmul_rn(x0, scale);
    const float xs1 = __fmul_rn(x1, scale);
    const float xs2 = __fmul_rn(x2, scale);
    const int v0 = __float2int_rd(xs0);
    const int v1 = __float2int_rd(xs1);
    const int v2 = __float2int_rd(xs2);
    cr.v[0] = v0;
    cr.v[1] = v1;
    cr.v[2] = v2;
    const float f0 = __fsub_rn(xs0, __int2float_rn(v0));
    const float f1 = __fsub_rn(xs1, __int2float_rn(v1));
    const float f2 = __fsub_rn(xs2, __int2float_rn(v2));
    cr.f[0] = f0;
    cr.f[1] = f1;
    cr.f[2] = f2;
    const uint32_t hx0 = (uint32_t)v0, hx1 = hx0 + 1u;
    const uint32_t hy0 = (uint32_t)v1 * kPrimeY, hy1 = hy0 + kPrimeY;
    const uint32_t hz0 = (uint32_t)v2 * kPrimeZ, hz1 = hz0 + kPrimeZ;
    const float g0 = 1.0f - f0, g1 = 1.0f - f1, g2 = 1.0f - f2;
    const float wxy[4] = {g0 * g1, f0 * g1, g0 * f1, f0 * f1};
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint32_t hx = (c & 1) ? hx1 : hx0;
        const uint32_t hy = (c & 2) ? hy1 : hy0;
        const uint32_t hz = (c & 4) ? hz1 : hz0;
        cr.idx[c] = (hx ^ hy ^ hz) & mask;
        cr.w[c] = wxy[c & 3] * ((c & 4) ? f2 : g2);
    }
}

// Stage rows [p0, p0 + nvalid) of a global [*, W] fp32 array into shared memory with row
// stride S (coalesced global reads, V-wide).
template <int V>
__device__ __forceinline__ void stage_rows_in(float* s, const float* __restrict__ gsrc,
                                              int64_t p0, int nvalid, int W, int S) {
    const int per_row = W / V;
    const int total = nvalid * per_row;
    const float* base = gsrc + p0 * (int64_t)W;
    for (int k = threadIdx.x; k < total; k += blockDim.x) {
        const int row = k / per_row;
        const int col = (k - row * per_row) * V;
        if (!in_bounds<kChkDout>(base + (int64_t)row * W + col, 4 * V)) continue;
        if constexpr (V == 4) {
            float4 v = __ldcs(reinterpret_cast<const float4*>(base + (int64_t)row * W + col));
            *reinterpret_cast<float4*>(s + row * S + col) = v;
        } else if constexpr (V == 2) {
            float2 v = __ldcs(reinterpret_cast<const float2*>(base + (int64_t)row * W + col));
            *reinterpret_cast<float2*>(s + row * S + col) = v;
        } else {
            s[row * S + col] = __ldcs(base + (int64_t)row * W + col);
        }
    }
}

template <int V>
__device__ __forceinline__ void stage_rows_out(const float* s, float* __restrict__ gdst,
                                               int64_t p0, int nvalid, int W, int S) {
    const int per_row = W / V;
    const int total = nvalid * per_row;
    float* base = gdst + p0 * (int64_t)W;
    for (int k = threadIdx.x; k < total; k += blockDim.x) {
        const int row = k / per_row;
        const int col = (k - row * per_row) * V;
        if (!in_bounds<kChkOut>(base + (int64_t)row * W + col, 4 * V)) continue;
        if constexpr (V == 4) {
            __stcs(reinterpret_cast<float4*>(base + (int64_t)row * W + col),
                   *reinterpret_cast<const float4*>(s + row * S + col));
        } else if constexpr (V == 2) {
            __stcs(reinterpret_cast<float2*>(base + (int64_t)row * W + col),
                   *reinterpret_cast<const float2*>(s + row * S + col));
        } else {
            __stcs(base + (int64_t)row * W + col, s[row * S + col]);
        }
    }
}

template <int F>
__device__ __forceinline__ void store_smem_entry(float* s, const float* v) {
    if constexpr (F == 1) {
        s[0] = v[0];
    } else if constexpr (F == 2) {
        *reinterpret_cast<float2*>(s) = make_float2(v[0], v[1]);
    } else {
#pragma unroll
        for (int j = 0; j < F; j += 4)
            *reinterpret_cast<float4*>(s + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
    }
}

template <int F>
__device__ __forceinline__ void load_smem_entry(const float* s, float* v) {
    if constexpr (F == 1) {
        v[0] = s[0];
    } else if constexpr (F == 2) {
        float2 a = *reinterpret_cast<const float2*>(s);
        v[0] = a.x; v[1] = a.y;
    } else {
#pragma unroll
        for (int j = 0; j < F; j += 4) {
            float4 a = *reinterpret_cast<const float4*>(s + j);
            v[j] = a.x; v[j + 1] = a.y; v[j + 2] = a.z; v[j + 3] = a.w;
        }
    }
}

// Dynamic shared memory of one block: x tile [BP*3] then a data tile [BP * S].
__host__ __device__ constexpr size_t tile_smem_bytes(int BP, int L, int F) {
    return sizeof(float) * ((size_t)BP * 3 + (size_t)BP * (L * F + row_pad(F)));
}

// ---------------------------------------------------------------------------------------
// Forward kernel. Grid: one block per BP-point tile.
// kGatherCorner: one F-wide load per corner. kGatherSector: one 256-bit sector load per
// x-corner pair plus a predicated load of the second corner when it lies in another sector
// (needs a 32-byte-aligned table). kGatherPair: the same with 16-byte units (entries of at
// most 8 bytes; wider entries load per corner).
// ---------------------------------------------------------------------------------------
enum GatherMode { kGatherCorner = 0, kGatherSector = 1, kGatherPair = 2, kGatherLanes = 3 };

// 16-byte read-only load.
__device__ __forceinline__ void ld_unit(const void* p, uint32_t (&w)[4]) {
    if (!in_bounds<kChkTable>(p, 16)) {
        w[0] = w[1] = w[2] = w[3] = 0u;
        return;
    }
    uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
}

// Entry j of a loaded 16-byte unit (entries of at most 8 bytes: 16 / E entries per unit).
template <int F, typename TT>
__device__ __forceinline__ void unit_entry(const uint32_t (&w)[4], uint32_t j, float* e) {
    constexpr int E = F * (int)sizeof(TT);
    static_assert(E <= 8, "a 16-byte unit holds at least two entries");
    uint32_t padded[8] = {w[0], w[1], w[2], w[3], w[0], w[1], w[2], w[3]};
    // reuse the sector decoder on the first half: entries beyond the unit never occur
    sector_entry<F, TT>(padded, j, e);
}

// The two 8-byte entries of a 16-byte unit (F = 2 fp32 or F = 4 fp16).
template <int F, typename TT>
__device__ __forceinline__ void unit8_entries(const uint4& u, float* lo, float* hi) {
    if constexpr (std::is_same<TT, float>::value) {
        lo[0] = __uint_as_float(u.x); lo[1] = __uint_as_float(u.y);
        hi[0] = __uint_as_float(u.z); hi[1] = __uint_as_float(u.w);
    } else {
        const float2 a = h2_bits_to_f2(u.x), b = h2_bits_to_f2(u.y), c = h2_bits_to_f2(u.z), d = h2_bits_to_f2(u.w);
        lo[0] = a.x; lo[1] = a.y; lo[2] = b.x; lo[3] = b.y;
        hi[0] = c.x; hi[1] = c.y; hi[2] = d.x; hi[3] = d.y;
    }
}

// kSplit (per-corner gathers of 8-byte entries only): the x prime is 1, so corners
// (v0, y, z) and (v0 + 1, y, z) hash to (v0 ^ K) and ((v0 + 1) ^ K), and all four x-pairs of
// a point differ by the same v0 ^ (v0 + 1). For even v0 that is 1 and each pair fills one
// aligned 16-byte unit: lanes with even v0 make four 16-byte loads instead of eight 8-byte
// ones, halving their L1 wavefronts, at the price of a divergent branch. Measured on B200
// (2^20 ray samples): faster inside the fused MLP kernel (309 -> 289 us), slower in the
// plain forward (250 -> 266 us) and dL/dx (285 -> 293 us), so only the MLP enables it, for
// fp32 tables (with fp16 ones the branch spills at 40 registers).
template <int F, typename TT, int kGather, bool kSplit = false>
__device__ __forceinline__ void gather_corners(const TT* __restrict__ tl, const Corners& cr,
                                               float (&e)[8][F]) {
    constexpr int E = F * (int)sizeof(TT);
    if constexpr (kGather == kGatherCorner && kSplit && E == 8) {
        if ((cr.idx[0] ^ cr.idx[1]) == 1u) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t a = cr.idx[2 * q];
                const TT* pu = tl + (uint64_t)(a & ~1u) * F;
                const uint4 u = in_bounds<kChkTable>(pu, 16) ? __ldg(reinterpret_cast<const uint4*>(pu))
                                                              : make_uint4(0u, 0u, 0u, 0u);
                float lo[F], hi[F];
                unit8_entries<F, TT>(u, lo, hi);
                const bool a_lo = (a & 1u) == 0;
#pragma unroll
                for (int f = 0; f < F; ++f) {
                    e[2 * q][f] = a_lo ? lo[f] : hi[f];
                    e[2 * q + 1][f] = a_lo ? hi[f] : lo[f];
                }
            }
        } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) EntryLoad<F, TT>::load(tl + (uint64_t)cr.idx[c] * F, e[c]);
        }
    } else if constexpr (kGather == kGatherCorner || (kGather == kGatherPair && E > 8)) {
#pragma unroll
        for (int c = 0; c < 8; ++c) EntryLoad<F, TT>::load(tl + (uint64_t)cr.idx[c] * F, e[c]);
    } else if constexpr (kGather == kGatherPair) {
        constexpr uint32_t kPer = 16 / E;  // entries per 16-byte unit
        uint32_t w[4][4];
        float far[4][F];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t a = cr.idx[2 * q], b = cr.idx[2 * q + 1];
            ld_unit(tl + (uint64_t)(a & ~(kPer - 1)) * F, w[q]);
            if ((a ^ b) >= kPer) EntryLoad<F, TT>::load(tl + (uint64_t)b * F, far[q]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t a = cr.idx[2 * q], b = cr.idx[2 * q + 1];
            unit_entry<F, TT>(w[q], a & (kPer - 1), e[2 * q]);
            float near[F];
            unit_entry<F, TT>(w[q], b & (kPer - 1), near);
            const bool same = (a ^ b) < kPer;
#pragma unroll
            for (int f = 0; f < F; ++f) e[2 * q + 1][f] = same ? near[f] : far[q][f];
        }
    } else {
        using S = Sector<F, TT>;
        constexpr uint32_t kPer = S::kPerSector;
        uint32_t w[4][8];
        float far[4][F];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t a = cr.idx[2 * q], b = cr.idx[2 * q + 1];
            ld_sector(tl + (uint64_t)(a & ~(kPer - 1)) * F, w[q]);
            if ((a ^ b) >= kPer) EntryLoad<F, TT>::load(tl + (uint64_t)b * F, far[q]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t a = cr.idx[2 * q], b = cr.idx[2 * q + 1];
            sector_entry<F, TT>(w[q], a & (kPer - 1), e[2 * q]);
            float near[F];
            sector_entry<F, TT>(w[q], b & (kPer - 1), near);
            const bool same = (a ^ b) < kPer;
#pragma unroll
            for (int f = 0; f < F; ++f) e[2 * q + 1][f] = same ? near[f] : far[q][f];
        }
    }
}

// Per-corner gathers run 3 blocks of 512 threads per SM (<= 42 registers: more warps keep
// more gathers in flight, measured 10-15% faster than the compiler's own choice); sector
// gathers and F = 8 need more registers: 2 blocks per SM (<= 64 registers), and one
// block for sector gathers of F = 8.
__host__ __device__ constexpr int forward_min_blocks(int F, int gather) {
    return gather == kGatherSector ? (F == 8 ? 1 : 2) : (gather == kGatherPair || F == 8) ? 2 : 3;
}

template <int F, typename TT, int BP, int kGather>
__global__ void __launch_bounds__(512, forward_min_blocks(F, kGather)) forward_kernel(LevelParams lp, const float* __restrict__ x,
                                                      int64_t N, const TT* __restrict__ table,
                                                      float* __restrict__ out) {
    extern __shared__ __align__(16) float smem[];
    const int L = lp.L;
    const int W = L * F;
    const int S = W + row_pad(F);
    float* xs = smem;
    float* os = smem + BP * 3;
    const int64_t p0 = (int64_t)blockIdx.x * BP;
    const int nvalid = (int)min((int64_t)BP, N - p0);

    stage_x(xs, x + p0 * 3, nvalid * 3);
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    const int items = (BP / 32) * L;
    for (int it = warp; it < items; it += nwarps) {
        const int q = it / L;
        const int l = it - q * L;
        const int pl = q * 32 + lane;
        if (pl < nvalid) {
            Corners cr;
            locate_corners(xs[pl * 3 + 0], xs[pl * 3 + 1], xs[pl * 3 + 2], lp.scale[l], lp.mask, cr);
            const TT* tl = table + (uint64_t)l * lp.T * F;
            float e[8][F];
            gather_corners<F, TT, kGather>(tl, cr, e);
            float o[F];
#pragma unroll
            for (int f = 0; f < F; ++f) {
                float acc = cr.w[0] * e[0][f];
#pragma unroll
                for (int c = 1; c < 8; ++c) acc = fmaf(cr.w[c], e[c][f], acc);
                o[f] = acc;
            }
            store_smem_entry<F>(os + pl * S + l * F, o);
        }
    }
    __syncthreads();
    stage_rows_out<(F < 4 ? F : 4)>(os, out, p0, nvalid, W, S);
}

// ---------------------------------------------------------------------------------------
// Lane-pair forward (kGatherLanes). The x prime is 1, so a corner and its x-neighbour hash to
// (v0 ^ K) and ((v0 + 1) ^ K) for the same K: their indices differ only below the lowest
// carry of v0 + 1, so the two entries share a 32-byte sector most of the time (F = 2 fp32:
// 3 times in 4) and a 128-byte line almost always (15 times in 16). Here two neighbouring
// lanes work on one (point, level): lane d0 = lane & 1 gathers the 4 corners whose x offset
// is d0. Each gather instruction then carries both x-neighbours of 16 cell edges, and the
// L1 serves a sector (and sends a line request to L2) once for both lanes, where one lane
// per point loads the two neighbours in different instructions. The pair adds its two
// partial sums with one shuffle and each lane stores half of the F outputs.
// ---------------------------------------------------------------------------------------
struct HalfCorners {
    uint32_t idx[4];  // corner k: y offset k & 1, z offset k >> 1 (full corner d0 + 2k)
    float w[4];
};

// The 4 corners with x offset d0 of one point at one level; weights are the same fp32
// products, in the same order, as locate_corners computes for those corners.
__device__ __forceinline__ void locate_half(float x0, float x1, float x2, float scale, uint32_t mask, uint32_t d0,
                                            HalfCorners& hc) {
    const float xs0 = __fmul_rn(x0, scale);
    const float xs1 = __fmul_rn(x1, scale);
    const float xs2 = __fmul_rn(x2, scale);
    const int v0 = __float2int_rd(xs0);
    const int v1 = __float2int_rd(xs1);
    const int v2 = __float2int_rd(xs2);
    const float f0 = __fsub_rn(xs0, __int2float_rn(v0));
    const float f1 = __fsub_rn(xs1, __int2float_rn(v1));
    const float f2 = __fsub_rn(xs2, __int2float_rn(v2));
    const uint32_t hx = (uint32_t)v0 + d0;
    const uint32_t hy0 = (uint32_t)v1 * kPrimeY, hy1 = hy0 + kPrimeY;
    const uint32_t hz0 = (uint32_t)v2 * kPrimeZ, hz1 = hz0 + kPrimeZ;
    const float wx = d0 ? f0 : 1.0f - f0;
    const float wxy[2] = {wx * (1.0f - f1), wx * f1};
    const float g2 = 1.0f - f2;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        hc.idx[k] = (hx ^ ((k & 1) ? hy1 : hy0) ^ ((k & 2) ? hz1 : hz0)) & mask;
        hc.w[k] = wxy[k & 1] * ((k & 2) ? f2 : g2);
    }
}

// Gathers and interpolates the lane's 4 corners; returns the pair's full sums in o (both
// lanes get the same values: a + b == b + a in IEEE arithmetic).
template <int F, typename TT>
__device__ __forceinline__ void interpolate_pair(const TT* __restrict__ tl, const HalfCorners& hc, unsigned pair,
                                                 float (&o)[F]) {
    float e[4][F];
#pragma unroll
    for (int k = 0; k < 4; ++k) EntryLoad<F, TT>::load(tl + (uint64_t)hc.idx[k] * F, e[k]);
#pragma unroll
    for (int f = 0; f < F; ++f) {
        float acc = hc.w[0] * e[0][f];
#pragma unroll
        for (int k = 1; k < 4; ++k) acc = fmaf(hc.w[k], e[k][f], acc);
        o[f] = acc + __shfl_xor_sync(pair, acc, 1);
    }
}

// Lane d0 of a pair writes outputs [d0 * F/2, (d0 + 1) * F/2) of the (point, level) at p
// (F = 1: lane 0 writes the one output).
template <int F, bool kStreaming>
__device__ __forceinline__ void store_half(float* p, const float (&o)[F], uint32_t d0) {
    if constexpr (F == 1) {
        if (d0 == 0) {
            if constexpr (kStreaming) {
                if (in_bounds<kChkOut>(p, 4)) __stcs(p, o[0]);
            } else {
                *p = o[0];
            }
        }
    } else {
        constexpr int H = F / 2;
        float v[H];
#pragma unroll
        for (int j = 0; j < H; ++j) v[j] = d0 ? o[H + j] : o[j];
        float* q = p + d0 * H;
        if constexpr (kStreaming) {
            if (!in_bounds<kChkOut>(q, 4 * H)) return;
        }
        if constexpr (H == 1) {
            if constexpr (kStreaming) __stcs(q, v[0]); else *q = v[0];
        } else if constexpr (H == 2) {
            const float2 t = make_float2(v[0], v[1]);
            if constexpr (kStreaming) __stcs(reinterpret_cast<float2*>(q), t); else *reinterpret_cast<float2*>(q) = t;
        } else {
            const float4 t = make_float4(v[0], v[1], v[2], v[3]);
            if constexpr (kStreaming) __stcs(reinterpret_cast<float4*>(q), t); else *reinterpret_cast<float4*>(q) = t;
        }
    }
}

// Lane pairs hold half a point's corners each, so fewer registers than one lane per point:
// 4 blocks of 512 threads per SM for F <= 2 (<= 32 registers), 3 for F = 4, 2 for F = 8.
__host__ __device__ constexpr int forward_lanes_min_blocks(int F) { return F <= 2 ? 4 : (F == 4 ? 3 : 2); }

template <int F, typename TT, int BP>
__global__ void __launch_bounds__(512, forward_lanes_min_blocks(F))
    forward_kernel_lanes(LevelParams lp, const float* __restrict__ x, int64_t N, const TT* __restrict__ table,
                         float* __restrict__ out) {
    extern __shared__ __align__(16) float smem[];
    const int L = lp.L;
    const int W = L * F;
    const int S = W + row_pad(F);
    float* xs = smem;
    float* os = smem + BP * 3;
    const int64_t p0 = (int64_t)blockIdx.x * BP;
    const int nvalid = (int)min((int64_t)BP, N - p0);

    // scalar loads here: the float4 staging of the other tile kernels measured 1% slower on
    // uniform points for this kernel (78.7 against 77.9 us per 2^18 points)
    for (int i = threadIdx.x; i < nvalid * 3; i += blockDim.x) xs[i] = ld_x(x + p0 * 3 + i);
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    const uint32_t d0 = lane & 1;
    const unsigned pair = 3u << (lane & 30);
    const int items = (BP / 16) * L;  // a warp item: 16 points at one level
    for (int it = warp; it < items; it += nwarps) {
        const int q = it / L;
        const int l = it - q * L;
        const int pl = q * 16 + (lane >> 1);
        if (pl < nvalid) {  // both lanes of a pair take the same branch
            HalfCorners hc;
            locate_half(xs[pl * 3 + 0], xs[pl * 3 + 1], xs[pl * 3 + 2], lp.scale[l], lp.mask, d0, hc);
            float o[F];
            interpolate_pair<F, TT>(table + (uint64_t)l * lp.T * F, hc, pair, o);
            store_half<F, false>(os + pl * S + l * F, o, d0);
        }
    }
    __syncthreads();
    stage_rows_out<(F < 4 ? F : 4)>(os, out, p0, nvalid, W, S);
}

// ---------------------------------------------------------------------------------------
// Backward kernel (table gradient). Grid: one block per BP-point tile. Each (point, level,
// corner) contributes w_c * dL_dout[p][l*F..] to the level's gradient table.
//
// Grouped reductions (coherent batches, e.g. consecutive samples along rays): a warp first
// groups its 32 x 8 contributions by 16-byte gradient unit, then issues one red.v4 per
// distinct unit. Consecutive samples of a ray share voxels at coarse levels and voxel faces
// at finer ones, so far fewer reductions reach L2, whose reduction rate bounds this pass.
// Grouping uses only integer shared-memory atomics (native; fp32 shared-memory atomics are
// compare-and-swap loops that serialise when lanes collide): a direct-mapped table of 512
// slots maps unit keys to slots (atomicCAS; a contribution whose slot already holds another
// key is reduced on its own right away, so there is no probing), each grouped contribution
// is pushed onto its slot's list (atomicExch), and after a warp barrier each lane walks the
// lists of its slots, summing in registers.
//
// Backward modes: kAtomicOnly -- every (point, level) reduces its own 8 contributions, the
// two x-corners of an edge merged into one 16-byte red when they share an aligned unit
// (red_pair). kGroupAlways -- every warp item is grouped. kAdaptive -- a warp item is
// grouped when at least half of its lanes sit in a voxel adjacent to (or equal to) the
// previous lane's voxel, i.e. when neighbouring points can share corners; otherwise it
// takes the kAtomicOnly path (uniformly scattered points never share corners in a warp).
// ---------------------------------------------------------------------------------------
enum BackwardMode { kAtomicOnly = 0, kAdaptive = 1, kGroupAlways = 2, kRunMerge = 3 };

constexpr int kGroupSlots = 512;
constexpr int kGroupItems = 256;           // 32 lanes x 8 corners
constexpr uint32_t kEmpty = 0xffffffffu;
constexpr uint32_t kEnd = 0xffffu;

// Shared memory of one warp: keys[512], head[512], next[256], occupied[256] (u32),
// values[F][256] (f32).
__host__ __device__ constexpr size_t group_smem_bytes(int warps, int F) {
    return (size_t)warps * (2 * kGroupSlots * sizeof(uint32_t) +
                            (size_t)kGroupItems * (2 * sizeof(uint32_t) + (size_t)F * sizeof(float)));
}

template <int F>
struct GroupWarp {
    static constexpr uint32_t kUnit = 4 / F;  // table entries per 16-byte unit
    uint32_t* keys;  // [kGroupSlots]
    uint32_t* head;  // [kGroupSlots]
    uint32_t* next;  // [kGroupItems], contribution id = corner * 32 + lane (conflict-free)
    uint32_t* occ;   // [kGroupItems], slots claimed in this warp item, in claim order
    float* vals;     // [F][kGroupItems] (structure of arrays: conflict-free)
    uint32_t nocc;   // number of claimed slots (warp-uniform)

    __device__ __forceinline__ GroupWarp(char* base, int warp) : nocc(0) {
        char* w = base + (size_t)warp * group_smem_bytes(1, F);
        keys = reinterpret_cast<uint32_t*>(w);
        head = keys + kGroupSlots;
        next = head + kGroupSlots;
        occ = next + kGroupItems;
        vals = reinterpret_cast<float*>(occ + kGroupItems);
    }

    __device__ __forceinline__ void clear(int lane) {
        for (int s = lane; s < kGroupSlots; s += 32) {
            keys[s] = kEmpty;
            head[s] = kEmpty;
        }
    }

    // The lane's 8 contributions v[c] (F values each) to entries idx[c] of level table dl.
    // The 8 slot claims and the 8 list pushes are each issued back to back.
    // `vmask` is the ballot of the lanes that push (a prefix of the warp).
    __device__ __forceinline__ void push8(float* dl, const uint32_t* idx, const float (*v)[F], int lane,
                                          uint32_t vmask) {
        uint32_t slot[8], prev[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint32_t key = idx[c] / kUnit;
            slot[c] = (key * 2654435761u) >> 23;  // 9 bits: kGroupSlots == 512
            prev[c] = atomicCAS(keys + slot[c], kEmpty, key);
        }
        // Record newly claimed slots (at most one claim per slot, <= 256 per item).
        const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const bool claimed = prev[c] == kEmpty;
            const uint32_t b = __ballot_sync(vmask, claimed);
            if (claimed) occ[nocc + __popc(b & lt)] = slot[c];
            nocc += __popc(b);
        }
        bool mine[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint32_t key = idx[c] / kUnit;
            mine[c] = prev[c] == kEmpty || prev[c] == key;
            if (!mine[c]) {  // slot taken by another unit: reduce this one directly
                RedAdd<F>::add(dl + (uint64_t)idx[c] * F, v[c]);
            } else {
#pragma unroll
                for (int f = 0; f < F; ++f) vals[f * kGroupItems + c * 32 + lane] = v[c][f];
            }
        }
        uint32_t old[8];
#pragma unroll
        for (int c = 0; c < 8; ++c)
            if (mine[c]) old[c] = atomicExch(head + slot[c], (uint32_t)(c * 32 + lane));
#pragma unroll
        for (int c = 0; c < 8; ++c)
            if (mine[c]) next[c * 32 + lane] = (old[c] & kEnd) | ((idx[c] & (kUnit - 1)) << 16);
    }

    // After __syncwarp(): one red.v4 per claimed slot, then the slots are emptied.
    __device__ __forceinline__ void flush(float* dl, int lane) {
        nocc = __shfl_sync(0xffffffffu, nocc, 0);  // lanes past the tail did not push
        for (uint32_t j = lane; j < nocc; j += 32) {
            const uint32_t s = occ[j];
            const uint32_t key = keys[s];
            float u[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t id = head[s] & kEnd;
            while (id != kEnd) {
                const uint32_t n = next[id];
                const uint32_t off = (n >> 16) * F;
#pragma unroll
                for (int f = 0; f < F; ++f) {
                    const float v = vals[f * kGroupItems + id];
#pragma unroll
                    for (int k = 0; k < 4; ++k) u[k] += (off + f == (uint32_t)k) ? v : 0.f;
                }
                id = n & kEnd;
            }
            RedAdd<4>::add(dl + (uint64_t)key * 4, u);
            keys[s] = kEmpty;
            head[s] = kEmpty;
        }
        nocc = 0;
    }
};

// Grouping modes run 8 warps per block (their tables take 8-10 KB of shared memory per
// warp): 3 blocks per SM, 2 for F = 4. The plain mode runs 16 warps per block.
__host__ __device__ constexpr int backward_threads(int mode) { return mode == kAtomicOnly ? 512 : 256; }

template <int F, int BP, int kMode, typename GT = float>
__device__ __forceinline__ void backward_body(const LevelParams& lp, const float* __restrict__ x,
                                              const float* __restrict__ dout, int64_t N,
                                              GT* __restrict__ dtable) {
    static_assert(kMode == kAtomicOnly || F <= 4, "grouped units are 16 bytes");
    extern __shared__ __align__(16) float smem[];
    const int L = lp.L;
    const int W = L * F;
    const int S = W + row_pad(F);
    float* xs = smem;
    float* gs = smem + BP * 3;
    const int64_t p0 = (int64_t)blockIdx.x * BP;
    const int nvalid = (int)min((int64_t)BP, N - p0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;

    constexpr int FG = F <= 4 ? F : 4;  // keeps GroupWarp instantiable for kAtomicOnly
    GroupWarp<FG> grp(reinterpret_cast<char*>(smem + BP * 3 + BP * S), warp);
    if constexpr (kMode != kAtomicOnly) grp.clear(lane);

    stage_x(xs, x + p0 * 3, nvalid * 3);
    stage_rows_in<(F < 4 ? F : 4)>(gs, dout, p0, nvalid, W, S);
    __syncthreads();

    const int items = (BP / 32) * L;
    for (int it = warp; it < items; it += nwarps) {
        const int q = it / L;
        const int l = it - q * L;
        const int pl = q * 32 + lane;
        const bool valid = pl < nvalid;
        const int pc = valid ? pl : 0;  // rows past the tail read row 0 and contribute nothing
        GT* dl = dtable + (uint64_t)l * lp.T * F;
        Corners cr;
        locate_corners(xs[pc * 3 + 0], xs[pc * 3 + 1], xs[pc * 3 + 2], lp.scale[l], lp.mask, cr);
        float g[F];
        load_smem_entry<F>(gs + pc * S + l * F, g);

        bool group = (kMode == kGroupAlways);
        if constexpr (kMode == kAdaptive) {
            const int u0 = __shfl_up_sync(0xffffffffu, cr.v[0], 1);
            const int u1 = __shfl_up_sync(0xffffffffu, cr.v[1], 1);
            const int u2 = __shfl_up_sync(0xffffffffu, cr.v[2], 1);
            const bool near = valid && lane > 0 && abs(cr.v[0] - u0) <= 1 && abs(cr.v[1] - u1) <= 1 &&
                              abs(cr.v[2] - u2) <= 1;
            group = __popc(__ballot_sync(0xffffffffu, near)) >= 16;
        }
        if constexpr (kMode != kAtomicOnly) {
            static_assert(sizeof(GT) == 4, "grouped reductions accumulate fp32 gradients");
            if (group) {
                const uint32_t vmask = __ballot_sync(0xffffffffu, valid);
                if (valid) {
                    float v[8][FG];
#pragma unroll
                    for (int c = 0; c < 8; ++c)
#pragma unroll
                        for (int f = 0; f < FG; ++f) v[c][f] = cr.w[c] * g[f < F ? f : 0];
                    grp.push8(dl, cr.idx, v, lane, vmask);
                }
                __syncwarp();
                grp.flush(dl, lane);
                __syncwarp();
                continue;
            }
        }
        if (valid) {
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                float va[F], vb[F];
#pragma unroll
                for (int f = 0; f < F; ++f) {
                    va[f] = cr.w[2 * qq] * g[f];
                    vb[f] = cr.w[2 * qq + 1] * g[f];
                }
                red_pair<F>(dl, cr.idx[2 * qq], cr.idx[2 * qq + 1], va, vb);
            }
        }
    }
}

template <int F, int BP, typename GT>
__global__ void __launch_bounds__(512) backward_kernel_atomic(LevelParams lp, const float* __restrict__ x,
                                                              const float* __restrict__ dout, int64_t N,
                                                              GT* __restrict__ dtable) {
    backward_body<F, BP, kAtomicOnly, GT>(lp, x, dout, N, dtable);
}

template <int F, int BP, int kMode>
__global__ void __launch_bounds__(256, F == 4 ? 2 : 3) backward_kernel_grouped(LevelParams lp, const float* __restrict__ x,
                                                                                const float* __restrict__ dout, int64_t N,
                                                                                float* __restrict__ dtable) {
    backward_body<F, BP, kMode>(lp, x, dout, N, dtable);
}

// ---------------------------------------------------------------------------------------
// Run-merged backward (ordered batches, e.g. consecutive samples along rays). A lane walks a
// run of kRun consecutive points at one level and keeps the current voxel's 8 corner sums
// in registers. A point in the same voxel only adds to them. A step to a face-adjacent
// voxel shares 4 corners: the 4 corners left behind are reduced into the table and the 4
// shared ones carry their sums over. Any other step reduces all 8. Reductions of the two
// x-corners of an edge are merged as in red_pair. Block: kRunTile points (32 runs) and 8
// warps; a warp item is one level for the block's 32 runs.
// Shared memory: x and the upstream-gradient rows, grouped by run with strides chosen so
// that the lanes' row reads (lane = run) fall in distinct banks.
// ---------------------------------------------------------------------------------------
constexpr int kRun = 8;                 // one-lane and level-major walks
constexpr int kRunTile = 32 * kRun;     // one-lane tile: a run per lane of a warp
// Lane-pair walks (backward_kernel_runs_lanes) take runs of 16 points, 16 runs per 256-point
// tile: at coarse levels a run's end flushes its corners even when the next sample shares
// the voxel, and runs of 16 halve those flushes (rays: 345 against 352 us). The level-major
// walk keeps runs of 8 (runs of 16 left too few lane pairs in flight there: 3.01 against
// 2.66 ms on the 1 GiB grid).
constexpr int kRunPair = 16;
constexpr int kRunPairTile = 256;

__host__ __device__ constexpr int run_x_stride(int run = kRun) { return run * 3 + 1; }
__host__ __device__ constexpr int run_row_stride(int L, int F) { return L * F + row_pad(F); }
__host__ __device__ constexpr int run_g_stride(int L, int F, int run = kRun) { return run * run_row_stride(L, F) + F; }
__host__ __device__ constexpr size_t run_smem_bytes(int L, int F, int runs = kRunTile / kRun, int run = kRun) {
    return sizeof(float) * ((size_t)runs * run_x_stride(run) + (size_t)runs * run_g_stride(L, F, run));
}

template <int F, bool kKeep = false, typename GT>
__device__ __forceinline__ void run_flush(GT* dl, const float (&acc)[8][F], const uint32_t (&cidx)[8],
                                          int ax, uint32_t leave_bit) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int a = 2 * q, b = 2 * q + 1;
        const bool fa = ax < 0 || (((uint32_t)a >> ax) & 1u) == leave_bit;
        const bool fb = ax < 0 || (((uint32_t)b >> ax) & 1u) == leave_bit;
        red_pair<F, kKeep>(dl, cidx[a], cidx[b], acc[a], acc[b], fa, fb);
    }
}

// Walk one run of `n` consecutive points at one level (scale, mask) and reduce into the
// level table dl. xp(j, x3) loads point j's 3 coordinates; gl(j, g) its F upstream
// gradients.
template <int F, bool kKeep = false, typename GT, class XP, class GL>
__device__ __forceinline__ void walk_run(GT* dl, float scale, uint32_t mask, int n, XP xp, GL gl) {
    float acc[8][F];
    uint32_t cidx[8];
    int cv0 = 0, cv1 = 0, cv2 = 0;
#pragma unroll
    for (int c = 0; c < 8; ++c)
#pragma unroll
        for (int f = 0; f < F; ++f) acc[c][f] = 0.f;
    for (int j = 0; j < n; ++j) {
        float x3[3];
        xp(j, x3);
        Corners cr;
        locate_corners(x3[0], x3[1], x3[2], scale, mask, cr);
        float g[F];
        gl(j, g);
        if (j > 0) {
            const int dx = cr.v[0] - cv0, dy = cr.v[1] - cv1, dz = cr.v[2] - cv2;
            if ((dx | dy | dz) != 0) {
                const bool face = abs(dx) + abs(dy) + abs(dz) == 1;
                const int ax = face ? (dx != 0 ? 0 : (dy != 0 ? 1 : 2)) : -1;
                const uint32_t leave_bit = (dx + dy + dz) > 0 ? 0u : 1u;
                run_flush<F, kKeep>(dl, acc, cidx, ax, leave_bit);
                // carried corners: the new corner c with bit ax == leave_bit is the old
                // corner c ^ (1 << ax); every other new corner starts from zero
                float old[8][F];
#pragma unroll
                for (int c = 0; c < 8; ++c)
#pragma unroll
                    for (int f = 0; f < F; ++f) old[c][f] = acc[c][f];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const bool keep = face && (((uint32_t)c >> ax) & 1u) == leave_bit;
#pragma unroll
                    for (int f = 0; f < F; ++f) {
                        const float from = ax == 0 ? old[c ^ 1][f] : (ax == 1 ? old[c ^ 2][f] : old[c ^ 4][f]);
                        acc[c][f] = keep ? from : 0.f;
                    }
                }
            }
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            cidx[c] = cr.idx[c];
#pragma unroll
            for (int f = 0; f < F; ++f) acc[c][f] = fmaf(cr.w[c], g[f], acc[c][f]);
        }
        cv0 = cr.v[0];
        cv1 = cr.v[1];
        cv2 = cr.v[2];
    }
    if (n > 0) run_flush<F, kKeep>(dl, acc, cidx, -1, 0u);
}

template <int F, typename GT>
__global__ void __launch_bounds__(256) backward_kernel_runs(LevelParams lp, const float* __restrict__ x,
                                                           const float* __restrict__ dout, int64_t N,
                                                           GT* __restrict__ dtable) {
    static_assert(F <= 4, "run merging keeps 8 x F sums in registers");
    extern __shared__ __align__(16) float smem[];
    const int L = lp.L;
    const int W = L * F;
    const int S = run_row_stride(L, F);
    const int G = run_g_stride(L, F);
    constexpr int XS = run_x_stride();
    float* xs = smem;
    float* gs = smem + 32 * XS;
    const int64_t p0 = (int64_t)blockIdx.x * kRunTile;
    const int nvalid = (int)min((int64_t)kRunTile, N - p0);

    stage_x(x + p0 * 3, nvalid * 3, [&](int k, float v) {
        const int p = k / 3, i = k - 3 * (k / 3);
        xs[(p / kRun) * XS + (p % kRun) * 3 + i] = v;
    });
    {
        constexpr int V = F < 4 ? F : 4;
        const int per_row = W / V;
        const float* base = dout + p0 * (int64_t)W;
        for (int k = threadIdx.x; k < nvalid * per_row; k += blockDim.x) {
            const int row = k / per_row;
            const int col = (k - row * per_row) * V;
            float* dst = gs + (row / kRun) * G + (row % kRun) * S + col;
            const float* src = base + (int64_t)row * W + col;
            if (!in_bounds<kChkDout>(src, 4 * V)) continue;
            if constexpr (V == 4) {
                *reinterpret_cast<float4*>(dst) = __ldcs(reinterpret_cast<const float4*>(src));
            } else if constexpr (V == 2) {
                *reinterpret_cast<float2*>(dst) = __ldcs(reinterpret_cast<const float2*>(src));
            } else {
                *dst = __ldcs(src);
            }
        }
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    const int jmax = min(kRun, nvalid - lane * kRun);  // points of this lane's run (may be <= 0)
    for (int l = warp; l < L; l += nwarps) {
        GT* dl = dtable + (uint64_t)l * lp.T * F;
        walk_run<F>(dl, lp.scale[l], lp.mask, jmax,
                    [&](int j, float* x3) {
                        const float* q = xs + lane * XS + j * 3;
                        x3[0] = q[0]; x3[1] = q[1]; x3[2] = q[2];
                    },
                    [&](int j, float* g) { load_smem_entry<F>(gs + lane * G + j * S + l * F, g); });
    }
}

// ---------------------------------------------------------------------------------------
// Lane-pair run walk. As walk_run, but the two lanes of a pair walk one run together: lane
// d0 = lane & 1 keeps the sums of the 4 corners whose x offset is d0 and reduces them
// itself, one F-wide reduction per corner. Both lanes see the same points, so they take the
// same decisions and issue the reductions of x-neighbouring corners in the same
// instruction. The x prime is 1, so those two entries share a 32-byte sector most of the
// time, and the L2 serves two reductions into one sector from one instruction faster than
// two from different instructions (measured on B200 with the probe kernels: 296 against
// 188 G lane-reductions per second for random 8-byte x-pairs). A step across an x face
// hands the shared face's 4 sums from one lane to the other with shuffles; y and z steps
// carry sums inside each lane, as in walk_run.
// ---------------------------------------------------------------------------------------
template <int F, typename GT, bool kKeep = false> struct RedLane;
template <int F, bool kKeep> struct RedLane<F, float, kKeep> {
    static __device__ __forceinline__ void add(float* p, const float (&v)[F]) { RedAdd<F, kKeep>::add(p, v); }
};
template <bool kKeep> struct RedLane<1, __half, kKeep> {
    static __device__ __forceinline__ void add(__half* p, const float (&v)[1]) {
        if (!in_bounds<kChkGrad>(p, 2)) return;
        const unsigned short h = __half_as_ushort(__float2half_rn(v[0]));
        if constexpr (kKeep) {
            asm volatile("red.global.add.L2::cache_hint.noftz.f16 [%0], %1, %2;" ::"l"(p), "h"(h),
                         "l"(l2_evict_last_policy())
                         : "memory");
        } else {
            asm volatile("red.global.add.noftz.f16 [%0], %1;" ::"l"(p), "h"(h) : "memory");
        }
    }
};
template <bool kKeep> struct RedLane<2, __half, kKeep> {
    static __device__ __forceinline__ void add(__half* p, const float (&v)[2]) {
        if (!in_bounds<kChkGrad>(p, 4)) return;
        __half2 h = __floats2half2_rn(v[0], v[1]);
        const uint32_t w = *reinterpret_cast<uint32_t*>(&h);
        if constexpr (kKeep) {
            asm volatile("red.global.add.L2::cache_hint.noftz.f16x2 [%0], %1, %2;" ::"l"(p), "r"(w),
                         "l"(l2_evict_last_policy())
                         : "memory");
        } else {
            asm volatile("red.global.add.noftz.f16x2 [%0], %1;" ::"l"(p), "r"(w) : "memory");
        }
    }
};
template <bool kKeep> struct RedLane<8, __half, kKeep> {
    static __device__ __forceinline__ void add(__half* p, const float (&v)[8]) { red_half_unit<kKeep>(p, v); }
};
template <bool kKeep> struct RedLane<4, __half, kKeep> {
    static __device__ __forceinline__ void add(__half* p, const float (&v)[4]) {
        if (!in_bounds<kChkGrad>(p, 8)) return;
        __half2 a = __floats2half2_rn(v[0], v[1]), b = __floats2half2_rn(v[2], v[3]);
        const uint32_t wa = *reinterpret_cast<uint32_t*>(&a), wb = *reinterpret_cast<uint32_t*>(&b);
        if constexpr (kKeep) {
            asm volatile("red.global.add.L2::cache_hint.noftz.v2.f16x2 [%0], {%1, %2}, %3;" ::"l"(p), "r"(wa),
                         "r"(wb), "l"(l2_evict_last_policy())
                         : "memory");
        } else {
            asm volatile("red.global.add.noftz.v2.f16x2 [%0], {%1, %2};" ::"l"(p), "r"(wa), "r"(wb) : "memory");
        }
    }
};

// locate_half plus the voxel (the walk compares voxels of consecutive points).
__device__ __forceinline__ void locate_half_voxel(float x0, float x1, float x2, float scale, uint32_t mask,
                                                  uint32_t d0, HalfCorners& hc, int (&v)[3]) {
    locate_half(x0, x1, x2, scale, mask, d0, hc);
    v[0] = __float2int_rd(__fmul_rn(x0, scale));
    v[1] = __float2int_rd(__fmul_rn(x1, scale));
    v[2] = __float2int_rd(__fmul_rn(x2, scale));
}

template <int F, bool kKeep = false, typename GT, class XP, class GL>
__device__ __forceinline__ void walk_run_pair(GT* dl, float scale, uint32_t mask, int n, uint32_t d0, unsigned pair,
                                              XP xp, GL gl) {
    float acc[4][F];
    uint32_t cidx[4];
    int cv[3] = {0, 0, 0};
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int f = 0; f < F; ++f) acc[k][f] = 0.f;
    for (int j = 0; j < n; ++j) {
        float x3[3];
        xp(j, x3);
        HalfCorners hc;
        int v[3];
        locate_half_voxel(x3[0], x3[1], x3[2], scale, mask, d0, hc, v);
        float g[F];
        gl(j, g);
        if (j > 0) {
            const int dx = v[0] - cv[0], dy = v[1] - cv[1], dz = v[2] - cv[2];
            if ((dx | dy | dz) != 0) {
                const bool face = abs(dx) + abs(dy) + abs(dz) == 1;
                if (face && dx != 0) {
                    // x face: the lane on the side left behind reduces its corners and takes
                    // over its partner's sums (they lie on the shared face); the partner
                    // starts from zero. dx = +1 leaves x offset 0 behind, dx = -1 offset 1.
                    const uint32_t leave = dx > 0 ? 0u : 1u;
                    if (d0 == leave) {
#pragma unroll
                        for (int k = 0; k < 4; ++k) RedLane<F, GT, kKeep>::add(dl + (uint64_t)cidx[k] * F, acc[k]);
                    }
#pragma unroll
                    for (int k = 0; k < 4; ++k)
#pragma unroll
                        for (int f = 0; f < F; ++f) {
                            const float other = __shfl_xor_sync(pair, acc[k][f], 1);
                            acc[k][f] = d0 == leave ? other : 0.f;
                        }
                } else if (face) {
                    // y or z face: corner bit b (0: y, 1: z) of the local corner number k;
                    // corners whose offset along the step's axis is leave_bit are left behind,
                    // the new corners with that offset take the sums of their face neighbours
                    const int b = dy != 0 ? 0 : 1;
                    const uint32_t leave_bit = (dy + dz) > 0 ? 0u : 1u;
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if ((((uint32_t)k >> b) & 1u) == leave_bit)
                            RedLane<F, GT, kKeep>::add(dl + (uint64_t)cidx[k] * F, acc[k]);
                    float old[4][F];
#pragma unroll
                    for (int k = 0; k < 4; ++k)
#pragma unroll
                        for (int f = 0; f < F; ++f) old[k][f] = acc[k][f];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const bool keep = (((uint32_t)k >> b) & 1u) == leave_bit;
#pragma unroll
                        for (int f = 0; f < F; ++f) acc[k][f] = keep ? (b == 0 ? old[k ^ 1][f] : old[k ^ 2][f]) : 0.f;
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        RedLane<F, GT, kKeep>::add(dl + (uint64_t)cidx[k] * F, acc[k]);
#pragma unroll
                        for (int f = 0; f < F; ++f) acc[k][f] = 0.f;
                    }
                }
            }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            cidx[k] = hc.idx[k];
#pragma unroll
            for (int f = 0; f < F; ++f) acc[k][f] = fmaf(hc.w[k], g[f], acc[k][f]);
        }
        cv[0] = v[0];
        cv[1] = v[1];
        cv[2] = v[2];
    }
    if (n > 0) {
#pragma unroll
        for (int k = 0; k < 4; ++k) RedLane<F, GT, kKeep>::add(dl + (uint64_t)cidx[k] * F, acc[k]);
    }
}

// Block: kRunPairTile points (16 runs of kRunPair) and 8 warps, shared memory laid out as in
// backward_kernel_runs; a warp item is 16 runs at one level (a lane pair per run).
template <int F, typename GT>
__global__ void __launch_bounds__(256) backward_kernel_runs_lanes(LevelParams lp, const float* __restrict__ x,
                                                                 const float* __restrict__ dout, int64_t N,
                                                                 GT* __restrict__ dtable) {
    static_assert(F <= 4, "run merging keeps 4 x F sums per lane in registers");
    extern __shared__ __align__(16) float smem[];
    const int L = lp.L;
    const int W = L * F;
    const int S = run_row_stride(L, F);
    constexpr int R = kRunPair;                   // points per run
    constexpr int NR = kRunPairTile / kRunPair;   // runs per tile
    const int G = run_g_stride(L, F, R);
    constexpr int XS = run_x_stride(R);
    float* xs = smem;
    float* gs = smem + NR * XS;
    const int64_t p0 = (int64_t)blockIdx.x * kRunPairTile;
    const int nvalid = (int)min((int64_t)kRunPairTile, N - p0);

    stage_x(x + p0 * 3, nvalid * 3, [&](int k, float v) {
        const int p = k / 3, i = k - 3 * (k / 3);
        xs[(p / R) * XS + (p % R) * 3 + i] = v;
    });
    {
        constexpr int V = F < 4 ? F : 4;
        const int per_row = W / V;
        const float* base = dout + p0 * (int64_t)W;
        for (int k = threadIdx.x; k < nvalid * per_row; k += blockDim.x) {
            const int row = k / per_row;
            const int col = (k - row * per_row) * V;
            float* dst = gs + (row / R) * G + (row % R) * S + col;
            const float* src = base + (int64_t)row * W + col;
            if (!in_bounds<kChkDout>(src, 4 * V)) continue;
            if constexpr (V == 4) {
                *reinterpret_cast<float4*>(dst) = __ldcs(reinterpret_cast<const float4*>(src));
            } else if constexpr (V == 2) {
                *reinterpret_cast<float2*>(dst) = __ldcs(reinterpret_cast<const float2*>(src));
            } else {
                *dst = __ldcs(src);
            }
        }
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    const uint32_t d0 = lane & 1;
    const unsigned pair = 3u << (lane & 30);
    for (int it = warp; it < (NR / 16) * L; it += nwarps) {
        const int h = it / L;
        const int l = it - h * L;
        const int run = h * 16 + (lane >> 1);
        const int jmax = min(R, nvalid - run * R);  // the same for both lanes of a pair
        GT* dl = dtable + (uint64_t)l * lp.T * F;
        walk_run_pair<F>(dl, lp.scale[l], lp.mask, jmax, d0, pair,
                         [&](int j, float* x3) {
                             const float* q = xs + run * XS + j * 3;
                             x3[0] = q[0]; x3[1] = q[1]; x3[2] = q[2];
                         },
                         [&](int j, float* g) { load_smem_entry<F>(gs + run * G + j * S + l * F, g); });
    }
}

// ---------------------------------------------------------------------------------------
// Level-major schedules, for tables larger than L2. Grid (tiles, L): blocks are issued with
// the tile index fastest, so the GPU works through the levels one after another and the
// current level's table slice (backward: its gradient slice) stays resident in L2 while
// every point visits it, instead of each point's fine-level gathers missing to DRAM. The
// price is re-reading x once per level and touching output / upstream-gradient rows in
// F-wide column slices.
// ---------------------------------------------------------------------------------------
// Streaming (evict-first) row accesses: x, output and upstream-gradient slices are touched
// once per level and must not push the level's table out of L2.
template <int F>
__device__ __forceinline__ void store_global_entry(float* p, const float* v) {
    if (!in_bounds<kChkOut>(p, 4 * F)) return;
    if constexpr (F == 1) {
        __stcs(p, v[0]);
    } else if constexpr (F == 2) {
        __stcs(reinterpret_cast<float2*>(p), make_float2(v[0], v[1]));
    } else {
#pragma unroll
        for (int j = 0; j < F; j += 4)
            __stcs(reinterpret_cast<float4*>(p + j), make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]));
    }
}

template <int F>
__device__ __forceinline__ void load_global_entry(const float* p, float* v) {
    if (!in_bounds<kChkDout>(p, 4 * F)) {
#pragma unroll
        for (int f = 0; f < F; ++f) v[f] = 0.f;
        return;
    }
    if constexpr (F == 1) {
        v[0] = __ldcs(p);
    } else if constexpr (F == 2) {
        float2 a = __ldcs(reinterpret_cast<const float2*>(p));
        v[0] = a.x; v[1] = a.y;
    } else {
#pragma unroll
        for (int j = 0; j < F; j += 4) {
            float4 a = __ldcs(reinterpret_cast<const float4*>(p + j));
            v[j] = a.x; v[j + 1] = a.y; v[j + 2] = a.z; v[j + 3] = a.w;
        }
    }
}

// F-wide fp32 / fp16 table entry load with an L2 cache policy.
template <int F, typename TT>
__device__ __forceinline__ void load_entry_policy(const TT* p, float* e, uint64_t pol) {
    constexpr int E = F * (int)sizeof(TT);
    if (!in_bounds<kChkTable>(p, E)) {
#pragma unroll
        for (int f = 0; f < F; ++f) e[f] = 0.f;
        return;
    }
    uint32_t w[8];
    if constexpr (E == 2) {
        unsigned short h;
        asm("ld.global.nc.L2::cache_hint.b16 %0, [%1], %2;" : "=h"(h) : "l"(p), "l"(pol));
        e[0] = __half2float(__ushort_as_half(h));
        return;
    } else if constexpr (E == 4) {
        asm("ld.global.nc.L2::cache_hint.b32 %0, [%1], %2;" : "=r"(w[0]) : "l"(p), "l"(pol));
    } else if constexpr (E == 8) {
        asm("ld.global.nc.L2::cache_hint.v2.b32 {%0, %1}, [%2], %3;" : "=r"(w[0]), "=r"(w[1]) : "l"(p), "l"(pol));
    } else {
#pragma unroll
        for (int k = 0; k < E / 16; ++k)
            asm("ld.global.nc.L2::cache_hint.v4.b32 {%0, %1, %2, %3}, [%4], %5;"
                : "=r"(w[4 * k]), "=r"(w[4 * k + 1]), "=r"(w[4 * k + 2]), "=r"(w[4 * k + 3])
                : "l"(reinterpret_cast<const char*>(p) + 16 * k), "l"(pol));
    }
    if constexpr (sizeof(TT) == 4) {
#pragma unroll
        for (int f = 0; f < F; ++f) e[f] = __uint_as_float(w[f]);
    } else {
#pragma unroll
        for (int k = 0; k < E / 4; ++k) {
            float2 v = h2_bits_to_f2(w[k]);
            e[2 * k] = v.x;
            e[2 * k + 1] = v.y;
        }
    }
}

constexpr int kLevelBlock = 256;

template <int F, typename TT>
__global__ void __launch_bounds__(kLevelBlock) forward_kernel_levels(LevelParams lp, const float* __restrict__ x,
                                                                    int64_t N, const TT* __restrict__ table,
                                                                    float* __restrict__ out) {
    const int l = blockIdx.y;
    const int64_t p = (int64_t)blockIdx.x * kLevelBlock + threadIdx.x;
    if (p >= N) return;
    Corners cr;
    locate_corners(ld_x(x + p * 3), ld_x(x + p * 3 + 1), ld_x(x + p * 3 + 2), lp.scale[l], lp.mask, cr);
    const TT* tl = table + (uint64_t)l * lp.T * F;
    const uint64_t pol = l2_evict_last_policy();
    float e[8][F];
#pragma unroll
    for (int c = 0; c < 8; ++c) load_entry_policy<F, TT>(tl + (uint64_t)cr.idx[c] * F, e[c], pol);
    float o[F];
#pragma unroll
    for (int f = 0; f < F; ++f) {
        float acc = cr.w[0] * e[0][f];
#pragma unroll
        for (int c = 1; c < 8; ++c) acc = fmaf(cr.w[c], e[c][f], acc);
        o[f] = acc;
    }
    store_global_entry<F>(out + p * (int64_t)(lp.L * F) + l * F, o);
}

// Level-major forward with lane pairs: two threads per point for the levels of group
// blockIdx.y, in order (x is read once per group, and a group's output pieces of a row
// are written back to back, so its sectors leave L2 whole).
template <int F, typename TT>
__global__ void __launch_bounds__(kLevelBlock) forward_kernel_levels_lanes(LevelParams lp, const float* __restrict__ x,
                                                                          int64_t N, const TT* __restrict__ table,
                                                                          float* __restrict__ out) {
    const int g = blockIdx.y;
    const int64_t p = ((int64_t)blockIdx.x * kLevelBlock + threadIdx.x) >> 1;
    if (p >= N) return;  // both lanes of a pair return together
    const uint32_t lane = threadIdx.x & 31;
    const uint32_t d0 = lane & 1;
    const unsigned pair = 3u << (lane & 30);
    const float x0 = ld_x(x + p * 3), x1 = ld_x(x + p * 3 + 1), x2 = ld_x(x + p * 3 + 2);
    const uint64_t pol = l2_evict_last_policy();
    for (int l = lp.group_lo[g]; l < lp.group_lo[g + 1]; ++l) {
        HalfCorners hc;
        locate_half(x0, x1, x2, lp.scale[l], lp.mask, d0, hc);
        const TT* tl = table + (uint64_t)l * lp.T * F;
        float e[4][F];
#pragma unroll
        for (int k = 0; k < 4; ++k) load_entry_policy<F, TT>(tl + (uint64_t)hc.idx[k] * F, e[k], pol);
        float o[F];
#pragma unroll
        for (int f = 0; f < F; ++f) {
            float acc = hc.w[0] * e[0][f];
#pragma unroll
            for (int k = 1; k < 4; ++k) acc = fmaf(hc.w[k], e[k][f], acc);
            o[f] = acc + __shfl_xor_sync(pair, acc, 1);
        }
        store_half<F, true>(out + p * (int64_t)(lp.L * F) + l * F, o, d0);
    }
}

template <int F, typename GT>
__global__ void __launch_bounds__(kLevelBlock) backward_kernel_atomic_levels(LevelParams lp, const float* __restrict__ x,
                                                                            const float* __restrict__ dout, int64_t N,
                                                                            GT* __restrict__ dtable) {
    const int l = blockIdx.y;
    const int64_t p = (int64_t)blockIdx.x * kLevelBlock + threadIdx.x;
    if (p >= N) return;
    Corners cr;
    locate_corners(ld_x(x + p * 3), ld_x(x + p * 3 + 1), ld_x(x + p * 3 + 2), lp.scale[l], lp.mask, cr);
    float g[F];
    load_global_entry<F>(dout + p * (int64_t)(lp.L * F) + l * F, g);
    GT* dl = dtable + (uint64_t)l * lp.T * F;
#pragma unroll
    for (int qq = 0; qq < 4; ++qq) {
        float va[F], vb[F];
#pragma unroll
        for (int f = 0; f < F; ++f) {
            va[f] = cr.w[2 * qq] * g[f];
            vb[f] = cr.w[2 * qq + 1] * g[f];
        }
        red_pair<F, true>(dl, cr.idx[2 * qq], cr.idx[2 * qq + 1], va, vb);
    }
}

// One thread walks one run of kRun consecutive points at level blockIdx.y.
template <int F, typename GT>
__global__ void __launch_bounds__(kLevelBlock) backward_kernel_runs_levels(LevelParams lp, const float* __restrict__ x,
                                                                          const float* __restrict__ dout, int64_t N,
                                                                          GT* __restrict__ dtable) {
    const int l = blockIdx.y;
    const int64_t p0 = ((int64_t)blockIdx.x * kLevelBlock + threadIdx.x) * kRun;
    if (p0 >= N) return;
    const int n = (int)min((int64_t)kRun, N - p0);
    const int64_t W = lp.L * F;
    GT* dl = dtable + (uint64_t)l * lp.T * F;
    walk_run<F, true>(dl, lp.scale[l], lp.mask, n,
                [&](int j, float* x3) {
                    const float* q = x + (p0 + j) * 3;
                    x3[0] = ld_x(q); x3[1] = ld_x(q + 1); x3[2] = ld_x(q + 2);
                },
                [&](int j, float* g) { load_global_entry<F>(dout + (p0 + j) * W + l * F, g); });
}

// Level-major lane-pair run walk: two threads per run of kRun consecutive points, walked at
// each level of group blockIdx.y in turn (the run's x and upstream-gradient rows are read
// from HBM for the group's first level and from the caches for the others).
template <int F, typename GT>
__global__ void __launch_bounds__(kLevelBlock) backward_kernel_runs_levels_lanes(LevelParams lp,
                                                                                const float* __restrict__ x,
                                                                                const float* __restrict__ dout,
                                                                                int64_t N, GT* __restrict__ dtable) {
    const int grp = blockIdx.y;
    const int64_t p0 = (((int64_t)blockIdx.x * kLevelBlock + threadIdx.x) >> 1) * kRun;
    if (p0 >= N) return;  // both lanes of a pair return together
    const int n = (int)min((int64_t)kRun, N - p0);
    const int64_t W = lp.L * F;
    const uint32_t lane = threadIdx.x & 31;
    for (int l = lp.group_lo[grp]; l < lp.group_lo[grp + 1]; ++l) {
        GT* dl = dtable + (uint64_t)l * lp.T * F;
        walk_run_pair<F, true>(dl, lp.scale[l], lp.mask, n, lane & 1, 3u << (lane & 30),
                               [&](int j, float* x3) {
                                   const float* q = x + (p0 + j) * 3;
                                   x3[0] = ld_x(q); x3[1] = ld_x(q + 1); x3[2] = ld_x(q + 2);
                               },
                               [&](int j, float* g) { load_global_entry<F>(dout + (p0 + j) * W + l * F, g); });
    }
}

// ---------------------------------------------------------------------------------------
// Gradient with respect to the input coordinates ([NeRFace-HG] section 3 runs the encoder
// on coordinates produced by a learned transform). Inside the voxel that floor() selects,
// d frac_i / d x_i = N_l, so with s_c = sum_f g_f e_c[f]:
//   dL/dx_i = sum_l N_l * sum_c s_c * (d_i ? +1 : -1) * prod_{j != i} (d_j ? frac_j : 1 - frac_j).
// Point-major: a block stages its x and upstream-gradient rows, each (point, level) thread
// gathers the 8 corners and writes its 3 partials to shared memory as [level][point][axis]
// (stride 3 across lanes: conflict-free), then one thread per (point, axis) sums the levels
// in order (consecutive words across lanes) and stores dL/dx.
// ---------------------------------------------------------------------------------------
__host__ __device__ constexpr size_t input_grad_smem_bytes(int BP, int L, int F) {
    return tile_smem_bytes(BP, L, F) + sizeof(float) * (size_t)BP * L * 3;
}

template <int F, typename TT, int BP>
__global__ void __launch_bounds__(512, F <= 2 ? 3 : 2) backward_input_kernel(LevelParams lp, const float* __restrict__ x,
                                                                const float* __restrict__ dout, int64_t N,
                                                                const TT* __restrict__ table,
                                                                float* __restrict__ dx) {
    extern __shared__ __align__(16) float smem[];
    const int L = lp.L;
    const int W = L * F;
    const int S = W + row_pad(F);
    float* xs = smem;
    float* gs = smem + BP * 3;
    float* part = gs + BP * S;  // [L][BP][3]
    const int64_t p0 = (int64_t)blockIdx.x * BP;
    const int nvalid = (int)min((int64_t)BP, N - p0);

    stage_x(xs, x + p0 * 3, nvalid * 3);
    stage_rows_in<(F < 4 ? F : 4)>(gs, dout, p0, nvalid, W, S);
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    const int items = (BP / 32) * L;
    for (int it = warp; it < items; it += nwarps) {
        const int q = it / L;
        const int l = it - q * L;
        const int pl = q * 32 + lane;
        if (pl < nvalid) {
            Corners cr;
            locate_corners(xs[pl * 3 + 0], xs[pl * 3 + 1], xs[pl * 3 + 2], lp.scale[l], lp.mask, cr);
            const TT* tl = table + (uint64_t)l * lp.T * F;
            float e[8][F];
            gather_corners<F, TT, kGatherCorner>(tl, cr, e);
            float g[F];
            load_smem_entry<F>(gs + pl * S + l * F, g);
            float sc[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                float t = g[0] * e[c][0];
#pragma unroll
                for (int f = 1; f < F; ++f) t = fmaf(g[f], e[c][f], t);
                sc[c] = t;
            }
            const float w0[2] = {1.0f - cr.f[0], cr.f[0]};
            const float w1[2] = {1.0f - cr.f[1], cr.f[1]};
            const float w2[2] = {1.0f - cr.f[2], cr.f[2]};
            float d0 = 0.f, d1 = 0.f, d2 = 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const int b0 = c & 1, b1 = (c >> 1) & 1, b2 = (c >> 2) & 1;
                const float s0 = b0 ? sc[c] : -sc[c];
                const float s1 = b1 ? sc[c] : -sc[c];
                const float s2 = b2 ? sc[c] : -sc[c];
                d0 = fmaf(s0, w1[b1] * w2[b2], d0);
                d1 = fmaf(s1, w0[b0] * w2[b2], d1);
                d2 = fmaf(s2, w0[b0] * w1[b1], d2);
            }
            const float n = lp.scale[l];
            float* pp = part + ((size_t)l * BP + pl) * 3;  // stride 3 across lanes: conflict-free
            pp[0] = n * d0;
            pp[1] = n * d1;
            pp[2] = n * d2;
        }
    }
    __syncthreads();
    for (int t = threadIdx.x; t < nvalid * 3; t += blockDim.x) {  // t = 3 * point + axis
        float s = 0.f;
        for (int l = 0; l < L; ++l) s += part[(size_t)l * BP * 3 + t];
        if (in_bounds<kChkOut>(dx + p0 * 3 + t, 4)) __stcs(dx + p0 * 3 + t, s);
    }
}

// ---------------------------------------------------------------------------------------
// Sparse Adam on the tables ([NeRFace-HG] sections 3-4: Adam, no weight decay, only the
// sampled entries receive gradient). Per element with nonzero gradient g:
//   m = b1 m + (1 - b1) g;  v = b2 v + (1 - b2) g^2;
//   theta -= lr * (m * c1) / (sqrt(v * c2) + eps),  c1 = 1/(1 - b1^t), c2 = 1/(1 - b2^t);
// elements with g == 0 are left unchanged. Optionally the consumed gradient is zeroed,
// which replaces a separate clear of the whole gradient table before the next backward.
// Elementwise over L*T*F elements (a multiple of 16), 4 per thread, grid-stride; a group
// of 4 zero gradients costs one 16-byte read.
// ---------------------------------------------------------------------------------------
struct AdamParams {
    float lr, b1, b2, eps, c1, c2;
};

__device__ __forceinline__ float adam_one(float& m, float& v, float theta, float g, const AdamParams& a) {
    m = fmaf(a.b1, m, (1.0f - a.b1) * g);
    v = fmaf(a.b2, v, (1.0f - a.b2) * g * g);
    const float denom = __fadd_rn(__fsqrt_rn(v * a.c2), a.eps);
    return theta - a.lr * __fdiv_rn(m * a.c1, denom);
}

// One 4-element group: the state is loaded first, the update and stores come later, so a
// thread can have two groups' loads in flight at once.
template <typename TT>
struct AdamGroup {
    float m[4], v[4], th[4];

    __device__ __forceinline__ void load(const TT* __restrict__ param, const float* __restrict__ mom1,
                                         const float* __restrict__ mom2, int64_t i) {
        if (!(in_bounds<kChkM>(mom1 + 4 * i, 16) & in_bounds<kChkV>(mom2 + 4 * i, 16) &
              in_bounds<kChkTable>(param + 4 * i, 4 * sizeof(TT)))) {
#pragma unroll
            for (int k = 0; k < 4; ++k) m[k] = v[k] = th[k] = 0.f;
            return;
        }
        const float4 mm = reinterpret_cast<const float4*>(mom1)[i];
        const float4 vv = reinterpret_cast<const float4*>(mom2)[i];
        m[0] = mm.x; m[1] = mm.y; m[2] = mm.z; m[3] = mm.w;
        v[0] = vv.x; v[1] = vv.y; v[2] = vv.z; v[3] = vv.w;
        if constexpr (sizeof(TT) == 4) {
            const float4 t = reinterpret_cast<const float4*>(param)[i];
            th[0] = t.x; th[1] = t.y; th[2] = t.z; th[3] = t.w;
        } else {
            const uint2 t = reinterpret_cast<const uint2*>(param)[i];
            const float2 lo = h2_bits_to_f2(t.x), hi = h2_bits_to_f2(t.y);
            th[0] = lo.x; th[1] = lo.y; th[2] = hi.x; th[3] = hi.y;
        }
    }

    __device__ __forceinline__ void update_store(TT* __restrict__ param, float* __restrict__ mom1,
                                                 float* __restrict__ mom2, float* __restrict__ grad, int64_t i,
                                                 const float4& g, const AdamParams& a, int zero_grad) {
        if (!(in_bounds<kChkM>(mom1 + 4 * i, 16) & in_bounds<kChkV>(mom2 + 4 * i, 16) &
              in_bounds<kChkTable>(param + 4 * i, 4 * sizeof(TT)) & in_bounds<kChkGrad>(grad + 4 * i, 16)))
            return;
        const float gv[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (gv[k] != 0.f) th[k] = adam_one(m[k], v[k], th[k], gv[k], a);
        reinterpret_cast<float4*>(mom1)[i] = make_float4(m[0], m[1], m[2], m[3]);
        reinterpret_cast<float4*>(mom2)[i] = make_float4(v[0], v[1], v[2], v[3]);
        if constexpr (sizeof(TT) == 4) {
            reinterpret_cast<float4*>(param)[i] = make_float4(th[0], th[1], th[2], th[3]);
        } else {
            const __half2 lo = __floats2half2_rn(th[0], th[1]), hi = __floats2half2_rn(th[2], th[3]);
            uint2 t;
            t.x = *reinterpret_cast<const uint32_t*>(&lo);
            t.y = *reinterpret_cast<const uint32_t*>(&hi);
            reinterpret_cast<uint2*>(param)[i] = t;
        }
        if (zero_grad) __stcs(reinterpret_cast<float4*>(grad) + i, make_float4(0.f, 0.f, 0.f, 0.f));
    }
};

__device__ __forceinline__ bool any_nonzero(const float4& g) {
    return g.x != 0.f || g.y != 0.f || g.z != 0.f || g.w != 0.f;
}

// Grid-stride over 4-element groups, two independent groups (i and i + stride) per step:
// both gradient loads first, then the state of the groups with a nonzero gradient, then
// the updates (measured latency-bound with one group per step).
template <typename TT>
__global__ void __launch_bounds__(256) adam_kernel(TT* __restrict__ param, float* __restrict__ mom1,
                                                   float* __restrict__ mom2, float* __restrict__ grad,
                                                   int64_t n4, AdamParams a, int zero_grad) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += 2 * stride) {
        const int64_t j = i + stride;
        const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 g0 = in_bounds<kChkGrad>(grad + 4 * i, 16) ? __ldcs(reinterpret_cast<const float4*>(grad) + i) : z4;
        const float4 g1 = j < n4 && in_bounds<kChkGrad>(grad + 4 * j, 16)
                              ? __ldcs(reinterpret_cast<const float4*>(grad) + j) : z4;
        const bool u0 = any_nonzero(g0), u1 = any_nonzero(g1);
        AdamGroup<TT> s0, s1;
        if (u0) s0.load(param, mom1, mom2, i);
        if (u1) s1.load(param, mom1, mom2, j);
        if (u0) s0.update_store(param, mom1, mom2, grad, i, g0, a, zero_grad);
        if (u1) s1.update_store(param, mom1, mom2, grad, j, g1, a, zero_grad);
    }
}

// Warp-owned lane-pair dL/dx: each warp owns 16 points for all levels. It stages its 16
// upstream-gradient rows in its own shared-memory tile (coalesced row loads), keeps x in
// registers, and each lane sums its half of the three derivatives over the levels in order
// in registers; the pair adds its halves at the end and one lane writes the point's dL/dx.
// No block-wide barrier and no per-level partials in shared memory (the per-(point, level)
// kernel above stores them and sums them in a second phase): measured 195 against 274 us
// per 2^20 ray samples for the lane-pair form of that two-phase kernel, 284 us for the
// one-lane-per-point form.
constexpr int kWarpPoints = 16;
template <int F, typename TT, int kWarps>
__global__ void __launch_bounds__(32 * kWarps, F <= 2 ? 3 : 2)
    backward_input_kernel_warp(LevelParams lp, const float* __restrict__ x, const float* __restrict__ dout,
                               int64_t N, const TT* __restrict__ table, float* __restrict__ dx) {
    extern __shared__ __align__(16) float smem[];
    const int L = lp.L;
    const int W = L * F;
    const int S = W + row_pad(F);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* gs = smem + warp * (kWarpPoints * S);
    const int64_t p0 = ((int64_t)blockIdx.x * kWarps + warp) * kWarpPoints;
    if (p0 >= N) return;  // whole warps only
    const int nvalid = (int)min((int64_t)kWarpPoints, N - p0);
    {
        constexpr int V = F < 4 ? F : 4;
        const int per_row = W / V;
        for (int k = lane; k < nvalid * per_row; k += 32) {
            const int row = k / per_row;
            const int col = (k - row * per_row) * V;
            const float* src = dout + (p0 + row) * (int64_t)W + col;
            if (!in_bounds<kChkDout>(src, 4 * V)) continue;
            if constexpr (V == 4) {
                *reinterpret_cast<float4*>(gs + row * S + col) = __ldcs(reinterpret_cast<const float4*>(src));
            } else if constexpr (V == 2) {
                *reinterpret_cast<float2*>(gs + row * S + col) = __ldcs(reinterpret_cast<const float2*>(src));
            } else {
                gs[row * S + col] = __ldcs(src);
            }
        }
    }
    __syncwarp();
    const uint32_t d0 = lane & 1;
    const unsigned pair = 3u << (lane & 30);
    const int pl = lane >> 1;
    if (pl >= nvalid) return;  // both lanes of a pair
    const float x0 = ld_x(x + (p0 + pl) * 3), x1 = ld_x(x + (p0 + pl) * 3 + 1), x2 = ld_x(x + (p0 + pl) * 3 + 2);
    float a0 = 0.f, a1 = 0.f, a2 = 0.f;
    for (int l = 0; l < L; ++l) {
        const float scale = lp.scale[l];
        HalfCorners hc;
        locate_half(x0, x1, x2, scale, lp.mask, d0, hc);
        const float xs0 = __fmul_rn(x0, scale), xs1 = __fmul_rn(x1, scale), xs2 = __fmul_rn(x2, scale);
        const float f0 = __fsub_rn(xs0, __int2float_rn(__float2int_rd(xs0)));
        const float f1 = __fsub_rn(xs1, __int2float_rn(__float2int_rd(xs1)));
        const float f2 = __fsub_rn(xs2, __int2float_rn(__float2int_rd(xs2)));
        const TT* tl = table + (uint64_t)l * lp.T * F;
        float e[4][F];
#pragma unroll
        for (int k = 0; k < 4; ++k) EntryLoad<F, TT>::load(tl + (uint64_t)hc.idx[k] * F, e[k]);
        float g[F];
        load_smem_entry<F>(gs + pl * S + l * F, g);
        const float w0 = d0 ? f0 : 1.0f - f0;
        const float w1[2] = {1.0f - f1, f1};
        const float w2[2] = {1.0f - f2, f2};
        float b0 = 0.f, b1 = 0.f, b2 = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int k1 = k & 1, k2 = k >> 1;
            float sc = g[0] * e[k][0];
#pragma unroll
            for (int f = 1; f < F; ++f) sc = fmaf(g[f], e[k][f], sc);
            b0 = fmaf(d0 ? sc : -sc, w1[k1] * w2[k2], b0);
            b1 = fmaf(k1 ? sc : -sc, w0 * w2[k2], b1);
            b2 = fmaf(k2 ? sc : -sc, w0 * w1[k1], b2);
        }
        a0 = fmaf(scale, b0, a0);
        a1 = fmaf(scale, b1, a1);
        a2 = fmaf(scale, b2, a2);
    }
    a0 += __shfl_xor_sync(pair, a0, 1);
    a1 += __shfl_xor_sync(pair, a1, 1);
    a2 += __shfl_xor_sync(pair, a2, 1);
    if (d0 == 0) {
        float* q = dx + (p0 + pl) * 3;
        if (in_bounds<kChkOut>(q, 12)) {
            __stcs(q, a0);
            __stcs(q + 1, a1);
            __stcs(q + 2, a2);
        }
    }
}

// ---------------------------------------------------------------------------------------
// Index export (tests and inspection): idx[(p*L + l)*8 + c]. One thread per (point, level).
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) indices_kernel(LevelParams lp, const float* __restrict__ x,
                                                      int64_t N, uint32_t* __restrict__ idx) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t total = N * lp.L;
    if (t >= total) return;
    const int64_t p = t / lp.L;
    const int l = (int)(t - p * lp.L);
    Corners cr;
    locate_corners(ld_x(x + p * 3 + 0), ld_x(x + p * 3 + 1), ld_x(x + p * 3 + 2), lp.scale[l], lp.mask, cr);
    uint4* dst = reinterpret_cast<uint4*>(idx + t * 8);
    if (!in_bounds<kChkOut>(dst, 32)) return;
    dst[0] = make_uint4(cr.idx[0], cr.idx[1], cr.idx[2], cr.idx[3]);
    dst[1] = make_uint4(cr.idx[4], cr.idx[5], cr.idx[6], cr.idx[7]);
}

}  // namespace hg
