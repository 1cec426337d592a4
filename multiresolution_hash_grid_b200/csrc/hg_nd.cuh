// hg_nd.cuh -- the encoding for D-dimensional inputs (D = 2 or 4) on sm_100a.
//
// [Repro-HG] section 2.2 writes the hash for coordinates of any dimension as the XOR over
// axes of coordinate_i * pi_i (mod T), and section 3 lists the primes (1, 2654435761,
// 805459861, 3674653429, 2097192037, 1434869437, 2165219737). A D-dimensional point
// interpolates the 2^D corners of its cell with multilinear weights
// prod_i (offset_i ? frac_i : 1 - frac_i); corner c has offset bit i = (c >> i) & 1.
// These kernels follow the 3-D ones in hg_device.cuh (tiles of 64 points staged in shared
// memory; by default lane pairs, two threads per (point, level) split by x offset, since the
// first prime is 1 here too; otherwise one thread per (point, level) with x-pair merged
// reductions), with per-corner gathers and per-point reductions only.
#pragma once

#include "hg_device.cuh"

namespace hg {
namespace nd {

__device__ __constant__ uint32_t kPrimes[7] = {1u, 2654435761u, 805459861u, 3674653429u,
                                               2097192037u, 1434869437u, 2165219737u};

template <int D>
struct CornersND {
    static constexpr int kC = 1 << D;
    uint32_t idx[kC];
    float w[kC];
    float f[D];
};

// Cell, corner indices and weights of one point at one level (x*N_l in fp32, never fused).
template <int D>
__device__ __forceinline__ void locate(const float* xp, float scale, uint32_t mask, CornersND<D>& cr) {
    uint32_t h0[D], h1[D];
    float g[D];
#pragma unroll
    for (int i = 0; i < D; ++i) {
        const float xs = __fmul_rn(xp[i], scale);
        const int v = __float2int_rd(xs);
        cr.f[i] = __fsub_rn(xs, __int2float_rn(v));
        g[i] = 1.0f - cr.f[i];
        h0[i] = (uint32_t)v * kPrimes[i];
        h1[i] = h0[i] + kPrimes[i];
    }
#pragma unroll
    for (int c = 0; c < CornersND<D>::kC; ++c) {
        uint32_t h = 0;
        float w = 1.0f;
#pragma unroll
        for (int i = 0; i < D; ++i) {
            const bool b = (c >> i) & 1;
            h ^= b ? h1[i] : h0[i];
            w *= b ? cr.f[i] : g[i];
        }
        cr.idx[c] = h & mask;
        cr.w[c] = w;
    }
}

// The 2^(D-1) corners with x offset d0 (lane d0 of a lane pair, as the 3-D lane-pair
// kernels): corner k of the half is full corner c = d0 | (k << 1); index and weight as locate
// computes them for that corner.
template <int D>
struct HalfCornersND {
    static constexpr int kC = 1 << (D - 1);
    uint32_t idx[kC];
    float w[kC];
    float f[D];
};

template <int D>
__device__ __forceinline__ void locate_half(const float* xp, float scale, uint32_t mask, uint32_t d0,
                                            HalfCornersND<D>& cr) {
    uint32_t h0[D], h1[D];
    float g[D];
#pragma unroll
    for (int i = 0; i < D; ++i) {
        const float xs = __fmul_rn(xp[i], scale);
        const int v = __float2int_rd(xs);
        cr.f[i] = __fsub_rn(xs, __int2float_rn(v));
        g[i] = 1.0f - cr.f[i];
        h0[i] = (uint32_t)v * kPrimes[i];
        h1[i] = h0[i] + kPrimes[i];
    }
#pragma unroll
    for (int k = 0; k < HalfCornersND<D>::kC; ++k) {
        const int c = (int)d0 | (k << 1);
        uint32_t h = 0;
        float w = 1.0f;
#pragma unroll
        for (int i = 0; i < D; ++i) {
            const bool b = (c >> i) & 1;
            h ^= b ? h1[i] : h0[i];
            w *= b ? cr.f[i] : g[i];
        }
        cr.idx[k] = h & mask;
        cr.w[k] = w;
    }
}

constexpr int kTile = 64;

__host__ __device__ constexpr size_t tile_smem_bytes(int D, int L, int F) {
    return sizeof(float) * ((size_t)kTile * D + (size_t)kTile * (L * F + row_pad(F)));
}

// kLanes: a warp item is 16 points at one level as 16 lane pairs, lane d handling the 2^(D-1)
// corners with x offset d (the x prime is 1 here too); the pair adds its halves.
template <int D, int F, typename TT, bool kLanes = false>
__global__ void __launch_bounds__(512) forward_kernel(LevelParams lp, const float* __restrict__ x, int64_t N,
                                                      const TT* __restrict__ table, float* __restrict__ out) {
    extern __shared__ __align__(16) float smem[];
    const int L = lp.L, W = L * F, S = W + row_pad(F);
    float* xs = smem;
    float* os = smem + kTile * D;
    const int64_t p0 = (int64_t)blockIdx.x * kTile;
    const int nvalid = (int)min((int64_t)kTile, N - p0);
    stage_x(xs, x + p0 * D, nvalid * D);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    if constexpr (kLanes) {
        const uint32_t d0 = lane & 1;
        const unsigned pair = 3u << (lane & 30);
        for (int it = warp; it < (kTile / 16) * L; it += nwarps) {
            const int q = it / L, l = it - q * L, pl = q * 16 + (lane >> 1);
            if (pl >= nvalid) continue;  // both lanes of a pair
            HalfCornersND<D> cr;
            locate_half<D>(xs + pl * D, lp.scale[l], lp.mask, d0, cr);
            const TT* tl = table + (uint64_t)l * lp.T * F;
            float o[F];
#pragma unroll
            for (int f = 0; f < F; ++f) o[f] = 0.f;
#pragma unroll
            for (int k = 0; k < HalfCornersND<D>::kC; ++k) {
                float e[F];
                EntryLoad<F, TT>::load(tl + (uint64_t)cr.idx[k] * F, e);
#pragma unroll
                for (int f = 0; f < F; ++f) o[f] = fmaf(cr.w[k], e[f], o[f]);
            }
#pragma unroll
            for (int f = 0; f < F; ++f) o[f] += __shfl_xor_sync(pair, o[f], 1);
            store_half<F, false>(os + pl * S + l * F, o, d0);
        }
    } else {
        for (int it = warp; it < (kTile / 32) * L; it += nwarps) {
            const int q = it / L, l = it - q * L, pl = q * 32 + lane;
            if (pl >= nvalid) continue;
            CornersND<D> cr;
            locate<D>(xs + pl * D, lp.scale[l], lp.mask, cr);
            const TT* tl = table + (uint64_t)l * lp.T * F;
            float o[F];
#pragma unroll
            for (int f = 0; f < F; ++f) o[f] = 0.f;
#pragma unroll
            for (int c = 0; c < CornersND<D>::kC; ++c) {
                float e[F];
                EntryLoad<F, TT>::load(tl + (uint64_t)cr.idx[c] * F, e);
#pragma unroll
                for (int f = 0; f < F; ++f) o[f] = fmaf(cr.w[c], e[f], o[f]);
            }
            store_smem_entry<F>(os + pl * S + l * F, o);
        }
    }
    __syncthreads();
    stage_rows_out<(F < 4 ? F : 4)>(os, out, p0, nvalid, W, S);
}

// kLanes: lane pairs as in the forward; each lane reduces its corners one F-wide reduction
// each, so x-neighbouring corners are reduced by the same instruction.
template <int D, int F, typename GT, bool kLanes = false>
__global__ void __launch_bounds__(512) backward_kernel(LevelParams lp, const float* __restrict__ x,
                                                       const float* __restrict__ dout, int64_t N, GT* __restrict__ dtable) {
    extern __shared__ __align__(16) float smem[];
    const int L = lp.L, W = L * F, S = W + row_pad(F);
    float* xs = smem;
    float* gs = smem + kTile * D;
    const int64_t p0 = (int64_t)blockIdx.x * kTile;
    const int nvalid = (int)min((int64_t)kTile, N - p0);
    stage_x(xs, x + p0 * D, nvalid * D);
    stage_rows_in<(F < 4 ? F : 4)>(gs, dout, p0, nvalid, W, S);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    if constexpr (kLanes) {
        const uint32_t d0 = lane & 1;
        for (int it = warp; it < (kTile / 16) * L; it += nwarps) {
            const int q = it / L, l = it - q * L, pl = q * 16 + (lane >> 1);
            if (pl >= nvalid) continue;
            HalfCornersND<D> cr;
            locate_half<D>(xs + pl * D, lp.scale[l], lp.mask, d0, cr);
            float g[F];
            load_smem_entry<F>(gs + pl * S + l * F, g);
            GT* dl = dtable + (uint64_t)l * lp.T * F;
#pragma unroll
            for (int k = 0; k < HalfCornersND<D>::kC; ++k) {
                float v[F];
#pragma unroll
                for (int f = 0; f < F; ++f) v[f] = cr.w[k] * g[f];
                RedLane<F, GT>::add(dl + (uint64_t)cr.idx[k] * F, v);
            }
        }
    } else {
        for (int it = warp; it < (kTile / 32) * L; it += nwarps) {
            const int q = it / L, l = it - q * L, pl = q * 32 + lane;
            if (pl >= nvalid) continue;
            CornersND<D> cr;
            locate<D>(xs + pl * D, lp.scale[l], lp.mask, cr);
            float g[F];
            load_smem_entry<F>(gs + pl * S + l * F, g);
            GT* dl = dtable + (uint64_t)l * lp.T * F;
#pragma unroll
            for (int c = 0; c < CornersND<D>::kC; c += 2) {
                float va[F], vb[F];
#pragma unroll
                for (int f = 0; f < F; ++f) {
                    va[f] = cr.w[c] * g[f];
                    vb[f] = cr.w[c + 1] * g[f];
                }
                red_pair<F>(dl, cr.idx[c], cr.idx[c + 1], va, vb);
            }
        }
    }
}

// dL/dx_i = sum_l N_l sum_c (sum_f g e_c[f]) (d_i ? +1 : -1) prod_{j != i} (d_j ? frac_j : 1 - frac_j)
// kLanes: lane pairs as in the forward; the pair adds its halves of the D derivative sums.
template <int D, int F, typename TT, bool kLanes = false>
__global__ void __launch_bounds__(512) backward_input_kernel(LevelParams lp, const float* __restrict__ x,
                                                             const float* __restrict__ dout, int64_t N,
                                                             const TT* __restrict__ table, float* __restrict__ dx) {
    extern __shared__ __align__(16) float smem[];
    const int L = lp.L, W = L * F, S = W + row_pad(F);
    float* xs = smem;
    float* gs = smem + kTile * D;
    float* part = gs + kTile * S;  // [L][D][kTile]
    const int64_t p0 = (int64_t)blockIdx.x * kTile;
    const int nvalid = (int)min((int64_t)kTile, N - p0);
    stage_x(xs, x + p0 * D, nvalid * D);
    stage_rows_in<(F < 4 ? F : 4)>(gs, dout, p0, nvalid, W, S);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    if constexpr (kLanes) {
        const uint32_t d0 = lane & 1;
        const unsigned pair = 3u << (lane & 30);
        for (int it = warp; it < (kTile / 16) * L; it += nwarps) {
            const int q = it / L, l = it - q * L, pl = q * 16 + (lane >> 1);
            if (pl >= nvalid) continue;  // both lanes of a pair
            HalfCornersND<D> cr;
            locate_half<D>(xs + pl * D, lp.scale[l], lp.mask, d0, cr);
            float g[F];
            load_smem_entry<F>(gs + pl * S + l * F, g);
            const TT* tl = table + (uint64_t)l * lp.T * F;
            float d[D];
#pragma unroll
            for (int i = 0; i < D; ++i) d[i] = 0.f;
#pragma unroll
            for (int k = 0; k < HalfCornersND<D>::kC; ++k) {
                const int c = (int)d0 | (k << 1);
                float e[F];
                EntryLoad<F, TT>::load(tl + (uint64_t)cr.idx[k] * F, e);
                float sc = g[0] * e[0];
#pragma unroll
                for (int f = 1; f < F; ++f) sc = fmaf(g[f], e[f], sc);
#pragma unroll
                for (int i = 0; i < D; ++i) {
                    float pw = ((c >> i) & 1) ? sc : -sc;
#pragma unroll
                    for (int j = 0; j < D; ++j)
                        if (j != i) pw *= ((c >> j) & 1) ? cr.f[j] : 1.0f - cr.f[j];
                    d[i] += pw;
                }
            }
#pragma unroll
            for (int i = 0; i < D; ++i) d[i] += __shfl_xor_sync(pair, d[i], 1);
            if (d0 == 0) {
#pragma unroll
                for (int i = 0; i < D; ++i) part[(l * D + i) * kTile + pl] = lp.scale[l] * d[i];
            }
        }
    } else {
    for (int it = warp; it < (kTile / 32) * L; it += nwarps) {
        const int q = it / L, l = it - q * L, pl = q * 32 + lane;
        if (pl >= nvalid) continue;
        CornersND<D> cr;
        locate<D>(xs + pl * D, lp.scale[l], lp.mask, cr);
        float g[F];
        load_smem_entry<F>(gs + pl * S + l * F, g);
        const TT* tl = table + (uint64_t)l * lp.T * F;
        float d[D];
#pragma unroll
        for (int i = 0; i < D; ++i) d[i] = 0.f;
#pragma unroll
        for (int c = 0; c < CornersND<D>::kC; ++c) {
            float e[F];
            EntryLoad<F, TT>::load(tl + (uint64_t)cr.idx[c] * F, e);
            float sc = g[0] * e[0];
#pragma unroll
            for (int f = 1; f < F; ++f) sc = fmaf(g[f], e[f], sc);
#pragma unroll
            for (int i = 0; i < D; ++i) {
                float pw = ((c >> i) & 1) ? sc : -sc;
#pragma unroll
                for (int j = 0; j < D; ++j)
                    if (j != i) pw *= ((c >> j) & 1) ? cr.f[j] : 1.0f - cr.f[j];
                d[i] += pw;
            }
        }
#pragma unroll
        for (int i = 0; i < D; ++i) part[(l * D + i) * kTile + pl] = lp.scale[l] * d[i];
    }
    }
    __syncthreads();
    for (int t = threadIdx.x; t < nvalid * D; t += blockDim.x) {
        const int pt = t / D, i = t - D * (t / D);
        float s = 0.f;
        for (int l = 0; l < L; ++l) s += part[(l * D + i) * kTile + pt];
        if (in_bounds<kChkOut>(dx + p0 * D + t, 4)) __stcs(dx + p0 * D + t, s);
    }
}

template <int D>
__global__ void __launch_bounds__(256) indices_kernel(LevelParams lp, const float* __restrict__ x, int64_t N,
                                                      uint32_t* __restrict__ idx) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= N * lp.L) return;
    const int64_t p = t / lp.L;
    const int l = (int)(t - p * lp.L);
    float xp[D];
#pragma unroll
    for (int i = 0; i < D; ++i) xp[i] = ld_x(x + p * D + i);
    CornersND<D> cr;
    locate<D>(xp, lp.scale[l], lp.mask, cr);
#pragma unroll
    for (int c = 0; c < CornersND<D>::kC; ++c)
        if (in_bounds<kChkOut>(idx + t * CornersND<D>::kC + c, 4)) idx[t * CornersND<D>::kC + c] = cr.idx[c];
}

}  // namespace nd
}  // namespace hg
