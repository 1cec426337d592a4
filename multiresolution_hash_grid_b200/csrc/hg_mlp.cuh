// hg_mlp.cuh -- encoding fused with the small MLP that consumes it, on the sm_100a tensor
// cores (tcgen05 + TMEM).
//
// [NeRFace-HG] section 3: after the hash features comes a three-layer network of 64 units
// with ReLU; [Repro-HG] section 4: Linear(in, 64), ReLU, Linear(64, 64), ReLU,
// Linear(64, 4). Per point:  e = enc(x) (L*F values, computed as in forward_kernel);
//   a1 = relu(W1 e + b1), a2 = relu(W2 a1 + b2), y = W3 a2 + b3.
// The three layers are dense contractions over a tile of 128 points, so each runs as
// tcgen05.mma (kind::f16, bf16 x bf16 -> fp32, M = 128 points = the 128 TMEM lanes), with
// the encoding and the hidden activations rounded to bf16 as MMA operands and fp32
// accumulation in tensor memory. The encoding never leaves the SM.
//
// Persistent CTAs of 512 threads, up to 3 per SM (3 x 64 of the 512 TMEM columns) so one
// CTA's encoding overlaps another's MMAs: the weights are staged in shared memory once; per tile of
// 128 points the 16 warps encode (4 threads per point, each a quarter of the levels) into
// the bf16 A operand, one thread issues the layer's MMAs and commits them to an mbarrier,
// and after the (bounded) wait the 16 warps read the accumulator rows back with
// tcgen05.ld (warp w reads TMEM lanes 32 (w % 4) .. + 31, columns 16 (w / 4) .. + 15),
// add the bias, apply ReLU and write the next layer's bf16 operand.
//
// Operand layout: the canonical no-swizzle K-major layout of the tensor cores. An R x K
// bf16 matrix is tiled into 8 x 8 core matrices of 128 contiguous bytes (8 rows of 16 B);
// core matrices adjacent in K are 128 B apart (the descriptor's leading byte offset) and
// 8-row groups are K/8 * 128 B apart (stride byte offset). One MMA consumes K = 16, so the
// descriptors advance by 256 B per K step.
#pragma once

#include <cuda_bf16.h>

#include "hg_device.cuh"

namespace hg {
namespace mlp {

constexpr int kM = 128;        // points per tile = MMA M = TMEM lanes used
constexpr int kHid = 64;       // hidden width
constexpr int kOut = 4;        // outputs per point
constexpr int kOutPad = 16;    // MMA N of the last layer (the smallest N for M = 128)
constexpr int kThreads = 512;  // 16 warps
constexpr int kTmemCols = 64;  // accumulator columns (fp32), reused by the three layers
constexpr uint32_t kWaitLimit = 1u << 22;

__host__ __device__ constexpr size_t smem_bytes(int K1) {
    return (size_t)kM * K1 * 2 + 2 * (size_t)kM * kHid * 2 + (size_t)kHid * K1 * 2 + (size_t)kHid * kHid * 2 +
           (size_t)kOutPad * kHid * 2 + sizeof(float) * (kHid + kHid + kOutPad) + 16 /* mbarrier + tmem slot */;
}

// Byte offset of element (r, k) of an R x K bf16 matrix in the canonical layout.
__device__ __forceinline__ uint32_t canon(int r, int k, int K) {
    return (uint32_t)((r >> 3) * (K >> 3) * 128 + (k >> 3) * 128 + (r & 7) * 16 + (k & 7) * 2);
}

// Shared-memory matrix descriptor: start address, leading byte offset (K direction),
// stride byte offset (8-row groups), descriptor version 1 (bits 46-47), no swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, int K) {
    const uint64_t lbo = 128, sbo = (uint64_t)(K / 8) * 128;
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | (((lbo >> 4) & 0x3FFFu) << 16) |
           (((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Instruction descriptor of kind::f16: D fp32 (bits 4-5 = 1), A and B bf16 (bits 7-9 and
// 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 in bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t instr_desc(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
}

__device__ __forceinline__ bool wait_parity(uint32_t mbar, uint32_t parity) {
    for (uint32_t it = 0; it < kWaitLimit; ++it) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(ok)
            : "r"(mbar), "r"(parity)
            : "memory");
        if (ok) return true;
        __nanosleep(32);
    }
    return false;
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 16 consecutive fp32 accumulator columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Copy a row-major [R][K] bf16 global matrix into the canonical layout (rows >= Rsrc zero).
__device__ __forceinline__ void stage_matrix(uint8_t* dst, const uint16_t* __restrict__ src, int R, int Rsrc, int K) {
    const int chunks = R * (K / 8);
    for (int i = threadIdx.x; i < chunks; i += blockDim.x) {
        const int r = i / (K / 8), kc = i - r * (K / 8);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < Rsrc) v = __ldg(reinterpret_cast<const uint4*>(src + (size_t)r * K + kc * 8));
        *reinterpret_cast<uint4*>(dst + canon(r, kc * 8, K)) = v;
    }
}

// Epilogue of a hidden layer: rows of the TMEM accumulator + bias, ReLU, -> bf16 operand.
__device__ __forceinline__ void hidden_epilogue(uint32_t tmem, const float* bias, uint8_t* dst, int warp,
                                                int lane) {
    const int q = warp & 3, cc = warp >> 2;
    float v[16];
    tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + 16 * cc, v);
    const int r = 32 * q + lane;
    uint32_t w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
        w[j] = pack_bf16(fmaxf(v[2 * j] + bias[16 * cc + 2 * j], 0.f), fmaxf(v[2 * j + 1] + bias[16 * cc + 2 * j + 1], 0.f));
    *reinterpret_cast<uint4*>(dst + canon(r, 16 * cc, kHid)) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4*>(dst + canon(r, 16 * cc + 8, kHid)) = make_uint4(w[4], w[5], w[6], w[7]);
}

template <int F, typename TT, int K1>
__global__ void __launch_bounds__(kThreads, F == 8 ? 2 : 3) mlp_forward_kernel(
    LevelParams lp, const float* __restrict__ x, int64_t N, const TT* __restrict__ table,
    const uint16_t* __restrict__ w1, const float* __restrict__ b1, const uint16_t* __restrict__ w2,
    const float* __restrict__ b2, const uint16_t* __restrict__ w3, const float* __restrict__ b3,
    float* __restrict__ y, int* __restrict__ status) {
    static_assert(K1 % 16 == 0 && K1 <= 64, "the encoding width must be a multiple of 16, at most 64");
    extern __shared__ __align__(1024) uint8_t sm[];
    uint8_t* A0 = sm;                               // [128][K1]  encoding
    uint8_t* A1 = A0 + kM * K1 * 2;                 // [128][64]  a1
    uint8_t* A2 = A1 + kM * kHid * 2;               // [128][64]  a2
    uint8_t* W1s = A2 + kM * kHid * 2;              // [64][K1]
    uint8_t* W2s = W1s + kHid * K1 * 2;             // [64][64]
    uint8_t* W3s = W2s + kHid * kHid * 2;           // [16][64]   (rows 4..15 zero)
    float* bias = reinterpret_cast<float*>(W3s + kOutPad * kHid * 2);  // b1[64] b2[64] b3[16]
    uint64_t* mbar = reinterpret_cast<uint64_t*>(bias + kHid + kHid + kOutPad);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(mbar + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    stage_matrix(W1s, w1, kHid, kHid, K1);
    stage_matrix(W2s, w2, kHid, kHid, kHid);
    stage_matrix(W3s, w3, kOutPad, kOut, kHid);
    for (int i = tid; i < kHid + kHid + kOutPad; i += kThreads)
        bias[i] = i < kHid ? b1[i] : (i < 2 * kHid ? b2[i - kHid] : (i - 2 * kHid < kOut ? b3[i - 2 * kHid] : 0.f));
    const uint32_t mbar_s = (uint32_t)__cvta_generic_to_shared(mbar);
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mbar_s) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         (uint32_t)__cvta_generic_to_shared(tslot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    fence_async_smem();
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t a0 = (uint32_t)__cvta_generic_to_shared(A0), a1s = (uint32_t)__cvta_generic_to_shared(A1),
                   a2s = (uint32_t)__cvta_generic_to_shared(A2), w1s = (uint32_t)__cvta_generic_to_shared(W1s),
                   w2s = (uint32_t)__cvta_generic_to_shared(W2s), w3s = (uint32_t)__cvta_generic_to_shared(W3s);
    constexpr uint32_t kIdHid = instr_desc(kM, kHid), kIdOut = instr_desc(kM, kOutPad);
    uint32_t phase = 0;
    bool failed = false;

    const int64_t ntiles = (N + kM - 1) / kM;
    for (int64_t tile = blockIdx.x; tile < ntiles && !failed; tile += gridDim.x) {
        const int64_t p0 = tile * kM;
        // ---- encoding: thread = (point tid % 128, levels tid / 128, + 4, + 8, ...) ----
        {
            const int pt = tid & (kM - 1), lg = tid >> 7;
            const bool valid = p0 + pt < N;
            const float x0 = valid ? __ldg(x + (p0 + pt) * 3) : 0.f;
            const float x1 = valid ? __ldg(x + (p0 + pt) * 3 + 1) : 0.f;
            const float x2 = valid ? __ldg(x + (p0 + pt) * 3 + 2) : 0.f;
            for (int l = lg; l < lp.L; l += kThreads / kM) {
                Corners cr;
                locate_corners(x0, x1, x2, lp.scale[l], lp.mask, cr);
                float e[8][F];
                gather_corners<F, TT, kGatherCorner>(table + (uint64_t)l * lp.T * F, cr, e);
                float o[F];
#pragma unroll
                for (int f = 0; f < F; ++f) {
                    float acc = cr.w[0] * e[0][f];
#pragma unroll
                    for (int c = 1; c < 8; ++c) acc = fmaf(cr.w[c], e[c][f], acc);
                    o[f] = acc;
                }
                if constexpr (F == 1) {
                    *reinterpret_cast<__nv_bfloat16*>(A0 + canon(pt, l, K1)) = __float2bfloat16_rn(o[0]);
                } else {
                    // F even: the pairs (l*F + 2j, + 1) are adjacent within one core-matrix row
#pragma unroll
                    for (int j = 0; j < F / 2; ++j)
                        *reinterpret_cast<uint32_t*>(A0 + canon(pt, l * F + 2 * j, K1)) = pack_bf16(o[2 * j], o[2 * j + 1]);
                }
            }
        }
        // ---- three layers ----
        for (int layer = 0; layer < 3 && !failed; ++layer) {
            fence_async_smem();
            fence_before();
            __syncthreads();
            if (tid == 0) {
                fence_after();
                const int K = layer == 0 ? K1 : kHid;
                const uint32_t as = layer == 0 ? a0 : (layer == 1 ? a1s : a2s);
                const uint32_t bs = layer == 0 ? w1s : (layer == 1 ? w2s : w3s);
                const uint32_t id = layer == 2 ? kIdOut : kIdHid;
                for (int kk = 0; kk < K / 16; ++kk)
                    mma(tmem, smem_desc(as + kk * 256, K), smem_desc(bs + kk * 256, K), id, kk > 0 ? 1u : 0u);
                commit(mbar_s);
            }
            const bool ok = wait_parity(mbar_s, phase);
            phase ^= 1u;
            failed = __syncthreads_or(!ok) != 0;
            if (failed) break;
            fence_after();
            if (layer < 2) {
                hidden_epilogue(tmem, bias + layer * kHid, layer == 0 ? A1 : A2, warp, lane);
            } else if (warp < 4) {
                float v[16];
                tmem_ld16(tmem + ((uint32_t)(32 * warp) << 16), v);
                const int64_t p = p0 + 32 * warp + lane;
                if (p < N) {
                    const float* bo = bias + 2 * kHid;
                    __stcs(reinterpret_cast<float4*>(y + p * kOut),
                           make_float4(v[0] + bo[0], v[1] + bo[1], v[2] + bo[2], v[3] + bo[3]));
                }
            }
        }
    }
    if (failed && tid == 0 && status != nullptr) atomicExch(status, 1);
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

}  // namespace mlp
}  // namespace hg
