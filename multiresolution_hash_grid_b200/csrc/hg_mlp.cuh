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
// Persistent CTAs, 2 per SM (2 x 64 of the 512 TMEM columns); the weights are staged in
// shared memory once. Warp-specialised per CTA (see the kernel): 20 producer warps (12 for
// F = 8) encode 128-point tiles into a double-buffered bf16 A operand, and 4
// consumer warps -- one per quarter of the 128 TMEM lanes -- issue each layer's MMAs
// (one elected thread, committed to an mbarrier, bounded waits) and read the accumulator
// rows back with tcgen05.ld to add the bias, apply ReLU and write the next layer's bf16
// operand, while the producers encode the next tile.
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
// Threads per CTA: 4 consumer warps + 20 producer warps (F <= 4, 40 registers a thread) or
// + 12 (F = 8, 64 registers); 2 CTAs per SM either way. Two CTAs of 768 rather than three
// of 512 gives more gathering warps per SM and leaves L1 more room beside shared memory.
// With lane-pair producers (F <= 4): 4 + 16 warps, so that the 256 producer pairs cover
// the 128 points of a tile exactly twice (48 registers a thread).
__host__ __device__ constexpr int block_threads(int F, bool lanes = false) {
    return lanes && F <= 4 ? 640 : (F == 8 ? 512 : 768);
}
constexpr int kCtasPerSm = 2;
constexpr int kTmemCols = 64;  // accumulator columns (fp32), reused by the three layers
constexpr uint32_t kWaitLimit = 1u << 22;

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

// Shared memory of the pipelined kernel: two encoding buffers, one hidden-activation buffer
// (a2 overwrites a1 once the second layer's MMAs have read it), the three weight matrices,
// the biases, five mbarriers and the TMEM address slot.
__host__ __device__ constexpr size_t ws_smem_bytes(int K1) {
    return 2 * (size_t)kM * K1 * 2 + (size_t)kM * kHid * 2 + (size_t)kHid * K1 * 2 + (size_t)kHid * kHid * 2 +
           (size_t)kOutPad * kHid * 2 + sizeof(float) * (kHid + kHid + kOutPad) + 5 * 8 + 8;
}

__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t mbar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}\n" ::"r"(mbar) : "memory");
}

// Named barrier 1 over the 4 consumer warps (barrier 0 is __syncthreads), reducing a
// predicate: true on every consumer thread if it was true on any of them.
__device__ __forceinline__ bool consumers_any(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.or.pred po, 1, 128, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)pred)
        : "memory");
    return r != 0;
}

// Warp-specialised pipeline. Warps 4..15 (producers) encode tile i into A0[i % 2], and each
// producer warp then arrives on full[i % 2]. Warps 0..3 (consumers, one per quarter of the
// 128 TMEM lanes) wait on it; one thread issues each layer's MMAs, the first layer's
// completion also arriving on empty[i % 2] to hand the buffer back to the producers for
// tile i + 2; the 4 warps run the epilogues. The encoding of the next tile thus overlaps
// the current tile's MMAs and epilogues. Every wait is bounded: a consumer that gives up
// makes all consumers stop together (the barrier vote) and raises the CTA's abort flag,
// which stops the producers before their next tile; the caller's status word is then set.
template <int F, typename TT, int K1, bool kLanes = false>
__global__ void __launch_bounds__(block_threads(F, kLanes), kCtasPerSm) mlp_forward_kernel(
    LevelParams lp, const float* __restrict__ x, int64_t N, const TT* __restrict__ table,
    const uint16_t* __restrict__ w1, const float* __restrict__ b1, const uint16_t* __restrict__ w2,
    const float* __restrict__ b2, const uint16_t* __restrict__ w3, const float* __restrict__ b3,
    float* __restrict__ y, int* __restrict__ status) {
    static_assert(K1 % 16 == 0 && K1 <= 64, "the encoding width must be a multiple of 16, at most 64");
    static_assert(!kLanes || F <= 4, "lane-pair producers need F <= 4");
    constexpr int kThreads = block_threads(F, kLanes);
    constexpr int kConsumers = kM;                     // 4 warps
    constexpr int kProducers = kThreads - kConsumers;  // 20 or 12 warps
    extern __shared__ __align__(1024) uint8_t sm[];
    // sm: A0[2][128][K1] encodings (buffer b at b * kM * K1 * 2), then the rest
    uint8_t* A1 = sm + 2 * kM * K1 * 2;             // [128][64] a1, then a2
    uint8_t* W1s = A1 + kM * kHid * 2;              // [64][K1]
    uint8_t* W2s = W1s + kHid * K1 * 2;             // [64][64]
    uint8_t* W3s = W2s + kHid * kHid * 2;           // [16][64] (rows 4..15 zero)
    float* bias = reinterpret_cast<float*>(W3s + kOutPad * kHid * 2);  // b1[64] b2[64] b3[16]
    uint64_t* bars = reinterpret_cast<uint64_t*>(bias + kHid + kHid + kOutPad);  // full[2] empty[2] mma
    uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 5);
    __shared__ int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    stage_matrix(W1s, w1, kHid, kHid, K1);
    stage_matrix(W2s, w2, kHid, kHid, kHid);
    stage_matrix(W3s, w3, kOutPad, kOut, kHid);
    for (int i = tid; i < kHid + kHid + kOutPad; i += kThreads)
        bias[i] = i < kHid ? b1[i] : (i < 2 * kHid ? b2[i - kHid] : (i - 2 * kHid < kOut ? b3[i - 2 * kHid] : 0.f));
    const uint32_t bar0 = (uint32_t)__cvta_generic_to_shared(bars);
    // mbarriers: full[b] at bar0 + 8 b, empty[b] at bar0 + 16 + 8 b, the MMA barrier at bar0 + 32
    const uint32_t mma_b = bar0 + 32;
    if (tid == 0) {
        abort_flag = 0;
        mbar_init(bar0, kProducers / 32);
        mbar_init(bar0 + 8, kProducers / 32);
        mbar_init(bar0 + 16, 1);
        mbar_init(bar0 + 24, 1);
        mbar_init(mma_b, 1);
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
    const int64_t ntiles = (N + kM - 1) / kM;
    const int my_tiles = blockIdx.x < ntiles ? (int)((ntiles - 1 - blockIdx.x) / gridDim.x + 1) : 0;

    if (warp >= kConsumers / 32) {
        // ------------------------------- producers -------------------------------
        // Thread pt keeps point q = pt % 128 of every tile (kProducers is a multiple of kM, so
        // x is read once per tile) and encodes every kStride-th level group of it; a warp
        // covers 32 consecutive points of one group. A group of G levels packs G*F bf16 values
        // into one 4-, 8- or 16-byte store within one core-matrix row.
        // With kLanes, a lane pair (the two threads 2j, 2j+1) shares one point of one level
        // group, thread d gathering the 4 corners with x offset d (as forward_kernel_lanes).
        constexpr int kPer = kLanes ? 2 : 1;  // threads per (point, group)
        static_assert(kProducers % (kM * kPer) == 0, "each producer thread (pair) owns one point of the tile");
        constexpr int G = F == 1 ? 2 : 1;
        constexpr int kStride = kProducers / (kM * kPer);
        const int pt = (tid - kConsumers) / kPer, q = pt & (kM - 1), ngroups = lp.L / G;
        const uint32_t d0 = (uint32_t)lane & 1u;
        const unsigned pair = 3u << (lane & 30);
        for (int i = 0; i < my_tiles; ++i) {
            const int b = i & 1;
            bool stop = i >= 2 && !wait_parity(bar0 + 16 + 8 * b, (uint32_t)(((i >> 1) - 1) & 1));
            stop = stop || *(volatile int*)&abort_flag != 0;
            if (__any_sync(0xffffffffu, stop)) {  // warp-uniform exit
                if (lane == 0) atomicExch(&abort_flag, 1);
                break;
            }
            const int64_t p = ((int64_t)blockIdx.x + (int64_t)i * gridDim.x) * kM + q;
            const bool valid = p < N;
            const bool xin = valid && in_bounds<kChkX>(x + p * 3, 12);
            const float x0 = xin ? __ldg(x + p * 3) : 0.f, x1 = xin ? __ldg(x + p * 3 + 1) : 0.f,
                        x2 = xin ? __ldg(x + p * 3 + 2) : 0.f;
            uint8_t* A0 = sm + b * (kM * K1 * 2);
            // The first group rotates with the tile, so that no warp always draws the extra
            // group when kStride does not divide the group count.
            for (int gi = (pt / kM + i) % kStride; gi < ngroups; gi += kStride) {
                float o[G * F];
                // One level at a time (not unrolled: two levels' gathers in flight would spill
                // at the 40 registers that 3 CTAs of 512 threads leave).
#pragma unroll 1
                for (int u = 0; u < G; ++u) {
                    const int l = gi * G + u;
                    float acc[F];
                    if constexpr (kLanes) {
                        HalfCorners hc;
                        locate_half(x0, x1, x2, lp.scale[l], lp.mask, d0, hc);
                        interpolate_pair<F, TT>(table + (uint64_t)l * lp.T * F, hc, pair, acc);
                    } else {
                        Corners cr;
                        locate_corners(x0, x1, x2, lp.scale[l], lp.mask, cr);
                        float e[8][F];
                        gather_corners<F, TT, kGatherCorner, std::is_same<TT, float>::value>(table + (uint64_t)l * lp.T * F, cr, e);
#pragma unroll
                        for (int f = 0; f < F; ++f) {
                            acc[f] = cr.w[0] * e[0][f];
#pragma unroll
                            for (int c = 1; c < 8; ++c) acc[f] = fmaf(cr.w[c], e[c][f], acc[f]);
                        }
                    }
#pragma unroll
                    for (int f = 0; f < F; ++f)
#pragma unroll
                        for (int uu = 0; uu < G; ++uu)  // constant indices: o stays in registers
                            if (uu == u) o[uu * F + f] = acc[f];
                }
                if (kLanes && d0 != 0) continue;  // both threads of a pair hold the sums; one stores
                uint8_t* dst = A0 + canon(q, gi * G * F, K1);  // G*F consecutive columns, one 16-byte row chunk
                if constexpr (G * F == 2) {
                    *reinterpret_cast<uint32_t*>(dst) = pack_bf16(o[0], o[1]);
                } else if constexpr (G * F == 4) {
                    *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]));
                } else {
                    *reinterpret_cast<uint4*>(dst) = make_uint4(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]),
                                                                pack_bf16(o[4], o[5]), pack_bf16(o[6], o[7]));
                }
            }
            fence_async_smem();  // this thread's operand writes -> visible to the tensor cores
            __syncwarp();
            if (lane == 0) mbar_arrive(bar0 + 8 * b);
        }
    } else {
        // ------------------------- consumers: MMAs + epilogues -------------------------
        const uint32_t sm0 = (uint32_t)__cvta_generic_to_shared(sm), a1s = (uint32_t)__cvta_generic_to_shared(A1), w1s = (uint32_t)__cvta_generic_to_shared(W1s),
                       w2s = (uint32_t)__cvta_generic_to_shared(W2s), w3s = (uint32_t)__cvta_generic_to_shared(W3s);
        constexpr uint32_t kIdHid = instr_desc(kM, kHid), kIdOut = instr_desc(kM, kOutPad);
        const uint32_t trow = tmem + ((uint32_t)(32 * warp) << 16);  // this warp's 32 TMEM lanes
        const int r = tid;                                            // accumulator row = TMEM lane
        uint32_t mma_phase = 0;
        bool ok = true, aborted = false;
        for (int i = 0; i < my_tiles && !aborted; ++i) {
            const int b = i & 1;
            const int64_t p0 = ((int64_t)blockIdx.x + (int64_t)i * gridDim.x) * kM;
            ok = wait_parity(bar0 + 8 * b, (uint32_t)((i >> 1) & 1)) && ok;
            for (int layer = 0; layer < 3; ++layer) {
                // The vote doubles as the barrier that orders the previous epilogue's TMEM
                // reads and operand writes before the next MMAs.
                fence_before();
                if (consumers_any(!ok)) {
                    aborted = true;
                    break;
                }
                if (tid == 0) {
                    fence_after();
                    const int K = layer == 0 ? K1 : kHid;
                    const uint32_t as = layer == 0 ? sm0 + b * (kM * K1 * 2) : a1s;
                    const uint32_t bs = layer == 0 ? w1s : (layer == 1 ? w2s : w3s);
                    for (int kk = 0; kk < K / 16; ++kk)
                        mma(tmem, smem_desc(as + kk * 256, K), smem_desc(bs + kk * 256, K),
                            layer == 2 ? kIdOut : kIdHid, kk > 0 ? 1u : 0u);
                    if (layer == 0) commit(bar0 + 16 + 8 * b);  // A0[b] may be refilled once these complete
                    commit(mma_b);
                }
                ok = wait_parity(mma_b, mma_phase);
                mma_phase ^= 1u;
                fence_after();
                const float* bl = bias + layer * kHid;
                if (layer < 2) {
#pragma unroll
                    for (int cc = 0; cc < kHid / 16; ++cc) {
                        float v[16];
                        tmem_ld16(trow + 16 * cc, v);
                        uint32_t w[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            w[j] = pack_bf16(fmaxf(v[2 * j] + bl[16 * cc + 2 * j], 0.f),
                                             fmaxf(v[2 * j + 1] + bl[16 * cc + 2 * j + 1], 0.f));
                        *reinterpret_cast<uint4*>(A1 + canon(r, 16 * cc, kHid)) = make_uint4(w[0], w[1], w[2], w[3]);
                        *reinterpret_cast<uint4*>(A1 + canon(r, 16 * cc + 8, kHid)) = make_uint4(w[4], w[5], w[6], w[7]);
                    }
                    fence_async_smem();
                } else {
                    float v[16];
                    tmem_ld16(trow, v);
                    const int64_t p = p0 + r;
                    if (ok && p < N && in_bounds<kChkOut>(y + p * kOut, 16))
                        __stcs(reinterpret_cast<float4*>(y + p * kOut),
                               make_float4(v[0] + bl[0], v[1] + bl[1], v[2] + bl[2], v[3] + bl[3]));
                }
            }
        }
        fence_before();
        if (!aborted) aborted = consumers_any(!ok);  // the last layer's wait
        if (aborted && tid == 0) atomicExch(&abort_flag, 1);
    }
    fence_before();
    __syncthreads();
    fence_after();
    if (tid == 0 && abort_flag != 0 && status != nullptr) atomicExch(status, 1);
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

}  // namespace mlp
}  // namespace hg
