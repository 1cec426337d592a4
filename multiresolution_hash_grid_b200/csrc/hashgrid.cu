// hashgrid.cu -- C ABI of libhashgrid.so (declared in include/hashgrid.h): handle, host-side
// validation and kernel launches for the multiresolution hash-grid encoding on sm_100a.
//
// Every argument is checked on the host before anything is launched: ranges, NULLs,
// 16-byte alignment, that each pointer is device-accessible memory of the current device,
// and (for cudaMalloc'd memory) that the whole extent the call will touch lies inside the
// pointer's allocation. A call either launches its kernels or returns an error having
// written nothing.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <initializer_list>
#include <new>
#include <string>
#include <type_traits>

#include "hashgrid.h"
#include "hg_device.cuh"
#include "hg_mlp.cuh"
#include "hg_nd.cuh"
#include "hg_probe.cuh"
#include "hashgrid_probe.h"

#ifdef HASHGRID_CHECKED
#define HASHGRID_VERSION_STRING "hashgrid-b200 0.2 (sm_100a, checked)"
#else
#define HASHGRID_VERSION_STRING "hashgrid-b200 0.2 (sm_100a)"
#endif

struct hashgrid_s {
    int D;  // input dimensions (3 for hashgrid_create)
    int L, F, log2T, N_min, N_max, dtype;
    int res[HASHGRID_MAX_LEVELS];
    int forward_gather;   // HASHGRID_GATHER_*
    int backward_mode;    // HASHGRID_BACKWARD_*
    int schedule;         // HASHGRID_SCHEDULE_*
    hg::LevelParams lp;
};

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

int ok() { return HASHGRID_OK; }

// Resolution schedule, [NeRFace-HG] section 2: b = exp((ln N_max - ln N_min)/(L - 1)),
// N_l = floor(N_min * b^l) of the exact-math value. In double, N_min * b^l can fall a few
// ulp short of an integer it equals exactly (16 * b^15 = 4095.99999... for N_max = 4096);
// a value within 1e-9 (relative) of an integer is taken as that integer, any other value
// is floored.
bool compute_resolutions(int L, int N_min, int N_max, int* res) {
    if (L == 1) {
        if (N_min != N_max) return false;
        res[0] = N_min;
        return true;
    }
    const double b = std::exp((std::log((double)N_max) - std::log((double)N_min)) / (double)(L - 1));
    for (int l = 0; l < L; ++l) {
        const double v = (double)N_min * std::pow(b, (double)l);
        const double r = std::nearbyint(v);
        res[l] = (int)((std::fabs(v - r) <= 1e-9 * v) ? r : std::floor(v));
    }
    return true;
}

// cuMemGetAddressRange through the runtime's driver entry-point query, so the library
// needs no link-time dependency on libcuda.
typedef CUresult (*PFN_memGetAddressRange)(CUdeviceptr*, size_t*, CUdeviceptr);

PFN_memGetAddressRange address_range_fn() {
    static PFN_memGetAddressRange fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            p = nullptr;
        }
        return reinterpret_cast<PFN_memGetAddressRange>(p);
    }();
    return fn;
}

// Checks one buffer argument that the call will access over [p, p + bytes): not NULL,
// 16-byte aligned, device memory of the current device or managed memory, and (where the
// driver reports the allocation's range) the whole extent inside the allocation.
int check_buffer(const void* p, size_t bytes, const char* name) {
    if (p == nullptr) return fail(HASHGRID_ERR_ARG, "%s is NULL", name);
    if (reinterpret_cast<uintptr_t>(p) % 16 != 0)
        return fail(HASHGRID_ERR_ALIGN, "%s (%p) is not 16-byte aligned", name, p);
    cudaPointerAttributes a;
    cudaError_t e = cudaPointerGetAttributes(&a, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(HASHGRID_ERR_ARG, "%s (%p): cudaPointerGetAttributes failed: %s", name, p,
                    cudaGetErrorString(e));
    }
    if (a.type == cudaMemoryTypeUnregistered || a.devicePointer == nullptr)
        return fail(HASHGRID_ERR_ARG, "%s (%p) is not device-accessible memory", name, p);
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return fail(HASHGRID_ERR_CUDA, "cudaGetDevice failed");
    }
    // Host memory (pinned or registered) is device-accessible but its extent cannot be
    // checked here, and the kernels would read it across the host link: not accepted.
    if (a.type == cudaMemoryTypeHost)
        return fail(HASHGRID_ERR_ARG, "%s (%p) is host memory; the library takes device memory", name, p);
    if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
        return fail(HASHGRID_ERR_ARG, "%s (%p) has unknown memory type %d", name, p, (int)a.type);
    if (a.type == cudaMemoryTypeDevice && a.device != dev)
        return fail(HASHGRID_ERR_ARG, "%s lives on device %d but device %d is current", name, a.device, dev);
    // The extent the call touches must lie inside the pointer's allocation. Device memory
    // whose range the driver cannot report (none is known) is accepted as before; managed
    // memory is accepted only when its range is known.
    PFN_memGetAddressRange range = address_range_fn();
    CUdeviceptr base = 0;
    size_t size = 0;
    const bool known = range != nullptr && range(&base, &size, (CUdeviceptr)(uintptr_t)p) == CUDA_SUCCESS;
    if (known) {
        const uintptr_t end = (uintptr_t)base + size;
        if ((uintptr_t)p + bytes > end || (uintptr_t)p + bytes < (uintptr_t)p)
            return fail(HASHGRID_ERR_ARG,
                        "%s: the call touches %zu bytes from %p but its allocation ends %zu bytes after it", name,
                        bytes, p, (size_t)(end - (uintptr_t)p));
    } else if (a.type == cudaMemoryTypeManaged) {
        return fail(HASHGRID_ERR_ARG, "%s (%p): the extent of this managed allocation cannot be checked", name, p);
    }
    return ok();
}

int check_handle(const hashgrid_s* h) {
    if (h == nullptr) return fail(HASHGRID_ERR_ARG, "handle is NULL");
    return ok();
}

int check_N(int64_t N, int BP) {
    if (N < 0) return fail(HASHGRID_ERR_ARG, "N = %lld is negative", (long long)N);
    if ((N + BP - 1) / BP > 0x7fffffffLL)
        return fail(HASHGRID_ERR_ARG, "N = %lld exceeds the largest launchable batch", (long long)N);
    return ok();
}

int launch_status(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return fail(HASHGRID_ERR_CUDA, "%s launch failed: %s", what, cudaGetErrorString(e));
    return ok();
}

constexpr int kTile = 64;      // points per block tile
constexpr int kMaxThreads = 512;

int tile_threads(int L) {
    const int items = (kTile / 32) * L;
    return items * 32 < kMaxThreads ? items * 32 : kMaxThreads;
}

template <typename K>
int prepare_smem(K kernel, size_t smem) {
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return fail(HASHGRID_ERR_CUDA, "cudaFuncSetAttribute(smem=%zu) failed: %s", smem,
                        cudaGetErrorString(e));
        }
    }
    return ok();
}

template <int F, typename TT>
int launch_forward(const hashgrid_s* h, const float* x, int64_t N, const void* table, float* out,
                   int gather, cudaStream_t s) {
    const size_t smem = hg::tile_smem_bytes(kTile, h->L, F);
    const unsigned blocks = (unsigned)((N + kTile - 1) / kTile);
    if (gather == hg::kGatherLanes) {
        auto k = hg::forward_kernel_lanes<F, TT, kTile>;
        if (int rc = prepare_smem(k, smem)) return rc;
        // a warp item is 16 points at one level: (kTile / 16) * L items per tile
        const int items = (kTile / 16) * h->L;
        const int threads = items * 32 < kMaxThreads ? items * 32 : kMaxThreads;
        k<<<blocks, threads, smem, s>>>(h->lp, x, N, static_cast<const TT*>(table), out);
        return launch_status("forward");
    }
    auto k = gather == hg::kGatherSector ? hg::forward_kernel<F, TT, kTile, hg::kGatherSector>
           : gather == hg::kGatherPair   ? hg::forward_kernel<F, TT, kTile, hg::kGatherPair>
                                         : hg::forward_kernel<F, TT, kTile, hg::kGatherCorner>;
    if (int rc = prepare_smem(k, smem)) return rc;
    k<<<blocks, tile_threads(h->L), smem, s>>>(h->lp, x, N, static_cast<const TT*>(table), out);
    return launch_status("forward");
}

template <int F, int kMode, typename GT = float>
int launch_backward_mode(const hashgrid_s* h, const float* x, const float* dout, int64_t N,
                         GT* dtable, cudaStream_t s) {
    const int cap = hg::backward_threads(kMode);
    const int threads = tile_threads(h->L) < cap ? tile_threads(h->L) : cap;
    const size_t smem = hg::tile_smem_bytes(kTile, h->L, F) +
                        (kMode == hg::kAtomicOnly ? 0 : hg::group_smem_bytes(threads / 32, F));
    const unsigned blocks = (unsigned)((N + kTile - 1) / kTile);
    if constexpr (kMode == hg::kAtomicOnly) {
        auto k = hg::backward_kernel_atomic<F, kTile, GT>;
        if (int rc = prepare_smem(k, smem)) return rc;
        k<<<blocks, threads, smem, s>>>(h->lp, x, dout, N, dtable);
    } else {
        auto k = hg::backward_kernel_grouped<F, kTile, kMode>;
        if (int rc = prepare_smem(k, smem)) return rc;
        k<<<blocks, threads, smem, s>>>(h->lp, x, dout, N, dtable);
    }
    return launch_status("backward");
}

// The forward kernel a handle's gather option selects (AUTO: lane pairs, measured fastest
// on every workload: per 2^20 ray samples 225 against 250 us per-corner, per 2^18 uniform
// points 81 against 95 us, fp16 table 1.02 against 1.23 ms per 2^22 points).
int forward_gather_kernel(const hashgrid_s* h) {
    switch (h->forward_gather) {
        case HASHGRID_GATHER_CORNER: return hg::kGatherCorner;
        case HASHGRID_GATHER_SECTOR: return hg::kGatherSector;
        case HASHGRID_GATHER_PAIR: return hg::kGatherPair;
        default: return hg::kGatherLanes;
    }
}

// The run walk a handle's backward option selects for F <= 4: lane pairs for AUTO and
// RUN_LANES (measured 356 against 424 us per 2^20 ray samples, 1.74 against 2.10 ms per
// 2^22 uniform points), one lane per run for RUN_MERGE.
bool run_lanes(const hashgrid_s* h) {
    return h->backward_mode == HASHGRID_BACKWARD_RUN_LANES || h->backward_mode == HASHGRID_BACKWARD_AUTO;
}

// Level-major when asked, or (AUTO) when the whole table is larger than most of L2.
constexpr size_t kLevelMajorTableBytes = 96u << 20;

// Level groups of the level-major lane-pair kernels. A level's points in the unit cube reach
// at most min(T, (N_l + 2)^3) entries, so the coarse levels of a large table touch only a
// few MB of their slices. Consecutive levels are grouped while the entries they can reach
// (counted at 4F bytes, the fp32 gradient's width) stay within 32 MB, a quarter of the L2;
// a level above that is a group of its own. One pass per group then reads x and writes the
// output rows once for all its levels. (1 GiB grid, L = 16, F = 4: levels 0-5 reach 26.5 MB
// together and form one group, levels 6-15 one group each.)
constexpr double kLevelGroupBytes = 32.0 * (1 << 20);

void compute_level_groups(hashgrid_s* h) {
    const double T = (double)((uint64_t)1 << h->log2T);
    int g = 0;
    double acc = 0.0;
    h->lp.group_lo[0] = 0;
    for (int l = 0; l < h->L; ++l) {
        const double v = (double)h->res[l] + 2.0;
        const double bytes = std::min(T, v * v * v) * h->F * 4.0;
        if (l > 0 && acc + bytes > kLevelGroupBytes) {
            h->lp.group_lo[++g] = l;
            acc = 0.0;
        }
        acc += bytes;
    }
    h->lp.group_lo[++g] = h->L;
    h->lp.ngroups = g;
}

bool level_major(const hashgrid_s* h) {
    if (h->schedule == HASHGRID_SCHEDULE_LEVEL_MAJOR) return true;
    if (h->schedule == HASHGRID_SCHEDULE_POINT_MAJOR) return false;
    const size_t bytes = (size_t)h->L * ((size_t)1 << h->log2T) * h->F * (h->dtype == HASHGRID_F16 ? 2 : 4);
    return bytes > kLevelMajorTableBytes;
}

template <int F, typename TT>
int launch_forward_levels(const hashgrid_s* h, const float* x, int64_t N, const void* table, float* out,
                          int gather, cudaStream_t s) {
    if (gather == hg::kGatherLanes) {  // two threads per point
        const dim3 grid((unsigned)((2 * N + hg::kLevelBlock - 1) / hg::kLevelBlock), (unsigned)h->lp.ngroups);
        hg::forward_kernel_levels_lanes<F, TT><<<grid, hg::kLevelBlock, 0, s>>>(h->lp, x, N, static_cast<const TT*>(table), out);
        return launch_status("forward");
    }
    const dim3 grid((unsigned)((N + hg::kLevelBlock - 1) / hg::kLevelBlock), (unsigned)h->L);
    hg::forward_kernel_levels<F, TT><<<grid, hg::kLevelBlock, 0, s>>>(h->lp, x, N, static_cast<const TT*>(table), out);
    return launch_status("forward");
}

// Run merging for every mode but ATOMIC (the warp-dedup modes have no level-major form);
// lane pairs for RUN_LANES.
template <int F, typename GT>
int launch_backward_levels(const hashgrid_s* h, const float* x, const float* dout, int64_t N, GT* dtable,
                           cudaStream_t s) {
    if constexpr (F <= 4) {
        if (run_lanes(h)) {
            const int64_t runs = (N + hg::kRun - 1) / hg::kRun;
            const dim3 grid((unsigned)((2 * runs + hg::kLevelBlock - 1) / hg::kLevelBlock), (unsigned)h->lp.ngroups);
            hg::backward_kernel_runs_levels_lanes<F, GT><<<grid, hg::kLevelBlock, 0, s>>>(h->lp, x, dout, N, dtable);
            return launch_status("backward");
        }
        if (h->backward_mode != HASHGRID_BACKWARD_ATOMIC) {
            const int64_t runs = (N + hg::kRun - 1) / hg::kRun;
            const dim3 grid((unsigned)((runs + hg::kLevelBlock - 1) / hg::kLevelBlock), (unsigned)h->L);
            hg::backward_kernel_runs_levels<F, GT><<<grid, hg::kLevelBlock, 0, s>>>(h->lp, x, dout, N, dtable);
            return launch_status("backward");
        }
    }
    const dim3 grid((unsigned)((N + hg::kLevelBlock - 1) / hg::kLevelBlock), (unsigned)h->L);
    hg::backward_kernel_atomic_levels<F, GT><<<grid, hg::kLevelBlock, 0, s>>>(h->lp, x, dout, N, dtable);
    return launch_status("backward");
}

template <int F, typename GT = float>
int launch_backward_runs(const hashgrid_s* h, const float* x, const float* dout, int64_t N,
                         GT* dtable, cudaStream_t s) {
    const bool lanes = run_lanes(h);
    auto k = lanes ? hg::backward_kernel_runs_lanes<F, GT> : hg::backward_kernel_runs<F, GT>;
    const size_t smem = lanes ? hg::run_smem_bytes(h->L, F, hg::kRunPairTile / hg::kRunPair, hg::kRunPair)
                              : hg::run_smem_bytes(h->L, F);
    if (int rc = prepare_smem(k, smem)) return rc;
    const int64_t tile = lanes ? hg::kRunPairTile : hg::kRunTile;
    const unsigned blocks = (unsigned)((N + tile - 1) / tile);
    k<<<blocks, 256, smem, s>>>(h->lp, x, dout, N, dtable);
    return launch_status("backward");
}

// fp16 gradient tables: run merging (every mode but ATOMIC) or per-point reductions.
template <int F>
int launch_backward_half(const hashgrid_s* h, const float* x, const float* dout, int64_t N, __half* dtable,
                         cudaStream_t s) {
    if (level_major(h)) return launch_backward_levels<F, __half>(h, x, dout, N, dtable, s);
    if constexpr (F <= 4) {
        if (h->backward_mode != HASHGRID_BACKWARD_ATOMIC) return launch_backward_runs<F, __half>(h, x, dout, N, dtable, s);
    }
    return launch_backward_mode<F, hg::kAtomicOnly, __half>(h, x, dout, N, dtable, s);
}

template <int F>
int launch_backward(const hashgrid_s* h, const float* x, const float* dout, int64_t N,
                    float* dtable, cudaStream_t s) {
    const bool grouped = h->backward_mode == HASHGRID_BACKWARD_WARP_DEDUP ||
                         h->backward_mode == HASHGRID_BACKWARD_WARP_DEDUP_ADAPTIVE;
    if (!grouped && level_major(h)) return launch_backward_levels<F, float>(h, x, dout, N, dtable, s);
    if constexpr (F <= 4) {
        if (h->backward_mode == HASHGRID_BACKWARD_RUN_MERGE || h->backward_mode == HASHGRID_BACKWARD_AUTO ||
            h->backward_mode == HASHGRID_BACKWARD_RUN_LANES)
            return launch_backward_runs<F>(h, x, dout, N, dtable, s);
        if (h->backward_mode == HASHGRID_BACKWARD_WARP_DEDUP)
            return launch_backward_mode<F, hg::kGroupAlways>(h, x, dout, N, dtable, s);
        if (h->backward_mode == HASHGRID_BACKWARD_WARP_DEDUP_ADAPTIVE)
            return launch_backward_mode<F, hg::kAdaptive>(h, x, dout, N, dtable, s);
    }
    return launch_backward_mode<F, hg::kAtomicOnly>(h, x, dout, N, dtable, s);
}

// dL/dx: warp-owned lane pairs when the gather option selects lane pairs (AUTO, LANES),
// else one thread per (point, level). A warp stages its 16 upstream-gradient rows: 16 warps
// per block for rows of up to 64 floats, 4 above (shared memory).
template <int F, typename TT, int kW>
int launch_backward_input_warp(const hashgrid_s* h, const float* x, const float* dout, int64_t N, const void* table,
                               float* dx, cudaStream_t s) {
    auto k = hg::backward_input_kernel_warp<F, TT, kW>;
    const size_t smem = sizeof(float) * (size_t)kW * hg::kWarpPoints * (h->L * F + hg::row_pad(F));
    if (int rc = prepare_smem(k, smem)) return rc;
    const int64_t pts = (int64_t)kW * hg::kWarpPoints;
    k<<<(unsigned)((N + pts - 1) / pts), 32 * kW, smem, s>>>(h->lp, x, dout, N, static_cast<const TT*>(table), dx);
    return launch_status("backward_input");
}

template <int F, typename TT>
int launch_backward_input(const hashgrid_s* h, const float* x, const float* dout, int64_t N, const void* table,
                          float* dx, cudaStream_t s) {
    if (forward_gather_kernel(h) == hg::kGatherLanes)
        return h->L * F <= 64 ? launch_backward_input_warp<F, TT, 16>(h, x, dout, N, table, dx, s)
                              : launch_backward_input_warp<F, TT, 4>(h, x, dout, N, table, dx, s);
    auto k = hg::backward_input_kernel<F, TT, kTile>;
    const size_t smem = hg::input_grad_smem_bytes(kTile, h->L, F);
    if (int rc = prepare_smem(k, smem)) return rc;
    const unsigned blocks = (unsigned)((N + kTile - 1) / kTile);
    k<<<blocks, tile_threads(h->L), smem, s>>>(h->lp, x, dout, N, static_cast<const TT*>(table), dx);
    return launch_status("backward_input");
}

template <int F, typename TT, int K1>
int launch_mlp_forward(const hashgrid_s* h, const float* x, int64_t N, const void* table, const void* w1,
                       const float* b1, const void* w2, const float* b2, const void* w3, const float* b3, float* y,
                       int* status, cudaStream_t s) {
    // lane-pair producers when the gather option selects lane pairs (F <= 4)
    constexpr bool kCanLanes = F <= 4;
    const bool lanes = kCanLanes && forward_gather_kernel(h) == hg::kGatherLanes;
    auto k = lanes ? hg::mlp::mlp_forward_kernel<F, TT, K1, kCanLanes> : hg::mlp::mlp_forward_kernel<F, TT, K1, false>;
    const size_t smem = hg::mlp::ws_smem_bytes(K1);
    if (int rc = prepare_smem(k, smem)) return rc;
    int dev = 0, sms = 148, smem_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    // Persistent grid: as many CTAs as fit per SM (registers allow 2; shared memory as
    // computed, with the 1 KB the runtime reserves per CTA). More would only queue behind the
    // resident ones.
    const int fit = (int)((size_t)smem_sm / (smem + 1024));
    const int per_sm = std::max(1, std::min(hg::mlp::kCtasPerSm, fit));
    const int64_t tiles = (N + hg::mlp::kM - 1) / hg::mlp::kM;
    const int64_t cap = (int64_t)sms * per_sm;
    const unsigned blocks = (unsigned)(tiles < cap ? tiles : cap);
    k<<<blocks, hg::mlp::block_threads(F, lanes), smem, s>>>(h->lp, x, N, static_cast<const TT*>(table),
                                               static_cast<const uint16_t*>(w1), b1, static_cast<const uint16_t*>(w2),
                                               b2, static_cast<const uint16_t*>(w3), b3, y, status);
    return launch_status("mlp_forward");
}

template <int F, typename TT>
int dispatch_mlp_forward(const hashgrid_s* h, const float* x, int64_t N, const void* table, const void* w1,
                         const float* b1, const void* w2, const float* b2, const void* w3, const float* b3, float* y,
                         int* status, cudaStream_t s) {
    switch (h->L * F) {
        case 16: return launch_mlp_forward<F, TT, 16>(h, x, N, table, w1, b1, w2, b2, w3, b3, y, status, s);
        case 32: return launch_mlp_forward<F, TT, 32>(h, x, N, table, w1, b1, w2, b2, w3, b3, y, status, s);
        case 48: return launch_mlp_forward<F, TT, 48>(h, x, N, table, w1, b1, w2, b2, w3, b3, y, status, s);
        case 64: return launch_mlp_forward<F, TT, 64>(h, x, N, table, w1, b1, w2, b2, w3, b3, y, status, s);
    }
    return fail(HASHGRID_ERR_ARG, "the MLP needs L*F in {16, 32, 48, 64}, got %d", h->L * F);
}

// D-dimensional inputs (D = 2, 4): per-corner gathers and per-point reductions, with lane
// pairs (two threads per (point, level), split by x offset) when the LANES gather option
// (forward, dL/dx) or the RUN_LANES backward option asks for them, and under AUTO for D = 4.
// Measured per 2^20 uniform points of the default grid: D = 4 forward 533 against 802 us,
// backward 784 against 927, dL/dx 569 against 764; D = 2 forward 185 against 161 us, backward
// 449 against 415 (4 corners: the duplicated locate and hash cost more than the shared
// sectors save).
bool nd_lanes_fwd(const hashgrid_s* h) {
    return h->forward_gather == HASHGRID_GATHER_LANES || (h->forward_gather == HASHGRID_GATHER_AUTO && h->D == 4);
}
bool nd_lanes_bwd(const hashgrid_s* h) {
    return h->backward_mode == HASHGRID_BACKWARD_RUN_LANES || (h->backward_mode == HASHGRID_BACKWARD_AUTO && h->D == 4);
}

int nd_threads(const hashgrid_s* h, bool lanes) {
    const int items = (hg::nd::kTile / (lanes ? 16 : 32)) * h->L;
    return items * 32 < kMaxThreads ? items * 32 : kMaxThreads;
}

template <int D, int F, typename TT>
int launch_nd_forward(const hashgrid_s* h, const float* x, int64_t N, const void* table, float* out, cudaStream_t s) {
    const bool lanes = nd_lanes_fwd(h);
    auto k = lanes ? hg::nd::forward_kernel<D, F, TT, true> : hg::nd::forward_kernel<D, F, TT, false>;
    const size_t smem = hg::nd::tile_smem_bytes(D, h->L, F);
    if (int rc = prepare_smem(k, smem)) return rc;
    k<<<(unsigned)((N + hg::nd::kTile - 1) / hg::nd::kTile), nd_threads(h, lanes), smem, s>>>(
        h->lp, x, N, static_cast<const TT*>(table), out);
    return launch_status("forward");
}

template <int D, int F, typename GT>
int launch_nd_backward(const hashgrid_s* h, const float* x, const float* dout, int64_t N, GT* dtable, cudaStream_t s) {
    const bool lanes = nd_lanes_bwd(h);
    auto k = lanes ? hg::nd::backward_kernel<D, F, GT, true> : hg::nd::backward_kernel<D, F, GT, false>;
    const size_t smem = hg::nd::tile_smem_bytes(D, h->L, F);
    if (int rc = prepare_smem(k, smem)) return rc;
    k<<<(unsigned)((N + hg::nd::kTile - 1) / hg::nd::kTile), nd_threads(h, lanes), smem, s>>>(h->lp, x, dout, N, dtable);
    return launch_status("backward");
}

template <int D, int F, typename TT>
int launch_nd_backward_input(const hashgrid_s* h, const float* x, const float* dout, int64_t N, const void* table,
                             float* dx, cudaStream_t s) {
    const bool lanes = nd_lanes_fwd(h);
    auto k = lanes ? hg::nd::backward_input_kernel<D, F, TT, true> : hg::nd::backward_input_kernel<D, F, TT, false>;
    const size_t smem = hg::nd::tile_smem_bytes(D, h->L, F) + sizeof(float) * (size_t)hg::nd::kTile * h->L * D;
    if (int rc = prepare_smem(k, smem)) return rc;
    k<<<(unsigned)((N + hg::nd::kTile - 1) / hg::nd::kTile), nd_threads(h, lanes), smem, s>>>(
        h->lp, x, dout, N, static_cast<const TT*>(table), dx);
    return launch_status("backward_input");
}

// Calls fn<D, F>() for the handle's D (2 or 4) and F.
template <class Fn>
int nd_dispatch(const hashgrid_s* h, Fn&& fn) {
#define HG_ND_CASE(DD, FF) \
    if (h->D == DD && h->F == FF) return fn(std::integral_constant<int, DD>(), std::integral_constant<int, FF>());
    HG_ND_CASE(2, 1) HG_ND_CASE(2, 2) HG_ND_CASE(2, 4) HG_ND_CASE(2, 8)
    HG_ND_CASE(4, 1) HG_ND_CASE(4, 2) HG_ND_CASE(4, 4) HG_ND_CASE(4, 8)
#undef HG_ND_CASE
    return fail(HASHGRID_ERR_ARG, "corrupt handle");
}

// Buffers of one call for the checked build's range checks: (role, base, bytes).
struct CheckBuf {
    int role;
    const void* p;
    size_t bytes;
};

// Runs fn (the call's launches). In the checked build (HASHGRID_CHECKED) the byte ranges
// of the call's buffers are first recorded for the kernels' range checks (roles the call
// does not use stay unrestricted), and after the launches the device status word is read
// back on the call's stream: a tripped check is cleared and reported as
// HASHGRID_ERR_DEVICE_CHECK. Calls are then synchronous, and calls running at the same
// time on several streams would share the recorded ranges: the checked build is for one
// stream at a time. In the regular build this only calls fn.
template <class Fn>
int run_checked(cudaStream_t s, std::initializer_list<CheckBuf> bufs, const char* what, Fn&& fn) {
#ifdef HASHGRID_CHECKED
    // the status word is read back after the kernel: not possible inside stream capture
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) {
        cudaGetLastError();
        return fail(HASHGRID_ERR_CUDA, "%s: cudaStreamIsCapturing failed", what);
    }
    if (cap != cudaStreamCaptureStatusNone)
        return fail(HASHGRID_ERR_ARG, "%s: the checked build cannot run inside stream capture", what);
    hg::CheckRanges r;
    for (int i = 0; i < hg::kChkRoles; ++i) {
        r.lo[i] = 0;
        r.hi[i] = ~0ull;
    }
    for (const CheckBuf& b : bufs) {
        r.lo[b.role] = (uint64_t)(uintptr_t)b.p;
        r.hi[b.role] = (uint64_t)(uintptr_t)b.p + b.bytes;
    }
    // Test hook: HASHGRID_CHECK_SHRINK_OUT=n records the output buffer n bytes shorter than
    // it is, so that a test can make the checks trip on accesses that still lie inside the
    // caller's buffer.
    if (const char* shrink = std::getenv("HASHGRID_CHECK_SHRINK_OUT")) {
        const uint64_t n = std::strtoull(shrink, nullptr, 10);
        if (r.hi[hg::kChkOut] != ~0ull) r.hi[hg::kChkOut] -= std::min<uint64_t>(n, r.hi[hg::kChkOut] - r.lo[hg::kChkOut]);
    }
    if (cudaMemcpyToSymbolAsync(hg::g_check_ranges, &r, sizeof r, 0, cudaMemcpyHostToDevice, s) != cudaSuccess) {
        cudaGetLastError();
        return fail(HASHGRID_ERR_CUDA, "%s: recording the checked ranges failed", what);
    }
    const int rc = fn();
    if (rc != HASHGRID_OK) return rc;
    unsigned int flags = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&flags, hg::g_check_flags, sizeof flags, 0, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(HASHGRID_ERR_CUDA, "%s: reading the device status failed: %s", what, cudaGetErrorString(e));
    }
    if (flags != 0) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(hg::g_check_flags, &zero, sizeof zero);
        static const char* names[hg::kChkRoles] = {"x", "table", "output", "dL_dout", "dL_dtable", "adam_m", "adam_v"};
        std::string which;
        for (int i = 0; i < hg::kChkRoles; ++i)
            if (flags & (1u << i)) which += std::string(which.empty() ? "" : ", ") + names[i];
        return fail(HASHGRID_ERR_DEVICE_CHECK, "%s: a device range check tripped on %s (the access was skipped)", what,
                    which.c_str());
    }
    return rc;
#else
    (void)s;
    (void)bufs;
    (void)what;
    return fn();
#endif
}

size_t table_bytes(const hashgrid_s* h) {
    return (size_t)h->L * ((size_t)1 << h->log2T) * (size_t)h->F * (h->dtype == HASHGRID_F16 ? 2 : 4);
}

}  // namespace

extern "C" {

int hashgrid_create(int L, int F, int log2T, int N_min, int N_max, int dtype, hashgrid_t* out) {
    if (out == nullptr) return fail(HASHGRID_ERR_ARG, "out handle pointer is NULL");
    *out = nullptr;
    if (L < 1 || L > HASHGRID_MAX_LEVELS)
        return fail(HASHGRID_ERR_ARG, "L = %d outside [1, %d]", L, HASHGRID_MAX_LEVELS);
    if (F != 1 && F != 2 && F != 4 && F != 8)
        return fail(HASHGRID_ERR_ARG, "F = %d not in {1, 2, 4, 8}", F);
    if (log2T < HASHGRID_MIN_LOG2T || log2T > HASHGRID_MAX_LOG2T)
        return fail(HASHGRID_ERR_ARG, "log2T = %d outside [%d, %d]", log2T, HASHGRID_MIN_LOG2T,
                    HASHGRID_MAX_LOG2T);
    if (N_min < 1 || N_max < N_min || N_max > HASHGRID_MAX_RESOLUTION)
        return fail(HASHGRID_ERR_ARG, "resolutions N_min = %d, N_max = %d outside 1 <= N_min <= N_max <= %d",
                    N_min, N_max, HASHGRID_MAX_RESOLUTION);
    if (dtype != HASHGRID_F32 && dtype != HASHGRID_F16)
        return fail(HASHGRID_ERR_ARG, "dtype = %d is neither HASHGRID_F32 nor HASHGRID_F16", dtype);
    if (L == 1 && N_min != N_max)
        return fail(HASHGRID_ERR_ARG, "L = 1 needs N_min == N_max (the growth factor divides by L - 1)");
    hashgrid_s* h = new (std::nothrow) hashgrid_s;
    if (h == nullptr) return fail(HASHGRID_ERR_OOM, "out of host memory");
    std::memset(h, 0, sizeof(*h));
    h->D = 3;
    h->L = L; h->F = F; h->log2T = log2T; h->N_min = N_min; h->N_max = N_max; h->dtype = dtype;
    compute_resolutions(L, N_min, N_max, h->res);
    h->lp.L = L;
    h->lp.T = (uint64_t)1 << log2T;
    h->lp.mask = (uint32_t)(h->lp.T - 1);
    for (int l = 0; l < L; ++l) h->lp.scale[l] = (float)h->res[l];
    compute_level_groups(h);
    *out = h;
    return ok();
}

int hashgrid_create_nd(int D, int L, int F, int log2T, int N_min, int N_max, int dtype, hashgrid_t* out) {
    if (out != nullptr) *out = nullptr;
    if (D != 2 && D != 3 && D != 4) return fail(HASHGRID_ERR_ARG, "D = %d is not 2, 3 or 4", D);
    int rc = hashgrid_create(L, F, log2T, N_min, N_max, dtype, out);
    if (rc == HASHGRID_OK) (*out)->D = D;
    return rc;
}

int hashgrid_dims(hashgrid_t h) { return h == nullptr ? 0 : h->D; }

int hashgrid_destroy(hashgrid_t h) {
    delete h;
    return ok();
}

int hashgrid_resolutions(hashgrid_t h, int* res_out) {
    if (int rc = check_handle(h)) return rc;
    if (res_out == nullptr) return fail(HASHGRID_ERR_ARG, "res_out is NULL");
    std::memcpy(res_out, h->res, sizeof(int) * h->L);
    return ok();
}

size_t hashgrid_table_elems(hashgrid_t h) {
    if (h == nullptr) return 0;
    return (size_t)h->L * ((size_t)1 << h->log2T) * (size_t)h->F;
}

int hashgrid_output_width(hashgrid_t h) { return h == nullptr ? 0 : h->L * h->F; }

int hashgrid_set_option(hashgrid_t h, int option, int value) {
    if (int rc = check_handle(h)) return rc;
    switch (option) {
        case HASHGRID_OPT_FORWARD_GATHER:
            if (value < HASHGRID_GATHER_AUTO || value > HASHGRID_GATHER_LANES)
                return fail(HASHGRID_ERR_ARG, "forward gather mode %d is not a HASHGRID_GATHER_* value", value);
            h->forward_gather = value;
            return ok();
        case HASHGRID_OPT_SCHEDULE:
            if (value < HASHGRID_SCHEDULE_AUTO || value > HASHGRID_SCHEDULE_LEVEL_MAJOR)
                return fail(HASHGRID_ERR_ARG, "schedule %d is not a HASHGRID_SCHEDULE_* value", value);
            h->schedule = value;
            return ok();
        case HASHGRID_OPT_BACKWARD_MODE:
            if (value < HASHGRID_BACKWARD_AUTO || value > HASHGRID_BACKWARD_RUN_LANES)
                return fail(HASHGRID_ERR_ARG, "backward mode %d is not a HASHGRID_BACKWARD_* value", value);
            if ((value == HASHGRID_BACKWARD_WARP_DEDUP || value == HASHGRID_BACKWARD_RUN_MERGE ||
                 value == HASHGRID_BACKWARD_WARP_DEDUP_ADAPTIVE || value == HASHGRID_BACKWARD_RUN_LANES) && h->F > 4)
                return fail(HASHGRID_ERR_ARG, "backward mode %d needs F <= 4, F = %d", value, h->F);
            h->backward_mode = value;
            return ok();
    }
    return fail(HASHGRID_ERR_ARG, "unknown option %d", option);
}

int hashgrid_get_option(hashgrid_t h, int option, int* value) {
    if (int rc = check_handle(h)) return rc;
    if (value == nullptr) return fail(HASHGRID_ERR_ARG, "value is NULL");
    switch (option) {
        case HASHGRID_OPT_FORWARD_GATHER: *value = h->forward_gather; return ok();
        case HASHGRID_OPT_BACKWARD_MODE: *value = h->backward_mode; return ok();
        case HASHGRID_OPT_SCHEDULE: *value = h->schedule; return ok();
    }
    return fail(HASHGRID_ERR_ARG, "unknown option %d", option);
}

int hashgrid_params(hashgrid_t h, int* L, int* F, int* log2T, int* N_min, int* N_max, int* dtype) {
    if (int rc = check_handle(h)) return rc;
    if (L) *L = h->L;
    if (F) *F = h->F;
    if (log2T) *log2T = h->log2T;
    if (N_min) *N_min = h->N_min;
    if (N_max) *N_max = h->N_max;
    if (dtype) *dtype = h->dtype;
    return ok();
}

int hashgrid_forward(hashgrid_t h, const float* x, int64_t N, const void* table, float* out,
                     void* cuda_stream) {
    if (int rc = check_handle(h)) return rc;
    if (int rc = check_N(N, kTile)) return rc;
    if (N == 0) return ok();
    const size_t W = (size_t)h->L * h->F;
    if (int rc = check_buffer(x, (size_t)N * h->D * sizeof(float), "x")) return rc;
    if (int rc = check_buffer(table, table_bytes(h), "table")) return rc;
    if (int rc = check_buffer(out, (size_t)N * W * sizeof(float), "out")) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    return run_checked(s, {{hg::kChkX, x, (size_t)N * h->D * sizeof(float)}, {hg::kChkTable, table, table_bytes(h)},
                           {hg::kChkOut, out, (size_t)N * W * sizeof(float)}},
                       "forward", [&]() -> int {
    const bool half = h->dtype == HASHGRID_F16;
    if (h->D != 3)
        return nd_dispatch(h, [&](auto d, auto f) {
            return half ? launch_nd_forward<decltype(d)::value, decltype(f)::value, __half>(h, x, N, table, out, s)
                        : launch_nd_forward<decltype(d)::value, decltype(f)::value, float>(h, x, N, table, out, s);
        });
    // Sector gathers issue 256-bit loads, which need a 32-byte-aligned table.
    const bool aligned32 = reinterpret_cast<uintptr_t>(table) % 32 == 0;
    if (h->forward_gather == HASHGRID_GATHER_SECTOR && !aligned32)
        return fail(HASHGRID_ERR_ALIGN, "sector gathers need a 32-byte-aligned table (%p)", table);
    const int sector = forward_gather_kernel(h);
    if (level_major(h)) {
        const int lg = sector == hg::kGatherLanes ? hg::kGatherLanes : hg::kGatherCorner;
        switch (h->F) {
            case 1: return half ? launch_forward_levels<1, __half>(h, x, N, table, out, lg, s) : launch_forward_levels<1, float>(h, x, N, table, out, lg, s);
            case 2: return half ? launch_forward_levels<2, __half>(h, x, N, table, out, lg, s) : launch_forward_levels<2, float>(h, x, N, table, out, lg, s);
            case 4: return half ? launch_forward_levels<4, __half>(h, x, N, table, out, lg, s) : launch_forward_levels<4, float>(h, x, N, table, out, lg, s);
            case 8: return half ? launch_forward_levels<8, __half>(h, x, N, table, out, lg, s) : launch_forward_levels<8, float>(h, x, N, table, out, lg, s);
        }
    }
    switch (h->F) {
        case 1: return half ? launch_forward<1, __half>(h, x, N, table, out, sector, s) : launch_forward<1, float>(h, x, N, table, out, sector, s);
        case 2: return half ? launch_forward<2, __half>(h, x, N, table, out, sector, s) : launch_forward<2, float>(h, x, N, table, out, sector, s);
        case 4: return half ? launch_forward<4, __half>(h, x, N, table, out, sector, s) : launch_forward<4, float>(h, x, N, table, out, sector, s);
        case 8: return half ? launch_forward<8, __half>(h, x, N, table, out, sector, s) : launch_forward<8, float>(h, x, N, table, out, sector, s);
    }
    return fail(HASHGRID_ERR_ARG, "corrupt handle");
    });
}

int hashgrid_backward(hashgrid_t h, const float* x, const float* dL_dout, int64_t N, float* dL_dtable,
                      void* cuda_stream) {
    if (int rc = check_handle(h)) return rc;
    if (int rc = check_N(N, kTile)) return rc;
    if (N == 0) return ok();
    const size_t W = (size_t)h->L * h->F;
    if (int rc = check_buffer(x, (size_t)N * h->D * sizeof(float), "x")) return rc;
    if (int rc = check_buffer(dL_dout, (size_t)N * W * sizeof(float), "dL_dout")) return rc;
    if (int rc = check_buffer(dL_dtable, hashgrid_table_elems(h) * sizeof(float), "dL_dtable")) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    return run_checked(s, {{hg::kChkX, x, (size_t)N * h->D * sizeof(float)}, {hg::kChkDout, dL_dout, (size_t)N * W * sizeof(float)},
                           {hg::kChkGrad, dL_dtable, hashgrid_table_elems(h) * sizeof(float)}},
                       "backward", [&]() -> int {
    if (h->D != 3)
        return nd_dispatch(h, [&](auto d, auto f) {
            return launch_nd_backward<decltype(d)::value, decltype(f)::value, float>(h, x, dL_dout, N, dL_dtable, s);
        });
    switch (h->F) {
        case 1: return launch_backward<1>(h, x, dL_dout, N, dL_dtable, s);
        case 2: return launch_backward<2>(h, x, dL_dout, N, dL_dtable, s);
        case 4: return launch_backward<4>(h, x, dL_dout, N, dL_dtable, s);
        case 8: return launch_backward<8>(h, x, dL_dout, N, dL_dtable, s);
    }
    return fail(HASHGRID_ERR_ARG, "corrupt handle");
    });
}

int hashgrid_backward_half(hashgrid_t h, const float* x, const float* dL_dout, int64_t N, void* dL_dtable,
                           void* cuda_stream) {
    if (int rc = check_handle(h)) return rc;
    if (int rc = check_N(N, kTile)) return rc;
    if (N == 0) return ok();
    const size_t W = (size_t)h->L * h->F;
    if (int rc = check_buffer(x, (size_t)N * h->D * sizeof(float), "x")) return rc;
    if (int rc = check_buffer(dL_dout, (size_t)N * W * sizeof(float), "dL_dout")) return rc;
    if (int rc = check_buffer(dL_dtable, hashgrid_table_elems(h) * 2, "dL_dtable")) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    __half* d = static_cast<__half*>(dL_dtable);
    return run_checked(s, {{hg::kChkX, x, (size_t)N * h->D * sizeof(float)}, {hg::kChkDout, dL_dout, (size_t)N * W * sizeof(float)},
                           {hg::kChkGrad, dL_dtable, hashgrid_table_elems(h) * 2}},
                       "backward_half", [&]() -> int {
    if (h->D != 3)
        return nd_dispatch(h, [&](auto dd, auto f) {
            return launch_nd_backward<decltype(dd)::value, decltype(f)::value, __half>(h, x, dL_dout, N, d, s);
        });
    switch (h->F) {
        case 1: return launch_backward_half<1>(h, x, dL_dout, N, d, s);
        case 2: return launch_backward_half<2>(h, x, dL_dout, N, d, s);
        case 4: return launch_backward_half<4>(h, x, dL_dout, N, d, s);
        case 8: return launch_backward_half<8>(h, x, dL_dout, N, d, s);
    }
    return fail(HASHGRID_ERR_ARG, "corrupt handle");
    });
}

int hashgrid_backward_input(hashgrid_t h, const float* x, const float* dL_dout, int64_t N, const void* table,
                            float* dL_dx, void* cuda_stream) {
    if (int rc = check_handle(h)) return rc;
    if (int rc = check_N(N, kTile)) return rc;
    if (N == 0) return ok();
    const size_t W = (size_t)h->L * h->F;
    if (int rc = check_buffer(x, (size_t)N * h->D * sizeof(float), "x")) return rc;
    if (int rc = check_buffer(dL_dout, (size_t)N * W * sizeof(float), "dL_dout")) return rc;
    if (int rc = check_buffer(table, table_bytes(h), "table")) return rc;
    if (int rc = check_buffer(dL_dx, (size_t)N * h->D * sizeof(float), "dL_dx")) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    return run_checked(s, {{hg::kChkX, x, (size_t)N * h->D * sizeof(float)}, {hg::kChkDout, dL_dout, (size_t)N * W * sizeof(float)},
                           {hg::kChkTable, table, table_bytes(h)}, {hg::kChkOut, dL_dx, (size_t)N * h->D * sizeof(float)}},
                       "backward_input", [&]() -> int {
    const bool half = h->dtype == HASHGRID_F16;
    if (h->D != 3)
        return nd_dispatch(h, [&](auto d, auto f) {
            constexpr int DD = decltype(d)::value, FF = decltype(f)::value;
            return half ? launch_nd_backward_input<DD, FF, __half>(h, x, dL_dout, N, table, dL_dx, s)
                        : launch_nd_backward_input<DD, FF, float>(h, x, dL_dout, N, table, dL_dx, s);
        });
    switch (h->F) {
        case 1: return half ? launch_backward_input<1, __half>(h, x, dL_dout, N, table, dL_dx, s) : launch_backward_input<1, float>(h, x, dL_dout, N, table, dL_dx, s);
        case 2: return half ? launch_backward_input<2, __half>(h, x, dL_dout, N, table, dL_dx, s) : launch_backward_input<2, float>(h, x, dL_dout, N, table, dL_dx, s);
        case 4: return half ? launch_backward_input<4, __half>(h, x, dL_dout, N, table, dL_dx, s) : launch_backward_input<4, float>(h, x, dL_dout, N, table, dL_dx, s);
        case 8: return half ? launch_backward_input<8, __half>(h, x, dL_dout, N, table, dL_dx, s) : launch_backward_input<8, float>(h, x, dL_dout, N, table, dL_dx, s);
    }
    return fail(HASHGRID_ERR_ARG, "corrupt handle");
    });
}

int hashgrid_adam_step(hashgrid_t h, void* table, float* adam_m, float* adam_v, float* dL_dtable, int64_t step,
                       float lr, float beta1, float beta2, float eps, int zero_grad, void* cuda_stream) {
    if (int rc = check_handle(h)) return rc;
    if (step < 1) return fail(HASHGRID_ERR_ARG, "step = %lld must be >= 1", (long long)step);
    if (!(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f))
        return fail(HASHGRID_ERR_ARG, "betas (%g, %g) must lie in [0, 1)", beta1, beta2);
    if (!(eps > 0.f) || !std::isfinite(eps) || !std::isfinite(lr))
        return fail(HASHGRID_ERR_ARG, "lr = %g and eps = %g must be finite, eps > 0", lr, eps);
    const size_t n = hashgrid_table_elems(h);
    if (int rc = check_buffer(table, table_bytes(h), "table")) return rc;
    if (int rc = check_buffer(adam_m, n * sizeof(float), "adam_m")) return rc;
    if (int rc = check_buffer(adam_v, n * sizeof(float), "adam_v")) return rc;
    if (int rc = check_buffer(dL_dtable, n * sizeof(float), "dL_dtable")) return rc;
    hg::AdamParams a;
    a.lr = lr;
    a.b1 = beta1;
    a.b2 = beta2;
    a.eps = eps;
    a.c1 = (float)(1.0 / (1.0 - std::pow((double)beta1, (double)step)));
    a.c2 = (float)(1.0 / (1.0 - std::pow((double)beta2, (double)step)));
    const int64_t n4 = (int64_t)(n / 4);  // L*T*F is a multiple of 16
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (n4 + 255) / 256;
    const unsigned blocks = (unsigned)(want < (int64_t)sms * 16 ? want : (int64_t)sms * 16);
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    return run_checked(s, {{hg::kChkTable, table, table_bytes(h)}, {hg::kChkM, adam_m, n * sizeof(float)},
                           {hg::kChkV, adam_v, n * sizeof(float)}, {hg::kChkGrad, dL_dtable, n * sizeof(float)}},
                       "adam_step", [&]() -> int {
        if (h->dtype == HASHGRID_F16)
            hg::adam_kernel<__half><<<blocks, 256, 0, s>>>(static_cast<__half*>(table), adam_m, adam_v, dL_dtable, n4, a, zero_grad);
        else
            hg::adam_kernel<float><<<blocks, 256, 0, s>>>(static_cast<float*>(table), adam_m, adam_v, dL_dtable, n4, a, zero_grad);
        return launch_status("adam_step");
    });
}

int hashgrid_mlp_forward(hashgrid_t h, const float* x, int64_t N, const void* table, const void* w1,
                         const float* b1, const void* w2, const float* b2, const void* w3, const float* b3, float* y,
                         int* device_status, void* cuda_stream) {
    if (int rc = check_handle(h)) return rc;
    if (h->D != 3) return fail(HASHGRID_ERR_ARG, "the MLP takes 3-D points, the handle has D = %d", h->D);
    const int K1 = h->L * h->F;
    if (K1 % 16 != 0 || K1 > 64)
        return fail(HASHGRID_ERR_ARG, "the MLP needs L*F in {16, 32, 48, 64}, got %d", K1);
    if (int rc = check_N(N, hg::mlp::kM)) return rc;
    if (N == 0) return ok();
    using namespace hg::mlp;
    if (int rc = check_buffer(x, (size_t)N * h->D * sizeof(float), "x")) return rc;
    if (int rc = check_buffer(table, table_bytes(h), "table")) return rc;
    if (int rc = check_buffer(w1, (size_t)kHid * K1 * 2, "w1")) return rc;
    if (int rc = check_buffer(b1, kHid * sizeof(float), "b1")) return rc;
    if (int rc = check_buffer(w2, (size_t)kHid * kHid * 2, "w2")) return rc;
    if (int rc = check_buffer(b2, kHid * sizeof(float), "b2")) return rc;
    if (int rc = check_buffer(w3, (size_t)kOut * kHid * 2, "w3")) return rc;
    if (int rc = check_buffer(b3, kOut * sizeof(float), "b3")) return rc;
    if (int rc = check_buffer(y, (size_t)N * kOut * sizeof(float), "y")) return rc;
    if (device_status != nullptr)
        if (int rc = check_buffer(device_status, sizeof(int), "device_status")) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    return run_checked(s, {{hg::kChkX, x, (size_t)N * h->D * sizeof(float)}, {hg::kChkTable, table, table_bytes(h)},
                           {hg::kChkOut, y, (size_t)N * kOut * sizeof(float)}},
                       "mlp_forward", [&]() -> int {
    const bool half = h->dtype == HASHGRID_F16;
    switch (h->F) {
        case 1: return half ? dispatch_mlp_forward<1, __half>(h, x, N, table, w1, b1, w2, b2, w3, b3, y, device_status, s)
                            : dispatch_mlp_forward<1, float>(h, x, N, table, w1, b1, w2, b2, w3, b3, y, device_status, s);
        case 2: return half ? dispatch_mlp_forward<2, __half>(h, x, N, table, w1, b1, w2, b2, w3, b3, y, device_status, s)
                            : dispatch_mlp_forward<2, float>(h, x, N, table, w1, b1, w2, b2, w3, b3, y, device_status, s);
        case 4: return half ? dispatch_mlp_forward<4, __half>(h, x, N, table, w1, b1, w2, b2, w3, b3, y, device_status, s)
                            : dispatch_mlp_forward<4, float>(h, x, N, table, w1, b1, w2, b2, w3, b3, y, device_status, s);
        case 8: return half ? dispatch_mlp_forward<8, __half>(h, x, N, table, w1, b1, w2, b2, w3, b3, y, device_status, s)
                            : dispatch_mlp_forward<8, float>(h, x, N, table, w1, b1, w2, b2, w3, b3, y, device_status, s);
    }
    return fail(HASHGRID_ERR_ARG, "corrupt handle");
    });
}

int hashgrid_debug_indices(hashgrid_t h, const float* x, int64_t N, uint32_t* idx_out, void* cuda_stream) {
    if (int rc = check_handle(h)) return rc;
    if (int rc = check_N(N, 1)) return rc;
    if (N == 0) return ok();
    if (int rc = check_buffer(x, (size_t)N * h->D * sizeof(float), "x")) return rc;
    if (int rc = check_buffer(idx_out, (size_t)N * h->L * ((size_t)1 << h->D) * sizeof(uint32_t), "idx_out")) return rc;
    const int64_t total = N * h->L;
    const int threads = 256;
    const int64_t blocks = (total + threads - 1) / threads;
    if (blocks > 0x7fffffffLL) return fail(HASHGRID_ERR_ARG, "N too large for the index export");
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    return run_checked(s, {{hg::kChkX, x, (size_t)N * h->D * sizeof(float)},
                           {hg::kChkOut, idx_out, (size_t)N * h->L * ((size_t)1 << h->D) * sizeof(uint32_t)}},
                       "debug_indices", [&]() -> int {
        if (h->D == 2)
            hg::nd::indices_kernel<2><<<(unsigned)blocks, threads, 0, s>>>(h->lp, x, N, idx_out);
        else if (h->D == 4)
            hg::nd::indices_kernel<4><<<(unsigned)blocks, threads, 0, s>>>(h->lp, x, N, idx_out);
        else
            hg::indices_kernel<<<(unsigned)blocks, threads, 0, s>>>(h->lp, x, N, idx_out);
        return launch_status("debug_indices");
    });
}

int hashgrid_probe(int kind, int width, int pattern, void* buf, size_t buf_bytes, int64_t ops, float* sink,
                   int64_t* ops_done, void* cuda_stream) {
    if (kind != HASHGRID_PROBE_GATHER && kind != HASHGRID_PROBE_RED && kind != HASHGRID_PROBE_RED_F16)
        return fail(HASHGRID_ERR_ARG, "probe kind %d is not a HASHGRID_PROBE_* kind", kind);
    const bool red = kind != HASHGRID_PROBE_GATHER;
    if (!(width == 4 || width == 8 || width == 16 || (width == 32 && !red)))
        return fail(HASHGRID_ERR_ARG, "probe width %d not supported by this kind", width);
    if (pattern < HASHGRID_PROBE_RANDOM || pattern > HASHGRID_PROBE_STREAM)
        return fail(HASHGRID_ERR_ARG, "probe pattern %d is not a HASHGRID_PROBE_* pattern", pattern);
    if ((pattern == HASHGRID_PROBE_SECTOR_PAIR || pattern == HASHGRID_PROBE_LINE_PAIR) && width != 16)
        return fail(HASHGRID_ERR_ARG, "the sector- and line-pair patterns take 16-byte units");
    if (buf_bytes < 256 || (buf_bytes & (buf_bytes - 1)) != 0 || buf_bytes / width > ((size_t)1 << 32))
        return fail(HASHGRID_ERR_ARG, "probe buffer of %zu bytes: need a power of two from 256 to 2^32 units",
                    buf_bytes);
    if (ops < 1) return fail(HASHGRID_ERR_ARG, "ops = %lld must be >= 1", (long long)ops);
    if (int rc = check_buffer(buf, buf_bytes, "buf")) return rc;
    if (width == 32 && reinterpret_cast<uintptr_t>(buf) % 32 != 0)
        return fail(HASHGRID_ERR_ALIGN, "32-byte gathers need a 32-byte-aligned buffer (%p)", buf);
    if (!red)
        if (int rc = check_buffer(sink, sizeof(float), "sink")) return rc;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t blocks = (int64_t)sms * 8;
    const int64_t per_iter = blocks * hg::probe::kThreads * hg::probe::kOpsPerIter;
    const int64_t iters = (ops + per_iter - 1) / per_iter;
    if (iters > 0x7fffffffLL) return fail(HASHGRID_ERR_ARG, "ops = %lld is too many", (long long)ops);
    if (ops_done != nullptr) *ops_done = iters * per_iter;
    const uint32_t mask = (uint32_t)(buf_bytes / width - 1);
    char* b = static_cast<char*>(buf);
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    const dim3 grid((unsigned)blocks), block(hg::probe::kThreads);
    const int it = (int)iters;
    const uint32_t seed = 0x2545f491u;
    using namespace hg::probe;
    if (kind == HASHGRID_PROBE_RED) {
        switch (width) {
            case 4: probe_kernel<4, kRedF32><<<grid, block, 0, s>>>(b, mask, pattern, it, seed, sink); break;
            case 8: probe_kernel<8, kRedF32><<<grid, block, 0, s>>>(b, mask, pattern, it, seed, sink); break;
            default: probe_kernel<16, kRedF32><<<grid, block, 0, s>>>(b, mask, pattern, it, seed, sink); break;
        }
    } else if (kind == HASHGRID_PROBE_RED_F16) {
        switch (width) {
            case 4: probe_kernel<4, kRedF16><<<grid, block, 0, s>>>(b, mask, pattern, it, seed, sink); break;
            case 8: probe_kernel<8, kRedF16><<<grid, block, 0, s>>>(b, mask, pattern, it, seed, sink); break;
            default: probe_kernel<16, kRedF16><<<grid, block, 0, s>>>(b, mask, pattern, it, seed, sink); break;
        }
    } else {
        switch (width) {
            case 4: probe_kernel<4, kGather><<<grid, block, 0, s>>>(b, mask, pattern, it, seed, sink); break;
            case 8: probe_kernel<8, kGather><<<grid, block, 0, s>>>(b, mask, pattern, it, seed, sink); break;
            case 16: probe_kernel<16, kGather><<<grid, block, 0, s>>>(b, mask, pattern, it, seed, sink); break;
            default: probe_kernel<32, kGather><<<grid, block, 0, s>>>(b, mask, pattern, it, seed, sink); break;
        }
    }
    return launch_status("probe");
}

const char* hashgrid_last_error(void) { return g_last_error.c_str(); }

const char* hashgrid_version(void) { return HASHGRID_VERSION_STRING; }

}  // extern "C"
