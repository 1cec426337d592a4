/*
 * hashgrid.h -- C ABI of libhashgrid.so: the multiresolution hash-grid encoding
 * (Instant-NGP style) on NVIDIA B200 (sm_100a), forward and backward.
 *
 * Sources, cited by page and section:
 *   [NeRFace-HG]  "NeRFace + Instant-NGP hash encoding" article (ipipp.com, 0929/63223),
 *                 section 2 (二): L levels, each a table of T learnable F-wide features;
 *                 resolution N_l growing geometrically from N_min to N_max; the point's voxel
 *                 and its 8 corners; corner hash with primes (1, 2654435761, 805459861);
 *                 trilinear interpolation; concatenation into an L*F vector. Section 3 (三)
 *                 and the end of section 2: only the sampled features receive gradient.
 *   [Repro-HG]    "Reproduce Instant-NGP's hash-encoding layer in PyTorch" (jsqmd.com,
 *                 news/998204): section 2.1 (level table), 2.2 (XOR-of-primes hash mod T),
 *                 3 (the layer, [B,3] -> [B,L*F]), 5 (half-precision tables; a custom CUDA
 *                 kernel for the hash).
 *   [Overview-HG] Instant-NGP overview (ijyty.com, news/1538821), section 2.2 (the hash
 *                 formula; hash queries run in parallel on the GPU), section 3.1 (irregular
 *                 table accesses are the memory bottleneck; cache hot buckets on chip).
 *
 * Conventions shared by every call:
 *   - All array pointers are DEVICE pointers (cudaMalloc'd, or PyTorch CUDA tensors) on the
 *     device that is current when the call is made, unless a parameter says otherwise.
 *     Pointers must be 16-byte aligned; otherwise the call returns HASHGRID_ERR_ALIGN.
 *     Host memory (pageable, pinned or registered) and pointers that the CUDA runtime does
 *     not report as device memory are rejected with HASHGRID_ERR_ARG before anything is
 *     launched; so is a buffer whose allocation is smaller than the extent the call
 *     touches. Managed (cudaMallocManaged) memory is accepted when the driver reports its
 *     allocation's range.
 *   - Layouts (row-major, element offsets):
 *       x          [N, 3]      fp32, x[p*3 + i]; the encoding's domain is [0,1]^3. Points
 *                               outside are not clamped: the same formula applies (int32
 *                               floor, uint32 hash wraparound). NaN/Inf, or |x*N_l| >= 2^31,
 *                               give unspecified (but in-bounds) results.
 *       table      [L, T, F]   fp32 or fp16 (the handle's dtype), table[(l*T + i)*F + f]
 *       out        [N, L*F]    fp32, out[p*L*F + l*F + f] (level l in columns l*F..l*F+F-1)
 *       dL_dout    [N, L*F]    fp32, same layout as out
 *       dL_dtable  [L, T, F]   fp32 for both table dtypes
 *   - Corner numbering: corner c in 0..7 has offsets (c & 1, (c >> 1) & 1, (c >> 2) & 1)
 *     along (x, y, z).
 *   - Calls are asynchronous on `cuda_stream` (a cudaStream_t; NULL = the legacy default
 *     stream), like a kernel launch. Nothing is synchronised.
 *   - Ownership: the caller owns every array and the stream; the library owns the handle.
 *   - Errors: every call returns a hashgrid_status. Invalid arguments are reported before
 *     any launch and nothing is written. A failed launch returns HASHGRID_ERR_CUDA.
 *     hashgrid_last_error() gives a message for the last failure on the calling thread.
 *   - N = 0 is a valid no-op (returns HASHGRID_OK, pointers may be NULL).
 *   - A handle may be used from several threads and streams at once; set its options before
 *     sharing it (hashgrid_set_option is not synchronised with running calls).
 *   - The compute calls may be captured into CUDA graphs: their host-side checks only query
 *     pointer attributes, and each call is a single kernel launch on cuda_stream.
 */
#ifndef HASHGRID_H
#define HASHGRID_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct hashgrid_s *hashgrid_t; /* opaque, library-owned */

/* Table storage type. fp16 tables are read as IEEE binary16 and converted exactly to fp32
 * (subnormals kept); interpolation and gradients are fp32 ([Repro-HG] section 5). */
enum hashgrid_dtype { HASHGRID_F32 = 0, HASHGRID_F16 = 1 };

enum hashgrid_status {
    HASHGRID_OK = 0,
    HASHGRID_ERR_ARG = 1,          /* invalid argument (shape, range, NULL, host pointer) */
    HASHGRID_ERR_ALIGN = 2,        /* a pointer is not 16-byte aligned */
    HASHGRID_ERR_CUDA = 3,         /* a CUDA runtime call or a launch failed */
    HASHGRID_ERR_OOM = 4,          /* host allocation of the handle failed */
    HASHGRID_ERR_DEVICE_CHECK = 5  /* checked build only: a device-side range check tripped */
};

/* The checked build (libhashgrid_checked.so, compiled with -DHASHGRID_CHECKED) tests every
 * global-memory access of the kernels against the extent of the buffer it belongs to. An
 * access outside it is skipped (a load reads zero) and the call returns
 * HASHGRID_ERR_DEVICE_CHECK, naming the buffers in hashgrid_last_error(). Its calls wait for
 * their kernel, since they read the device status word back. They are meant for one stream
 * at a time, and they return HASHGRID_ERR_ARG, before any work, on a stream that is being
 * captured into a CUDA graph. The regular build (libhashgrid.so) has none of this and never
 * returns HASHGRID_ERR_DEVICE_CHECK. */

/* Parameter limits checked by hashgrid_create. The pages use L = 16 to 32 levels
 * ([Repro-HG] section 5, [Overview-HG] section 2.1) and F = 2 to 4 features. */
#define HASHGRID_MAX_LEVELS 32
#define HASHGRID_MIN_LOG2T 4
#define HASHGRID_MAX_LOG2T 24
#define HASHGRID_MAX_RESOLUTION (1 << 20)

/*
 * hashgrid_create -- build a handle for an encoding of L levels, F features per level,
 * T = 2^log2T entries per level table, resolutions from N_min to N_max, table dtype.
 *
 * [NeRFace-HG] section 2: growth factor b = exp((ln N_max - ln N_min)/(L - 1)) and
 * N_l = floor(N_min * b^l). The floor is taken of the exact-math value: a double result
 * within 1e-9 (relative) of an integer is that integer (so N_{L-1} = N_max even where a
 * literal double computation gives 4095.99999 for 4096); otherwise it is floored. L = 1
 * requires N_min == N_max (b is undefined; N_0 = N_min).
 *
 * Valid ranges: 1 <= L <= 32; F in {1, 2, 4, 8}; 4 <= log2T <= 24;
 * 1 <= N_min <= N_max <= 2^20; dtype in hashgrid_dtype. T is a power of two, so the
 * pages' "mod T" is a mask of the hash's low bits.
 * On success writes a new handle to *out and returns HASHGRID_OK. Does not touch the GPU.
 */
int hashgrid_create(int L, int F, int log2T, int N_min, int N_max, int dtype, hashgrid_t *out);

/*
 * hashgrid_create_nd -- hashgrid_create for D-dimensional points, D in {2, 3, 4}.
 *
 * [Repro-HG] section 2.2 writes the hash for any dimension d as the XOR over axes of
 * coordinate_i * pi_i (mod T) and section 3 lists the primes (1, 2654435761, 805459861,
 * 3674653429, 2097192037, 1434869437, 2165219737); axis i uses the i-th. A point
 * interpolates the 2^D corners of its cell with multilinear weights
 * prod_i (offset_i ? frac_i : 1 - frac_i), corner c having offset bit i = (c >> i) & 1.
 * x is then [N, D] and dL_dx [N, D]; hashgrid_debug_indices writes [N, L, 2^D].
 * D = 3 is hashgrid_create. For D != 3 the forward pass gathers per corner and the backward
 * passes reduce per point, with lane pairs (two threads per point and level, split by x
 * offset) under the LANES gather option (forward, dL/dx) and the RUN_LANES backward option,
 * and under AUTO for D = 4 (for D = 2 one thread per point and level measured faster); the
 * schedule option and the other backward modes apply to D = 3 only, and
 * hashgrid_mlp_forward is not available.
 */
int hashgrid_create_nd(int D, int L, int F, int log2T, int N_min, int N_max, int dtype,
                       hashgrid_t *out);

/* Input dimensions D of a handle (0 for a NULL handle). */
int hashgrid_dims(hashgrid_t h);

/* Free a handle (NULL is allowed). The caller must not destroy a handle while calls that
 * use it are still being issued from other threads; work already launched is unaffected. */
int hashgrid_destroy(hashgrid_t h);

/* Copy the L per-level resolutions N_l into res_out (host array of L ints). */
int hashgrid_resolutions(hashgrid_t h, int *res_out);

/* Handle parameters, for callers that allocate buffers: L*T*F, the number of elements of
 * a table (and of dL_dtable); and L*F, the width of an output row. 0 for a NULL handle. */
size_t hashgrid_table_elems(hashgrid_t h);
int hashgrid_output_width(hashgrid_t h);

/* The create arguments of a handle, written to the non-NULL pointers (host ints). */
int hashgrid_params(hashgrid_t h, int *L, int *F, int *log2T, int *N_min, int *N_max, int *dtype);

/*
 * hashgrid_forward -- encode N points.
 *
 * [NeRFace-HG] section 2, [Repro-HG] section 3: for each point p and level l,
 *   xs = fp32(x * N_l) per axis, v = floor(xs), frac = xs - v;
 *   corner c = v + offsets(c); index_c = hash(corner_c) mod T, with
 *   hash(c) = c0*1 XOR c1*2654435761 XOR c2*805459861 in uint32 wraparound
 *   ([Repro-HG] section 2.2, [Overview-HG] section 2.2);
 *   w_c = prod over axes of (frac_i if offset_i else 1 - frac_i);
 *   out[p][l*F + f] = sum_c w_c * table[l][index_c][f]   (fp32 arithmetic).
 *
 * x: [N,3] fp32; table: [L,T,F] of the handle's dtype; out: [N,L*F] fp32 (overwritten).
 */
int hashgrid_forward(hashgrid_t h, const float *x, int64_t N, const void *table, float *out,
                     void *cuda_stream);

/*
 * hashgrid_backward -- gradient of a loss with respect to the tables.
 *
 * The forward pass is linear in the table, and only the entries a point's corners read
 * receive gradient ([NeRFace-HG] end of section 2 and section 3):
 *   dL_dtable[l][index_c][f] += w_c * dL_dout[p][l*F + f]   for every p, l, c.
 * dL_dtable is ACCUMULATED into (fp32 atomic reductions; the caller zeroes it first when
 * a fresh gradient is wanted). Colliding corners each add their own contribution. The
 * summation order is unspecified, so results vary in the last bits from run to run.
 *
 * x: [N,3] fp32; dL_dout: [N,L*F] fp32; dL_dtable: [L,T,F] fp32 (for both table dtypes).
 */
int hashgrid_backward(hashgrid_t h, const float *x, const float *dL_dout, int64_t N,
                      float *dL_dtable, void *cuda_stream);

/*
 * hashgrid_backward_half -- hashgrid_backward into an fp16 gradient table.
 *
 * The same contributions as hashgrid_backward (computed in fp32, merged in fp32 registers
 * by the run walk), rounded to fp16 and reduced with packed fp16 reductions
 * (red.global.add.noftz f16 / f16x2; round to nearest, subnormals kept): half the gradient
 * memory. Each reduction rounds the running sum to fp16, so the result is accurate to
 * about 2^-11 * sqrt(contributions per entry) relative; values beyond fp16 range overflow
 * to infinity. Backward modes as for hashgrid_backward: ATOMIC = per-point reductions
 * (16-byte units shared by x-neighbours), RUN_MERGE = run walk with 16-byte units, AUTO and
 * RUN_LANES = lane-pair run walk (one F-wide reduction per corner; the default), the other
 * modes = RUN_MERGE; the schedule option applies.
 *
 * x: [N,3] fp32; dL_dout: [N,L*F] fp32; dL_dtable: [L,T,F] fp16 (IEEE binary16),
 * ACCUMULATED into.
 */
int hashgrid_backward_half(hashgrid_t h, const float *x, const float *dL_dout, int64_t N,
                           void *dL_dtable, void *cuda_stream);

/*
 * hashgrid_backward_input -- gradient of a loss with respect to the input coordinates.
 *
 * [NeRFace-HG] section 3 applies the encoder to coordinates produced by a learned
 * transform, which needs dL/dx. Inside the voxel that floor() selects,
 * d frac_i / d x_i = N_l, so
 *   dL_dx[p][i] = sum_l N_l * sum_c (sum_f dL_dout[p][l*F + f] * table[l][index_c][f])
 *                 * (offset_i(c) ? +1 : -1) * prod_{j != i} (offset_j(c) ? frac_j : 1 - frac_j).
 * On a voxel face the encoding has a kink; this is the derivative from the voxel that
 * contains x (the one-sided derivative towards +x). fp32 arithmetic, levels summed in order.
 *
 * x: [N,3] fp32; dL_dout: [N,L*F] fp32; table: [L,T,F] of the handle's dtype;
 * dL_dx: [N,3] fp32, OVERWRITTEN. Always point-major (schedule option ignored); the gather
 * option selects lane pairs (AUTO, LANES) or one thread per (point, level) (any other).
 */
int hashgrid_backward_input(hashgrid_t h, const float *x, const float *dL_dout, int64_t N,
                            const void *table, float *dL_dx, void *cuda_stream);

/*
 * hashgrid_adam_step -- one sparse Adam step on the tables, fused with clearing the
 * consumed gradient.
 *
 * [NeRFace-HG] sections 3 and 4: the tables are trained with Adam, without weight decay,
 * at a learning rate several times the MLP's, and only the sampled entries receive
 * gradient in a step; [Overview-HG] sections 4-5 use Adam with lr 1e-2 .. 1e-3. For every
 * element (L*T*F of them) with a nonzero gradient g, at step t >= 1:
 *   m = beta1 m + (1 - beta1) g;   v = beta2 v + (1 - beta2) g^2;
 *   table -= lr * (m / (1 - beta1^t)) / (sqrt(v / (1 - beta2^t)) + eps);
 * elements whose gradient is exactly zero were not sampled and are left unchanged (table,
 * m and v). fp32 arithmetic with correctly rounded sqrt and division; fp16 tables are
 * updated in fp32 and stored rounded to nearest. If zero_grad != 0 the consumed gradient
 * elements are set to zero, so dL_dtable is all zeros afterwards and the next backward can
 * accumulate into it without a separate clear.
 *
 * table: [L,T,F] of the handle's dtype (updated); adam_m, adam_v: [L,T,F] fp32 moments
 * (updated; zero them before step 1); dL_dtable: [L,T,F] fp32. step >= 1,
 * 0 <= beta1, beta2 < 1, eps > 0, lr finite; otherwise HASHGRID_ERR_ARG.
 */
int hashgrid_adam_step(hashgrid_t h, void *table, float *adam_m, float *adam_v, float *dL_dtable,
                       int64_t step, float lr, float beta1, float beta2, float eps, int zero_grad,
                       void *cuda_stream);

/*
 * hashgrid_mlp_forward -- the encoding fused with the small MLP that consumes it, on the
 * tensor cores.
 *
 * [NeRFace-HG] section 3: a three-layer network of 64 units with ReLU follows the hash
 * features; [Repro-HG] section 4: Linear(in, 64), ReLU, Linear(64, 64), ReLU,
 * Linear(64, 4). With e = the encoding of x (as hashgrid_forward computes it, L*F values):
 *   y = W3 relu(W2 relu(W1 e + b1) + b2) + b3.
 * The encoding stays on chip; each layer runs on the tcgen05 tensor cores over tiles of
 * 128 points with bf16 operands (the encoding and the hidden activations are rounded to
 * bf16) and fp32 accumulation. The pages' extra MLP inputs (an expression code, raw x)
 * are not part of this call.
 *
 * x: [N,3] fp32; table: [L,T,F] of the handle's dtype; w1: [64][L*F], w2: [64][64],
 * w3: [4][64] bf16 (uint16 bit patterns), row-major [out][in] like a torch Linear weight;
 * b1: [64], b2: [64], b3: [4] fp32; y: [N,4] fp32 (overwritten). L*F must be 16, 32, 48
 * or 64 (HASHGRID_ERR_ARG otherwise). device_status: NULL or a device int the caller sets
 * to 0; the kernel sets it to 1 if a bounded wait inside it ran out (on the tensor cores'
 * completion or on the hand-off between its encoding and MMA warps); it then stops early
 * and y is incomplete.
 */
int hashgrid_mlp_forward(hashgrid_t h, const float *x, int64_t N, const void *table, const void *w1,
                         const float *b1, const void *w2, const float *b2, const void *w3,
                         const float *b3, float *y, int *device_status, void *cuda_stream);

/*
 * hashgrid_debug_indices -- export the hash index of every corner: idx_out[(p*L + l)*8 + c]
 * = index_c of point p at level l (uint32, < T), computed by the same device code as the
 * forward and backward passes. For tests and inspection. idx_out: [N, L, 8] uint32.
 */
int hashgrid_debug_indices(hashgrid_t h, const float *x, int64_t N, uint32_t *idx_out,
                           void *cuda_stream);

/* Message describing the last failed call on the calling thread ("" if none). The pointer
 * stays valid until the next call on this thread. */
const char *hashgrid_last_error(void);

/*
 * Execution options of a handle (defaults: AUTO). Options only select among kernels that
 * compute the same result; set them before issuing calls with the handle (they are not
 * synchronised with calls running on other threads).
 *
 * HASHGRID_OPT_FORWARD_GATHER -- how the forward pass reads table entries:
 *   HASHGRID_GATHER_CORNER: one F-wide load per corner;
 *   HASHGRID_GATHER_SECTOR: one 256-bit load of the aligned 32-byte sector holding corner
 *     (v0, y, z), which often also holds corner (v0 + 1, y, z) because the x prime is 1
 *     ([NeRFace-HG] section 2: primes (1, 2654435761, 805459861)); the second corner is
 *     loaded separately only when it is not in that sector. Needs a 32-byte-aligned table
 *     (HASHGRID_ERR_ALIGN otherwise);
 *   HASHGRID_GATHER_PAIR: as SECTOR with 16-byte units: one 128-bit load of the aligned
 *     16-byte unit holding corner (v0, y, z), plus a load of corner (v0 + 1, y, z) when it
 *     is not in that unit (entries wider than 8 bytes load per corner);
 *   HASHGRID_GATHER_LANES: two neighbouring threads per (point, level), thread d gathering
 *     the 4 corners with x offset d, so that each load instruction carries both x-neighbours
 *     of an edge; the two entries usually share a sector and a line (the x prime is 1), and
 *     the L1 fetches a shared sector once for both threads. The pair adds its partial sums;
 *     applies to both schedules;
 *   HASHGRID_GATHER_AUTO: LANES (measured fastest on every workload: per 2^20 ray samples
 *     221 us against 250 us for CORNER, per 2^18 uniform points 78 against 95 us).
 * HASHGRID_OPT_BACKWARD_MODE -- how the backward pass reduces into dL_dtable:
 *   HASHGRID_BACKWARD_ATOMIC: each (point, level) reduces its 8 corner contributions, the
 *     two x-corners merged into one 16-byte reduction when they share an aligned unit;
 *   HASHGRID_BACKWARD_WARP_DEDUP: each warp (32 consecutive points at one level) first sums
 *     its contributions per distinct 16-byte gradient unit in shared memory, then issues one
 *     reduction per unit. Pays off for coherent batches (consecutive samples along rays)
 *     where neighbouring points share corners. Needs F <= 4;
 *   HASHGRID_BACKWARD_RUN_MERGE: each thread walks 8 consecutive points at one level and
 *     keeps the current voxel's corner sums in registers; it reduces a corner into the table
 *     only when the walk leaves it (a step to a face-adjacent voxel keeps the 4 shared
 *     corners). Pays off when consecutive points are close, as for samples ordered along
 *     rays. Needs F <= 4;
 *   HASHGRID_BACKWARD_WARP_DEDUP_ADAPTIVE: per warp and level, WARP_DEDUP when at least
 *     half of the warp's points lie in a voxel adjacent to the previous point's voxel, else
 *     ATOMIC. Needs F <= 4;
 *   HASHGRID_BACKWARD_RUN_LANES: RUN_MERGE with two threads per run, thread d keeping the
 *     sums of the 4 corners with x offset d, each corner reduced on its own (F-wide);
 *     x-neighbouring corners, which usually share a sector (the x prime is 1), are reduced
 *     by the same instruction. Runs are 16 points long under the point-major schedule and
 *     8 under the level-major one. Needs F <= 4. The schedule option applies;
 *   HASHGRID_BACKWARD_AUTO: RUN_LANES for F <= 4 (measured fastest on every workload: per
 *     2^20 ray samples 345 us against 424 us for RUN_MERGE, per 2^22 uniform points 1.74
 *     against 2.10 ms), ATOMIC for F = 8.
 * HASHGRID_OPT_SCHEDULE -- the order in which (point, level) pairs are visited:
 *   HASHGRID_SCHEDULE_POINT_MAJOR: a block handles all levels of a tile of points (best
 *     when the table fits in L2: the x and upstream-gradient rows are read once and the
 *     output rows are written whole);
 *   HASHGRID_SCHEDULE_LEVEL_MAJOR: blocks sweep all points for the first group of levels,
 *     then the next group, ..., so the group's table slices (and gradient slices) stay in
 *     L2 while every point visits them (best for tables much larger than L2). A group is a
 *     run of consecutive levels whose entries reachable from the unit cube,
 *     min(T, (N_l + 2)^3) per level at 4F bytes, fit in 32 MB together: the coarse levels
 *     of a large table share one pass, the fine levels have one pass each; x is read once
 *     per group. The forward pass then gathers with lane pairs (AUTO, LANES) or per corner
 *     (any other gather option), whose kernels take one level per pass; the warp-dedup
 *     backward modes keep their point-major schedule;
 *   HASHGRID_SCHEDULE_AUTO: LEVEL_MAJOR when the table is larger than 96 MB, else
 *     POINT_MAJOR.
 * Returns HASHGRID_ERR_ARG for an unknown option or value.
 */
enum hashgrid_option {
    HASHGRID_OPT_FORWARD_GATHER = 0,
    HASHGRID_OPT_BACKWARD_MODE = 1,
    HASHGRID_OPT_SCHEDULE = 2
};
enum hashgrid_schedule {
    HASHGRID_SCHEDULE_AUTO = 0,
    HASHGRID_SCHEDULE_POINT_MAJOR = 1,
    HASHGRID_SCHEDULE_LEVEL_MAJOR = 2
};
enum hashgrid_gather {
    HASHGRID_GATHER_AUTO = 0,
    HASHGRID_GATHER_CORNER = 1,
    HASHGRID_GATHER_SECTOR = 2,
    HASHGRID_GATHER_PAIR = 3,
    HASHGRID_GATHER_LANES = 4
};
enum hashgrid_backward_mode {
    HASHGRID_BACKWARD_AUTO = 0,
    HASHGRID_BACKWARD_ATOMIC = 1,
    HASHGRID_BACKWARD_WARP_DEDUP = 2,
    HASHGRID_BACKWARD_RUN_MERGE = 3,
    HASHGRID_BACKWARD_WARP_DEDUP_ADAPTIVE = 4,
    HASHGRID_BACKWARD_RUN_LANES = 5
};
int hashgrid_set_option(hashgrid_t h, int option, int value);
int hashgrid_get_option(hashgrid_t h, int option, int *value);

/* Library version string. */
const char *hashgrid_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HASHGRID_H */
