/*
 * hashgrid_probe.h -- measurement entry point of libhashgrid.so: the memory-system rates
 * that the encoding's kernels are held against (their roofline denominators), measured by
 * kernels that issue the encoding's kind of access and nothing else.
 *
 * [Overview-HG] section 3.1 ("Instant-NGP overview", ijyty.com, news/1538821): the cost of
 * the hash-grid encoding is its irregular table accesses. The forward pass gathers one
 * F-wide entry per corner from random slots of a level table; the backward pass adds one
 * F-wide fp32 contribution per corner into random slots of the gradient table. Which
 * memory serves them depends on the table's size: tables that fit in L2 are served by L2,
 * larger ones by HBM. This call measures the rate of such accesses on a buffer of the
 * caller's choosing (a buffer smaller than L2 measures L2; a larger one, HBM), so that a
 * kernel's time can be compared with the time the same number of accesses needs at the
 * device's own rate.
 *
 * Same conventions as hashgrid.h (device pointers on the current device, status codes,
 * hashgrid_last_error, asynchronous on cuda_stream).
 */
#ifndef HASHGRID_PROBE_H
#define HASHGRID_PROBE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* What each operation of the probe does, at one lane (thread). */
enum hashgrid_probe_kind {
    HASHGRID_PROBE_GATHER = 0,  /* one read-only load of `width` bytes (4, 8, 16 or 32) */
    HASHGRID_PROBE_RED = 1,     /* one red.global.add of width/4 fp32 values of 1.0 (width 4, 8 or 16) */
    HASHGRID_PROBE_RED_F16 = 2  /* one red.global.add.noftz of width/2 fp16 values of 1.0, packed in
                                   half pairs (width 4, 8 or 16) */
};

/* Which width-byte unit of the buffer each operation touches. */
enum hashgrid_probe_pattern {
    HASHGRID_PROBE_RANDOM = 0,      /* every lane an independent uniformly random unit */
    HASHGRID_PROBE_XPAIR = 1,       /* lanes 2k, 2k+1: units (v XOR K) and ((v + 1) XOR K) for one
                                       random v and K -- the x-neighbour pattern of the hash */
    HASHGRID_PROBE_SECTOR_PAIR = 2, /* lanes 2k, 2k+1: the two 16-byte halves of one random
                                       32-byte sector (width 16 only) */
    HASHGRID_PROBE_LINE_PAIR = 3,   /* lanes 2k, 2k+1: two different 32-byte sectors of one random
                                       128-byte line (width 16 only) */
    HASHGRID_PROBE_STREAM = 4       /* consecutive lanes take consecutive units (coalesced) */
};

/*
 * hashgrid_probe -- run one probe kernel: about `ops` operations of `kind` with `pattern`
 * on `buf`.
 *
 * buf: device buffer of buf_bytes bytes; buf_bytes a power of two, at least 256. Gathers
 * read it; reductions add 1.0 to fp32 elements of it (its contents change). Every access
 * stays inside [buf, buf + buf_bytes). width 32 needs a 32-byte-aligned buf.
 * ops: requested number of lane operations (>= 1); the kernel runs a persistent grid
 * (8 blocks of 256 threads per SM) in which every thread performs the same number of
 * operations, so the count is rounded up; *ops_done (host int64, may be NULL) receives
 * the count performed.
 * fp16 reductions add to binary16 elements, which count exactly up to 2048.
 * sink: a device float that gathers may write (they do only if the loaded values sum to
 * -3e38, which a buffer of zeros or small values never does); unused by reductions, may be
 * NULL for them.
 * Time the call with CUDA events on cuda_stream; rate = *ops_done / time.
 * Returns HASHGRID_ERR_ARG for an unknown kind or pattern, a width the kind does not
 * support, a pair pattern with another width than 16, or a bad buffer.
 */
int hashgrid_probe(int kind, int width, int pattern, void *buf, size_t buf_bytes, int64_t ops, float *sink,
                   int64_t *ops_done, void *cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* HASHGRID_PROBE_H */
