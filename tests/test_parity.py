"""GPU parity: the CUDA path, called through the C ABI, against the CPU oracle.

Bars (from the method's arithmetic, see the design notes):
  - hash indices: bit-exact;
  - forward: |gpu - ref| <= rtol * sum_c w_c |e_c| + 1e-30 per element, with rtol 1e-6 for
    fp32 tables and 2e-3 for fp16 tables. sum_c w_c |e_c| is the oracle's encoding of the
    absolute-value table; an error bound relative to it stays meaningful when features
    cancel to near zero, where a plain relative error is ill-conditioned;
  - backward: ||g - g_ref||_2 / ||g_ref||_2 <= 1e-5 over the gradient table (fp32 atomics
    accumulate in an unspecified order).
Reduced sizes span many 64-point tiles plus a ragged tail; full sizes run the library's
own launch configuration (the one the benchmark times) and compare sampled rows, level
subsets of the gradient, and the adjoint identity, which holds at any size.
"""
import os
import subprocess
import sys

import numpy as np
import pytest

import oracle
import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

FWD_RTOL = {"f32": 1e-6, "f16": 2e-3}
BWD_REL_L2 = 1e-5
THREADS = oracle.default_threads()


def hgmod():
    import multiresolution_hash_grid_b200 as hg
    return hg


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


# every kernel variant (forward gather mode, backward reduction mode) is held to the same bars
GATHERS = ["corner", "sector", "pair", "lanes"]
BACKWARDS = ["atomic", "auto", "dedup", "runs", "dedup_adaptive", "run_lanes"]


def make_pair(L, F, log2T, N_min, N_max, dtype="f32", gather="auto", backward="auto", schedule="auto"):
    hg = hgmod()
    dt = hg.HASHGRID_F16 if dtype == "f16" else hg.HASHGRID_F32
    gm = {"auto": hg.HASHGRID_GATHER_AUTO, "corner": hg.HASHGRID_GATHER_CORNER,
          "sector": hg.HASHGRID_GATHER_SECTOR, "pair": hg.HASHGRID_GATHER_PAIR,
          "lanes": hg.HASHGRID_GATHER_LANES}[gather]
    bm = {"auto": hg.HASHGRID_BACKWARD_AUTO, "atomic": hg.HASHGRID_BACKWARD_ATOMIC,
          "dedup": hg.HASHGRID_BACKWARD_WARP_DEDUP if F <= 4 else hg.HASHGRID_BACKWARD_ATOMIC,
          "runs": hg.HASHGRID_BACKWARD_RUN_MERGE if F <= 4 else hg.HASHGRID_BACKWARD_ATOMIC,
          "dedup_adaptive": hg.HASHGRID_BACKWARD_WARP_DEDUP_ADAPTIVE if F <= 4 else hg.HASHGRID_BACKWARD_ATOMIC,
          "run_lanes": hg.HASHGRID_BACKWARD_RUN_LANES if F <= 4 else hg.HASHGRID_BACKWARD_ATOMIC}[backward]
    sm = {"auto": hg.HASHGRID_SCHEDULE_AUTO, "point": hg.HASHGRID_SCHEDULE_POINT_MAJOR,
          "level": hg.HASHGRID_SCHEDULE_LEVEL_MAJOR}[schedule]
    return (hg.HashGrid(L, F, log2T, N_min, N_max, dt, forward_gather=gm, backward_mode=bm, schedule=sm),
            oracle.Grid(L, F, log2T, N_min, N_max, oracle.F16 if dtype == "f16" else oracle.F32))


def gpu_forward(grid, x, table):
    out = grid.forward(dev(x), dev(table))
    torch.cuda.synchronize()
    return out.cpu().numpy()


def gpu_backward(grid, x, g):
    d = grid.backward(dev(x), dev(g))
    torch.cuda.synchronize()
    return d.cpu().numpy()


def abs_table(table):
    return np.abs(table)


def check_forward(og, x, table, got, dtype, rows=None):
    ref = og.forward(x, table, nthreads=THREADS)
    bound = og.forward(x, abs_table(table), nthreads=THREADS)
    if rows is not None:
        got = got[rows]
    err = np.abs(got.astype(np.float64) - ref)
    lim = FWD_RTOL[dtype] * bound + 1e-30
    bad = np.argwhere(err > lim)
    assert bad.size == 0, f"{len(bad)} elements off; first {bad[:5].tolist()} err {err[tuple(bad[0])]:.3e} lim {lim[tuple(bad[0])]:.3e}"
    return ref


def rel_l2(got, ref):
    ref = ref.astype(np.float64)
    den = np.linalg.norm(ref.ravel())
    return np.linalg.norm(got.astype(np.float64).ravel() - ref.ravel()) / max(den, 1e-300)


def check_gradient(got, ref, levels=None):
    """Relative L2 error <= 1e-5 over the whole table and over every level's slice on its
    own (so that an error in a fine level cannot hide under the coarse levels' larger
    gradients); levels = (l0, l1) restricts the check to those slices of got and ref."""
    l0, l1 = levels or (0, ref.shape[0])
    assert rel_l2(got[l0:l1], ref[l0:l1]) <= BWD_REL_L2
    for l in range(l0, l1):
        if np.any(ref[l] != 0):
            assert rel_l2(got[l], ref[l]) <= BWD_REL_L2, l


# ---------------------------------------------------------------------------------------
# The five workloads at reduced sizes (several tiles + a ragged tail)
# ---------------------------------------------------------------------------------------

REDUCED_N = 4096 + 37


@pytest.fixture(scope="module")
def reduced_inputs():
    cache = {}

    def get(name):
        if name not in cache:
            w = workloads.WORKLOADS[name]
            n = w.n_points if w.n_points <= 4096 else REDUCED_N
            cache[name] = (w, workloads.make_inputs(w, seed=0, n_points=n, grads=True))
        return cache[name]
    return get


@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_indices_bit_exact(name, reduced_inputs):
    w, inp = reduced_inputs(name)
    grid, og = make_pair(w.L, w.F, w.log2T, w.N_min, w.N_max, w.dtype)
    got = grid.indices(dev(inp.x)).cpu().numpy().view(np.uint32)
    want = og.indices(inp.x)
    np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("gather", GATHERS + ["level", "lanes/level"])
@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_forward_parity(name, gather, reduced_inputs):
    w, inp = reduced_inputs(name)
    if gather == "level":
        grid, og = make_pair(w.L, w.F, w.log2T, w.N_min, w.N_max, w.dtype, schedule="level")
    elif gather == "lanes/level":
        grid, og = make_pair(w.L, w.F, w.log2T, w.N_min, w.N_max, w.dtype, gather="lanes", schedule="level")
    else:
        grid, og = make_pair(w.L, w.F, w.log2T, w.N_min, w.N_max, w.dtype, gather=gather, schedule="point")
    got = gpu_forward(grid, inp.x, inp.table)
    check_forward(og, inp.x, inp.table, got, w.dtype)


@pytest.mark.parametrize("mode", BACKWARDS + ["runs/level", "atomic/level", "run_lanes/level"])
@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_backward_parity(name, mode, reduced_inputs):
    w, inp = reduced_inputs(name)
    bm, _, sched = mode.partition("/")
    grid, og = make_pair(w.L, w.F, w.log2T, w.N_min, w.N_max, w.dtype, backward=bm, schedule=sched or "point")
    got = gpu_backward(grid, inp.x, inp.g)
    ref = og.backward(inp.x, inp.g, nthreads=THREADS)
    check_gradient(got, ref)
    # untouched entries stay exactly zero; touched ones are nonzero on both sides
    np.testing.assert_array_equal(got == 0, ref == 0)


# ---------------------------------------------------------------------------------------
# Full sizes, in the launch configuration the benchmark times
# ---------------------------------------------------------------------------------------

FULL_LEVELS = {   # gradient levels the oracle recomputes at full size: all of them, in groups
    "tiny_L4F2T10": [(0, 4)],
    "rays_L16F2T19": [(0, 16)],
    "half_L16F2T19": [(0, 16)],
    "large_L16F4T22": [(0, 8), (8, 16)],   # one fp64 table (2 GiB) filled half at a time
}


@pytest.mark.parametrize("modes", [("auto", "auto", "auto"), ("corner", "dedup", "point"), ("sector", "runs", "point"),
                                   ("auto", "auto", "level"), ("lanes", "run_lanes", "point"), ("lanes", "run_lanes", "level")])
@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_full_size(name, modes):
    w = workloads.WORKLOADS[name]
    inp = workloads.make_inputs(w, seed=0, grads=True)
    grid, og = make_pair(w.L, w.F, w.log2T, w.N_min, w.N_max, w.dtype, gather=modes[0], backward=modes[1], schedule=modes[2])
    x_d, t_d, g_d = dev(inp.x), dev(inp.table), dev(inp.g)
    out_d = grid.forward(x_d, t_d)
    dt_d = grid.backward(x_d, g_d)
    torch.cuda.synchronize()
    # forward: sampled rows (random, first and last tiles)
    N = inp.x.shape[0]
    rng = np.random.default_rng(99)
    rows = np.unique(np.concatenate([rng.choice(N, 2048, replace=False), np.arange(64), np.arange(N - 64, N)]))
    got_rows = out_d[torch.from_numpy(rows).cuda()].cpu().numpy()
    check_forward(og, inp.x[rows], inp.table, got_rows, w.dtype)
    # adjoint identity <g, fwd(t)> == <bwd(g), t>, computed in fp64 on the device
    tf = t_d.double()
    lhs = float(torch.sum(g_d.double() * out_d.double()))
    rhs = float(torch.sum(dt_d.double() * tf))
    assert abs(lhs - rhs) <= 1e-5 * max(abs(lhs), abs(rhs), 1e-30)
    # gradient: level subsets against the oracle
    if name in FULL_LEVELS:
        got = dt_d.cpu().numpy()
        ref = np.zeros((w.L, w.T, w.F))
        for l0, l1 in FULL_LEVELS[name]:
            ref[l0:l1] = 0.0
            og.backward(inp.x, inp.g, levels=(l0, l1), nthreads=THREADS, dtable=ref)
            check_gradient(got, ref, levels=(l0, l1))
        del ref


# ---------------------------------------------------------------------------------------
# Edge cases
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("modes", [("corner", "atomic", "point"), ("sector", "dedup", "point"), ("auto", "auto", "point"),
                                   ("pair", "runs", "point"), ("auto", "auto", "level"), ("auto", "atomic", "level"),
                                   ("lanes", "run_lanes", "point"), ("lanes", "run_lanes", "level")])
@pytest.mark.parametrize("N", [1, 2, 31, 32, 33, 63, 64, 65, 127, 129, 1000])
def test_ragged_batch_sizes(N, modes):
    grid, og = make_pair(16, 2, 19, 16, 512, gather=modes[0], backward=modes[1], schedule=modes[2])
    rng = np.random.default_rng(N)
    table = workloads.table_values(rng, 16, 2**19, 2)
    x = workloads.uniform_points(rng, N)
    g = workloads.upstream_grads(rng, N, 32)
    check_forward(og, x, table, gpu_forward(grid, x, table), "f32")
    check_gradient(gpu_backward(grid, x, g), og.backward(x, g, nthreads=THREADS))


@pytest.mark.parametrize("modes", [("corner", "atomic", "point"), ("sector", "dedup", "point"), ("auto", "auto", "point"),
                                   ("pair", "runs", "point"), ("auto", "auto", "level"), ("auto", "atomic", "level"),
                                   ("lanes", "run_lanes", "point"), ("lanes", "run_lanes", "level")])
def test_special_coordinates(modes):
    """x = 0, the largest fp32 below 1, exactly 1 (voxel N_l, corner N_l + 1), points
    outside the cube (no clamping), and grid vertices (bit-exact table entries)."""
    grid, og = make_pair(4, 2, 10, 2, 16, gather=modes[0], backward=modes[1], schedule=modes[2])
    rng = np.random.default_rng(5)
    table = rng.standard_normal((4, 1024, 2)).astype(np.float32)
    vals = np.array([0.0, 1.0 - 2**-24, 1.0, 0.5, 0.25, -0.3, 1.7, -2.0, 3.25], dtype=np.float32)
    x = np.stack(np.meshgrid(vals, vals, vals, indexing="ij"), -1).reshape(-1, 3).astype(np.float32)
    got = gpu_forward(grid, x, table)
    check_forward(og, x, table, got, "f32")
    np.testing.assert_array_equal(grid.indices(dev(x)).cpu().numpy().view(np.uint32), og.indices(x))
    # vertices: x = k/2 lands on a vertex at every level of the 2->16 grid
    k = rng.integers(0, 3, size=(200, 3))
    xv = (k / 2.0).astype(np.float32)
    np.testing.assert_array_equal(gpu_forward(grid, xv, table), og.forward(xv, table).astype(np.float32))
    g = rng.standard_normal((x.shape[0], 8)).astype(np.float32)
    check_gradient(gpu_backward(grid, x, g), og.backward(x, g))


@pytest.mark.parametrize("modes", [("corner", "atomic", "point"), ("sector", "dedup", "point"), ("auto", "auto", "point"),
                                   ("pair", "runs", "point"), ("auto", "auto", "level"), ("auto", "atomic", "level"),
                                   ("lanes", "run_lanes", "point"), ("lanes", "run_lanes", "level")])
@pytest.mark.parametrize("F", [1, 2, 4, 8])
@pytest.mark.parametrize("dtype", ["f32", "f16"])
def test_feature_widths_and_dtypes(F, dtype, modes):
    grid, og = make_pair(5, F, 12, 3, 200, dtype, gather=modes[0], backward=modes[1], schedule=modes[2])
    rng = np.random.default_rng(F)
    table = workloads.table_values(rng, 5, 2**12, F, dtype)
    x = workloads.uniform_points(rng, 3000)
    g = workloads.upstream_grads(rng, 3000, 5 * F)
    check_forward(og, x, table, gpu_forward(grid, x, table), dtype)
    check_gradient(gpu_backward(grid, x, g), og.backward(x, g, nthreads=THREADS))


@pytest.mark.parametrize("shape", [
    (1, 2, 10, 64, 64),          # L = 1, N_min == N_max
    (32, 2, 14, 16, 2**20),      # most levels, largest resolution
    (3, 2, 4, 4, 64),            # T = 16: corners of one point collide
    (2, 1, 24, 512, 2**16),      # largest table
    (32, 8, 8, 2, 300),          # widest output row (256 floats, > 48 KB of shared memory)
])
@pytest.mark.parametrize("modes", [("corner", "atomic", "point"), ("sector", "dedup", "point"), ("auto", "auto", "point"),
                                   ("pair", "runs", "point"), ("auto", "auto", "level"), ("auto", "atomic", "level"),
                                   ("lanes", "run_lanes", "point"), ("lanes", "run_lanes", "level")])
def test_extreme_shapes(shape, modes):
    L, F, log2T, a, b = shape
    grid, og = make_pair(L, F, log2T, a, b, gather=modes[0], backward=modes[1], schedule=modes[2])
    rng = np.random.default_rng(L * 100 + F)
    table = workloads.table_values(rng, L, 2**log2T, F)
    x = workloads.uniform_points(rng, 777)
    g = workloads.upstream_grads(rng, 777, L * F)
    np.testing.assert_array_equal(grid.indices(dev(x)).cpu().numpy().view(np.uint32), og.indices(x))
    check_forward(og, x, table, gpu_forward(grid, x, table), "f32")
    check_gradient(gpu_backward(grid, x, g), og.backward(x, g, nthreads=THREADS))


def test_backward_accumulates_and_side_stream():
    grid, og = make_pair(16, 2, 19, 16, 512)
    w = workloads.WORKLOADS["rays_L16F2T19"]
    inp = workloads.make_inputs(w, seed=3, n_points=2000)
    s = torch.cuda.Stream()
    x_d, g_d = dev(inp.x), dev(inp.g)
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        d = torch.zeros((16, 2**19, 2), device="cuda")
        grid.backward(x_d, g_d, d)
        grid.backward(x_d, g_d, d)
        out = grid.forward(x_d, dev(inp.table))
    s.synchronize()
    ref = og.backward(inp.x, inp.g, nthreads=THREADS)
    check_gradient(d.cpu().numpy(), 2 * ref)
    check_forward(og, inp.x, inp.table, out.cpu().numpy(), "f32")


def test_sector_gather_alignment():
    """AUTO falls back to per-corner gathers for a table that is only 16-byte aligned;
    forcing sector gathers on it is an alignment error (no launch)."""
    hg = hgmod()
    grid, og = make_pair(4, 2, 10, 2, 16)
    rng = np.random.default_rng(8)
    table = rng.standard_normal((4, 1024, 2)).astype(np.float32)
    x = rng.random((500, 3), dtype=np.float32)
    buf = torch.zeros(4 * 1024 * 2 + 4, device="cuda")
    t16 = buf[4:]                                     # 16 bytes past a 512-byte boundary
    assert t16.data_ptr() % 32 == 16
    t16.copy_(torch.from_numpy(table.ravel()).cuda())
    out = grid.forward(dev(x), t16)
    torch.cuda.synchronize()
    check_forward(og, x, table, out.cpu().numpy(), "f32")
    hg.hashgrid_set_option(grid.handle, hg.HASHGRID_OPT_FORWARD_GATHER, hg.HASHGRID_GATHER_SECTOR)
    o2 = torch.full((500, 8), 3.0, device="cuda")
    rc = hg.lib.hashgrid_forward(grid.handle, dev(x).data_ptr(), 500, t16.data_ptr(), o2.data_ptr(), None)
    torch.cuda.synchronize()
    assert rc == hg.HASHGRID_ERR_ALIGN and bool(torch.all(o2 == 3.0))


def test_errors_on_device():
    hg = hgmod()
    grid = hg.HashGrid(4, 2, 10, 2, 16)
    x = torch.rand(100, 3, device="cuda")
    t = torch.zeros(4, 1024, 2, device="cuda")
    out = torch.full((100, 8), 7.0, device="cuda")
    L = hg.lib
    # host memory
    xh = np.zeros((100, 3), dtype=np.float32)
    assert L.hashgrid_forward(grid.handle, xh.ctypes.data, 100, t.data_ptr(), out.data_ptr(), None) == hg.HASHGRID_ERR_ARG
    # misaligned device pointer
    assert L.hashgrid_forward(grid.handle, x.data_ptr() + 4, 99, t.data_ptr(), out.data_ptr(), None) == hg.HASHGRID_ERR_ALIGN
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)


def test_allocation_too_small_is_rejected():
    """With torch's caching allocator off every tensor is its own cudaMalloc, so the
    library's allocation-range check must reject a batch larger than x's allocation. The
    case is sized so that, were the check missing, the over-read would stay inside the
    allocation's page (no fault); the assertion on the status would then fail."""
    code = r"""
import torch, numpy as np, multiresolution_hash_grid_b200 as hg
g = hg.HashGrid(4, 2, 10, 2, 16)
x = torch.rand(1000, 3, device="cuda")
t = torch.zeros(4, 1024, 2, device="cuda")
out = torch.full((2000, 8), 7.0, device="cuda")
rc = hg.lib.hashgrid_forward(g.handle, x.data_ptr(), 2000, t.data_ptr(), out.data_ptr(), None)
torch.cuda.synchronize()
assert rc == hg.HASHGRID_ERR_ARG, rc
assert "allocation" in hg.hashgrid_last_error()
assert bool(torch.all(out == 7.0))
print("ok")
"""
    env = dict(os.environ, PYTORCH_NO_CUDA_MEMORY_CACHING="1")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], env=env, cwd=root, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr


def test_host_memory_is_rejected():
    """Pinned host buffers are device-accessible, but the library takes device memory: each
    buffer argument given pinned host memory (correctly sized, or too small for the call)
    is an argument error before any launch, and nothing is written. The undersized case
    stays inside the pinned allocation's rounding, so a missing check could not fault."""
    hg = hgmod()
    g = hg.HashGrid(4, 2, 10, 2, 16)
    x = torch.rand(1000, 3, device="cuda")
    t = torch.zeros(4, 1024, 2, device="cuda")
    out = torch.full((1100, 8), 7.0, device="cuda")
    xh = x.cpu().pin_memory()
    th = t.cpu().pin_memory()
    outh = torch.full((1000, 8), 7.0).pin_memory()
    cases = [(xh, t, out, 1000), (xh, t, out, 1100), (x, th, out, 1000), (x, t, outh, 1000)]
    for xa, ta, oa, n in cases:
        rc = hg.lib.hashgrid_forward(g.handle, xa.data_ptr(), n, ta.data_ptr(), oa.data_ptr(), None)
        assert rc == hg.HASHGRID_ERR_ARG, rc
        assert "host memory" in hg.hashgrid_last_error()
    torch.cuda.synchronize()
    assert bool(torch.all(out == 7.0)) and bool(torch.all(outh == 7.0))


def test_managed_memory_extent_is_checked():
    """Managed memory (cuMemAllocManaged through the driver API): a buffer too small for the
    call is an argument error before any launch (the over-read a missing check would make
    stays inside the allocation's page); a large enough one is either accepted and gives
    the device path's result, or refused because its range cannot be checked."""
    import ctypes
    hg = hgmod()
    try:
        cu = ctypes.CDLL("libcuda.so.1")
    except OSError:
        pytest.skip("no driver library")
    torch.cuda.init()
    torch.zeros(1, device="cuda")           # primary context current on this thread
    ptr = ctypes.c_uint64()
    assert cu.cuMemAllocManaged(ctypes.byref(ptr), ctypes.c_size_t(1000 * 3 * 4), ctypes.c_uint(1)) == 0
    try:
        rng = np.random.default_rng(8)
        xs = workloads.uniform_points(rng, 1000)
        ctypes.memmove(ptr.value, xs.ctypes.data, xs.nbytes)
        g = hg.HashGrid(4, 2, 10, 2, 16)
        t = dev(workloads.table_values(rng, 4, 1024, 2))
        out = torch.full((1100, 8), 7.0, device="cuda")
        # 1020 points read 12240 bytes of the 12000-byte allocation: still inside its 4 KiB page
        rc = hg.lib.hashgrid_forward(g.handle, ptr.value, 1020, t.data_ptr(), out.data_ptr(), None)
        assert rc == hg.HASHGRID_ERR_ARG, rc
        torch.cuda.synchronize()
        assert bool(torch.all(out == 7.0))
        rc = hg.lib.hashgrid_forward(g.handle, ptr.value, 1000, t.data_ptr(), out.data_ptr(), None)
        torch.cuda.synchronize()
        if rc == hg.HASHGRID_OK:
            want = g.forward(dev(xs), t)
            torch.cuda.synchronize()
            assert torch.equal(out[:1000], want)
        else:
            assert rc == hg.HASHGRID_ERR_ARG and "managed" in hg.hashgrid_last_error()
    finally:
        torch.cuda.synchronize()
        cu.cuMemFree_v2(ctypes.c_uint64(ptr.value))


# ---------------------------------------------------------------------------------------
# Gradient with respect to the coordinates
# ---------------------------------------------------------------------------------------

def check_backward_x(og, x, table, g, got):
    """|gpu - ref| <= 1e-5 * B_i, B_i = sum_l N_l * 2 * sum_f |g[l, f]| * max|table|: a bound
    on the sum of absolute values of the terms (the 8 corner weight derivatives along one
    axis have absolute sum 2 * N_l). fp32 products and sums stay within ~30 ulp of it."""
    ref = og.backward_x(x, table, g, nthreads=THREADS)
    tmax = float(np.max(np.abs(np.asarray(table, dtype=np.float64))))
    F = og.F
    B = np.zeros(x.shape[0])
    for l, n in enumerate(og.res):
        B += float(n) * 2.0 * np.sum(np.abs(g[:, l * F:(l + 1) * F].astype(np.float64)), axis=1) * tmax
    err = np.abs(got.astype(np.float64) - ref)
    lim = 1e-5 * B[:, None] + 1e-30
    bad = np.argwhere(err > lim)
    assert bad.size == 0, f"{len(bad)} off; first {bad[:3].tolist()}"


@pytest.mark.parametrize("gather", ["corner", "lanes"])
@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_backward_input_parity(name, gather, reduced_inputs):
    w, inp = reduced_inputs(name)
    grid, og = make_pair(w.L, w.F, w.log2T, w.N_min, w.N_max, w.dtype, gather=gather)
    got = grid.backward_input(dev(inp.x), dev(inp.g), dev(inp.table))
    torch.cuda.synchronize()
    check_backward_x(og, inp.x, inp.table, inp.g, got.cpu().numpy())


@pytest.mark.parametrize("gather", ["corner", "lanes"])
@pytest.mark.parametrize("F", [1, 2, 4, 8])
@pytest.mark.parametrize("dtype", ["f32", "f16"])
def test_backward_input_widths_edges(F, dtype, gather):
    grid, og = make_pair(5, F, 12, 3, 200, dtype, gather=gather)
    rng = np.random.default_rng(40 + F)
    table = workloads.table_values(rng, 5, 2**12, F, dtype)
    vals = np.array([0.0, 1.0 - 2**-24, 1.0, 0.5, -0.3, 1.7], dtype=np.float32)
    xe = np.stack(np.meshgrid(vals, vals, vals, indexing="ij"), -1).reshape(-1, 3)
    x = np.concatenate([workloads.uniform_points(rng, 777), xe]).astype(np.float32)
    g = workloads.upstream_grads(rng, x.shape[0], 5 * F)
    got = grid.backward_input(dev(x), dev(g), dev(table))
    torch.cuda.synchronize()
    check_backward_x(og, x, table, g, got.cpu().numpy())


@pytest.mark.parametrize("gather", ["corner", "lanes"])
@pytest.mark.parametrize("shape", [(32, 2, 12, 4, 4096), (32, 4, 10, 2, 300), (32, 8, 8, 2, 300), (1, 2, 10, 64, 64)])
def test_backward_input_row_widths(shape, gather):
    """Rows of 64 to 256 floats (the lane-pair kernel stages a warp's upstream-gradient rows
    in shared memory, with fewer warps per block above 64 floats) and a single level."""
    L, F, log2T, a, b = shape
    grid, og = make_pair(L, F, log2T, a, b, gather=gather)
    rng = np.random.default_rng(L * 10 + F)
    table = workloads.table_values(rng, L, 2**log2T, F)
    x = workloads.uniform_points(rng, 1000 + 13)
    g = workloads.upstream_grads(rng, x.shape[0], L * F)
    got = grid.backward_input(dev(x), dev(g), dev(table))
    torch.cuda.synchronize()
    check_backward_x(og, x, table, g, got.cpu().numpy())


@pytest.mark.parametrize("gather", ["auto", "corner"])
def test_backward_input_full_size_sampled(gather):
    """2^20 ray samples through the library's launch configuration; sampled rows checked."""
    w = workloads.WORKLOADS["rays_L16F2T19"]
    inp = workloads.make_inputs(w, seed=0)
    grid, og = make_pair(w.L, w.F, w.log2T, w.N_min, w.N_max, gather=gather)
    got = grid.backward_input(dev(inp.x), dev(inp.g), dev(inp.table)).cpu().numpy()
    rows = np.unique(np.concatenate([np.random.default_rng(3).choice(inp.x.shape[0], 3000, replace=False),
                                     np.arange(70), np.arange(inp.x.shape[0] - 70, inp.x.shape[0])]))
    check_backward_x(og, inp.x[rows], inp.table, inp.g[rows], got[rows])


# ---------------------------------------------------------------------------------------
# Sparse Adam
# ---------------------------------------------------------------------------------------

def run_adam_steps(dtype, zero_grad, L, F, log2T, steps, zero_frac, seed):
    """``steps`` sparse Adam steps on the GPU, each compared with the oracle's step from the
    GPU's current state: m and v within 1e-6 of (|old| + |input term|); untouched elements
    bit-identical; the gradient zeroed exactly when asked. The parameter, fp32 tables: the
    rounding error of the fp32 update, propagated from its terms (u = 2^-24): m' carries
    2u (|b1 m| + |(1 - b1) g|), v' 3u (|b2 v| + (1 - b2) g^2), the step lr c1 m' / (sqrt(c2 v')
    + eps) that error through lr c1 / denom plus ~7u of its own size (products, square root,
    division, c1 and c2 rounded to fp32) and half the relative error of v', and the new
    parameter u |theta'| more; the test allows twice that. (A bound relative to |m'| alone
    fails where b1 m and (1 - b1) g nearly cancel.) fp16 tables: one fp16 ulp of theta' plus
    1e-6 of the step."""
    hg = hgmod()
    grid, _ = make_pair(L, F, log2T, 2, 64, dtype)
    rng = np.random.default_rng(seed)
    table = workloads.table_values(rng, L, 2**log2T, F, dtype)
    n = table.size
    t_d = dev(table)
    m_d = torch.zeros(n, device="cuda")
    v_d = torch.zeros(n, device="cuda")
    # the C ABI takes the hyperparameters as fp32: the oracle gets those same values (as
    # exact doubles), not the unrounded decimals (1 - 0.99f differs from 0.01 by 1e-6)
    lr, b1, b2, eps = (float(np.float32(c)) for c in (1e-2, 0.9, 0.99, 1e-15))
    for step in range(1, steps + 1):
        g = rng.standard_normal(n).astype(np.float32)
        g[rng.random(n) < zero_frac] = 0.0
        g[-4:] = rng.standard_normal(4).astype(np.float32)   # the last group is always touched
        g_d = dev(g)
        p_in = t_d.cpu().numpy().astype(np.float64).ravel()
        m_in, v_in = m_d.cpu().numpy().astype(np.float64), v_d.cpu().numpy().astype(np.float64)
        hg.hashgrid_adam_step(grid.handle, t_d, m_d, v_d, g_d, step, lr, b1, b2, eps, zero_grad)
        torch.cuda.synchronize()
        p_ref, m_ref, v_ref = oracle.adam_step(p_in, m_in, v_in, g, step, lr, b1, b2, eps)
        p_got = t_d.cpu().numpy().astype(np.float64).ravel()
        m_got, v_got = m_d.cpu().numpy().astype(np.float64), v_d.cpu().numpy().astype(np.float64)
        touched = g != 0
        np.testing.assert_array_equal(p_got[~touched], p_in[~touched])
        np.testing.assert_array_equal(m_got[~touched], m_in[~touched])
        np.testing.assert_array_equal(v_got[~touched], v_in[~touched])
        gd = g.astype(np.float64)
        assert np.all(np.abs(m_got - m_ref) <= 1e-6 * (np.abs(m_in) + np.abs(gd)) + 1e-30)
        assert np.all(np.abs(v_got - v_ref) <= 1e-6 * (np.abs(v_in) + gd * gd) + 1e-30)
        if dtype == "f32":
            u = 2.0 ** -24
            c1, c2 = 1.0 / (1.0 - b1 ** step), 1.0 / (1.0 - b2 ** step)
            vt = np.where(touched, v_ref, 1.0)
            denom = np.sqrt(vt * c2) + eps
            e_m = 2 * u * (np.abs(b1 * m_in) + np.abs((1 - b1) * gd))
            e_v_rel = 3 * u * (np.abs(b2 * v_in) + (1 - b2) * gd * gd) / vt
            e_step = lr * c1 * e_m / denom + np.abs(p_ref - p_in) * (0.5 * e_v_rel + 7 * u)
            lim = np.where(touched, 2 * (u * np.abs(p_ref) + e_step), 0.0) + 1e-30
        else:
            spacing = np.maximum(np.abs(p_ref), 2.0**-14) * 2.0**-10   # one fp16 ulp (subnormals: 2^-24)
            lim = spacing + 1e-6 * np.abs(p_ref - p_in)
        assert np.all(np.abs(p_got - p_ref) <= lim), float(np.max(np.abs(p_got - p_ref) - lim))
        g_after = g_d.cpu().numpy()
        if zero_grad:
            assert np.all(g_after == 0)
        else:
            np.testing.assert_array_equal(g_after, g)


@pytest.mark.parametrize("dtype", ["f32", "f16"])
@pytest.mark.parametrize("zero_grad", [True, False])
def test_adam_step_parity(dtype, zero_grad):
    """Three steps on a small table with a sparse gradient (70% exact zeros)."""
    run_adam_steps(dtype, zero_grad, 4, 2, 12, 3, 0.7, 50)


@pytest.mark.parametrize("dtype", ["f32", "f16"])
def test_adam_step_parity_large_table(dtype):
    """The default grid's table (16.8 M elements, 4.2 M four-element groups): more groups
    than twice the kernel's grid (148 SMs x 16 blocks x 256 threads), so every thread
    updates groups i and i + stride in each grid-stride step, several steps over, and the
    last group sits in the tail. Every element of parameter, m and v is compared."""
    run_adam_steps(dtype, True, 16, 2, 19, 2, 0.9, 51)


def test_training_step_with_fused_clear():
    """forward -> backward -> Adam (with the fused gradient clear), twice, on the ray
    workload's grid: the second backward accumulates into the gradient the first Adam step
    cleared, and matches the oracle's fresh gradient."""
    hg = hgmod()
    w = workloads.WORKLOADS["rays_L16F2T19"]
    inp = workloads.make_inputs(w, seed=9, n_points=5000)
    grid, og = make_pair(w.L, w.F, w.log2T, w.N_min, w.N_max)
    x_d, t_d, g_d = dev(inp.x), dev(inp.table), dev(inp.g)
    n = inp.table.size
    m_d, v_d = torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda")
    dt = torch.zeros((w.L, w.T, w.F), device="cuda")
    for step in (1, 2):
        grid.forward(x_d, t_d)
        grid.backward(x_d, g_d, dt)
        torch.cuda.synchronize()
        ref = og.backward(inp.x, inp.g, nthreads=THREADS)
        check_gradient(dt.cpu().numpy(), ref)
        hg.hashgrid_adam_step(grid.handle, t_d, m_d, v_d, dt, step, 1e-2)
        torch.cuda.synchronize()
        assert float(dt.abs().max()) == 0.0


# ---------------------------------------------------------------------------------------
# Encoding + MLP on the tensor cores
# ---------------------------------------------------------------------------------------

def bf16_bits(a):
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + ((u >> 16) & 1) + 0x7FFF) >> 16).astype(np.uint16)


def bf16_values(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def mlp_weights(rng, K):
    w1 = bf16_bits(rng.standard_normal((64, K)) * (2.0 / K) ** 0.5)
    w2 = bf16_bits(rng.standard_normal((64, 64)) * (2.0 / 64) ** 0.5)
    w3 = bf16_bits(rng.standard_normal((4, 64)) * (1.0 / 64) ** 0.5)
    b1, b2, b3 = (rng.standard_normal(n).astype(np.float32) * 0.1 for n in (64, 64, 4))
    return w1, b1, w2, b2, w3, b3


def check_mlp(og, x, table, wts, got):
    """|gpu - ref| <= 2 Ey + 1e-6. With u = 2^-8 (twice the bf16 rounding bound) the error
    of each bf16 operand is propagated through |W|: E0 = u|e|,
    E1 = |W1|E0 + u(|W1||e| + |b1|), E2 = |W2|E1 + u(|W2||a1| + |b2|),
    Ey = |W3|E2 + 1e-6(|W3||a2| + |b3|) (fp32 accumulation), on the exact activations."""
    w1, b1, w2, b2, w3, b3 = wts
    ref = og.mlp_forward(x, table, *wts, nthreads=THREADS)
    e = og.forward(x, table, nthreads=THREADS)
    W1, W2, W3 = (np.abs(bf16_values(w)) for w in (w1, w2, w3))
    a1 = np.maximum(e @ bf16_values(w1).T + b1, 0)
    a2 = np.maximum(a1 @ bf16_values(w2).T + b2, 0)
    u = 2.0 ** -8
    E1 = np.abs(e) @ W1.T * u + u * (np.abs(e) @ W1.T + np.abs(b1))
    E2 = E1 @ W2.T + u * (a1 @ W2.T + np.abs(b2))
    Ey = E2 @ W3.T + 1e-6 * (a2 @ W3.T + np.abs(b3))
    err = np.abs(got.astype(np.float64) - ref)
    lim = 2 * Ey + 1e-6
    bad = np.argwhere(err > lim)
    assert bad.size == 0, f"{len(bad)} of {err.size} off; first {bad[:3].tolist()} err {err[tuple(bad[0])]:.3e} lim {lim[tuple(bad[0])]:.3e} ref {ref[tuple(bad[0])]:.3e} got {got[tuple(bad[0])]:.3e}"


@pytest.mark.parametrize("shape", [(16, 2, 19, 16, 512, "f32"), (8, 2, 12, 4, 128, "f32"), (24, 2, 12, 4, 600, "f32"),
                                   (16, 4, 14, 16, 4096, "f32"), (16, 2, 19, 16, 512, "f16"),
                                   (16, 1, 12, 16, 512, "f32"), (32, 1, 10, 8, 1000, "f16"),     # F = 1: two levels per store
                                   (4, 8, 12, 4, 200, "f32"), (8, 8, 12, 4, 300, "f16"),         # F = 8: 512-thread CTAs
                                   (12, 4, 12, 4, 300, "f16")])
@pytest.mark.parametrize("gather", ["auto", "corner"])
def test_mlp_forward_parity(shape, gather):
    """Lane-pair producers (AUTO, F <= 4) and per-corner producers (CORNER, and F = 8)."""
    hg = hgmod()
    L, F, log2T, a, b, dtype = shape
    grid, og = make_pair(L, F, log2T, a, b, dtype, gather=gather)
    rng = np.random.default_rng(70 + L * F)
    table = (rng.standard_normal((L, 2**log2T, F)) * 0.3).astype(np.float32)
    if dtype == "f16":
        table = table.astype(np.float16)
    x = np.concatenate([workloads.ray_points(rng, 40), workloads.uniform_points(rng, 1000)]).astype(np.float32)
    wts = mlp_weights(rng, L * F)
    N = x.shape[0]
    y = torch.full((N, 4), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    hg.hashgrid_mlp_forward(grid.handle, dev(x), N, dev(table), *[dev(w) for w in wts], y, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    check_mlp(og, x, table, wts, y.cpu().numpy())


def test_mlp_forward_full_size_sampled():
    hg = hgmod()
    w = workloads.WORKLOADS["rays_L16F2T19"]
    inp = workloads.make_inputs(w, seed=0, grads=False)
    grid, og = make_pair(w.L, w.F, w.log2T, w.N_min, w.N_max)
    rng = np.random.default_rng(71)
    table = (inp.table * 3000).astype(np.float32)       # features of order 0.3, as after training
    wts = mlp_weights(rng, 32)
    N = inp.x.shape[0]
    y = torch.empty((N, 4), device="cuda")
    hg.hashgrid_mlp_forward(grid.handle, dev(inp.x), N, dev(table), *[dev(w) for w in wts], y)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([rng.choice(N, 3000, replace=False), np.arange(130), np.arange(N - 130, N)]))
    check_mlp(og, inp.x[rows], table, wts, y.cpu().numpy()[rows])


@pytest.mark.parametrize("gather", ["auto", "corner"])
@pytest.mark.parametrize("N", [0, 1, 127, 128, 129, 3 * 2 * 148 * 128 + 77])
def test_mlp_forward_tile_edges(N, gather):
    """Below, at and above one 128-point tile, and enough tiles that every persistent CTA
    cycles both encoding buffers at least once (3+ tiles per CTA): every row against the
    oracle; N = 0 writes nothing. Two calls give bit-identical results (no atomics)."""
    hg = hgmod()
    w = workloads.WORKLOADS["rays_L16F2T19"]
    grid, og = make_pair(w.L, w.F, w.log2T, w.N_min, w.N_max, gather=gather)
    rng = np.random.default_rng(72)
    table = (rng.standard_normal((w.L, w.T, w.F)) * 0.3).astype(np.float32)
    x = workloads.ray_points(rng, (N + 63) // 64)[:N].astype(np.float32).reshape(-1, 3)
    wts = mlp_weights(rng, 32)
    y = torch.full((max(N, 1), 4), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    args = (dev(x) if N else torch.empty((1, 3), device="cuda"), N, dev(table), *[dev(v) for v in wts])
    hg.hashgrid_mlp_forward(grid.handle, *args, y, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    if N == 0:
        assert torch.isnan(y).all()
        return
    first = y.clone()
    hg.hashgrid_mlp_forward(grid.handle, *args, y, status)
    torch.cuda.synchronize()
    assert torch.equal(first, y)
    check_mlp(og, x, table, wts, y.cpu().numpy())


def test_mlp_forward_graph_capture():
    """The fused MLP captured in a CUDA graph and replayed equals the eager call bit for bit."""
    hg = hgmod()
    w = workloads.WORKLOADS["rays_L16F2T19"]
    grid, _ = make_pair(w.L, w.F, w.log2T, w.N_min, w.N_max)
    rng = np.random.default_rng(73)
    table = dev((rng.standard_normal((w.L, w.T, w.F)) * 0.3).astype(np.float32))
    x = dev(workloads.ray_points(rng, 300).astype(np.float32))
    wts = [dev(v) for v in mlp_weights(rng, 32)]
    N = x.shape[0]
    eager = torch.empty((N, 4), device="cuda")
    hg.hashgrid_mlp_forward(grid.handle, x, N, table, *wts, eager)
    y = torch.empty((N, 4), device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        hg.hashgrid_mlp_forward(grid.handle, x, N, table, *wts, y, stream=s.cuda_stream)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    y.fill_(float("nan"))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        hg.hashgrid_mlp_forward(grid.handle, x, N, table, *wts, y, stream=s.cuda_stream)
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(y, eager)


# ---------------------------------------------------------------------------------------
# fp16 gradient tables (packed f16x2 reductions)
# ---------------------------------------------------------------------------------------

def check_half_gradient(og, x, g, got):
    """fp16 accumulation model. Each reduction rounds its operand and the running sum to
    fp16 (unit roundoff 2^-11, subnormal spacing 2^-24). With A_e = sum of |contributions|
    into element e (the oracle's gradient of |g|, weights being >= 0) and n_e the number of
    contributions: |err_e| <= 2^-11 (n_e + 1) A_e + 2^-24 (n_e + 1) (worst case), and per
    level the relative L2 error <= 3 * 2^-11 sqrt(mean n_e) + 2^-11 (rounding errors of a
    running sum add like a random walk)."""
    ref = og.backward(x, g, nthreads=THREADS)
    A = og.backward(x, np.abs(g), nthreads=THREADS)
    idx = og.indices(x)
    got = got.astype(np.float64)
    u = 2.0 ** -11
    for l in range(og.L):
        n = np.bincount(idx[:, l, :].ravel(), minlength=og.T).astype(np.float64)[:, None]
        err = np.abs(got[l] - ref[l])
        lim = u * (n + 1) * A[l] + 2.0 ** -24 * (n + 1)
        assert np.all(err <= lim), (l, float(np.max(err - lim)))
        touched = n[:, 0] > 0
        den = np.linalg.norm(ref[l][touched])
        if den > 0:
            rel = np.linalg.norm((got[l] - ref[l])[touched]) / den
            assert rel <= 3 * u * np.sqrt(np.mean(n[touched])) + u, (l, rel)


@pytest.mark.parametrize("mode", ["auto", "atomic", "runs/level", "atomic/level", "run_lanes", "run_lanes/level"])
@pytest.mark.parametrize("name", ["tiny_L4F2T10", "rays_L16F2T19", "half_L16F2T19"])
def test_backward_half_parity(name, mode, reduced_inputs):
    hg = hgmod()
    w, inp = reduced_inputs(name)
    bm, _, sched = mode.partition("/")
    grid, og = make_pair(w.L, w.F, w.log2T, w.N_min, w.N_max, w.dtype, backward=bm if bm != "auto" else "auto",
                         schedule=sched or "point")
    d = torch.zeros((w.L, w.T, w.F), dtype=torch.float16, device="cuda")
    hg.hashgrid_backward_half(grid.handle, dev(inp.x), dev(inp.g), inp.x.shape[0], d)
    torch.cuda.synchronize()
    check_half_gradient(og, inp.x, inp.g, d.cpu().numpy())


@pytest.mark.parametrize("mode", ["auto", "run_lanes"])
@pytest.mark.parametrize("F", [1, 4, 8])
def test_backward_half_widths(F, mode):
    hg = hgmod()
    grid, og = make_pair(5, F, 12, 3, 200, backward=mode)
    rng = np.random.default_rng(80 + F)
    x = workloads.uniform_points(rng, 2000)
    g = workloads.upstream_grads(rng, 2000, 5 * F)
    d = torch.zeros((5, 2**12, F), dtype=torch.float16, device="cuda")
    hg.hashgrid_backward_half(grid.handle, dev(x), dev(g), 2000, d)
    torch.cuda.synchronize()
    check_half_gradient(og, x, g, d.cpu().numpy())


# ---------------------------------------------------------------------------------------
# D-dimensional inputs
# ---------------------------------------------------------------------------------------

ND_MODES = {"auto": {}, "lanes": {"forward_gather": 4, "backward_mode": 5},           # LANES, RUN_LANES
            "one-lane": {"forward_gather": 1, "backward_mode": 1}}                      # CORNER, ATOMIC


@pytest.mark.parametrize("mode", list(ND_MODES))
@pytest.mark.parametrize("F", [1, 2, 4, 8])
@pytest.mark.parametrize("D", [2, 4])
def test_nd_parity(D, F, mode):
    """Indices bit-exact, forward within 1e-6 of sum_c w_c |e_c| (2^D products of D-1
    fp32 roundings and 2^D fma: ~(D + 2^D) ulp), fp32 and fp16 gradients, and dL/dx, for
    D = 2 and 4 against the oracle's D-dimensional functions; lane-pair kernels (LANES,
    RUN_LANES), one thread per (point, level) (CORNER gathers, ATOMIC reductions) and AUTO."""
    hg = hgmod()
    L, log2T = 6, 12
    opts = dict(ND_MODES[mode])
    if F > 4 and opts.get("backward_mode") == 5:   # RUN_LANES takes F <= 4 (AUTO covers D = 4, F = 8 lanes)
        opts["backward_mode"] = 1
    grid = hg.HashGrid(L, F, log2T, 3, 150, D=D, **opts)
    og = oracle.GridND(D, L, F, log2T, 3, 150)
    rng = np.random.default_rng(100 + 10 * D + F)
    table = workloads.table_values(rng, L, 2**log2T, F)
    x = rng.random((2000 + 37, D), dtype=np.float32)
    x[:4] = np.float32(1.0)
    x[4:8] = -rng.random((4, D), dtype=np.float32)
    g = workloads.upstream_grads(rng, x.shape[0], L * F)
    x_d, t_d, g_d = dev(x), dev(table), dev(g)
    np.testing.assert_array_equal(grid.indices(x_d).cpu().numpy().view(np.uint32), og.indices(x))
    out = grid.forward(x_d, t_d).cpu().numpy().astype(np.float64)
    ref = og.forward(x, table, nthreads=THREADS)
    bound = og.forward(x, np.abs(table), nthreads=THREADS)
    assert np.all(np.abs(out - ref) <= 1e-6 * bound + 1e-30)
    dref = og.backward(x, g, nthreads=THREADS)
    check_gradient(grid.backward(x_d, g_d).cpu().numpy(), dref)
    dh = torch.zeros((L, 2**log2T, F), dtype=torch.float16, device="cuda")
    hg.hashgrid_backward_half(grid.handle, x_d, g_d, x.shape[0], dh)
    torch.cuda.synchronize()
    check_half_gradient(og, x, g, dh.cpu().numpy())
    dx = grid.backward_input(x_d, g_d, t_d).cpu().numpy().astype(np.float64)
    dxref = og.backward_x(x, table, g, nthreads=THREADS)
    tmax = float(np.max(np.abs(table)))
    B = np.zeros(x.shape[0])
    for l, n in enumerate(og.res):
        B += float(n) * 2.0 * np.sum(np.abs(g[:, l * F:(l + 1) * F].astype(np.float64)), axis=1) * tmax
    assert np.all(np.abs(dx - dxref) <= 1e-5 * B[:, None] * 2 ** (D - 3) + 1e-30)


@pytest.mark.parametrize("mode", list(ND_MODES))
@pytest.mark.parametrize("F", [2, 4])
@pytest.mark.parametrize("D", [2, 4])
def test_nd_parity_fp16_table(D, F, mode):
    """fp16 tables with D = 2 and 4: the entries are decoded exactly, so the forward holds
    the fp32 bound (1e-6 of sum_c w_c |e_c|) and dL/dx the same bound as with fp32 tables."""
    hg = hgmod()
    L, log2T = 6, 12
    grid = hg.HashGrid(L, F, log2T, 3, 150, dtype=hg.HASHGRID_F16, D=D, **ND_MODES[mode])
    og = oracle.GridND(D, L, F, log2T, 3, 150, dtype=oracle.F16)
    rng = np.random.default_rng(120 + 10 * D + F)
    table = (rng.standard_normal((L, 2**log2T, F)) * 0.5).astype(np.float16)
    x = rng.random((1500 + 11, D), dtype=np.float32)
    g = workloads.upstream_grads(rng, x.shape[0], L * F)
    x_d, t_d, g_d = dev(x), dev(table), dev(g)
    out = grid.forward(x_d, t_d).cpu().numpy().astype(np.float64)
    ref = og.forward(x, table, nthreads=THREADS)
    bound = og.forward(x, np.abs(table), nthreads=THREADS)
    assert np.all(np.abs(out - ref) <= 1e-6 * bound + 1e-30)
    check_gradient(grid.backward(x_d, g_d).cpu().numpy(), og.backward(x, g, nthreads=THREADS))
    dx = grid.backward_input(x_d, g_d, t_d).cpu().numpy().astype(np.float64)
    dxref = og.backward_x(x, table, g, nthreads=THREADS)
    tmax = float(np.max(np.abs(table.astype(np.float64))))
    B = np.zeros(x.shape[0])
    for l, n in enumerate(og.res):
        B += float(n) * 2.0 * np.sum(np.abs(g[:, l * F:(l + 1) * F].astype(np.float64)), axis=1) * tmax
    assert np.all(np.abs(dx - dxref) <= 1e-5 * B[:, None] * 2 ** (D - 3) + 1e-30)


def test_nd_mlp_rejected():
    hg = hgmod()
    grid = hg.HashGrid(16, 2, 12, 16, 512, D=2)
    z = torch.zeros(64 * 64, device="cuda")
    rc = hg.lib.hashgrid_mlp_forward(grid.handle, z.data_ptr(), 4, z.data_ptr(), z.data_ptr(), z.data_ptr(),
                                     z.data_ptr(), z.data_ptr(), z.data_ptr(), z.data_ptr(), z.data_ptr(), None, None)
    assert rc == hg.HASHGRID_ERR_ARG


# ---------------------------------------------------------------------------------------
# CUDA graph capture
# ---------------------------------------------------------------------------------------

def test_cuda_graph_capture_and_replay():
    """Forward + zero + backward captured in a CUDA graph (torch's default capture mode)
    and replayed: the forward is bit-identical to an eager call, the gradient matches the
    oracle, and replays with new inputs copied into the captured buffers follow them."""
    w = workloads.WORKLOADS["rays_L16F2T19"]
    grid, og = make_pair(w.L, w.F, w.log2T, w.N_min, w.N_max)
    inp = workloads.make_inputs(w, seed=11, n_points=3000)
    x_d, t_d, g_d = dev(inp.x), dev(inp.table), dev(inp.g)
    out = torch.empty((3000, 32), device="cuda")
    d = torch.zeros((w.L, w.T, w.F), device="cuda")
    eager = grid.forward(x_d, t_d).clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):                 # warm-up outside the capture
        grid.forward(x_d, t_d, out)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        d.zero_()
        grid.forward(x_d, t_d, out)
        grid.backward(x_d, g_d, d)
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)
    check_gradient(d.cpu().numpy(), og.backward(inp.x, inp.g, nthreads=THREADS))
    inp2 = workloads.make_inputs(w, seed=12, n_points=3000)
    x_d.copy_(torch.from_numpy(inp2.x))
    g_d.copy_(torch.from_numpy(inp2.g))
    graph.replay()
    torch.cuda.synchronize()
    check_forward(og, inp2.x, inp.table, out.cpu().numpy(), "f32")
    check_gradient(d.cpu().numpy(), og.backward(inp2.x, inp2.g, nthreads=THREADS))


# ---------------------------------------------------------------------------------------
# The README's usage example runs as written
# ---------------------------------------------------------------------------------------

def test_readme_usage_example():
    import os
    import re
    readme = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "README.md")
    block = re.search(r"```python\n(.*?)```", open(readme).read(), re.S).group(1)
    scope = {}
    exec(compile(block, "README.md", "exec"), scope)
    torch.cuda.synchronize()
    assert scope["out"].shape == (1 << 20, 32) and torch.isfinite(scope["out"]).all()
    assert scope["dL_dx"].shape == (1 << 20, 3) and torch.isfinite(scope["y"]).all()
    assert int(torch.count_nonzero(scope["dL_dtable"])) == 0      # the Adam step cleared it
