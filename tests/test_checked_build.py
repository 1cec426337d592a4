"""The checked build (libhashgrid_checked.so, -DHASHGRID_CHECKED): every global-memory access
of the kernels is range-checked against the buffers of its call; an access outside them
is skipped and the call returns HASHGRID_ERR_DEVICE_CHECK. The GPU tests run the small
parity cases under it (no check may trip on valid inputs) and trip a check on purpose by
recording the output buffer shorter than it is (the skipped writes still lie inside the
caller's buffer, so nothing outside any allocation is touched either way)."""
import ctypes
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CHECKED_LIB = os.path.join(ROOT, "multiresolution_hash_grid_b200", "libhashgrid_checked.so")

SMALL_PARITY = ("forward_parity or backward_parity or ragged or special_coordinates or feature_widths or "
                "extreme_shapes or backward_input_parity or backward_input_widths or backward_half or nd_parity or "
                "indices_bit_exact or mlp_forward_parity or mlp_forward_tile_edges or "
                "(adam_step_parity and not large)")


def checked_env(**extra):
    return dict(os.environ, HASHGRID_CHECKED="1", **extra)


def test_checked_library_exports_the_same_calls():
    from tests.test_abi_host import declared_functions
    lib = ctypes.CDLL(CHECKED_LIB)
    assert not [n for n in declared_functions() if not hasattr(lib, n)]
    lib.hashgrid_version.restype = ctypes.c_char_p
    assert b"checked" in lib.hashgrid_version()
    r = subprocess.run([sys.executable, "-c", "import multiresolution_hash_grid_b200 as hg; print(hg.hashgrid_version())"],
                       cwd=ROOT, env=checked_env(), capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and "checked" in r.stdout, r.stderr


@pytest.mark.gpu
@pytest.mark.timeout(1800)
def test_small_parity_cases_pass_under_the_checked_build():
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_parity.py", "-m", "gpu", "-q", "-x", "-p",
                        "no:cacheprovider", "-k", SMALL_PARITY], cwd=ROOT, env=checked_env(), capture_output=True,
                       text=True, timeout=1700)
    tail = r.stdout[-3000:] + r.stderr[-2000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout, tail


TRIP = r"""
import numpy as np, torch, multiresolution_hash_grid_b200 as hg, workloads
assert "checked" in hg.hashgrid_version()
g = hg.HashGrid(4, 2, 10, 2, 16)
rng = np.random.default_rng(3)
x = torch.from_numpy(workloads.uniform_points(rng, 1000)).cuda()
t = torch.from_numpy(workloads.table_values(rng, 4, 1024, 2)).cuda()
want = g.forward(x, t)          # HASHGRID_CHECK_SHRINK_OUT is read per call: 0 for this one
torch.cuda.synchronize()
import os
os.environ["HASHGRID_CHECK_SHRINK_OUT"] = "4096"   # the last 128 rows (32 B each) fall outside
for attempt in range(2):           # the status word is cleared after each report
    out = torch.full((1000, 8), 7.0, device="cuda")
    rc = hg.lib.hashgrid_forward(g.handle, x.data_ptr(), 1000, t.data_ptr(), out.data_ptr(), None)
    torch.cuda.synchronize()
    assert rc == hg.HASHGRID_ERR_DEVICE_CHECK, rc
    assert "output" in hg.hashgrid_last_error(), hg.hashgrid_last_error()
    assert torch.equal(out[:872], want[:872])             # inside the recorded range: written
    assert bool(torch.all(out[872:] == 7.0))              # outside it: skipped
del os.environ["HASHGRID_CHECK_SHRINK_OUT"]
out = g.forward(x, t)
torch.cuda.synchronize()
assert torch.equal(out, want)
print("ok")
"""


@pytest.mark.gpu
def test_a_tripped_check_is_reported_and_the_access_skipped():
    r = subprocess.run([sys.executable, "-c", TRIP], cwd=ROOT, env=checked_env(), capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr


CAPTURE = r"""
import numpy as np, torch, multiresolution_hash_grid_b200 as hg, workloads
assert "checked" in hg.hashgrid_version()
g = hg.HashGrid(4, 2, 10, 2, 16)
rng = np.random.default_rng(4)
x = torch.from_numpy(workloads.uniform_points(rng, 500)).cuda()
t = torch.from_numpy(workloads.table_values(rng, 4, 1024, 2)).cuda()
want = g.forward(x, t)
torch.cuda.synchronize()
out = torch.zeros((500, 8), device="cuda")
s = torch.cuda.Stream()
graph = torch.cuda.CUDAGraph()
codes = []
with torch.cuda.graph(graph, stream=s):
    codes.append(hg.lib.hashgrid_forward(g.handle, x.data_ptr(), 500, t.data_ptr(), out.data_ptr(),
                                         torch.cuda.current_stream().cuda_stream))
assert codes == [hg.HASHGRID_ERR_ARG], codes
assert "stream capture" in hg.hashgrid_last_error(), hg.hashgrid_last_error()
graph.replay()                      # the call issued nothing into the graph
torch.cuda.synchronize()
assert bool(torch.all(out == 0))
assert torch.equal(g.forward(x, t), want)   # eager calls still work
print("ok")
"""


@pytest.mark.gpu
def test_stream_capture_is_refused_before_any_work():
    """The checked build reads its status word back after every kernel, which stream
    capture does not allow: a call on a capturing stream returns HASHGRID_ERR_ARG and
    issues nothing, and the capture and later eager calls are unaffected."""
    r = subprocess.run([sys.executable, "-c", CAPTURE], cwd=ROOT, env=checked_env(), capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr
