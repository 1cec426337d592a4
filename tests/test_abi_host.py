"""Host-side tests of the C ABI (no GPU needed, no compute calls): the library loads and
exports every function that include/hashgrid.h declares, handles report their parameters,
the library's resolution schedule agrees with the oracle's and with exact integer floors,
and invalid arguments are rejected with the documented status before any launch."""
import ctypes
import glob
import os
import re
import shutil
import subprocess
import sys

import numpy as np
import pytest

import oracle
import multiresolution_hash_grid_b200 as hg
from tests.test_oracle_pins import exact_floor_resolution, near_integer_from_below

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE_DIR = os.path.join(ROOT, "include")
HEADER = os.path.join(INCLUDE_DIR, "hashgrid.h")
LIB_PATH = os.path.join(ROOT, "multiresolution_hash_grid_b200", "libhashgrid.so")


def declared_functions(headers=None):
    """Every hashgrid_* function declared in include/*.h (comments stripped)."""
    names = set()
    for path in headers or sorted(glob.glob(os.path.join(INCLUDE_DIR, "*.h"))):
        text = re.sub(r"/\*.*?\*/", "", open(path).read(), flags=re.S)
        names |= set(re.findall(r"\b(hashgrid_\w+)\s*\(", text))
    return sorted(names)


def test_library_exports_every_declared_function():
    names = declared_functions()
    assert "hashgrid_forward" in names and "hashgrid_backward" in names and "hashgrid_create" in names
    assert "hashgrid_probe" in names
    lib = ctypes.CDLL(hg.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    if shutil.which("nm"):
        out = subprocess.run(["nm", "-D", "--defined-only", hg.LIB_PATH], capture_output=True, text=True).stdout
        exported = set(re.findall(r" T (hashgrid_\w+)", out))
        assert set(names) <= exported


def test_library_is_sm100a_build():
    assert "sm_100a" in hg.hashgrid_version()


def test_create_params_and_sizes():
    h = hg.hashgrid_create(16, 2, 19, 16, 512, hg.HASHGRID_F32)
    try:
        assert hg.hashgrid_params(h) == dict(L=16, F=2, log2T=19, N_min=16, N_max=512, dtype=0)
        assert hg.hashgrid_table_elems(h) == 16 * 2**19 * 2
        assert hg.hashgrid_output_width(h) == 32
        assert hg.hashgrid_resolutions(h) == [16, 20, 25, 32, 40, 50, 64, 80, 101, 128, 161, 203, 256, 322, 406, 512]
    finally:
        hg.hashgrid_destroy(h)
    grid = hg.HashGrid(16, 4, 22, 16, 4096)
    assert grid.resolutions[-1] == 4096 and grid.resolutions[6] == 147
    assert hg.hashgrid_table_elems(0) == 0 and hg.hashgrid_output_width(0) == 0
    assert hg.lib.hashgrid_destroy(None) == hg.HASHGRID_OK


def test_resolutions_match_oracle_and_exact_floor():
    """The library computes the schedule in its own code; it must agree with the oracle on
    every level, and with the exact-integer floor where that is unambiguous."""
    rng = np.random.default_rng(20)
    cases = [(4, 2, 16), (16, 16, 512), (16, 16, 4096), (1, 7, 7), (32, 1, 2**20), (2, 3, 3)]
    for _ in range(200):
        L = int(rng.integers(2, 33))
        a = int(rng.integers(1, 2**12))
        cases.append((L, a, int(rng.integers(a, 2**20 + 1))))
    for L, a, b in cases:
        h = hg.hashgrid_create(L, 2, 10, a, b)
        try:
            got = hg.hashgrid_resolutions(h)
        finally:
            hg.hashgrid_destroy(h)
        assert got == oracle.resolutions(L, a, b), (L, a, b)
        for l in range(L):
            if L > 1 and not near_integer_from_below(L, a, b, l):
                assert got[l] == exact_floor_resolution(L, a, b, l)


@pytest.mark.parametrize("args", [
    (0, 2, 19, 16, 512, 0), (33, 2, 19, 16, 512, 0),             # L out of range
    (16, 3, 19, 16, 512, 0), (16, 0, 19, 16, 512, 0), (16, 16, 19, 16, 512, 0),  # F
    (16, 2, 3, 16, 512, 0), (16, 2, 25, 16, 512, 0),             # log2T
    (16, 2, 19, 0, 512, 0), (16, 2, 19, 600, 512, 0), (16, 2, 19, 16, 2**20 + 1, 0),
    (16, 2, 19, 16, 512, 2), (16, 2, 19, 16, 512, -1),           # dtype
    (1, 2, 19, 16, 512, 0),                                      # L = 1 needs N_min == N_max
])
def test_create_rejects_invalid(args):
    h = ctypes.c_void_p(1234)
    rc = hg.lib.hashgrid_create(*args, ctypes.byref(h))
    assert rc == hg.HASHGRID_ERR_ARG
    assert h.value is None
    assert hg.hashgrid_last_error() != ""
    with pytest.raises(hg.HashGridError) as e:
        hg.hashgrid_create(*args)
    assert e.value.code == hg.HASHGRID_ERR_ARG


def test_create_nd():
    for D in (2, 3, 4):
        h = hg.hashgrid_create_nd(D, 8, 2, 12, 4, 128)
        try:
            assert hg.hashgrid_dims(h) == D
            assert hg.hashgrid_resolutions(h) == oracle.resolutions(8, 4, 128)
        finally:
            hg.hashgrid_destroy(h)
    assert hg.hashgrid_dims(hg.hashgrid_create(4, 2, 10, 2, 16)) == 3
    for D in (0, 1, 5, 7):
        h = ctypes.c_void_p(99)
        assert hg.lib.hashgrid_create_nd(D, 8, 2, 12, 4, 128, 0, ctypes.byref(h)) == hg.HASHGRID_ERR_ARG
        assert h.value is None
    assert hg.hashgrid_dims(0) == 0


def test_options():
    h = hg.hashgrid_create(16, 2, 19, 16, 512)
    try:
        assert hg.hashgrid_get_option(h, hg.HASHGRID_OPT_FORWARD_GATHER) == hg.HASHGRID_GATHER_AUTO
        assert hg.hashgrid_get_option(h, hg.HASHGRID_OPT_BACKWARD_MODE) == hg.HASHGRID_BACKWARD_AUTO
        hg.hashgrid_set_option(h, hg.HASHGRID_OPT_FORWARD_GATHER, hg.HASHGRID_GATHER_SECTOR)
        hg.hashgrid_set_option(h, hg.HASHGRID_OPT_BACKWARD_MODE, hg.HASHGRID_BACKWARD_WARP_DEDUP)
        assert hg.hashgrid_get_option(h, hg.HASHGRID_OPT_FORWARD_GATHER) == hg.HASHGRID_GATHER_SECTOR
        assert hg.hashgrid_get_option(h, hg.HASHGRID_OPT_BACKWARD_MODE) == hg.HASHGRID_BACKWARD_WARP_DEDUP
        assert hg.hashgrid_get_option(h, hg.HASHGRID_OPT_SCHEDULE) == hg.HASHGRID_SCHEDULE_AUTO
        hg.hashgrid_set_option(h, hg.HASHGRID_OPT_SCHEDULE, hg.HASHGRID_SCHEDULE_LEVEL_MAJOR)
        assert hg.hashgrid_get_option(h, hg.HASHGRID_OPT_SCHEDULE) == hg.HASHGRID_SCHEDULE_LEVEL_MAJOR
        for opt, val in [(hg.HASHGRID_OPT_SCHEDULE, 3), (hg.HASHGRID_OPT_FORWARD_GATHER, 5), (hg.HASHGRID_OPT_BACKWARD_MODE, -1), (hg.HASHGRID_OPT_BACKWARD_MODE, 6), (7, 0)]:
            assert hg.lib.hashgrid_set_option(h, opt, val) == hg.HASHGRID_ERR_ARG
        assert hg.lib.hashgrid_set_option(None, 0, 0) == hg.HASHGRID_ERR_ARG
    finally:
        hg.hashgrid_destroy(h)
    h8 = hg.hashgrid_create(4, 8, 10, 2, 16)
    try:   # warp dedup works on 16-byte gradient units: F <= 4 only
        assert hg.lib.hashgrid_set_option(h8, hg.HASHGRID_OPT_BACKWARD_MODE, hg.HASHGRID_BACKWARD_WARP_DEDUP) == hg.HASHGRID_ERR_ARG
        assert hg.lib.hashgrid_set_option(h8, hg.HASHGRID_OPT_BACKWARD_MODE, hg.HASHGRID_BACKWARD_RUN_MERGE) == hg.HASHGRID_ERR_ARG
        assert hg.lib.hashgrid_set_option(h8, hg.HASHGRID_OPT_BACKWARD_MODE, hg.HASHGRID_BACKWARD_RUN_LANES) == hg.HASHGRID_ERR_ARG
    finally:
        hg.hashgrid_destroy(h8)


def test_calls_validate_before_any_launch():
    h = hg.hashgrid_create(4, 2, 10, 2, 16)
    try:
        L = hg.lib
        # NULL handle
        assert L.hashgrid_forward(None, 0x1000, 1, 0x1000, 0x1000, None) == hg.HASHGRID_ERR_ARG
        assert L.hashgrid_backward(None, 0x1000, 0x1000, 1, 0x1000, None) == hg.HASHGRID_ERR_ARG
        assert L.hashgrid_resolutions(None, None) == hg.HASHGRID_ERR_ARG
        # N < 0, N too large for a launch
        assert L.hashgrid_forward(h, 0x1000, -1, 0x1000, 0x1000, None) == hg.HASHGRID_ERR_ARG
        assert L.hashgrid_forward(h, 0x1000, 2**62, 0x1000, 0x1000, None) == hg.HASHGRID_ERR_ARG
        # N == 0 is a no-op, any pointers
        assert L.hashgrid_forward(h, None, 0, None, None, None) == hg.HASHGRID_OK
        assert L.hashgrid_backward(h, None, None, 0, None, None) == hg.HASHGRID_OK
        assert L.hashgrid_debug_indices(h, None, 0, None, None) == hg.HASHGRID_OK
        # NULL buffers
        assert L.hashgrid_forward(h, None, 5, 0x1000, 0x1000, None) == hg.HASHGRID_ERR_ARG
        assert "x is NULL" in hg.hashgrid_last_error()
        assert L.hashgrid_backward(h, 0x1000, None, 5, 0x1000, None) in (hg.HASHGRID_ERR_ARG,)
        # misaligned pointers are rejected before the runtime is consulted
        assert L.hashgrid_forward(h, 0x1004, 5, 0x1000, 0x1000, None) == hg.HASHGRID_ERR_ALIGN
        assert L.hashgrid_forward(h, 0x1000, 5, 0x1008, 0x1000, None) in (hg.HASHGRID_ERR_ALIGN, hg.HASHGRID_ERR_ARG)
        assert L.hashgrid_debug_indices(h, 0x100c, 5, 0x1000, None) == hg.HASHGRID_ERR_ALIGN
        # ordinary host memory is not device memory
        a = np.zeros(1024, dtype=np.float32)
        assert a.ctypes.data % 16 == 0
        assert L.hashgrid_forward(h, a.ctypes.data, 5, a.ctypes.data, a.ctypes.data, None) == hg.HASHGRID_ERR_ARG
        assert L.hashgrid_backward(h, a.ctypes.data, a.ctypes.data, 5, a.ctypes.data, None) == hg.HASHGRID_ERR_ARG
        assert np.all(a == 0)
    finally:
        hg.hashgrid_destroy(h)


def test_adam_and_input_gradient_validate_arguments():
    h = hg.hashgrid_create(4, 2, 10, 2, 16)
    try:
        L = hg.lib
        f = ctypes.c_float
        assert L.hashgrid_adam_step(h, 0x1000, 0x1000, 0x1000, 0x1000, 0, f(1e-2), f(0.9), f(0.99), f(1e-15), 1, None) == hg.HASHGRID_ERR_ARG
        assert L.hashgrid_adam_step(h, 0x1000, 0x1000, 0x1000, 0x1000, 1, f(1e-2), f(1.0), f(0.99), f(1e-15), 1, None) == hg.HASHGRID_ERR_ARG
        assert L.hashgrid_adam_step(h, 0x1000, 0x1000, 0x1000, 0x1000, 1, f(1e-2), f(0.9), f(0.99), f(0.0), 1, None) == hg.HASHGRID_ERR_ARG
        assert L.hashgrid_adam_step(h, None, 0x1000, 0x1000, 0x1000, 1, f(1e-2), f(0.9), f(0.99), f(1e-15), 1, None) == hg.HASHGRID_ERR_ARG
        assert L.hashgrid_adam_step(None, 0x1000, 0x1000, 0x1000, 0x1000, 1, f(1e-2), f(0.9), f(0.99), f(1e-15), 1, None) == hg.HASHGRID_ERR_ARG
        assert L.hashgrid_backward_input(h, None, None, 0, None, None, None) == hg.HASHGRID_OK
        assert L.hashgrid_backward_input(h, 0x1004, 0x1000, 3, 0x1000, 0x1000, None) == hg.HASHGRID_ERR_ALIGN
        a = np.zeros(4096, dtype=np.float32)
        assert L.hashgrid_backward_input(h, a.ctypes.data, a.ctypes.data, 3, a.ctypes.data, a.ctypes.data, None) == hg.HASHGRID_ERR_ARG
    finally:
        hg.hashgrid_destroy(h)


def test_binding_fails_loudly_without_library(tmp_path):
    """A copy of the binding with no built library beside it must raise ImportError on
    import: there is no fallback path."""
    pkg = tmp_path / "multiresolution_hash_grid_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(os.path.dirname(hg.__file__), "__init__.py"), pkg / "__init__.py")
    r = subprocess.run([sys.executable, "-c", "import multiresolution_hash_grid_b200"], cwd=tmp_path,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "ImportError" in r.stderr and "not built" in r.stderr


C_CLIENT = r"""
#include <stdio.h>
#include "hashgrid.h"
#include "hashgrid_probe.h"

int main(void)
{
    hashgrid_t h = NULL;
    int res[16], L, F, log2T, nmin, nmax, dtype;
    if (hashgrid_create(16, 2, 19, 16, 512, HASHGRID_F32, &h) != HASHGRID_OK) {
        fprintf(stderr, "%s\n", hashgrid_last_error());
        return 1;
    }
    if (hashgrid_resolutions(h, res) != HASHGRID_OK || res[0] != 16 || res[15] != 512) return 2;
    if (hashgrid_params(h, &L, &F, &log2T, &nmin, &nmax, &dtype) != HASHGRID_OK || L != 16 || F != 2) return 3;
    if (hashgrid_table_elems(h) != (size_t)16 * 524288 * 2 || hashgrid_output_width(h) != 32) return 4;
    /* an invalid call is an error code before any launch, with a message */
    if (hashgrid_forward(h, NULL, 4, NULL, NULL, NULL) == HASHGRID_OK || hashgrid_last_error()[0] == 0) return 5;
    if (hashgrid_probe(7, 8, HASHGRID_PROBE_RANDOM, NULL, 1024, 1, NULL, NULL, NULL) != HASHGRID_ERR_ARG) return 6;
    hashgrid_destroy(h);
    printf("%s\n", hashgrid_version());
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc missing")
def test_header_is_plain_c_and_links(tmp_path):
    """A C99 client compiled with gcc -Wall -Werror against include/*.h links to the
    library and uses it without a GPU (create, queries, an argument error, destroy)."""
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE_DIR, str(src), "-o", str(exe),
                    "-L", libdir, "-lhashgrid", f"-Wl,-rpath,{libdir}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stderr)
    assert "sm_100a" in r.stdout
