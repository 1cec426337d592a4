"""CPU oracle for the multiresolution hash-grid encoding (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package. The CUDA library never imports, links or calls it, and this
package imports nothing from the library. The arithmetic lives in ``hashgrid_oracle.c``
(plain C, fp64); this module only marshals numpy arrays through ctypes.

Every function here names the page section it follows in the C source. Inputs are numpy
arrays; outputs are fp64 numpy arrays (or uint32 for hash indices).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None

F32 = 0
F16 = 1


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i32, i64, vp = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p
        lib.oracle_resolutions.argtypes = [i32, i32, i32, vp]
        lib.oracle_resolutions.restype = i32
        lib.oracle_hash3.argtypes = [i64, i64, i64]
        lib.oracle_hash3.restype = ctypes.c_uint32
        lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_half_to_double.restype = ctypes.c_double
        lib.oracle_indices.argtypes = [i32, i32, vp, vp, i64, i32, i32, vp]
        lib.oracle_indices.restype = None
        lib.oracle_forward.argtypes = [i32, i32, i32, vp, i32, vp, vp, i64, i32, i32, vp, i32]
        lib.oracle_forward.restype = None
        lib.oracle_backward.argtypes = [i32, i32, i32, vp, vp, vp, i64, i32, i32, vp, i32]
        lib.oracle_backward.restype = None
        lib.oracle_backward_x.argtypes = [i32, i32, i32, vp, i32, vp, vp, vp, i64, i32, i32, vp, i32]
        lib.oracle_backward_x.restype = None
        dbl = ctypes.c_double
        lib.oracle_adam_step.argtypes = [i64, vp, vp, vp, vp, i64, dbl, dbl, dbl, dbl]
        lib.oracle_adam_step.restype = None
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_double.restype = ctypes.c_double
        lib.oracle_mlp_forward.argtypes = [i32, i32, i32, vp, i32, vp, vp, i64, vp, vp, vp, vp, vp, vp, vp, i32]
        lib.oracle_mlp_forward.restype = None
        lib.oracle_hash_nd.argtypes = [i32, vp]
        lib.oracle_hash_nd.restype = ctypes.c_uint32
        lib.oracle_indices_nd.argtypes = [i32, i32, i32, vp, vp, i64, vp]
        lib.oracle_indices_nd.restype = None
        lib.oracle_forward_nd.argtypes = [i32, i32, i32, i32, vp, i32, vp, vp, i64, vp, i32]
        lib.oracle_forward_nd.restype = None
        lib.oracle_backward_nd.argtypes = [i32, i32, i32, i32, vp, vp, vp, i64, vp, i32]
        lib.oracle_backward_nd.restype = None
        lib.oracle_backward_x_nd.argtypes = [i32, i32, i32, i32, vp, i32, vp, vp, vp, i64, vp, i32]
        lib.oracle_backward_x_nd.restype = None
        _LIB = lib
    return _LIB


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def default_threads() -> int:
    return len(os.sched_getaffinity(0))


def resolutions(L: int, N_min: int, N_max: int) -> list[int]:
    """Per-level grid resolutions N_l (NeRFace-HG section 2, reading R1 in the C file)."""
    out = np.zeros(max(L, 1), dtype=np.int32)
    rc = _lib().oracle_resolutions(L, N_min, N_max, _ptr(out))
    if rc != 0:
        raise ValueError(f"invalid resolution arguments L={L} N_min={N_min} N_max={N_max}")
    return [int(v) for v in out[:L]]


def hash3(c0: int, c1: int, c2: int) -> int:
    """uint32 spatial hash of one vertex (Repro-HG section 2.2, Overview-HG section 2.2)."""
    return int(_lib().oracle_hash3(int(c0), int(c1), int(c2)))


def half_to_double(bits: int) -> float:
    """IEEE binary16 bit pattern -> float, decoded from the format's definition."""
    return float(_lib().oracle_half_to_double(int(bits) & 0xFFFF))


def hash_nd(coords) -> int:
    """uint32 hash of a D-dimensional vertex with the 7-prime list (Repro-HG sections 2.2, 3)."""
    c = np.ascontiguousarray(np.asarray(coords, dtype=np.int64))
    return int(_lib().oracle_hash_nd(c.size, _ptr(c)))


class GridND:
    """D-dimensional encoding (D in 2..7 for the hash; 2^D corners, multilinear weights)."""

    def __init__(self, D: int, L: int, F: int, log2T: int, N_min: int, N_max: int, dtype: int = F32):
        self.D, self.L, self.F, self.log2T, self.N_min, self.N_max, self.dtype = D, L, F, log2T, N_min, N_max, dtype
        self.T = 1 << log2T
        self.res = np.asarray(resolutions(L, N_min, N_max), dtype=np.int32)

    def _x(self, x):
        return np.ascontiguousarray(x, dtype=np.float32).reshape(-1, self.D)

    def _table(self, table):
        return Grid._check_table(self, table)

    def indices(self, x):
        x = self._x(x)
        idx = np.zeros((x.shape[0], self.L, 1 << self.D), dtype=np.uint32)
        _lib().oracle_indices_nd(self.D, self.L, self.log2T, _ptr(self.res), _ptr(x), x.shape[0], _ptr(idx))
        return idx

    def forward(self, x, table, nthreads: int = 1):
        x, table = self._x(x), self._table(table)
        out = np.zeros((x.shape[0], self.L * self.F))
        _lib().oracle_forward_nd(self.D, self.L, self.F, self.log2T, _ptr(self.res), self.dtype, _ptr(table), _ptr(x),
                                 x.shape[0], _ptr(out), nthreads)
        return out

    def backward(self, x, g, nthreads: int = 1):
        x = self._x(x)
        g = np.ascontiguousarray(g, dtype=np.float32).reshape(x.shape[0], self.L * self.F)
        d = np.zeros((self.L, self.T, self.F))
        _lib().oracle_backward_nd(self.D, self.L, self.F, self.log2T, _ptr(self.res), _ptr(x), _ptr(g), x.shape[0],
                                  _ptr(d), nthreads)
        return d

    def backward_x(self, x, table, g, nthreads: int = 1):
        x, table = self._x(x), self._table(table)
        g = np.ascontiguousarray(g, dtype=np.float32).reshape(x.shape[0], self.L * self.F)
        dx = np.zeros((x.shape[0], self.D))
        _lib().oracle_backward_x_nd(self.D, self.L, self.F, self.log2T, _ptr(self.res), self.dtype, _ptr(table),
                                    _ptr(x), _ptr(g), x.shape[0], _ptr(dx), nthreads)
        return dx


def bf16_to_double(bits: int) -> float:
    """bfloat16 bit pattern -> float (the upper half of a binary32)."""
    return float(_lib().oracle_bf16_to_double(int(bits) & 0xFFFF))


def adam_step(param: np.ndarray, m: np.ndarray, v: np.ndarray, grad: np.ndarray, step: int,
              lr: float, beta1: float = 0.9, beta2: float = 0.99, eps: float = 1e-15):
    """Sparse Adam (NeRFace-HG sections 3-4): fp64 copies of param/m/v updated where the
    fp32 gradient is nonzero. Returns (param, m, v) as new fp64 arrays."""
    p = np.array(param, dtype=np.float64).ravel()
    mm = np.array(m, dtype=np.float64).ravel()
    vv = np.array(v, dtype=np.float64).ravel()
    g = np.ascontiguousarray(grad, dtype=np.float32).ravel()
    assert p.size == mm.size == vv.size == g.size
    _lib().oracle_adam_step(p.size, _ptr(p), _ptr(mm), _ptr(vv), _ptr(g), int(step), lr, beta1, beta2, eps)
    return p, mm, vv


class Grid:
    """Grid parameters as the C-ABI's create call takes them."""

    def __init__(self, L: int, F: int, log2T: int, N_min: int, N_max: int, dtype: int = F32):
        self.L, self.F, self.log2T, self.N_min, self.N_max, self.dtype = L, F, log2T, N_min, N_max, dtype
        self.T = 1 << log2T
        self.res = np.asarray(resolutions(L, N_min, N_max), dtype=np.int32)

    def _levels(self, levels):
        if levels is None:
            return 0, self.L
        l0, l1 = levels
        assert 0 <= l0 <= l1 <= self.L
        return l0, l1

    def _check_table(self, table: np.ndarray) -> np.ndarray:
        want = np.float32 if self.dtype == F32 else np.uint16
        if self.dtype == F16 and table.dtype == np.float16:
            table = table.view(np.uint16)
        assert table.dtype == want, (table.dtype, want)
        assert table.size == self.L * self.T * self.F
        return np.ascontiguousarray(table)

    def indices(self, x: np.ndarray, levels=None) -> np.ndarray:
        """uint32 [N, L, 8] hash indices, corner c = (c&1, c>>1&1, c>>2&1) offsets."""
        x = np.ascontiguousarray(x, dtype=np.float32).reshape(-1, 3)
        N = x.shape[0]
        l0, l1 = self._levels(levels)
        idx = np.zeros((N, self.L, 8), dtype=np.uint32)
        _lib().oracle_indices(self.L, self.log2T, _ptr(self.res), _ptr(x), N, l0, l1, _ptr(idx))
        return idx

    def forward(self, x: np.ndarray, table: np.ndarray, levels=None, nthreads: int = 1) -> np.ndarray:
        """fp64 [N, L*F] encoding (NeRFace-HG section 2; Repro-HG section 3)."""
        x = np.ascontiguousarray(x, dtype=np.float32).reshape(-1, 3)
        table = self._check_table(table)
        N = x.shape[0]
        l0, l1 = self._levels(levels)
        out = np.zeros((N, self.L * self.F), dtype=np.float64)
        _lib().oracle_forward(self.L, self.F, self.log2T, _ptr(self.res), self.dtype, _ptr(table),
                              _ptr(x), N, l0, l1, _ptr(out), nthreads)
        return out

    def backward(self, x: np.ndarray, g: np.ndarray, levels=None, nthreads: int = 1,
                 dtable: np.ndarray | None = None) -> np.ndarray:
        """fp64 [L, T, F] table gradient, accumulated into ``dtable`` (zeros if None)."""
        x = np.ascontiguousarray(x, dtype=np.float32).reshape(-1, 3)
        g = np.ascontiguousarray(g, dtype=np.float32).reshape(x.shape[0], self.L * self.F)
        N = x.shape[0]
        l0, l1 = self._levels(levels)
        if dtable is None:
            dtable = np.zeros((self.L, self.T, self.F), dtype=np.float64)
        assert dtable.dtype == np.float64 and dtable.size == self.L * self.T * self.F
        _lib().oracle_backward(self.L, self.F, self.log2T, _ptr(self.res), _ptr(x), _ptr(g), N,
                               l0, l1, _ptr(dtable), nthreads)
        return dtable

    def backward_x(self, x: np.ndarray, table: np.ndarray, g: np.ndarray, levels=None,
                   nthreads: int = 1) -> np.ndarray:
        """fp64 [N, 3] gradient of <g, encoding> with respect to x (NeRFace-HG section 3;
        derivative of the trilinear weights inside the voxel that contains x)."""
        x = np.ascontiguousarray(x, dtype=np.float32).reshape(-1, 3)
        table = self._check_table(table)
        g = np.ascontiguousarray(g, dtype=np.float32).reshape(x.shape[0], self.L * self.F)
        N = x.shape[0]
        l0, l1 = self._levels(levels)
        dx = np.zeros((N, 3), dtype=np.float64)
        _lib().oracle_backward_x(self.L, self.F, self.log2T, _ptr(self.res), self.dtype, _ptr(table),
                                 _ptr(x), _ptr(g), N, l0, l1, _ptr(dx), nthreads)
        return dx

    def mlp_forward(self, x: np.ndarray, table: np.ndarray, w1: np.ndarray, b1: np.ndarray, w2: np.ndarray,
                    b2: np.ndarray, w3: np.ndarray, b3: np.ndarray, nthreads: int = 1) -> np.ndarray:
        """fp64 [N, 4] = W3 relu(W2 relu(W1 enc(x) + b1) + b2) + b3 (NeRFace-HG section 3,
        Repro-HG section 4). Weights: uint16 bf16 bit patterns [out][in]; biases fp32."""
        x = np.ascontiguousarray(x, dtype=np.float32).reshape(-1, 3)
        table = self._check_table(table)
        K = self.L * self.F
        w1 = np.ascontiguousarray(w1, dtype=np.uint16).reshape(64, K)
        w2 = np.ascontiguousarray(w2, dtype=np.uint16).reshape(64, 64)
        w3 = np.ascontiguousarray(w3, dtype=np.uint16).reshape(4, 64)
        b1 = np.ascontiguousarray(b1, dtype=np.float32).reshape(64)
        b2 = np.ascontiguousarray(b2, dtype=np.float32).reshape(64)
        b3 = np.ascontiguousarray(b3, dtype=np.float32).reshape(4)
        N = x.shape[0]
        y = np.zeros((N, 4), dtype=np.float64)
        _lib().oracle_mlp_forward(self.L, self.F, self.log2T, _ptr(self.res), self.dtype, _ptr(table), _ptr(x), N,
                                  _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2), _ptr(w3), _ptr(b3), _ptr(y), nthreads)
        return y
