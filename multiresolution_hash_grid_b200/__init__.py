"""Python binding of libhashgrid.so, the B200 (sm_100a) multiresolution hash-grid encoding.

Argument marshalling only: every step of the encoding runs in the library's CUDA kernels.
PyTorch supplies device memory and streams. The functions carry the C ABI's names
(``include/hashgrid.h`` documents semantics, layouts and errors) and take either torch
CUDA tensors or raw integer device pointers; ``stream`` defaults to torch's current
stream. A nonzero status raises ``HashGridError`` with the library's message.

The library must be built (``python multiresolution_hash_grid_b200/build.py``); importing
this package without it raises ImportError. There is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# HASHGRID_CHECKED=1 loads the checked build (every global access of the kernels range-checked,
# violations returned as HASHGRID_ERR_DEVICE_CHECK; synchronous, for testing).
CHECKED = os.environ.get("HASHGRID_CHECKED", "0") not in ("", "0")
LIB_PATH = os.path.join(HERE, "libhashgrid_checked.so" if CHECKED else "libhashgrid.so")

HASHGRID_F32 = 0
HASHGRID_F16 = 1

HASHGRID_OK = 0
HASHGRID_ERR_ARG = 1
HASHGRID_ERR_ALIGN = 2
HASHGRID_ERR_CUDA = 3
HASHGRID_ERR_OOM = 4
HASHGRID_ERR_DEVICE_CHECK = 5

MAX_LEVELS = 32

HASHGRID_OPT_FORWARD_GATHER = 0
HASHGRID_OPT_BACKWARD_MODE = 1
HASHGRID_OPT_SCHEDULE = 2
HASHGRID_SCHEDULE_AUTO = 0
HASHGRID_SCHEDULE_POINT_MAJOR = 1
HASHGRID_SCHEDULE_LEVEL_MAJOR = 2
HASHGRID_GATHER_AUTO = 0
HASHGRID_GATHER_CORNER = 1
HASHGRID_GATHER_SECTOR = 2
HASHGRID_GATHER_PAIR = 3
HASHGRID_GATHER_LANES = 4
HASHGRID_BACKWARD_AUTO = 0
HASHGRID_BACKWARD_ATOMIC = 1
HASHGRID_BACKWARD_WARP_DEDUP = 2
HASHGRID_BACKWARD_RUN_MERGE = 3
HASHGRID_BACKWARD_WARP_DEDUP_ADAPTIVE = 4
HASHGRID_BACKWARD_RUN_LANES = 5
HASHGRID_PROBE_GATHER = 0
HASHGRID_PROBE_RED = 1
HASHGRID_PROBE_RED_F16 = 2
HASHGRID_PROBE_RANDOM = 0
HASHGRID_PROBE_XPAIR = 1
HASHGRID_PROBE_SECTOR_PAIR = 2
HASHGRID_PROBE_LINE_PAIR = 3
HASHGRID_PROBE_STREAM = 4


class HashGridError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"hashgrid error {code}: {message}")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built: run `python multiresolution_hash_grid_b200/build.py"
                          f"{' --checked' if CHECKED else ''}`")
    lib = ctypes.CDLL(LIB_PATH)
    i32, i64, vp, sz = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t
    protos = {
        "hashgrid_create": (i32, [i32, i32, i32, i32, i32, i32, ctypes.POINTER(vp)]),
        "hashgrid_create_nd": (i32, [i32, i32, i32, i32, i32, i32, i32, ctypes.POINTER(vp)]),
        "hashgrid_dims": (i32, [vp]),
        "hashgrid_destroy": (i32, [vp]),
        "hashgrid_resolutions": (i32, [vp, ctypes.POINTER(i32)]),
        "hashgrid_table_elems": (sz, [vp]),
        "hashgrid_output_width": (i32, [vp]),
        "hashgrid_params": (i32, [vp] + [ctypes.POINTER(i32)] * 6),
        "hashgrid_set_option": (i32, [vp, i32, i32]),
        "hashgrid_get_option": (i32, [vp, i32, ctypes.POINTER(i32)]),
        "hashgrid_forward": (i32, [vp, vp, i64, vp, vp, vp]),
        "hashgrid_backward": (i32, [vp, vp, vp, i64, vp, vp]),
        "hashgrid_backward_input": (i32, [vp, vp, vp, i64, vp, vp, vp]),
        "hashgrid_backward_half": (i32, [vp, vp, vp, i64, vp, vp]),
        "hashgrid_adam_step": (i32, [vp, vp, vp, vp, vp, i64, ctypes.c_float, ctypes.c_float, ctypes.c_float,
                                     ctypes.c_float, i32, vp]),
        "hashgrid_mlp_forward": (i32, [vp, vp, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "hashgrid_debug_indices": (i32, [vp, vp, i64, vp, vp]),
        "hashgrid_probe": (i32, [i32, i32, i32, vp, sz, i64, vp, ctypes.POINTER(i64), vp]),
        "hashgrid_last_error": (ctypes.c_char_p, []),
        "hashgrid_version": (ctypes.c_char_p, []),
    }
    for name, (res, args) in protos.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


lib = _load()


def _check(rc: int) -> None:
    if rc != HASHGRID_OK:
        raise HashGridError(rc, lib.hashgrid_last_error().decode())


def _ptr(a) -> int | None:
    if a is None:
        return None
    if isinstance(a, int):
        return a
    return a.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def hashgrid_version() -> str:
    return lib.hashgrid_version().decode()


def hashgrid_last_error() -> str:
    return lib.hashgrid_last_error().decode()


def hashgrid_create(L: int, F: int, log2T: int, N_min: int, N_max: int, dtype: int = HASHGRID_F32) -> int:
    h = ctypes.c_void_p()
    _check(lib.hashgrid_create(L, F, log2T, N_min, N_max, dtype, ctypes.byref(h)))
    return h.value


def hashgrid_create_nd(D: int, L: int, F: int, log2T: int, N_min: int, N_max: int, dtype: int = HASHGRID_F32) -> int:
    h = ctypes.c_void_p()
    _check(lib.hashgrid_create_nd(D, L, F, log2T, N_min, N_max, dtype, ctypes.byref(h)))
    return h.value


def hashgrid_dims(h: int) -> int:
    return int(lib.hashgrid_dims(h))


def hashgrid_destroy(h: int) -> None:
    _check(lib.hashgrid_destroy(h))


def hashgrid_params(h: int) -> dict:
    vals = [ctypes.c_int() for _ in range(6)]
    _check(lib.hashgrid_params(h, *[ctypes.byref(v) for v in vals]))
    return dict(zip(("L", "F", "log2T", "N_min", "N_max", "dtype"), (v.value for v in vals)))


def hashgrid_resolutions(h: int) -> list[int]:
    arr = (ctypes.c_int * MAX_LEVELS)()
    _check(lib.hashgrid_resolutions(h, arr))
    return list(arr[: hashgrid_params(h)["L"]])


def hashgrid_set_option(h: int, option: int, value: int) -> None:
    _check(lib.hashgrid_set_option(h, option, value))


def hashgrid_get_option(h: int, option: int) -> int:
    v = ctypes.c_int()
    _check(lib.hashgrid_get_option(h, option, ctypes.byref(v)))
    return v.value


def hashgrid_table_elems(h: int) -> int:
    return int(lib.hashgrid_table_elems(h))


def hashgrid_output_width(h: int) -> int:
    return int(lib.hashgrid_output_width(h))


def hashgrid_forward(h: int, x, N: int, table, out, stream=None) -> None:
    _check(lib.hashgrid_forward(h, _ptr(x), N, _ptr(table), _ptr(out), _stream(stream)))


def hashgrid_backward(h: int, x, dL_dout, N: int, dL_dtable, stream=None) -> None:
    _check(lib.hashgrid_backward(h, _ptr(x), _ptr(dL_dout), N, _ptr(dL_dtable), _stream(stream)))


def hashgrid_backward_half(h: int, x, dL_dout, N: int, dL_dtable, stream=None) -> None:
    _check(lib.hashgrid_backward_half(h, _ptr(x), _ptr(dL_dout), N, _ptr(dL_dtable), _stream(stream)))


def hashgrid_backward_input(h: int, x, dL_dout, N: int, table, dL_dx, stream=None) -> None:
    _check(lib.hashgrid_backward_input(h, _ptr(x), _ptr(dL_dout), N, _ptr(table), _ptr(dL_dx), _stream(stream)))


def hashgrid_adam_step(h: int, table, adam_m, adam_v, dL_dtable, step: int, lr: float, beta1: float = 0.9,
                       beta2: float = 0.99, eps: float = 1e-15, zero_grad: bool = True, stream=None) -> None:
    _check(lib.hashgrid_adam_step(h, _ptr(table), _ptr(adam_m), _ptr(adam_v), _ptr(dL_dtable), step, lr, beta1,
                                  beta2, eps, 1 if zero_grad else 0, _stream(stream)))


def hashgrid_mlp_forward(h: int, x, N: int, table, w1, b1, w2, b2, w3, b3, y, device_status=None,
                         stream=None) -> None:
    _check(lib.hashgrid_mlp_forward(h, _ptr(x), N, _ptr(table), _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2), _ptr(w3),
                                    _ptr(b3), _ptr(y), _ptr(device_status), _stream(stream)))


def hashgrid_debug_indices(h: int, x, N: int, idx_out, stream=None) -> None:
    _check(lib.hashgrid_debug_indices(h, _ptr(x), N, _ptr(idx_out), _stream(stream)))


def hashgrid_probe(kind: int, width: int, pattern: int, buf, buf_bytes: int, ops: int, sink=None,
                   stream=None) -> int:
    """Runs one memory-system probe (include/hashgrid_probe.h); returns the number of lane
    operations the kernel performs."""
    done = ctypes.c_int64()
    _check(lib.hashgrid_probe(kind, width, pattern, _ptr(buf), buf_bytes, ops, _ptr(sink), ctypes.byref(done),
                              _stream(stream)))
    return done.value


class HashGrid:
    """Owns a handle and allocates outputs with torch; the encoding itself runs in the
    library. ``table`` arguments are CUDA tensors of shape [L, T, F] (float32 or float16,
    matching ``dtype``)."""

    def __init__(self, L: int = 16, F: int = 2, log2T: int = 19, N_min: int = 16, N_max: int = 512,
                 dtype: int = HASHGRID_F32, forward_gather: int = HASHGRID_GATHER_AUTO,
                 backward_mode: int = HASHGRID_BACKWARD_AUTO, schedule: int = HASHGRID_SCHEDULE_AUTO, D: int = 3):
        self.L, self.F, self.log2T, self.N_min, self.N_max, self.dtype, self.D = L, F, log2T, N_min, N_max, dtype, D
        self.T = 1 << log2T
        self.handle = hashgrid_create_nd(D, L, F, log2T, N_min, N_max, dtype)
        hashgrid_set_option(self.handle, HASHGRID_OPT_FORWARD_GATHER, forward_gather)
        hashgrid_set_option(self.handle, HASHGRID_OPT_BACKWARD_MODE, backward_mode)
        hashgrid_set_option(self.handle, HASHGRID_OPT_SCHEDULE, schedule)

    def __del__(self):
        h = getattr(self, "handle", None)
        if h and lib is not None:  # the module may already be torn down at interpreter exit
            lib.hashgrid_destroy(h)
            self.handle = None

    @property
    def resolutions(self) -> list[int]:
        return hashgrid_resolutions(self.handle)

    def forward(self, x, table, out=None, stream=None):
        import torch
        N = x.shape[0]
        if out is None:
            out = torch.empty((N, self.L * self.F), dtype=torch.float32, device=x.device)
        hashgrid_forward(self.handle, x, N, table, out, stream)
        return out

    def backward(self, x, dL_dout, dL_dtable=None, stream=None):
        import torch
        if dL_dtable is None:
            dL_dtable = torch.zeros((self.L, self.T, self.F), dtype=torch.float32, device=x.device)
        hashgrid_backward(self.handle, x, dL_dout, x.shape[0], dL_dtable, stream)
        return dL_dtable

    def backward_input(self, x, dL_dout, table, dL_dx=None, stream=None):
        import torch
        if dL_dx is None:
            dL_dx = torch.empty((x.shape[0], self.D), dtype=torch.float32, device=x.device)
        hashgrid_backward_input(self.handle, x, dL_dout, x.shape[0], table, dL_dx, stream)
        return dL_dx

    def indices(self, x, stream=None):
        import torch
        idx = torch.empty((x.shape[0], self.L, 1 << self.D), dtype=torch.int32, device=x.device)
        hashgrid_debug_indices(self.handle, x, x.shape[0], idx, stream)
        return idx
