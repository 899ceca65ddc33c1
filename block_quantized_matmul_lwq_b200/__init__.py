"""Python binding of liblwq.so, the block-quantized matmul for B200 (sm_100a).

Argument marshalling only: every step of y = x . dequant(Wq)^T runs in the
library's CUDA kernels.  The names mirror the C ABI in include/lwq.h.
Pointer arguments accept plain integers or objects with ``data_ptr()`` (torch
tensors); ``stream`` accepts an integer cudaStream_t, an object with a
``cuda_stream`` attribute (torch.cuda.Stream), or None (legacy default stream).
The library is loaded on first use; any call fails loudly (ImportError)
when it has not been built -- there is no fallback of any kind.
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblwq.so")

# codes (include/lwq.h)
LWQ_Q8_0, LWQ_Q4_0, LWQ_Q4_K, LWQ_Q6_K, LWQ_Q5_K, LWQ_Q2_K = 1, 2, 3, 4, 5, 6
LWQ_ACT_F32, LWQ_ACT_F16, LWQ_ACT_BF16 = 0x000, 0x100, 0x200
LWQ_FLAG_OVERLAP = 0x1000   # weights constant: allow programmatic dependent launch
LWQ_FLAG_ACT_I8 = 0x2000    # int8 activation blocks of 32 (integer block dot products)
LWQ_OK = 0
LWQ_ERR_INVALID_ARG = 1
LWQ_ERR_UNSUPPORTED = 2
LWQ_ERR_MISALIGNED = 3
LWQ_ERR_NOT_INITIALIZED = 4
LWQ_ERR_WORKSPACE_TOO_SMALL = 5
LWQ_ERR_CUDA = 6
LWQ_ERR_DEVICE_TIMEOUT = 7
STATUS = {0: "LWQ_OK", 1: "LWQ_ERR_INVALID_ARG", 2: "LWQ_ERR_UNSUPPORTED", 3: "LWQ_ERR_MISALIGNED",
          4: "LWQ_ERR_NOT_INITIALIZED", 5: "LWQ_ERR_WORKSPACE_TOO_SMALL", 6: "LWQ_ERR_CUDA",
          7: "LWQ_ERR_DEVICE_TIMEOUT"}
WEIGHT_FORMATS = {"q8_0": LWQ_Q8_0, "q4_0": LWQ_Q4_0, "q4_k": LWQ_Q4_K, "q6_k": LWQ_Q6_K, "q5_k": LWQ_Q5_K,
                  "q2_k": LWQ_Q2_K}
ACT_DTYPES = {"f32": LWQ_ACT_F32, "f16": LWQ_ACT_F16, "bf16": LWQ_ACT_BF16}

# every symbol the header declares
EXPORTS = ["lwq_row_bytes", "lwq_workspace_size", "lwq_init", "lwq_shutdown", "lwq_matmul",
           "lwq_select_config", "lwq_matmul_config", "lwq_status_string", "lwq_get_device_error",
           "lwq_selftest_timeout", "lwq_last_launch_count", "lwq_version", "lwq_matmul_noalloc",
           "lwq_attention_workspace_size", "lwq_attention_decode"]


class LwqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({lwq_status_string(status)})")


class lwq_config(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int), ("warps", ctypes.c_int), ("stages", ctypes.c_int),
                ("splits", ctypes.c_int), ("ctas", ctypes.c_int), ("tile_n", ctypes.c_int),
                ("tile_m", ctypes.c_int), ("reserved", ctypes.c_int * 5)]

    def as_dict(self) -> dict:
        return {f: getattr(self, f) for f, _ in self._fields_ if f != "reserved"}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m block_quantized_matmul_lwq_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    c = ctypes
    vp, i = c.c_void_p, c.c_int
    lib.lwq_row_bytes.restype, lib.lwq_row_bytes.argtypes = c.c_size_t, [i, c.c_int64]
    lib.lwq_workspace_size.restype, lib.lwq_workspace_size.argtypes = c.c_size_t, [i, i, i, i]
    lib.lwq_init.restype, lib.lwq_init.argtypes = i, [vp, c.c_size_t]
    lib.lwq_shutdown.restype, lib.lwq_shutdown.argtypes = i, []
    lib.lwq_matmul.restype, lib.lwq_matmul.argtypes = i, [i, vp, vp, vp, i, i, i, vp]
    lib.lwq_select_config.restype = i
    lib.lwq_select_config.argtypes = [i, i, i, i, c.POINTER(lwq_config)]
    lib.lwq_matmul_config.restype = i
    lib.lwq_matmul_config.argtypes = [i, vp, vp, vp, i, i, i, c.POINTER(lwq_config), vp]
    lib.lwq_status_string.restype, lib.lwq_status_string.argtypes = c.c_char_p, [i]
    lib.lwq_get_device_error.restype, lib.lwq_get_device_error.argtypes = i, []
    lib.lwq_selftest_timeout.restype, lib.lwq_selftest_timeout.argtypes = i, [c.c_uint, vp]
    lib.lwq_last_launch_count.restype, lib.lwq_last_launch_count.argtypes = i, []
    lib.lwq_version.restype, lib.lwq_version.argtypes = i, []
    lib.lwq_matmul_noalloc.restype, lib.lwq_matmul_noalloc.argtypes = i, [i, vp, vp, vp, i, i, i, vp]
    lib.lwq_attention_workspace_size.restype = c.c_size_t
    lib.lwq_attention_workspace_size.argtypes = [i, i, i, i, i]
    lib.lwq_attention_decode.restype = i
    lib.lwq_attention_decode.argtypes = [i, vp, vp, vp, vp, vp, i, i, i, i, i, c.c_float, vp]
    return lib


_lib_handle = None


def lib() -> ctypes.CDLL:
    global _lib_handle
    if _lib_handle is None:
        _lib_handle = _load()
    return _lib_handle


class _LazyLib:
    def __getattr__(self, name):
        return getattr(lib(), name)


_lib = _LazyLib()


def _ptr(p) -> int:
    if p is None:
        return 0
    if isinstance(p, int):
        return p
    return int(p.data_ptr())


def _stream(s) -> int:
    if s is None:
        return 0
    if isinstance(s, int):
        return s
    return int(s.cuda_stream)


def _check(rc: int, where: str) -> int:
    if rc != LWQ_OK:
        raise LwqError(rc, where)
    return rc


def fmt_code(weights: str, act: str) -> int:
    """``fmt`` for the C ABI from names: weights in q8_0/q4_0/q4_k/q6_k/q5_k/q2_k, act in f32/f16/bf16."""
    return WEIGHT_FORMATS[weights] | ACT_DTYPES[act]


def lwq_status_string(status: int) -> str:
    return _lib.lwq_status_string(status).decode()


def lwq_row_bytes(fmt: int, K: int) -> int:
    return _lib.lwq_row_bytes(fmt, K)


def lwq_workspace_size(fmt: int, max_M: int, max_N: int, max_K: int) -> int:
    return _lib.lwq_workspace_size(fmt, max_M, max_N, max_K)


def lwq_init(workspace, nbytes: int) -> None:
    _check(_lib.lwq_init(_ptr(workspace), nbytes), "lwq_init")


def lwq_shutdown() -> None:
    _check(_lib.lwq_shutdown(), "lwq_shutdown")


def lwq_matmul(fmt: int, Wq, x, y, M: int, N: int, K: int, stream=None) -> None:
    _check(_lib.lwq_matmul(fmt, _ptr(Wq), _ptr(x), _ptr(y), M, N, K, _stream(stream)), "lwq_matmul")


def lwq_select_config(fmt: int, M: int, N: int, K: int) -> lwq_config:
    cfg = lwq_config()
    _check(_lib.lwq_select_config(fmt, M, N, K, ctypes.byref(cfg)), "lwq_select_config")
    return cfg


def lwq_matmul_config(fmt: int, Wq, x, y, M: int, N: int, K: int, cfg: lwq_config, stream=None) -> None:
    _check(_lib.lwq_matmul_config(fmt, _ptr(Wq), _ptr(x), _ptr(y), M, N, K, ctypes.byref(cfg), _stream(stream)),
           "lwq_matmul_config")


def lwq_get_device_error() -> int:
    """LWQ_OK, or LWQ_ERR_DEVICE_TIMEOUT (and clears it); synchronize first."""
    return _lib.lwq_get_device_error()


def lwq_selftest_timeout(timeout_us: int, stream=None) -> None:
    _check(_lib.lwq_selftest_timeout(timeout_us, _stream(stream)), "lwq_selftest_timeout")


def lwq_last_launch_count() -> int:
    return _lib.lwq_last_launch_count()


def lwq_version() -> int:
    return _lib.lwq_version()


def lwq_matmul_noalloc(fmt: int, Wq, x, y, M: int, N: int, K: int, stream=None) -> None:
    """lwq_matmul for callers that cannot allocate: no workspace, static 4 MiB scratch (see include/lwq.h)."""
    _check(_lib.lwq_matmul_noalloc(fmt, _ptr(Wq), _ptr(x), _ptr(y), M, N, K, _stream(stream)),
           "lwq_matmul_noalloc")


def lwq_attention_workspace_size(B: int, H: int, Hkv: int, Lmax: int, D: int) -> int:
    return _lib.lwq_attention_workspace_size(B, H, Hkv, Lmax, D)


def lwq_attention_decode(act: int, q, k, v, seq_lens, out, B: int, H: int, Hkv: int, Lmax: int, D: int,
                         scale: float, stream=None) -> None:
    """Decode attention through the C ABI (act: LWQ_ACT_F16 or LWQ_ACT_BF16; seq_lens may be None)."""
    _check(_lib.lwq_attention_decode(act, _ptr(q), _ptr(k), _ptr(v), _ptr(seq_lens), _ptr(out), B, H, Hkv, Lmax, D,
                                     float(scale), _stream(stream)), "lwq_attention_decode")
