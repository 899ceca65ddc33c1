"""CPU oracle for the block-quantized matmul -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The library under
``block_quantized_matmul_lwq_b200`` never does, and shares no code with it.

The arithmetic lives in ``lwq_oracle.c`` (plain C, fp64 accumulation, one
OpenMP loop over output rows); this module only builds it with gcc and
marshals numpy arrays through ctypes.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lwq_oracle.c")
_LIB = os.path.join(_HERE, "liblwq_oracle.so")

FMT = {"q8_0": 1, "q4_0": 2, "q4_k": 3, "q6_k": 4, "q5_k": 5, "q2_k": 6}
ACT = {"f32": 0, "f16": 1, "bf16": 2}

CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-shared", "-fPIC", "-std=c11"]


def build(out: str = _LIB, extra: list[str] | None = None) -> str:
    """Compile the oracle with gcc (no-op when the .so is newer than the source)."""
    if extra is None and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(_SRC):
        return out
    cmd = ["gcc", *CFLAGS, *(extra or []), _SRC, "-o", out + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


_lib = None


def _bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    c = ctypes
    lib.lwq_oracle_f16.restype = c.c_double
    lib.lwq_oracle_f16.argtypes = [c.c_uint16]
    lib.lwq_oracle_bf16.restype = c.c_double
    lib.lwq_oracle_bf16.argtypes = [c.c_uint16]
    lib.lwq_oracle_row_bytes.restype = c.c_long
    lib.lwq_oracle_row_bytes.argtypes = [c.c_int, c.c_long]
    lib.lwq_oracle_q4k_scale_min.restype = None
    lib.lwq_oracle_q4k_scale_min.argtypes = [c.c_void_p, c.c_int, c.POINTER(c.c_int), c.POINTER(c.c_int)]
    lib.lwq_oracle_dequant_row.restype = c.c_int
    lib.lwq_oracle_dequant_row.argtypes = [c.c_int, c.c_void_p, c.c_long, c.c_void_p]
    lib.lwq_oracle_matmul.restype = c.c_int
    lib.lwq_oracle_matmul.argtypes = [c.c_int, c.c_int, c.c_void_p, c.c_void_p, c.c_long, c.c_long,
                                      c.c_long, c.c_void_p, c.c_void_p, c.c_int]
    lib.lwq_oracle_matmul_sampled.restype = c.c_int
    lib.lwq_oracle_matmul_sampled.argtypes = [c.c_int, c.c_int, c.c_void_p, c.c_void_p, c.c_long,
                                              c.c_long, c.c_long, c.c_void_p, c.c_void_p, c.c_long,
                                              c.c_void_p, c.c_void_p, c.c_int]
    lib.lwq_oracle_attention.restype = c.c_int
    lib.lwq_oracle_attention.argtypes = [c.c_int, c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_long, c.c_long,
                                         c.c_long, c.c_long, c.c_long, c.c_double, c.c_void_p, c.c_void_p]
    lib.lwq_oracle_max_threads.restype = c.c_int
    lib.lwq_oracle_max_threads.argtypes = []
    return lib


def load(path: str | None = None) -> ctypes.CDLL:
    """Load (building first if needed) the oracle library; ``path`` loads another build."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _act_of(x: np.ndarray, act: str | None) -> str:
    if act is not None:
        return act
    if x.dtype == np.float32:
        return "f32"
    if x.dtype == np.float16:
        return "f16"
    raise ValueError("uint16 activations are ambiguous: pass act='bf16' or 'f16'")


def f16(code: int, lib=None) -> float:
    return (lib or load()).lwq_oracle_f16(code)


def bf16(code: int, lib=None) -> float:
    return (lib or load()).lwq_oracle_bf16(code)


def row_bytes(fmt: str, K: int, lib=None) -> int:
    return (lib or load()).lwq_oracle_row_bytes(FMT[fmt], K)


def q4k_scale_min(scales12: np.ndarray, j: int, lib=None) -> tuple[int, int]:
    s = np.ascontiguousarray(scales12, dtype=np.uint8)
    assert s.size == 12
    sc, m = ctypes.c_int(), ctypes.c_int()
    (lib or load()).lwq_oracle_q4k_scale_min(_ptr(s), j, ctypes.byref(sc), ctypes.byref(m))
    return sc.value, m.value


def dequant(fmt: str, Wq: np.ndarray, K: int, lib=None) -> np.ndarray:
    """Decode packed rows [N][row_bytes] to fp32 [N][K]."""
    lib = lib or load()
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8)
    rb = lib.lwq_oracle_row_bytes(FMT[fmt], K)
    if rb < 0:
        raise ValueError(f"bad K={K} for {fmt}")
    Wq = Wq.reshape(-1, rb)
    out = np.empty((Wq.shape[0], K), dtype=np.float32)
    for n in range(Wq.shape[0]):
        rc = lib.lwq_oracle_dequant_row(FMT[fmt], _ptr(Wq[n]), K, _ptr(out[n]))
        if rc:
            raise ValueError("dequant failed")
    return out


def matmul(fmt: str, Wq: np.ndarray, x: np.ndarray, K: int | None = None, act: str | None = None,
           nthreads: int = 0, lib=None):
    """(y, den): fp64 [M][N] reference output and sum_k |x*w|."""
    lib = lib or load()
    act = _act_of(x, act)
    x = np.ascontiguousarray(x)
    M = x.shape[0]
    K = x.shape[1] if K is None else K
    rb = lib.lwq_oracle_row_bytes(FMT[fmt], K)
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8).reshape(-1, rb)
    N = Wq.shape[0]
    y = np.empty((M, N), dtype=np.float64)
    den = np.empty((M, N), dtype=np.float64)
    rc = lib.lwq_oracle_matmul(FMT[fmt], ACT[act], _ptr(Wq), _ptr(x), M, N, K, _ptr(y), _ptr(den), nthreads)
    if rc:
        raise ValueError("oracle matmul failed")
    return y, den


def matmul_sampled(fmt: str, Wq: np.ndarray, x: np.ndarray, ms, ns, K: int | None = None,
                   act: str | None = None, nthreads: int = 0, lib=None):
    """(y, den) fp64 for the listed outputs (ms[i], ns[i])."""
    lib = lib or load()
    act = _act_of(x, act)
    x = np.ascontiguousarray(x)
    M = x.shape[0]
    K = x.shape[1] if K is None else K
    rb = lib.lwq_oracle_row_bytes(FMT[fmt], K)
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8).reshape(-1, rb)
    N = Wq.shape[0]
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    y = np.empty(ms.shape[0], dtype=np.float64)
    den = np.empty(ms.shape[0], dtype=np.float64)
    rc = lib.lwq_oracle_matmul_sampled(FMT[fmt], ACT[act], _ptr(Wq), _ptr(x), M, N, K, _ptr(ms), _ptr(ns),
                                       ms.shape[0], _ptr(y), _ptr(den), nthreads)
    if rc:
        raise ValueError("oracle sampled matmul failed")
    return y, den


# ------------------------------------------------ int8 activations
# "Compute Shaders con WebGPU para Inferencia ML" lists quantized arithmetic
# without runtime dequantization among the reasons to write the kernels by hand,
# and its quantized matmul scales groups of 32.  The reading implemented here,
# and by the library under LWQ_FLAG_ACT_I8: each run of 32 activations along K
# of one row becomes int8 codes q with one fp32 scale d, and the matmul uses
# x_q = q * d in place of x.  Per block, in fp32 with round-to-nearest-even:
#   amax = max |x|;  if amax < 2^-100: d = 0 and q = 0;
#   else d = amax / 127, s = 127 / amax, q = rint(x * s) (clamped to +-127).
# 16-bit activations are first converted to fp32 (exactly).

ACT_Q8_BLOCK = 32
ACT_Q8_TINY = np.float32(2.0 ** -100)


def activations_f32(x: np.ndarray, act: str | None = None) -> np.ndarray:
    """Activations as fp32 (f16 and bf16 widen exactly)."""
    act = _act_of(x, act)
    x = np.ascontiguousarray(x)
    if act == "f32":
        return x.astype(np.float32, copy=False)
    if act == "f16":
        return x.view(np.float16).astype(np.float32)
    return (x.view(np.uint16).astype(np.uint32) << 16).view(np.float32)


def quantize_act_q8(x: np.ndarray, act: str | None = None):
    """(q, d): int8 codes [M][K] and fp32 scales [M][K/32] of the activations."""
    xf = activations_f32(x, act)
    M, K = xf.shape
    if K % ACT_Q8_BLOCK:
        raise ValueError("K must be a multiple of 32")
    blk = xf.reshape(M, K // ACT_Q8_BLOCK, ACT_Q8_BLOCK)
    amax = np.max(np.abs(blk), axis=2)
    tiny = amax < ACT_Q8_TINY
    safe = np.where(tiny, np.float32(1), amax)
    d = np.where(tiny, np.float32(0), amax / np.float32(127)).astype(np.float32)
    s = np.where(tiny, np.float32(0), np.float32(127) / safe).astype(np.float32)
    prod = (blk * s[:, :, None]).astype(np.float32)
    q = np.clip(np.rint(prod), -127, 127).astype(np.int8)
    return q.reshape(M, K), d


def matmul_q8act(fmt: str, Wq: np.ndarray, x: np.ndarray, K: int | None = None, act: str | None = None,
                 lib=None):
    """(y, den) in fp64 with the activations replaced by their int8 blocks:
    y[m,n] = sum_k w[n,k] * q[m,k] * d[m,k/32], den = sum_k |w * q * d|."""
    q, d = quantize_act_q8(x, act)
    M, Kx = q.shape
    K = Kx if K is None else K
    xq = q.astype(np.float64) * np.repeat(d.astype(np.float64), ACT_Q8_BLOCK, axis=1)
    W = dequant(fmt, Wq, K, lib=lib).astype(np.float64)
    return xq @ W.T, np.abs(xq) @ np.abs(W).T


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, lens, scale: float, act: str | None = None, lib=None):
    """Decode attention (see ``lwq_oracle_attention``): q [B][H][D], k/v [B][Hkv][Lmax][D] as fp16
    arrays or bf16 codes (uint16), lens [B].  Returns (out, den), fp64 [B][H][D]."""
    lib = lib or load()
    if act is None:
        act = "f16" if q.dtype == np.float16 else "bf16"
    B, H, D = q.shape
    Hkv, Lmax = k.shape[1], k.shape[2]
    lens = np.ascontiguousarray(np.asarray(lens, dtype=np.int32))
    q16 = np.ascontiguousarray(q).view(np.uint16)
    k16 = np.ascontiguousarray(k).view(np.uint16)
    v16 = np.ascontiguousarray(v).view(np.uint16)
    out = np.empty((B, H, D), dtype=np.float64)
    den = np.empty((B, H, D), dtype=np.float64)
    rc = lib.lwq_oracle_attention(ACT[act], _ptr(q16), _ptr(k16), _ptr(v16), _ptr(lens), B, H, Hkv, Lmax, D,
                                  float(scale), _ptr(out), _ptr(den))
    if rc:
        raise ValueError("bad attention arguments")
    return out, den


def max_threads(lib=None) -> int:
    return (lib or load()).lwq_oracle_max_threads()


def normalised_error(y_gpu: np.ndarray, y_ref: np.ndarray, den: np.ndarray) -> float:
    """max |y - y_ref| / den over all outputs; where den == 0 the output must be exactly 0.

    Returns +inf if any output with den == 0 is nonzero or any value is not finite.
    """
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    if not np.all(np.isfinite(y_gpu)):
        return float("inf")
    zero = den == 0
    if np.any(y_gpu[zero] != 0):
        return float("inf")
    if np.all(zero):
        return 0.0
    err = np.abs(y_gpu[~zero] - y_ref[~zero]) / den[~zero]
    return float(err.max()) if err.size else 0.0
