"""Helpers shared by the GPU tests: run one problem through the C ABI and
score it against the oracle on the same seeded inputs."""

from __future__ import annotations

import numpy as np
import torch

import block_quantized_matmul_lwq_b200 as lwq
import oracle
from block_quantized_matmul_lwq_b200 import inputs

TOL_GEMV = 1e-4   # tensor-core GEMV and simple GEMV (exact 16-bit products, fp32 sums)
TOL_GEMM = 5e-3   # tcgen05 GEMM (weights rounded once to bf16/fp16)


def to_device(a: np.ndarray, dev) -> torch.Tensor:
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def tolerance(fmt: int, M: int, N: int, K: int) -> float:
    return TOL_GEMM if lwq.lwq_select_config(fmt, M, N, K).path == 2 else TOL_GEMV


def run_gpu(w: str, a: str, Wq: np.ndarray, x: np.ndarray, M: int, N: int, K: int, dev, cfg=None,
            y: torch.Tensor | None = None) -> torch.Tensor:
    fmt = lwq.fmt_code(w, a)
    Wd, xd = to_device(Wq, dev), to_device(x, dev)
    if y is None:
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
    if cfg is None:
        lwq.lwq_matmul(fmt, Wd, xd, y, M, N, K)
    else:
        lwq.lwq_matmul_config(fmt, Wd, xd, y, M, N, K, cfg)
    torch.cuda.synchronize(dev)
    return y


def check_full(w, a, M, N, K, dev, seed=0, cfg=None, tol=None):
    Wq, x = inputs.make_problem(w, a, M, N, K, seed=seed)
    y = run_gpu(w, a, Wq, x, M, N, K, dev, cfg=cfg).cpu().numpy()
    y_ref, den = oracle.matmul(w, Wq, x, act=a)
    err = oracle.normalised_error(y, y_ref, den)
    if tol is None:
        tol = tolerance(lwq.fmt_code(w, a), M, N, K)
    assert err <= tol, f"{w}/{a} M={M} N={N} K={K} cfg={cfg and cfg.as_dict()}: err {err:.3e} > {tol}"
    return err


def sample_indices(M, N, count, seed):
    g = np.random.default_rng(seed)
    ms = list(g.integers(0, M, count))
    ns = list(g.integers(0, N, count))
    # every activation row at the first, last and tile-edge weight rows
    for m in range(M):
        for n in (0, 1, 15, 16, N // 2, N - 17, N - 16, N - 1):
            if 0 <= n < N:
                ms.append(m)
                ns.append(n)
    return np.array(ms), np.array(ns)


def check_sampled(w, a, M, N, K, dev, seed=0, count=2000, tol=None, Wq=None, x=None):
    if Wq is None:
        Wq, x = inputs.make_problem(w, a, M, N, K, seed=seed)
    y = run_gpu(w, a, Wq, x, M, N, K, dev).cpu().numpy()
    assert np.all(np.isfinite(y)), "non-finite output"
    ms, ns = sample_indices(M, N, count, seed + 1)
    y_ref, den = oracle.matmul_sampled(w, Wq, x, ms, ns, act=a)
    err = oracle.normalised_error(y[ms, ns], y_ref, den)
    if tol is None:
        tol = tolerance(lwq.fmt_code(w, a), M, N, K)
    assert err <= tol, f"{w}/{a} M={M} N={N} K={K} sampled: err {err:.3e} > {tol}"
    return err, y
