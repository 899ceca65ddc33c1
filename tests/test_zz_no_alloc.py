"""lwq_matmul_noalloc: the decode GEMV for callers that cannot allocate.

Such callers (code that may not call the CUDA allocator, fixed memory pools,
plugins that receive only input and output pointers) cannot provide the
workspace that lwq_matmul's split-K needs, so this entry point keeps its
scratch in a static device array.  These tests call it through the C ABI and
check its outputs against lwq_matmul's on the same inputs and against the
oracle, for two calls in a row.  This file is collected last on purpose.
"""

import numpy as np
import pytest
import torch

import block_quantized_matmul_lwq_b200 as lwq
import oracle
from block_quantized_matmul_lwq_b200 import inputs
from gpu_util import TOL_GEMV, to_device

pytestmark = pytest.mark.gpu

CASES = [("q4_k", "f16", 1, 4096, 11008),    # split-K
         ("q4_0", "f32", 4, 11008, 4096),    # two column tiles
         ("q8_0", "f32", 1, 4096, 4096),
         ("q4_0", "bf16", 16, 333, 6144),    # 16 activation rows, split-K, ragged N
         ("q6_k", "f16", 2, 500, 8192),      # per-superblock boxes, split-K
         ("q5_k", "bf16", 3, 300, 4096),
         ("q6_k", "bf16", 2, 96, 11008),     # row slots (9030-byte rows), split-K
         ("q2_k", "f32", 3, 120, 11008)]     # row slots (3612-byte rows)


@pytest.fixture(scope="module")
def dev():
    d = torch.device("cuda:0")
    torch.cuda.set_device(d)
    return d


def _run_both(dev, w, a, M, N, K, seed):
    fmt = lwq.fmt_code(w, a)
    Wq, x = inputs.make_problem(w, a, M, N, K, seed=seed)
    Wd, xd = to_device(Wq, dev), to_device(x, dev)
    ws_bytes = lwq.lwq_workspace_size(fmt, M, N, K)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    lwq.lwq_init(ws, ws_bytes)
    y_ref = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
    lwq.lwq_matmul(fmt, Wd, xd, y_ref, M, N, K)
    outs = []
    for _ in range(2):  # two calls in a row share the static scratch
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
        rc = lwq.lib().lwq_matmul_noalloc(fmt, Wd.data_ptr(), xd.data_ptr(), y.data_ptr(), M, N, K, None)
        assert rc == lwq.LWQ_OK, lwq.lwq_status_string(rc)
        outs.append(y)
    torch.cuda.synchronize(dev)
    lwq.lwq_shutdown()
    y_oracle, den = oracle.matmul(w, Wq, x, act=a)
    ref = y_ref.cpu().numpy()
    for y in outs:
        got = y.cpu().numpy()
        # against the existing entry point's output on the same inputs ...
        err = oracle.normalised_error(got, ref.astype(np.float64), den)
        assert err <= TOL_GEMV, f"{w}/{a} M={M} N={N} K={K}: {err:.3e} against lwq_matmul"
        # ... and against the oracle itself
        err = oracle.normalised_error(got, y_oracle, den)
        assert err <= TOL_GEMV, f"{w}/{a} M={M} N={N} K={K}: {err:.3e} against the oracle"
    return ref, [y.cpu().numpy() for y in outs]


@pytest.mark.parametrize("w,a,M,N,K", CASES)
def test_noalloc_matches_lwq_matmul(dev, w, a, M, N, K):
    _run_both(dev, w, a, M, N, K, seed=N + M)


def test_noalloc_back_to_back_shapes(dev):
    """Different shapes one after another share the scratch array and both stay correct."""
    for w, a, M, N, K in CASES[::-1]:
        _run_both(dev, w, a, M, N, K, seed=K)


def test_noalloc_rejects_oversize_and_other_paths(dev):
    fmt = lwq.fmt_code("q4_0", "f16")
    buf = torch.zeros(64, dtype=torch.float32, device=dev)
    p = buf.data_ptr()
    # split-K scratch beyond the 4 MiB array: 16 rows x 32000 x K=14336 (14 splits) needs ~29 MB
    rc = lwq.lib().lwq_matmul_noalloc(fmt, p, p, p, 16, 32000, 14336, None)
    assert rc == 5, lwq.lwq_status_string(rc)
    # prefill shapes are not offered here
    rc = lwq.lib().lwq_matmul_noalloc(fmt, p, p, p, 64, 4096, 4096, None)
    assert rc == 2, lwq.lwq_status_string(rc)
    rc = lwq.lib().lwq_matmul_noalloc(fmt, p + 2, p, p, 1, 4096, 4096, None)
    assert rc == 3
