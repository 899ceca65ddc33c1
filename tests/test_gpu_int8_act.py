"""GPU parity of the int8-activation GEMV (LWQ_FLAG_ACT_I8; Q4_0, Q8_0 and Q4_K weights)
against the oracle's definition (oracle.quantize_act_q8 / matmul_q8act).

The activation codes are integer decisions taken in fp32 on both sides with the
same operations, so they must agree exactly; what remains is fp32 rounding of
the per-block scale products and of the sums: TOL_I8 = 1e-5 of sum |x_q w|
(the kernel's sums run over at most 8 blocks per warp, 16 warps and the splits,
a few tens of fp32 roundings of 2^-24 each).
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import block_quantized_matmul_lwq_b200 as lwq
import oracle
from block_quantized_matmul_lwq_b200 import inputs
from gpu_util import run_gpu, to_device

pytestmark = pytest.mark.gpu

TOL_I8 = 1e-5
WS_BYTES = 64 << 20


@pytest.fixture(scope="module")
def dev():
    d = torch.device("cuda", 0)
    ws = torch.zeros(WS_BYTES, dtype=torch.uint8, device=d)
    lwq.lwq_init(ws, WS_BYTES)
    yield d
    torch.cuda.synchronize(d)
    assert lwq.lwq_get_device_error() == lwq.LWQ_OK


def run_i8(a, Wq, x, M, N, K, dev, noalloc=False, w="q4_0"):
    fmt = lwq.fmt_code(w, a) | lwq.LWQ_FLAG_ACT_I8
    Wd, xd = to_device(Wq, dev), to_device(x, dev)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
    if noalloc:
        lwq.lwq_matmul_noalloc(fmt, Wd, xd, y, M, N, K)
    else:
        lwq.lwq_matmul(fmt, Wd, xd, y, M, N, K)
    torch.cuda.synchronize(dev)
    return y.cpu().numpy()


def check(a, M, N, K, dev, seed, noalloc=False, x=None, w="q4_0"):
    Wq, x0 = inputs.make_problem(w, a, M, N, K, seed=seed)
    x = x0 if x is None else x
    y = run_i8(a, Wq, x, M, N, K, dev, noalloc=noalloc, w=w)
    y_ref, den = oracle.matmul_q8act(w, Wq, x, act=a)
    err = oracle.normalised_error(y, y_ref, den)
    assert err <= TOL_I8, f"{a} M={M} N={N} K={K}: err {err:.3e} > {TOL_I8}"
    return y, Wq, x


@pytest.mark.parametrize("w", ["q4_0", "q8_0", "q4_k"])
@pytest.mark.parametrize("a", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("M,N,K", [(1, 211, 3072), (2, 1000, 4096), (5, 47, 11008), (8, 300, 4096),
                                   (9, 130, 2048), (16, 64, 4352)])
def test_parity(dev, w, a, M, N, K):
    check(a, M, N, K, dev, seed=M * 31 + K, w=w)


@pytest.mark.parametrize("w", ["q4_0", "q8_0", "q4_k"])
@pytest.mark.parametrize("M", [17, 40, 130])
def test_many_rows_in_passes(dev, w, M):
    """M > 16: passes of 8 activation rows, each streaming the weights."""
    check("bf16", M, 300, 2048, dev, seed=M, w=w)


def test_q8_0_gemv_4096x4096(dev):
    """Q8_0 4096 x 4096 at M = 1 with int8 activation blocks, every output."""
    check("f32", 1, 4096, 4096, dev, seed=0, w="q8_0")


def test_q4_k_7b_layer_shapes(dev):
    """Q4_K at the 7B layer's three shapes, fp16 activations as int8 blocks, every output (split-K at K = 11008)."""
    for N, K in ((4096, 4096), (11008, 4096), (4096, 11008)):
        check("f16", 1, N, K, dev, seed=N + K, w="q4_k")


def test_headline_shape_against_exact_product(dev):
    # Q4_0 11008 x 4096 at M = 8: parity with the int8 definition, and within 1e-2 of the exact product
    M, N, K = 8, 11008, 4096
    y, Wq, x = check("f32", M, N, K, dev, seed=0)
    y_exact, den = oracle.matmul("q4_0", Wq, x)
    assert oracle.normalised_error(y, y_exact, den) < 1e-2


def test_zero_and_extreme_blocks(dev):
    M, N, K = 3, 70, 1024
    Wq, x = inputs.make_problem("q4_0", "f32", M, N, K, seed=4)
    x = x.copy()
    x[0] = 0.0                                  # all-zero row: y exactly 0
    x[1, 100:132] = 0.0
    x[1, 96] = 3.0e4                            # one block ruled by a large value
    x[2, :32] = np.float32(2.0 ** -101)         # a block below 2^-100 quantizes to zero
    y, _, _ = check("f32", M, N, K, dev, seed=4, x=x)
    assert (y[0] == 0).all()


def test_noalloc_and_deterministic(dev):
    M, N, K = 4, 500, 4096
    Wq, x = inputs.make_problem("q4_0", "bf16", M, N, K, seed=8)
    ys = [run_i8("bf16", Wq, x, M, N, K, dev) for _ in range(2)]
    ys.append(run_i8("bf16", Wq, x, M, N, K, dev, noalloc=True))
    assert np.array_equal(ys[0], ys[1]) and np.array_equal(ys[0], ys[2])
    y_ref, den = oracle.matmul_q8act("q4_0", Wq, x, act="bf16")
    assert oracle.normalised_error(ys[0], y_ref, den) <= TOL_I8


@pytest.mark.parametrize("w,M,K", [("q2_k", 1, 4096), ("q5_k", 1, 4096), ("q6_k", 1, 4096), ("q4_0", 1, 288)])
def test_unsupported(dev, w, M, K):
    fmt = lwq.fmt_code(w, "f16") | lwq.LWQ_FLAG_ACT_I8
    N = 64
    Wd = torch.zeros(N * lwq.lwq_row_bytes(fmt, K), dtype=torch.uint8, device=dev)
    xd = torch.zeros((M, K), dtype=torch.float16, device=dev)
    y = torch.zeros((M, N), dtype=torch.float32, device=dev)
    with pytest.raises(lwq.LwqError) as e:
        lwq.lwq_matmul(fmt, Wd, xd, y, M, N, K)
    assert e.value.status == lwq.LWQ_ERR_UNSUPPORTED
