"""The GEMV carries activations exactly, whatever their spread, and a weight of
zero contributes exactly nothing.

* Outliers meeting zero weights: one activation of 2^30 (fp32, bf16; fp16:
  2^15) per 256-element chunk, at a position where every weight row holds a
  zero weight (Q4_0 nibble 8, Q8_0 code 0, Q4_K sub-block with scale and min
  0).  The normalised error |y - y_ref| / sum |x w| is then made of the other
  activations alone, so any rounding of the outlier, or any cancellation of
  it against an offset, shows at once.
* Mixed magnitudes inside a chunk: activations N(0,1) * 2^u with u drawn per
  element.
* den = 0: Q4_0 rows whose bytes are all 0x88 decode to zero weights; their
  outputs must be exactly 0 on every path (GEMV one row and several rows,
  split-K, prefill GEMM, simple kernel).
* 24 significant bits: with weights +-d (d a power of two) and one nonzero
  activation per row, every output is an exact fp32 product; the GPU must
  return it bit for bit, which a 22-bit activation would not.
"""

import numpy as np
import pytest
import torch

import block_quantized_matmul_lwq_b200 as lwq
import oracle
from block_quantized_matmul_lwq_b200 import inputs
from gpu_util import TOL_GEMM, TOL_GEMV, run_gpu

pytestmark = pytest.mark.gpu

WS_BYTES = 64 << 20


@pytest.fixture(scope="module")
def dev():
    d = torch.device("cuda:0")
    torch.cuda.set_device(d)
    ws = torch.zeros(WS_BYTES, dtype=torch.uint8, device=d)
    lwq.lwq_init(ws, WS_BYTES)
    yield d
    torch.cuda.synchronize(d)
    assert lwq.lwq_get_device_error() == lwq.LWQ_OK
    lwq.lwq_shutdown()
    del ws


def _x_store(v: np.ndarray, a: str) -> np.ndarray:
    """fp32 activations as stored for activation type a (round to nearest even)."""
    if a == "f32":
        return v.astype(np.float32)
    if a == "f16":
        return v.astype(np.float16).view(np.uint16)
    u = v.astype(np.float32).view(np.uint32)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def _zero_weights_at(w: str, Wq: np.ndarray, K: int, cols: list[int]) -> np.ndarray:
    """Make the weight of every row at element positions `cols` exactly zero."""
    Wq = Wq.copy()
    N = Wq.shape[0]
    if w == "q4_0":
        blk = Wq.reshape(N, K // 32, 18)
        for k in cols:
            b, i = divmod(k, 32)
            byte = 2 + (i % 16)
            if i < 16:
                blk[:, b, byte] = (blk[:, b, byte] & 0xF0) | 0x08
            else:
                blk[:, b, byte] = (blk[:, b, byte] & 0x0F) | 0x80
    elif w == "q8_0":
        blk = Wq.reshape(N, K // 32, 34)
        for k in cols:
            b, i = divmod(k, 32)
            blk[:, b, 2 + i] = 0
    else:
        # Q4_K: the sub-block holding k gets scale 0 and min 0 (all its weights are zero)
        blk = Wq.reshape(N, K // 256, 144)
        for k in cols:
            sb, r = divmod(k, 256)
            j = r // 32
            s = blk[:, sb, 4:16]
            if j < 4:
                s[:, j] &= 0xC0          # sc_j = s[j] & 63
                s[:, j + 4] &= 0xC0      # m_j = s[j+4] & 63
            else:
                s[:, j + 4] = 0          # low nibbles of sc_j and m_j
                s[:, j - 4] &= 0x3F      # high bits of sc_j
                s[:, j] &= 0x3F          # high bits of m_j
            blk[:, sb, 4:16] = s
    return Wq


def _outlier_problem(w, a, M, N, K, seed):
    g = inputs.rng(seed)
    Wq = inputs.make_weights(w, g, N, K)
    v = g.standard_normal((M, K), dtype=np.float32)
    big = np.float32(2.0 ** 15 if a == "f16" else 2.0 ** 30)
    cols = [c * 256 + int(g.integers(0, 256)) for c in range(K // 256)]
    for k in cols:
        v[:, k] = big * np.where(g.random(M) < 0.5, -1, 1).astype(np.float32)
    return _zero_weights_at(w, Wq, K, cols), _x_store(v, a)


def _check(w, a, Wq, x, M, N, K, dev, tol, cfg=None):
    y = run_gpu(w, a, Wq, x, M, N, K, dev, cfg=cfg).cpu().numpy()
    y_ref, den = oracle.matmul(w, Wq, x, act=a)
    err = oracle.normalised_error(y, y_ref, den)
    assert err <= tol, f"{w}/{a} M={M} N={N} K={K}: err {err:.3e} > {tol}"
    return err


@pytest.mark.parametrize("w", ["q4_0", "q8_0", "q4_k"])
@pytest.mark.parametrize("a", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("M", [1, 4, 8, 16])
def test_outliers_at_zero_weights(dev, w, a, M):
    N, K = 200, 4096
    Wq, x = _outlier_problem(w, a, M, N, K, seed=M * 31 + len(w) + len(a))
    _check(w, a, Wq, x, M, N, K, dev, TOL_GEMV)


@pytest.mark.parametrize("w,a", [("q4_0", "bf16"), ("q4_0", "f16"), ("q8_0", "bf16"), ("q4_k", "f16")])
def test_outliers_at_zero_weights_prefill(dev, w, a):
    """The tcgen05 GEMM (weights rounded once to bf16/fp16; zero stays zero)."""
    M, N, K = 48, 256, 4096
    Wq, x = _outlier_problem(w, a, M, N, K, seed=5)
    assert lwq.lwq_select_config(lwq.fmt_code(w, a), M, N, K).path == 2
    _check(w, a, Wq, x, M, N, K, dev, TOL_GEMM)


@pytest.mark.parametrize("w", ["q4_0", "q8_0", "q4_k"])
@pytest.mark.parametrize("a,span", [("f32", 40), ("bf16", 60), ("f16", 12)])
@pytest.mark.parametrize("M", [1, 3, 8])
def test_mixed_magnitudes_in_chunk(dev, w, a, span, M):
    N, K = 150, 2048
    g = inputs.rng(100 + M + span)
    Wq = inputs.make_weights(w, g, N, K)
    v = g.standard_normal((M, K), dtype=np.float32) * np.exp2(g.integers(-span, span + 1, (M, K))).astype(np.float32)
    _check(w, a, Wq, _x_store(v, a), M, N, K, dev, TOL_GEMV)


@pytest.mark.parametrize("a,e", [("f32", -110), ("f32", 100), ("bf16", -110), ("bf16", 100)])
@pytest.mark.parametrize("M", [1, 8])
def test_extreme_scales(dev, a, e, M):
    """Activations scaled far outside [2^-60, 2^60] take the power-of-two rescale of the warp's slice."""
    w, N, K = "q4_0", 64, 1024
    g = inputs.rng(7 + M)
    Wq = inputs.make_weights(w, g, N, K)
    v = g.standard_normal((M, K), dtype=np.float32) * np.float32(2.0 ** e)
    _check(w, a, Wq, _x_store(v, a), M, N, K, dev, TOL_GEMV)


@pytest.mark.parametrize("case", ["one_row", "rows4_f32", "rows8_f32", "rows16_f16", "split_k", "gemm", "simple"])
def test_den_zero_rows_are_exactly_zero(dev, case):
    """Q4_0 rows of all-0x88 bytes (any d) give y == 0 exactly; the other rows match the oracle."""
    a, M, N, K = {"one_row": ("f32", 1, 300, 4096), "rows4_f32": ("f32", 4, 300, 4096),
                  "rows8_f32": ("f32", 8, 300, 4096), "rows16_f16": ("f16", 16, 300, 4096),
                  "split_k": ("bf16", 2, 300, 11008), "gemm": ("bf16", 64, 300, 4096),
                  "simple": ("f32", 3, 300, 96)}[case]
    g = inputs.rng(len(case))
    Wq = inputs.make_weights("q4_0", g, N, K)
    zero_rows = np.arange(0, N, 3)
    blk = Wq.reshape(N, K // 32, 18)
    blk[zero_rows, :, 2:] = 0x88
    x = inputs.activations(g, M, K, a)
    cfg = lwq.lwq_select_config(lwq.fmt_code("q4_0", a), M, N, K)
    expect_path = {"gemm": 2, "simple": 3}.get(case, 1)
    assert cfg.path == expect_path
    if case == "split_k":
        assert cfg.splits > 1
    y = run_gpu("q4_0", a, Wq, x, M, N, K, dev).cpu().numpy()
    assert np.all(y[:, zero_rows] == 0.0), "a row of zero weights gave a nonzero output"
    y_ref, den = oracle.matmul("q4_0", Wq, x, act=a)
    assert np.all(den[:, zero_rows] == 0.0)
    keep = np.setdiff1d(np.arange(N), zero_rows)
    tol = TOL_GEMM if cfg.path == 2 else TOL_GEMV
    assert oracle.normalised_error(y[:, keep], y_ref[:, keep], den[:, keep]) <= tol


def _pm_one_weights(w, g, N, K, log2d):
    """Packed weights equal to +-2^log2d: Q4_0 nibbles 7 or 9, Q8_0 codes -1 or 1; d = 2^log2d."""
    d16 = np.float16(2.0 ** log2d).view(np.uint16)
    sgn = g.random((N, K)) < 0.5
    if w == "q4_0":
        q = np.where(sgn, 7, 9).astype(np.uint8).reshape(N, K // 32, 32)
        blk = np.empty((N, K // 32, 18), dtype=np.uint8)
        blk[..., 0] = d16 & 0xFF
        blk[..., 1] = d16 >> 8
        blk[..., 2:] = q[..., :16] | (q[..., 16:] << 4)
    else:
        q = np.where(sgn, -1, 1).astype(np.int8).reshape(N, K // 32, 32)
        blk = np.empty((N, K // 32, 34), dtype=np.uint8)
        blk[..., 0] = d16 & 0xFF
        blk[..., 1] = d16 >> 8
        blk[..., 2:] = q.view(np.uint8)
    return blk.reshape(N, -1)


@pytest.mark.parametrize("w", ["q4_0", "q8_0"])
@pytest.mark.parametrize("a", ["f32", "bf16"])
@pytest.mark.parametrize("M", [1, 2, 5, 8])
def test_every_activation_bit_reaches_the_product(dev, w, a, M):
    """One nonzero activation per row, weights +-2^-3: each output is the exact fp32 product
    w * x, which needs every significand bit of x (24 for fp32) -- returned bit for bit."""
    N, K = 96, 2048
    g = inputs.rng(300 + M)
    Wq = _pm_one_weights(w, g, N, K, -3)
    bits = g.integers(0, 1 << 23, M).astype(np.uint32) | np.uint32(0x3F800001)   # [1, 2), low bit set
    v = np.zeros((M, K), dtype=np.float32)
    ks = g.integers(0, K, M)
    v[np.arange(M), ks] = bits.view(np.float32) * np.float32(2.0 ** 20) * np.where(g.random(M) < 0.5, -1, 1)
    x = _x_store(v, a)
    y = run_gpu(w, a, Wq, x, M, N, K, dev).cpu().numpy()
    y_ref, den = oracle.matmul(w, Wq, x, act=a)
    assert np.array_equal(y, y_ref.astype(np.float32)), "an output differs from the exact product"
    assert np.array_equal(y_ref.astype(np.float32).astype(np.float64), y_ref)   # the products are exact in fp32
