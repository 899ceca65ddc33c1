"""Decode attention on the GPU against the oracle (element by element).

Error measure: |out - out_ref| / den with den = sum_j p_j |v_j| / sum_j p_j,
the oracle's softmax weights p (fp64); the bound 1e-4 covers fp32 dot
products and exponentials (about 1e-6 is typical).
"""

import numpy as np
import pytest
import torch

import block_quantized_matmul_lwq_b200 as lwq
import oracle
from block_quantized_matmul_lwq_b200 import inputs
from gpu_util import to_device

pytestmark = pytest.mark.gpu

TOL_ATTN = 1e-4
WS_BYTES = 64 << 20


_ARENA = []   # the registered workspace, kept alive for the module


@pytest.fixture(scope="module")
def dev():
    d = torch.device("cuda:0")
    torch.cuda.set_device(d)
    _ARENA.append(torch.zeros(WS_BYTES, dtype=torch.uint8, device=d))
    lwq.lwq_init(_ARENA[0], WS_BYTES)
    yield d
    torch.cuda.synchronize(d)
    lwq.lwq_shutdown()
    _ARENA.clear()


def run(dev, act, q, k, v, lens, scale, pass_lens=True):
    B, H, D = q.shape
    Hkv, Lmax = k.shape[1], k.shape[2]
    qd, kd, vd = to_device(q, dev), to_device(k, dev), to_device(v, dev)
    ld = torch.from_numpy(np.asarray(lens, dtype=np.int32)).to(dev) if pass_lens else None
    out = torch.full((B, H, D), float("nan"), dtype=torch.float32, device=dev)
    code = lwq.LWQ_ACT_F16 if act == "f16" else lwq.LWQ_ACT_BF16
    lwq.lwq_attention_decode(code, qd, kd, vd, ld, out, B, H, Hkv, Lmax, D, scale)
    torch.cuda.synchronize(dev)
    return out.cpu().numpy()


def check(dev, act, B, H, Hkv, Lmax, D, lens=None, seed=0, scale=None, pass_lens=True):
    q, k, v, lens = inputs.attention_problem(B, H, Hkv, Lmax, D, act, seed=seed, lens=lens)
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    out = run(dev, act, q, k, v, lens, scale, pass_lens)
    clamped = np.clip(lens, 1, Lmax)
    ref, den = oracle.attention(q, k, v, clamped, scale, act=act)
    assert np.all(np.isfinite(out))
    err = float(np.max(np.abs(out - ref) / den))
    assert err <= TOL_ATTN, f"B={B} H={H} Hkv={Hkv} L={Lmax} D={D} {act}: {err:.3e}"
    return out


@pytest.mark.parametrize("act", ["f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("H,Hkv", [(4, 4), (8, 4), (8, 2), (16, 2)])
@pytest.mark.parametrize("Lmax", [1, 7, 33, 300])
def test_small(dev, act, D, H, Hkv, Lmax):
    check(dev, act, 2, H, Hkv, Lmax, D, seed=Lmax + H)


@pytest.mark.parametrize("act", ["f16", "bf16"])
def test_ragged_lengths(dev, act):
    """Sequences of different lengths in one call: 1, a partial 4-key group, a split edge, the maximum."""
    check(dev, act, 6, 8, 2, 2000, 128, lens=[1, 3, 255, 256, 1999, 2000], seed=3)


def test_lengths_clamped(dev):
    """A length of 0 counts as 1 and one beyond Lmax as Lmax (no read outside the cache)."""
    check(dev, "f16", 3, 4, 4, 64, 64, lens=[0, 65, 10], seed=4)


def test_null_lengths_mean_full_cache(dev):
    check(dev, "bf16", 2, 8, 8, 700, 128, seed=5, pass_lens=False)


def test_page_shape(dev):
    """The pages' example: 512 tokens, 12 heads, head dimension 64."""
    check(dev, "f16", 1, 12, 12, 512, 64, seed=6)


@pytest.mark.parametrize("B,H,Hkv,L", [(4, 32, 32, 4096), (2, 32, 4, 8192), (16, 32, 8, 1024)])
def test_7b_decode_shapes(dev, B, H, Hkv, L):
    """Llama-7B-shaped decode batches (head dimension 128, multi-head and grouped), split over CTAs."""
    check(dev, "f16", B, H, Hkv, L, 128, seed=B + L)


def test_large_scores_do_not_overflow(dev):
    """Scores of several hundred: the running maximum keeps every exponential finite."""
    check(dev, "f16", 1, 4, 4, 300, 64, seed=7, scale=8.0)


def test_deterministic(dev):
    q, k, v, lens = inputs.attention_problem(3, 16, 4, 3000, 128, "bf16", seed=8)
    a = run(dev, "bf16", q, k, v, lens, 0.09)
    b = run(dev, "bf16", q, k, v, lens, 0.09)
    np.testing.assert_array_equal(a, b)


def test_argument_errors(dev):
    buf = torch.zeros(1 << 16, dtype=torch.float32, device=dev)
    p = buf.data_ptr()
    f = lwq.lib().lwq_attention_decode
    assert f(lwq.LWQ_ACT_F16, p, p, p, None, p, 1, 4, 4, 16, 96, 0.1, None) == lwq.LWQ_ERR_UNSUPPORTED   # D
    assert f(lwq.LWQ_ACT_F16, p, p, p, None, p, 1, 12, 4, 16, 64, 0.1, None) == lwq.LWQ_ERR_UNSUPPORTED  # G = 3
    assert f(lwq.LWQ_ACT_F16, p, p, p, None, p, 1, 6, 4, 16, 64, 0.1, None) == lwq.LWQ_ERR_INVALID_ARG   # H % Hkv
    assert f(lwq.LWQ_ACT_F32, p, p, p, None, p, 1, 4, 4, 16, 64, 0.1, None) == lwq.LWQ_ERR_UNSUPPORTED   # dtype
    assert f(lwq.LWQ_ACT_F16, p + 8, p, p, None, p, 1, 4, 4, 16, 64, 0.1, None) == lwq.LWQ_ERR_MISALIGNED
    assert f(lwq.LWQ_ACT_F16, p, p, p, None, p, 0, 4, 4, 16, 64, 0.1, None) == lwq.LWQ_ERR_INVALID_ARG
    assert f(lwq.LWQ_ACT_F16, p, p, p, None, p, 1, 4, 4, 16, 64, float("inf"), None) == lwq.LWQ_ERR_INVALID_ARG
    torch.cuda.synchronize(dev)


def test_workspace_needed_for_splits(dev):
    """A long sequence is split; without a large enough workspace the call is refused, not run."""
    B, H, Hkv, L, D = 1, 8, 8, 16384, 128
    need = lwq.lwq_attention_workspace_size(B, H, Hkv, L, D)
    assert need > 0
    small = torch.zeros(256, dtype=torch.uint8, device=dev)
    lwq.lwq_init(small, 256)
    try:
        buf = torch.zeros(B * Hkv * L * D, dtype=torch.float16, device=dev)
        out = torch.zeros(B * H * D, dtype=torch.float32, device=dev)
        rc = lwq.lib().lwq_attention_decode(lwq.LWQ_ACT_F16, buf.data_ptr(), buf.data_ptr(), buf.data_ptr(), None,
                                            out.data_ptr(), B, H, Hkv, L, D, 0.1, None)
        assert rc == lwq.LWQ_ERR_WORKSPACE_TOO_SMALL
    finally:
        lwq.lwq_init(_ARENA[0], WS_BYTES)
