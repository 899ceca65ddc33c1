"""GPU path vs the CPU oracle, element by element, on the same seeded inputs.

Small cases span several row tiles, K chunks and split-K slices and end in
ragged tails; the full workload sizes are checked on sampled outputs (plus
every tile edge) in the configuration the benchmark times.
"""

import ctypes
import functools

import numpy as np
import pytest
import torch

import block_quantized_matmul_lwq_b200 as lwq
import oracle
from block_quantized_matmul_lwq_b200 import inputs
from gpu_util import TOL_GEMV, check_full, check_sampled, run_gpu, to_device

pytestmark = pytest.mark.gpu

WS_BYTES = 256 << 20


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


# every weight format with every activation type (all take the tensor-core GEMV when K % 256 == 0)
FAST = [(w, a) for w in ("q4_0", "q8_0", "q4_k") for a in ("f32", "f16", "bf16")]


@pytest.mark.parametrize("w,a", FAST)
@pytest.mark.parametrize("M,N,K", [(1, 1, 256), (1, 37, 512), (3, 100, 1024), (8, 333, 4096), (5, 61, 2816),
                                   (16, 50, 768), (12, 130, 4352), (1, 17, 6144)])
def test_small_shapes(dev, w, a, M, N, K):
    check_full(w, a, M, N, K, dev, seed=M * 1000 + N)


@pytest.mark.parametrize("w,a", FAST)
@pytest.mark.parametrize("M", [2, 3, 4, 5, 6, 7, 8, 9, 15, 16])
def test_every_column_layout(dev, w, a, M):
    # row counts at and around the boundaries of the GEMV's column layouts (fp32: 3 parts per
    # row, so 1, 2 and 3 tiles of 8 columns at M <= 2, 5 and 8; 16-bit: 8 rows per tile)
    check_full(w, a, M, 45, 1024, dev, seed=100 + M)


def _scaled_problem(w, a, M, N, K, seed, e):
    """make_problem with the activations multiplied by 2**e (exact in every activation type)."""
    Wq, x = inputs.make_problem(w, a, M, N, K, seed=seed)
    if a == "f32":
        return Wq, (x * np.float32(2.0 ** e)).astype(np.float32)
    if a == "f16":
        v = x.view(np.float16).astype(np.float32) * np.float32(2.0 ** e)
        assert np.all(np.isfinite(v.astype(np.float16)))
        return Wq, v.astype(np.float16).view(np.uint16)
    v = (x.astype(np.uint32) << 16).view(np.float32) * np.float32(2.0 ** e)
    return Wq, (v.view(np.uint32) >> 16).astype(np.uint16)


@pytest.mark.parametrize("w,a,e", [("q4_0", "f32", -40), ("q4_0", "f32", 40), ("q4_0", "f16", -12),
                                   ("q4_0", "f16", 12), ("q8_0", "f16", -12), ("q4_k", "f16", 12),
                                   ("q4_0", "bf16", -60), ("q8_0", "f32", 30)])
@pytest.mark.parametrize("M", [1, 3, 8])
def test_activation_magnitudes(dev, w, a, e, M):
    # the per-warp power-of-two activation scale must hold tiny and huge inputs
    N, K = 40, 1024
    Wq, x = _scaled_problem(w, a, M, N, K, 11 + M, e)
    y = run_gpu(w, a, Wq, x, M, N, K, dev).cpu().numpy()
    y_ref, den = oracle.matmul(w, Wq, x, act=a)
    err = oracle.normalised_error(y, y_ref, den)
    assert err <= TOL_GEMV, f"{w}/{a} x*2^{e} M={M}: err {err:.3e}"


@pytest.mark.parametrize("w,a", [("q4_0", "f32"), ("q8_0", "f16"), ("q4_0", "bf16")])
@pytest.mark.parametrize("M,N,K", [(1, 9, 32), (2, 40, 96), (4, 7, 320), (17, 33, 480)])
def test_k_not_multiple_of_256(dev, w, a, M, N, K):
    check_full(w, a, M, N, K, dev, seed=7)


@pytest.mark.parametrize("w,a", FAST)
@pytest.mark.parametrize("M", [20, 33])
def test_many_activation_rows(dev, w, a, M):
    check_full(w, a, M, 70, 1024, dev, seed=M)


@pytest.mark.parametrize("w,a", FAST)
@pytest.mark.parametrize("warps,splits,stages", [(1, 0, 2), (2, 0, 3), (4, 3, 2), (8, 2, 4), (3, 4, 2)])
def test_forced_gemv_configs(dev, w, a, warps, splits, stages):
    cfg = lwq.lwq_config()
    cfg.path, cfg.warps, cfg.splits, cfg.stages = 1, warps, splits, stages
    M, N, K = 5, 211, 3072
    Wq, x = inputs.make_problem(w, a, M, N, K, seed=11)
    Wd, xd = to_device(Wq, dev), to_device(x, dev)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
    rc = lwq.lib().lwq_matmul_config(lwq.fmt_code(w, a), Wd.data_ptr(), xd.data_ptr(), y.data_ptr(), M, N, K,
                                     ctypes.byref(cfg), None)
    if rc == lwq.LWQ_ERR_UNSUPPORTED:
        pytest.skip("configuration leaves a chunk without a warp")
    assert rc == lwq.LWQ_OK, lwq.lwq_status_string(rc)
    torch.cuda.synchronize(dev)
    y_ref, den = oracle.matmul(w, Wq, x, act=a)
    assert oracle.normalised_error(y.cpu().numpy(), y_ref, den) <= TOL_GEMV


@pytest.mark.parametrize("w,a", [("q4_0", "bf16"), ("q4_k", "f16"), ("q8_0", "bf16")])
@pytest.mark.parametrize("M,N,K,splits", [(40, 300, 2048, 0), (64, 1000, 4096, 0), (96, 130, 3072, 3),
                                          (33, 257, 4096, 2), (200, 384, 6144, 5)])
def test_gemm_split_k(dev, w, a, M, N, K, splits):
    # few output tiles: the GEMM splits K into slices whose fp32 partials a follow-up kernel adds
    cfg = None
    if splits:
        cfg = lwq.lwq_config()
        cfg.path, cfg.splits = 2, splits
    else:
        assert lwq.lwq_select_config(lwq.fmt_code(w, a), M, N, K).splits > 1
    check_full(w, a, M, N, K, dev, seed=M + N, cfg=cfg)


GEMM_256_CASES = [
    (40, 300, 2048, 48, 0, 0),        # N ends inside the second half of the only weight tile
    (130, 1000, 1024, 64, 0, 3),      # two accumulator buffers (2 x 2 x 64 columns), several tiles per CTA
    (300, 700, 1536, 176, 0, 2),      # one accumulator buffer, the epilogue before the next tile's MMAs
    (96, 513, 3072, 96, 3, 0),        # K slices: fp32 partials added by the follow-up kernel
    (257, 256, 512, 256, 0, 1)]       # widest token tile, one CTA walks both token tiles


# Q8_0's packed chunks of 256 rows (2 x 68 KB) leave room for token tiles up to 96 only
@pytest.mark.parametrize("w,a,M,N,K,bn,splits,ctas",
                         [(w, a) + c for w, a in [("q4_0", "bf16"), ("q4_k", "f16"), ("q4_0", "f16")]
                          for c in GEMM_256_CASES] +
                         [("q8_0", "bf16", 130, 1000, 1024, 64, 0, 3), ("q8_0", "f16", 96, 513, 3072, 96, 3, 0)])
def test_gemm_256_row_tiles(dev, w, a, M, N, K, bn, splits, ctas):
    """256-row weight tiles (two UMMAs per K step share the activation tile) against the oracle."""
    cfg = lwq.lwq_config()
    cfg.path, cfg.tile_n, cfg.tile_m, cfg.splits, cfg.ctas = 2, 256, bn, splits, ctas
    check_full(w, a, M, N, K, dev, seed=M + N + bn, cfg=cfg)


@pytest.mark.parametrize("w,a,M", [("q4_0", "f32", 1), ("q4_k", "f16", 1), ("q8_0", "f16", 16)])
def test_split_k_deterministic(dev, w, a, M):
    """Repeated calls (split-K: partials added in split order by a follow-up kernel) are bitwise identical."""
    N, K = 300, 11008
    Wq, x = inputs.make_problem(w, a, M, N, K, seed=3)
    assert lwq.lwq_select_config(lwq.fmt_code(w, a), M, N, K).splits > 1
    ys = [run_gpu(w, a, Wq, x, M, N, K, dev).cpu().numpy() for _ in range(3)]
    assert np.array_equal(ys[0], ys[1]) and np.array_equal(ys[1], ys[2])
    y_ref, den = oracle.matmul(w, Wq, x, act=a)
    assert oracle.normalised_error(ys[0], y_ref, den) <= TOL_GEMV


# ----------------------------------------------------------- full workloads

def test_q8_0_gemv_4096x4096(dev):
    """Q8_0 decode GEMV, M=1, K=N=4096, fp32 activations, seed 0 -- every output."""
    check_full("q8_0", "f32", 1, 4096, 4096, dev, seed=0)


@pytest.mark.parametrize("M", [1, 4, 8])
def test_q4_0_gemv_11008x4096(dev, M):
    """Q4_0 decode GEMV, M in {1,4,8}, N=11008, K=4096, fp32 activations -- every output."""
    check_full("q4_0", "f32", M, 11008, 4096, dev, seed=0)


def test_q4_k_7b_layer_decode(dev):
    """Q4_K decode over the seven projections of a 7B layer, fp16 activations -- every output."""
    spec = inputs.WORKLOADS["q4_k_7b_layer_decode"]
    for (N, K), seed in zip(spec["shapes"], spec["seeds"]):
        check_full("q4_k", "f16", 1, N, K, dev, seed=seed)


@pytest.mark.parametrize("M,N,K", [(512, 11008, 4096), (2048, 4096, 11008)])
def test_q4_0_prefill_gemm(dev, M, N, K):
    """Q4_0 prefill GEMM, bf16 activations -- sampled outputs plus every tile edge."""
    check_sampled("q4_0", "bf16", M, N, K, dev, seed=0, count=1500)


@functools.lru_cache(maxsize=2)
def _sweep_weights(w, N, K):
    return inputs.make_weights(w, inputs.rng(11), N, K)


@pytest.mark.parametrize("M", inputs.SWEEP_MS)
@pytest.mark.parametrize("K,N", inputs.SWEEP_SHAPES_KN)
@pytest.mark.parametrize("w", inputs.SWEEP_FMTS)
def test_sweep_points_sampled(dev, w, K, N, M):
    """Every point of the format x batch sweep (fp16 activations), in the configuration the sweep times."""
    Wq = _sweep_weights(w, N, K)
    x = inputs.activations(inputs.rng(12 + M), M, K, "f16")
    check_sampled(w, "f16", M, N, K, dev, seed=M + K, count=400, Wq=Wq, x=x)


# ------------------------------------------------------------ error paths

def test_misaligned_pointers(dev):
    fmt = lwq.fmt_code("q4_0", "f32")
    W = torch.zeros(64 * 2304 + 16, dtype=torch.uint8, device=dev)
    x = torch.zeros(4096 + 4, dtype=torch.float32, device=dev)
    y = torch.zeros(64 + 4, dtype=torch.float32, device=dev)
    rc = lwq.lib().lwq_matmul(fmt, W.data_ptr() + 1, x.data_ptr(), y.data_ptr(), 1, 64, 4096, None)
    assert rc == 3
    rc = lwq.lib().lwq_matmul(fmt, W.data_ptr(), x.data_ptr() + 4, y.data_ptr(), 1, 64, 4096, None)
    assert rc == 3


def test_workspace_errors(dev):
    """A split-K call needs the workspace: missing -> NOT_INITIALIZED, small -> TOO_SMALL."""
    w, a, M, N, K = "q4_k", "f16", 1, 256, 11008
    fmt = lwq.fmt_code(w, a)
    assert lwq.lwq_select_config(fmt, M, N, K).splits > 1
    Wq, x = inputs.make_problem(w, a, M, N, K, seed=1)
    Wd, xd = to_device(Wq, dev), to_device(x, dev)
    y = torch.zeros((M, N), dtype=torch.float32, device=dev)
    lwq.lwq_shutdown()
    try:
        assert lwq.lib().lwq_matmul(fmt, Wd.data_ptr(), xd.data_ptr(), y.data_ptr(), M, N, K, None) == 4
        small = torch.zeros(256, dtype=torch.uint8, device=dev)
        lwq.lwq_init(small, 256)
        assert lwq.lib().lwq_matmul(fmt, Wd.data_ptr(), xd.data_ptr(), y.data_ptr(), M, N, K, None) == 5
    finally:
        ws = torch.zeros(WS_BYTES, dtype=torch.uint8, device=dev)
        lwq.lwq_init(ws, WS_BYTES)
        dev_ws_keepalive.append(ws)


dev_ws_keepalive = []


def test_plan_without_split_when_workspace_is_short(dev):
    """The fastest plan splits K (Q4_K, two tiles, half chunks) but no workspace is registered: the call takes
    the plan with a warp per chunk, which needs none, and stays correct."""
    w, a, M, N, K = "q4_k", "f16", 12, 300, 4096
    fmt = lwq.fmt_code(w, a)
    assert lwq.lwq_select_config(fmt, M, N, K).splits > 1
    Wq, x = inputs.make_problem(w, a, M, N, K, seed=9)
    Wd, xd = to_device(Wq, dev), to_device(x, dev)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
    lwq.lwq_shutdown()
    try:
        rc = lwq.lib().lwq_matmul(fmt, Wd.data_ptr(), xd.data_ptr(), y.data_ptr(), M, N, K, None)
        assert rc == lwq.LWQ_OK, lwq.lwq_status_string(rc)
        assert lwq.lwq_last_launch_count() == 1   # no split-K sum
        torch.cuda.synchronize(dev)
    finally:
        ws = torch.zeros(WS_BYTES, dtype=torch.uint8, device=dev)
        lwq.lwq_init(ws, WS_BYTES)
        dev_ws_keepalive.append(ws)
    y_ref, den = oracle.matmul(w, Wq, x, act=a)
    assert oracle.normalised_error(y.cpu().numpy(), y_ref, den) <= TOL_GEMV


def test_bounded_wait_reports_timeout(dev):
    """A wait on an mbarrier that nothing arrives at ends after its bound and reports."""
    torch.cuda.synchronize(dev)
    assert lwq.lwq_get_device_error() == lwq.LWQ_OK
    lwq.lwq_selftest_timeout(2000)
    torch.cuda.synchronize(dev)
    assert lwq.lwq_get_device_error() == lwq.LWQ_ERR_DEVICE_TIMEOUT
    assert lwq.lwq_get_device_error() == lwq.LWQ_OK
    # the context is still usable
    check_full("q4_0", "f32", 1, 64, 512, dev, seed=5)


def test_stream_argument(dev):
    """Calls honour the caller's stream."""
    w, a, M, N, K = "q4_0", "f16", 2, 500, 4096
    Wq, x = inputs.make_problem(w, a, M, N, K, seed=9)
    Wd, xd = to_device(Wq, dev), to_device(x, dev)
    y = torch.zeros((M, N), dtype=torch.float32, device=dev)
    s = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(s):
        lwq.lwq_matmul(lwq.fmt_code(w, a), Wd, xd, y, M, N, K, stream=s)
    s.synchronize()
    y_ref, den = oracle.matmul(w, Wq, x, act=a)
    assert oracle.normalised_error(y.cpu().numpy(), y_ref, den) <= TOL_GEMV


def test_overlap_flag_chains(dev):
    """LWQ_FLAG_OVERLAP (programmatic dependent launch) gives bitwise the same results as plain
    launches, for a chain where each call reads the previous call's output (read after write)
    and later calls overwrite a buffer an earlier call read (write after read)."""
    g = np.random.default_rng(17)
    K = 4096
    W1 = to_device(inputs.make_weights("q4_0", g, 4096, K), dev)
    W2 = to_device(inputs.make_weights("q8_0", g, 4096, K), dev)
    W3 = to_device(inputs.make_weights("q4_k", g, 2048, K), dev)
    x0 = torch.from_numpy(inputs.activations(g, 4, K, "f32")).to(dev)

    def chain(flag):
        a = x0.clone()
        b = torch.full((4, 4096), float("nan"), device=dev)
        c = torch.full((4, 2048), float("nan"), device=dev)
        lwq.lwq_matmul(lwq.fmt_code("q4_0", "f32") | flag, W1, a, b, 4, 4096, K)    # b = f(a)
        lwq.lwq_matmul(lwq.fmt_code("q8_0", "f32") | flag, W2, b, a, 4, 4096, K)    # a = f(b): RAW on b, WAR on a
        lwq.lwq_matmul(lwq.fmt_code("q4_k", "f32") | flag, W3, a, c, 4, 2048, K)    # c = f(a): RAW on a
        lwq.lwq_matmul(lwq.fmt_code("q4_0", "f32") | flag, W1, a, b, 1, 4096, K)    # one-row kernel, RAW on a
        torch.cuda.synchronize(dev)
        return a.cpu().numpy(), b.cpu().numpy(), c.cpu().numpy()

    plain = chain(0)
    for _ in range(3):
        over = chain(lwq.LWQ_FLAG_OVERLAP)
        for p_, o_ in zip(plain, over):
            assert np.array_equal(p_, o_)
    assert all(np.all(np.isfinite(p_)) for p_ in plain)


@pytest.mark.parametrize("w,a,M", [("q4_k", "f16", 1), ("q4_0", "f32", 4), ("q8_0", "bf16", 8)])
def test_fused_projections_equal_separate_calls(dev, w, a, M):
    """One call over weights stacked row-wise (q, k, v in one) gives, bit for bit, the
    separate calls' outputs side by side: a row's result depends only on its own weights."""
    K, parts = 4096, (4096, 1024, 1024)
    Ws = [inputs.make_weights(w, inputs.rng(40 + i), n, K) for i, n in enumerate(parts)]
    x = inputs.activations(inputs.rng(49), M, K, a)
    ys = [run_gpu(w, a, Wq, x, M, n, K, dev).cpu().numpy() for Wq, n in zip(Ws, parts)]
    stacked = np.concatenate(Ws, axis=0)
    y = run_gpu(w, a, stacked, x, M, sum(parts), K, dev).cpu().numpy()
    assert np.array_equal(y, np.concatenate(ys, axis=1))
    y_ref, den = oracle.matmul(w, stacked, x, act=a)
    assert oracle.normalised_error(y, y_ref, den) <= TOL_GEMV


# Two column tiles with a K slice of 8 chunks or fewer: half a chunk of K per warp (all 16 compute warps work).
HALF_CHUNK_CASES = [
    ("q4_0", "f16", 16, 300, 4096), ("q4_0", "bf16", 9, 257, 2048), ("q4_0", "f32", 4, 130, 2048),
    ("q8_0", "f16", 12, 300, 4096), ("q8_0", "f32", 4, 211, 4096), ("q8_0", "bf16", 16, 64, 1024),
    ("q4_k", "f16", 16, 300, 4096), ("q4_k", "bf16", 10, 129, 2048), ("q4_k", "f32", 5, 96, 2048),
    ("q5_k", "f16", 12, 300, 4096), ("q5_k", "f32", 4, 211, 4096), ("q5_k", "bf16", 16, 33, 1024),
    ("q6_k", "f16", 9, 300, 4096), ("q6_k", "f32", 4, 160, 4096), ("q6_k", "bf16", 16, 136, 4352),
    ("q2_k", "f16", 16, 300, 4096), ("q2_k", "f32", 3, 96, 2048), ("q2_k", "bf16", 11, 160, 2048),
]


@pytest.mark.parametrize("w,a,M,N,K", HALF_CHUNK_CASES)
def test_half_chunk_warps(dev, w, a, M, N, K):
    """The two-tile GEMV with half a chunk of K per warp, every format, against the oracle (Q6_K with K = 4352
    and Q2_K stream as row slots); the plan must be the one under test."""
    cfg = lwq.lwq_select_config(lwq.fmt_code(w, a), M, N, K)
    nchunks = K // 256
    cps = -(-nchunks // cfg.splits)
    assert cfg.path == 1 and cps <= 8 and cfg.warps == 2 * cps, cfg.as_dict()
    check_full(w, a, M, N, K, dev, seed=M + N + K)
