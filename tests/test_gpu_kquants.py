"""More K-quant formats (Q5_K, Q6_K, Q2_K) on the GPU against the oracle.

Q5_K has tensor-core decoders (the GEMV and the tcgen05 GEMM).  Q6_K and Q2_K
superblocks are 210 and 84 bytes, so their rows are not 16-byte multiples in
general.  Q6_K rows of K a multiple of 2048 are, and take per-chunk TMA boxes
(and the tcgen05 GEMM); other Q6_K rows, and every Q2_K row, stream as slots of
the flat matrix whenever the whole matrix is a 16-byte multiple, else take the
simple kernel.  Every case is scored element by element against the oracle on
the same seeded inputs.
"""

import ctypes

import pytest
import torch

import block_quantized_matmul_lwq_b200 as lwq
from gpu_util import check_full, check_sampled

pytestmark = pytest.mark.gpu

WS_BYTES = 256 << 20
ACTS = ("f32", "f16", "bf16")


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


@pytest.mark.parametrize("w", ["q5_k", "q6_k", "q2_k"])
@pytest.mark.parametrize("a", ACTS)
@pytest.mark.parametrize("M,N,K", [(1, 1, 256), (1, 37, 512), (3, 100, 1024), (8, 333, 4096), (5, 61, 2816),
                                   (16, 50, 768), (12, 130, 4352), (1, 17, 6144)])
def test_small_shapes(dev, w, a, M, N, K):
    check_full(w, a, M, N, K, dev, seed=M * 1000 + N + K)


@pytest.mark.parametrize("a", ACTS)
@pytest.mark.parametrize("M", [2, 3, 4, 5, 6, 7, 8, 9, 15, 16])
def test_q5_k_every_column_layout(dev, a, M):
    assert lwq.lwq_select_config(lwq.fmt_code("q5_k", a), M, 45, 1024).path == 1
    check_full("q5_k", a, M, 45, 1024, dev, seed=200 + M)


@pytest.mark.parametrize("a", ACTS)
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 6, 8, 9, 16])
@pytest.mark.parametrize("K", [2048, 6144])
def test_q6_k_tensor_core_gemv(dev, a, M, K):
    """Q6_K rows of whole 16-byte multiples (K % 2048 == 0): per-chunk TMA boxes whose superblock
    starts 0..14 bytes in (both word alignments), every column layout, ragged N."""
    assert lwq.lwq_select_config(lwq.fmt_code("q6_k", a), M, 45, K).path == 1
    check_full("q6_k", a, M, 45, K, dev, seed=300 + M + K)


@pytest.mark.parametrize("a", ["bf16", "f16"])
@pytest.mark.parametrize("M,N,K,tile_n", [(40, 300, 2048, 0), (130, 1000, 4096, 0), (200, 520, 6144, 128),
                                          (64, 700, 4096, 256)])
def test_q6_k_gemm(dev, a, M, N, K, tile_n):
    """Q6_K on the tcgen05 GEMM (K a multiple of 2048): per-superblock boxes at both word alignments."""
    cfg = None
    if tile_n:
        cfg = lwq.lwq_config()
        cfg.path, cfg.tile_n = 2, tile_n
    assert lwq.lwq_select_config(lwq.fmt_code("q6_k", a), M, N, K).path == 2
    check_full("q6_k", a, M, N, K, dev, seed=M + K, cfg=cfg)


@pytest.mark.parametrize("a", ["bf16", "f16"])
@pytest.mark.parametrize("M,N,K,tile_n", [(40, 300, 1024, 0), (130, 1000, 4096, 0), (200, 520, 3072, 128),
                                          (64, 700, 4096, 256), (17, 96, 2048, 0)])
def test_q2_k_gemm(dev, a, M, N, K, tile_n):
    """Q2_K on the tcgen05 GEMM (K a multiple of 1024): per-superblock 96-byte boxes whose superblock
    starts 0, 4, 8 or 12 bytes in."""
    cfg = None
    if tile_n:
        cfg = lwq.lwq_config()
        cfg.path, cfg.tile_n = 2, tile_n
    assert lwq.lwq_select_config(lwq.fmt_code("q2_k", a), M, N, K).path == 2
    check_full("q2_k", a, M, N, K, dev, seed=M + K + 1, cfg=cfg)


@pytest.mark.parametrize("w", ["q6_k", "q2_k"])
@pytest.mark.parametrize("a", ["bf16", "f16"])
@pytest.mark.parametrize("M,N,K,tile_n,splits", [(40, 48, 2816, 0, 0), (130, 296, 4352, 0, 0), (64, 520, 11008, 256, 0),
                                                 (200, 136, 1536, 128, 3), (17, 264, 11008, 0, 0)])
def test_row_slot_gemm(dev, w, a, M, N, K, tile_n, splits):
    """Q6_K and Q2_K rows that are not 16-byte multiples on the tcgen05 GEMM: one bulk copy per row and
    superblock, superblocks starting at every 2-byte (Q6_K) or 4-byte (Q2_K) offset, rows past N."""
    cfg = None
    if tile_n or splits:
        cfg = lwq.lwq_config()
        cfg.path, cfg.tile_n, cfg.splits = 2, tile_n, splits
    assert lwq.lwq_select_config(lwq.fmt_code(w, a), M, N, K).path == 2
    check_full(w, a, M, N, K, dev, seed=M + N + K, cfg=cfg)


@pytest.mark.parametrize("w", ["q6_k", "q2_k"])
def test_row_slot_prefill_down_projection(dev, w):
    """The 7B down projection (K = 11008) at 512 tokens, sampled outputs plus every tile edge."""
    M, N, K = 512, 4096, 11008
    assert lwq.lwq_select_config(lwq.fmt_code(w, "bf16"), M, N, K).path == 2
    check_sampled(w, "bf16", M, N, K, dev, seed=23, count=2000)


def test_q2_k_prefill_gemm_sampled(dev):
    M, N, K = 512, 11008, 4096
    assert lwq.lwq_select_config(lwq.fmt_code("q2_k", "bf16"), M, N, K).path == 2
    check_sampled("q2_k", "bf16", M, N, K, dev, seed=19, count=2000)


def test_q6_k_prefill_gemm_sampled(dev):
    M, N, K = 512, 11008, 4096
    assert lwq.lwq_select_config(lwq.fmt_code("q6_k", "bf16"), M, N, K).path == 2
    check_sampled("q6_k", "bf16", M, N, K, dev, seed=9, count=2000)


@pytest.mark.parametrize("a", ACTS)
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 6, 8, 9, 16])
@pytest.mark.parametrize("K", [256, 1024, 4352, 11008])
def test_q2_k_tensor_core_gemv(dev, a, M, K):
    """Q2_K row slots: 44 rows (a 16-byte multiple whatever K), slices that start 0, 4, 8 or 12
    bytes into their slot, every column layout, a ragged last row tile, split-K at K = 11008."""
    assert lwq.lwq_select_config(lwq.fmt_code("q2_k", a), M, 44, K).path == 1
    check_full("q2_k", a, M, 44, K, dev, seed=400 + M + K)


@pytest.mark.parametrize("a", ACTS)
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 6, 8, 9, 16])
@pytest.mark.parametrize("K", [256, 2816, 4352, 11008])
def test_q6_k_row_slot_gemv(dev, a, M, K):
    """Q6_K rows that are not 16-byte multiples: row slots whose superblocks start at either word
    alignment, row by row, every column layout, a ragged last row tile, split-K at K = 11008."""
    assert lwq.lwq_select_config(lwq.fmt_code("q6_k", a), M, 56, K).path == 1
    check_full("q6_k", a, M, 56, K, dev, seed=500 + M + K)


@pytest.mark.parametrize("warps,splits,stages", [(1, 0, 2), (3, 0, 2), (8, 2, 3), (4, 3, 2), (16, 0, 4)])
def test_q6_k_row_slot_forced_configs(dev, warps, splits, stages):
    cfg = lwq.lwq_config()
    cfg.path, cfg.warps, cfg.splits, cfg.stages = 1, warps, splits, stages
    check_full("q6_k", "bf16", 3, 72, 4352, dev, seed=warps + splits, cfg=cfg)


@pytest.mark.parametrize("warps,splits,stages", [(1, 0, 2), (3, 0, 2), (8, 2, 3), (4, 3, 2), (16, 0, 4)])
def test_q2_k_forced_gemv_configs(dev, warps, splits, stages):
    cfg = lwq.lwq_config()
    cfg.path, cfg.warps, cfg.splits, cfg.stages = 1, warps, splits, stages
    check_full("q2_k", "f32", 5, 120, 4352, dev, seed=warps + splits, cfg=cfg)


def test_q2_k_routing(dev):
    """Q2_K takes the tensor-core GEMV when N * row bytes is a 16-byte multiple, else the simple kernel."""
    f = lwq.fmt_code("q2_k", "f16")
    assert lwq.lwq_select_config(f, 1, 4096, 11008).path == 1
    assert lwq.lwq_select_config(f, 1, 37, 11008).path == 3      # 37 x 3612 bytes
    assert lwq.lwq_select_config(f, 1, 37, 4096).path == 1       # 1344-byte rows
    check_full("q2_k", "f16", 2, 37, 11008, dev, seed=3)


@pytest.mark.parametrize("warps,splits,stages", [(1, 0, 2), (3, 0, 2), (8, 2, 3), (4, 3, 2)])
def test_q6_k_forced_gemv_configs(dev, warps, splits, stages):
    cfg = lwq.lwq_config()
    cfg.path, cfg.warps, cfg.splits, cfg.stages = 1, warps, splits, stages
    check_full("q6_k", "f16", 3, 100, 4096, dev, seed=warps + splits, cfg=cfg)


@pytest.mark.parametrize("w", ["q5_k", "q6_k", "q2_k"])
def test_7b_layer_shapes(dev, w):
    """The 7B layer's three projection shapes at M = 1 with fp16 activations, every output."""
    for N, K in ((4096, 4096), (11008, 4096), (4096, 11008)):
        check_full(w, "f16", 1, N, K, dev, seed=N + K)


@pytest.mark.parametrize("w,a", [("q5_k", "bf16"), ("q5_k", "f16"), ("q6_k", "bf16"), ("q2_k", "f16")])
@pytest.mark.parametrize("M,N,K", [(40, 300, 2048), (130, 1000, 1024), (300, 700, 1536)])
def test_prefill_shapes(dev, w, a, M, N, K):
    check_full(w, a, M, N, K, dev, seed=M + N)


def test_q5_k_prefill_gemm_sampled(dev):
    """Q5_K at the prefill shape (tcgen05 GEMM, 256-row tiles), sampled outputs."""
    M, N, K = 512, 11008, 4096
    cfg = lwq.lwq_select_config(lwq.fmt_code("q5_k", "bf16"), M, N, K)
    assert cfg.path == 2
    check_sampled("q5_k", "bf16", M, N, K, dev, seed=7, count=2000)


@pytest.mark.parametrize("tile_n,bn,splits", [(128, 64, 0), (256, 96, 0), (256, 48, 3), (128, 176, 2)])
def test_q5_k_forced_gemm_tiles(dev, tile_n, bn, splits):
    cfg = lwq.lwq_config()
    cfg.path, cfg.tile_n, cfg.tile_m, cfg.splits = 2, tile_n, bn, splits
    check_full("q5_k", "f16", 150, 520, 3072, dev, seed=tile_n + bn, cfg=cfg)


def test_q5_k_split_k_gemv(dev):
    """Small N, long K: the GEMV splits K over CTAs and a follow-up kernel adds the partials."""
    fmt = lwq.fmt_code("q5_k", "f32")
    assert lwq.lwq_select_config(fmt, 4, 300, 11008).splits > 1
    check_full("q5_k", "f32", 4, 300, 11008, dev, seed=5)


def test_forced_path_without_decoder_is_refused(dev):
    """Forcing the tensor-core GEMV where its weight stream cannot go (a Q6_K or Q2_K matrix that is
    not a whole number of 16-byte units) returns LWQ_ERR_UNSUPPORTED before anything runs."""
    cfg = lwq.lwq_config()
    cfg.path = 1
    buf = torch.zeros(1024, dtype=torch.float32, device="cuda:0")
    p = buf.data_ptr()
    for w, N in (("q6_k", 15), ("q2_k", 1), ("q2_k", 5)):   # 15 x 210, 84, 5 x 84 bytes
        rc = lwq.lib().lwq_matmul_config(lwq.fmt_code(w, "f16"), p, p, p, 1, N, 256, ctypes.byref(cfg), None)
        assert rc == lwq.LWQ_ERR_UNSUPPORTED, w

