"""Host-side checks of the C-ABI library: it loads, exports every symbol the
header declares, and its argument checks / configuration table behave.  No
call here reaches a GPU (every checked call returns before any device work)."""

import os
import re

import pytest

import block_quantized_matmul_lwq_b200 as lwq
from block_quantized_matmul_lwq_b200 import inputs
from block_quantized_matmul_lwq_b200 import build as lwq_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    lwq_build.build()


def header_functions():
    with open(os.path.join(ROOT, "include", "lwq.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lwq_[a-z_]+)\s*\(", src)))


def test_exports_every_header_symbol():
    names = header_functions()
    assert len(names) >= 10
    lib = lwq.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(lwq.EXPORTS) == names


def test_row_bytes():
    f = lwq.fmt_code
    assert lwq.lwq_row_bytes(f("q8_0", "f32"), 4096) == 4352
    assert lwq.lwq_row_bytes(f("q4_0", "f32"), 4096) == 2304
    assert lwq.lwq_row_bytes(f("q4_k", "f16"), 11008) == 6192
    assert lwq.lwq_row_bytes(f("q4_k", "f16"), 128) == 0
    assert lwq.lwq_row_bytes(f("q4_0", "f32"), 48) == 0
    assert lwq.lwq_row_bytes(f("q4_0", "f32"), -32) == 0
    assert lwq.lwq_row_bytes(0x7, 4096) == 0


FAKE = 0x10000  # 16-byte aligned host integer; never dereferenced by the checks below


@pytest.mark.parametrize("args,status", [
    ((lwq.fmt_code("q4_0", "f32"), FAKE, FAKE, FAKE, 0, 8, 64), 1),
    ((lwq.fmt_code("q4_0", "f32"), FAKE, FAKE, FAKE, 1, -8, 64), 1),
    ((lwq.fmt_code("q4_0", "f32"), FAKE, FAKE, FAKE, 1, 8, 48), 1),
    ((lwq.fmt_code("q4_k", "f16"), FAKE, FAKE, FAKE, 1, 8, 128), 1),
    ((0x9, FAKE, FAKE, FAKE, 1, 8, 64), 2),
    ((lwq.LWQ_Q4_0 | 0x300, FAKE, FAKE, FAKE, 1, 8, 64), 2),
    ((lwq.LWQ_Q4_0 | 0x10000, FAKE, FAKE, FAKE, 1, 8, 64), 2),
    ((lwq.fmt_code("q4_0", "f32"), FAKE + 2, FAKE, FAKE, 1, 8, 64), 3),
    ((lwq.fmt_code("q4_0", "f32"), FAKE, FAKE + 4, FAKE, 1, 8, 64), 3),
    ((lwq.fmt_code("q4_0", "f32"), FAKE, FAKE, FAKE + 8, 1, 8, 64), 3),
    ((lwq.fmt_code("q4_0", "f32"), 0, FAKE, FAKE, 1, 8, 64), 1),
])
def test_argument_checks(args, status):
    fmt, W, x, y, M, N, K = args
    rc = lwq.lib().lwq_matmul(fmt, W, x, y, M, N, K, None)
    assert rc == status, (rc, lwq.lwq_status_string(rc))


def test_status_strings():
    for s in range(8):
        assert lwq.lwq_status_string(s)
    assert "unknown" in lwq.lwq_status_string(99)


@pytest.mark.parametrize("w,a", [("q4_0", "f32"), ("q8_0", "f32"), ("q4_k", "f16"), ("q4_0", "bf16"),
                                 ("q8_0", "f16"), ("q4_k", "bf16")])
@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (8, 11008, 4096), (1, 4096, 11008), (16, 32000, 4096),
                                   (4, 4096, 14336), (1, 5, 256), (3, 70, 512), (16, 4096, 14336)])
def test_config_table(w, a, M, N, K):
    fmt = lwq.fmt_code(w, a)
    cfg = lwq.lwq_select_config(fmt, M, N, K).as_dict()
    assert cfg["path"] in (1, 2, 3)
    if cfg["path"] == 1:
        assert 1 <= cfg["warps"] <= 16 and cfg["stages"] >= 2 and cfg["splits"] >= 1
        nchunks = K // 256
        cps = -(-nchunks // cfg["splits"])
        assert cps <= cfg["warps"]            # every chunk of a split has a compute warp
        assert cfg["ctas"] % cfg["splits"] == 0
        ws = lwq.lwq_workspace_size(fmt, M, N, K)
        assert ws >= 256
        if cfg["splits"] > 1:
            m_group = min(M, 8 if a == "f32" else 16)   # activation rows per GEMV pass
            assert ws >= cfg["splits"] * m_group * N * 4
    if K % 256 == 0 and M <= 16:
        assert cfg["path"] == 1               # every format and activation type has the tensor-core GEMV


def test_workspace_size_monotone():
    fmt = lwq.fmt_code("q4_k", "f16")
    a = lwq.lwq_workspace_size(fmt, 1, 4096, 11008)
    b = lwq.lwq_workspace_size(fmt, 16, 11008, 14336)
    assert 0 < a <= b
    assert lwq.lwq_workspace_size(fmt, 0, 1, 256) == 0
    assert lwq.lwq_workspace_size(fmt, 1, 1, 100) == 0


def test_python_constants_match_the_header():
    """Every status code and #define of include/lwq.h has the same value in the binding."""
    import re

    import block_quantized_matmul_lwq_b200 as lwq

    hdr = open(os.path.join(ROOT, "include", "lwq.h")).read()
    found = 0
    for name, val in re.findall(r"\b(LWQ_(?:OK|ERR_[A-Z_]+))\s*=\s*(\d+)", hdr):
        assert getattr(lwq, name) == int(val), name
        found += 1
    for name, val in re.findall(r"#define\s+(LWQ_[A-Z0-9_]+)\s+(0x[0-9A-Fa-f]+|\d+)", hdr):
        if hasattr(lwq, name):
            assert getattr(lwq, name) == int(val, 0), name
            found += 1
    assert found >= 14


@pytest.mark.parametrize("w,a,M,N,K,warps,splits,stages", [
    ("q4_0", "f32", 1, 11008, 4096, 16, 1, 4),     # 3 columns (fp32 parts): one tile, a chunk per warp, K in one CTA
    ("q4_0", "f32", 4, 11008, 4096, 16, 1, 2),     # 12 columns: two tiles, still a chunk per warp (2 stages fit)
    ("q4_0", "f32", 8, 11008, 4096, 16, 2, 4),     # 24 columns: three tiles, half a chunk per warp
    ("q4_0", "f16", 16, 4096, 4096, 16, 2, 4),     # 16 rows of 16-bit activations: the staged slice limits a CTA to
                                                   # 14 chunks, so 2 splits, evened out to 8 chunks with room for 4
                                                   # stages, and half a chunk per warp so that all 16 warps work
    ("q8_0", "f32", 4, 4096, 4096, 16, 2, 4),      # Q8_0, fp32 x, 4 rows: 8 chunks a CTA, half a chunk per warp
    ("q4_0", "f16", 12, 4096, 4096, 16, 1, 2),     # 12 rows: 16 chunks fit, a chunk per warp
    ("q8_0", "f32", 1, 4096, 4096, 16, 1, 2),      # Q8_0 chunks are twice as large: 2 stages
    ("q8_0", "f16", 1, 32000, 4096, 16, 1, 2),
    ("q4_k", "f16", 1, 4096, 11008, 11, 4, 4),     # K = 43 chunks: 4 splits of 11 balance the CTAs better than 3
    ("q4_0", "f16", 1, 4096, 14336, 14, 4, 4),     # K = 56 chunks: 4 splits of 14
])
def test_config_table_rules(w, a, M, N, K, warps, splits, stages):
    """The GEMV rows of the per-shape table (148 SMs when no GPU is present): up to 16 compute warps,
    the split count from the per-CTA work model, and a 4-stage ring where shared memory allows."""
    if lwq.lwq_select_config(lwq.fmt_code("q4_0", "f32"), 1, 11008, 4096).ctas != 148:
        pytest.skip("a device with another SM count is present")
    cfg = lwq.lwq_select_config(lwq.fmt_code(w, a), M, N, K)
    assert (cfg.path, cfg.warps, cfg.splits, cfg.stages) == (1, warps, splits, stages)


@pytest.mark.parametrize("w,a,M,N,K,tile_n,tile_m,ctas", [
    # 256 weight rows x 176 tokens: 43 x 3 = 129 tiles, one round (measured 52 us; 128 x 176 took 70 us)
    ("q4_0", "bf16", 512, 11008, 4096, 256, 176, 129),
    # 256 x 240: 16 x 9 = 144 tiles, one round (measured 157 us; 128 x 256, two rounds, 172 us)
    ("q4_0", "bf16", 2048, 4096, 11008, 256, 240, 144),
])
def test_gemm_table_rules(w, a, M, N, K, tile_n, tile_m, ctas):
    """The GEMM rows of the per-shape table (148 SMs when no GPU is present): the weight and token tiles
    with the least modelled time, rounds of the persistent grid x the time of one tile."""
    if lwq.lwq_select_config(lwq.fmt_code("q4_0", "f32"), 1, 11008, 4096).ctas != 148:
        pytest.skip("a device with another SM count is present")
    cfg = lwq.lwq_select_config(lwq.fmt_code(w, a), M, N, K)
    assert (cfg.path, cfg.tile_n, cfg.tile_m, cfg.ctas, cfg.splits) == (2, tile_n, tile_m, ctas, 1)


def test_gemm_tile_choices_are_valid():
    """Every GEMM row of the sweep has a 128- or 256-row weight tile and a token tile that is a
    multiple of 16 in [32, 256]."""
    for w in ("q8_0", "q4_0", "q4_k"):
        for K, N in ((4096, 4096), (4096, 14336), (14336, 4096), (4096, 32000)):
            for M in (17, 64, 256, 1024):
                cfg = lwq.lwq_select_config(lwq.fmt_code(w, "f16"), M, N, K)
                assert cfg.path == 2
                assert cfg.tile_n in (128, 256)
                assert 32 <= cfg.tile_m <= 256 and cfg.tile_m % 16 == 0
                assert cfg.stages >= 2 and cfg.splits >= 1 and 1 <= cfg.ctas <= 148


def test_more_kquant_formats_routing_and_row_bytes():
    """Q5_K takes the tensor-core paths; Q6_K and Q2_K the tensor-core GEMV and the tcgen05 GEMM too,
    their rows streamed as row slots where they are not 16-byte multiples; they fall back to the
    simple kernel (any M) only when the whole matrix is not a 16-byte multiple; row bytes follow the
    superblock sizes 176, 210 and 84."""
    for M, path in ((1, 1), (16, 1), (17, 2), (512, 2)):
        assert lwq.lwq_select_config(lwq.fmt_code("q5_k", "f16"), M, 4096, 4096).path == path
    for M, K, path in ((1, 4096, 1), (16, 14336, 1), (1, 11008, 1), (8, 2816, 1), (17, 4096, 1), (40, 11008, 1)):
        assert lwq.lwq_select_config(lwq.fmt_code("q6_k", "f32"), M, 4096, K).path == path
    assert lwq.lwq_select_config(lwq.fmt_code("q6_k", "f32"), 1, 4095, 11008).path == 3   # 4095 x 9030 bytes
    # 16-bit activations, M > 16: the tcgen05 GEMM where the rows allow it, else the GEMV in passes
    assert lwq.lwq_select_config(lwq.fmt_code("q6_k", "bf16"), 17, 4096, 4096).path == 2
    assert lwq.lwq_select_config(lwq.fmt_code("q6_k", "bf16"), 512, 4096, 11008).path == 2   # row slots
    assert lwq.lwq_select_config(lwq.fmt_code("q6_k", "bf16"), 512, 4095, 11008).path == 3   # not 16-byte units
    for M in (1, 16, 17, 512):
        # the tcgen05 GEMM for M > 16 when the rows are 16-byte multiples (K % 1024 == 0)
        assert lwq.lwq_select_config(lwq.fmt_code("q2_k", "f16"), M, 4096, 4096).path == (1 if M <= 16 else 2)
        assert lwq.lwq_select_config(lwq.fmt_code("q2_k", "f16"), M, 4096, 11008).path == (1 if M <= 16 else 2)
        assert lwq.lwq_select_config(lwq.fmt_code("q2_k", "f16"), M, 4097, 11008).path == 3
    for w, K, rb in (("q6_k", 4096, 3360), ("q6_k", 11008, 9030), ("q5_k", 4096, 2816), ("q2_k", 11008, 3612)):
        assert lwq.lwq_row_bytes(lwq.fmt_code(w, "f16"), K) == rb == inputs.row_bytes(w, K)
    assert lwq.lwq_row_bytes(lwq.fmt_code("q6_k", "f16"), 288) == 0


def test_workspace_size_covers_smaller_shapes():
    """lwq_workspace_size(fmt, max_M, N, K) covers every M <= max_M: the split-K partials of each
    sweep point (splits x rows of a pass x N fp32) fit the size taken at the sweep's largest M."""
    for w in inputs.SWEEP_FMTS:
        for K, N in inputs.SWEEP_SHAPES_KN:
            fmt = lwq.fmt_code(w, "f16")
            top = lwq.lwq_workspace_size(fmt, max(inputs.SWEEP_MS), N, K)
            for M in list(range(1, 40)) + inputs.SWEEP_MS:
                c = lwq.lwq_select_config(fmt, M, N, K)
                rows = M if c.path == 2 else min(M, 16)
                need = c.splits * rows * N * 4 if c.splits > 1 else 0
                assert need <= top, (w, K, N, M, need, top)


def test_int8_flag_plan():
    i8 = lwq.fmt_code("q4_0", "bf16") | lwq.LWQ_FLAG_ACT_I8
    cfg = lwq.lwq_select_config(i8, 16, 4096, 4096)
    assert cfg.path == 1
    # passes of 8 rows: the workspace for M=16 is that of one 8-row pass
    assert lwq.lwq_workspace_size(i8, 16, 4096, 11008) == lwq.lwq_workspace_size(i8, 8, 4096, 11008)
    assert lwq.lwq_select_config(i8, 17, 4096, 4096).path == 1              # M > 16: GEMV passes of 8 rows
    assert lwq.lwq_select_config(lwq.fmt_code("q8_0", "f16") | lwq.LWQ_FLAG_ACT_I8, 1, 4096, 4096).path == 1
    assert lwq.lwq_select_config(lwq.fmt_code("q4_k", "f16") | lwq.LWQ_FLAG_ACT_I8, 1, 4096, 4096).path == 1
    for fmt, M, K in ((lwq.fmt_code("q6_k", "f16") | lwq.LWQ_FLAG_ACT_I8, 1, 4096), (i8, 1, 288)):
        with pytest.raises(lwq.LwqError) as e:
            lwq.lwq_select_config(fmt, M, 64, K)
        assert e.value.status == lwq.LWQ_ERR_UNSUPPORTED


@pytest.mark.parametrize("B,H,Hkv,L,D,splits", [
    (1, 32, 8, 32768, 128, 18),   # 8 (sequence, kv head) pairs: one CTA per SM, 148 // 8 splits
    (2, 32, 4, 16384, 128, 18),
    (2, 8, 4, 300, 64, 5),        # at most one split per 64 keys
    (4, 32, 8, 8192, 128, 9),     # 32 pairs: the wave model (288 CTAs, two per SM)
    (16, 32, 8, 4096, 128, 2),
    (64, 32, 8, 2048, 128, 1),    # enough pairs: no split, no workspace
    (16, 32, 32, 4096, 128, 2),   # one query head per kv head: about four CTAs per SM
])
def test_attention_split_plan(B, H, Hkv, L, D, splits):
    """The decode-attention work division, read back through the workspace it needs ([B][H][S][D + 2] fp32
    partials when the keys are split).  Without a GPU the planner takes a B200's 148 SMs."""
    ws = lwq.lwq_attention_workspace_size(B, H, Hkv, L, D)
    assert ws == (B * H * splits * (D + 2) * 4 if splits > 1 else 0)


@pytest.mark.parametrize("w", ["q4_0", "q8_0", "q4_k", "q5_k", "q6_k", "q2_k"])
@pytest.mark.parametrize("a", ["f32", "f16", "bf16"])
def test_gemv_warps_per_chunk(w, a):
    """The GEMV plan's K per warp, read back as warps / chunks per CTA: half a chunk (two warps per chunk) at
    three column tiles, and at two when a CTA's K slice has 8 chunks or fewer or a K-quant has K <= 4096;
    otherwise a warp per chunk.  Never more than 16 compute warps."""
    kq = w in ("q4_k", "q5_k", "q6_k", "q2_k")
    fmt = lwq.fmt_code(w, a)
    parts, mmax = (3, 8) if a == "f32" else (1, 16)
    for M in range(1, 17):
        for N, K in ((4096, 4096), (4096, 2048), (11008, 4096), (4096, 11008), (300, 1024), (4096, 14336)):
            cfg = lwq.lwq_select_config(fmt, M, N, K)
            if cfg.path != 1:
                continue
            cps = -(-(K // 256) // cfg.splits)
            wpc, rem = divmod(cfg.warps, cps)
            assert rem == 0 and wpc in (1, 2) and cfg.warps <= 16, (M, N, K, cfg.as_dict())
            nt = -(-min(M, mmax) * parts // 8)
            half = nt == 3 or (nt == 2 and (cps <= 8 or (kq and K <= 4096)))
            assert (wpc == 2) == half, (M, N, K, cfg.as_dict())
