"""Seeded synthetic inputs for the block-quantized matmul y = x . dequant(Wq)^T.

This module is the one place that both the CUDA path's tests/benchmarks and
the CPU oracle take their inputs from.  It draws random numbers and packs
them into the block formats' byte layouts; it never decodes a block and never
computes a product, so it holds none of the matmul's arithmetic.

Formats (the llama.cpp "legacy" and "K-quant" families that "Llamas na Web"
names in its problem statement and in "3. Design de Shader Consciente de
Quantizacao"):

* Q8_0 -- 32 weights per 34-byte block: little-endian fp16 ``d`` then 32
  int8 codes ``q``; the weight is ``q*d``.
* Q4_0 -- 32 weights per 18-byte block: fp16 ``d`` then 16 bytes; byte ``i``
  holds element ``i`` in its low nibble and element ``i+16`` in its high
  nibble; the weight is ``(nibble-8)*d``.
* Q4_K -- 256 weights per 144-byte superblock: fp16 ``d``, fp16 ``dmin``,
  12 bytes holding eight 6-bit (scale, min) pairs, 128 bytes of nibbles.
* Q6_K -- 256 weights per 210-byte superblock: 128 bytes of low nibbles, 64
  bytes of 2-bit high parts, 16 int8 scales (one per 16 weights), fp16 ``d``.
* Q5_K -- 256 weights per 176-byte superblock: fp16 ``d``, fp16 ``dmin``, the
  12 scale/min bytes of Q4_K, 32 bytes of fifth bits, 128 bytes of nibbles.
* Q2_K -- 256 weights per 84-byte superblock: 16 bytes of 4-bit (scale, min)
  pairs, 64 bytes of 2-bit codes, fp16 ``d``, fp16 ``dmin``.

Draw order for one tensor: a fresh ``numpy.random.default_rng(seed)``
(PCG64) draws the weight tensor first (row-major [N][K]) and then the
activations ([M][K]).
"""

from __future__ import annotations

import numpy as np

QK = 32          # weights per Q8_0 / Q4_0 block
QK_K = 256       # weights per Q4_K superblock
BLOCK_BYTES = {"q8_0": 34, "q4_0": 18, "q4_k": 144, "q6_k": 210, "q5_k": 176, "q2_k": 84}
BLOCK_WEIGHTS = {"q8_0": QK, "q4_0": QK, "q4_k": QK_K, "q6_k": QK_K, "q5_k": QK_K, "q2_k": QK_K}


def row_bytes(fmt: str, K: int) -> int:
    """Bytes of one packed weight row of K weights."""
    bw = BLOCK_WEIGHTS[fmt]
    if K % bw:
        raise ValueError(f"K={K} is not a multiple of the {fmt} block ({bw})")
    return K // bw * BLOCK_BYTES[fmt]


def rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def normal_weights(g: np.random.Generator, N: int, K: int, std: float = 0.02) -> np.ndarray:
    """fp32 weights ~ N(0, std^2), row-major [N][K]."""
    return (g.standard_normal((N, K), dtype=np.float32) * np.float32(std)).astype(np.float32)


def _f16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to fp16 (nearest-even, numpy's cast) and return the 16-bit codes."""
    return np.ascontiguousarray(a.astype(np.float16)).view(np.uint16)


def _round_half_away(v: np.ndarray) -> np.ndarray:
    return (np.sign(v) * np.floor(np.abs(v) + np.float32(0.5))).astype(np.float32)


def quantize_q8_0(w: np.ndarray) -> np.ndarray:
    """Pack fp32 weights [N][K] into Q8_0 bytes [N][K/32*34].

    Per block of 32: d32 = max|w| / 127 in fp32, stored as fp16(d32);
    q = round(w / d32), halves away from zero, clamped to [-127, 127];
    an all-zero block stores d = 0, q = 0.
    """
    N, K = w.shape
    nb = K // QK
    wb = w.reshape(N, nb, QK).astype(np.float32)
    amax = np.abs(wb).max(axis=-1)
    d32 = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(d32 > 0, d32, np.float32(1.0))
    q = _round_half_away(wb / safe[..., None])
    q = np.clip(q, -127, 127)
    q = np.where(d32[..., None] > 0, q, 0).astype(np.int8)
    out = np.empty((N, nb, 34), dtype=np.uint8)
    out[..., 0:2] = _f16_bits(d32).view(np.uint8).reshape(N, nb, 2)
    out[..., 2:34] = q.view(np.uint8)
    return out.reshape(N, nb * 34)


def quantize_q4_0(w: np.ndarray) -> np.ndarray:
    """Pack fp32 weights [N][K] into Q4_0 bytes [N][K/32*18].

    Per block of 32: amax = the signed weight of largest magnitude (first
    index wins a tie); d32 = amax / -8 in fp32, stored as fp16(d32);
    q = min(15, round(w/d32 + 8)) with halves rounded up, floored at 0;
    an all-zero block stores d = 0 and every code 8.
    """
    N, K = w.shape
    nb = K // QK
    wb = w.reshape(N, nb, QK).astype(np.float32)
    idx = np.abs(wb).argmax(axis=-1)
    amax = np.take_along_axis(wb, idx[..., None], axis=-1)[..., 0]
    d32 = (amax / np.float32(-8.0)).astype(np.float32)
    safe = np.where(d32 != 0, d32, np.float32(1.0))
    v = (wb / safe[..., None] + np.float32(8.0)).astype(np.float32)
    q = np.floor(v + np.float32(0.5))
    q = np.clip(q, 0, 15)
    q = np.where(d32[..., None] != 0, q, 8).astype(np.uint8)
    packed = (q[..., :16] | (q[..., 16:] << 4)).astype(np.uint8)
    out = np.empty((N, nb, 18), dtype=np.uint8)
    out[..., 0:2] = _f16_bits(d32).view(np.uint8).reshape(N, nb, 2)
    out[..., 2:18] = packed
    return out.reshape(N, nb * 18)


def random_q4_k(g: np.random.Generator, N: int, K: int) -> np.ndarray:
    """Random Q4_K bytes [N][K/256*144].

    d and dmin ~ U(0, 0.01) drawn in fp32 and rounded to fp16; the 12
    scale/min bytes and the 128 nibble bytes are uniform random bytes (every
    bit of the 12 bytes belongs to exactly one 6-bit field, so uniform bytes
    give uniform 6-bit scales and mins).  Draw order: d[N][nb], dmin[N][nb],
    scale bytes[N][nb][12], nibble bytes[N][nb][128].
    """
    nb = K // QK_K
    if K % QK_K:
        raise ValueError("Q4_K needs K % 256 == 0")
    d = g.uniform(0.0, 0.01, size=(N, nb)).astype(np.float32)
    dmin = g.uniform(0.0, 0.01, size=(N, nb)).astype(np.float32)
    sc = g.integers(0, 256, size=(N, nb, 12), dtype=np.uint8)
    qs = g.integers(0, 256, size=(N, nb, 128), dtype=np.uint8)
    out = np.empty((N, nb, 144), dtype=np.uint8)
    out[..., 0:2] = _f16_bits(d).view(np.uint8).reshape(N, nb, 2)
    out[..., 2:4] = _f16_bits(dmin).view(np.uint8).reshape(N, nb, 2)
    out[..., 4:16] = sc
    out[..., 16:144] = qs
    return out.reshape(N, nb * 144)


def _superblocks(fmt: str, K: int) -> int:
    if K % QK_K:
        raise ValueError(f"{fmt} needs K % 256 == 0")
    return K // QK_K


def random_q6_k(g: np.random.Generator, N: int, K: int) -> np.ndarray:
    """Random Q6_K bytes [N][K/256*210].

    d ~ U(0, 0.01) drawn in fp32 and rounded to fp16; the 16 int8 scales,
    the 128 low-nibble bytes and the 64 high-bit bytes are uniform random
    bytes (uniform 6-bit codes and int8 scales).  Draw order: d[N][nb],
    scale bytes[N][nb][16], low bytes[N][nb][128], high bytes[N][nb][64].
    Layout: low bytes at 0, high bytes at 128, scales at 192, d at 208.
    """
    nb = _superblocks("q6_k", K)
    d = g.uniform(0.0, 0.01, size=(N, nb)).astype(np.float32)
    sc = g.integers(0, 256, size=(N, nb, 16), dtype=np.uint8)
    ql = g.integers(0, 256, size=(N, nb, 128), dtype=np.uint8)
    qh = g.integers(0, 256, size=(N, nb, 64), dtype=np.uint8)
    out = np.empty((N, nb, 210), dtype=np.uint8)
    out[..., 0:128] = ql
    out[..., 128:192] = qh
    out[..., 192:208] = sc
    out[..., 208:210] = _f16_bits(d).view(np.uint8).reshape(N, nb, 2)
    return out.reshape(N, nb * 210)


def random_q5_k(g: np.random.Generator, N: int, K: int) -> np.ndarray:
    """Random Q5_K bytes [N][K/256*176].

    d and dmin ~ U(0, 0.01) rounded to fp16; scale/min, fifth-bit and nibble
    bytes uniform.  Draw order: d[N][nb], dmin[N][nb], scale bytes[N][nb][12],
    fifth-bit bytes[N][nb][32], nibble bytes[N][nb][128].  Layout: d at 0,
    dmin at 2, scales at 4, fifth bits at 16, nibbles at 48.
    """
    nb = _superblocks("q5_k", K)
    d = g.uniform(0.0, 0.01, size=(N, nb)).astype(np.float32)
    dmin = g.uniform(0.0, 0.01, size=(N, nb)).astype(np.float32)
    sc = g.integers(0, 256, size=(N, nb, 12), dtype=np.uint8)
    qh = g.integers(0, 256, size=(N, nb, 32), dtype=np.uint8)
    qs = g.integers(0, 256, size=(N, nb, 128), dtype=np.uint8)
    out = np.empty((N, nb, 176), dtype=np.uint8)
    out[..., 0:2] = _f16_bits(d).view(np.uint8).reshape(N, nb, 2)
    out[..., 2:4] = _f16_bits(dmin).view(np.uint8).reshape(N, nb, 2)
    out[..., 4:16] = sc
    out[..., 16:48] = qh
    out[..., 48:176] = qs
    return out.reshape(N, nb * 176)


def random_q2_k(g: np.random.Generator, N: int, K: int) -> np.ndarray:
    """Random Q2_K bytes [N][K/256*84].

    d and dmin ~ U(0, 0.01) rounded to fp16; scale/min bytes and code bytes
    uniform.  Draw order: d[N][nb], dmin[N][nb], scale bytes[N][nb][16], code
    bytes[N][nb][64].  Layout: scales at 0, codes at 16, d at 80, dmin at 82.
    """
    nb = _superblocks("q2_k", K)
    d = g.uniform(0.0, 0.01, size=(N, nb)).astype(np.float32)
    dmin = g.uniform(0.0, 0.01, size=(N, nb)).astype(np.float32)
    sc = g.integers(0, 256, size=(N, nb, 16), dtype=np.uint8)
    qs = g.integers(0, 256, size=(N, nb, 64), dtype=np.uint8)
    out = np.empty((N, nb, 84), dtype=np.uint8)
    out[..., 0:16] = sc
    out[..., 16:80] = qs
    out[..., 80:82] = _f16_bits(d).view(np.uint8).reshape(N, nb, 2)
    out[..., 82:84] = _f16_bits(dmin).view(np.uint8).reshape(N, nb, 2)
    return out.reshape(N, nb * 84)


def activations(g: np.random.Generator, M: int, K: int, act: str) -> np.ndarray:
    """x ~ N(0,1) drawn in fp32 [M][K], then stored in ``act``.

    Returns float32 for "f32", float16 for "f16" and the uint16 bit codes of
    bf16 (round to nearest even) for "bf16".
    """
    x = g.standard_normal((M, K), dtype=np.float32)
    if act == "f32":
        return np.ascontiguousarray(x)
    if act == "f16":
        return np.ascontiguousarray(x.astype(np.float16))
    if act == "bf16":
        return f32_to_bf16_bits(x)
    raise ValueError(act)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 codes, round to nearest even (finite inputs)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    r = (b + 0x7FFF + lsb) >> 16
    return r.astype(np.uint16)


def make_weights(fmt: str, g: np.random.Generator, N: int, K: int) -> np.ndarray:
    """Packed weights for one tensor, drawn from ``g`` as each format's workload specifies."""
    if fmt == "q8_0":
        return quantize_q8_0(normal_weights(g, N, K))
    if fmt == "q4_0":
        return quantize_q4_0(normal_weights(g, N, K))
    if fmt == "q4_k":
        return random_q4_k(g, N, K)
    if fmt == "q6_k":
        return random_q6_k(g, N, K)
    if fmt == "q5_k":
        return random_q5_k(g, N, K)
    if fmt == "q2_k":
        return random_q2_k(g, N, K)
    raise ValueError(fmt)


def make_problem(fmt: str, act: str, M: int, N: int, K: int, seed: int = 0):
    """(Wq bytes [N][row_bytes], x [M][K] in ``act``) from one seeded stream: W first, then x."""
    g = rng(seed)
    Wq = make_weights(fmt, g, N, K)
    x = activations(g, M, K, act)
    return Wq, x


def attention_problem(B: int, H: int, Hkv: int, Lmax: int, D: int, act: str, seed: int = 0, lens=None):
    """Decode-attention inputs from one seeded stream: q [B][H][D], then the key cache and the
    value cache [B][Hkv][Lmax][D], all ~ N(0, 1) drawn in fp32 and stored in ``act`` (fp16, or
    bf16 codes).  Sequence lengths: ``lens`` as given, else Lmax for every sequence."""
    g = rng(seed)

    def draw(shape):
        a = g.standard_normal(shape, dtype=np.float32)
        return np.ascontiguousarray(a.astype(np.float16)) if act == "f16" else f32_to_bf16_bits(a)

    q = draw((B, H, D))
    k = draw((B, Hkv, Lmax, D))
    v = draw((B, Hkv, Lmax, D))
    lens = np.full(B, Lmax, dtype=np.int32) if lens is None else np.asarray(lens, dtype=np.int32)
    return q, k, v, lens


# The workloads, by what they are (format, activation dtype, shapes, seed).
WORKLOADS = {
    "q8_0_gemv_4096x4096": dict(fmt="q8_0", act="f32", Ms=[1], shapes=[(4096, 4096)], seeds=[0]),
    "q4_0_gemv_11008x4096": dict(fmt="q4_0", act="f32", Ms=[1, 4, 8], shapes=[(11008, 4096)], seeds=[0]),
    "q4_k_7b_layer_decode": dict(
        fmt="q4_k", act="f16", Ms=[1],
        # (N, K) of q, k, v, o, gate, up, down
        shapes=[(4096, 4096)] * 4 + [(11008, 4096), (11008, 4096), (4096, 11008)],
        seeds=[0, 1, 2, 3, 4, 5, 6]),
    # the same layer with q, k, v stored as one [12288][row] weight and gate, up as one
    # [22016][row] weight (rows concatenated in that order): four calls instead of seven
    "q4_k_7b_layer_decode_fused": dict(
        fmt="q4_k", act="f16", Ms=[1],
        shapes=[(12288, 4096), (4096, 4096), (22016, 4096), (4096, 11008)],
        seeds=[(0, 1, 2), 3, (4, 5), 6]),
    # the headline decode step with int8 activation blocks (LWQ_FLAG_ACT_I8)
    "q4_0_gemv_11008x4096_act_i8": dict(fmt="q4_0", act="f32:i8", Ms=[1, 4, 8], shapes=[(11008, 4096)], seeds=[0]),
    # the Q4_K layer with its fp16 activations taken as int8 blocks
    "q4_k_7b_layer_decode_act_i8": dict(
        fmt="q4_k", act="f16:i8", Ms=[1],
        shapes=[(4096, 4096)] * 4 + [(11008, 4096), (11008, 4096), (4096, 11008)],
        seeds=[0, 1, 2, 3, 4, 5, 6]),
    "q4_0_prefill_gemm": dict(fmt="q4_0", act="bf16", Ms=[512, 2048],
                              shapes=[(11008, 4096), (4096, 11008)], seeds=[0, 0]),
    # the other K-quant formats over the same 7B layer (fp16 activations, one token)
    "q6_k_7b_layer_decode": dict(fmt="q6_k", act="f16", Ms=[1],
                                 shapes=[(4096, 4096)] * 4 + [(11008, 4096), (11008, 4096), (4096, 11008)],
                                 seeds=[0, 1, 2, 3, 4, 5, 6]),
    "q5_k_7b_layer_decode": dict(fmt="q5_k", act="f16", Ms=[1],
                                 shapes=[(4096, 4096)] * 4 + [(11008, 4096), (11008, 4096), (4096, 11008)],
                                 seeds=[0, 1, 2, 3, 4, 5, 6]),
    "q2_k_7b_layer_decode": dict(fmt="q2_k", act="f16", Ms=[1],
                                 shapes=[(4096, 4096)] * 4 + [(11008, 4096), (11008, 4096), (4096, 11008)],
                                 seeds=[0, 1, 2, 3, 4, 5, 6]),
    # and their prefill GEMM at the up- and down-projection shapes (bf16 activations, 512 tokens; the
    # down projection's Q6_K and Q2_K rows are not 16-byte multiples and stream as row slots)
    "q6_k_prefill_gemm": dict(fmt="q6_k", act="bf16", Ms=[512, 512], shapes=[(11008, 4096), (4096, 11008)],
                              seeds=[0, 0]),
    "q5_k_prefill_gemm": dict(fmt="q5_k", act="bf16", Ms=[512, 512], shapes=[(11008, 4096), (4096, 11008)],
                              seeds=[0, 0]),
    "q2_k_prefill_gemm": dict(fmt="q2_k", act="bf16", Ms=[512, 512], shapes=[(11008, 4096), (4096, 11008)],
                              seeds=[0, 0]),
}

# Decode attention workloads: one query token per sequence against its key/value cache.
#  * the pages' example ("Compute Shaders con WebGPU para Inferencia ML", "El Mecanismo de
#    Atencion"): 512 tokens, 12 heads, head dimension 64;
#  * a 7B-shaped decode batch: 16 sequences of 4096 cached tokens, 32 heads of 128, each with
#    its own kv head (multi-head) or 4 query heads per kv head (grouped).
ATTENTION_WORKLOADS = {
    "attention_decode_page": dict(B=1, H=12, Hkv=12, L=512, D=64, act="f16"),
    "attention_decode_7b_mha": dict(B=16, H=32, Hkv=32, L=4096, D=128, act="f16"),
    "attention_decode_7b_gqa": dict(B=16, H=32, Hkv=8, L=4096, D=128, act="f16"),
}

SWEEP_FMTS = ["q8_0", "q4_0", "q4_k"]
SWEEP_MS = [1, 2, 4, 8, 16, 64, 256, 1024]
SWEEP_SHAPES_KN = [(4096, 4096), (4096, 14336), (14336, 4096), (4096, 32000)]
