"""Checks that pin the CPU oracle to facts outside itself.

Each ``pin_*`` function takes a loaded oracle library handle and raises
AssertionError when the oracle disagrees with a fact fixed by the block
layouts, by IEEE-754, by mathematics, or by an independent library routine.
``test_oracle_pins.py`` runs them against the real oracle (all must pass);
``test_oracle_mutants.py`` runs them against copies of the oracle with one
planted mistake each (each copy must fail at least one).
"""

from __future__ import annotations

import os

import math

import numpy as np
import torch

import oracle
from block_quantized_matmul_lwq_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------- fixtures

def _parse_bytes(spec: str) -> bytes:
    out = bytearray()
    for piece in spec.split("."):
        if "*" in piece:
            b, n = piece.split("*")
            out += bytes([int(b, 16)]) * int(n)
        else:
            out += bytes.fromhex(piece)
    return bytes(out)


def _parse_values(spec: str) -> list[float]:
    vals: list[float] = []
    for tok in spec.split(","):
        tok = tok.strip()
        if "*" in tok:
            v, n = tok.rsplit("*", 1)
            vals += [float(v)] * int(n)
        else:
            vals.append(float(tok))
    return vals


def hand_blocks():
    """(name, fmt, K, block bytes, expected weights) from tests/golden/hand_blocks.txt."""
    rows = []
    with open(os.path.join(GOLDEN, "hand_blocks.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, vals = line.split(":")
            name, fmt, K, spec = head.split()
            rows.append((name, fmt, int(K), _parse_bytes(spec), _parse_values(vals)))
    return rows


# ------------------------------------------------- independent decoders
# Written separately from the oracle's C code, vectorised, from the layouts.

def indep_f16(codes: np.ndarray) -> np.ndarray:
    return np.asarray(codes, dtype=np.uint16).view(np.float16).astype(np.float64)


def indep_bf16(codes: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.asarray(codes, dtype=np.uint16).view(np.int16).copy())
    return t.view(torch.bfloat16).to(torch.float64).numpy()


def indep_decode(fmt: str, Wq: np.ndarray, K: int) -> np.ndarray:
    """Decode packed rows with numpy only; returns fp64 exact values [N][K]."""
    rb = inputs.row_bytes(fmt, K)
    W = np.asarray(Wq, dtype=np.uint8).reshape(-1, rb)
    N = W.shape[0]
    if fmt == "q8_0":
        b = W.reshape(N, K // 32, 34)
        d = indep_f16(b[..., 0:2].copy().view(np.uint16)[..., 0])
        q = b[..., 2:].view(np.int8).astype(np.float64)
        return (q * d[..., None]).reshape(N, K)
    if fmt == "q4_0":
        b = W.reshape(N, K // 32, 18)
        d = indep_f16(b[..., 0:2].copy().view(np.uint16)[..., 0])
        nib = b[..., 2:]
        q = np.concatenate([(nib & 15), (nib >> 4)], axis=-1).astype(np.float64) - 8.0
        return (q * d[..., None]).reshape(N, K)
    if fmt == "q4_k":
        b = W.reshape(N, K // 256, 144)
        d = indep_f16(b[..., 0:2].copy().view(np.uint16)[..., 0])
        dmin = indep_f16(b[..., 2:4].copy().view(np.uint16)[..., 0])
        s = b[..., 4:16].astype(np.int64)
        sc = np.empty(s.shape[:-1] + (8,), dtype=np.int64)
        mn = np.empty_like(sc)
        sc[..., :4] = s[..., 0:4] & 63
        mn[..., :4] = s[..., 4:8] & 63
        sc[..., 4:] = (s[..., 8:12] & 15) | ((s[..., 0:4] >> 6) << 4)
        mn[..., 4:] = (s[..., 8:12] >> 4) | ((s[..., 4:8] >> 6) << 4)
        qs = b[..., 16:].reshape(N, K // 256, 4, 32).astype(np.int64)
        q = np.stack([qs & 15, qs >> 4], axis=3).reshape(N, K // 256, 8, 32)  # sub-block j = 2g + half
        w = d[..., None, None] * sc[..., None] * q - dmin[..., None, None] * mn[..., None]
        return w.reshape(N, K)
    if fmt == "q6_k":
        b = W.reshape(N, K // 256, 210)
        d = indep_f16(b[..., 208:210].copy().view(np.uint16)[..., 0])
        sc = b[..., 192:208].view(np.int8).astype(np.float64)              # [N][nb][16]
        ql = b[..., 0:128].reshape(N, K // 256, 2, 2, 32).astype(np.int64)  # [half][ql quarter][l]
        qh = b[..., 128:192].reshape(N, K // 256, 2, 1, 32).astype(np.int64)
        low = np.concatenate([ql & 15, ql >> 4], axis=3)                   # [half][g = 2*nibble + quarter][l]
        high = (qh >> (2 * np.arange(4)[None, None, None, :, None])) & 3
        q = (low | (high << 4)).reshape(N, K // 256, 256).astype(np.float64) - 32.0
        return (d[..., None] * np.repeat(sc, 16, axis=-1) * q).reshape(N, K)
    if fmt == "q5_k":
        b = W.reshape(N, K // 256, 176)
        d = indep_f16(b[..., 0:2].copy().view(np.uint16)[..., 0])
        dmin = indep_f16(b[..., 2:4].copy().view(np.uint16)[..., 0])
        s = b[..., 4:16].astype(np.int64)
        sc = np.empty(s.shape[:-1] + (8,), dtype=np.int64)
        mn = np.empty_like(sc)
        sc[..., :4] = s[..., 0:4] & 63
        mn[..., :4] = s[..., 4:8] & 63
        sc[..., 4:] = (s[..., 8:12] & 15) | ((s[..., 0:4] >> 6) << 4)
        mn[..., 4:] = (s[..., 8:12] >> 4) | ((s[..., 4:8] >> 6) << 4)
        qh = b[..., 16:48].astype(np.int64)                                # [N][nb][32]
        qs = b[..., 48:176].reshape(N, K // 256, 4, 32).astype(np.int64)
        nib = np.stack([qs & 15, qs >> 4], axis=3)                         # [g][h][l]
        bit = np.stack([(qh[..., None, :] >> (2 * np.arange(4)[:, None] + h)) & 1 for h in (0, 1)], axis=3)
        q = (nib | (bit << 4)).reshape(N, K // 256, 8, 32)                 # sub-block j = 2g + h
        w = d[..., None, None] * sc[..., None] * q - dmin[..., None, None] * mn[..., None]
        return w.reshape(N, K)
    if fmt == "q2_k":
        b = W.reshape(N, K // 256, 84)
        s = b[..., 0:16].astype(np.int64)
        d = indep_f16(b[..., 80:82].copy().view(np.uint16)[..., 0])
        dmin = indep_f16(b[..., 82:84].copy().view(np.uint16)[..., 0])
        qs = b[..., 16:80].reshape(N, K // 256, 2, 1, 32).astype(np.int64)
        q = ((qs >> (2 * np.arange(4)[None, None, None, :, None])) & 3).reshape(N, K // 256, 256)
        scale = np.repeat(s & 15, 16, axis=-1)
        mins = np.repeat(s >> 4, 16, axis=-1)
        w = d[..., None] * scale * q - dmin[..., None] * mins
        return w.reshape(N, K)
    raise ValueError(fmt)


def pack_q4k_scales(sc: list[int], m: list[int]) -> np.ndarray:
    """12 bytes holding eight 6-bit scales and mins (inverse of the unpack rule)."""
    s = np.zeros(12, dtype=np.uint8)
    for j in range(4):
        s[j] = (sc[j] & 63) | ((sc[j + 4] >> 4) << 6)
        s[j + 4] = (m[j] & 63) | ((m[j + 4] >> 4) << 6)
        s[j + 8] = (sc[j + 4] & 15) | ((m[j + 4] & 15) << 4)
    return s


# ------------------------------------------------------------------ pins

def pin_hand_blocks(lib):
    """Hand-built blocks decode to their hand-derived values."""
    for name, fmt, K, raw, expect in hand_blocks():
        got = oracle.dequant(fmt, np.frombuffer(raw, dtype=np.uint8), K, lib=lib)[0]
        assert got.shape[0] == len(expect), name
        np.testing.assert_array_equal(got.astype(np.float64), np.array(expect), err_msg=name)


def pin_f16_exhaustive(lib):
    """All 65,536 fp16 codes decode as numpy's IEEE binary16 does."""
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = indep_f16(codes)
    got = np.array([lib.lwq_oracle_f16(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def pin_bf16_exhaustive(lib):
    """All 65,536 bf16 codes decode as torch.bfloat16 does."""
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = indep_bf16(codes)
    got = np.array([lib.lwq_oracle_bf16(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def pin_q4k_scale_roundtrip(lib):
    """pack(sc, m) -> 12 bytes -> unpack returns (sc, m): all-0, all-63, single bits, random."""
    cases = [([0] * 8, [0] * 8), ([63] * 8, [63] * 8)]
    for j in range(8):
        for bit in range(6):
            sc = [0] * 8
            mm = [0] * 8
            sc[j] = 1 << bit
            cases.append((sc, [0] * 8))
            mm[j] = 1 << bit
            cases.append(([0] * 8, mm))
    g = np.random.default_rng(1234)
    for _ in range(2000):
        cases.append((list(g.integers(0, 64, 8)), list(g.integers(0, 64, 8))))
    for sc, mm in cases:
        s = pack_q4k_scales(sc, mm)
        for j in range(8):
            assert oracle.q4k_scale_min(s, j, lib=lib) == (sc[j], mm[j]), (sc, mm, j)


def pin_roundtrip_q8_0(lib):
    """Quantize -> oracle decode stays within the Q8_0 rounding bound on 10^5 random blocks."""
    g = np.random.default_rng(7)
    w = (g.standard_normal((3125, 1024), dtype=np.float32) * np.float32(0.02)).astype(np.float32)
    Wq = inputs.quantize_q8_0(w)
    got = oracle.dequant("q8_0", Wq, 1024, lib=lib).astype(np.float64)
    wb = w.reshape(-1, 32).astype(np.float64)
    d32 = np.abs(w.reshape(-1, 32)).max(axis=1).astype(np.float32) / np.float32(127)
    d16 = d32.astype(np.float16).astype(np.float64)
    d32 = d32.astype(np.float64)
    # |w - q d| <= |w - q d32| + |q| |d32 - d| <= d32/2 + 127 |d32 - d|  (+ fp32 slop)
    bound = d32 / 2 + 127 * np.abs(d32 - d16) + 4 * np.spacing(np.abs(wb).max(axis=1).astype(np.float32))
    err = np.abs(got.reshape(-1, 32) - wb).max(axis=1)
    assert np.all(err <= bound), float((err - bound).max())


def pin_roundtrip_q4_0(lib):
    """Quantize -> oracle decode stays within the Q4_0 rounding bound on 10^5 random blocks."""
    g = np.random.default_rng(8)
    w = (g.standard_normal((3125, 1024), dtype=np.float32) * np.float32(0.02)).astype(np.float32)
    Wq = inputs.quantize_q4_0(w)
    got = oracle.dequant("q4_0", Wq, 1024, lib=lib).astype(np.float64).reshape(-1, 32)
    wb = w.reshape(-1, 32).astype(np.float64)
    idx = np.abs(wb).argmax(axis=1)
    amax = wb[np.arange(wb.shape[0]), idx]
    d32 = (amax.astype(np.float32) / np.float32(-8)).astype(np.float64)
    d16 = d32.astype(np.float16).astype(np.float64)
    slop = 4 * np.spacing(np.abs(wb).max(axis=1).astype(np.float32))
    # codes within [0, 15]: |w - (q-8)d| <= |d32|/2 + 8|d32 - d|; the clamped code 16 -> 15 adds |d32|/2
    bound = np.abs(d32) + 8 * np.abs(d32 - d16) + slop
    err = np.abs(got - wb).max(axis=1)
    assert np.all(err <= bound), float((err - bound).max())
    # the element equal to amax decodes to -8 d exactly
    got_amax = got[np.arange(wb.shape[0]), idx]
    np.testing.assert_array_equal(got_amax, (-8.0 * d16).astype(np.float32).astype(np.float64))


def pin_bruteforce_one_block(lib):
    """K = one block, N, M <= 3: oracle y equals Python-loop sums over an independent decode."""
    g = np.random.default_rng(99)
    for fmt, K in (("q8_0", 32), ("q4_0", 32), ("q4_k", 256), ("q6_k", 256), ("q5_k", 256), ("q2_k", 256)):
        for act in ("f32", "f16", "bf16"):
            for M, N in ((1, 1), (2, 3), (3, 2)):
                Wq = inputs.make_weights(fmt, g, N, K)
                x = inputs.activations(g, M, K, act)
                y, den = oracle.matmul(fmt, Wq, x, K=K, act=act, lib=lib)
                W = indep_decode(fmt, Wq, K)
                W32 = W.astype(np.float32).astype(np.float64)  # the oracle rounds w once to fp32
                xd = {"f32": lambda a: a.astype(np.float64), "f16": lambda a: a.astype(np.float64),
                      "bf16": indep_bf16}[act](x)
                for m in range(M):
                    for n in range(N):
                        acc = 0.0
                        acc_abs = 0.0
                        for k in range(K):
                            p = float(xd[m, k]) * float(W32[n, k])
                            acc += p
                            acc_abs += abs(p)
                        assert y[m, n] == acc, (fmt, act, m, n, y[m, n], acc)
                        assert den[m, n] == acc_abs, (fmt, act, m, n)


def pin_library_matmul(lib):
    """Oracle y equals torch.matmul (fp64) of the independently decoded W, to 1e-12 relative to den."""
    g = np.random.default_rng(5)
    for fmt, K in (("q8_0", 512), ("q4_0", 512), ("q4_k", 512), ("q6_k", 512), ("q5_k", 512), ("q2_k", 512)):
        for act in ("f32", "f16", "bf16"):
            M, N = 5, 37
            Wq = inputs.make_weights(fmt, g, N, K)
            x = inputs.activations(g, M, K, act)
            y, den = oracle.matmul(fmt, Wq, x, act=act, lib=lib)
            W = torch.from_numpy(indep_decode(fmt, Wq, K).astype(np.float32).astype(np.float64))
            xd = torch.from_numpy(indep_bf16(x) if act == "bf16" else x.astype(np.float64))
            ref = (xd @ W.T).numpy()
            ref_den = (xd.abs() @ W.abs().T).numpy()
            assert np.all(np.abs(y - ref) <= 1e-12 * ref_den), fmt
            assert np.all(np.abs(den - ref_den) <= 1e-12 * ref_den), fmt


def pin_linearity(lib):
    """y(a x1 + b x2) == a y(x1) + b y(x2) exactly when every sum is exact (dyadic grid)."""
    g = np.random.default_rng(11)
    K, N = 256, 9
    # blocks with power-of-two d and small-integer x: every partial sum is exact in fp64
    for fmt in ("q8_0", "q4_0", "q4_k"):
        Wq = inputs.make_weights(fmt, g, N, K).reshape(N, -1).copy()
        bb, bw = inputs.BLOCK_BYTES[fmt], inputs.BLOCK_WEIGHTS[fmt]
        blk = Wq.reshape(N, K // bw, bb)
        e = g.integers(-8, -2, size=blk.shape[:2])
        dcode = (np.exp2(e).astype(np.float16)).view(np.uint16)
        blk[..., 0:2] = dcode.view(np.uint8).reshape(blk.shape[:2] + (2,))
        if fmt == "q4_k":
            blk[..., 2:4] = (np.exp2(e - 1).astype(np.float16)).view(np.uint16).view(np.uint8).reshape(blk.shape[:2] + (2,))
        Wq = blk.reshape(N, -1)
        x1 = g.integers(-8, 9, size=(3, K)).astype(np.float32)
        x2 = g.integers(-8, 9, size=(3, K)).astype(np.float32)
        a, b = np.float32(2.0), np.float32(-0.5)
        y1, _ = oracle.matmul(fmt, Wq, x1, lib=lib)
        y2, _ = oracle.matmul(fmt, Wq, x2, lib=lib)
        y12, _ = oracle.matmul(fmt, Wq, (a * x1 + b * x2).astype(np.float32), lib=lib)
        np.testing.assert_array_equal(y12, 2.0 * y1 - 0.5 * y2, err_msg=fmt)
        # a unit vector picks out one decoded weight: y(e_k)[n] == w_hat[n][k]
        W = oracle.dequant(fmt, Wq, K, lib=lib)
        ks = [0, 1, 15, 16, 17, 31, 32, 100, 255]
        eye = np.zeros((len(ks), K), dtype=np.float32)
        eye[np.arange(len(ks)), ks] = 1.0
        ye, _ = oracle.matmul(fmt, Wq, eye, lib=lib)
        np.testing.assert_array_equal(ye, W[:, ks].T.astype(np.float64), err_msg=fmt)


def pin_zero_denominator(lib):
    """All-eight Q4_0 rows and zero activations give y == 0 and den == 0 exactly."""
    K, N = 128, 4
    blk = np.zeros((N, K // 32, 18), dtype=np.uint8)
    blk[..., 0:2] = np.frombuffer(bytes.fromhex("003c"), dtype=np.uint8)
    blk[..., 2:] = 0x88
    x = np.random.default_rng(3).standard_normal((2, K)).astype(np.float32)
    y, den = oracle.matmul("q4_0", blk.reshape(N, -1), x, lib=lib)
    assert np.all(y == 0) and np.all(den == 0)
    Wq = inputs.make_weights("q4_k", np.random.default_rng(4), N, 256)
    y, den = oracle.matmul("q4_k", Wq, np.zeros((2, 256), dtype=np.float16), lib=lib)
    assert np.all(y == 0) and np.all(den == 0)
    # Q6_K: every code 32 (low nibbles 0, high bits 2) is zero whatever the scales and d
    blk = np.asarray(inputs.make_weights("q6_k", np.random.default_rng(5), N, 512)).reshape(N, 2, 210).copy()
    blk[..., 0:128] = 0
    blk[..., 128:192] = 0xAA
    y, den = oracle.matmul("q6_k", blk.reshape(N, -1), np.random.default_rng(6).standard_normal((2, 512)).astype(np.float32), lib=lib)
    assert np.all(y == 0) and np.all(den == 0)


def pin_sampled_equals_full(lib):
    """The sampled entry point returns bit-identical values to the full product."""
    g = np.random.default_rng(21)
    for fmt, K in (("q8_0", 256), ("q4_0", 288), ("q4_k", 512), ("q6_k", 768), ("q5_k", 512), ("q2_k", 256)):
        M, N = 3, 23
        Wq = inputs.make_weights(fmt, g, N, K)
        x = inputs.activations(g, M, K, "f16")
        y, den = oracle.matmul(fmt, Wq, x, lib=lib)
        ms = g.integers(0, M, 40)
        ns = g.integers(0, N, 40)
        ys, dens = oracle.matmul_sampled(fmt, Wq, x, ms, ns, lib=lib)
        np.testing.assert_array_equal(ys, y[ms, ns])
        np.testing.assert_array_equal(dens, den[ms, ns])


def pin_row_bytes(lib):
    for fmt, K, rb in (("q8_0", 4096, 4352), ("q4_0", 4096, 2304), ("q4_k", 4096, 2304),
                       ("q4_0", 11008, 6192), ("q4_k", 11008, 6192), ("q8_0", 14336, 15232)):
        assert lib.lwq_oracle_row_bytes(oracle.FMT[fmt], K) == rb
    for fmt, K, rb in (("q6_k", 4096, 3360), ("q6_k", 11008, 9030), ("q5_k", 4096, 2816), ("q2_k", 4096, 1344)):
        assert lib.lwq_oracle_row_bytes(oracle.FMT[fmt], K) == rb
    assert lib.lwq_oracle_row_bytes(oracle.FMT["q4_k"], 128) == -1
    assert lib.lwq_oracle_row_bytes(oracle.FMT["q4_0"], 48) == -1
    assert lib.lwq_oracle_row_bytes(oracle.FMT["q6_k"], 288) == -1


# ------------------------------------------------------ decode attention pins

def _f16(a):
    return np.asarray(a, dtype=np.float16)


def pin_attn_one_key(lib):
    """One key: its softmax weight is 1, so out is that key's value row exactly (den its |row|)."""
    q, k, v, _ = inputs.attention_problem(2, 4, 2, 5, 16, "f16", seed=1)
    out, den = oracle.attention(q, k, v, [1, 1], 0.25, lib=lib)
    for b in range(2):
        for h in range(4):
            np.testing.assert_array_equal(out[b, h], v[b, h // 2, 0].astype(np.float64))
            np.testing.assert_array_equal(den[b, h], np.abs(v[b, h // 2, 0].astype(np.float64)))


def pin_attn_zero_query_is_mean(lib):
    """q = 0 makes every score 0: out is the plain mean of the value rows of the sequence."""
    q, k, v, _ = inputs.attention_problem(1, 2, 1, 9, 8, "f16", seed=2)
    q[:] = 0
    out, _ = oracle.attention(q, k, v, [7], 0.3, lib=lib)
    ref = v[0, 0, :7].astype(np.float64).mean(axis=0)
    assert np.allclose(out[0, 0], ref, rtol=0, atol=1e-15)


def pin_attn_two_keys(lib):
    """Scores 0 and s: out = (v0 + e^s v1) / (1 + e^s)."""
    D = 4
    q = np.zeros((1, 1, D), dtype=np.float16)
    q[0, 0, 0] = 1.0
    k = np.zeros((1, 1, 2, D), dtype=np.float16)
    k[0, 0, 1, 0] = 1.0986328125          # an fp16 value near ln 3
    v = _f16([[[[1, 2, -3, 0.5], [5, -6, 7, 0.25]]]])
    out, _ = oracle.attention(q, k, v, [2], 1.0, lib=lib)
    r = math.exp(1.0986328125)
    ref = (v[0, 0, 0].astype(np.float64) + r * v[0, 0, 1].astype(np.float64)) / (1 + r)
    assert np.allclose(out[0, 0], ref, rtol=1e-15, atol=0)


def pin_attn_dominant_key(lib):
    """A score 1000 above every other one takes all the weight (exp(-1000) is 0 in fp64), and
    the maximum is subtracted first (exp(1000) would overflow)."""
    q, k, v, _ = inputs.attention_problem(1, 1, 1, 6, 8, "f16", seed=3)
    q[:] = 0
    q[0, 0, 0] = 1.0
    k[0, 0, :, 0] = 0
    k[0, 0, 4, 0] = 1000.0
    out, _ = oracle.attention(q, k, v, [6], 1.0, lib=lib)
    np.testing.assert_array_equal(out[0, 0], v[0, 0, 4].astype(np.float64))


def pin_attn_gqa_heads(lib):
    """Query head h reads kv head h / (H / Hkv): value rows all 2^g in kv head g give out = 2^g."""
    q, k, v, _ = inputs.attention_problem(2, 6, 3, 5, 8, "bf16", seed=4)
    for g in range(3):
        v[:, g] = inputs.f32_to_bf16_bits(np.full((2, 5, 8), 2.0 ** g, dtype=np.float32))
    out, _ = oracle.attention(q, k, v, [5, 3], 0.5, act="bf16", lib=lib)
    for h in range(6):
        assert np.all(out[:, h] == 2.0 ** (h // 2)), h


def pin_attn_linear_in_v(lib):
    """out is linear in the value rows (small halves: the sums of two caches are exact in fp16)."""
    g = np.random.default_rng(5)
    q, k, _, _ = inputs.attention_problem(1, 2, 2, 11, 8, "f16", seed=5)
    v1 = _f16(g.integers(-8, 9, size=(1, 2, 11, 8)) / 2)
    v2 = _f16(g.integers(-8, 9, size=(1, 2, 11, 8)) / 2)
    o1, _ = oracle.attention(q, k, v1, [11], 0.35, lib=lib)
    o2, _ = oracle.attention(q, k, v2, [11], 0.35, lib=lib)
    o12, _ = oracle.attention(q, k, _f16(v1.astype(np.float32) + v2.astype(np.float32)), [11], 0.35, lib=lib)
    assert np.allclose(o12, o1 + o2, rtol=0, atol=1e-13)


def pin_attn_length_respected(lib):
    """Keys past a sequence's length change nothing."""
    q, k, v, _ = inputs.attention_problem(2, 2, 2, 12, 8, "f16", seed=6)
    out, _ = oracle.attention(q, k, v, [5, 12], 0.4, lib=lib)
    k2, v2 = k.copy(), v.copy()
    k2[0, :, 5:] = 60000.0
    v2[0, :, 5:] = -60000.0
    out2, _ = oracle.attention(q, k2, v2, [5, 12], 0.4, lib=lib)
    np.testing.assert_array_equal(out, out2)


def pin_attn_logsumexp_bruteforce(lib):
    """Tiny case against Python floats in the log-sum-exp form: out = sum_j exp(s_j - lse) v_j."""
    q, k, v, _ = inputs.attention_problem(1, 2, 1, 3, 4, "f16", seed=7)
    scale = 0.7
    out, _ = oracle.attention(q, k, v, [3], scale, lib=lib)
    for h in range(2):
        s = [scale * sum(float(q[0, h, d]) * float(k[0, 0, j, d]) for d in range(4)) for j in range(3)]
        lse = math.log(sum(math.exp(x) for x in s))
        ref = [sum(math.exp(s[j] - lse) * float(v[0, 0, j, d]) for j in range(3)) for d in range(4)]
        assert np.allclose(out[0, h], ref, rtol=1e-13, atol=1e-15)


ALL_PINS = [pin_hand_blocks, pin_f16_exhaustive, pin_bf16_exhaustive, pin_q4k_scale_roundtrip,
            pin_roundtrip_q8_0, pin_roundtrip_q4_0, pin_bruteforce_one_block, pin_library_matmul,
            pin_linearity, pin_zero_denominator, pin_sampled_equals_full, pin_row_bytes,
            pin_attn_one_key, pin_attn_zero_query_is_mean, pin_attn_two_keys, pin_attn_dominant_key,
            pin_attn_gqa_heads, pin_attn_linear_in_v, pin_attn_length_respected, pin_attn_logsumexp_bruteforce]
