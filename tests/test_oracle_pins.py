"""Pins for the CPU oracle: each check ties the oracle to something other than itself.

Sources: values the pages print (golden fixtures), library float conversions
(numpy float16, torch bfloat16 / float8 types), exact rational brute force
(``fractions.Fraction``), closed forms (one-hot inputs, row sums) and invariants
(Q8_0 round-trip error <= scale/2).
"""
import math
import os
import random
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from block_quantized_weight_qgemm_b200 import inputs

E2M1_MAG = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3),
            Fraction(4), Fraction(6)]


# ------------------------------------------------------------------------------------------
# Element / scale decoders
# ------------------------------------------------------------------------------------------

def test_e2m1_table_and_f16_low_byte(golden):
    g = golden("fp4_fp8_exactness.json")
    vals = [oracle.e2m1(c) for c in range(16)]
    assert vals[:8] == g["e2m1_magnitudes"]
    assert vals[8:] == [-v for v in g["e2m1_magnitudes"]]
    assert math.copysign(1.0, vals[8]) == -1.0  # code 8 is negative zero
    # page fact: f16 of every E2M1 value has a zero low byte
    for v in vals:
        bits = int(np.array([v], dtype=np.float16).view(np.uint16)[0])
        assert bits & 0xFF == 0


def test_e4m3_all_bytes_against_torch_and_page_rule(golden):
    g = golden("fp4_fp8_exactness.json")
    allb = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = allb.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    non_nan = 0
    for b in range(256):
        v = oracle.e4m3(b)
        if math.isnan(ref[b]):
            assert math.isnan(v), b
            assert b in g["e4m3_nan_bytes"]
            continue
        non_nan += 1
        assert v == ref[b], (b, v, ref[b])
        # page rule: f16 bits = (byte & 0x7f) << 7, then times 256 (sign separately)
        mag16 = np.array([(b & 0x7F) << 7], dtype=np.uint16).view(np.float16)[0]
        assert float(mag16) * 256.0 == abs(v)
    assert non_nan == g["e4m3_non_nan_bytes"]
    assert oracle.e4m3(0x7E) == g["e4m3_max"]
    assert oracle.e4m3(0x00) == 0.0 and oracle.e4m3(0x01) == 2.0 ** -9 and oracle.e4m3(0x08) == 2.0 ** -6


def test_e4m3_times_e2m1_products_exact_in_f16_and_bf16(golden):
    # page fact: all 254 non-NaN scale bytes x 16 codes are exact in f16 (subnormals incl.)
    count = 0
    for b in range(256):
        s = oracle.e4m3(b)
        if math.isnan(s):
            continue
        for c in range(16):
            p = s * oracle.e2m1(c)  # exact in fp64
            assert float(np.float16(p)) == p, (b, c)
            assert float(torch.tensor(p, dtype=torch.float64).to(torch.float32).to(torch.bfloat16).double()) == p
            count += 1
    assert count == 254 * 16


def test_e8m0_landmarks_and_torch():
    assert oracle.e8m0(0) == 2.0 ** -127
    assert oracle.e8m0(127) == 1.0
    assert oracle.e8m0(254) == 2.0 ** 127
    assert math.isnan(oracle.e8m0(255))
    if hasattr(torch, "float8_e8m0fnu"):
        ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e8m0fnu).to(torch.float64)
        for b in range(255):
            assert oracle.e8m0(b) == float(ref[b])


def test_f16_decode_all_codes_against_numpy():
    ref = np.arange(65536, dtype=np.uint32).astype(np.uint16).view(np.float16).astype(np.float64)
    for h in range(0, 65536, 1):
        v = oracle.f16(h)
        if math.isnan(ref[h]):
            assert math.isnan(v)
        else:
            assert v == ref[h], h


def test_bf16_decode_all_codes_against_torch():
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.bfloat16).to(torch.float64).numpy()
    tab = oracle.bf16_table()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(tab), nan)
    assert np.array_equal(tab[~nan], ref[~nan])


# ------------------------------------------------------------------------------------------
# Encoders
# ------------------------------------------------------------------------------------------

def test_f16_encode_against_numpy_rne():
    rng = np.random.default_rng(0)
    vals = list(rng.standard_normal(4000) * 10.0 ** rng.integers(-9, 5, 4000))
    # exact midpoints between adjacent f16 values (ties to even) and just around them
    for h in list(range(1, 0x7BFF, 97)) + [0x0001, 0x03FF, 0x0400, 0x3C00, 0x7BFE]:
        a, b = oracle.f16(h), oracle.f16(h + 1)
        mid = (a + b) / 2
        vals += [mid, np.nextafter(mid, 0), np.nextafter(mid, np.inf), -mid]
    for v in vals:
        ref = int(np.array([v], dtype=np.float64).astype(np.float16).view(np.uint16)[0])
        if abs(v) >= 65520.0:
            continue  # IEEE overflows to inf; the oracle saturates (checked below)
        assert oracle.f16_encode_satfinite(float(v)) == ref, v
    assert oracle.f16_encode_satfinite(1e9) == 0x7BFF
    assert oracle.f16_encode_satfinite(-1e9) == 0xFBFF


def test_bf16_encode_roundtrip_and_ties():
    for h in list(range(0, 0x7F80, 37)) + [0x0001, 0x007F, 0x0080, 0x3F80, 0x7F7F]:
        assert oracle.bf16_encode(oracle.bf16(h)) == h
        assert oracle.bf16_encode(-oracle.bf16(h)) == (h | 0x8000 if h else 0x8000)
        if h < 0x7F7F:
            a, b = Fraction(oracle.bf16(h)), Fraction(oracle.bf16(h + 1))
            mid = float((a + b) / 2)
            even = h if h % 2 == 0 else h + 1
            assert oracle.bf16_encode(mid) == even
            assert oracle.bf16_encode(float(np.nextafter(mid, 0))) == h
            assert oracle.bf16_encode(float(np.nextafter(mid, np.inf))) == h + 1


def test_e4m3_encode_against_torch_and_ties():
    rng = np.random.default_rng(1)
    vals = np.abs(rng.standard_normal(3000).astype(np.float32) * np.float32(2.0) ** rng.integers(-12, 9, 3000).astype(np.float32))
    vals = vals[vals < 448.0]
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for v, r in zip(vals, ref):
        assert oracle.e4m3_encode_pos(float(v)) == int(r), v
    for b in range(0, 0x7E):
        a, c = Fraction(oracle.e4m3(b)), Fraction(oracle.e4m3(b + 1))
        mid = float((a + c) / 2)
        assert oracle.e4m3_encode_pos(mid) == (b if b % 2 == 0 else b + 1)
    assert oracle.e4m3_encode_pos(449.0) == 0x7E
    assert oracle.e4m3_encode_pos(1e30) == 0x7E


def test_e4m3_signed_encode_against_torch_and_sign_rule():
    # the FP8 weight encoder: torch's float -> float8_e4m3fn conversion (round to nearest even)
    # on values of both signs within the finite range, and the sign rule for zero
    rng = np.random.default_rng(3)
    vals = (rng.standard_normal(4000).astype(np.float32)
            * np.float32(2.0) ** rng.integers(-14, 9, 4000).astype(np.float32))
    vals = vals[np.abs(vals) < 448.0]
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for v, r in zip(vals, ref):
        if int(r) & 0x7F:   # a non-zero result: torch and the oracle agree on sign and magnitude
            assert oracle.e4m3_encode(float(v)) == int(r), v
        else:               # rounds to zero: the oracle keeps the sign bit of v
            assert oracle.e4m3_encode(float(v)) == (0x80 if v < 0 else 0x00), v
    assert oracle.e4m3_encode(-448.0) == 0xFE and oracle.e4m3_encode(-1e9) == 0xFE
    assert oracle.e4m3_encode(-2.0 ** -10) == 0x80 and oracle.e4m3_encode(2.0 ** -10) == 0x00
    assert oracle.e4m3_encode(-(2.0 ** -10 + 2.0 ** -20)) == 0x81  # above half the subnormal step


def _e2m1_nearest_code(v: Fraction) -> int:
    """Brute force: nearest E2M1 magnitude, ties to the even code, saturate at 6."""
    a = abs(v)
    best = min(range(8), key=lambda c: (abs(a - E2M1_MAG[c]), c & 1))
    return (8 if v < 0 else 0) | best


def test_e2m1_encode_brute_force():
    cases = [Fraction(k, 8) for k in range(-64, 65)] + [Fraction(7), Fraction(100), Fraction(-9)]
    rng = random.Random(2)
    cases += [Fraction(rng.uniform(-7, 7)) for _ in range(2000)]
    for v in cases:
        assert oracle.e2m1_encode(float(v)) == _e2m1_nearest_code(v), v
    # the ties named in the reading: 2.5 -> 2, 5 -> 4, 0.25 -> 0, 0.75 -> 1
    assert oracle.e2m1_encode(2.5) == 4 and oracle.e2m1_encode(5.0) == 6
    assert oracle.e2m1_encode(0.25) == 0 and oracle.e2m1_encode(0.75) == 2


# ------------------------------------------------------------------------------------------
# Packers
# ------------------------------------------------------------------------------------------

def _rows_with_specials(N, K, seed):
    W = inputs.weights(N, K, seed=seed).numpy().copy()
    W[0, :32] = 0.0                      # all-zero block
    W[1, 32:64] = 0.0
    W[1, 40] = 1e-3                      # single non-zero element
    W[2, :16] *= 1e-6                    # tiny block
    W[3, 64:96] = np.float32(0.75) * 0.02  # equal elements (ties in the FP4 grids)
    return W


def test_q8_0_pack_invariant_and_scale():
    N, K = 6, 256
    W = _rows_with_specials(N, K, 11)
    codes, scales, _ = oracle.pack("q8_0", W)
    for n in range(N):
        for kb in range(K // 32):
            blk = W[n, kb * 32:(kb + 1) * 32].astype(np.float64)
            h = int(scales[n, 2 * kb]) | (int(scales[n, 2 * kb + 1]) << 8)
            assert h == int(np.array([np.abs(blk).max() / 127.0]).astype(np.float16).view(np.uint16)[0])
            d = Fraction(float(np.array([h], dtype=np.uint16).view(np.float16)[0]))
            q = codes[n, kb * 32:(kb + 1) * 32].view(np.int8).astype(int)
            assert np.all(np.abs(q) <= 127)
            for i in range(32):
                err = abs(Fraction(float(blk[i])) - q[i] * d)
                assert err <= d / 2, (n, kb, i)
            if d == 0:
                assert np.all(q == 0)


def test_nvfp4_pack_brute_force():
    N, K = 5, 128
    W = _rows_with_specials(N, K, 12)
    codes, scales, ts = oracle.pack("nvfp4", W)
    amax = float(np.abs(W.astype(np.float64)).max())
    assert ts == float(np.float32(amax / 2688.0))
    e4m3_vals = [Fraction(oracle.e4m3(b)) for b in range(0x7F)]
    for n in range(N):
        for kb in range(K // 16):
            blk = [Fraction(float(v)) for v in W[n, kb * 16:(kb + 1) * 16]]
            ab = max(abs(v) for v in blk)
            s = int(scales[n, kb])
            if ab == 0:
                assert s == 0
            else:
                target = ab / (6 * Fraction(ts))
                want = min(range(0x7F), key=lambda b: (abs(target - e4m3_vals[b]), b & 1))
                assert s == want, (n, kb)
            sv = e4m3_vals[s]
            for i in range(16):
                byte = int(codes[n, (kb * 16 + i) // 2])
                c = byte & 0xF if i % 2 == 0 else byte >> 4
                if sv == 0:
                    assert c == 0
                else:
                    assert c == _e2m1_nearest_code(blk[i] / (sv * Fraction(ts))), (n, kb, i)


def test_mxfp4_pack_brute_force():
    N, K = 5, 128
    W = _rows_with_specials(N, K, 13)
    W[4, :32] *= 1000.0   # large block: exercises saturation at 6 after scaling
    codes, scales, _ = oracle.pack("mxfp4", W)
    for n in range(N):
        for kb in range(K // 32):
            blk = [Fraction(float(v)) for v in W[n, kb * 32:(kb + 1) * 32]]
            ab = max(abs(v) for v in blk)
            e = int(scales[n, kb])
            if ab == 0:
                assert e == 0
                want_e = 0
            else:
                m, ex = math.frexp(float(ab))
                want_e = min(max(ex - 1 - 2 + 127, 0), 254)
            assert e == want_e
            sc = Fraction(2) ** (e - 127)
            for i in range(32):
                byte = int(codes[n, (kb * 32 + i) // 2])
                c = byte & 0xF if i % 2 == 0 else byte >> 4
                if ab == 0:
                    assert c == 0
                else:
                    assert c == _e2m1_nearest_code(blk[i] / sc), (n, kb, i)


def test_pitches_and_footprint(golden):
    # padded row pitches keep every row start 16-byte aligned
    for fmt in ("q8_0", "nvfp4", "mxfp4"):
        for K in (32, 64, 96, 1024, 5120, 17408):
            if fmt != "nvfp4" and K % 32:
                continue
            assert oracle.code_pitch(fmt, K) % 16 == 0 and oracle.scale_pitch(fmt, K) % 16 == 0
    # model-card fact: 22.7B MXFP4 params occupy ~12.05B packed bytes (17/32 B per param)
    g = golden("mxfp4_footprint.json")
    K = 17408
    per_param = (oracle.code_pitch("mxfp4", K) + oracle.scale_pitch("mxfp4", K)) / K
    assert per_param == 17 / 32
    assert abs(g["params_approx_g"] * per_param - g["packed_u8_bytes_approx_g"]) < 0.02


# ------------------------------------------------------------------------------------------
# Dequantisation and GEMM
# ------------------------------------------------------------------------------------------

def test_fp8_pack_brute_force():
    # per-tensor scale ts = fp32(amax/448); each code the E4M3 value nearest to w/ts in exact
    # arithmetic (ties to the even code, saturating at 448), with the sign of w
    N, K = 5, 96
    W = _rows_with_specials(N, K, 14)
    W[4, 5] = -np.abs(W).max() * 1.5      # the matrix maximum is negative
    W[4, 6] = np.float32(1e-12)           # far below the smallest subnormal step
    W[4, 7] = np.float32(-1e-12)
    codes, scales, ts = oracle.pack("fp8", W)
    assert scales.shape == (N, 0)
    amax = float(np.abs(W.astype(np.float64)).max())
    assert ts == float(np.float32(amax / 448.0))
    vals = [Fraction(oracle.e4m3(b)) for b in range(0x7F)]   # the finite non-negative values
    for n in range(N):
        for k in range(K):
            q = Fraction(float(W[n, k])) / Fraction(ts)
            want = min(range(0x7F), key=lambda b: (abs(abs(q) - vals[b]), b & 1))
            want |= 0x80 if q < 0 else 0
            assert int(codes[n, k]) == want, (n, k)
    assert int(codes[4, 5]) == 0xFE      # -amax -> -448 (saturated after the fp32 rounding of ts)
    assert int(codes[4, 6]) == 0x00 and int(codes[4, 7]) == 0x80
    # a zero matrix: ts = 0 and all codes 0
    c0, _, t0 = oracle.pack("fp8", np.zeros((2, 32), dtype=np.float32))
    assert t0 == 0.0 and not c0.any()


def test_dequant_hand_built_rows():
    K = 32
    # Q8_0: codes -127, 1, 5 with scale 1.0 (0x3C00) and 0.5 (0x3800) in block 2
    codes = np.zeros((1, oracle.code_pitch("q8_0", 64)), dtype=np.uint8)
    scales = np.zeros((1, oracle.scale_pitch("q8_0", 64)), dtype=np.uint8)
    codes[0, 0] = np.uint8(0x81)
    codes[0, 1] = 1
    codes[0, 33] = 5
    scales[0, 0:2] = [0x00, 0x3C]
    scales[0, 2:4] = [0x00, 0x38]
    Wd = oracle.dequant("q8_0", codes, scales, 1.0, 1, 64)
    assert Wd[0, 0] == -127.0 and Wd[0, 1] == 1.0 and Wd[0, 33] == 2.5 and Wd[0, 2] == 0.0
    # NVFP4: element 0 = low nibble of byte 0; scale 0x38 = 1.0; ts = 0.5
    codes = np.zeros((1, oracle.code_pitch("nvfp4", K)), dtype=np.uint8)
    scales = np.zeros((1, oracle.scale_pitch("nvfp4", K)), dtype=np.uint8)
    codes[0, 0] = 0x7F          # element 0: 0xF (-6), element 1: 0x7 (+6)
    codes[0, 8] = 0x01          # element 16: 0x1 (0.5)
    scales[0, 0] = 0x38
    scales[0, 1] = 0x40         # e4m3 0x40 = 2.0
    Wd = oracle.dequant("nvfp4", codes, scales, 0.5, 1, K)
    assert Wd[0, 0] == -3.0 and Wd[0, 1] == 3.0 and Wd[0, 16] == 0.5 and Wd[0, 17] == 0.0
    # MXFP4: e = 128 -> 2.0
    codes = np.zeros((1, oracle.code_pitch("mxfp4", K)), dtype=np.uint8)
    scales = np.zeros((1, oracle.scale_pitch("mxfp4", K)), dtype=np.uint8)
    codes[0, 0] = 0x97          # element 0: 0x7 (6), element 1: 0x9 (-0.5)
    scales[0, 0] = 128
    Wd = oracle.dequant("mxfp4", codes, scales, 1.0, 1, K)
    assert Wd[0, 0] == 12.0 and Wd[0, 1] == -1.0
    # FP8: E4M3 0x38 = 1.0, 0xC0 = -2.0, 0x7E = 448, 0x01 = 2^-9, 0x80 = -0; ts = 0.25
    codes = np.zeros((1, oracle.code_pitch("fp8", K)), dtype=np.uint8)
    scales = np.zeros((1, 0), dtype=np.uint8)
    codes[0, :5] = [0x38, 0xC0, 0x7E, 0x01, 0x80]
    Wd = oracle.dequant("fp8", codes, scales, 0.25, 1, K)
    assert list(Wd[0, :6]) == [0.25, -0.5, 112.0, 2.0 ** -11, 0.0, 0.0]


def _fraction_gemm(x16, Wd):
    B, K = x16.shape
    N = Wd.shape[0]
    xf = [[Fraction(oracle.bf16(int(x16[b, k]))) for k in range(K)] for b in range(B)]
    wf = [[Fraction(float(Wd[n, k])) for k in range(K)] for n in range(N)]
    return [[sum(xf[b][k] * wf[n][k] for k in range(K)) for n in range(N)] for b in range(B)]


@pytest.mark.parametrize("fmt", ["q8_0", "nvfp4", "mxfp4", "fp8"])
@pytest.mark.parametrize("K", [32, 64])
def test_gemm_brute_force_rational(fmt, K):
    N, B = 4, 3
    W = inputs.weights(N, K, seed=21).numpy()
    codes, scales, ts = oracle.pack(fmt, W)
    Wd = oracle.dequant(fmt, codes, scales, ts, N, K)
    x16 = inputs.bf16_bits(inputs.activations(B, K, seed=22))
    y = oracle.gemm(x16, Wd, nthreads=2)
    exact = _fraction_gemm(x16, Wd)
    for b in range(B):
        for n in range(N):
            bound = K * 2.0 ** -52 * float(sum(abs(Fraction(oracle.bf16(int(x16[b, k]))) * Fraction(float(Wd[n, k])))
                                               for k in range(K)))
            assert abs(Fraction(float(y[b, n])) - exact[b][n]) <= Fraction(bound)


@pytest.mark.parametrize("fmt", ["q8_0", "nvfp4", "mxfp4", "fp8"])
def test_gemm_one_hot_and_ones(fmt):
    N, K = 7, 96
    W = inputs.weights(N, K, seed=23).numpy()
    codes, scales, ts = oracle.pack(fmt, W)
    Wd = oracle.dequant(fmt, codes, scales, ts, N, K)
    cols = [0, 1, 15, 16, 31, 32, 33, 95]
    x16 = inputs.bf16_bits(inputs.one_hot(len(cols), K, cols))
    y = oracle.gemm(x16, Wd)
    for b, c in enumerate(cols):
        assert np.array_equal(y[b], Wd[:, c])       # exact: one non-zero product
    ones = inputs.bf16_bits(torch.ones(1, K, dtype=torch.bfloat16))
    y1 = oracle.gemm(ones, Wd)
    for n in range(N):
        assert abs(y1[0, n] - math.fsum(Wd[n])) <= 1e-15 * max(1.0, float(np.abs(Wd[n]).sum()))


def test_gemm_chunked_equals_unchunked(golden):
    # the PR's boundary matrix, replayed on the oracle: 70 = 64 + 6, 256 = 4 x 64
    g = golden("q8_boundary_matrix.json")
    N, K = 8, 64
    W = inputs.weights(N, K, seed=24).numpy()
    codes, scales, ts = oracle.pack("q8_0", W)
    Wd = oracle.dequant("q8_0", codes, scales, ts, N, K)
    x16 = inputs.bf16_bits(inputs.activations(256, K, seed=25))
    full = oracle.gemm(x16, Wd)
    for width in g["widths"]:
        parts = g["chunk_decompositions"].get(str(width), [width])
        rows, o = [], 0
        for p in parts:
            rows.append(oracle.gemm(x16[o:o + p], Wd))
            o += p
        assert np.array_equal(np.concatenate(rows), full[:width])


def test_normalised_error_metric():
    x16 = inputs.bf16_bits(torch.tensor([[3.0, 4.0]], dtype=torch.bfloat16))
    Wd = np.array([[1.0, 0.0], [0.0, 0.0]])
    y_ref = np.array([[3.0, 0.0]])
    assert oracle.normalised_error(y_ref + np.array([[0.05, 0.0]]), y_ref, x16, Wd) == pytest.approx(0.01)
    assert oracle.normalised_error(y_ref + np.array([[0.0, 0.5]]), y_ref, x16, Wd) == pytest.approx(0.5)


# ------------------------------------------------------------------------------------------
# Fused FFN
# ------------------------------------------------------------------------------------------

def test_silu_closed_forms():
    assert oracle.silu(0.0) == 0.0
    assert oracle.silu(1.0) == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-15)
    assert oracle.silu(-40.0) == pytest.approx(-40.0 * math.exp(-40.0), rel=1e-9)
    assert oracle.silu(40.0) == pytest.approx(40.0, rel=1e-15)


def test_ffn_special_cases_and_rounding():
    M, K, N = 3, 64, 5
    x16 = inputs.bf16_bits(inputs.activations(M, K, seed=31))
    Wg = oracle.dequant("nvfp4", *oracle.pack("nvfp4", inputs.weights(N, K, seed=32).numpy()), N, K)
    Wu = oracle.dequant("nvfp4", *oracle.pack("nvfp4", inputs.weights(N, K, seed=33).numpy()), N, K)
    zero = np.zeros_like(Wg)
    _, _, h = oracle.ffn_gate_up(x16, zero, Wu)
    assert np.all((h & 0x7FFF) == 0)           # SiLU(0) * u = 0
    _, _, h = oracle.ffn_gate_up(x16, Wg, zero)
    assert np.all((h & 0x7FFF) == 0)
    g, u, h = oracle.ffn_gate_up(x16, Wg, Wu)
    assert np.array_equal(g, oracle.gemm(x16, Wg)) and np.array_equal(u, oracle.gemm(x16, Wu))
    for i in range(M):
        for j in range(N):
            v = g[i, j] / (1.0 + math.exp(-g[i, j])) * u[i, j]
            hv = Fraction(oracle.bf16(int(h[i, j])))
            lo = Fraction(oracle.bf16(int(h[i, j]) - 1)) if (int(h[i, j]) & 0x7FFF) else -hv
            # h is the bf16 value nearest to v: no neighbour is closer
            assert abs(Fraction(v) - hv) <= abs(Fraction(v) - Fraction(oracle.bf16(int(h[i, j]) + 1)))
            assert abs(Fraction(v) - hv) <= abs(Fraction(v) - lo)


# --------------------------------------------------------------------------------------
# the pins catch planted mistakes: each variant of the oracle is compiled with one known
# error (ORC_MUTATE) and run through the same checks, which must now fail
# --------------------------------------------------------------------------------------
def _mutant(tmp_path, m):
    import ctypes
    import subprocess
    src = os.path.join(os.path.dirname(oracle.__file__), "qgemm_oracle.c")
    so = str(tmp_path / ("liboracle_mut%d.so" % m))
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-fno-fast-math",
                           "-ffp-contract=off", "-pthread", "-DORC_MUTATE=%d" % m, src, "-o", so,
                           "-lm"])
    lib = ctypes.CDLL(so)
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    lib.orc_dequant.argtypes = [ctypes.c_int, vp, vp, ctypes.c_float, i64, i64, vp]
    lib.orc_gemm.argtypes = [vp, i64, i64, vp, i64, vp, ctypes.c_int]
    return lib


def _dequant_with(lib, fmt, codes, scales, ts, N, K):
    Wd = np.zeros((N, K), dtype=np.float64)
    lib.orc_dequant(oracle.FORMATS[fmt], codes.ctypes.data, scales.ctypes.data, ts, N, K,
                    Wd.ctypes.data)
    return Wd


def _hand_rows_hold(lib):
    # the hand-built rows of test_dequant_hand_built_rows, through `lib`
    K = 64
    ok = True
    codes = np.zeros((1, oracle.code_pitch("q8_0", K)), dtype=np.uint8)
    scales = np.zeros((1, oracle.scale_pitch("q8_0", K)), dtype=np.uint8)
    codes[0, 0] = 0x81
    codes[0, 1] = 1
    scales[0, 0:2] = [0x00, 0x3C]  # fp16 1.0
    Wd = _dequant_with(lib, "q8_0", codes, scales, 1.0, 1, K)
    ok &= bool(Wd[0, 0] == -127.0 and Wd[0, 1] == 1.0)
    codes = np.zeros((1, oracle.code_pitch("nvfp4", K)), dtype=np.uint8)
    scales = np.zeros((1, oracle.scale_pitch("nvfp4", K)), dtype=np.uint8)
    codes[0, 0] = 0x7F
    scales[0, 0] = 0x38
    Wd = _dequant_with(lib, "nvfp4", codes, scales, 0.5, 1, K)
    ok &= bool(Wd[0, 0] == -3.0 and Wd[0, 1] == 3.0)
    codes = np.zeros((1, oracle.code_pitch("fp8", K)), dtype=np.uint8)
    scales = np.zeros((1, 16), dtype=np.uint8)
    codes[0, :2] = [0x38, 0xC0]
    Wd = _dequant_with(lib, "fp8", codes, scales, 0.25, 1, K)
    ok &= bool(Wd[0, 0] == 0.25 and Wd[0, 1] == -0.5)
    return ok


def _gemm_matches_fractions(lib):
    N, K, B = 4, 32, 3
    W = inputs.weights(N, K, seed=21).numpy()
    codes, scales, ts = oracle.pack("q8_0", W)
    Wd = oracle.dequant("q8_0", codes, scales, ts, N, K)
    x16 = np.ascontiguousarray(inputs.bf16_bits(inputs.activations(B, K, seed=22)))
    y = np.zeros((B, N), dtype=np.float64)
    lib.orc_gemm(x16.ctypes.data, B, K, Wd.ctypes.data, N, y.ctypes.data, 1)
    exact = _fraction_gemm(x16, Wd)
    return all(abs(Fraction(float(y[b, n])) - exact[b][n]) <= Fraction(1e-12)
               for b in range(B) for n in range(N))


def test_pins_catch_planted_mistakes(tmp_path):
    assert _hand_rows_hold(_mutant(tmp_path, 0)) and _gemm_matches_fractions(_mutant(tmp_path, 0))
    assert not _hand_rows_hold(_mutant(tmp_path, 1))        # nibble order swapped
    assert not _hand_rows_hold(_mutant(tmp_path, 2))        # NVFP4 tensor scale dropped
    assert not _gemm_matches_fractions(_mutant(tmp_path, 3))  # last term of each sum dropped
    assert not _hand_rows_hold(_mutant(tmp_path, 4))        # Q8_0 scale bytes swapped
    assert not _hand_rows_hold(_mutant(tmp_path, 5))        # FP8 tensor scale dropped
    assert not _hand_rows_hold(_mutant(tmp_path, 6))        # FP8 sign bit ignored


# ------------------------------------------------------------------------------------------
# Activation split for a block-scaled MMA (the decision input of the block-scaled path)
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("elem,top", [("e4m3", 7), ("e2m1", 2)])
def test_activation_split_first_term_brute_force(elem, top):
    # one term: each element is the code value nearest to x / 2^e (ties to the even code,
    # saturating), e = floor(log2 max|block|) - top, computed here from the definitions
    x16 = inputs.bf16_bits(inputs.activations(3, 96, seed=51))
    xs = oracle.split_x(x16, elem, 1)
    if elem == "e4m3":
        vals = [Fraction(oracle.e4m3(b)) for b in range(0x7F)]
    else:
        vals = [Fraction(v) for v in E2M1_MAG]
    for b in range(3):
        for k0 in range(0, 96, 32):
            blk = [Fraction(oracle.bf16(int(v))) for v in x16[b, k0:k0 + 32]]
            amax = max(abs(v) for v in blk)
            _, ex = math.frexp(float(amax))
            sc = Fraction(2) ** ((ex - 1) - top)
            for i, v in enumerate(blk):
                a = abs(v) / sc
                best = min(range(len(vals)), key=lambda c: (abs(a - vals[c]), c & 1))
                want = vals[best] * sc * (1 if v >= 0 else -1)
                assert Fraction(float(xs[b, k0 + i])) == want, (b, k0 + i)


def test_activation_split_accuracy_for_the_block_scaled_path():
    # the 1e-3 bar of the method, for x ~ N(0, 1) in bf16 and NVFP4 / MXFP4 weights, at the
    # 27B FFN reduction lengths: one E4M3 term is not enough, two are exact for all but a
    # handful of elements; three E2M1 terms keep a wide margin
    for K in (5120, 17408):
        x16 = inputs.bf16_bits(inputs.activations(4, K, seed=52))
        xd = oracle.bf16_decode_array(x16)
        for fmt in ("nvfp4", "mxfp4"):
            W = inputs.weights(16, K, seed=53).numpy()
            Wd = oracle.dequant(fmt, *oracle.pack(fmt, W), 16, K)
            y = oracle.gemm(x16, Wd)
            err = {}
            for elem, t in (("e4m3", 1), ("e4m3", 2), ("e4m3", 3), ("e2m1", 3), ("e2m1", 4)):
                xs = oracle.split_x(x16, elem, t)
                err[(elem, t)] = oracle.normalised_error(oracle.gemm_f64(xs, Wd), y, x16, Wd)
            assert err[("e4m3", 1)] > 1e-4
            assert err[("e4m3", 2)] < 1e-8 and err[("e4m3", 3)] < 1e-10
            assert err[("e2m1", 3)] < 2e-4 and err[("e2m1", 4)] < 2e-5
            assert np.array_equal(oracle.split_x(x16, "e4m3", 3), xd)  # three terms: exact


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "fp8"])
def test_block_scaled_split_first_term_brute_force(fmt):
    # one term, from the definitions: xe = floor(log2 max|row|) - xshift, each block's
    # e = floor(log2 max|x 2^-xe|) - top, the nearest code value of x 2^-xe / 2^e (E2M1, top 2,
    # or E4M3, top 7; ties to the even code, saturating), times 2^e 2^xe; blocks with e below the
    # smallest scale are zero
    blk, xshift, emin, elem, _ = oracle.BS_SPLIT[fmt]
    top = 7 if elem == 0 else 2
    x = inputs.activations(3, 96, seed=61)
    x[1, 16:32] *= 2.0 ** -40  # a block far below its row maximum
    x16 = inputs.bf16_bits(x)
    xs = oracle.split_x_bs(x16, fmt, 1)
    vals = ([Fraction(oracle.e4m3(b)) for b in range(0x7F)] if elem == 0
            else [Fraction(v) for v in E2M1_MAG])
    for b in range(3):
        row = [Fraction(oracle.bf16(int(v))) for v in x16[b]]
        _, ex = math.frexp(float(max(abs(v) for v in row)))
        xe = (ex - 1) - xshift
        for k0 in range(0, 96, blk):
            r = [v / Fraction(2) ** xe for v in row[k0:k0 + blk]]
            _, ex = math.frexp(float(max(abs(v) for v in r)))
            e = (ex - 1) - top
            for i, v in enumerate(r):
                if e < emin:
                    want = Fraction(0)
                else:
                    a = abs(v) / Fraction(2) ** e
                    best = min(range(len(vals)), key=lambda c: (abs(a - vals[c]), c & 1))
                    want = vals[best] * Fraction(2) ** (e + xe) * (1 if v >= 0 else -1)
                assert Fraction(float(xs[b, k0 + i])) == want, (fmt, b, k0 + i)
    if fmt == "nvfp4":
        assert not xs[1, 16:32].any()  # 2^-40 below the maximum: below the UE4M3 range


def test_block_scaled_split_prescale_invariance_and_mxfp4_reduction():
    # a power-of-two factor on a row scales its split by the same factor (the prescale absorbs
    # it); with MXFP4's parameters and no dropped block the split is the plain per-block peel
    x = inputs.activations(4, 640, seed=62)
    x16 = inputs.bf16_bits(x)
    for fmt in ("mxfp4", "nvfp4", "fp8"):
        base = oracle.split_x_bs(x16, fmt)
        for k in (-60, 7, 90):
            xk = inputs.bf16_bits(x * 2.0 ** k)
            assert np.array_equal(oracle.split_x_bs(xk, fmt), np.ldexp(base, k)), (fmt, k)
    assert np.array_equal(oracle.split_x_bs(x16, "mxfp4", 3), oracle.split_x(x16, "e2m1", 3))
    assert np.array_equal(oracle.split_x_bs(x16, "fp8", 2), oracle.split_x(x16, "e4m3", 2))


def test_block_scaled_split_accuracy():
    # three E2M1 terms (FP4 weights) and two E4M3 terms (FP8 weights) stay well inside the
    # 1e-3 bar at the 27B lengths
    for K in (5120, 17408):
        x16 = inputs.bf16_bits(inputs.activations(4, K, seed=63))
        for fmt in ("nvfp4", "mxfp4", "fp8"):
            W = inputs.weights(16, K, seed=64).numpy()
            Wd = oracle.dequant(fmt, *oracle.pack(fmt, W), 16, K)
            y = oracle.gemm(x16, Wd)
            err = oracle.normalised_error(oracle.gemm_f64(oracle.split_x_bs(x16, fmt), Wd), y, x16, Wd)
            assert err < (1e-8 if fmt == "fp8" else 2e-4), (K, fmt, err)
