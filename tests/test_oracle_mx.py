"""Pins for the oracle's MX formats (oracle/mx.py) against published values,
hand-computed roundings, exhaustive round trips and closed-form invariants."""
import math
import os

import numpy as np
import pytest

from oracle import mx

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mx_formats.txt")


def _golden():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        fmt, code, val = line.split()
        rows.append((fmt, int(code, 0), float(val)))
    return rows


def _same(a, b):
    if math.isnan(b):
        return math.isnan(a)
    return a == b and math.copysign(1, a) == math.copysign(1, b)


def test_published_values():
    for fmt, code, val in _golden():
        if fmt == "e2m1":
            got = mx.E2M1_TABLE[code]
            assert _same(got, val), (fmt, code, got, val)
            assert _same(mx.E2M1_TABLE[code | 8], -val)      # sign bit is bit 3
        elif fmt == "e4m3":
            assert _same(mx.E4M3_TABLE[code], val), (fmt, hex(code))
        else:
            assert _same(float(mx.e8m0_value(code)), val), (fmt, code)


def test_e4m3_structure():
    t = mx.E4M3_TABLE
    finite = t[~np.isnan(t)]
    assert len(finite) == 254                       # 256 codes minus two NaNs
    assert np.max(finite) == 448.0 and np.min(finite) == -448.0
    pos = t[:127]
    assert np.all(np.diff(pos) > 0)                 # code order is value order
    # spacing: 2^-9 in the subnormal range and the first binade, doubling after
    assert pos[1] - pos[0] == 2.0 ** -9
    assert pos[16] - pos[15] == 2.0 ** -9
    assert pos[126] - pos[125] == 32.0


def test_e2m1_rne_cases():
    # block whose amax makes the scale exponent 0 for E2M1: amax in [4, 8)
    cases = {2.5: 2.0, 5.0: 4.0, 0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0,
             7.0: 6.0, 6.5: 6.0, 2.75: 3.0, 3.5: 4.0, 0.3: 0.5, -2.5: -2.0}
    for v, want in cases.items():
        blk = np.zeros(32)
        blk[0] = 4.0
        blk[1] = v
        codes, sc = mx.quantize_mx(blk[None], "e2m1")
        assert sc[0, 0] == 127
        assert mx.E2M1_TABLE[codes[0, 1]] == want, (v, mx.E2M1_TABLE[codes[0, 1]])


def test_e2m1_saturation_block():
    # {7, 0, ...}: floor(log2 7) = 2 = emax -> scale 2^0, and 7 saturates to 6
    blk = np.zeros(32)
    blk[0] = 7.0
    codes, sc = mx.quantize_mx(blk[None], "e2m1")
    assert sc[0, 0] == 127 and codes[0, 0] == 7 and mx.E2M1_TABLE[7] == 6.0


def test_e4m3_rne_and_saturation():
    blk = np.zeros(32)
    blk[0] = 480.0 * 2.0 ** 5                       # amax in [2^8, 2^9) * 2^5 -> e = 5
    blk[1] = 17.0 * 2.0 ** 5                        # tie between 16 and 18 -> 16 (even)
    blk[2] = 19.0 * 2.0 ** 5                        # tie between 18 and 20 -> 20 (even)
    blk[3] = -(2.0 ** -10) * 2.0 ** 5               # tiny negative -> -0 (sign kept)
    blk[4] = 3.0 * 2.0 ** -10 * 2.0 ** 5            # 1.5 * 2^-9 tie -> 2^-8 (even code 2)
    codes, sc = mx.quantize_mx(blk[None], "e4m3")
    assert sc[0, 0] == 127 + 5
    vals = mx.E4M3_TABLE[codes[0]]
    assert vals[0] == 448.0 and codes[0, 0] == 0x7E
    assert vals[1] == 16.0 and vals[2] == 20.0
    assert codes[0, 3] == 0x80
    assert vals[4] == 2.0 ** -8


def test_zero_block_and_signed_zero():
    blk = np.zeros((1, 32))
    blk[0, 3] = -0.0
    codes, sc = mx.quantize_mx(blk, "e4m3")
    assert sc[0, 0] == 0
    assert codes[0, 3] == 0x80 and np.all(np.delete(codes[0], 3) == 0)


@pytest.mark.parametrize("fmt,table,emax,maxcode", [
    ("e2m1", mx.E2M1_TABLE, 2, 7), ("e4m3", mx.E4M3_TABLE, 8, 0x7E)])
def test_round_trip_every_code_and_scale(fmt, table, emax, maxcode):
    """Every finite code times 2^s, in a block that also holds the max code,
    quantises back to the same code and scale byte 127+s."""
    codes = [c for c in range(len(table)) if not np.isnan(table[c])]
    for s in range(-10, 11):
        for start in range(0, len(codes), 31):
            chunk = codes[start:start + 31]
            blk_codes = np.array([maxcode] + chunk + [0] * (31 - len(chunk)))
            vals = table[blk_codes] * 2.0 ** s
            q, sc = mx.quantize_mx(vals[None], fmt)
            assert sc[0, 0] == 127 + s
            assert np.array_equal(q[0], blk_codes.astype(np.uint8)), (fmt, s, start)


def test_scale_covariance():
    rng = np.random.default_rng(0)
    v = rng.standard_normal((4, 64)) * 3
    for fmt in ("e4m3", "e2m1"):
        q0, s0 = mx.quantize_mx(v, fmt)
        for n in (-7, 1, 13):
            q1, s1 = mx.quantize_mx(v * 2.0 ** n, fmt)
            assert np.array_equal(q0, q1)
            assert np.array_equal(s1.astype(int), s0.astype(int) + n)


def test_quantisation_error_bound():
    """|v - dequant(quant(v))| <= half a code step at the block's scale, except
    for saturated elements (which land on the max magnitude)."""
    rng = np.random.default_rng(1)
    v = rng.standard_normal((16, 256))
    for fmt, mant, emax, mxv in (("e4m3", 3, 8, 448.0), ("e2m1", 1, 2, 6.0)):
        q, s = mx.quantize_mx(v, fmt)
        r = mx.dequantize_mx(q, s, fmt)
        scale = np.repeat(mx.e8m0_value(s), 32, axis=-1)
        a = np.abs(v) / scale
        # step at |a|: 2^(floor(log2 a) - mant), floor at the subnormal step
        sub_exp = 1 - (7 if fmt == "e4m3" else 1)
        ex = np.floor(np.log2(np.maximum(a, 2.0 ** sub_exp)))
        step = 2.0 ** (ex - mant) * scale
        ok = (np.abs(v - r) <= step / 2 + 1e-300) | (a >= mxv)
        assert np.all(ok), fmt
        # the scale exponent is floor(log2 amax) - emax
        amax = np.max(np.abs(v.reshape(16, -1, 32)), axis=-1)
        assert np.array_equal(s.astype(int) - 127, np.floor(np.log2(amax)).astype(int) - emax)


def test_nibble_packing():
    codes = np.arange(16, dtype=np.uint8)[None].repeat(2, 0)
    p = mx.pack_e2m1(codes)
    assert p.shape == (2, 8) and p[0, 0] == 0x10 and p[0, 7] == 0xFE
    assert np.array_equal(mx.unpack_e2m1(p), codes)


def test_bf16_round():
    import torch
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.standard_normal(10000) * 10.0 ** rng.integers(-30, 30, 10000),
                        [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -1.0 - 2.0 ** -8, 0.0]])
    got = mx.bf16_round(v)
    # exact fp64 -> bf16 rounding checked against torch for values that are exact in fp32
    v32 = v.astype(np.float32)
    exact = v32.astype(np.float64) == v
    ref = torch.from_numpy(v32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(got[exact], ref[exact])
    assert got[-4] == 1.0 and got[-3] == 1.0 + 2.0 ** -6 and got[-2] == -1.0
    # a value a hair above the tie rounds up (no double rounding through fp32)
    hair = 1.0 + 2.0 ** -8 + 2.0 ** -40
    assert mx.bf16_round(np.array([hair]))[0] == 1.0 + 2.0 ** -7


# ------------------------------------------------------------------ the C restatement (oracle/cmx.c)
def test_c_quantiser_matches_the_numpy_definition():
    """oracle/cmx.c restates quantize_mx for fp32 input; it must give the same codes and
    scales on random data over a wide range of magnitudes, on ties and saturation, and on
    signed zeros and bf16/fp32 subnormals."""
    from oracle import cmx
    g = np.random.default_rng(12)
    x = (g.standard_normal((64, 512)) * np.logspace(-40, 38, 512)[None, :]).astype(np.float32)
    x[0] = 0.0
    x[1, :32] = -0.0
    x[2, :32] = np.float32(448.0 * 2.0 ** 10)
    x[3, :32] *= np.float32(1e-38)
    x[3, 5] = np.float32(2.0 ** -149)                    # fp32 subnormal
    x[4, :32] = [17.0, 19.0, -17.0, 480.0] * 8           # E4M3 ties and saturation
    x[5, :32] = [2.5, 5.0, 0.25, 0.75, 1.25, 1.75, -2.5, 7.0] * 4   # E2M1 ties
    # every E2M1 / E4M3 value times a spread of scales, and the midpoints between them
    vals = np.concatenate([mx._E2M1_POS, -mx._E2M1_POS, mx._E4M3_POS, -mx._E4M3_POS])
    mids = (mx._E4M3_POS[1:] + mx._E4M3_POS[:-1]) / 2
    extra = np.concatenate([vals, mids, -mids])
    extra = np.resize(extra, (len(extra) + 31) // 32 * 32).reshape(-1, 32)
    extra = np.concatenate([extra * 2.0 ** s for s in (-20, -3, 0, 5, 30)]).astype(np.float32)
    for data in (x, extra, g.standard_normal((300, 96)).astype(np.float32) * 0.02):
        for fmt in ("e2m1", "e4m3"):
            c1, s1 = cmx.quantize_mx_f32(data, fmt)
            c0, s0 = mx.quantize_mx(data, fmt)
            assert np.array_equal(s1, s0), fmt
            assert np.array_equal(c1, c0), fmt


def test_c_quantiser_round_trips_every_code():
    """Every finite code of both formats, scaled by 2^s: quantising the decoded value gives
    back the code and the scale (the exhaustive pin of quantize_mx, applied to the C
    restatement)."""
    from oracle import cmx
    for fmt, top in (("e2m1", 8), ("e4m3", 127)):
        pos = mx._E2M1_POS if fmt == "e2m1" else mx._E4M3_POS
        for s in (-20, 0, 17):
            for c in range(1, top):
                # block: the largest code sets the scale, the tested code sits beside it
                blk = np.zeros(32)
                blk[0] = pos[top - 1] * 2.0 ** s
                blk[1] = pos[c] * 2.0 ** s
                blk[2] = -pos[c] * 2.0 ** s
                codes, scales = cmx.quantize_mx_f32(blk[None, :].astype(np.float32), fmt)
                assert scales[0, 0] == s + 127       # amax = largest value x 2^s: exponent s
                dec = mx.dequantize_mx(codes, scales, fmt)
                assert dec[0, 1] == blk[1] and dec[0, 2] == blk[2], (fmt, s, c)


def test_c_decoder_matches_the_numpy_definition():
    """oracle/cmx.c's decoder gives dequantize_mx's values: every code with a spread of
    scale bytes, the NaN scale (0xFF) and the E4M3 NaN codes included."""
    from oracle import cmx
    g = np.random.default_rng(13)
    for fmt, ncodes in (("e2m1", 16), ("e4m3", 256)):
        codes = g.integers(0, ncodes, size=(64, 256)).astype(np.uint8)
        codes[0, :ncodes] = np.arange(ncodes)
        scales = g.integers(0, 256, size=(64, 8)).astype(np.uint8)
        scales[1] = 255
        scales[2] = [0, 1, 126, 127, 128, 253, 254, 255]
        a = cmx.dequantize_mx_f64(codes, scales, fmt)
        b = mx.dequantize_mx(codes, scales, fmt)
        assert np.array_equal(a, b, equal_nan=True), fmt
