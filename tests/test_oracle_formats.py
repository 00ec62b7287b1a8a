"""Pins of the oracle's number formats against library casts, the formats'
closed-form tables and brute-force nearest-value search."""
import numpy as np
import pytest
import torch

from oracle import csa_oracle as O


def _rng(s=0):
    return np.random.default_rng(s)


# ---------------------------------------------------------------- BF16

def test_bf16_matches_torch_cast():
    r = _rng(1)
    x = np.concatenate([
        r.standard_normal(20000).astype(np.float32) * 10.0,
        # exact ties between two BF16 neighbours (low 16 bits == 0x8000)
        (np.arange(1, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, 1e-38], dtype=np.float32),
    ])
    ours = O.bf16_bits_from_f32(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(O.bf16_value(ours),
                          torch.from_numpy(ours.view(np.int16)).view(torch.bfloat16)
                          .to(torch.float64).numpy())


# ---------------------------------------------------------------- FP8 E4M3

def test_e4m3_decode_all_codes_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_value(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2                         # 0x7F and 0xFF
    assert np.array_equal(ours[~nan], ref[~nan])
    assert O.e4m3_value(np.uint8(0x7E)) == 448.0   # largest finite
    assert O.e4m3_value(np.uint8(0x01)) == 2.0 ** -9
    assert O.e4m3_value(np.uint8(0x08)) == 2.0 ** -6


def test_e4m3_encode_matches_torch_cast_in_range():
    r = _rng(2)
    finite = O.e4m3_value(np.arange(0, 0x7F, dtype=np.uint8))   # 0 .. 448
    mids = (finite[1:] + finite[:-1]) / 2.0                      # exact ties
    x = np.concatenate([r.uniform(-448, 448, 30000), r.standard_normal(30000) * 1e-2,
                        mids, -mids, finite, -finite, [0.0, -0.0]])
    x = x.astype(np.float32)
    ours = O.e4m3_code(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_saturates_and_is_nearest():
    assert O.e4m3_code(1e6) == 0x7E and O.e4m3_code(-1e6) == 0xFE
    assert O.e4m3_code(464.0) == 0x7E                 # tie 448/480 -> even (448)
    vals = O.e4m3_value(np.arange(0, 0x7F, dtype=np.uint8))
    r = _rng(3)
    for y in r.uniform(0, 448, 2000):
        got = O.e4m3_value(O.e4m3_code(y))
        assert abs(got - y) == np.min(np.abs(vals - y))


# ---------------------------------------------------------------- FP4 E2M1 / E8M0

def test_e2m1_table_and_roundtrip():
    mags = O.e2m1_value(np.arange(8, dtype=np.uint8))
    assert list(mags) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]   # OCP MX E2M1 table
    assert list(O.e2m1_value(np.arange(8, 16, dtype=np.uint8))) == [-v for v in mags]
    for c in range(16):
        assert O.e2m1_code(O.e2m1_value(np.uint8(c))) == c


@pytest.mark.parametrize("y,expect", [(0.25, 0.0), (0.75, 1.0), (1.25, 1.0), (1.75, 2.0),
                                      (2.5, 2.0), (3.5, 4.0), (5.0, 4.0), (5.5, 6.0),
                                      (7.0, 6.0), (100.0, 6.0), (-5.0, -4.0), (0.3, 0.5)])
def test_e2m1_ties_to_even_and_saturation(y, expect):
    assert O.e2m1_value(O.e2m1_code(y)) == expect


def test_e2m1_is_nearest_brute_force():
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    for y in _rng(4).uniform(-6, 6, 5000):
        got = O.e2m1_value(O.e2m1_code(y))
        assert abs(got - y) == np.min(np.abs(np.concatenate([mags, -mags]) - y))


def test_ue8m0():
    assert O.ue8m0_value(127) == 1.0
    assert O.ue8m0_value(0) == 2.0 ** -127
    assert O.ue8m0_value(130) == 8.0


# ---------------------------------------------------------------- MXFP4 blocks

def test_mxfp4_scale_rule_and_brute_force():
    r = _rng(5)
    x = r.standard_normal((50, 128)) * np.exp2(r.integers(-6, 6, (50, 1)))
    q = O.quantize_mxfp4(x)
    x32 = O.f32(x).astype(np.float64).reshape(50, 4, 32)
    grid = np.concatenate([O._E2M1_MAGS, -O._E2M1_MAGS])
    for i in range(50):
        for b in range(4):
            amax = np.max(np.abs(x32[i, b]))
            e = int(np.floor(np.log2(amax))) - 2
            assert q.scales[i, b] == e + 127
            # brute force: nearest grid value of x / 2^e, clamped to +-6
            y = x32[i, b] / 2.0 ** e
            for jj in range(32):
                v = O.e2m1_value(q.codes[i, b * 32 + jj])
                assert abs(v - y[jj]) == np.min(np.abs(grid - y[jj]))
    deq = O.dequantize_mxfp4(q)
    # |x / 2^e| < 8: spacing 2 above 4, saturation at 6 -> error below 2 * 2^e
    assert np.all(np.abs(deq - x32.reshape(50, 128)) <
                  np.repeat(np.exp2(q.scales.astype(float) - 127), 32, axis=1) * 2.0)


def test_mxfp4_zero_block():
    q = O.quantize_mxfp4(np.zeros((1, 32)))
    assert q.scales[0, 0] == 127 and np.all(q.codes == 0)


def test_mxfp4_exact_values_roundtrip():
    r = _rng(6)
    codes = r.integers(0, 16, (10, 64)).astype(np.uint8)
    codes[:, 0] = 7                             # amax 6 * 2^e -> exponent e exactly
    codes[:, 32] = 7
    e = r.integers(-10, 10, (10, 2))
    x = O.e2m1_value(codes).reshape(10, 2, 32) * np.exp2(e)[..., None]
    q = O.quantize_mxfp4(x.reshape(10, 64))
    assert np.array_equal(O.dequantize_mxfp4(q), x.reshape(10, 64))


# ---------------------------------------------------------------- KV rows

def test_kv_row_quantiser():
    r = _rng(7)
    D, R = 512, 64
    x = r.standard_normal((40, D)) * 0.3
    kv = O.quantize_kv(x, R)
    deq = O.dequantize_kv(kv)
    # the element of largest magnitude maps to the largest finite code
    amax_idx = np.argmax(np.abs(O.f32(x[:, :-R])), axis=1)
    assert np.all((kv.fp8[np.arange(40), amax_idx] & 0x7F) == 0x7E)
    # E4M3 has 3 mantissa bits: half-ulp relative bound 2^-4 in the normal
    # range; absolute bound of half a subnormal step below it
    err = np.abs(deq[:, :-R] - x[:, :-R])
    bound = np.maximum(np.abs(x[:, :-R]) * 2.0 ** -4, kv.scale[:, None] * 2.0 ** -10) * 1.0001
    assert np.all(err <= bound)
    # the RoPE dims are BF16: exact for BF16-representable input
    xb = O.bf16_round(x)
    assert np.array_equal(O.dequantize_kv(O.quantize_kv(xb, R))[:, -R:], xb[:, -R:])


def test_kv_row_rope_dims_are_torch_bf16():
    """The RoPE dims of a stored row are the BF16 round-to-nearest-even of
    the fp32 value: torch's own cast, ties and all."""
    r = _rng(8)
    D, R = 128, 64
    x = (r.standard_normal((30, D)) * 3.0).astype(np.float32)
    x[:, -R:][:, :8] = (np.arange(1, 9, dtype=np.uint32) << 16 | 0x8000).view(np.float32)   # exact ties
    kv = O.quantize_kv(x.astype(np.float64), R)
    ref = torch.from_numpy(np.ascontiguousarray(x[:, -R:])).to(torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(kv.rope, ref.view(np.uint16))


def test_kv_row_zero():
    kv = O.quantize_kv(np.zeros((1, 128)), 64)
    assert kv.scale[0] == 1.0 and np.all(kv.fp8 == 0)
