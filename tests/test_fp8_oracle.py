"""Pins for the CPU statement of the FP8 latent cache (oracle/fp8_cache.py),
without a GPU: the E4M3 format from its definition, nearest rounding by brute
force, the per-token power-of-two scale, and the error bound of the encoding.
"""
import math

import numpy as np
import pytest
import torch

from oracle import fp8_cache as f8


def test_known_codes():
    # from the format: bias 7, 3 mantissa bits, subnormals m * 2^-9
    assert f8.e4m3_value(0x00) == 0.0
    assert f8.e4m3_value(0x01) == 2.0 ** -9
    assert f8.e4m3_value(0x07) == 7 * 2.0 ** -9
    assert f8.e4m3_value(0x08) == 2.0 ** -6
    assert f8.e4m3_value(0x38) == 1.0
    assert f8.e4m3_value(0x39) == 1.125
    assert f8.e4m3_value(0x7E) == 448.0
    assert f8.e4m3_value(0xFE) == -448.0
    assert math.isnan(f8.e4m3_value(0x7F)) and math.isnan(f8.e4m3_value(0xFF))
    assert math.copysign(1.0, f8.e4m3_value(0x80)) == -1.0
    finite = [c for c in range(256) if not math.isnan(f8.e4m3_value(c))]
    assert len(finite) == 254


def test_every_finite_code_round_trips():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)])
    vals = f8.decode_codes(codes)
    np.testing.assert_array_equal(f8.e4m3_round(vals), codes.astype(np.uint8))


def brute_nearest(y):
    """argmin over all finite codes of |value - y|, ties to the even code."""
    best = None
    for c in range(256):
        v = f8.e4m3_value(c)
        if math.isnan(v) or (c & 0x80) != (0x80 if math.copysign(1.0, y) < 0 else 0):
            continue
        d = abs(v - y)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0 and best[1] % 2 == 1):
            best = (d, c)
    return best[1]


def test_rounding_matches_brute_force():
    g = np.random.default_rng(0)
    mags = np.ldexp(g.random(400) + 0.5, g.integers(-12, 9, size=400))
    ys = np.concatenate([mags, -mags, [0.0, -0.0, 448.0, 2.0 ** -10, 2.0 ** -11, 3 * 2.0 ** -11]])
    ys = ys[np.abs(ys) <= 448]
    got = f8.e4m3_round(ys)
    for y, c in zip(ys, got):
        assert c == brute_nearest(y), y


def test_ties_go_to_even_codes():
    codes = np.arange(0x00, 0x7E)
    lo, hi = f8.decode_codes(codes), f8.decode_codes(codes + 1)
    mid = (lo + hi) / 2
    got = f8.e4m3_round(mid)
    want = np.where(codes % 2 == 0, codes, codes + 1)
    np.testing.assert_array_equal(got, want.astype(np.uint8))
    np.testing.assert_array_equal(f8.e4m3_round(-mid), (want | 0x80).astype(np.uint8))


@pytest.mark.parametrize("amax", [1e-30, 0.001, 0.75, 1.0, 3.9, 224.0, 224.5, 448.0, 449.0,
                                  1e4, 3.0e38])
def test_scale_exponent_is_the_smallest_fitting_power(amax):
    k = f8.scale_exponent(amax)
    assert amax <= 448.0 * 2.0 ** k
    assert amax > 448.0 * 2.0 ** (k - 1)
    assert 224.0 < amax * 2.0 ** -k <= 448.0


def test_encoding_error_is_half_a_step():
    g = torch.Generator().manual_seed(3)
    rows = (torch.randn((40, 576), generator=g) * torch.logspace(-3, 3, 40)[:, None]).to(
        torch.bfloat16).double().numpy()
    codes, scales = f8.encode_rows(rows)
    deq = f8.dequantize(codes, scales)
    for x, d, s in zip(rows, deq, scales):
        # E4M3 spacing is 2^-3 relative for normal values and 2^-9 absolute below
        # 2^-6, scaled by s; nearest rounding is off by at most half of that
        bound = np.maximum(np.abs(x) * 2.0 ** -4, s * 2.0 ** -10)
        assert np.all(np.abs(x - d) <= bound)
        assert np.max(np.abs(d)) <= 448 * s
        assert np.max(np.abs(x)) > 224 * s
    # the dequantised values are exact in bf16 (4 significant bits times a power of two)
    t = torch.from_numpy(deq)
    assert torch.equal(t.to(torch.bfloat16).double(), t)


def test_zero_row_and_signed_zero():
    codes, scale = f8.encode_row(np.zeros(576))
    assert scale == 1.0 and not codes.any()
    # row max 1.0: the smallest k with 1 <= 448 * 2^k is -8, and 1.0 * 2^8 = 256
    # is code 0x78 (exponent field 15, mantissa 0); -1e-9 * 2^8 rounds to -0
    codes, scale = f8.encode_row(np.array([-1e-9, 1.0] + [0.0] * 574))
    assert scale == 2.0 ** -8
    assert codes[0] == 0x80 and codes[1] == 0x78 and not codes[2:].any()


MUTATIONS = {
    "ties_to_odd": ("(_POS_CODES[hi] % 2 == 0)", "(_POS_CODES[hi] % 2 == 1)"),
    "scale_one_step_small": ("    return k\n", "    return k - 1\n"),
    "sign_dropped": ("np.where(np.signbit(y), 0x80, 0)", "np.where(np.signbit(y), 0, 0)"),
    "subnormal_step_wrong": ("return sign * m * 2.0 ** -9", "return sign * m * 2.0 ** -10"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_reject_mutation(name, tmp_path):
    import importlib.util
    old, new = MUTATIONS[name]
    src = open(f8.__file__).read()
    assert src.count(old) >= 1, old
    path = tmp_path / f"mut_{name}.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"mut_{name}", path)
    failed = False
    try:
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        saved = f8.__dict__.copy()
        f8.__dict__.update({k: v for k, v in mod.__dict__.items() if not k.startswith("__")})
        try:
            for t in (test_known_codes, test_every_finite_code_round_trips,
                      test_rounding_matches_brute_force, test_ties_go_to_even_codes,
                      test_encoding_error_is_half_a_step, test_grid_rounding_equals_table_rounding):
                t()
            for a in (0.75, 224.5, 1e4):
                test_scale_exponent_is_the_smallest_fitting_power(a)
        finally:
            f8.__dict__.update(saved)
    except (AssertionError, ValueError):
        failed = True
    assert failed, f"mutation {name} went undetected"


def test_block_encoder_equals_row_encoder():
    g = torch.Generator().manual_seed(5)
    rows = (torch.randn((50, 576), generator=g) * torch.logspace(-5, 5, 50)[:, None]).to(
        torch.bfloat16).double().numpy()
    codes, scales = f8.encode_rows(rows, chunk=7)
    for n in range(50):
        c, s = f8.encode_row(rows[n])
        np.testing.assert_array_equal(codes[n], c)
        assert scales[n] == s


def test_block_scale_rule_equals_scalar_rule():
    amax = np.concatenate([[0.0, 448.0, 392.0, 392.0001, 224.0, 1.0, 0.875, 0.8750001],
                           np.ldexp(np.random.default_rng(1).random(2000) + 0.5,
                                    np.random.default_rng(2).integers(-140, 120, 2000))])
    rows = np.zeros((amax.size, 576))
    rows[:, 7] = amax
    _, scales = f8.encode_rows(rows, chunk=333)
    for a, s in zip(amax, scales):
        assert s == 2.0 ** f8.scale_exponent(a), a


def test_grid_rounding_equals_table_rounding():
    g = np.random.default_rng(4)
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)])
    vals = f8.decode_codes(codes)
    lo, hi = f8.decode_codes(np.arange(0, 0x7E)), f8.decode_codes(np.arange(1, 0x7F))
    mids = (lo + hi) / 2
    rand = np.ldexp(g.random(200000) + 0.5, g.integers(-14, 9, 200000))
    rand = rand[rand <= 448] * np.where(g.random(rand.size) < 0.5, -1, 1)
    for y in (vals, mids, -mids, rand, np.array([0.0, -0.0, 2.0 ** -12, -2.0 ** -12])):
        np.testing.assert_array_equal(f8.e4m3_round_grid(y), f8.e4m3_round(y))


def test_format_agrees_with_torch_float8_e4m3fn():
    # an independent implementation of the same format (OCP E4M3, "fn": no
    # infinities, NaN at S.1111.111): every code's value, and nearest-even
    # rounding of float32 values inside the range, including exact midpoints
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    lib_vals = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = f8.decode_codes(codes.numpy())
    finite = ~np.isnan(lib_vals)
    assert finite.sum() == 254
    np.testing.assert_array_equal(np.isnan(ours), ~finite)
    np.testing.assert_array_equal(ours[finite], lib_vals[finite])
    np.testing.assert_array_equal(np.signbit(ours[finite]), np.signbit(lib_vals[finite]))

    g = np.random.default_rng(7)
    mags = np.ldexp(g.random(20000) + 0.5, g.integers(-14, 9, size=20000)).astype(np.float32)
    vals = np.sort(f8.decode_codes(np.arange(0x00, 0x7F)))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)      # exact in float32
    ys = np.concatenate([mags, -mags, mids, -mids]).astype(np.float32)
    ys = ys[np.abs(ys) <= 448]
    lib_codes = torch.from_numpy(ys).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(f8.e4m3_round(ys.astype(np.float64)), lib_codes)
