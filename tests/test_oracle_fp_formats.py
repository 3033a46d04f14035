"""Pins of the oracle's fp8 (E4M3 + one fp16 scale per vector) and nvfp4 (E2M1
+ an E4M3 scale per 16 values) codecs, against things other than the oracle:

- E4M3 decode of all 256 codes and E4M3 encode against torch's float8_e4m3fn
  conversion (a library routine);
- E2M1 decode against the value list of the format (0, 0.5, 1, 1.5, 2, 3, 4, 6)
  and E2M1 encode against a brute-force nearest-value search with ties to the
  even code;
- the quantisers' scales against numpy / torch conversions of max|x| / 448 and
  max|x| / 6, their error bounds, and the byte counts printed on the pages
  (516 and 288 bytes per position).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")
E2M1_VALUES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _torch_e4m3(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    got = oracle.e4m3_to_f32(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2          # S.1111.111
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(40)
    x = np.concatenate([
        rng.standard_normal(20000) * np.exp(rng.uniform(-12, 6, 20000)),
        oracle.e4m3_to_f32(np.arange(256, dtype=np.uint8)),                  # every grid value
        # midpoints between neighbours: ties go to the even code
        (oracle.e4m3_to_f32(np.arange(0, 126, dtype=np.uint8)).astype(np.float64)
         + oracle.e4m3_to_f32(np.arange(1, 127, dtype=np.uint8))) / 2,
        [0.0, -0.0, 2.0 ** -10, 2.0 ** -10 * 3, 447.9, -447.9, 448.0, -448.0],
    ]).astype(np.float32)
    x = x[np.isfinite(x) & (np.abs(x) <= 448.0)]
    assert np.array_equal(oracle.f32_to_e4m3(x), _torch_e4m3(x))


def test_e4m3_encode_saturates():
    x = np.array([449.0, 463.9, 464.0, 1e6, 3e38, -500.0, -1e9], np.float32)
    got = oracle.f32_to_e4m3(x)
    assert np.array_equal(got, np.array([0x7E] * 5 + [0xFE] * 2, np.uint8))


def test_e2m1_decode_is_the_value_list():
    got = oracle.e2m1_to_f32(np.arange(16, dtype=np.uint8))
    assert np.array_equal(got[:8], np.array(E2M1_VALUES, np.float32))
    assert np.array_equal(got[8:], -np.array(E2M1_VALUES, np.float32))
    assert np.signbit(got[8])                                               # code 8 is -0


def _e2m1_brute(v: float) -> int:
    a = min(abs(v), 6.0)
    best = None
    for code, val in enumerate(E2M1_VALUES):
        d = abs(a - val)
        if best is None or d < best[0] or (d == best[0] and code % 2 == 0):
            best = (d, code)
    return best[1] | (8 if np.signbit(v) else 0)


def test_e2m1_encode_matches_brute_force():
    rng = np.random.default_rng(41)
    x = np.concatenate([rng.uniform(-8, 8, 5000), rng.standard_normal(2000),
                        np.arange(-70, 71) / 10.0, [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -5.0, 7.0, -0.0]])
    x = x.astype(np.float32)
    want = np.array([_e2m1_brute(float(v)) for v in x], np.uint8)
    assert np.array_equal(oracle.f32_to_e2m1(x), want)


def test_quant_fp8_scale_codes_and_error_bound():
    rng = np.random.default_rng(42)
    for i in range(100):
        x = (rng.standard_normal(256) * np.exp(rng.uniform(-10, 8))).astype(np.float32)
        if i == 0:
            x[:] = 0
        c, s = oracle.quant_fp8(x)
        amax = np.float32(np.max(np.abs(x)))
        want_s = np.array([np.float32(amax / np.float32(448.0))], np.float32).astype(np.float16).view(np.uint16)
        assert s[0] == want_s[0]
        d = np.float32(np.float16(s.view(np.float16)[0]))
        if d == 0:
            assert np.all(c == 0)
            continue
        assert np.array_equal(c, _torch_e4m3(np.clip(x / d, -448, 448)))
        xhat = oracle.e4m3_to_f32(c).astype(np.float64) * d
        # E4M3 keeps 3 fraction bits: error <= 2^-4 of the value (normals) or
        # half a subnormal step 2^-10 d, plus the fp16 rounding of d
        bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * d) + np.abs(x) * 2.0 ** -10
        assert np.all(np.abs(xhat - x) <= bound)
        assert np.array_equal(oracle.dequant_rows("e4m3", c[None], s[None])[0], xhat)


def test_quant_nvfp4_scales_codes_and_error_bound():
    rng = np.random.default_rng(43)
    for i in range(100):
        x = (rng.standard_normal(256) * np.exp(rng.uniform(-8, 8))).astype(np.float32)
        if i == 0:
            x[16:32] = 0                                                      # a zero block
        c, s = oracle.quant_nvfp4(x)
        xb = x.reshape(16, 16)
        amax = np.max(np.abs(xb), axis=1).astype(np.float32)
        # saturating conversion: torch gives NaN past 448, so clip first
        assert np.array_equal(s.astype(np.uint8), _torch_e4m3(np.minimum(amax / np.float32(6.0), 448.0)))
        sd = torch.from_numpy(s.astype(np.uint8)).view(torch.float8_e4m3fn).float().numpy()
        for b in range(16):
            blk = c[16 * b:16 * b + 16]
            if sd[b] == 0:
                assert np.all(blk == 0)
                continue
            want = np.array([_e2m1_brute(float(np.float32(v / sd[b]))) for v in xb[b]], np.uint8)
            assert np.array_equal(blk, want)
            xhat = oracle.e2m1_to_f32(blk).astype(np.float64) * sd[b]
            # inside +-6 s the E2M1 grid step is at most 2 s (between 4 and 6),
            # so the error is at most s; above it the value saturates to 6 s
            # (the scale can round below max|x| / 6, and far below it when it
            # falls into E4M3's subnormal range)
            ax = np.abs(xb[b]).astype(np.float64)
            bound = np.maximum(1.0 * sd[b], ax - 6.0 * sd[b]) * (1 + 1e-6)
            assert np.all(np.abs(xhat - xb[b]) <= bound)
            assert np.all(np.abs(xhat) <= 6.0 * sd[b])
        got = oracle.dequant_rows("e2m1", c[None], s[None])[0]
        assert np.array_equal(got, oracle.e2m1_to_f32(c).astype(np.float64) * np.repeat(sd.astype(np.float64), 16))


def test_fp_formats_byte_counts_are_the_printed_ones():
    g = json.load(open(GOLDEN))
    assert oracle.format_bytes_per_token_head("fp8") == g["fp8_kv_bytes_per_position"]["bytes_per_position"]
    f = g["four_bit_16_value_fp8_scale_kv"]
    assert oracle.format_bytes_per_token_head("nvfp4") == f["bytes_per_position"]
    per_token = f["positions_per_token"] * oracle.format_bytes_per_token_head("nvfp4")
    assert round(per_token * 163840 / 2 ** 30, 2) == f["gib_at_163840"]
    assert round(per_token * 262144 / 2 ** 30, 2) == f["gib_at_262144"]


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_fp_formats_are_not_rotated(fmt):
    rng = np.random.default_rng(44)
    k = rng.standard_normal((2, 256)).astype(np.float32)
    v = rng.standard_normal((2, 256)).astype(np.float32)
    kc, ks, vc, vs = oracle.append_rows(fmt, k, v)
    q = oracle.QUANT[oracle.PARTS[fmt][0]]
    for i in range(2):
        ck, sk = q(k[i])
        cv, sv = q(v[i])
        assert np.array_equal(kc[i], ck) and np.array_equal(ks[i], sk)
        assert np.array_equal(vc[i], cv) and np.array_equal(vs[i], sv)
