"""Pins of the C oracle to things other than itself.

Every check here compares the oracle with an independent fact: a library
routine (numpy float16, torch bfloat16, torch SDPA in fp64), a closed form, an
exact integer identity, a hand-computed case, or a figure printed on the pages.
No GPU is used.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")


def sylvester(n=256):
    i = np.arange(n)
    pc = np.vectorize(lambda v: bin(v).count("1"))(i[:, None] & i[None, :])
    return np.where(pc % 2 == 0, 1, -1).astype(np.int64)


H = sylvester()


# --------------------------------------------------------------------------
# fp16 / bf16 conversions against library conversions
# --------------------------------------------------------------------------
def _edge_floats():
    rng = np.random.default_rng(7)
    vals = [0.0, -0.0, 1.0, -1.0, 65504.0, 65519.99, 65520.0, 70000.0, -70000.0, 1e-8, 2.0 ** -24,
            2.0 ** -25, 2.0 ** -25 * 1.0000001, 3 * 2.0 ** -25, 2.0 ** -14, 2.0 ** -14 * (1 - 2 ** -11),
            6.1e-5, 5.96e-8, 1e-40, np.float32(np.inf), -np.float32(np.inf), 0.1, 1 / 3, 1024.5, 2049.0, 2051.0]
    # exact ties between adjacent binary16 values
    for e in range(-24, 16):
        base = np.float32(2.0 ** e)
        vals += [float(base * np.float32(1 + 2 ** -11)), float(base * np.float32(1 + 3 * 2 ** -11))]
    vals = np.array(vals, np.float32)
    rnd = (rng.standard_normal(20000) * np.exp(rng.uniform(-20, 12, 20000))).astype(np.float32)
    bits = rng.integers(0, 2 ** 32, 20000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    bits = bits[np.isfinite(bits)]
    return np.concatenate([vals, rnd, bits])


def test_f32_to_f16_matches_numpy():
    x = _edge_floats()
    got = oracle.f32_to_f16_bits(x)
    want = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want)


def test_f16_to_f32_matches_numpy_all_finite_codes():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f16 = h.view(np.float16)
    h = h[np.isfinite(f16)]
    got = oracle.f16_bits_to_f32(h)
    want = h.view(np.float16).astype(np.float32)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_f32_to_bf16_matches_torch():
    x = _edge_floats()
    got = oracle.f32_to_bf16_bits(x)
    want = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)


# --------------------------------------------------------------------------
# FWHT-256 (the rotation of the Strata page's 4-bit section)
# --------------------------------------------------------------------------
def test_hadamard_integer_identity():
    assert np.array_equal(H @ H, 256 * np.eye(256, dtype=np.int64))


def test_fwht_exact_on_integer_inputs():
    rng = np.random.default_rng(1)
    x = rng.integers(-3000, 3000, (64, 256))
    got = oracle.fwht256_f32(x.astype(np.float32))
    want = (x @ H.T).astype(np.float64) / 16.0      # every partial sum is an exact integer < 2^24
    assert np.array_equal(got.astype(np.float64), want)


def test_fwht_columns_closed_form():
    for j in (0, 1, 77, 128, 255):
        e = np.zeros(256, np.float32)
        e[j] = 1.0
        got = oracle.fwht256_f32(e)[0]
        assert np.array_equal(got, H[:, j].astype(np.float32) / 16)
    assert np.array_equal(oracle.fwht256_f32(np.eye(256, dtype=np.float32)[0])[0], np.full(256, 1 / 16, np.float32))


def test_fwht_random_within_fp32_rounding_and_involution():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((32, 256)).astype(np.float32) * 3
    y = oracle.fwht256_f32(x).astype(np.float64)
    exact = x.astype(np.float64) @ H.T.astype(np.float64) / 16
    # 8 rounded additions on values of size <= sum|x|: bound 8 * 2^-24 * sum|x| / 16
    bound = 8 * 2.0 ** -24 * np.abs(x).sum(1, keepdims=True) / 16
    assert np.all(np.abs(y - exact) <= bound)
    back = oracle.fwht256_f32(y.astype(np.float32)).astype(np.float64)
    assert np.max(np.abs(back - x)) < 1e-5 * np.abs(x).max()
    yd = oracle.fwht256_f64(x.astype(np.float64))
    assert np.allclose(yd, exact, rtol=0, atol=1e-12)


def test_rotation_preserves_dot_product():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((16, 256)).astype(np.float32)
    k = rng.standard_normal((16, 256)).astype(np.float32)
    qr = oracle.fwht256_f32(q).astype(np.float64)
    kr = oracle.fwht256_f32(k).astype(np.float64)
    d0 = np.sum(q.astype(np.float64) * k, 1)
    d1 = np.sum(qr * kr, 1)
    norm = np.linalg.norm(q, axis=1) * np.linalg.norm(k, axis=1)
    assert np.all(np.abs(d1 - d0) <= 1e-6 * norm)


# --------------------------------------------------------------------------
# q4_0 and int8 codecs: hand-computed cases and error bounds
# --------------------------------------------------------------------------
def test_q4_0_hand_cases():
    x = np.zeros(256, np.float32)
    # block 0: signed max -8 -> d = 1.0; ties round half to even
    x[0:8] = [-8.0, 2.5, 3.5, -0.5, 0.5, 1.5, 7.5, -7.5]
    # block 1: signed max +8 -> d = -1.0 (codes mirror)
    x[32:36] = [8.0, 2.5, -2.5, 4.0]
    # block 2: all zero -> d = 0 / -8 = -0.0 (IEEE sign rule), every code 8
    # block 3: one non-zero value
    x[96 + 5] = 3.25
    # block 4: constant block
    x[128:160] = -1.75
    # block 5: |x| tie, first index wins (positive first -> d negative)
    x[160] = 2.0
    x[161] = -2.0
    c, s = oracle.quant_q4_0(x)
    assert s[0] == 0x3C00 and list(c[0:8]) == [0, 10, 12, 8, 8, 10, 15, 0] and all(c[8:32] == 8)
    assert s[1] == 0xBC00 and list(c[32:36]) == [0, 6, 10, 4]
    assert s[2] == 0x8000 and all(c[64:96] == 8)
    assert c[101] == 0 and all(np.delete(c[96:128], 5) == 8)
    assert np.float32(np.uint16(s[3]).view(np.float16)) == np.float32(3.25 / -8)
    assert all(c[128:160] == 0)
    assert s[5] == np.float16(-0.25).view(np.uint16) and c[160] == 0 and c[161] == 15
    # block 6: true division, not a multiply by the reciprocal: with d = 6.1835938
    # (an fp16 value) x = 21.642578 gives x/d = 3.5 exactly (a tie, rounds to 4),
    # while x * fl(1/d) = 3.4999998 would round to 3
    y = np.zeros(256, np.float32)
    y[192] = np.float32(-49.46875)
    y[193] = np.float32(21.642578)
    c, s = oracle.quant_q4_0(y)
    assert s[6] == np.float16(6.1835938).view(np.uint16) and c[192] == 0 and c[193] == 12


def test_int8_hand_cases():
    x = np.zeros(256, np.float32)
    x[0:5] = [127.0, 2.5, -2.5, 126.5, -127.0]       # d = 1.0
    x[64 + 9] = -0.3                                  # single value -> -127
    # group 2 all zero
    x[192:256] = 0.5                                  # constant -> 127
    c, s = oracle.quant_int8(x)
    assert s[0] == 0x3C00 and list(c[0:5]) == [127, 2, -2, 126, -127]
    assert c[73] == -127 and all(np.delete(c[64:128], 9) == 0)
    assert s[2] == 0 and all(c[128:192] == 0)
    assert all(c[192:256] == 127)
    # a subnormal fp16 scale: d32 = 1.4 * 2^-24 rounds to 2^-24, so |x| / d = 177.8
    # and the code saturates at -127 (never -128)
    y = np.zeros(256, np.float32)
    y[64] = np.float32(-127 * 1.4 * 2.0 ** -24)
    c, s = oracle.quant_int8(y)
    assert s[1] == 1 and c[64] == -127


def _f16(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def test_q4_0_error_bound():
    rng = np.random.default_rng(4)
    for _ in range(200):
        x = (rng.standard_normal(256) * np.exp(rng.uniform(-6, 6))).astype(np.float32)
        c, s = oracle.quant_q4_0(x)
        d = np.repeat(_f16(s), 32)
        xhat = (c.astype(np.int64) - 8) * d
        err = np.abs(xhat - x)
        # inside the code range the error is at most d/2 (plus the fp16 scale
        # rounding, at most 2^-11 relative per unit of code); the +8 side is
        # clamped to code 15, an error of at most |d| (plus the same term)
        slack = 8.5 * np.abs(d) * 2.0 ** -10
        clamped = c == 15
        assert np.all(err[~clamped] <= np.abs(d[~clamped]) / 2 + slack[~clamped])
        assert np.all(err[clamped] <= np.abs(d[clamped]) + slack[clamped])
        # decoding through the oracle's own dequantiser gives the same values
        assert np.array_equal(oracle.dequant_rows(True, c[None], s[None])[0], xhat)


def test_int8_error_bound():
    rng = np.random.default_rng(5)
    for _ in range(200):
        x = (rng.standard_normal(256) * np.exp(rng.uniform(-6, 6))).astype(np.float32)
        c, s = oracle.quant_int8(x)
        d = np.repeat(_f16(s), 64)
        xhat = c.astype(np.float64) * d
        slack = 128 * d * 2.0 ** -10
        assert np.all(np.abs(xhat - x) <= d / 2 + slack)
        assert np.array_equal(oracle.dequant_rows(False, c.view(np.uint8)[None], s[None])[0], xhat)


def test_append_formats_compose_rotation_and_codec():
    rng = np.random.default_rng(6)
    k = rng.standard_normal((3, 256)).astype(np.float32)
    v = rng.standard_normal((3, 256)).astype(np.float32)
    for fmt, (kp, vp, krot, vrot) in oracle.PARTS.items():
        kc, ks, vc, vs = oracle.append_rows(fmt, k, v)
        for i in range(3):
            kk = oracle.fwht256_f32(k[i])[0] if krot else k[i]
            vv = oracle.fwht256_f32(v[i])[0] if vrot else v[i]
            ck, sk = oracle.QUANT[kp](kk)
            cv, sv = oracle.QUANT[vp](vv)
            assert np.array_equal(kc[i], ck.view(np.uint8)) and np.array_equal(ks[i], sk)
            assert np.array_equal(vc[i], cv.view(np.uint8)) and np.array_equal(vs[i], sv)
    # q4_0 rotates Q with the same transform; the other formats leave it alone
    q = rng.standard_normal((2, 256)).astype(np.float32)
    assert np.array_equal(oracle.q_prepare("q4_0", q), oracle.fwht256_f32(q))
    assert np.array_equal(oracle.q_prepare("int8", q), q)
    assert np.array_equal(oracle.q_prepare("k8v4", q), q)
    assert np.array_equal(oracle.q_prepare("fp8", q), q)
    assert np.array_equal(oracle.q_prepare("nvfp4", q), q)


# --------------------------------------------------------------------------
# attention: library routine (torch SDPA, fp64), closed forms, invariants
# --------------------------------------------------------------------------
def _encoded(fmt, T, rng, scale=1.0, qscale=1.0, G=6):
    k = (rng.standard_normal((T, 256)) * scale).astype(np.float32)
    v = (rng.standard_normal((T, 256)) * scale).astype(np.float32)
    q = (rng.standard_normal((G, 256)) * qscale).astype(np.float32)
    kc, ks, vc, vs = oracle.append_rows(fmt, k, v)
    return oracle.q_prepare(fmt, q), kc, ks, vc, vs


def _sdpa(qp, khat, vhat):
    qt = torch.from_numpy(qp.astype(np.float64))[None, :, None, :]
    kt = torch.from_numpy(khat)[None, None].expand(1, qp.shape[0], -1, -1)
    vt = torch.from_numpy(vhat)[None, None].expand(1, qp.shape[0], -1, -1)
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[0, :, 0].numpy()


@pytest.mark.parametrize("fmt", ["int8", "q4_0", "k8v4", "fp8", "nvfp4"])
@pytest.mark.parametrize("T", [1, 7, 300])
def test_attention_matches_torch_sdpa_fp64(fmt, T):
    rng = np.random.default_rng(10 + T)
    qp, kc, ks, vc, vs = _encoded(fmt, T, rng, qscale=2.0)
    kq4, vq4, krot, vrot = oracle.PARTS[fmt]
    khat = oracle.dequant_rows(kq4, kc, ks)
    vhat = oracle.dequant_rows(vq4, vc, vs)
    ref = _sdpa(qp, khat, vhat)
    if vrot:                                  # un-rotate with the explicit Sylvester matrix
        ref = ref @ (H.T / 16.0)
    got = oracle.attn_decode(fmt, qp, kc, ks, vc, vs)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_attention_single_token_is_that_value():
    rng = np.random.default_rng(11)
    qp, kc, ks, vc, vs = _encoded("int8", 1, rng)
    got = oracle.attn_decode("int8", qp, kc, ks, vc, vs)
    vhat = oracle.dequant_rows(False, vc, vs)[0]
    assert np.allclose(got, np.broadcast_to(vhat, got.shape), rtol=0, atol=1e-13)


def test_attention_identical_keys_give_mean_value():
    rng = np.random.default_rng(12)
    T = 9
    k = np.repeat(rng.standard_normal((1, 256)).astype(np.float32), T, 0)
    v = rng.standard_normal((T, 256)).astype(np.float32)
    kc, ks, vc, vs = oracle.append_rows("int8", k, v)
    q = rng.standard_normal((3, 256)).astype(np.float32)
    got = oracle.attn_decode("int8", q, kc, ks, vc, vs)
    mean = oracle.dequant_rows(False, vc, vs).mean(0)
    assert np.allclose(got, np.broadcast_to(mean, got.shape), rtol=0, atol=1e-12)


def test_attention_two_tokens_logistic_closed_form():
    rng = np.random.default_rng(13)
    qp, kc, ks, vc, vs = _encoded("int8", 2, rng, qscale=3.0, G=2)
    khat = oracle.dequant_rows(False, kc, ks)
    vhat = oracle.dequant_rows(False, vc, vs)
    got = oracle.attn_decode("int8", qp, kc, ks, vc, vs)
    for h in range(2):
        s0 = float(qp[h].astype(np.float64) @ khat[0]) / 16
        s1 = float(qp[h].astype(np.float64) @ khat[1]) / 16
        w0 = 1.0 / (1.0 + np.exp(s1 - s0))
        assert np.allclose(got[h], w0 * vhat[0] + (1 - w0) * vhat[1], rtol=0, atol=1e-12)


def test_attention_dominant_token():
    rng = np.random.default_rng(14)
    T = 50
    k = rng.standard_normal((T, 256)).astype(np.float32) * 0.01
    k[17] = 1.0
    v = rng.standard_normal((T, 256)).astype(np.float32)
    kc, ks, vc, vs = oracle.append_rows("int8", k, v)
    q = np.full((1, 256), 40.0, np.float32)           # score of token 17 is about 640 higher
    got = oracle.attn_decode("int8", q, kc, ks, vc, vs)
    assert np.allclose(got[0], oracle.dequant_rows(False, vc[17:18], vs[17:18])[0], rtol=0, atol=1e-12)


@pytest.mark.parametrize("fmt", ["int8", "q4_0", "k8v4", "fp8", "nvfp4"])
def test_attention_split_invariance_and_permutation(fmt):
    rng = np.random.default_rng(15)
    T = 97
    qp, kc, ks, vc, vs = _encoded(fmt, T, rng, qscale=4.0)
    full = oracle.attn_decode(fmt, qp, kc, ks, vc, vs)
    a = oracle.attn_partial(fmt, qp, 0, 40, kc, ks, vc, vs)
    b = oracle.attn_partial(fmt, qp, 40, T, kc, ks, vc, vs)
    m, l, o = oracle.merge_partials(a, b)
    assert np.allclose(oracle.finish(fmt, l, o), full, rtol=0, atol=1e-12)
    perm = rng.permutation(T)
    permuted = oracle.attn_decode(fmt, qp, kc[perm], ks[perm], vc[perm], vs[perm])
    assert np.allclose(permuted, full, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# sizes: the pages' printed figures
# --------------------------------------------------------------------------
def test_kv_size_formula_reproduces_printed_figures():
    g = json.load(open(GOLDEN))
    s = g["model_27b_shape"]
    fig = g["kv_256k_27b_GB"]
    for key in ("fp16", "q8_0", "q4_0"):
        b = oracle.kv_cache_bytes(s["full_attention_layers"], s["kv_heads"], s["head_dim"],
                                  fig["bytes_per_elem"][key], fig["context"])
        assert round(b / 1e9, 1) == fig[key], key
    b64 = oracle.kv_cache_bytes(g["kv_256k_all_full_attention_fp16_GB"]["layers"], 4, 256, 2.0, 262144)
    assert round(b64 / 1e9, 1) == g["kv_256k_all_full_attention_fp16_GB"]["value"]
    b1m = oracle.kv_cache_bytes(16, 4, 256, 0.5625, g["kv_1m_q4_0_GB"]["context"])
    assert round(b1m / 1e9) == g["kv_1m_q4_0_GB"]["value"]


def test_format_bytes_reproduce_strata_figures():
    g = json.load(open(GOLDEN))["strata_bytes_per_token_layer_two_kv_heads"]
    assert 2 * oracle.format_bytes_per_token_head("int8") == g["int8"]
    assert 2 * oracle.format_bytes_per_token_head("q4_0") == g["q4_0"]
    k8v4 = 2 * oracle.format_bytes_per_token_head("k8v4")
    assert round(100 * (1 - k8v4 / g["int8"])) == g["k8v4_saving_vs_int8_percent"]
    # bytes per element consistent with the generic size formula
    for fmt in ("int8", "q4_0", "k8v4"):
        per_elem = oracle.format_bytes_per_token_head(fmt) / (2 * 256)
        assert oracle.kv_cache_bytes(1, 1, 256, per_elem, 1) == oracle.format_bytes_per_token_head(fmt)


def test_full_window_q4_0_is_the_printed_4_8_GB():
    g = json.load(open(GOLDEN))
    per_token = 16 * 4 * oracle.format_bytes_per_token_head("q4_0")
    total = per_token * 262144
    assert round(total / 1e9, 1) == g["kv_256k_27b_GB"]["q4_0"]
    f = g["four_bit_16_value_fp8_scale_kv"]
    assert oracle.format_bytes_per_token_head("q4_0") == f["bytes_per_position"]
    assert round(f["positions_per_token"] * f["bytes_per_position"] * 262144 / 2 ** 30, 2) == f["gib_at_262144"]
    assert round(f["positions_per_token"] * f["bytes_per_position"] * 163840 / 2 ** 30, 2) == f["gib_at_163840"]


def test_strata_host_kv_implies_about_13_layers():
    g = json.load(open(GOLDEN))
    per_layer = 2 * oracle.format_bytes_per_token_head("int8")
    hk = g["strata_host_kv"]
    layers = hk["kb_per_token"] * 1000 / per_layer
    assert abs(layers - 13) < 0.05
    assert round(13 * per_layer * hk["context"] / 2 ** 30, 1) == hk["gb_at_128k"]


def test_pcie_estimate_arithmetic():
    p = json.load(open(GOLDEN))["pcie_estimate"]
    per_layer = oracle.kv_cache_bytes(1, 4, 256, 1.0, p["context"])
    assert per_layer / 2 ** 20 == p["mib_per_layer"]
    assert oracle.kv_cache_bytes(1, 4, 256, 1.0, 1) == p["bytes_per_token_layer"]
    total = p["layers"] * per_layer
    assert total / 2 ** 30 == p["gib_total"]
    assert round(p["pcie_gib_per_s"] * 2 ** 30 / total) == p["tok_per_s"]
