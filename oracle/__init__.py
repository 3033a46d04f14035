"""Python view of the C oracle (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path never does.

``build()`` compiles ``kvq_oracle.c`` with gcc into ``liboracle_kvq.so`` next
to it (``-ffp-contract=off``: no fused multiply-add, so every fp32 step is one
correctly rounded IEEE operation).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Tuple

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kvq_oracle.c")
LIB = os.path.join(HERE, "liboracle_kvq.so")
# A test may point the wrapper at another build of the oracle (for example one
# with a deliberately planted mistake) through this variable.
_OVERRIDE = os.environ.get("KVQ_ORACLE_LIB")

FMT = {"int8": 0, "q4_0": 1, "k8v4": 2, "fp8": 3, "nvfp4": 4}
# How K and V are stored: "i8" (int8, fp16 scale per 64), "q4" (q4_0, fp16
# scale per 32), "e4m3" (fp8 codes, one fp16 scale), "e2m1" (fp4 codes, an
# E4M3 scale per 16).
PART_ID = {"i8": 0, "q4": 1, "e4m3": 2, "e2m1": 3}
N_SCALES = {"i8": 4, "q4": 8, "e4m3": 1, "e2m1": 16}
# (K part, V part, K rotated, V rotated) per format
PARTS = {"int8": ("i8", "i8", False, False), "q4_0": ("q4", "q4", True, True), "k8v4": ("i8", "q4", False, True),
         "fp8": ("e4m3", "e4m3", False, False), "nvfp4": ("e2m1", "e2m1", False, False)}

_lib = None


def build(force: bool = False) -> str:
    if _OVERRIDE:
        return _OVERRIDE
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
               "-Wall", "-Wextra", "-o", LIB, SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return LIB


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        L.oracle_f32_to_f16.argtypes = [ctypes.c_float]
        L.oracle_f32_to_f16.restype = ctypes.c_uint16
        L.oracle_f16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_f16_to_f32.restype = ctypes.c_float
        L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.oracle_fwht256_f32.argtypes = [P, P]
        L.oracle_fwht256_f64.argtypes = [P, P]
        L.oracle_quant_q4_0.argtypes = [P, P, P]
        L.oracle_quant_int8.argtypes = [P, P, P]
        L.oracle_quant_fp8.argtypes = [P, P, P]
        L.oracle_quant_nvfp4.argtypes = [P, P, P]
        L.oracle_e4m3_to_f32.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_to_f32.restype = ctypes.c_float
        L.oracle_e2m1_to_f32.argtypes = [ctypes.c_uint8]
        L.oracle_e2m1_to_f32.restype = ctypes.c_float
        L.oracle_f32_to_e4m3.argtypes = [ctypes.c_float]
        L.oracle_f32_to_e4m3.restype = ctypes.c_uint8
        L.oracle_f32_to_e2m1.argtypes = [ctypes.c_float]
        L.oracle_f32_to_e2m1.restype = ctypes.c_uint8
        L.oracle_append_rows.argtypes = [ctypes.c_int, ctypes.c_long, P, P, P, P, P, P]
        L.oracle_append_rows.restype = ctypes.c_int
        L.oracle_q_prepare.argtypes = [ctypes.c_int, P, P, ctypes.c_long]
        L.oracle_q_prepare.restype = ctypes.c_int
        L.oracle_dequant_rows.argtypes = [ctypes.c_int, ctypes.c_long, P, P, P]
        L.oracle_attn_partial.argtypes = [ctypes.c_int, P, ctypes.c_int, ctypes.c_long, ctypes.c_long,
                                          P, P, P, P, P, P, P]
        L.oracle_attn_partial.restype = ctypes.c_int
        L.oracle_merge_partials.argtypes = [ctypes.c_int, P, P, P, P, P, P]
        L.oracle_finish.argtypes = [ctypes.c_int, ctypes.c_int, P, P, P]
        L.oracle_finish.restype = ctypes.c_int
        L.oracle_attn_decode.argtypes = [ctypes.c_int, P, ctypes.c_int, ctypes.c_long, P, P, P, P, P]
        L.oracle_attn_decode.restype = ctypes.c_int
        L.oracle_kv_cache_bytes.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                            ctypes.c_double]
        L.oracle_kv_cache_bytes.restype = ctypes.c_double
        L.oracle_format_bytes_per_token_head.argtypes = [ctypes.c_int]
        L.oracle_format_bytes_per_token_head.restype = ctypes.c_long
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# --- scalar conversions ------------------------------------------------------
def f32_to_f16_bits(x: np.ndarray) -> np.ndarray:
    L = lib()
    x = np.asarray(x, np.float32).ravel()
    return np.array([L.oracle_f32_to_f16(float(v)) for v in x], np.uint16)


def f16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    L = lib()
    h = np.asarray(h, np.uint16).ravel()
    return np.array([L.oracle_f16_to_f32(int(v)) for v in h], np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    L = lib()
    x = np.asarray(x, np.float32).ravel()
    return np.array([L.oracle_f32_to_bf16(float(v)) for v in x], np.uint16)


def e4m3_to_f32(b: np.ndarray) -> np.ndarray:
    L = lib()
    return np.array([L.oracle_e4m3_to_f32(int(v)) for v in np.asarray(b, np.uint8).ravel()], np.float32)


def e2m1_to_f32(c: np.ndarray) -> np.ndarray:
    L = lib()
    return np.array([L.oracle_e2m1_to_f32(int(v)) for v in np.asarray(c, np.uint8).ravel()], np.float32)


def f32_to_e4m3(x: np.ndarray) -> np.ndarray:
    L = lib()
    return np.array([L.oracle_f32_to_e4m3(float(v)) for v in np.asarray(x, np.float32).ravel()], np.uint8)


def f32_to_e2m1(x: np.ndarray) -> np.ndarray:
    L = lib()
    return np.array([L.oracle_f32_to_e2m1(float(v)) for v in np.asarray(x, np.float32).ravel()], np.uint8)


# --- transform / codecs ------------------------------------------------------
def fwht256_f32(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float32).reshape(-1, 256)
    out = np.empty_like(x)
    for i in range(x.shape[0]):
        lib().oracle_fwht256_f32(_p(x[i]), _p(out[i]))
    return out


def fwht256_f64(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float64).reshape(-1, 256)
    out = np.empty_like(x)
    for i in range(x.shape[0]):
        lib().oracle_fwht256_f64(_p(x[i]), _p(out[i]))
    return out


def quant_q4_0(x: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """256-vector -> (codes uint8[256] in 0..15, fp16 scale bits uint16[8])."""
    x = np.ascontiguousarray(x, np.float32).reshape(256)
    c = np.empty(256, np.uint8)
    s = np.empty(8, np.uint16)
    lib().oracle_quant_q4_0(_p(x), _p(c), _p(s))
    return c, s


def quant_int8(x: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """256-vector -> (codes int8[256] in -127..127, fp16 scale bits uint16[4])."""
    x = np.ascontiguousarray(x, np.float32).reshape(256)
    c = np.empty(256, np.int8)
    s = np.empty(4, np.uint16)
    lib().oracle_quant_int8(_p(x), _p(c), _p(s))
    return c, s


def quant_fp8(x: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """256-vector -> (E4M3 codes uint8[256], fp16 scale bits uint16[1])."""
    x = np.ascontiguousarray(x, np.float32).reshape(256)
    c = np.empty(256, np.uint8)
    s = np.empty(1, np.uint16)
    lib().oracle_quant_fp8(_p(x), _p(c), _p(s))
    return c, s


def quant_nvfp4(x: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """256-vector -> (E2M1 codes uint8[256] in 0..15, E4M3 block scales uint16[16])."""
    x = np.ascontiguousarray(x, np.float32).reshape(256)
    c = np.empty(256, np.uint8)
    s = np.empty(16, np.uint16)
    lib().oracle_quant_nvfp4(_p(x), _p(c), _p(s))
    return c, s


QUANT = {"i8": quant_int8, "q4": quant_q4_0, "e4m3": quant_fp8, "e2m1": quant_nvfp4}


def _part(p) -> str:
    """A part name; True / False stand for "q4" / "i8"."""
    if isinstance(p, (bool, np.bool_)):
        return "q4" if p else "i8"
    return p


def n_scales(part) -> int:
    return N_SCALES[_part(part)]


def append_rows(fmt: str, k: np.ndarray, v: np.ndarray):
    """Encode n tokens of one KV head.  k, v: [n, 256] float32.

    Returns (kc uint8[n,256], ks uint16[n,nk], vc uint8[n,256], vs uint16[n,nv]);
    int8 codes are returned as their two's-complement bytes.
    """
    kp, vp, _, _ = PARTS[fmt]
    k = np.ascontiguousarray(k, np.float32).reshape(-1, 256)
    v = np.ascontiguousarray(v, np.float32).reshape(-1, 256)
    n = k.shape[0]
    kc = np.empty((n, 256), np.uint8)
    vc = np.empty((n, 256), np.uint8)
    ks = np.empty((n, n_scales(kp)), np.uint16)
    vs = np.empty((n, n_scales(vp)), np.uint16)
    rc = lib().oracle_append_rows(FMT[fmt], n, _p(k), _p(v), _p(kc), _p(ks), _p(vc), _p(vs))
    assert rc == 0
    return kc, ks, vc, vs


def q_prepare(fmt: str, q: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, np.float32).reshape(-1, 256)
    out = np.empty_like(q)
    assert lib().oracle_q_prepare(FMT[fmt], _p(q), _p(out), q.shape[0]) == 0
    return out


def dequant_rows(part, codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    part = _part(part)
    codes = np.ascontiguousarray(codes).view(np.uint8).reshape(-1, 256)
    scales = np.ascontiguousarray(scales, np.uint16).reshape(codes.shape[0], n_scales(part))
    out = np.empty((codes.shape[0], 256), np.float64)
    lib().oracle_dequant_rows(PART_ID[part], codes.shape[0], _p(codes), _p(scales), _p(out))
    return out


def _kv_args(kc, ks, vc, vs):
    return (np.ascontiguousarray(kc).view(np.uint8), np.ascontiguousarray(ks, np.uint16),
            np.ascontiguousarray(vc).view(np.uint8), np.ascontiguousarray(vs, np.uint16))


def attn_decode(fmt: str, qp: np.ndarray, kc, ks, vc, vs) -> np.ndarray:
    """Split-free decode attention of G query heads over T tokens of one KV head.

    qp: prepared query [G,256] float32 (rotated for q4_0).  Returns [G,256] fp64.
    """
    qp = np.ascontiguousarray(qp, np.float32).reshape(-1, 256)
    G = qp.shape[0]
    kc, ks, vc, vs = _kv_args(kc, ks, vc, vs)
    T = kc.reshape(-1, 256).shape[0]
    out = np.empty((G, 256), np.float64)
    rc = lib().oracle_attn_decode(FMT[fmt], _p(qp), G, T, _p(kc), _p(ks), _p(vc), _p(vs), _p(out))
    assert rc == 0, rc
    return out


def attn_partial(fmt: str, qp: np.ndarray, t0: int, t1: int, kc, ks, vc, vs):
    qp = np.ascontiguousarray(qp, np.float32).reshape(-1, 256)
    G = qp.shape[0]
    kc, ks, vc, vs = _kv_args(kc, ks, vc, vs)
    m = np.empty(G, np.float64)
    l = np.empty(G, np.float64)
    o = np.empty((G, 256), np.float64)
    rc = lib().oracle_attn_partial(FMT[fmt], _p(qp), G, t0, t1, _p(kc), _p(ks), _p(vc), _p(vs),
                                   _p(m), _p(l), _p(o))
    assert rc == 0, rc
    return m, l, o


def merge_partials(a, b):
    ma, la, oa = (np.array(x, copy=True) for x in a)
    mb, lb, ob = (np.ascontiguousarray(x) for x in b)
    lib().oracle_merge_partials(ma.shape[0], _p(ma), _p(la), _p(oa), _p(mb), _p(lb), _p(ob))
    return ma, la, oa


def finish(fmt: str, l: np.ndarray, o: np.ndarray) -> np.ndarray:
    l = np.ascontiguousarray(l, np.float64)
    o = np.ascontiguousarray(o, np.float64)
    out = np.empty_like(o)
    assert lib().oracle_finish(FMT[fmt], l.shape[0], _p(l), _p(o), _p(out)) == 0
    return out


def kv_cache_bytes(layers: int, kv_heads: int, head_dim: int, bytes_per_elem: float, context: float) -> float:
    return lib().oracle_kv_cache_bytes(layers, kv_heads, head_dim, bytes_per_elem, context)


def format_bytes_per_token_head(fmt: str) -> int:
    return lib().oracle_format_bytes_per_token_head(FMT[fmt])
