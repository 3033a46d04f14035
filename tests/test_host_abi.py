"""Host-side tests of the C ABI: the library loads and exports every declared
symbol, sizes and layout, the split plan, and argument validation.  Every call
here fails validation or is host-only, so no GPU is touched."""
import ctypes
import os
import re

import numpy as np
import pytest

import kvq_inputs
import oracle
import quantized_kv_cache_17_b200 as kvq
from tests import kvq_layout

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from quantized_kv_cache_17_b200 import build
    build.build()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "kvq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("q_rotate", "kv_append", "paged_decode_attn_int8", "paged_decode_attn_q4_0", "paged_decode_attn_k8v4",
              "attn_combine", "kvq_pool_bytes", "kvq_pool_layout", "kvq_decode_plan", "kv_append_q_rotate",
              "paged_decode_step_int8", "paged_decode_step_q4_0", "paged_decode_step_k8v4"):
        assert n in names


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(kvq.LIB_PATH)
    for n in declared_functions():
        assert hasattr(L, n), n
    assert kvq.lib().kvq_version().startswith(b"kvq")


@pytest.mark.parametrize("fmt", ["int8", "q4_0", "k8v4", "fp8", "nvfp4"])
def test_pool_bytes_match_format_sizes(fmt):
    d = kvq.make_desc(3, 2, 12, 5, fmt)
    L = kvq.pool_layout(d)
    assert L.bytes_per_token_head == oracle.format_bytes_per_token_head(fmt)
    assert kvq.pool_bytes(d) == 3 * 5 * 2 * 256 * L.bytes_per_token_head
    assert L.page_bytes == 256 * L.bytes_per_token_head and L.page_bytes % 256 == 0
    kc, ks, vc, vs, tb = kvq_layout.tile_sections(fmt)
    assert (L.tile_bytes, L.k_codes_off, L.k_scales_off, L.v_codes_off, L.v_scales_off) == (tb, kc, ks, vc, vs)
    for off in (L.k_scales_off, L.v_codes_off, L.v_scales_off, L.tile_bytes):
        assert off % 16 == 0


def test_full_window_pool_is_the_printed_size():
    w = kvq_inputs.workload("qwen27b_q4_0_262k")
    d = kvq.make_desc(w.n_layers, w.n_kv_heads, w.n_q_heads, w.pages_needed(), w.fmt)
    assert round(kvq.pool_bytes(d) / 1e9, 1) == 4.8
    two_heads = kvq.pool_layout(kvq.make_desc(1, 2, 16, 1, "int8")).bytes_per_token_head * 2
    assert two_heads == 1056


@pytest.mark.parametrize("part,side", [(p, s) for p in ("q4", "i8", "f8", "f4") for s in ("k", "v")])
def test_layout_decoder_is_a_bijection(part, side):
    off, sh = kvq_layout.code_map(part, side)
    keys = off * 8 + sh
    assert len(np.unique(keys)) == 8 * 256
    assert off.max() < kvq_layout.CODE_BYTES[part]
    so = kvq_layout.scale_map(part)
    width = 1 if part == "f4" else 2                      # E4M3 byte or fp16 scale
    cover = np.unique((so[..., None] + np.arange(width)).ravel())
    assert len(cover) == so.size * width and so.max() + width <= kvq_layout.SCALE_BYTES[part]


def _check_plan(plan, info, seq_lens, n_kv, n_ctas):
    n = info.n_units
    assert plan[0] == 0x4B565131 and plan[1] == n and plan[2] == len(seq_lens) and plan[3] == n_kv
    units = plan[8:8 + 4 * n].reshape(n, 4)
    start = plan[8 + 4 * n:]
    assert len(start) == len(seq_lens) * n_kv + 1 and info.plan_len == len(plan)
    assert n <= max(n_ctas, len(seq_lens) * n_kv)
    for b, T in enumerate(seq_lens):
        for g in range(n_kv):
            us = units[start[b * n_kv + g]:start[b * n_kv + g + 1]]
            assert (us[:, 0] == b).all() and (us[:, 1] == g).all()
            assert us[0, 2] == 0 and us[-1, 3] == T
            assert (us[1:, 2] == us[:-1, 3]).all()          # contiguous, no overlap, no gap
            assert (us[:, 2] % 64 == 0).all() and (us[:, 3] > us[:, 2]).all()
            assert ((us[:, 3] - us[:, 2]) <= info.chunk_tokens).all()
    G = plan[4]
    counters = (len(seq_lens) * n_kv * 4 + 15) // 16 * 16
    assert info.workspace_bytes == n * (G * 256 + 16) * 4 + counters


@pytest.mark.parametrize("seq_lens,n_ctas", [([1024], 148), ([262144], 148), ([32768], 148), ([131072], 148),
                                              ([8192, 65536, 200000, 262144], 148), ([1], 148), ([1025, 3, 64], 7),
                                              ([100] * 50, 20)])
def test_decode_plan_properties(seq_lens, n_ctas):
    d = kvq.make_desc(1, 4, 24, 4096, "q4_0")
    plan, info = kvq.decode_plan(d, seq_lens, max_pages=1024, n_ctas=n_ctas)
    _check_plan(plan, info, seq_lens, 4, n_ctas)


def test_decode_plan_balance_full_window():
    d = kvq.make_desc(16, 4, 24, 1024, "q4_0")
    plan, info = kvq.decode_plan(d, [262144], max_pages=1024, n_ctas=148)
    units = plan[8:8 + 4 * info.n_units].reshape(-1, 4)
    sizes = units[:, 3] - units[:, 2]
    assert info.n_units == 148
    assert sizes.max() - sizes.min() <= 64


def test_validation_errors_without_a_gpu():
    L = kvq.lib()
    bad = kvq.make_desc(1, 4, 24, 8, "q4_0")
    bad.head_dim = 128
    assert L.kvq_pool_bytes(ctypes.byref(bad), ctypes.byref(ctypes.c_uint64())) == -2
    bad = kvq.make_desc(1, 4, 22, 8, "q4_0")
    assert L.kvq_pool_bytes(ctypes.byref(bad), ctypes.byref(ctypes.c_uint64())) == -1
    bad = kvq.make_desc(1, 1, 16, 8, "q4_0")            # group 16 > 8
    assert L.kvq_pool_bytes(ctypes.byref(bad), ctypes.byref(ctypes.c_uint64())) == -2
    d = kvq.make_desc(1, 4, 24, 8, "q4_0")
    info = kvq.PlanInfo()
    for lens in ([0], [8 * 256 + 1], [-5]):
        sl = np.array(lens, np.int32)
        assert L.kvq_decode_plan(ctypes.byref(d), 1, sl.ctypes.data, 8, 148, None, 0, ctypes.byref(info)) == -1
    assert L.q_rotate(None, None, 4, None) == -1
    assert L.q_rotate(0x1008, 0x2000, 4, None) == -3
    assert L.q_rotate(None, None, 0, None) == 0
    assert L.q_rotate(None, None, -1, None) == -1
    pool = kvq.Pool(0x10000, d)
    assert L.kv_append(ctypes.byref(pool), 1, 0x1000, 0x1000, 1, None, 0x1000, 0x1000, 8, 1, None, None) == -1
    assert L.kv_append(ctypes.byref(kvq.Pool(0x10008, d)), 0, 0x1000, 0x1000, 1, None, 0x1000, 0x1000, 8, 1,
                       None, None) == -3
    plan, info = kvq.decode_plan(d, [1000], max_pages=8, n_ctas=148)
    args = (ctypes.byref(pool), 0, 0x1000, 0x2000, 8, 0x3000, ctypes.byref(info), 0x4000)
    assert L.paged_decode_attn_int8(*args, info.workspace_bytes, None, None) == -1          # wrong format
    assert L.paged_decode_attn_q4_0(*args, info.workspace_bytes - 1, None, None) == -5      # workspace too small
    assert L.paged_decode_attn_q4_0(ctypes.byref(pool), 0, 0x1004, 0x2000, 8, 0x3000, ctypes.byref(info), 0x4000,
                                    info.workspace_bytes, None, None) == -3
    assert L.attn_combine(None, 0x3000, ctypes.byref(info), 1, 0x5000, None, None) == -1
    assert L.paged_decode_attn_cudacore(7, *args, info.workspace_bytes, None, None) == -1
    # the CUDA-core control decodes the integer-code formats only
    for f in (kvq.FP8, kvq.NVFP4):
        assert L.paged_decode_attn_cudacore(f, *args, info.workspace_bytes, None, None) == -2
    assert L.paged_decode_attn_fp8(*args, info.workspace_bytes, None, None) == -1           # pool is q4_0
    assert L.paged_decode_attn_nvfp4(*args, info.workspace_bytes, None, None) == -1
    bad = kvq.make_desc(1, 4, 24, 8, 5)                                                     # no such format
    assert L.kvq_pool_bytes(ctypes.byref(bad), ctypes.byref(ctypes.c_uint64())) == -1


@pytest.mark.parametrize("pos0,n_tok", [(32256, 512), (0, 512), (100, 512), (64, 100), (1000, 1), (261632, 512),
                                        (5000, 3000), (63, 1), (64, 1)])
def test_prefill_split_choice(pos0, n_tok):
    """kvq_prefill_split: a valid cut (multiples of 64, all at or below pos0),
    the workspace it needs, and never more waves x longest part than no split."""
    d = kvq.make_desc(1, 4, 24, 1100, "q4_0")
    ns, wb = kvq.prefill_split(d, pos0, n_tok)
    assert 1 <= ns <= 8
    assert wb == (ns * 4 * n_tok * 6 * 260 * 4 if ns > 1 else 0)
    if ns > 1:
        t_end = pos0 + n_tok
        share = -(-t_end // (64 * ns)) * 64
        st = min(share, ((pos0 // 64 * 64) // (ns - 1)) // 64 * 64)
        assert st >= 64 and (ns - 1) * st <= pos0 and st % 64 == 0
        ctas = -(-n_tok * 6 // 64) * 4
        assert -(-ctas * ns // 148) * max(st, t_end - (ns - 1) * st) < -(-ctas // 148) * t_end
    if pos0 < 64:
        assert ns == 1


def test_prefill_validation_without_a_gpu():
    L = kvq.lib()
    d = kvq.make_desc(1, 2, 12, 8, "q4_0")
    pool = kvq.Pool(0x10000, d)
    args = (ctypes.byref(pool), 0, 0x1000, 0, 256, 4, 0x2000, 8, 1)
    tail = (0x3000, 0x4000, None, None)
    assert L.paged_prefill_attn(*args, 0, None, 0, *tail) == -1            # n_split 0
    assert L.paged_prefill_attn(*args, 9, None, 0, *tail) == -1            # above 8
    assert L.paged_prefill_attn(*args, 2, None, 0, *tail) == -1            # split without a workspace
    assert L.paged_prefill_attn(*args, 2, 0x5000, 100, *tail) == -5        # workspace too small
    assert L.paged_prefill_attn(*args, 2, 0x5008, 1 << 30, *tail) == -3    # unaligned workspace
    args_low = (ctypes.byref(pool), 0, 0x1000, 0, 100, 4, 0x2000, 8, 1)
    assert L.paged_prefill_attn(*args_low, 3, 0x5000, 1 << 30, *tail) == -1   # no cut at or below pos0
    ns, wb = ctypes.c_int(), ctypes.c_uint64()
    assert L.kvq_prefill_split(ctypes.byref(d), -1, 4, 0, ctypes.byref(ns), ctypes.byref(wb)) == -1
    assert L.kvq_prefill_split(ctypes.byref(d), 0, 0, 0, ctypes.byref(ns), ctypes.byref(wb)) == -1
