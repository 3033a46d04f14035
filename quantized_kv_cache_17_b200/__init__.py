"""Python binding of the quantized paged decode-attention library (libkvq.so).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Tensors are PyTorch device tensors (memory and streams come from
PyTorch); the library itself never allocates.  If the compiled library is
missing, importing the binding's functions raises ``KVQError`` at once: there
is no fallback implementation.

Names follow the C ABI in ``include/kvq.h``: ``q_rotate``, ``kv_append``,
``paged_decode_attn_{int8,q4_0,k8v4,fp8,nvfp4}``, ``attn_combine`` plus the host
helpers ``pool_bytes``, ``pool_layout`` and ``decode_plan``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

INT8, Q4_0, K8V4, FP8, NVFP4 = 0, 1, 2, 3, 4
FORMATS = {"int8": INT8, "q4_0": Q4_0, "k8v4": K8V4, "fp8": FP8, "nvfp4": NVFP4}
HEAD_DIM = 256
PAGE_TOKENS = 256

STATUS_BAD_SLOT, STATUS_BAD_PLAN, STATUS_TIMEOUT = 1, 2, 4
ERRORS = {-1: "KVQ_EINVAL", -2: "KVQ_EUNSUPPORTED", -3: "KVQ_EALIGN", -4: "KVQ_ECUDA", -5: "KVQ_ESIZE"}

# entry points declared in include/kvq.h
EXPORTS = ["kvq_version", "kvq_pool_bytes", "kvq_pool_layout", "q_rotate", "kv_append", "kv_append_q_rotate",
           "kvq_decode_plan",
           "paged_decode_attn_int8", "paged_decode_attn_q4_0", "paged_decode_attn_k8v4",
           "paged_decode_attn_fp8", "paged_decode_attn_nvfp4",
           "paged_decode_attn_int8_combined", "paged_decode_attn_q4_0_combined", "paged_decode_attn_k8v4_combined",
           "paged_decode_attn_fp8_combined", "paged_decode_attn_nvfp4_combined",
           "paged_decode_attn_q4_0_noalloc", "paged_decode_attn_cudacore", "attn_combine",
           "paged_decode_step_int8", "paged_decode_step_q4_0", "paged_decode_step_k8v4",
           "paged_decode_step_fp8", "paged_decode_step_nvfp4", "paged_prefill_attn", "kvq_prefill_split",
           "kvq_resident_state_bytes", "kvq_resident_init", "kvq_resident_map", "kvq_resident_load",
           "kvq_resident_query", "kvq_resident_stats"]
_FMT_NAMES = ("int8", "q4_0", "k8v4", "fp8", "nvfp4")


class KVQError(RuntimeError):
    pass


class PoolDesc(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("page_tokens", ctypes.c_int32), ("n_pages", ctypes.c_int32),
                ("fmt", ctypes.c_int32)]


class Pool(ctypes.Structure):
    _fields_ = [("base", ctypes.c_void_p), ("desc", PoolDesc)]


class Layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in
                ("tile_bytes", "k_codes_off", "k_scales_off", "v_codes_off", "v_scales_off", "page_bytes",
                 "head_stride", "slot_stride", "layer_stride", "total_bytes", "bytes_per_token_head")]


class PlanInfo(ctypes.Structure):
    _fields_ = [("n_units", ctypes.c_int32), ("n_seq", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("group", ctypes.c_int32), ("plan_len", ctypes.c_int32), ("chunk_tokens", ctypes.c_int32),
                ("workspace_bytes", ctypes.c_uint64)]


_lib = None


def lib():
    """The loaded libkvq.so (raises KVQError when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise KVQError(f"{LIB_PATH} is missing: run `python -m quantized_kv_cache_17_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        L.kvq_version.restype = ctypes.c_char_p
        L.kvq_pool_bytes.argtypes = [ctypes.POINTER(PoolDesc), ctypes.POINTER(ctypes.c_uint64)]
        L.kvq_pool_layout.argtypes = [ctypes.POINTER(PoolDesc), ctypes.POINTER(Layout)]
        L.q_rotate.argtypes = [P, P, I64, P]
        L.kv_append.argtypes = [ctypes.POINTER(Pool), I32, P, P, I64, P, P, P, I32, I32, P, P]
        L.kv_append_q_rotate.argtypes = [ctypes.POINTER(Pool), I32, P, P, I64, P, P, P, I32, I32, P, P, I64, P, P]
        L.kvq_decode_plan.argtypes = [ctypes.POINTER(PoolDesc), I32, P, I32, I32, P, I32, ctypes.POINTER(PlanInfo)]
        dec = [ctypes.POINTER(Pool), I32, P, P, I32, P, ctypes.POINTER(PlanInfo), P, ctypes.c_uint64, P, P]
        for f in _FMT_NAMES:
            getattr(L, "paged_decode_attn_" + f).argtypes = dec
            getattr(L, "paged_decode_attn_" + f + "_combined").argtypes = dec[:-2] + [P, P] + dec[-2:]
        L.paged_decode_attn_q4_0_noalloc.argtypes = dec[:7] + [P, P, P, P]
        L.paged_decode_attn_cudacore.argtypes = [I32] + dec
        for f in _FMT_NAMES:
            getattr(L, "paged_decode_step_" + f).argtypes = [ctypes.POINTER(Pool), I32, P, P, P, P, I32, P,
                                                             ctypes.POINTER(PlanInfo), P, ctypes.c_uint64, P, P, P, P]
        L.attn_combine.argtypes = [P, P, ctypes.POINTER(PlanInfo), I32, P, P, P]
        L.paged_prefill_attn.argtypes = [ctypes.POINTER(Pool), I32, P, I32, I32, I32, P, I32, I32, I32, P,
                                         ctypes.c_uint64, P, P, P, P]
        L.kvq_prefill_split.argtypes = [ctypes.POINTER(PoolDesc), I32, I32, I32, ctypes.POINTER(ctypes.c_int),
                                        ctypes.POINTER(ctypes.c_uint64)]
        L.kvq_resident_init.argtypes = [P, ctypes.c_uint64, ctypes.POINTER(Pool), ctypes.POINTER(Pool)]
        L.kvq_resident_map.argtypes = [P, I32, P, I32, I32, P, P, P, I32, ctypes.POINTER(ctypes.c_int)]
        L.kvq_resident_load.argtypes = [P, I32, P, I32, P]
        L.kvq_resident_query.argtypes = [P, I32, I32, ctypes.POINTER(ctypes.c_int)]
        L.kvq_resident_stats.argtypes = [P] + [ctypes.POINTER(ctypes.c_int64)] * 3
        for n in EXPORTS[1:]:
            getattr(L, n).restype = ctypes.c_int
        L.kvq_resident_state_bytes.argtypes = [I32, I32, I32]
        L.kvq_resident_state_bytes.restype = ctypes.c_uint64
        _lib = L
    return _lib


def _check(rc: int, what: str):
    if rc != 0:
        raise KVQError(f"{what} failed: {ERRORS.get(rc, rc)}")


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def make_desc(n_layers: int, n_kv_heads: int, n_q_heads: int, n_pages: int, fmt) -> PoolDesc:
    f = FORMATS[fmt] if isinstance(fmt, str) else int(fmt)
    return PoolDesc(n_layers, n_kv_heads, n_q_heads, HEAD_DIM, PAGE_TOKENS, n_pages, f)


def pool_bytes(desc: PoolDesc) -> int:
    b = ctypes.c_uint64()
    _check(lib().kvq_pool_bytes(ctypes.byref(desc), ctypes.byref(b)), "kvq_pool_bytes")
    return b.value


def pool_layout(desc: PoolDesc) -> Layout:
    L = Layout()
    _check(lib().kvq_pool_layout(ctypes.byref(desc), ctypes.byref(L)), "kvq_pool_layout")
    return L


@dataclass
class KVPool:
    """A pool descriptor plus the caller-owned device buffer that holds it."""
    desc: PoolDesc
    buf: object   # torch.uint8 device tensor of pool_bytes(desc) bytes

    @staticmethod
    def allocate(desc: PoolDesc, device="cuda"):
        """device="pinned" gives a pool in pinned, device-mapped host memory."""
        import torch
        if device == "pinned":
            return KVPool(desc, torch.zeros(pool_bytes(desc), dtype=torch.uint8).pin_memory())
        return KVPool(desc, torch.zeros(pool_bytes(desc), dtype=torch.uint8, device=device))

    def c_pool(self) -> Pool:
        return Pool(self.buf.data_ptr(), self.desc)

    @property
    def fmt(self) -> int:
        return self.desc.fmt


def q_rotate(q, out=None, stream=None):
    """q_rot = (H/16) q for [..., 256] fp32 device tensors; out may alias q."""
    if out is None:
        out = q.new_empty(q.shape)
    n = q.numel() // HEAD_DIM
    _check(lib().q_rotate(_ptr(q), _ptr(out), n, _stream(stream)), "q_rotate")
    return out


def kv_append(pool: KVPool, layer: int, k, v, row_pos, page_table, row_seq=None, status=None, stream=None):
    """Rotate/quantise/scatter rows k, v ([n_rows, n_kv_heads, 256] fp32)."""
    n_rows = k.shape[0]
    n_seq, max_pages = page_table.shape
    cp = pool.c_pool()
    _check(lib().kv_append(ctypes.byref(cp), layer, _ptr(k), _ptr(v), n_rows, _ptr(row_seq), _ptr(row_pos),
                           _ptr(page_table), max_pages, n_seq, _ptr(status), _stream(stream)), "kv_append")


def kv_append_q_rotate(pool: KVPool, layer: int, k, v, row_pos, page_table, q, q_rot=None, row_seq=None,
                       status=None, stream=None):
    """kv_append of rows k, v and q_rotate of q ([..., 256] fp32) in one launch; returns q_rot."""
    if q_rot is None:
        q_rot = q.new_empty(q.shape)
    n_rows = 0 if k is None else k.shape[0]
    n_seq, max_pages = page_table.shape
    cp = pool.c_pool()
    _check(lib().kv_append_q_rotate(ctypes.byref(cp), layer, _ptr(k), _ptr(v), n_rows, _ptr(row_seq), _ptr(row_pos),
                                    _ptr(page_table), max_pages, n_seq, _ptr(q), _ptr(q_rot), q.numel() // HEAD_DIM,
                                    _ptr(status), _stream(stream)), "kv_append_q_rotate")
    return q_rot


def decode_plan(desc: PoolDesc, seq_lens: Sequence[int], max_pages: int, n_ctas: int = 0):
    """Host split plan: returns (plan int32 numpy array, PlanInfo)."""
    sl = np.ascontiguousarray(np.asarray(seq_lens, np.int32))
    info = PlanInfo()
    rc = lib().kvq_decode_plan(ctypes.byref(desc), len(sl), sl.ctypes.data, max_pages, n_ctas, None, 0,
                               ctypes.byref(info))
    if rc != -5:
        _check(rc, "kvq_decode_plan")
    plan = np.zeros(info.plan_len, np.int32)
    _check(lib().kvq_decode_plan(ctypes.byref(desc), len(sl), sl.ctypes.data, max_pages, n_ctas,
                                 plan.ctypes.data, len(plan), ctypes.byref(info)), "kvq_decode_plan")
    return plan, info


_DECODE = {FORMATS[f]: "paged_decode_attn_" + f for f in _FMT_NAMES}
NOALLOC_WS_BYTES = 8 << 20


def paged_decode_attn_q4_0_noalloc(pool: KVPool, layer: int, q, page_table, plan_dev, info: PlanInfo, out_bf16,
                                   out_f32=None, status=None, stream=None):
    """The q4_0 decode with the merge fused in, using the library's own scratch
    array instead of a caller workspace (for callers that cannot allocate)."""
    cp = pool.c_pool()
    _check(lib().paged_decode_attn_q4_0_noalloc(ctypes.byref(cp), layer, _ptr(q), _ptr(page_table),
                                                page_table.shape[1], _ptr(plan_dev), ctypes.byref(info),
                                                _ptr(out_bf16), _ptr(out_f32), _ptr(status), _stream(stream)),
           "paged_decode_attn_q4_0_noalloc")


def paged_decode_attn_combined(pool: KVPool, layer: int, q, page_table, plan_dev, info: PlanInfo, workspace,
                               out_bf16, out_f32=None, status=None, stream=None):
    """Decode with the combine fused in; workspace must have been zero-filled
    once before its first use (the call leaves its counters at zero)."""
    cp = pool.c_pool()
    name = _DECODE[pool.fmt] + "_combined"
    _check(getattr(lib(), name)(ctypes.byref(cp), layer, _ptr(q), _ptr(page_table), page_table.shape[1],
                                _ptr(plan_dev), ctypes.byref(info), _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _ptr(out_bf16), _ptr(out_f32),
                                _ptr(status), _stream(stream)), name)


_STEP = {FORMATS[f]: "paged_decode_step_" + f for f in _FMT_NAMES}


def paged_decode_step(pool: KVPool, layer: int, q, k_new, v_new, page_table, plan_dev, info: PlanInfo, workspace,
                      out_bf16, out_f32=None, status=None, stream=None):
    """One decode step of a layer in one launch: append every sequence's newest
    token (k_new, v_new [n_seq, n_kv_heads, 256] at position seq_len - 1),
    rotate the raw query q where the format does, decode and merge."""
    cp = pool.c_pool()
    name = _STEP[pool.fmt]
    _check(getattr(lib(), name)(ctypes.byref(cp), layer, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(page_table),
                                page_table.shape[1], _ptr(plan_dev), ctypes.byref(info), _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _ptr(out_bf16), _ptr(out_f32),
                                _ptr(status), _stream(stream)), name)


def paged_decode_attn(pool: KVPool, layer: int, q, page_table, plan_dev, info: PlanInfo, workspace, status=None,
                      stream=None, cudacore: bool = False):
    """Split-K decode attention of the pool's format (tensor-core kernel, or
    the CUDA-core control when cudacore=True); partials go to workspace."""
    cp = pool.c_pool()
    args = (ctypes.byref(cp), layer, _ptr(q), _ptr(page_table), page_table.shape[1], _ptr(plan_dev),
            ctypes.byref(info), _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
            _stream(stream))
    if cudacore:
        _check(lib().paged_decode_attn_cudacore(pool.fmt, *args), "paged_decode_attn_cudacore")
    else:
        _check(getattr(lib(), _DECODE[pool.fmt])(*args), _DECODE[pool.fmt])


def paged_decode_attn_int8(pool, layer, q, page_table, plan_dev, info, workspace, status=None, stream=None):
    assert pool.fmt == INT8
    paged_decode_attn(pool, layer, q, page_table, plan_dev, info, workspace, status, stream)


def paged_decode_attn_q4_0(pool, layer, q, page_table, plan_dev, info, workspace, status=None, stream=None):
    assert pool.fmt == Q4_0
    paged_decode_attn(pool, layer, q, page_table, plan_dev, info, workspace, status, stream)


def paged_decode_attn_k8v4(pool, layer, q, page_table, plan_dev, info, workspace, status=None, stream=None):
    assert pool.fmt == K8V4
    paged_decode_attn(pool, layer, q, page_table, plan_dev, info, workspace, status, stream)


def paged_decode_attn_fp8(pool, layer, q, page_table, plan_dev, info, workspace, status=None, stream=None):
    assert pool.fmt == FP8
    paged_decode_attn(pool, layer, q, page_table, plan_dev, info, workspace, status, stream)


def paged_decode_attn_nvfp4(pool, layer, q, page_table, plan_dev, info, workspace, status=None, stream=None):
    assert pool.fmt == NVFP4
    paged_decode_attn(pool, layer, q, page_table, plan_dev, info, workspace, status, stream)


def prefill_split(desc: PoolDesc, pos0: int, n_tok: int, n_sms: int = 0):
    """(n_split, workspace bytes) the library suggests for a prefill chunk."""
    ns, wb = ctypes.c_int(), ctypes.c_uint64()
    _check(lib().kvq_prefill_split(ctypes.byref(desc), pos0, n_tok, n_sms, ctypes.byref(ns), ctypes.byref(wb)),
           "kvq_prefill_split")
    return ns.value, wb.value


def paged_prefill_attn(pool: KVPool, layer: int, q, seq: int, pos0: int, page_table, out_bf16, out_f32=None,
                       status=None, stream=None, n_split=None, workspace=None):
    """Chunked-prefill attention: q [n_tok, n_q_heads, 256] (prepared as for
    the decode) of sequence seq at positions pos0 .. pos0 + n_tok - 1, whose
    keys are already in the pool, attends causally over the sequence's cache.
    n_split None takes kvq_prefill_split's choice; a workspace the split needs
    and the caller does not pass is allocated here (as a torch tensor)."""
    cp = pool.c_pool()
    n_tok = q.shape[0]
    if n_split is None:
        n_split, wb = prefill_split(pool.desc, pos0, n_tok)
    else:
        wb = n_split * pool.desc.n_q_heads * n_tok * 260 * 4 if n_split > 1 else 0
    if n_split > 1 and workspace is None:
        import torch
        workspace = torch.empty(wb // 4, dtype=torch.float32, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().paged_prefill_attn(ctypes.byref(cp), layer, _ptr(q), seq, pos0, n_tok, _ptr(page_table),
                                    page_table.shape[1], page_table.shape[0], n_split, _ptr(workspace), ws_bytes,
                                    _ptr(out_bf16), _ptr(out_f32), _ptr(status), _stream(stream)),
           "paged_prefill_attn")


def attn_combine(workspace, plan_dev, info: PlanInfo, inverse_fwht: bool, out_bf16, out_f32=None, stream=None):
    """Merge the partials; out_bf16 is a bf16 (or int16/uint16) tensor [n_seq, n_q_heads, 256]."""
    _check(lib().attn_combine(_ptr(workspace), _ptr(plan_dev), ctypes.byref(info), 1 if inverse_fwht else 0,
                              _ptr(out_bf16), _ptr(out_f32), _stream(stream)), "attn_combine")


def rotated_v(fmt) -> bool:
    f = FORMATS[fmt] if isinstance(fmt, str) else int(fmt)
    return f in (Q4_0, K8V4)


def rotated_q(fmt) -> bool:
    f = FORMATS[fmt] if isinstance(fmt, str) else int(fmt)
    return f == Q4_0


class ResidentCache:
    """Host-resident KV with a device page cache: the state of the residency
    table and CLOCK hand (host memory owned here), over a pinned host pool and a
    one-layer device cache pool that the caller owns."""

    def __init__(self, host_pool: KVPool, cache_pool: KVPool = None, *, host_desc: PoolDesc = None,
                 cache_desc: PoolDesc = None, host_base: int = None, cache_base: int = None):
        # host_desc/cache_desc with raw base addresses: planning only (no pool memory behind them)
        if host_pool is not None:
            host_desc, host_base = host_pool.desc, host_pool.buf.data_ptr()
            cache_desc, cache_base = cache_pool.desc, cache_pool.buf.data_ptr()
        self.host_desc, self.cache_desc = host_desc, cache_desc
        n = lib().kvq_resident_state_bytes(host_desc.n_layers, host_desc.n_pages, cache_desc.n_pages)
        if n == 0:
            raise KVQError("kvq_resident_state_bytes failed: KVQ_EINVAL")
        self._state = np.zeros((n + 7) // 8, np.uint64)
        self.state = self._state.ctypes.data
        hp, cp = Pool(host_base, host_desc), Pool(cache_base, cache_desc)
        _check(lib().kvq_resident_init(self.state, self._state.nbytes, ctypes.byref(hp), ctypes.byref(cp)),
               "kvq_resident_init")

    def map(self, layer: int, host_page_table, seq_lens):
        """Host planning: returns (cache_page_table, loads) as int32 numpy
        arrays ([n_seq, max_pages] and [n_loads, 2] of (host page, slot))."""
        hpt = np.ascontiguousarray(np.asarray(host_page_table, np.int32))
        sl = np.ascontiguousarray(np.asarray(seq_lens, np.int32))
        n_seq, max_pages = hpt.shape
        cpt = np.empty_like(hpt)
        loads = np.empty((self.cache_desc.n_pages, 2), np.int32)
        nl = ctypes.c_int()
        _check(lib().kvq_resident_map(self.state, layer, hpt.ctypes.data, n_seq, max_pages, sl.ctypes.data,
                                      cpt.ctypes.data, loads.ctypes.data, len(loads), ctypes.byref(nl)),
               "kvq_resident_map")
        return cpt, loads[:nl.value].copy()

    def load(self, layer: int, loads, stream=None):
        """Enqueue the page-in of the (host page, slot) pairs in loads."""
        ld = np.ascontiguousarray(np.asarray(loads, np.int32).reshape(-1, 2))
        _check(lib().kvq_resident_load(self.state, layer, ld.ctypes.data if len(ld) else None, len(ld),
                                       _stream(stream)), "kvq_resident_load")

    def slot_of(self, layer: int, host_page: int) -> int:
        s = ctypes.c_int()
        _check(lib().kvq_resident_query(self.state, layer, host_page, ctypes.byref(s)), "kvq_resident_query")
        return s.value

    def stats(self):
        """(hits, misses, evictions) since construction."""
        v = [ctypes.c_int64() for _ in range(3)]
        _check(lib().kvq_resident_stats(self.state, *[ctypes.byref(x) for x in v]), "kvq_resident_stats")
        return tuple(x.value for x in v)
