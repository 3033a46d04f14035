"""Device-side workload construction: the GPU twin of the seeded generator and
the helpers that fill a pool through the library's public ``kv_append``.

Shared by the GPU tests, ``__graft_entry__.smoke()`` and ``bench.py``.  It
holds none of the method's arithmetic: values come from the counter-based
generator, the pool is filled only by calling the library.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import List, Optional

import numpy as np
import torch

from . import ChannelTable, Workload

_HERE = os.path.dirname(os.path.abspath(__file__))
GEN_LIB = os.path.join(_HERE, "libkvq_gen.so")
_gen = None


def gen_lib():
    global _gen
    if _gen is None:
        if not os.path.exists(GEN_LIB):
            raise RuntimeError(f"{GEN_LIB} missing: run `python -m quantized_kv_cache_17_b200.build`")
        L = ctypes.CDLL(GEN_LIB)
        L.kvq_gen_rows.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_uint64,
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p]
        L.kvq_gen_rows.restype = ctypes.c_int
        _gen = L
    return _gen


class DeviceTable:
    """A ChannelTable resident on the device."""

    def __init__(self, t: ChannelTable, device="cuda"):
        self.mul = torch.from_numpy(np.ascontiguousarray(t.mul.reshape(-1))).to(device)
        self.kind = torch.from_numpy(np.ascontiguousarray(t.kind.reshape(-1))).to(device)
        self.post = float(t.post)
        self.H = t.mul.shape[0]


def gen_rows_device(key: int, table: DeviceTable, row0: int, n_rows: int, out: Optional[torch.Tensor] = None):
    """Rows [row0, row0+n_rows) of a [rows, H, 256] fp32 tensor, on the device."""
    if out is None:
        out = torch.empty((n_rows, table.H, 256), dtype=torch.float32, device=table.mul.device)
    rc = gen_lib().kvq_gen_rows(out.data_ptr(), row0, n_rows, table.H, key, table.mul.data_ptr(),
                                table.kind.data_ptr(), table.post, torch.cuda.current_stream().cuda_stream)
    if rc != 0:
        raise RuntimeError(f"kvq_gen_rows failed: {rc}")
    return out


@dataclass
class DeviceWorkload:
    w: Workload
    pool: object               # quantized_kv_cache_17_b200.KVPool
    page_table: torch.Tensor   # int32 [B, max_pages] on the device
    page_table_host: np.ndarray
    seq_lens: List[int]
    layers: List[int]


def build_pool(w: Workload, layers: Optional[List[int]] = None, extra_slots: int = 0, chunk_rows: int = 8192,
               prefill_last: bool = False, device="cuda") -> DeviceWorkload:
    """Allocate a pool for workload w and fill tokens [0, T_b - 1) of every
    sequence (all T_b tokens if prefill_last) in the given layers through
    kv_append.  Other layers of the pool are left zero."""
    import quantized_kv_cache_17_b200 as kvq
    layers = list(range(w.n_layers)) if layers is None else list(layers)
    n_slots = w.pages_needed() + extra_slots
    pt_host = w.page_table(n_slots)
    desc = kvq.make_desc(w.n_layers, w.n_kv_heads, w.n_q_heads, n_slots, w.fmt)
    pool = kvq.KVPool.allocate(desc, device)
    pt = torch.from_numpy(pt_host).to(device)
    for layer in layers:
        tab = DeviceTable(w.kv_table(layer), device)
        for b, T in enumerate(w.seq_lens):
            n_fill = T if prefill_last else T - 1
            for r0 in range(0, n_fill, chunk_rows):
                n = min(chunk_rows, n_fill - r0)
                k = gen_rows_device(w.k_key(layer, b), tab, r0, n)
                v = gen_rows_device(w.v_key(layer, b), tab, r0, n)
                pos = torch.arange(r0, r0 + n, dtype=torch.int32, device=device)
                seq = torch.full((n,), b, dtype=torch.int32, device=device)
                kvq.kv_append(pool, layer, k, v, pos, pt, row_seq=seq)
    torch.cuda.synchronize()
    return DeviceWorkload(w, pool, pt, pt_host, list(w.seq_lens), layers)


def step_inputs(w: Workload, layers: List[int], device="cuda"):
    """This step's inputs per layer: q [B, Hq, 256], k_new/v_new [B, Hkv, 256]
    (the generator rows at position T_b - 1), pos [B]."""
    qs, ks, vs = [], [], []
    for layer in layers:
        qt = DeviceTable(w.q_table(layer), device)
        kt = DeviceTable(w.kv_table(layer), device)
        q = torch.empty((w.batch, w.n_q_heads, 256), dtype=torch.float32, device=device)
        k = torch.empty((w.batch, w.n_kv_heads, 256), dtype=torch.float32, device=device)
        v = torch.empty_like(k)
        for b, T in enumerate(w.seq_lens):
            q[b] = gen_rows_device(w.q_key(layer, b), qt, 0, 1)[0]
            k[b] = gen_rows_device(w.k_key(layer, b), kt, T - 1, 1)[0]
            v[b] = gen_rows_device(w.v_key(layer, b), kt, T - 1, 1)[0]
        qs.append(q)
        ks.append(k)
        vs.append(v)
    pos = torch.tensor([T - 1 for T in w.seq_lens], dtype=torch.int32, device=device)
    return torch.stack(qs), torch.stack(ks), torch.stack(vs), pos
