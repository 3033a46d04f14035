"""Host-resident KV with a device page cache, on the GPU ([Strata] "KV 从显存搬进内存
之后发生了什么": attention over the cached pages gives the same result as over a
fully resident cache, bit for bit).

A device pool D holds every layer; a pinned host pool H starts as a byte copy of
it; a cache C of fewer slots than the layers' pages together is fed from H by
kvq_resident_map / kvq_resident_load.  Each decode step appends the new token to
D, H and C and decodes D and C: the outputs must be the same bits, and every
cached page the same bytes as its host page.
"""
import dataclasses

import numpy as np
import pytest
import torch

import kvq_inputs
import quantized_kv_cache_17_b200 as kvq
from kvq_inputs import device as kdev

pytestmark = pytest.mark.gpu

FORMATS = ["int8", "q4_0", "k8v4", "fp8", "nvfp4"]


@pytest.fixture(scope="module", autouse=True)
def built():
    from quantized_kv_cache_17_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _decode(pool, layer, q, page_table, lens):
    plan, info = kvq.decode_plan(pool.desc, lens, page_table.shape[1])
    plan_d = torch.from_numpy(plan).cuda()
    ws = torch.zeros(info.workspace_bytes // 4, dtype=torch.float32, device="cuda")
    out_bf = torch.empty((len(lens), pool.desc.n_q_heads, 256), dtype=torch.bfloat16, device="cuda")
    out_f = torch.empty((len(lens), pool.desc.n_q_heads, 256), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvq.paged_decode_attn_combined(pool, layer, q, page_table, plan_d, info, ws, out_bf, out_f, status)
    return out_f, out_bf, status


@pytest.mark.parametrize("fmt,n_slots", [(f, 20) for f in FORMATS] + [("q4_0", 60), ("k8v4", 18)])
def test_resident_decode_is_bit_identical(fmt, n_slots):
    base = dataclasses.replace(kvq_inputs.workload("ragged4_q4_0"), fmt=fmt)
    w = kvq_inputs.scaled(base, [1500, 700, 2040], n_layers=3)   # 6 + 3 + 8 = 17 pages a layer
    dw = kdev.build_pool(w)
    D = dw.pool
    H = kvq.KVPool.allocate(D.desc, "pinned")
    H.buf.copy_(D.buf)
    C = kvq.KVPool.allocate(kvq.make_desc(1, w.n_kv_heads, w.n_q_heads, n_slots, fmt))
    rc = kvq.ResidentCache(H, C)
    layout = kvq.pool_layout(D.desc)
    S = layout.slot_stride
    lens0 = list(w.seq_lens)
    pages_per_layer = sum((T + 255) // 256 for T in lens0)
    for step in range(3):
        lens = [T + step for T in lens0]
        for layer in range(w.n_layers):
            qt = kdev.DeviceTable(w.q_table(layer), "cuda")
            kt = kdev.DeviceTable(w.kv_table(layer), "cuda")
            q = torch.stack([kdev.gen_rows_device(w.q_key(layer, b), qt, step, 1)[0] for b in range(w.batch)])
            k = torch.stack([kdev.gen_rows_device(w.k_key(layer, b), kt, T - 1, 1)[0] for b, T in enumerate(lens)])
            v = torch.stack([kdev.gen_rows_device(w.v_key(layer, b), kt, T - 1, 1)[0] for b, T in enumerate(lens)])
            pos = torch.tensor([T - 1 for T in lens], dtype=torch.int32, device="cuda")
            qp = kvq.q_rotate(q) if kvq.rotated_q(fmt) else q

            cpt, loads = rc.map(layer, dw.page_table_host, lens)
            if n_slots >= 3 * pages_per_layer and step > 0:
                assert len(loads) == 0                          # everything stays resident
            rc.load(layer, loads)
            cpt_d = torch.from_numpy(cpt).cuda()
            kvq.kv_append(D, layer, k, v, pos, dw.page_table)
            kvq.kv_append(H, layer, k, v, pos, dw.page_table)
            kvq.kv_append(C, 0, k, v, pos, cpt_d)

            f_d, bf_d, st_d = _decode(D, layer, qp, dw.page_table, lens)
            f_c, bf_c, st_c = _decode(C, 0, qp, cpt_d, lens)
            torch.cuda.synchronize()
            assert int(st_d.item()) == 0 and int(st_c.item()) == 0
            assert torch.equal(f_d.view(torch.int32), f_c.view(torch.int32)), (fmt, step, layer)
            assert torch.equal(bf_d.view(torch.int16), bf_c.view(torch.int16))
            # every page the call reads: cache slot == host page == device page
            for b, T in enumerate(lens):
                for p in range((T + 255) // 256):
                    hp, sl = int(dw.page_table_host[b, p]), int(cpt[b, p])
                    off = layer * layout.layer_stride + hp * S
                    hpage = H.buf[off:off + S].cuda()
                    assert torch.equal(C.buf[sl * S:(sl + 1) * S], hpage)
                    assert torch.equal(D.buf[off:off + S], hpage)
    hits, misses, ev = rc.stats()
    assert misses >= 3 * pages_per_layer or n_slots < 3 * pages_per_layer
    if n_slots < 3 * pages_per_layer:
        assert ev > 0 and misses > 3 * pages_per_layer
    else:
        assert ev == 0 and misses == 3 * pages_per_layer


def test_resident_load_rejects_device_memory_as_host_pool():
    d = kvq.make_desc(1, 2, 16, 4, "q4_0")
    fake_host = kvq.KVPool.allocate(d)                               # device memory, not pinned host memory
    C = kvq.KVPool.allocate(kvq.make_desc(1, 2, 16, 2, "q4_0"))
    rc = kvq.ResidentCache(fake_host, C)
    _, loads = rc.map(0, np.array([[0]], np.int32), [10])
    with pytest.raises(kvq.KVQError, match="EINVAL"):
        rc.load(0, loads)


@pytest.mark.parametrize("fmt", ["q4_0", "k8v4"])
def test_resident_prefill_is_bit_identical(fmt):
    """A prompt chunk appended and attended through the page cache gives the same
    bits as through the full device pool, unsplit and with a key-range split."""
    base = dataclasses.replace(kvq_inputs.workload("ragged4_q4_0"), fmt=fmt)
    w = kvq_inputs.scaled(base, [1800, 900], n_layers=2)
    dw = kdev.build_pool(w)
    D = dw.pool
    H = kvq.KVPool.allocate(D.desc, "pinned")
    H.buf.copy_(D.buf)
    C = kvq.KVPool.allocate(kvq.make_desc(1, w.n_kv_heads, w.n_q_heads, 12, fmt))
    rc = kvq.ResidentCache(H, C)
    n_tok = 40
    for layer in range(w.n_layers):
        T = w.seq_lens[0]
        pos0 = T - 1 - n_tok            # the chunk ends one token before the pool's fill
        cpt, loads = rc.map(layer, dw.page_table_host, [T, w.seq_lens[1]])
        rc.load(layer, loads)
        cpt_d = torch.from_numpy(cpt).cuda()
        qt = kdev.DeviceTable(w.q_table(layer), "cuda")
        q = kdev.gen_rows_device(w.q_key(layer, 0), qt, 0, n_tok)
        qp = kvq.q_rotate(q) if kvq.rotated_q(fmt) else q
        for n_split in (1, 3):
            outs = []
            for pool, lay, pt in ((D, layer, dw.page_table), (C, 0, cpt_d)):
                o_bf = torch.empty((n_tok, w.n_q_heads, 256), dtype=torch.bfloat16, device="cuda")
                o_f = torch.empty((n_tok, w.n_q_heads, 256), dtype=torch.float32, device="cuda")
                st = torch.zeros(1, dtype=torch.int32, device="cuda")
                kvq.paged_prefill_attn(pool, lay, qp, 0, pos0, pt, o_bf, o_f, status=st, n_split=n_split)
                torch.cuda.synchronize()
                assert int(st.item()) == 0
                outs.append((o_f, o_bf))
            assert torch.equal(outs[0][0].view(torch.int32), outs[1][0].view(torch.int32)), (fmt, layer, n_split)
            assert torch.equal(outs[0][1].view(torch.int16), outs[1][1].view(torch.int16))
