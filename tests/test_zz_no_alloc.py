"""The workspace-free q4_0 decode entry point.

Some callers cannot allocate device memory (a host that owns all device memory
and passes a library only the buffers of the call), so they cannot provide the
split-K workspace.  paged_decode_attn_q4_0_noalloc uses a scratch array inside
the library instead.  This test calls it through the C ABI twice in a row and
checks each output against the entry point that takes a caller workspace.  Both
run the same deterministic kernel on the same plan, so the outputs must agree
bit for bit (a tolerance would hide a wrong scratch offset or a stale counter
that moves the result by less than the attention tolerance).  The file sits on
its own and pytest collects it last.
"""
import numpy as np
import pytest
import torch

import kvq_inputs
import quantized_kv_cache_17_b200 as kvq
from kvq_inputs import device as kdev
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from quantized_kv_cache_17_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_noalloc_matches_workspace_entry_point():
    w = kvq_inputs.Workload(name="noalloc_q4_0", index=9, fmt="q4_0", n_layers=1, n_q_heads=24, n_kv_heads=4,
                            seq_lens=[1, 77, 300, 1025, 4000], page_order="permuted", n_outlier=8,
                            outlier_kind="student_t", q_post=1 / 16, q_outliers=False)
    dw = kdev.build_pool(w, extra_slots=3)
    q, k, v, pos = kdev.step_inputs(w, [0])
    kvq.kv_append(dw.pool, 0, k[0], v[0], pos, dw.page_table)
    plan, info = kvq.decode_plan(dw.pool.desc, dw.seq_lens, dw.page_table.shape[1], 0)
    assert info.workspace_bytes <= kvq.NOALLOC_WS_BYTES
    plan_d = torch.from_numpy(plan).cuda()
    qp = kvq.q_rotate(q[0])
    shape = (w.batch, w.n_q_heads, 256)

    ws = torch.zeros(info.workspace_bytes // 4, dtype=torch.float32, device="cuda")
    ref_bf = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    ref_f = torch.empty(shape, dtype=torch.float32, device="cuda")
    kvq.paged_decode_attn_combined(dw.pool, 0, qp, dw.page_table, plan_d, info, ws, ref_bf, ref_f)
    torch.cuda.synchronize()
    ref = ref_f.cpu().numpy()

    for _ in range(2):
        out_bf = torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")
        out_f = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        kvq.paged_decode_attn_q4_0_noalloc(dw.pool, 0, qp, dw.page_table, plan_d, info, out_bf, out_f, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        got = out_f.cpu().numpy()
        assert np.isfinite(got).all()
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), "fp32 output differs from the workspace path"
        assert torch.equal(out_bf.cpu().view(torch.int16), ref_bf.cpu().view(torch.int16)), "bf16 output differs"
        gc.assert_close(got, ref, "noalloc vs workspace entry point")


def test_noalloc_rejects_a_plan_larger_than_its_scratch():
    d = kvq.make_desc(1, 4, 24, 1024, "q4_0")
    plan, info = kvq.decode_plan(d, [262144], max_pages=1024, n_ctas=4000)
    assert info.workspace_bytes > kvq.NOALLOC_WS_BYTES
    pool = kvq.KVPool(d, torch.empty(16, dtype=torch.uint8, device="cuda"))
    with pytest.raises(kvq.KVQError, match="KVQ_ESIZE"):
        kvq.paged_decode_attn_q4_0_noalloc(pool, 0, torch.empty(24, 256, device="cuda"),
                                           torch.zeros((1, 1024), dtype=torch.int32, device="cuda"),
                                           torch.from_numpy(plan).cuda(), info,
                                           torch.empty((1, 24, 256), dtype=torch.bfloat16, device="cuda"))


def test_noalloc_rejects_an_info_that_does_not_match_its_plan_sizes():
    """An info whose workspace size is not the one its unit and group counts
    give is refused before the scratch array is touched (the counter clear is
    sized from it)."""
    w = kvq_inputs.Workload(name="noalloc_bad_info", index=9, fmt="q4_0", n_layers=1, n_q_heads=24, n_kv_heads=4,
                            seq_lens=[300], page_order="contiguous", n_outlier=8, outlier_kind="student_t",
                            q_post=1 / 16, q_outliers=False)
    dw = kdev.build_pool(w)
    plan, info = kvq.decode_plan(dw.pool.desc, dw.seq_lens, dw.page_table.shape[1], 0)
    plan_d = torch.from_numpy(plan).cuda()
    q = torch.zeros((1, 24, 256), dtype=torch.float32, device="cuda")
    out = torch.empty((1, 24, 256), dtype=torch.bfloat16, device="cuda")
    bad = kvq.PlanInfo(info.n_units + 1000, info.n_seq, info.n_kv_heads, info.group, info.plan_len,
                       info.chunk_tokens, info.workspace_bytes)
    with pytest.raises(kvq.KVQError, match="KVQ_EINVAL"):
        kvq.paged_decode_attn_q4_0_noalloc(dw.pool, 0, q, dw.page_table, plan_d, bad, out)
    small = kvq.PlanInfo(info.n_units, info.n_seq, info.n_kv_heads, info.group, info.plan_len,
                         info.chunk_tokens, 64)
    with pytest.raises(kvq.KVQError, match="KVQ_EINVAL"):
        kvq.paged_decode_attn_q4_0_noalloc(dw.pool, 0, q, dw.page_table, plan_d, small, out)
