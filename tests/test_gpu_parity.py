"""GPU vs oracle parity at sizes the oracle finishes in seconds.

Bit-exact: the device generator against numpy, q_rotate and the codes and
fp16 scales written by kv_append.  Within the tolerance (fp32 output vs the
fp64 oracle on the GPU's own codes: relative L2 <= 1e-3 per output vector and
max-abs <= 2e-3): decode + combine for every format, on both the tensor-core
kernels and the CUDA-core control, across several tiles, pages, ragged tails,
split counts, group sizes and permuted page tables.  All calls go through the
C ABI (via the ctypes binding).
"""
import numpy as np
import pytest
import torch

import kvq_inputs
import oracle
import quantized_kv_cache_17_b200 as kvq
from kvq_inputs import device as kdev
from tests import gpu_common as gc
from tests import kvq_layout

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from quantized_kv_cache_17_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


FORMATS = ["int8", "q4_0", "k8v4", "fp8", "nvfp4"]
FP_FORMATS = ("fp8", "nvfp4")          # the CUDA-core control does not decode these


def small(fmt, Hq, Hkv, seq_lens, order="permuted", outlier="mul20", q_post=1.0, q_outliers=True, n_out=4,
          layers=1, name=None):
    return kvq_inputs.Workload(name=name or f"small_{fmt}_{Hq}_{Hkv}_{'_'.join(map(str, seq_lens))}", index=9,
                               fmt=fmt, n_layers=layers, n_q_heads=Hq, n_kv_heads=Hkv, seq_lens=list(seq_lens),
                               page_order=order, n_outlier=n_out, outlier_kind=outlier, q_post=q_post,
                               q_outliers=q_outliers)


# ---------------------------------------------------------------------------
def test_device_generator_bit_exact():
    w = kvq_inputs.workload("qwen27b_q4_0_262k")
    for tab, key, row0 in [(w.kv_table(3), w.k_key(3, 0), 262000), (w.q_table(1), w.q_key(1, 0), 0),
                           (kvq_inputs.workload("tiny_q4_0_1k").kv_table(0), 12345, 17),
                           (kvq_inputs.workload("qwen27b_int8_32k").kv_table(0), 999, 5)]:
        dt = kdev.DeviceTable(tab)
        got = kdev.gen_rows_device(key, dt, row0, 37).cpu().numpy()
        want = kvq_inputs.gen_rows(key, tab, row0, 37)
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("n_vec", [1, 3, 24, 1000])
def test_q_rotate_bit_exact(n_vec):
    w = kvq_inputs.workload("tiny_q4_0_1k")
    qh = kvq_inputs.gen_rows(77, w.q_table(0), 0, n_vec).reshape(-1, 256)[:n_vec].copy()
    q = torch.from_numpy(qh).cuda()
    got = kvq.q_rotate(q).cpu().numpy()
    want = oracle.fwht256_f32(qh)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    kvq.q_rotate(q, out=q)            # in place
    assert np.array_equal(q.cpu().numpy().view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("fmt", FORMATS)
def test_kv_append_bit_exact(fmt):
    w = small(fmt, 12, 2, [700, 1025], outlier="student_t", n_out=8)
    dw = kdev.build_pool(w, extra_slots=3, prefill_last=True)
    for b, T in enumerate(w.seq_lens):
        for g in range(w.n_kv_heads):
            kc, ks, vc, vs = gc.pool_codes(dw, 0, b, g)
            k = w.k_rows(0, b, 0, T)[:, g]
            v = w.v_rows(0, b, 0, T)[:, g]
            okc, oks, ovc, ovs = oracle.append_rows(fmt, k, v)
            assert np.array_equal(kc, okc) and np.array_equal(ks, oks)
            assert np.array_equal(vc, ovc) and np.array_equal(vs, ovs)


@pytest.mark.parametrize("fmt", FORMATS)
def test_kv_append_single_rows_match_batch(fmt):
    """Decode-style appends (one row per sequence per call) give the same bytes."""
    w = small(fmt, 8, 2, [40, 300])
    a = kdev.build_pool(w, prefill_last=True)
    bpool = kdev.build_pool(w, prefill_last=False)
    _, k, v, pos = kdev.step_inputs(w, [0])
    kvq.kv_append(bpool.pool, 0, k[0], v[0], pos, bpool.page_table)
    torch.cuda.synchronize()
    layout = kvq.pool_layout(a.pool.desc)
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            x = kvq_layout.gather_sequence(fmt, a.pool.buf, layout, 0, g, a.page_table_host[b], w.seq_lens[b])
            y = kvq_layout.gather_sequence(fmt, bpool.pool.buf, layout, 0, g, bpool.page_table_host[b],
                                           w.seq_lens[b])
            for p, r in zip(x, y):
                assert np.array_equal(p, r)


def test_kv_append_bad_slot_sets_status():
    w = small("q4_0", 4, 1, [300])
    dw = kdev.build_pool(w)
    pt = dw.page_table.clone()
    pt[0, 1] = 10_000                     # outside the pool: the row must be skipped, not written
    before = dw.pool.buf.clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    k = torch.randn(1, 1, 256, device="cuda")
    kvq.kv_append(dw.pool, 0, k, k, torch.tensor([299], dtype=torch.int32, device="cuda"), pt, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & kvq.STATUS_BAD_SLOT
    assert torch.equal(before, dw.pool.buf)


# ---------------------------------------------------------------------------
CASES = {
    # name: (workload, n_ctas values)
    "tiny_1k": (kvq_inputs.workload("tiny_q4_0_1k"), [0, 3]),
    "cross_page_1025": (kvq_inputs.scaled(kvq_inputs.workload("tiny_q4_0_1k"), [1025]), [0, 1]),
    "ragged_g6": (small("q4_0", 24, 4, [1, 77, 300, 1025], outlier="student_t", q_post=1 / 16,
                        q_outliers=False, n_out=8), [0, 5]),
    "ragged_g8": (small("q4_0", 16, 2, [513, 64, 8]), [0, 2]),
    # 300 steps split 300 ways: more units in one group than the merge takes in one pass
    "many_units_300": (small("q4_0", 6, 1, [19200], outlier="student_t", q_post=1 / 16, q_outliers=False, n_out=8),
                       [300]),
}


def _case(name, fmt):
    w, nctas = CASES[name]
    if fmt != w.fmt:
        import dataclasses
        w = dataclasses.replace(w, fmt=fmt, name=w.name + "_" + fmt)
    return w, nctas


@pytest.mark.parametrize("impl", ["mma", "mma_fused", "alu"])
@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("case", list(CASES))
def test_decode_matches_oracle(case, fmt, impl):
    if impl == "alu" and fmt in FP_FORMATS:
        pytest.skip("the CUDA-core control covers int8, q4_0 and k8v4 (KVQ_EUNSUPPORTED otherwise)")
    w, nctas = _case(case, fmt)
    mode = "fused" if impl == "mma_fused" else "split"
    dw = kdev.build_pool(w, extra_slots=2)
    q, k, v, pos = kdev.step_inputs(w, [0])
    kvq.kv_append(dw.pool, 0, k[0], v[0], pos, dw.page_table)          # this step's token
    refs = {}
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            refs[b, g] = gc.oracle_group(dw, 0, b, g)
    for n_ctas in nctas:
        out_f, out_bf, status, plan, info = gc.decode_step(dw, 0, q[0], impl=impl.split("_")[0], n_ctas=n_ctas,
                                                           mode=mode, repeat=2 if mode == "fused" else 1)
        assert status == 0
        G = w.group
        for (b, g), ref in refs.items():
            gc.assert_close(out_f[b, g * G:(g + 1) * G], ref, f"{case}/{fmt}/{impl}/nctas={n_ctas} b={b} g={g}")
        ref_all = np.stack([np.concatenate([refs[b, g] for g in range(w.n_kv_heads)]) for b in range(w.batch)])
        gc.assert_bf16_consistent(out_f, out_bf, ref_all)


@pytest.mark.parametrize("G", [1, 2, 3, 5, 7])
@pytest.mark.parametrize("fmt", ["int8", "q4_0", "k8v4", "fp8", "nvfp4"])
def test_decode_every_group_size(fmt, G):
    """Group sizes the shipped configurations do not use (1 = one query head
    per KV head, up to 7), in the split and fused forms and as the one-launch
    step, against the oracle."""
    w = small(fmt, 2 * G, 2, [700, 1, 257], outlier="student_t", q_post=1 / 16, q_outliers=False, n_out=8,
              name=f"groups_{fmt}_{G}")
    dw = kdev.build_pool(w, extra_slots=1)
    q, k, v, pos = kdev.step_inputs(w, [0])
    kvq.kv_append(dw.pool, 0, k[0], v[0], pos, dw.page_table)
    refs = {(b, g): gc.oracle_group(dw, 0, b, g) for b in range(w.batch) for g in range(w.n_kv_heads)}
    for mode, n_ctas in (("split", 0), ("fused", 7)):
        out_f, out_bf, status, _, _ = gc.decode_step(dw, 0, q[0], n_ctas=n_ctas, mode=mode)
        assert status == 0
        for (b, g), ref in refs.items():
            gc.assert_close(out_f[b, g * G:(g + 1) * G], ref, f"G={G}/{fmt}/{mode} b={b} g={g}")
    # the step appends the same token again (same bytes) and must give the same answer
    out_s, _, status, _, _ = gc.decode_step(dw, 0, q[0], mode="step", k_new=k[0], v_new=v[0])
    assert status == 0
    for (b, g), ref in refs.items():
        gc.assert_close(out_s[b, g * G:(g + 1) * G], ref, f"G={G}/{fmt}/step b={b} g={g}")


def test_decode_single_token_context():
    """T = 1: the output is that token's dequantised value, un-rotated."""
    w = small("q4_0", 6, 1, [1])
    dw = kdev.build_pool(w)
    q, k, v, pos = kdev.step_inputs(w, [0])
    kvq.kv_append(dw.pool, 0, k[0], v[0], pos, dw.page_table)
    out_f, _, status, _, _ = gc.decode_step(dw, 0, q[0])
    kc, ks, vc, vs = gc.pool_codes(dw, 0, 0, 0)
    vhat = oracle.fwht256_f64(oracle.dequant_rows(True, vc, vs))[0]
    for h in range(6):
        gc.assert_close(out_f[0, h], vhat, "T=1")
    assert status == 0


def test_decode_bad_page_slot_reports_status():
    w = small("q4_0", 4, 1, [600])
    dw = kdev.build_pool(w, prefill_last=True)
    dw.page_table[0, 1] = -7
    q, _, _, _ = kdev.step_inputs(w, [0])
    out_f, _, status, _, _ = gc.decode_step(dw, 0, q[0])
    assert status & kvq.STATUS_BAD_SLOT
    assert np.isfinite(out_f).all()


def test_decode_bad_plan_reports_status():
    w = small("int8", 4, 1, [300])
    dw = kdev.build_pool(w, prefill_last=True)
    plan, info = kvq.decode_plan(dw.pool.desc, dw.seq_lens, dw.page_table.shape[1], 0)
    plan[8 + 2] = 32            # unit start not on a 64-token step
    plan_d = torch.from_numpy(plan).cuda()
    ws = torch.empty(info.workspace_bytes // 4, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, _, _, _ = kdev.step_inputs(w, [0])
    kvq.paged_decode_attn(dw.pool, 0, q[0], dw.page_table, plan_d, info, ws, status)
    torch.cuda.synchronize()
    assert int(status.item()) & kvq.STATUS_BAD_PLAN


@pytest.mark.parametrize("mode", ["split", "fused"])
@pytest.mark.parametrize("G,n_ctas", [(4, 300), (6, 300), (4, 0)])
def test_group_merge_is_deterministic(mode, G, n_ctas):
    """The merge of a group's partials gives the same bits on every run: with
    several warps per head their sums are added in a fixed order, also over
    more units than one merge pass takes (300 units of one step each; n_ctas 0:
    100 units and the cooperative merge)."""
    w = small("q4_0", G, 1, [19200], outlier="student_t", q_post=1 / 16, q_outliers=False, n_out=8)
    dw = kdev.build_pool(w, prefill_last=True)
    q, _, _, _ = kdev.step_inputs(w, [0])
    runs = [gc.decode_step(dw, 0, q[0], n_ctas=n_ctas, mode=mode) for _ in range(6)]
    for out_f, out_bf, status, _, _ in runs:
        assert status == 0
        assert np.array_equal(out_f.view(np.int32), runs[0][0].view(np.int32))
        assert torch.equal(out_bf.view(torch.int16), runs[0][1].view(torch.int16))


@pytest.mark.parametrize("fmt", FORMATS)
def test_kv_append_q_rotate_matches_separate_calls(fmt):
    """The combined launch writes the same pool bytes and the same rotated query."""
    w = small(fmt, 12, 2, [300, 513])
    a = kdev.build_pool(w, prefill_last=False)
    b = kdev.build_pool(w, prefill_last=False)
    q, k, v, pos = kdev.step_inputs(w, [0])
    kvq.kv_append(a.pool, 0, k[0], v[0], pos, a.page_table)
    qa = kvq.q_rotate(q[0])
    qb = kvq.kv_append_q_rotate(b.pool, 0, k[0], v[0], pos, b.page_table, q[0])
    torch.cuda.synchronize()
    assert torch.equal(a.pool.buf, b.pool.buf)
    assert torch.equal(qa.view(torch.int32), qb.view(torch.int32))
    want = oracle.fwht256_f32(q[0].cpu().numpy().reshape(-1, 256))
    assert np.array_equal(qb.cpu().numpy().reshape(-1, 256).view(np.uint32), want.view(np.uint32))
    qc = kvq.kv_append_q_rotate(b.pool, 0, None, None, pos, b.page_table, q[0])    # rotation only
    torch.cuda.synchronize()
    assert torch.equal(qc.view(torch.int32), qa.view(torch.int32))


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("case", ["ragged_g6", "ragged_g8", "cross_page_1025", "many_units_300"])
def test_decode_step_matches_the_three_calls(case, fmt):
    """paged_decode_step = kv_append of the newest tokens + q_rotate + the
    combined decode: the same pool bytes and the same output bits, and the
    output within the tolerance of the oracle, for every plan size of the case
    (one unit per SM: cooperative group merge; 300 units: more than can be
    resident, so the last CTA of a group merges it, and units of one step)."""
    w, nctas = _case(case, fmt)
    for n_ctas in nctas:
        a = kdev.build_pool(w, extra_slots=2, prefill_last=False)
        b = kdev.build_pool(w, extra_slots=2, prefill_last=False)
        q, k, v, pos = kdev.step_inputs(w, [0])
        # stale bytes in the new token's row, which the step's copy of that tile may read
        for dw in (a, b):
            kvq.kv_append(dw.pool, 0, (-2.0 * k[0]).contiguous(), (0.5 * v[0].flip(-1)).contiguous(), pos,
                          dw.page_table)
        plan, info = kvq.decode_plan(a.pool.desc, a.seq_lens, a.page_table.shape[1], n_ctas)
        plan_d = torch.from_numpy(plan).cuda()
        outs = []
        for dw, fused_step in ((a, False), (b, True)):
            ws = torch.zeros(info.workspace_bytes // 4, dtype=torch.float32, device="cuda")
            status = torch.zeros(1, dtype=torch.int32, device="cuda")
            out_bf = torch.empty((w.batch, w.n_q_heads, 256), dtype=torch.bfloat16, device="cuda")
            out_f = torch.empty((w.batch, w.n_q_heads, 256), dtype=torch.float32, device="cuda")
            if fused_step:
                kvq.paged_decode_step(dw.pool, 0, q[0], k[0], v[0], dw.page_table, plan_d, info, ws, out_bf, out_f,
                                      status)
            else:
                kvq.kv_append(dw.pool, 0, k[0], v[0], pos, dw.page_table, status=status)
                qp = kvq.q_rotate(q[0]) if kvq.rotated_q(fmt) else q[0]
                kvq.paged_decode_attn_combined(dw.pool, 0, qp, dw.page_table, plan_d, info, ws, out_bf, out_f,
                                               status)
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            outs.append((out_f.cpu(), out_bf.cpu()))
        tag = f"step/{case}/{fmt}/nctas={n_ctas}"
        assert torch.equal(a.pool.buf, b.pool.buf), tag
        assert torch.equal(outs[0][0].view(torch.int32), outs[1][0].view(torch.int32)), tag
        assert torch.equal(outs[0][1].view(torch.int16), outs[1][1].view(torch.int16)), tag
        G = w.group
        got = outs[1][0].numpy()
        for bb in range(w.batch):
            for g in range(w.n_kv_heads):
                gc.assert_close(got[bb, g * G:(g + 1) * G], gc.oracle_group(b, 0, bb, g), f"{tag} b={bb} g={g}")


def test_group_wait_times_out_and_recovers():
    """Cooperative group merge with one unit of the group rejected by its plan
    check: that CTA never counts in, the group's other CTAs give up after their
    wait limit and report KVQ_STATUS_TIMEOUT (a bounded wait on the device, not
    a hang), the launch completes without a fault, and once the counters are
    zeroed again a good plan on the same workspace gives the oracle's result."""
    w = small("q4_0", 6, 1, [19200], outlier="student_t", q_post=1 / 16, q_outliers=False, n_out=8)
    dw = kdev.build_pool(w, prefill_last=True)
    q, _, _, _ = kdev.step_inputs(w, [0])
    qp = kvq.q_rotate(q[0])
    plan, info = kvq.decode_plan(dw.pool.desc, dw.seq_lens, dw.page_table.shape[1], 0)
    assert 2 <= info.n_units <= 148           # one group, cooperative merge
    bad = plan.copy()
    bad[8 + 4 * 1 + 2] += 32                  # unit 1 no longer starts on a step boundary
    ws = torch.zeros(info.workspace_bytes // 4, dtype=torch.float32, device="cuda")
    out_bf = torch.empty((1, 6, 256), dtype=torch.bfloat16, device="cuda")
    out_f = torch.empty((1, 6, 256), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvq.paged_decode_attn_combined(dw.pool, 0, qp, dw.page_table, torch.from_numpy(bad).cuda(), info, ws, out_bf,
                                   out_f, status)
    torch.cuda.synchronize()                  # completes: every wait is bounded
    st = int(status.item())
    assert st & kvq.STATUS_BAD_PLAN and st & kvq.STATUS_TIMEOUT
    ws.zero_()                                # a timeout leaves the group counter set
    status.zero_()
    out_f.fill_(float("nan"))
    kvq.paged_decode_attn_combined(dw.pool, 0, qp, dw.page_table, torch.from_numpy(plan).cuda(), info, ws, out_bf,
                                   out_f, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    gc.assert_close(out_f.cpu().numpy()[0], gc.oracle_group(dw, 0, 0, 0), "after the timeout")
