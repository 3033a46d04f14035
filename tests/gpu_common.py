"""Helpers shared by the GPU tests: run one decode step through the C ABI and
compute the oracle's answer for the same (layer, sequence, KV head)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import quantized_kv_cache_17_b200 as kvq
from tests import kvq_layout

REL_L2 = 1e-3     # attention output tolerance, fp32 output vs fp64 oracle
MAX_ABS = 2e-3


def decode_step(dw, layer, q, impl="mma", n_ctas=0, status=None, mode="split", repeat=1, k_new=None, v_new=None):
    """q: [B, Hq, 256] fp32 device (unrotated).  mode 'split': decode then
    attn_combine; 'fused': the *_combined entry point (run `repeat` times on the
    same workspace); 'step': paged_decode_step, which also appends k_new / v_new
    ([B, Hkv, 256], the token at seq_len - 1) and rotates q itself.
    Returns (out_f32, out_bf16, status, plan, info)."""
    w = dw.w
    plan, info = kvq.decode_plan(dw.pool.desc, dw.seq_lens, dw.page_table.shape[1], n_ctas)
    plan_d = torch.from_numpy(plan).cuda()
    ws = torch.zeros(info.workspace_bytes // 4, dtype=torch.float32, device="cuda")
    qp = kvq.q_rotate(q) if kvq.rotated_q(w.fmt) and mode != "step" else q
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out_bf = torch.empty((w.batch, w.n_q_heads, 256), dtype=torch.bfloat16, device="cuda")
    out_f = torch.empty((w.batch, w.n_q_heads, 256), dtype=torch.float32, device="cuda")
    for _ in range(repeat):
        out_bf.fill_(float("nan"))
        out_f.fill_(float("nan"))
        if mode == "step":
            kvq.paged_decode_step(dw.pool, layer, q, k_new, v_new, dw.page_table, plan_d, info, ws, out_bf, out_f,
                                  status)
        elif mode == "fused":
            kvq.paged_decode_attn_combined(dw.pool, layer, qp, dw.page_table, plan_d, info, ws, out_bf, out_f, status)
        else:
            kvq.paged_decode_attn(dw.pool, layer, qp, dw.page_table, plan_d, info, ws, status,
                                  cudacore=(impl == "alu"))
            kvq.attn_combine(ws, plan_d, info, kvq.rotated_v(w.fmt), out_bf, out_f)
    torch.cuda.synchronize()
    return out_f.cpu().numpy(), out_bf.cpu(), int(status.item()), plan, info


def pool_codes(dw, layer, b, g):
    """GPU codes/scales of sequence b, KV head g, decoded with the tests' layout decoder."""
    layout = kvq.pool_layout(dw.pool.desc)
    return kvq_layout.gather_sequence(dw.w.fmt, dw.pool.buf, layout, layer, g, dw.page_table_host[b],
                                      dw.seq_lens[b])


def oracle_group(dw, layer, b, g, codes=None):
    """fp64 oracle output [G, 256] for (layer, sequence b, KV head g) on the GPU's codes."""
    w = dw.w
    G = w.group
    kc, ks, vc, vs = codes if codes is not None else pool_codes(dw, layer, b, g)
    q = w.q_row(layer, b)[g * G:(g + 1) * G]
    qp = oracle.q_prepare(w.fmt, q)
    return oracle.attn_decode(w.fmt, qp, kc, ks, vc, vs)


def assert_close(got: np.ndarray, ref: np.ndarray, what=""):
    got = np.asarray(got, np.float64).reshape(-1, 256)
    ref = np.asarray(ref, np.float64).reshape(-1, 256)
    err = got - ref
    rel = np.linalg.norm(err, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-30)
    mabs = np.abs(err).max()
    assert rel.max() <= REL_L2 and mabs <= MAX_ABS, f"{what}: rel-L2 {rel.max():.3e}, max-abs {mabs:.3e}"
    return rel.max(), mabs


def assert_bf16_consistent(out_f: np.ndarray, out_bf: torch.Tensor, ref: np.ndarray):
    """bf16 output = round-to-nearest-even of the f32 output, and therefore no
    farther from the oracle than half a bf16 ulp plus the f32 output's error."""
    bits = out_bf.view(torch.int16).numpy().view(np.uint16).reshape(-1)
    f = np.asarray(out_f, np.float32).reshape(-1)
    want = oracle.f32_to_bf16_bits(f)
    assert np.array_equal(bits, want)
    g = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    r = np.asarray(ref, np.float64).reshape(-1)
    half_ulp = np.maximum(np.abs(f), np.abs(r)) * 2.0 ** -8
    assert np.all(np.abs(g - r) <= half_ulp + np.abs(f - r) + 1e-30)
