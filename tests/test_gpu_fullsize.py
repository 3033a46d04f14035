"""Parity at the full workload sizes, in the launch configuration the benchmark
times (plan with one unit per SM, the decode step kernel), on sampled
outputs the oracle computes one at a time: whole (sequence, KV head) groups of
attention output over the full context, and bit-exact codes for sampled token
positions regenerated on the CPU."""
import numpy as np
import pytest
import torch

import kvq_inputs
import oracle
from kvq_inputs import device as kdev
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu

# workload -> sampled (sequence, KV head) pairs
SAMPLES = {
    "qwen27b_int8_32k": [(0, 0), (0, 3)],
    "flashnext_k8v4_128k": [(0, 1)],
    "qwen27b_q4_0_262k": [(0, 0), (0, 2)],
    "ragged4_q4_0": [(0, 1), (2, 2), (3, 3)],
    "ragged4_k8v4": [(1, 0), (2, 3)],
    "qwen27b_fp8_262k": [(0, 1)],
    "qwen27b_nvfp4_262k": [(0, 3)],
}


@pytest.fixture(scope="module", autouse=True)
def built():
    from quantized_kv_cache_17_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("mode", ["step", "fused"])
@pytest.mark.parametrize("name", list(SAMPLES))
def test_full_size_sampled(name, mode):
    """mode 'step': paged_decode_step, the launch the benchmark times (it
    appends the newest token itself); 'fused': kv_append, then the combined
    decode."""
    w = kvq_inputs.workload(name)
    layer = w.n_layers - 1
    dw = kdev.build_pool(w, layers=[layer], extra_slots=7)
    q, k, v, pos = kdev.step_inputs(w, [layer])
    import quantized_kv_cache_17_b200 as kvq
    if mode == "fused":
        kvq.kv_append(dw.pool, layer, k[0], v[0], pos, dw.page_table)
    out_f, out_bf, status, plan, info = gc.decode_step(dw, layer, q[0], mode=mode, k_new=k[0], v_new=v[0])
    assert status == 0
    rng = np.random.default_rng(w.seed)
    G = w.group
    for b, g in SAMPLES[name]:
        T = w.seq_lens[b]
        codes = gc.pool_codes(dw, layer, b, g)
        toks = np.unique(np.concatenate([rng.integers(0, T, 40), [0, T - 1, T // 2]]))
        kk = np.stack([w.k_rows(layer, b, int(t), 1)[0, g] for t in toks])
        vv = np.stack([w.v_rows(layer, b, int(t), 1)[0, g] for t in toks])
        okc, oks, ovc, ovs = oracle.append_rows(w.fmt, kk, vv)
        kc, ks, vc, vs = codes
        assert np.array_equal(kc[toks], okc) and np.array_equal(ks[toks], oks)
        assert np.array_equal(vc[toks], ovc) and np.array_equal(vs[toks], ovs)
        ref = gc.oracle_group(dw, layer, b, g, codes)
        gc.assert_close(out_f[b, g * G:(g + 1) * G], ref, f"{name} b={b} g={g}")
        gc.assert_bf16_consistent(out_f[b, g * G:(g + 1) * G], out_bf[b, g * G:(g + 1) * G], ref)
