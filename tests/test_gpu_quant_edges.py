"""GPU quantiser on the edge cases the oracle is pinned on, bit for bit.

The seeded N(0,1) and Student-t rows of the other tests almost never produce
these cases, so they are crafted here: an all-zero block (q4_0 scale -0, codes
8; int8 scale 0, codes 0), ties in |x| inside one lane and across lanes (the
first index sets the sign of the q4_0 scale), x/d landing exactly on k + 1/2
(round half to even), the true-division case where x * (1/d) would round the
other way, subnormal fp16 scales, int8 codes that saturate at -127, constant
blocks and single non-zero values.

Both GPU encoders are checked against the oracle: kv_append, and the encode of
the newest token inside paged_decode_step.  For the rotated parts (q4_0 K and
V, k8v4 V) the crafted values are the ones the quantiser must see after the
rotation, so the input is x = H/16 y computed with the oracle's fp32 transform;
the test first checks that the transform of x gives y back exactly, so the
edge cases really reach the quantiser.
"""
import numpy as np
import pytest
import torch

import kvq_inputs
import oracle
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


def q4_rows():
    """Vectors whose 32-value blocks hit the q4_0 edge cases (the values the
    quantiser sees).  Each vector only mixes values whose rotation sums are
    exact in fp32, so that it survives the round trip through the transform."""
    a = np.zeros(256, np.float32)
    a[0:8] = [-8.0, 2.5, 3.5, -0.5, 0.5, 1.5, 7.5, -7.5]      # d = 1, ties round half to even
    a[32:36] = [8.0, 2.5, -2.5, 4.0]                          # d = -1
    # block 2 all zero: d = 0/-8 = -0, codes 8
    a[96 + 5] = 3.25                                          # single value
    a[128:160] = -1.75                                        # constant block
    a[160] = 2.0                                              # |x| tie across lanes (dims 160 / 168):
    a[168] = -2.0                                             #   the first index wins, d = -0.25
    a[224] = -3.0                                             # the same with the signs swapped: d = 0.375
    a[233] = 3.0
    b = np.zeros(256, np.float32)
    b[0] = np.float32(-49.46875)                              # true division: d = 6.1835938 and
    b[1] = np.float32(21.642578)                              #   x/d = 3.5 exactly (x * fl(1/d) is not)
    c = np.zeros(256, np.float32)
    c[32] = np.float32(8 * 2.0 ** -20)                        # subnormal fp16 scale d = -2^-20
    c[33] = np.float32(-3 * 2.0 ** -20)
    c[34] = np.float32(2.5 * 2.0 ** -20)                      #   with a tie at x/d = -2.5
    d = np.zeros(256, np.float32)
    d[64:68] = [5.0, -5.0, 5.0, -5.0]                         # tie inside one lane: the first (+5) wins
    d[100] = -6.0                                             # tie of the block max across lanes,
    d[120] = 6.0                                              #   negative first
    e = np.zeros(256, np.float32)
    e[160:192] = np.float32(0.1)                              # constant non-dyadic block
    return [a, b, c, d, e]


def i8_rows():
    """Vectors whose 64-value groups hit the int8 edge cases."""
    a = np.zeros(256, np.float32)
    a[0:5] = [127.0, 2.5, -2.5, 126.5, -127.0]                # d = 1, ties, -127
    a[64 + 9] = -0.3                                          # single value -> -127
    # group 2 all zero: d = 0, codes 0
    a[192:256] = 0.5                                          # constant -> 127
    b = np.zeros(256, np.float32)
    b[64] = np.float32(-127 * 1.4 * 2.0 ** -24)               # subnormal d = 2^-24; |x|/d = 177.8 saturates
    b[0:3] = [-1.5, 0.5, 190.5]                               # x/d on halves with d = 1.5
    b[128:192] = -0.7                                         # constant negative group
    return [a, b]


def f8_rows():
    """Vectors that hit the fp8 edge cases (one fp16 scale d per vector)."""
    a = np.zeros(256, np.float32)
    a[0] = 448.0                                              # d = 1: codes are the E4M3 of x itself
    a[1:9] = [2.0 ** -9, 3 * 2.0 ** -10, 2.0 ** -10, -2.0 ** -11, 1.0625, 17.0, -18.0, 232.0]   # subnormals, ties
    a[9:12] = [-0.0, 1e-30, -1e-30]                           # signed zeros out of underflow
    b = np.zeros(256, np.float32)                             # all zero: d = 0, codes +0
    c = np.zeros(256, np.float32)
    c[5] = np.float32(448.0 * (1 + 0.9 * 2.0 ** -11))         # d rounds down: x / d > 448 saturates
    c[6] = -c[5]
    c[7] = 3.0
    d = (np.arange(256, dtype=np.float32) - 128) * np.float32(0.37)    # a ramp
    return [a, b, c, d]


def f4_rows():
    """Vectors whose 16-value blocks hit the nvfp4 edge cases (E4M3 scale s per block)."""
    a = np.zeros(256, np.float32)
    a[0:8] = [6.0, 0.25, 0.75, 1.25, 2.5, 3.5, 5.0, -5.0]    # s = 1: ties go to the even code
    a[16:20] = [6.0, -0.0, 7.0, -1.75]                        # s = 1 again; 7 saturates to 6 s
    # block 2 all zero: s = 0, codes +0
    a[48:64] = np.float32(0.01)                               # s in the E4M3 subnormal range
    a[64] = np.float32(6.0 * 448.0 * 1.5)                     # max|x| / 6 above 448: s saturates, codes too
    a[65] = -1000.0
    a[80:96] = np.linspace(-3, 3, 16, dtype=np.float32)
    a[96:112] = np.float32(6.0 * 2.0 ** -12)                  # s underflows to 0
    b = (np.arange(256, dtype=np.float32) % 17 - 8) * np.float32(0.61)
    return [a, b]


ROWS = {"q4": q4_rows, "i8": i8_rows, "e4m3": f8_rows, "e2m1": f4_rows}


def stored_domain(fmt):
    """(K rows, V rows) as the quantiser must see them, and the inputs that
    produce them (rotated parts pass through the inverse transform)."""
    kp, vp, k_rot, v_rot = oracle.PARTS[fmt]
    kq = ROWS[kp]()
    vq = ROWS[vp]()
    n = max(len(kq), len(vq))
    kq = [kq[i % len(kq)] for i in range(n)]
    vq = [vq[i % len(vq)] for i in range(n)]

    def to_input(y, rot):
        y = np.stack(y)
        if not rot:
            return y
        x = oracle.fwht256_f32(y)
        assert np.array_equal(oracle.fwht256_f32(x).view(np.uint32), y.view(np.uint32)), \
            "the crafted rows do not survive the rotation exactly"
        return x

    return to_input(kq, k_rot), to_input(vq, v_rot), np.stack(kq), np.stack(vq)


def small(fmt, T):
    return kvq_inputs.Workload(name=f"edges_{fmt}", index=9, fmt=fmt, n_layers=1, n_q_heads=8, n_kv_heads=1,
                               seq_lens=[T], page_order="permuted", n_outlier=4, outlier_kind="mul20",
                               q_post=1.0, q_outliers=True)


def _check_codes(dw, fmt, pos, k_in, v_in, k_seen, v_seen, tag):
    kc, ks, vc, vs = gc.pool_codes(dw, 0, 0, 0)
    okc, oks, ovc, ovs = oracle.append_rows(fmt, k_in, v_in)
    sl = slice(pos, pos + len(k_in))
    assert np.array_equal(kc[sl], okc), f"{tag}: K codes"
    assert np.array_equal(ks[sl], oks), f"{tag}: K scales"
    assert np.array_equal(vc[sl], ovc), f"{tag}: V codes"
    assert np.array_equal(vs[sl], ovs), f"{tag}: V scales"
    # the oracle itself on the values the quantiser saw (no rotation involved)
    quant_k = oracle.QUANT[oracle.PARTS[fmt][0]]
    quant_v = oracle.QUANT[oracle.PARTS[fmt][1]]
    for i in range(len(k_in)):
        c, s = quant_k(k_seen[i])
        assert np.array_equal(okc[i].view(np.uint8), c.view(np.uint8)) and np.array_equal(oks[i], s)
        c, s = quant_v(v_seen[i])
        assert np.array_equal(ovc[i].view(np.uint8), c.view(np.uint8)) and np.array_equal(ovs[i], s)


@pytest.mark.parametrize("fmt", ["int8", "q4_0", "k8v4", "fp8", "nvfp4"])
def test_kv_append_edge_cases_bit_exact(fmt):
    k_in, v_in, k_seen, v_seen = stored_domain(fmt)
    n = len(k_in)
    # rows at positions 5..5+n-1 and again at 255..: inside a tile and across a page boundary
    for pos in (5, 255):
        w = small(fmt, 300)
        dw = kdev.build_pool(w, prefill_last=True)
        k = torch.from_numpy(k_in[:, None, :].copy()).cuda()
        v = torch.from_numpy(v_in[:, None, :].copy()).cuda()
        p = torch.arange(pos, pos + n, dtype=torch.int32, device="cuda")
        seq = torch.zeros(n, dtype=torch.int32, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        kvq.kv_append(dw.pool, 0, k, v, p, dw.page_table, row_seq=seq, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        _check_codes(dw, fmt, pos, k_in, v_in, k_seen, v_seen, f"kv_append/{fmt}/pos={pos}")


@pytest.mark.parametrize("fmt", ["int8", "q4_0", "k8v4", "fp8", "nvfp4"])
def test_decode_step_encodes_edge_cases_bit_exact(fmt):
    """The decode step's own encode of the newest token, one crafted row per
    step, and the step's output against the oracle on the resulting codes."""
    k_in, v_in, k_seen, v_seen = stored_domain(fmt)
    for i in range(len(k_in)):
        T = 300 + 37 * i
        w = small(fmt, T)
        dw = kdev.build_pool(w)
        q, _, _, _ = kdev.step_inputs(w, [0])
        plan, info = kvq.decode_plan(dw.pool.desc, dw.seq_lens, dw.page_table.shape[1], 0)
        plan_d = torch.from_numpy(plan).cuda()
        ws = torch.zeros(info.workspace_bytes // 4, dtype=torch.float32, device="cuda")
        out_bf = torch.empty((1, 8, 256), dtype=torch.bfloat16, device="cuda")
        out_f = torch.empty((1, 8, 256), dtype=torch.float32, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        kn = torch.from_numpy(k_in[i][None, None, :].copy()).cuda()
        vn = torch.from_numpy(v_in[i][None, None, :].copy()).cuda()
        kvq.paged_decode_step(dw.pool, 0, q[0], kn, vn, dw.page_table, plan_d, info, ws, out_bf, out_f, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        _check_codes(dw, fmt, T - 1, k_in[i:i + 1], v_in[i:i + 1], k_seen[i:i + 1], v_seen[i:i + 1],
                     f"step/{fmt}/row {i}")
        gc.assert_close(out_f.cpu().numpy()[0], gc.oracle_group(dw, 0, 0, 0), f"step/{fmt}/row {i} output")
