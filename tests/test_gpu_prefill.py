"""Chunked prefill over the quantised cache (paged_prefill_attn), after the
chunk's multi-token kv_append, against the fp64 oracle.

Each chunk token i (position pos0 + i) must equal the oracle's single-query
attention over the sequence's first pos0 + i + 1 tokens, on the GPU's own codes
(the decode's contract, per token).  The chunk's codes come from one kv_append
call of all its rows and must be bit-exact against the oracle's append.
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

FORMATS = ["int8", "q4_0", "k8v4", "fp8", "nvfp4"]


@pytest.fixture(scope="module", autouse=True)
def built():
    from quantized_kv_cache_17_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _workload(fmt, Hq, Hkv, T, name, order="permuted", outlier="mul20", q_post=1.0, q_outliers=True, n_out=4):
    return kvq_inputs.Workload(name=name, index=9, fmt=fmt, n_layers=1, n_q_heads=Hq, n_kv_heads=Hkv, seq_lens=[T],
                               page_order=order, n_outlier=n_out, outlier_kind=outlier, q_post=q_post,
                               q_outliers=q_outliers)


def _prefill(w, n_tok, split=None, n_split=None):
    """Pool with the sequence's tokens [0, T - 1); the chunk [T - n_tok, T) appended
    in one kv_append call; then the prefill of the chunk (in calls of `split`
    tokens when given).  Returns (dw, pos0, out_f32 [n_tok, Hq, 256], out_bf16)."""
    T = w.seq_lens[0]
    pos0 = T - n_tok
    dw = kdev.build_pool(w)
    kt = kdev.DeviceTable(w.kv_table(0), "cuda")
    k = kdev.gen_rows_device(w.k_key(0, 0), kt, pos0, n_tok)
    v = kdev.gen_rows_device(w.v_key(0, 0), kt, pos0, n_tok)
    pos = torch.arange(pos0, T, dtype=torch.int32, device="cuda")
    kvq.kv_append(dw.pool, 0, k, v, pos, dw.page_table, row_seq=torch.zeros(n_tok, dtype=torch.int32, device="cuda"))
    qt = kdev.DeviceTable(w.q_table(0), "cuda")
    q = kdev.gen_rows_device(w.q_key(0, 0), qt, 0, n_tok)                 # chunk token i: query step i
    qp = kvq.q_rotate(q) if kvq.rotated_q(w.fmt) else q
    out_f = torch.full((n_tok, w.n_q_heads, 256), float("nan"), dtype=torch.float32, device="cuda")
    out_bf = torch.empty((n_tok, w.n_q_heads, 256), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    step = split or n_tok
    for c0 in range(0, n_tok, step):
        c1 = min(n_tok, c0 + step)
        kvq.paged_prefill_attn(dw.pool, 0, qp[c0:c1].contiguous(), 0, pos0 + c0, dw.page_table, out_bf[c0:c1],
                               out_f[c0:c1], status=status, n_split=n_split)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return dw, pos0, out_f.cpu().numpy(), out_bf.cpu()


def _check_rows(w, dw, pos0, out_f, out_bf, tokens, heads):
    G = w.group
    for g in heads:
        kc, ks, vc, vs = gc.pool_codes(dw, 0, 0, g)
        refs = []
        for i in tokens:
            T = pos0 + i + 1
            q = w.q_row(0, 0, i)[g * G:(g + 1) * G]
            ref = oracle.attn_decode(w.fmt, oracle.q_prepare(w.fmt, q), kc[:T], ks[:T], vc[:T], vs[:T])
            gc.assert_close(out_f[i, g * G:(g + 1) * G], ref, f"{w.name} token {i} head {g}")
            refs.append(ref)
        sel = out_f[np.array(tokens)][:, g * G:(g + 1) * G]
        bsel = out_bf[torch.tensor(tokens)][:, g * G:(g + 1) * G].contiguous()
        gc.assert_bf16_consistent(sel, bsel, np.stack(refs))


@pytest.mark.parametrize("n_tok", [1, 29, 64])
@pytest.mark.parametrize("fmt", FORMATS)
def test_prefill_matches_oracle(fmt, n_tok):
    w = _workload(fmt, 12, 2, 700, f"prefill_{fmt}_{n_tok}")
    dw, pos0, out_f, out_bf = _prefill(w, n_tok)
    # the chunk's codes: one kv_append of all its rows, bit-exact
    for g in range(w.n_kv_heads):
        kc, ks, vc, vs = gc.pool_codes(dw, 0, 0, g)
        kk = np.stack([w.k_rows(0, 0, pos0 + i, 1)[0, g] for i in range(n_tok)])
        vv = np.stack([w.v_rows(0, 0, pos0 + i, 1)[0, g] for i in range(n_tok)])
        okc, oks, ovc, ovs = oracle.append_rows(fmt, kk, vv)
        sl = slice(pos0, pos0 + n_tok)
        assert np.array_equal(kc[sl], okc) and np.array_equal(ks[sl], oks)
        assert np.array_equal(vc[sl], ovc) and np.array_equal(vs[sl], ovs)
    _check_rows(w, dw, pos0, out_f, out_bf, list(range(n_tok)), list(range(w.n_kv_heads)))


@pytest.mark.parametrize("n_tok", [1, 64, 512])
def test_prefill_32k_chunks(n_tok):
    """The 27B shape (24 Q / 4 KV heads, q4_0 + FWHT) with a 32,768-token
    context whose last n_tok tokens are the chunk; sampled rows."""
    w = _workload("q4_0", 24, 4, 32768, f"prefill32k_{n_tok}", order="contiguous", outlier="student_t",
                  q_post=1 / 16, q_outliers=False, n_out=8)
    dw, pos0, out_f, out_bf = _prefill(w, n_tok)
    rng = np.random.default_rng(n_tok)
    toks = sorted(set([0, n_tok - 1, n_tok // 2] + [int(x) for x in rng.integers(0, n_tok, 3)]))
    _check_rows(w, dw, pos0, out_f, out_bf, toks, [0, 3])


@pytest.mark.parametrize("fmt", ["q4_0", "k8v4"])
def test_prefill_in_smaller_chunks_is_bit_identical(fmt):
    """Without a key-range split each row's result depends only on its own
    keys: cutting the chunk into calls of 16 and 40 tokens gives the same bits
    as one call."""
    w = _workload(fmt, 12, 2, 900, f"prefill_split_{fmt}")
    _, _, one, one_bf = _prefill(w, 80, n_split=1)
    for split in (16, 40):
        _, _, parts, parts_bf = _prefill(w, 80, split=split, n_split=1)
        assert np.array_equal(parts.view(np.uint32), one.view(np.uint32))
        assert torch.equal(parts_bf.view(torch.int16), one_bf.view(torch.int16))


@pytest.mark.parametrize("n_split", [1, 2, 3, 8])
@pytest.mark.parametrize("fmt", FORMATS)
def test_prefill_key_split_matches_oracle(fmt, n_split):
    """The key range cut into n_split parts (cuts at multiples of 64 at or below
    pos0), partials merged by the second kernel: every row against the oracle."""
    w = _workload(fmt, 12, 2, 1400, f"prefill_ks_{fmt}_{n_split}")
    dw, pos0, out_f, out_bf = _prefill(w, 37, n_split=n_split)
    _check_rows(w, dw, pos0, out_f, out_bf, list(range(37)), list(range(w.n_kv_heads)))


@pytest.mark.parametrize("fmt", ["q4_0", "nvfp4"])
def test_prefill_from_the_first_token(fmt):
    """A whole prompt as one chunk (pos0 = 0): row i sees keys 0 .. i only, the
    first row a single key."""
    w = _workload(fmt, 12, 2, 300, f"prefill_first_{fmt}")
    dw, pos0, out_f, out_bf = _prefill(w, 300)
    assert pos0 == 0
    _check_rows(w, dw, pos0, out_f, out_bf, [0, 1, 2, 63, 64, 65, 255, 256, 299], list(range(w.n_kv_heads)))


@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (8, 1), (6, 2), (14, 2)])
def test_prefill_group_sizes(Hq, Hkv):
    """Group sizes 1, 8, 3 and 7: the rows r = i G + h of a CTA span token
    boundaries differently for each."""
    w = _workload("q4_0", Hq, Hkv, 900, f"prefill_g_{Hq}_{Hkv}")
    for n_split in (1, 2):
        dw, pos0, out_f, out_bf = _prefill(w, 23, n_split=n_split)
        _check_rows(w, dw, pos0, out_f, out_bf, list(range(23)), list(range(w.n_kv_heads)))


def test_prefill_default_split_at_32k():
    """The split kvq_prefill_split picks for a 512-token chunk at 32,768 (the
    bench's case) against the unsplit kernel and the oracle on sampled rows."""
    w = _workload("q4_0", 24, 4, 32768, "prefill32k_auto", order="contiguous", outlier="student_t",
                  q_post=1 / 16, q_outliers=False, n_out=8)
    n_split, wb = kvq.prefill_split(kvq.make_desc(1, 4, 24, 128, "q4_0"), 32768 - 512, 512)
    assert n_split > 1 and wb > 0
    dw, pos0, out_f, out_bf = _prefill(w, 512)
    _, _, one_f, _ = _prefill(w, 512, n_split=1)
    gc.assert_close(out_f.reshape(-1, 256), one_f.reshape(-1, 256), "split vs unsplit")
    _check_rows(w, dw, pos0, out_f, out_bf, [0, 255, 511], [0, 3])


def test_prefill_rejects_bad_arguments():
    w = _workload("q4_0", 12, 2, 300, "prefill_bad")
    dw = kdev.build_pool(w)
    q = torch.zeros((4, 12, 256), dtype=torch.float32, device="cuda")
    out = torch.empty((4, 12, 256), dtype=torch.bfloat16, device="cuda")
    for pos0 in (-1, dw.page_table.shape[1] * 256 - 3):
        with pytest.raises(kvq.KVQError, match="KVQ_EINVAL"):
            kvq.paged_prefill_attn(dw.pool, 0, q, 0, pos0, dw.page_table, out)
    with pytest.raises(kvq.KVQError, match="KVQ_EINVAL"):
        kvq.paged_prefill_attn(dw.pool, 0, q, 1, 0, dw.page_table, out)           # seq out of range
    for bad in (0, 9):
        with pytest.raises(kvq.KVQError, match="KVQ_EINVAL"):
            kvq.paged_prefill_attn(dw.pool, 0, q, 0, 200, dw.page_table, out, n_split=bad)
    with pytest.raises(kvq.KVQError, match="KVQ_EINVAL"):                           # no cut at or below pos0
        kvq.paged_prefill_attn(dw.pool, 0, q, 0, 100, dw.page_table, out, n_split=3)
    small = torch.empty(16, dtype=torch.float32, device="cuda")
    with pytest.raises(kvq.KVQError, match="KVQ_ESIZE"):
        kvq.paged_prefill_attn(dw.pool, 0, q, 0, 200, dw.page_table, out, n_split=2, workspace=small)
