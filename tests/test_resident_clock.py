"""Host-side tests of the residency table and CLOCK (second chance) policy of
the host-resident KV cache ([Strata] "KV 从显存搬进内存之后发生了什么": KV kept in
host memory, the GPU holds the pages attention reads, CLOCK chooses what to
evict).  kvq_resident_map is host-only, so the pools here are descriptors over
addresses that are never dereferenced.

The policy is checked against a plain model written here from the textbook
CLOCK algorithm (a circular list of frames with one reference bit each; on a
miss the hand clears set bits and stops at the first clear one), with the one
addition a batched cache needs: the pages one call reads are all resident at
once, so they are skipped by the hand while that call is planned."""
import itertools

import numpy as np
import pytest

import quantized_kv_cache_17_b200 as kvq

PAGE = 256


@pytest.fixture(scope="module", autouse=True)
def built():
    from quantized_kv_cache_17_b200 import build
    build.build()


def make(n_layers, n_host_pages, n_slots, fmt="q4_0"):
    h = kvq.make_desc(n_layers, 2, 16, n_host_pages, fmt)
    c = kvq.make_desc(1, 2, 16, n_slots, fmt)
    return kvq.ResidentCache(None, host_desc=h, cache_desc=c, host_base=0x100000, cache_base=0x200000)


class ClockModel:
    """Frames 0..n-1, a hand, one reference bit per frame."""

    def __init__(self, n_slots):
        self.frame = [None] * n_slots
        self.bit = [0] * n_slots
        self.hand = 0
        self.where = {}
        self.hits = self.misses = self.evictions = 0

    def call(self, refs):
        """refs: the (layer, page) keys one call reads, in reference order.
        Returns (slot of each ref, [(page, slot) loaded])."""
        batch = set(refs)
        busy = {self.where[k] for k in batch if k in self.where}
        for f in busy:
            self.bit[f] = 1
        loads, out = [], []
        for k in refs:
            if k in self.where:
                self.hits += 1
            else:
                self.misses += 1
                while True:
                    f = self.hand
                    self.hand = (self.hand + 1) % len(self.frame)
                    if f in busy:
                        continue
                    if self.bit[f]:
                        self.bit[f] = 0
                        continue
                    break
                if self.frame[f] is not None:
                    del self.where[self.frame[f]]
                    self.evictions += 1
                self.frame[f], self.bit[f] = k, 1
                self.where[k] = f
                busy.add(f)
                loads.append((k[1], f))
            out.append(self.where[k])
        return out, loads


def run_call(rc, layer, seqs, max_pages=None):
    """seqs: list of host-page lists; each sequence reads all its pages."""
    max_pages = max_pages or max(len(s) for s in seqs)
    hpt = np.full((len(seqs), max_pages), -7, np.int32)
    lens = []
    for b, s in enumerate(seqs):
        hpt[b, :len(s)] = s
        lens.append(len(s) * PAGE - (b % 3) * 40 if s else 0)   # ragged last pages
    cpt, loads = rc.map(layer, hpt, lens)
    for b, s in enumerate(seqs):
        assert (cpt[b, len(s):] == -1).all()
    return [list(cpt[b, :len(s)]) for b, s in enumerate(seqs)], [tuple(x) for x in loads]


def test_textbook_trace_second_chance():
    """Three frames, pages 1 2 3 4 2 5 one per call, worked by hand from the
    definition: 4 clears all three bits and replaces 1; 2 hits and sets its bit;
    5 passes 2 (clearing it) and replaces 3 -- where FIFO would replace 2."""
    rc = make(1, 8, 3)
    got = [run_call(rc, 0, [[p]])[1] for p in (1, 2, 3, 4, 2, 5)]
    assert got == [[(1, 0)], [(2, 1)], [(3, 2)], [(4, 0)], [], [(5, 2)]]
    assert [rc.slot_of(0, p) for p in range(8)] == [-1, -1, 1, -1, 0, 2, -1, -1]
    assert rc.stats() == (1, 5, 2)


def test_loop_larger_than_cache_always_misses():
    """A cyclic scan over n+1 pages with n frames misses on every reference
    (CLOCK degenerates to FIFO on a loop), and a scan over n pages hits on
    every reference after the first pass."""
    rc = make(1, 16, 4)
    for _ in range(3):
        for p in range(5):
            assert len(run_call(rc, 0, [[p]])[1]) == 1
    assert rc.stats() == (0, 15, 11)
    rc = make(1, 16, 4)
    for it in range(3):
        for p in range(4):
            assert len(run_call(rc, 0, [[p]])[1]) == (1 if it == 0 else 0)


@pytest.mark.parametrize("seed", range(6))
def test_matches_the_model_on_random_traces(seed):
    rng = np.random.default_rng(seed)
    n_layers, n_host, n_slots = 3, 40, int(rng.integers(8, 30))
    rc, model = make(n_layers, n_host, n_slots), ClockModel(n_slots)
    hot = rng.choice(n_host, 6, replace=False)
    for call in range(120):
        layer = int(rng.integers(n_layers))
        seqs = []
        budget = n_slots
        for _ in range(int(rng.integers(1, 4))):
            k = int(rng.integers(1, 6))
            pages = list(rng.choice(hot, 2, replace=False)) if rng.random() < 0.5 else []
            pages += list(rng.choice(n_host, k, replace=False))
            if len(set(itertools.chain(pages, *seqs))) > budget:
                break
            seqs.append([int(p) for p in pages])
        if not seqs:
            continue
        slots, loads = run_call(rc, layer, seqs)
        refs = [(layer, p) for s in seqs for p in s]
        want_slots, want_loads = model.call(refs)
        assert [x for s in slots for x in s] == want_slots
        assert loads == want_loads
        # table and slots agree, no slot holds two pages
        for l in range(n_layers):
            for p in range(n_host):
                assert rc.slot_of(l, p) == model.where.get((l, p), -1)
    assert rc.stats() == (model.hits, model.misses, model.evictions)


def test_batch_pages_are_never_evicted_by_their_own_call():
    """A call that needs every slot, after the cache is full of other pages:
    every page loads, none is loaded twice, all end in distinct slots."""
    rc = make(2, 32, 8)
    run_call(rc, 0, [list(range(8))])
    slots, loads = run_call(rc, 1, [[3, 1, 4], [1, 5, 9, 2, 6]])      # page 1 read by both sequences
    assert len(loads) == 7 and len({s for _, s in loads}) == 7
    assert slots[0][1] == slots[1][0]
    # a call mixing resident and missing pages keeps the resident ones
    slots2, loads2 = run_call(rc, 1, [[3, 1, 4, 20, 21]])
    assert [p for p, _ in loads2] == [20, 21]
    assert slots2[0][:3] == slots[0]


def test_layers_are_separate_keys():
    rc = make(3, 8, 6)
    for l in range(3):
        _, loads = run_call(rc, l, [[0, 1]])
        assert [p for p, _ in loads] == [0, 1]
    assert {rc.slot_of(l, p) for l in range(3) for p in (0, 1)} == set(range(6))


def test_errors_leave_the_state_unchanged():
    rc = make(2, 16, 4)
    run_call(rc, 0, [[0, 1, 2]])
    before = rc._state.copy()
    L = kvq.lib()
    n = np.zeros(1, np.int32)
    import ctypes
    nl = ctypes.c_int()
    cpt = np.zeros((1, 8), np.int32)
    loads = np.zeros((8, 2), np.int32)

    def m(layer, pages, T, cap=8, ld=loads):
        hpt = np.full((1, 8), 0, np.int32)
        hpt[0, :len(pages)] = pages
        return L.kvq_resident_map(rc.state, layer, hpt.ctypes.data, 1, 8, np.array([T], np.int32).ctypes.data,
                                  cpt.ctypes.data, None if ld is None else ld.ctypes.data, cap, ctypes.byref(nl))

    assert m(0, [0, 1, 2, 3, 4], 5 * PAGE) == -5                 # five pages, four slots
    assert m(0, [0, 16], 2 * PAGE) == -1                         # host page out of range
    assert m(0, [0, -1], 2 * PAGE) == -1
    assert m(2, [0], PAGE) == -1                                 # no such layer
    assert m(0, [0], 8 * PAGE + 1) == -1                         # longer than the table row
    assert m(0, [0], -1) == -1
    assert m(1, [5, 6], 2 * PAGE, cap=1) == -5 and nl.value == 2  # list too short: the count comes back
    assert m(1, [5, 6], 2 * PAGE, cap=0, ld=None) == -5 and nl.value == 2
    assert m(1, [5], PAGE, cap=3, ld=None) == -1                 # capacity without a list
    assert np.array_equal(rc._state, before)
    assert m(0, [0, 1], 2 * PAGE, cap=0, ld=None) == 0 and nl.value == 0   # all resident: no list needed
    assert L.kvq_resident_load(rc.state, 0, None, 0, None) == 0
    assert L.kvq_resident_load(rc.state, 0, np.array([[16, 0]], np.int32).ctypes.data, 1, None) == -1
    assert L.kvq_resident_load(rc.state, 0, np.array([[0, 4]], np.int32).ctypes.data, 1, None) == -1
    assert L.kvq_resident_load(rc.state, 5, None, 0, None) == -1
    assert L.kvq_resident_load(None, 0, None, 0, None) == -1


def test_init_validation():
    L = kvq.lib()
    h = kvq.make_desc(2, 2, 16, 16, "q4_0")
    n = L.kvq_resident_state_bytes(2, 16, 4)
    assert n > 0 and L.kvq_resident_state_bytes(0, 16, 4) == 0
    st = np.zeros(n // 8 + 1, np.uint64)
    import ctypes

    def init(cdesc, hb=0x1000, cb=0x2000, nbytes=n):
        return L.kvq_resident_init(st.ctypes.data, nbytes, ctypes.byref(kvq.Pool(hb, h)),
                                   ctypes.byref(kvq.Pool(cb, cdesc)))

    assert init(kvq.make_desc(1, 2, 16, 4, "q4_0")) == 0
    assert init(kvq.make_desc(1, 2, 16, 4, "int8")) == -1        # format differs
    assert init(kvq.make_desc(2, 2, 16, 4, "q4_0")) == -1        # cache must be one layer
    assert init(kvq.make_desc(1, 1, 8, 4, "q4_0")) == -1         # heads differ
    assert init(kvq.make_desc(1, 2, 16, 4, "q4_0"), nbytes=n - 1) == -5
    assert init(kvq.make_desc(1, 2, 16, 4, "q4_0"), hb=0x1008) == -3
    assert init(kvq.make_desc(1, 2, 16, 4, "q4_0"), hb=0) == -1
