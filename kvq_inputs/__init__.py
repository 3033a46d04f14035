"""Seeded synthetic inputs for the quantized paged decode-attention path.

This module is shared by the oracle-side tests and by the CUDA-side tests and
benchmark.  It holds NO arithmetic of the method (no rotation, no
quantisation, no attention): only

* a counter-based random generator (SplitMix64 finaliser, Steele, Lea & Flood,
  "Fast splittable pseudorandom number generators", OOPSLA 2014) evaluated at
  explicit counters so that any element can be regenerated on its own;
* an approximately normal variate from the Irwin-Hall sum of twelve 24-bit
  uniforms, computed in integers and converted to fp32 once (round to nearest);
* a Student-t(3) variate built as Z / sqrt(chi2_3 / 3) from four such normals,
  every fp32 operation a single correctly rounded IEEE operation;
* the per-workload recipes (shapes, seeds, outlier channels, page tables).

The same element definition is implemented a second time in CUDA
(``kvq_inputs/csrc/kvq_gen.cu``) so that multi-gigabyte K/V streams can be
produced on the device; the two are bit-identical by construction and a GPU
test checks it.

Element definition (tensor with ``H`` heads of 256 channels, rows = token
positions or decode steps)::

    e        = (row * H + head) * 256 + ch                 # global counter
    u(k, i)  = mix64(k + (i + 1) * GAMMA)                  # 64-bit draw
    N(k, j)  = fp32(sum_{r<6} hi24(u(k,6j+r)) + lo24(u(k,6j+r)) - 6*2^24) * 2^-24
    normal channel :  z = N(key, e)
    t channel      :  s = (N(kt,3e)^2 + N(kt,3e+1)^2) + N(kt,3e+2)^2 ; kt = mix64(key ^ TKEY)
                      z = N(key, e) / sqrt(s / 3)   (0 if the root is 0), clamped to +-4096
    x = (z * mul[head, ch]) * post
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence

import numpy as np

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
MIX1 = 0xBF58476D1CE4E5B9
MIX2 = 0x94D049BB133111EB
TKEY = 0xD1B54A32D192ED03
T_CLAMP = 4096.0
HEAD_DIM = 256
PAGE_TOKENS = 256

# tensor ids used to derive independent streams
TENSOR_Q, TENSOR_K, TENSOR_V, TENSOR_CHANNELS, TENSOR_PAGES = 1, 2, 3, 4, 5

_U64 = np.uint64


def mix64_int(z: int) -> int:
    """SplitMix64 output function on a Python int (mod 2^64)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * MIX1) & MASK64
    z = ((z ^ (z >> 27)) * MIX2) & MASK64
    return z ^ (z >> 31)


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function on a uint64 array (wrap-around arithmetic)."""
    z = z.astype(_U64, copy=True)
    with np.errstate(over="ignore"):
        z ^= z >> _U64(30)
        z *= _U64(MIX1)
        z ^= z >> _U64(27)
        z *= _U64(MIX2)
        z ^= z >> _U64(31)
    return z


def stream_key(seed: int, tensor: int, layer: int = 0, sub: int = 0) -> int:
    """64-bit key of one tensor stream (host only; passed to the device as is)."""
    k = mix64_int(seed * GAMMA + 0x243F6A8885A308D3)
    k = mix64_int(k + ((tensor << 40) | (layer << 20) | sub) * GAMMA)
    return k


def draws(key: int, idx: np.ndarray) -> np.ndarray:
    """u(key, i) for an array of counters i (uint64)."""
    i = idx.astype(_U64, copy=False)
    with np.errstate(over="ignore"):
        z = _U64(key) + (i + _U64(1)) * _U64(GAMMA)
    return mix64(z)


def normal_at(key: int, j: np.ndarray) -> np.ndarray:
    """Irwin-Hall approximate N(0,1) at counters j, as float32."""
    j = np.asarray(j, dtype=_U64)
    acc = np.zeros(j.shape, dtype=np.int64)
    with np.errstate(over="ignore"):
        base = j * _U64(6)
    for r in range(6):
        with np.errstate(over="ignore"):
            u = draws(key, base + _U64(r))
        acc += (u >> _U64(40)).astype(np.int64)
        acc += ((u >> _U64(16)) & _U64(0xFFFFFF)).astype(np.int64)
    acc -= 6 * (1 << 24)
    return acc.astype(np.float32) * np.float32(2.0 ** -24)


def student_t3_at(key: int, e: np.ndarray) -> np.ndarray:
    """Student-t(3) variate at counters e, float32, each op one IEEE fp32 op."""
    e = np.asarray(e, dtype=_U64)
    kt = mix64_int(key ^ TKEY)
    z0 = normal_at(key, e)
    with np.errstate(over="ignore"):
        e3 = e * _U64(3)
    z1 = normal_at(kt, e3)
    z2 = normal_at(kt, e3 + _U64(1))
    z3 = normal_at(kt, e3 + _U64(2))
    s = (z1 * z1 + z2 * z2) + z3 * z3
    s = s / np.float32(3.0)
    r = np.sqrt(s).astype(np.float32)
    out = np.zeros_like(z0)
    np.divide(z0, r, out=out, where=r > 0)
    return np.clip(out, np.float32(-T_CLAMP), np.float32(T_CLAMP)).astype(np.float32)


@dataclasses.dataclass
class ChannelTable:
    """Per-head channel recipe: multiplier and kind (0 normal, 1 Student-t)."""
    mul: np.ndarray   # float32 [H, 256]
    kind: np.ndarray  # uint8   [H, 256]
    post: float       # final scale applied to every element


def gen_rows(key: int, table: ChannelTable, row0: int, n_rows: int) -> np.ndarray:
    """Rows [row0, row0+n_rows) of a [rows, H, 256] float32 tensor."""
    H = table.mul.shape[0]
    rows = np.arange(row0, row0 + n_rows, dtype=np.int64)
    e = (rows[:, None, None] * H + np.arange(H)[None, :, None]) * HEAD_DIM + np.arange(HEAD_DIM)[None, None, :]
    e = e.astype(_U64)
    kind = np.broadcast_to(table.kind[None], e.shape)
    z = normal_at(key, e)
    if np.any(table.kind):
        tmask = kind == 1
        if np.any(tmask):
            z[tmask] = student_t3_at(key, e[tmask])
    x = z * np.broadcast_to(table.mul[None], e.shape).astype(np.float32)
    x = x * np.float32(table.post)
    return x.astype(np.float32)


def pick_channels(seed: int, layer: int, head: int, n: int) -> List[int]:
    """n distinct seeded channel indices in [0, 256)."""
    key = stream_key(seed, TENSOR_CHANNELS, layer, head)
    out: List[int] = []
    i = 0
    while len(out) < n:
        c = int(draws(key, np.array([i], dtype=_U64))[0] % _U64(HEAD_DIM))
        if c not in out:
            out.append(c)
        i += 1
    return out


@dataclasses.dataclass
class Workload:
    """One synthetic workload: shapes, format and value recipe."""
    name: str
    index: int                  # 1-based position in the workload list
    fmt: str                    # 'int8' | 'q4_0' | 'k8v4' | 'fp8' | 'nvfp4'
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    seq_lens: List[int]         # attended length per sequence (includes the appended token)
    page_order: str             # 'contiguous' | 'permuted'
    n_outlier: int              # outlier channels per (layer, kv head)
    outlier_kind: str           # 'mul20' | 'mul10' | 'student_t'
    q_post: float               # scale on Q (1/16 where the recipe says N(0,1)/16)
    q_outliers: bool            # Q heads share their group's outlier channels
    description: str = ""

    @property
    def seed(self) -> int:
        return 1000 + self.index

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def batch(self) -> int:
        return len(self.seq_lens)

    def max_pages(self) -> int:
        return max((t + PAGE_TOKENS - 1) // PAGE_TOKENS for t in self.seq_lens)

    def pages_needed(self) -> int:
        return sum((t + PAGE_TOKENS - 1) // PAGE_TOKENS for t in self.seq_lens)

    # -- value recipes -------------------------------------------------------
    def kv_table(self, layer: int) -> ChannelTable:
        mul = np.ones((self.n_kv_heads, HEAD_DIM), np.float32)
        kind = np.zeros((self.n_kv_heads, HEAD_DIM), np.uint8)
        for g in range(self.n_kv_heads):
            for c in pick_channels(self.seed, layer, g, self.n_outlier):
                if self.outlier_kind == "student_t":
                    kind[g, c] = 1
                elif self.outlier_kind == "mul20":
                    mul[g, c] = 20.0
                elif self.outlier_kind == "mul10":
                    mul[g, c] = 10.0
                else:
                    raise ValueError(self.outlier_kind)
        return ChannelTable(mul, kind, 1.0)

    def q_table(self, layer: int) -> ChannelTable:
        mul = np.ones((self.n_q_heads, HEAD_DIM), np.float32)
        kind = np.zeros((self.n_q_heads, HEAD_DIM), np.uint8)
        if self.q_outliers:
            kv = self.kv_table(layer)
            for h in range(self.n_q_heads):
                mul[h] = kv.mul[h // self.group]
        return ChannelTable(mul, kind, self.q_post)

    def k_key(self, layer: int, seq: int) -> int:
        return stream_key(self.seed, TENSOR_K, layer, seq)

    def v_key(self, layer: int, seq: int) -> int:
        return stream_key(self.seed, TENSOR_V, layer, seq)

    def q_key(self, layer: int, seq: int) -> int:
        return stream_key(self.seed, TENSOR_Q, layer, seq)

    def k_rows(self, layer: int, seq: int, row0: int, n: int) -> np.ndarray:
        return gen_rows(self.k_key(layer, seq), self.kv_table(layer), row0, n)

    def v_rows(self, layer: int, seq: int, row0: int, n: int) -> np.ndarray:
        return gen_rows(self.v_key(layer, seq), self.kv_table(layer), row0, n)

    def q_row(self, layer: int, seq: int, step: int = 0) -> np.ndarray:
        return gen_rows(self.q_key(layer, seq), self.q_table(layer), step, 1)[0]

    # -- page tables ---------------------------------------------------------
    def page_table(self, n_slots: Optional[int] = None) -> np.ndarray:
        """int32 [B, max_pages]; unused entries are -1.

        'contiguous': sequence b owns consecutive slots after the previous one.
        'permuted'  : the same slot set is shuffled by a seeded Fisher-Yates.
        """
        need = self.pages_needed()
        n_slots = need if n_slots is None else n_slots
        slots = np.arange(n_slots, dtype=np.int64)
        if self.page_order == "permuted":
            key = stream_key(self.seed, TENSOR_PAGES)
            u = draws(key, np.arange(n_slots, dtype=_U64))
            for i in range(n_slots - 1, 0, -1):
                j = int(u[i] % _U64(i + 1))
                slots[i], slots[j] = slots[j], slots[i]
        pt = np.full((self.batch, self.max_pages()), -1, np.int32)
        k = 0
        for b, t in enumerate(self.seq_lens):
            n = (t + PAGE_TOKENS - 1) // PAGE_TOKENS
            pt[b, :n] = slots[k:k + n]
            k += n
        return pt


def _w(**kw) -> Workload:
    return Workload(**kw)


# The five workloads.  Shapes and value distributions follow the decode-attention
# workloads the pages describe (27B: 24 Q heads, 4 KV heads, head_dim 256, 16
# full-attention layers, 262,144-token window; the Flash-Next-like shape with two
# KV heads; the three Strata KV formats).  No public dataset is involved.
WORKLOADS: Dict[str, Workload] = {
    "tiny_q4_0_1k": _w(name="tiny_q4_0_1k", index=1, fmt="q4_0", n_layers=1, n_q_heads=4, n_kv_heads=1,
                       seq_lens=[1024], page_order="contiguous", n_outlier=4, outlier_kind="mul20",
                       q_post=1.0, q_outliers=True,
                       description="1 layer, Hq=4, Hkv=1, 1,024 tokens in 4 pages, q4_0 + FWHT"),
    "qwen27b_int8_32k": _w(name="qwen27b_int8_32k", index=2, fmt="int8", n_layers=16, n_q_heads=24, n_kv_heads=4,
                           seq_lens=[32768], page_order="contiguous", n_outlier=5, outlier_kind="mul10",
                           q_post=1.0 / 16, q_outliers=False,
                           description="27B full-attention shape, int8/64, 32,768 tokens, contiguous pages"),
    "flashnext_k8v4_128k": _w(name="flashnext_k8v4_128k", index=3, fmt="k8v4", n_layers=16, n_q_heads=16,
                              n_kv_heads=2, seq_lens=[131072], page_order="permuted", n_outlier=4,
                              outlier_kind="mul20", q_post=1.0, q_outliers=True,
                              description="Flash-Next-like shape, k8v4, 131,072 tokens, permuted pages"),
    "qwen27b_q4_0_262k": _w(name="qwen27b_q4_0_262k", index=4, fmt="q4_0", n_layers=16, n_q_heads=24,
                            n_kv_heads=4, seq_lens=[262144], page_order="contiguous", n_outlier=8,
                            outlier_kind="student_t", q_post=1.0 / 16, q_outliers=False,
                            description="27B shape at the full 262,144 window, q4_0 + FWHT on Q/K/V"),
    "ragged4_q4_0": _w(name="ragged4_q4_0", index=5, fmt="q4_0", n_layers=16, n_q_heads=24, n_kv_heads=4,
                       seq_lens=[8192, 65536, 200000, 262144], page_order="permuted", n_outlier=8,
                       outlier_kind="student_t", q_post=1.0 / 16, q_outliers=False,
                       description="4 ragged sequences, shared pool, random page-to-slot map, q4_0"),
    "ragged4_k8v4": _w(name="ragged4_k8v4", index=5, fmt="k8v4", n_layers=16, n_q_heads=24, n_kv_heads=4,
                       seq_lens=[8192, 65536, 200000, 262144], page_order="permuted", n_outlier=8,
                       outlier_kind="student_t", q_post=1.0 / 16, q_outliers=False,
                       description="4 ragged sequences, shared pool, random page-to-slot map, k8v4"),
    # the two floating-point formats the smzdm roundup measures (FP8 516 B and
    # NVFP4 288 B per position) on the same 27B full-window shape
    "qwen27b_fp8_262k": _w(name="qwen27b_fp8_262k", index=6, fmt="fp8", n_layers=16, n_q_heads=24, n_kv_heads=4,
                           seq_lens=[262144], page_order="contiguous", n_outlier=8, outlier_kind="student_t",
                           q_post=1.0 / 16, q_outliers=False,
                           description="27B shape at the full 262,144 window, fp8 E4M3 KV, one fp16 scale per vector"),
    "qwen27b_nvfp4_262k": _w(name="qwen27b_nvfp4_262k", index=7, fmt="nvfp4", n_layers=16, n_q_heads=24,
                             n_kv_heads=4, seq_lens=[262144], page_order="contiguous", n_outlier=8,
                             outlier_kind="student_t", q_post=1.0 / 16, q_outliers=False,
                             description="27B shape at the full 262,144 window, nvfp4 KV (E2M1 + E4M3 per 16)"),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def scaled(w: Workload, seq_lens: Sequence[int], n_layers: Optional[int] = None, name: Optional[str] = None) -> Workload:
    """Same recipe (format, heads, value distribution, seed) at other lengths."""
    return dataclasses.replace(w, seq_lens=list(seq_lens), n_layers=n_layers or w.n_layers,
                               name=name or f"{w.name}@{'+'.join(map(str, seq_lens))}")
