"""Test-side decoder of the pool layout documented in include/kvq.h and the
kernel sources: turns the bytes of a page block back into one code per
(token, dim) and one fp16 scale per (token, block).  Written from the layout
description only; it shares no code with the CUDA path or the oracle.
"""
from __future__ import annotations

import functools

import numpy as np

Q4, I8, F8, F4 = "q4", "i8", "f8", "f4"
PARTS = {"int8": (I8, I8), "q4_0": (Q4, Q4), "k8v4": (I8, Q4), "fp8": (F8, F8), "nvfp4": (F4, F4)}
CODE_BYTES = {Q4: 1024, I8: 2048, F8: 2048, F4: 1024}
SCALE_BYTES = {Q4: 128, I8: 64, F8: 16, F4: 128}
N_SCALES = {Q4: 8, I8: 4, F8: 1, F4: 16}


def tile_sections(fmt):
    kp, vp = PARTS[fmt]
    kc = 0
    ks = kc + CODE_BYTES[kp]
    vc = ks + SCALE_BYTES[kp]
    vs = vc + CODE_BYTES[vp]
    return kc, ks, vc, vs, vs + SCALE_BYTES[vp]


@functools.lru_cache(None)
def code_map(part: str, side: str):
    """(byte offset, bit shift) of the code of (token r in tile, dim d): arrays [8, 256]."""
    if part == F8:                       # E4M3 bytes where int8 bytes would be
        return code_map(I8, side)
    if part == F4 and side == "v":       # E2M1 nibbles where q4_0 nibbles would be
        return code_map(Q4, side)
    off = np.full((8, 256), -1, np.int64)
    sh = np.zeros((8, 256), np.int64)
    if part == F4 and side == "k":
        # word (r, b, j) at the q4_0 place; byte q: dims 32b + 8q + 2j (low
        # nibble) and + 1 (high nibble)
        for r in range(8):
            for b in range(8):
                for j in range(4):
                    for q in range(4):
                        for h in range(2):
                            d = 32 * b + 8 * q + 2 * j + h
                            off[r, d] = (b >> 2) * 512 + (r * 4 + j) * 16 + (b & 3) * 4 + q
                            sh[r, d] = 4 * h
    elif part == Q4 and side == "k":
        for r in range(8):
            for b in range(8):
                for j in range(4):
                    for n in range(8):
                        d = 32 * b + 8 * (n & 3) + (n >> 2) + 2 * j
                        off[r, d] = (b >> 2) * 512 + (r * 4 + j) * 16 + (b & 3) * 4 + (n >> 1)
                        sh[r, d] = 4 * (n & 1)
    elif part == Q4 and side == "v":
        for p in range(4):
            for b in range(8):
                for g in range(8):
                    for n in range(8):
                        r = 2 * p + (n >> 2)
                        d = 32 * b + g + 8 * (n & 3)
                        off[r, d] = (b >> 2) * 512 + (g * 4 + p) * 16 + (b & 3) * 4 + (n >> 1)
                        sh[r, d] = 4 * (n & 1)
    elif part == I8 and side == "k":
        for r in range(8):
            for s in range(16):
                for j in range(4):
                    for n, dd in enumerate((0, 1, 8, 9)):
                        d = 16 * s + 2 * j + dd
                        off[r, d] = (s >> 2) * 512 + (r * 4 + j) * 16 + (s & 3) * 4 + n
    elif part == I8 and side == "v":
        for p in range(4):
            for m in range(16):
                for g in range(8):
                    for n in range(4):
                        r = 2 * p + (n & 1)
                        d = 16 * m + g + 8 * (n >> 1)
                        off[r, d] = (m >> 2) * 512 + (g * 4 + p) * 16 + (m & 3) * 4 + n
    else:
        raise ValueError((part, side))
    assert (off >= 0).all()
    return off, sh


@functools.lru_cache(None)
def scale_map(part: str):
    """byte offset of the scale of (token r, block q): [8, n_scales] (fp16 for
    q4 / i8 / f8, one E4M3 byte for f4)."""
    ns = N_SCALES[part]
    off = np.zeros((8, ns), np.int64)
    for r in range(8):
        for q in range(ns):
            if part == F8:
                off[r, q] = 2 * r
            elif part == F4:
                off[r, q] = (r >> 1) * 32 + q * 2 + (r & 1)
            else:
                stride = 32 if part == Q4 else 16
                off[r, q] = (r >> 1) * stride + q * 4 + (r & 1) * 2
    return off


def _decode_codes(sec: np.ndarray, part: str, side: str) -> np.ndarray:
    """sec: uint8 [n_tiles, code_bytes] -> codes [n_tiles*8, 256] (uint8; int8 as bytes)."""
    off, sh = code_map(part, side)
    raw = sec[:, off]                              # [n_tiles, 8, 256]
    if part in (Q4, F4):
        raw = (raw >> sh[None]) & 0xF
    return raw.reshape(-1, 256).astype(np.uint8)


def _decode_scales(sec: np.ndarray, part: str) -> np.ndarray:
    off = scale_map(part)
    lo = sec[:, off].astype(np.uint16)
    if part == F4:
        return lo.reshape(-1, N_SCALES[part])
    hi = sec[:, off + 1].astype(np.uint16)
    return (lo | (hi << 8)).reshape(-1, N_SCALES[part])


def decode_page_blocks(fmt: str, blocks: np.ndarray):
    """blocks: uint8 [n_blocks, page_bytes] (each a (layer, slot, kv head) block).

    Returns kc [n*256, 256] uint8, ks [n*256, nk] uint16, vc, vs, in token order.
    """
    kp, vp = PARTS[fmt]
    kc, ks, vc, vs, tb = tile_sections(fmt)
    tiles = blocks.reshape(-1, tb)
    return (_decode_codes(tiles[:, kc:ks], kp, "k"), _decode_scales(tiles[:, ks:vc], kp),
            _decode_codes(tiles[:, vc:vs], vp, "v"), _decode_scales(tiles[:, vs:tb], vp))


def page_block_offset(layout, layer: int, slot: int, head: int) -> int:
    return layer * layout.layer_stride + slot * layout.slot_stride + head * layout.head_stride


def gather_sequence(fmt: str, pool_u8, layout, layer: int, head: int, page_row, T: int):
    """Codes/scales of tokens [0, T) of one sequence from a torch uint8 pool (any device)."""
    import torch
    n_pages = (T + 255) // 256
    pb = layout.page_bytes
    parts = [pool_u8[o:o + pb] for o in (page_block_offset(layout, layer, int(page_row[p]), head)
                                         for p in range(n_pages))]
    blocks = torch.stack(parts).cpu().numpy()
    kc, ks, vc, vs = decode_page_blocks(fmt, blocks)
    return kc[:T], ks[:T], vc[:T], vs[:T]
