"""Mask descriptors for attn_plan(): one constructor per kind of ``attn_mask_desc_t``.

Every constructor returns a ``Mask``; attn_plan() and attn_classify_host() marshal it
field by field into the C descriptor (include/attn.h). Coordinates are sequence-local,
ranges half-open, and one mask is shared by every head of a sequence.

    causal()                                  key j visible to query i iff j <= pos(i),
                                              pos(i) = i + L_k - L_q (queries are the last
                                              L_q positions of the keys)
    sliding_window(w)                         causal and pos(i) - j < w ("feat: add Gemma2
                                              sliding-window (local/global) attention")
    prefix_lm(p | [p_b])                      j < p or causal ("[Attention] feat: support
                                              PrefixLM")
    chunk_causal(q0, q1, k0, k1, cs)          causal before q0, then chunks of cs rows that see
                                              every key up to their chunk's end ("Feature
                                              request: chunk-causal mask type for Flex Flash
                                              Attention", Desired representation)
    ranges([[(q0, q1, k0, k1, type, cs)]])    union of typed ranges per sequence (same page,
                                              Proposed API); type FULL, CAUSAL, INV_CAUSAL,
                                              BI_CAUSAL or CHUNK_CAUSAL
    custom(bits, word_offsets)                bit-packed rows ("Custom mask slows down
                                              attention."); pack_custom() packs booleans
    block_sparse(bq, bk, row_ptr, col_idx)    listed (bq x bk) blocks visible (same page, the
                                              sparse API)

pack_custom() is input preparation only (the layout the planner reads); the classification
of tiles and all of the attention arithmetic run on the GPU.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence, Tuple

import numpy as np

RANGE_FULL = 0
RANGE_CAUSAL = 1
RANGE_INV_CAUSAL = 2
RANGE_BI_CAUSAL = 3
RANGE_CHUNK_CAUSAL = 4

Range = Tuple[int, int, int, int, int, int]   # q_start, q_end, k_start, k_end, type, chunk_size


@dataclasses.dataclass
class Mask:
    """Fields of attn_mask_desc_t; only those of ``kind`` are read."""
    kind: str
    window: int = 0
    prefix_len: int = 0
    prefix_lens: Optional[np.ndarray] = None
    chunk: Optional[Range] = None
    ranges: Optional[List[List[Range]]] = None
    bits: Optional[object] = None              # numpy uint32 words (host) or a device int32/uint32 tensor
    word_offsets: Optional[np.ndarray] = None
    block_q: int = 0
    block_k: int = 0
    bsr_row_ptr: Optional[np.ndarray] = None
    bsr_col_idx: Optional[np.ndarray] = None


def full() -> Mask:
    return Mask("FULL")


def causal() -> Mask:
    return Mask("CAUSAL")


def sliding_window(window: int) -> Mask:
    if window < 1:
        raise ValueError("window must be >= 1")
    return Mask("SLIDING_WINDOW", window=int(window))


def prefix_lm(prefix_len) -> Mask:
    """prefix_len: one length for every sequence, or a sequence of per-sequence lengths."""
    if np.ndim(prefix_len) == 0:
        if prefix_len < 0:
            raise ValueError("prefix_len must be >= 0")
        return Mask("PREFIX_LM", prefix_len=int(prefix_len))
    p = np.asarray(prefix_len, dtype=np.int32)
    if (p < 0).any():
        raise ValueError("prefix lengths must be >= 0")
    return Mask("PREFIX_LM", prefix_lens=p)


def chunk_causal(q_start: int, q_end: int, k_start: int, k_end: int, chunk_size: int) -> Mask:
    if chunk_size < 1:
        raise ValueError("chunk_size must be >= 1")
    return Mask("CHUNK_CAUSAL", chunk=(int(q_start), int(q_end), int(k_start), int(k_end),
                                       RANGE_CHUNK_CAUSAL, int(chunk_size)))


def ranges(per_sequence: Sequence[Sequence[Range]]) -> Mask:
    """per_sequence[b]: the ranges of sequence b as (q_start, q_end, k_start, k_end, type,
    chunk_size) tuples; chunk_size is read for RANGE_CHUNK_CAUSAL only."""
    rs = [[tuple(int(x) for x in r) for r in per] for per in per_sequence]
    for per in rs:
        for r in per:
            if len(r) != 6:
                raise ValueError("a range has six fields")
    return Mask("RANGES", ranges=rs)


def pack_custom(dense_per_sequence: Sequence[np.ndarray]) -> Tuple[np.ndarray, np.ndarray]:
    """Boolean [L_q, L_k] arrays, one per sequence -> (uint32 words, int64 word offsets [B+1])
    in the CUSTOM layout: row-major [L_q][ceil(L_k / 32)] words per sequence, key j of row i
    in bit j % 32 of word i * W + j // 32, least significant bit first."""
    words, offsets = [], [0]
    for dense in dense_per_sequence:
        dense = np.asarray(dense, dtype=bool)
        if dense.ndim != 2:
            raise ValueError("each sequence's mask is [L_q, L_k]")
        lq, lk = dense.shape
        w = (lk + 31) // 32
        # 8 keys per byte, lowest key in the least significant bit; 4 bytes little-endian
        # per word, so key j lands in bit j % 32 of word j // 32
        by = np.packbits(dense, axis=1, bitorder="little")
        padded = np.zeros((lq, w * 4), dtype=np.uint8)
        padded[:, :by.shape[1]] = by
        words.append(padded.view("<u4").reshape(-1).astype(np.uint32))
        offsets.append(offsets[-1] + lq * w)
    flat = np.concatenate(words) if words else np.zeros(0, np.uint32)
    return flat, np.asarray(offsets, dtype=np.int64)


def custom(bits, word_offsets) -> Mask:
    """bits: packed words (numpy uint32 on the host, or a device tensor of 32-bit words);
    word_offsets: int64 [B+1], sequence b's words start at word_offsets[b]."""
    off = np.asarray(word_offsets, dtype=np.int64)
    if off.ndim != 1 or (off.size and (np.diff(off) < 0).any()):
        raise ValueError("word_offsets must be a non-decreasing [B+1] array")
    return Mask("CUSTOM", bits=bits, word_offsets=off)


def block_sparse(block_q: int, block_k: int, bsr_row_ptr, bsr_col_idx) -> Mask:
    """BSR over the block rows of all sequences in order (sequence b has ceil(L_q / block_q)
    block rows); column indices are sequence-local block columns."""
    if block_q < 1 or block_k < 1:
        raise ValueError("block sizes must be >= 1")
    return Mask("BLOCK_SPARSE", block_q=int(block_q), block_k=int(block_k),
                bsr_row_ptr=np.asarray(bsr_row_ptr, dtype=np.int32),
                bsr_col_idx=np.asarray(bsr_col_idx, dtype=np.int32))
