"""Oracle for the masked attention forward: TEST INFRASTRUCTURE ONLY.

A plain, slow, fp64 CPU statement of what the library computes, written
from the definitions on the pages, sharing no code with the CUDA path.
Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import it; the library itself never does.

Contents
  masks.py      dense boolean mask per descriptor kind, bit unpacking,
                128x128 tile classes and unmasked-pair counts from the dense mask
  attention.py  O = softmax(scale * Q K^T + mask) V and the row log-sum-exp, fp64
  backward.py   dQ, dK, dV of that forward for a given dO (chain rule through the row
                softmax), fp64
  fp8.py        e4m3 byte decoding (inputs of the fp8 forward)

Every function is pinned by the CPU tests (tests/test_oracle_*.py) to facts
the pages or the mathematics fix: the pages' worked chunk-causal example,
the mask equivalences the pages state, closed forms, a brute-force loop on
tiny inputs and the library softmax on unmasked rows.
"""
from .masks import (dense_mask_rows, dense_mask, unpack_rows, tile_classes, unmasked_pairs,
                    CLASS_EMPTY, CLASS_FULL, CLASS_PARTIAL)
from .attention import attention_one_head, masked_attention, sampled_attention
from .backward import attention_backward_one_head, masked_attention_backward, sampled_backward
from .fp8 import decode_e4m3

__all__ = ["dense_mask_rows", "dense_mask", "unpack_rows", "tile_classes", "unmasked_pairs",
           "CLASS_EMPTY", "CLASS_FULL", "CLASS_PARTIAL",
           "attention_one_head", "masked_attention", "sampled_attention",
           "attention_backward_one_head", "masked_attention_backward", "sampled_backward", "decode_e4m3"]
