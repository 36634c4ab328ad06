"""CPU tests of the package's mask constructors (masked_flash_attention_attn_b200.mask).

A Mask built by a constructor must give, through the host planner, the same 128 x 128
tile classes and unmasked pair counts as the oracle derives from the same parameters;
pack_custom() must produce the CUSTOM word layout the oracle unpacks.
"""
import numpy as np
import pytest

import workloads as W
from oracle import masks as OM
from masked_flash_attention_attn_b200 import mask as MK


def _lengths(cq, ck):
    return [(int(cq[b + 1] - cq[b]), int(ck[b + 1] - ck[b])) for b in range(len(cq) - 1)]


def _from_spec(spec):
    """The constructor call a user would write for the parameters of an oracle spec."""
    if spec.kind == "FULL":
        return MK.full()
    if spec.kind == "CAUSAL":
        return MK.causal()
    if spec.kind == "SLIDING_WINDOW":
        return MK.sliding_window(spec.window)
    if spec.kind == "PREFIX_LM":
        return MK.prefix_lm(spec.prefix_lens if spec.prefix_lens is not None else spec.prefix_len)
    if spec.kind == "CHUNK_CAUSAL":
        q0, q1, k0, k1, _, cs = spec.chunk
        return MK.chunk_causal(q0, q1, k0, k1, cs)
    if spec.kind == "RANGES":
        return MK.ranges(spec.ranges)
    if spec.kind == "BLOCK_SPARSE":
        return MK.block_sparse(spec.block_q, spec.block_k, spec.bsr_row_ptr, spec.bsr_col_idx)
    raise ValueError(spec.kind)


@pytest.mark.parametrize("kind", ["FULL", "CAUSAL", "SLIDING_WINDOW", "PREFIX_LM", "CHUNK_CAUSAL", "RANGES",
                                  "BLOCK_SPARSE"])
@pytest.mark.parametrize("seed", range(3))
def test_constructors_classify_like_the_oracle(attn_lib, kind, seed):
    rng = np.random.default_rng(1000 + seed)
    lq = rng.integers(1, 600, size=3)
    lk = lq.copy() if seed % 2 == 0 else np.maximum(lq, rng.integers(1, 600, size=3))
    spec = W.random_mask_spec(rng, kind, lq, lk)
    cq, ck = W.cu_from_lengths(lq), W.cu_from_lengths(lk)
    cls, pairs = attn_lib.attn_classify_host(hq=4, hkv=2, head_dim=64, cu_seqlens_q=cq, cu_seqlens_k=ck,
                                             mask=_from_spec(spec))
    assert np.array_equal(cls, OM.tile_classes(spec, _lengths(cq, ck)))
    assert pairs == OM.unmasked_pairs(spec, _lengths(cq, ck))


def test_range_type_codes_match_the_oracle():
    assert (MK.RANGE_FULL, MK.RANGE_CAUSAL, MK.RANGE_INV_CAUSAL, MK.RANGE_BI_CAUSAL, MK.RANGE_CHUNK_CAUSAL) == \
        (OM.R_FULL, OM.R_CAUSAL, OM.R_INV_CAUSAL, OM.R_BI_CAUSAL, OM.R_CHUNK)


@pytest.mark.parametrize("shape", [(1, 1), (3, 31), (5, 32), (4, 33), (130, 257), (0, 7), (2, 0)])
def test_pack_custom_layout(shape):
    rng = np.random.default_rng(shape[0] * 1000 + shape[1])
    a = rng.random(shape) < 0.5
    b = rng.random((shape[0] + 1, shape[1] + 40)) < 0.3
    words, off = MK.pack_custom([a, b])
    assert words.dtype == np.uint32 and off.dtype == np.int64
    wa, wb = (shape[1] + 31) // 32, (shape[1] + 40 + 31) // 32
    assert list(off) == [0, shape[0] * wa, shape[0] * wa + (shape[0] + 1) * wb]
    assert np.array_equal(OM.unpack_rows(words[off[0]:off[1]], shape[0], shape[1]), a)
    assert np.array_equal(OM.unpack_rows(words[off[1]:off[2]], shape[0] + 1, shape[1] + 40), b)


def test_pack_custom_bit_order_closed_form():
    """Key j of a row sets bit j % 32 of word j // 32: one visible key per row gives the
    power of two at that position and zeros elsewhere."""
    lk = 70
    dense = np.eye(lk, dtype=bool)
    words, _ = MK.pack_custom([dense])
    w = words.reshape(lk, 3)
    for j in range(lk):
        expect = np.zeros(3, np.uint32)
        expect[j // 32] = np.uint32(1) << np.uint32(j % 32)
        assert np.array_equal(w[j], expect)


def test_custom_mask_tile_classes_through_the_oracle():
    """A Mask built by custom(pack_custom(...)) is read by the oracle as the same booleans:
    its tile classes equal the classes counted directly on the dense masks (an empty
    column block and full tiles included)."""
    rng = np.random.default_rng(7)
    lq = [300, 129]
    dense = [rng.random((n, n)) < 0.6 for n in lq]
    dense[0][:, 200:] = False
    dense[0][:128, :128] = True
    m = MK.custom(*MK.pack_custom(dense))
    expect = []
    for d in dense:
        nt = (d.shape[0] + 127) // 128
        for a in range(nt):
            for b in range(nt):
                t = d[a * 128:(a + 1) * 128, b * 128:(b + 1) * 128]
                expect.append(0 if not t.any() else (1 if t.all() else 2))
    assert np.array_equal(OM.tile_classes(m, [(n, n) for n in lq]), np.asarray(expect, np.uint8))


def test_constructor_validation():
    with pytest.raises(ValueError):
        MK.sliding_window(0)
    with pytest.raises(ValueError):
        MK.prefix_lm(-1)
    with pytest.raises(ValueError):
        MK.chunk_causal(0, 8, 0, 8, 0)
    with pytest.raises(ValueError):
        MK.ranges([[(0, 1, 0, 1, 0)]])
    with pytest.raises(ValueError):
        MK.custom(np.zeros(4, np.uint32), [0, 3, 2])
    with pytest.raises(ValueError):
        MK.block_sparse(0, 16, [0], [])
