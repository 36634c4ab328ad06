"""Pins of the oracle's attention arithmetic (CPU).

The oracle is checked against: a brute-force pure-Python loop on tiny inputs,
closed forms (one visible key; zero queries), the library softmax/logsumexp
on unmasked rows, the log-sum-exp merge identity over disjoint key sets, the
GQA head sharing, and the fully masked row convention. A few tests plant
plausible mistakes in a copy of the oracle and check that a pin catches them.
"""
import math

import numpy as np
import pytest
import torch

import workloads as W
import oracle
from oracle import attention as OA
from oracle import masks as OM


def _brute(q, k, v, mask, scale):
    """Independent triple loop: q [n][d], k/v [L][d] as Python floats."""
    n, L, d = len(q), len(k), len(q[0])
    out, lse = [], []
    for i in range(n):
        s = [scale * sum(q[i][t] * k[j][t] for t in range(d)) for j in range(L)]
        vis = [j for j in range(L) if mask[i][j]]
        if not vis:
            out.append([0.0] * d)
            lse.append(-math.inf)
            continue
        mx = max(s[j] for j in vis)
        z = sum(math.exp(s[j] - mx) for j in vis)
        li = mx + math.log(z)
        out.append([sum(math.exp(s[j] - li) * v[j][t] for j in vis) for t in range(d)])
        lse.append(li)
    return np.array(out), np.array(lse)


@pytest.mark.parametrize("kind", ["FULL", "CAUSAL", "SLIDING_WINDOW", "PREFIX_LM", "CHUNK_CAUSAL",
                                  "RANGES", "CUSTOM", "BLOCK_SPARSE"])
def test_brute_force_tiny(kind):
    wl = W.random_small(seed=11 + len(kind), kind=kind, batch=3, hq=4, hkv=2, d=8, lmin=1, lmax=13)
    spec = wl.masks[0]
    out, lse = oracle.masked_attention(wl, spec)
    g = wl.hq // wl.hkv
    for b in range(wl.batch):
        lq, lk = wl.lq(b), wl.lk(b)
        q0 = int(wl.cu_seqlens_q[b])
        kk, vv = wl.kv_of_seq(b)
        m = OM.dense_mask(spec, b, lq, lk)
        for h in range(wl.hq):
            qh = wl.q[q0:q0 + lq, h].double().tolist()
            o, l = _brute(qh, kk[:, h // g].double().tolist(), vv[:, h // g].double().tolist(),
                          m.tolist(), wl.scale)
            np.testing.assert_allclose(out[q0:q0 + lq, h], o, rtol=0, atol=1e-12)
            fin = np.isfinite(l)
            assert np.array_equal(fin, np.isfinite(lse[q0:q0 + lq, h]))
            np.testing.assert_allclose(lse[q0:q0 + lq, h][fin], l[fin], rtol=0, atol=1e-12)


def test_single_visible_key_closed_form():
    rng = np.random.default_rng(0)
    n, L, d, scale = 6, 9, 16, 0.3
    q, k, v = rng.normal(size=(n, d)), rng.normal(size=(L, d)), rng.normal(size=(L, d))
    pick = rng.integers(0, L, size=n)
    mask = np.zeros((n, L), bool)
    mask[np.arange(n), pick] = True
    out, lse = OA.attention_one_head(q, k, v, mask, scale)
    np.testing.assert_allclose(out, v[pick], atol=1e-14)
    np.testing.assert_allclose(lse, scale * np.einsum("nd,nd->n", q, k[pick]), atol=1e-13)


def test_zero_query_is_uniform_average():
    rng = np.random.default_rng(1)
    n, L, d = 5, 12, 4
    k, v = rng.normal(size=(L, d)), rng.normal(size=(L, d))
    mask = rng.random((n, L)) < 0.5
    mask[:, 0] = True
    out, lse = OA.attention_one_head(np.zeros((n, d)), k, v, mask, 0.7)
    for i in range(n):
        np.testing.assert_allclose(out[i], v[mask[i]].mean(0), atol=1e-14)
        assert abs(lse[i] - math.log(mask[i].sum())) < 1e-14


def test_full_mask_equals_library_softmax():
    g = torch.Generator().manual_seed(2)
    q = torch.randn(33, 64, generator=g, dtype=torch.float64)
    k = torch.randn(47, 64, generator=g, dtype=torch.float64)
    v = torch.randn(47, 64, generator=g, dtype=torch.float64)
    s = 0.125 * q @ k.T
    ref = torch.softmax(s, dim=-1) @ v
    out, lse = OA.attention_one_head(q.numpy(), k.numpy(), v.numpy(), np.ones((33, 47), bool), 0.125)
    np.testing.assert_allclose(out, ref.numpy(), atol=1e-13)
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), atol=1e-13)


def test_masked_rows_equal_library_attention():
    """With a random boolean mask (every row keeps at least one key) the oracle equals
    torch's scaled_dot_product_attention in fp64 given the same boolean mask."""
    g = torch.Generator().manual_seed(12)
    n, L, d = 29, 53, 32
    q = torch.randn(n, d, generator=g, dtype=torch.float64)
    k = torch.randn(L, d, generator=g, dtype=torch.float64)
    v = torch.randn(L, d, generator=g, dtype=torch.float64)
    mask = torch.rand(n, L, generator=g) < 0.3
    mask[torch.arange(n), torch.randint(0, L, (n,), generator=g)] = True
    ref = torch.nn.functional.scaled_dot_product_attention(q[None, None], k[None, None], v[None, None],
                                                           attn_mask=mask[None, None], scale=0.3)[0, 0]
    out, _ = OA.attention_one_head(q.numpy(), k.numpy(), v.numpy(), mask.numpy(), 0.3)
    np.testing.assert_allclose(out, ref.numpy(), atol=1e-12)


def test_lse_merge_over_disjoint_key_sets():
    rng = np.random.default_rng(3)
    n, L, d = 7, 40, 8
    q, k, v = rng.normal(size=(n, d)), rng.normal(size=(L, d)), rng.normal(size=(L, d))
    mask = rng.random((n, L)) < 0.6
    mask[:, 0] = mask[:, 39] = True
    split = rng.random((n, L)) < 0.5
    split[:, 0], split[:, 39] = True, False
    oa, la = OA.attention_one_head(q, k, v, mask & split, 2.0)
    ob, lb = OA.attention_one_head(q, k, v, mask & ~split, 2.0)
    o, l = OA.attention_one_head(q, k, v, mask, 2.0)
    lm = np.logaddexp(la, lb)
    np.testing.assert_allclose(lm, l, atol=1e-12)
    np.testing.assert_allclose(np.exp(la - lm)[:, None] * oa + np.exp(lb - lm)[:, None] * ob, o, atol=1e-12)


def test_fully_masked_row_is_zero_and_minus_inf():
    out, lse = OA.attention_one_head(np.ones((2, 3)), np.ones((4, 3)), np.ones((4, 3)),
                                     np.array([[0, 0, 0, 0], [0, 1, 0, 0]], bool), 1.0)
    assert np.all(out[0] == 0) and lse[0] == -np.inf
    np.testing.assert_allclose(out[1], 1.0)
    out, lse = OA.attention_one_head(np.ones((2, 3)), np.ones((0, 3)), np.ones((0, 3)),
                                     np.zeros((2, 0), bool), 1.0)
    assert np.all(out == 0) and np.all(lse == -np.inf)


def test_gqa_heads_share_their_kv_head():
    wl = W.random_small(seed=5, kind="CAUSAL", batch=2, hq=4, hkv=2, d=16, lmin=5, lmax=20)
    wl.q[:, 1] = wl.q[:, 0]      # heads 0, 1 -> kv head 0; heads 2, 3 -> kv head 1
    wl.q[:, 3] = wl.q[:, 2]
    wl.q[:, 2] = wl.q[:, 0]
    out, lse = oracle.masked_attention(wl, wl.masks[0])
    np.testing.assert_array_equal(out[:, 0], out[:, 1])
    assert not np.allclose(out[:, 0], out[:, 2])   # same query, different kv head


def test_sampled_rows_match_full_oracle():
    wl = W.random_small(seed=6, kind="PREFIX_LM", batch=3, hq=4, hkv=1, d=16, lmin=3, lmax=40)
    out, lse = oracle.masked_attention(wl, wl.masks[0])
    samples = [(b, h, i) for b in range(3) for h in (0, 3) for i in (0, wl.lq(b) - 1)]
    so, sl = oracle.sampled_attention(wl, wl.masks[0], samples)
    for n, (b, h, i) in enumerate(samples):
        t = int(wl.cu_seqlens_q[b]) + i
        np.testing.assert_allclose(so[n], out[t, h], rtol=0, atol=1e-13)   # BLAS blocking only
        assert abs(sl[n] - lse[t, h]) < 1e-13


def test_biting_window_changes_output_inert_does_not():
    L = 256
    wl = W.random_small(seed=7, kind="CAUSAL", batch=1, hq=2, hkv=2, d=16, lmin=L, lmax=L, equal_qk=True)
    oc, _ = oracle.masked_attention(wl, W.MaskSpec("CAUSAL"))
    oi, _ = oracle.masked_attention(wl, W.MaskSpec("SLIDING_WINDOW", window=4096))
    ob, _ = oracle.masked_attention(wl, W.MaskSpec("SLIDING_WINDOW", window=64))
    assert np.array_equal(oc, oi)
    assert np.abs(ob - oc).max() > 1e-2


# ---- planted mistakes: each must be caught by one of the pins above ------------------

def test_planted_mistakes_are_caught(monkeypatch):
    good = OA.attention_one_head

    def no_scale(q, k, v, mask, scale):
        return good(q, k, v, mask, 1.0)

    def off_by_one_max(q, k, v, mask, scale):
        o, l = good(q, k, v, mask, scale)
        return o, l - 1e-3

    caught = 0
    for bad in (no_scale, off_by_one_max):
        monkeypatch.setattr(OA, "attention_one_head", bad)
        try:
            test_single_visible_key_closed_form()
        except AssertionError:
            caught += 1
        monkeypatch.setattr(OA, "attention_one_head", good)
    assert caught == 2

    # an off-by-one window (keeps w + 1 keys) is caught by the per-row key count pin
    good_rows = OM.dense_mask_rows

    def wide_window(spec, b, lq, lk, r0, r1):
        if spec.kind == "SLIDING_WINDOW":
            spec = W.MaskSpec("SLIDING_WINDOW", window=spec.window + 1)
        return good_rows(spec, b, lq, lk, r0, r1)

    monkeypatch.setattr(OM, "dense_mask_rows", wide_window)
    from tests import test_oracle_masks as TM
    with pytest.raises(AssertionError):
        TM.test_sliding_window_inert_equals_causal_and_biting_differs()
    monkeypatch.setattr(OM, "dense_mask_rows", good_rows)

    # a chunk that forgets full attention inside the chunk (i.e. plain causal) is caught
    good_or = OM._range_or_into

    def chunk_as_causal(m, rng, r0, r1):
        rng = tuple(rng)
        if rng[4] == OM.R_CHUNK:
            rng = rng[:4] + (OM.R_CAUSAL, 0)
        return good_or(m, rng, r0, r1)

    monkeypatch.setattr(OM, "_range_or_into", chunk_as_causal)
    with pytest.raises(AssertionError):
        TM.test_chunk_causal_worked_example_matches_printed_full_ranges()
    monkeypatch.setattr(OM, "_range_or_into", good_or)
