"""Pins of the fp64 backward oracle (oracle/backward.py) to facts outside itself:
central finite differences of the pinned forward oracle, the autograd of the library
softmax / matmul on unmasked and causal rows, the softmax-gradient invariant
(sum_j ds_ij = 0, hence sum_j dk_j = 0), zero gradients for rows that see no key, and
the grouped-query sum. Planted mistakes (a dropped D term, a missing scale, a transposed
ds) must each fail one of them."""
import numpy as np
import pytest
import torch

import oracle
import oracle.backward as OB
import workloads as W


def _case(seed, n=5, lk=7, d=4, density=0.6, empty_row=True):
    rng = np.random.default_rng(seed)
    q, k, v, do = (rng.standard_normal(s) for s in ((n, d), (lk, d), (lk, d), (n, d)))
    mask = rng.random((n, lk)) < density
    mask[0, :] = True
    if empty_row:
        mask[1, :] = False
    return q, k, v, do, mask


def _loss(q, k, v, mask, scale, do):
    out, _ = oracle.attention_one_head(q, k, v, mask, scale)
    return float(np.sum(out * do))


def _fd(f, x, h=1e-6):
    g = np.zeros_like(x)
    for idx in np.ndindex(*x.shape):
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        g[idx] = (f(xp) - f(xm)) / (2 * h)
    return g


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_finite_differences(seed):
    q, k, v, do, mask = _case(seed)
    scale = 0.7
    dq, dk, dv = OB.attention_backward_one_head(q, k, v, mask, scale, do)
    assert np.allclose(dq, _fd(lambda x: _loss(x, k, v, mask, scale, do), q), rtol=1e-6, atol=1e-8)
    assert np.allclose(dk, _fd(lambda x: _loss(q, x, v, mask, scale, do), k), rtol=1e-6, atol=1e-8)
    assert np.allclose(dv, _fd(lambda x: _loss(q, k, x, mask, scale, do), v), rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("causal", [False, True])
def test_library_autograd(causal):
    rng = np.random.default_rng(7)
    n, d = 9, 6
    q, k, v, do = (rng.standard_normal((n, d)) for _ in range(4))
    scale = 0.4
    mask = np.tril(np.ones((n, n), bool)) if causal else np.ones((n, n), bool)
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    add = torch.zeros(n, n, dtype=torch.float64).masked_fill(torch.from_numpy(~mask), float("-inf"))
    out = torch.softmax(scale * tq @ tk.T + add, dim=-1) @ tv
    out.backward(torch.from_numpy(do))
    dq, dk, dv = OB.attention_backward_one_head(q, k, v, mask, scale, do)
    for a, b in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.allclose(a, b.numpy(), rtol=1e-12, atol=1e-12)


def test_invariants():
    q, k, v, do, mask = _case(3, n=12, lk=20, d=8)
    dq, dk, dv = OB.attention_backward_one_head(q, k, v, mask, 0.5, do)
    assert np.allclose(dk.sum(axis=0), 0.0, atol=1e-12)      # sum_j ds_ij = 0 for every row
    assert np.all(dq[1] == 0.0)                               # row 1 sees no key
    # dv_j = sum_i p_ij dout_i: the column sums of p are the weights of dout
    out, lse = oracle.attention_one_head(q, k, v, mask, 0.5)
    assert np.allclose(dv.sum(axis=0), (do * np.isfinite(lse)[:, None]).sum(axis=0), atol=1e-12)


def test_gqa_sum_over_query_heads():
    wl = W.random_small(seed=4, kind="CAUSAL", batch=2, hq=4, hkv=2, d=16, lmin=3, lmax=20)
    rng = np.random.default_rng(4)
    do = rng.standard_normal((int(wl.cu_seqlens_q[-1]), wl.hq, wl.d))
    dq, dk, dv = oracle.masked_attention_backward(wl, wl.masks[0], do)
    b, g = 1, 2
    lq, lk = wl.lq(b), wl.lk(b)
    q0, k0 = int(wl.cu_seqlens_q[b]), int(wl.cu_seqlens_k[b])
    m = oracle.dense_mask(wl.masks[0], b, lq, lk)
    kk, vv = (t.to(torch.float64).numpy() for t in wl.kv_of_seq(b))
    acc_k = np.zeros((lk, wl.d))
    for h in (2, 3):   # the query heads of key/value head 1
        _, a, _ = OB.attention_backward_one_head(wl.q[q0:q0 + lq, h].double().numpy(), kk[:, 1], vv[:, 1], m,
                                                 wl.scale, do[q0:q0 + lq, h])
        acc_k += a
    assert np.allclose(dk[k0:k0 + lk, 1], acc_k, atol=1e-12)


def test_planted_mistakes_are_caught(monkeypatch):
    good = OB.attention_backward_one_head

    def no_d_term(q, k, v, mask, scale, dout):
        out, lse = oracle.attention_one_head(q, k, v, mask, scale)
        has = np.isfinite(lse)
        p = np.where(mask & has[:, None], np.exp(np.where(mask, scale * q @ k.T, 0) - np.where(has, lse, 0)[:, None]), 0)
        ds = p * (dout @ v.T)
        return scale * ds @ k, scale * ds.T @ q, p.T @ dout

    def no_scale(q, k, v, mask, scale, dout):
        a, b, c = good(q, k, v, mask, scale, dout)
        return a / scale, b / scale, c

    def transposed(q, k, v, mask, scale, dout):
        a, b, c = good(q, k, v, mask, scale, dout)
        return a, b[::-1].copy(), c

    caught = 0
    for bad in (no_d_term, no_scale, transposed):
        monkeypatch.setattr(OB, "attention_backward_one_head", bad)
        try:
            test_finite_differences(0)
        except AssertionError:
            caught += 1
        monkeypatch.setattr(OB, "attention_backward_one_head", good)
    assert caught == 3


def test_sampled_backward_matches_full():
    wl = W.random_small(seed=9, kind="SLIDING_WINDOW", batch=2, hq=4, hkv=2, d=16, lmin=40, lmax=90)
    rng = np.random.default_rng(9)
    do = rng.standard_normal((int(wl.cu_seqlens_q[-1]), wl.hq, wl.d))
    dq, dk, dv = oracle.masked_attention_backward(wl, wl.masks[0], do)
    qs = [(b, int(rng.integers(0, wl.hq)), int(rng.integers(0, wl.lq(b)))) for b in (0, 1) for _ in range(4)]
    ks = [(b, int(rng.integers(0, wl.hkv)), int(rng.integers(0, wl.lk(b)))) for b in (0, 1) for _ in range(4)]
    sq, sk, sv = OB.sampled_backward(wl, wl.masks[0], do, qs, ks, row_block=16)
    for n, (b, h, i) in enumerate(qs):
        assert np.allclose(sq[n], dq[int(wl.cu_seqlens_q[b]) + i, h], atol=1e-12)
    for n, (b, kh, j) in enumerate(ks):
        assert np.allclose(sk[n], dk[int(wl.cu_seqlens_k[b]) + j, kh], atol=1e-12)
        assert np.allclose(sv[n], dv[int(wl.cu_seqlens_k[b]) + j, kh], atol=1e-12)


@pytest.mark.parametrize("seed", [0, 4])
def test_finite_differences_with_lse_gradient(seed):
    # loss = sum dout . out + sum over rows with keys of dlse . lse
    q, k, v, do, mask = _case(seed)
    rng = np.random.default_rng(seed + 100)
    dl = rng.standard_normal(q.shape[0])
    scale = 0.6

    def loss(qq, kk, vv):
        out, lse = oracle.attention_one_head(qq, kk, vv, mask, scale)
        fin = np.isfinite(lse)
        return float(np.sum(out * do) + np.sum(dl[fin] * lse[fin]))

    dq, dk, dv = OB.attention_backward_one_head(q, k, v, mask, scale, do, dl)
    assert np.allclose(dq, _fd(lambda x: loss(x, k, v), q), rtol=1e-6, atol=1e-8)
    assert np.allclose(dk, _fd(lambda x: loss(q, x, v), k), rtol=1e-6, atol=1e-8)
    assert np.allclose(dv, _fd(lambda x: loss(q, k, x), v), rtol=1e-6, atol=1e-8)


def test_paged_gradients_are_the_contiguous_ones_through_the_page_table():
    """A paged cache's gradients: the same keys laid out contiguously give the same per-key
    dk / dv, and the paged oracle puts key j of sequence b at cache row (page_table[b, j //
    page_size], j % page_size); rows no sequence reads (spare pages, the tail of a last
    page) are exactly zero."""
    wl = W.random_small(seed=91, kind="CAUSAL", batch=3, hq=4, hkv=2, d=16, lmin=5, lmax=70, paged=True,
                        page_size=16)
    kv = [wl.kv_of_seq(b) for b in range(wl.batch)]
    lk = np.asarray([wl.lk(b) for b in range(wl.batch)])
    twin = W.Workload(name="contiguous twin", hq=wl.hq, hkv=wl.hkv, d=wl.d, scale=wl.scale,
                      cu_seqlens_q=wl.cu_seqlens_q, q=wl.q, masks=wl.masks, cu_seqlens_k=W.cu_from_lengths(lk),
                      k=torch.cat([a for a, _ in kv]), v=torch.cat([b for _, b in kv]), seed=wl.seed)
    dout = torch.randn(int(wl.cu_seqlens_q[-1]), wl.hq, wl.d, generator=torch.Generator().manual_seed(5),
                       dtype=torch.float64)
    dq_p, dk_p, dv_p = oracle.masked_attention_backward(wl, wl.masks[0], dout)
    dq_c, dk_c, dv_c = oracle.masked_attention_backward(twin, twin.masks[0], dout)
    assert np.array_equal(dq_p, dq_c)
    assert dk_p.shape == (wl.k_cache.shape[0], wl.page_size, wl.hkv, wl.d)
    used = np.zeros(dk_p.shape[:2], bool)
    for b in range(wl.batch):
        k0 = int(twin.cu_seqlens_k[b])
        for j in range(int(lk[b])):
            pg, sl = int(wl.page_table[b, j // wl.page_size]), j % wl.page_size
            used[pg, sl] = True
            assert np.array_equal(dk_p[pg, sl], dk_c[k0 + j]) and np.array_equal(dv_p[pg, sl], dv_c[k0 + j])
    assert not dk_p[~used].any() and not dv_p[~used].any()
    assert (~used).sum() >= 7 * wl.page_size   # the spare pages are among the unread rows
