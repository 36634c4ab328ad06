"""fp64 gradients of the masked attention forward (oracle; test infrastructure only).

The forward (oracle.attention) is, per sequence and query head h with key/value head
kh = floor(h / g), g = Hq / Hkv:

    s_ij = scale * q_i . k_j,  p_ij = exp(s_ij - lse_i) on visible (i, j), 0 elsewhere,
    out_i = sum_j p_ij v_j.

For a loss whose gradient with respect to out is dout (lse treated as an output without
a gradient of its own), the chain rule through the row softmax gives

    dv_j  = sum_i p_ij dout_i
    dp_ij = dout_i . v_j
    D_i   = sum_j p_ij dp_ij  ( = dout_i . out_i )
    ds_ij = p_ij (dp_ij - D_i)
    dq_i  = scale * sum_j ds_ij k_j
    dk_j  = scale * sum_i ds_ij q_i

and dk, dv of a key/value head are the sums over the g query heads that read it. A row
that sees no key has p = 0 and contributes nothing. When the loss also depends on lse
with gradient dlse_i, d lse_i / d s_ij = p_ij adds p_ij dlse_i to ds_ij, i.e. D_i becomes
D_i - dlse_i. These are the textbook derivatives of
softmax(scale Q K^T + mask) V; nothing here is taken from the CUDA path.
"""
from __future__ import annotations

import numpy as np

from .attention import attention_one_head, _f64
from .masks import dense_mask, dense_mask_rows


def attention_backward_one_head(q, k, v, mask, scale, dout, dlse=None):
    """q [n, d], k, v [L_k, d], mask bool [n, L_k], dout [n, d], dlse [n] or None; fp64.
    Returns (dq [n, d], dk [L_k, d], dv [L_k, d])."""
    out, lse = attention_one_head(q, k, v, mask, scale)
    has = np.isfinite(lse)
    s = scale * (q @ k.T)
    p = np.where(mask & has[:, None], np.exp(np.where(mask, s, 0.0) - np.where(has, lse, 0.0)[:, None]), 0.0)
    dv = p.T @ dout
    dp = dout @ v.T
    big_d = np.sum(p * dp, axis=1)
    if dlse is not None:
        big_d = big_d - np.asarray(dlse, np.float64)
    ds = p * (dp - big_d[:, None])
    dq = scale * (ds @ k)
    dk = scale * (ds.T @ q)
    return dq, dk, dv


def masked_attention_backward(wl, spec, dout, dlse=None):
    """Gradients: dout [total_q, Hq, d], dlse [total_q, Hq] or None (torch or numpy).
    Returns dq fp64 [total_q, Hq, d] and dk, dv fp64 shaped like the keys: [total_k, Hkv, d]
    for contiguous K/V; for a paged cache [num_pages, page_size, Hkv, d], key j of sequence b
    being cache row (page_table[b, j // page_size], j % page_size) -- a cache entry's
    gradient is the sum over the keys stored there, and entries no sequence reads get 0."""
    dout = dout.to(__import__("torch").float64).numpy() if hasattr(dout, "numpy") else np.asarray(dout, np.float64)
    if dlse is not None:
        dlse = dlse.to(__import__("torch").float64).numpy() if hasattr(dlse, "numpy") else np.asarray(dlse, np.float64)
    g = wl.hq // wl.hkv
    total_q = int(wl.cu_seqlens_q[-1])
    dq = np.zeros((total_q, wl.hq, wl.d))
    if wl.paged:
        dk = np.zeros((wl.k_cache.shape[0], wl.page_size, wl.hkv, wl.d))
    else:
        dk = np.zeros((int(wl.cu_seqlens_k[-1]), wl.hkv, wl.d))
    dv = np.zeros_like(dk)
    for b in range(wl.batch):
        lq, lk = wl.lq(b), wl.lk(b)
        q0 = int(wl.cu_seqlens_q[b])
        if lq == 0 or lk == 0:
            continue
        m = dense_mask(spec, b, lq, lk)
        kk, vv = wl.kv_of_seq(b)
        kk, vv = _f64(kk), _f64(vv)
        if wl.paged:   # cache (page, slot) of every key of the sequence
            keys = np.arange(lk)
            rows = (np.asarray(wl.page_table[b], np.int64)[keys // wl.page_size], keys % wl.page_size)
        else:
            k0 = int(wl.cu_seqlens_k[b])
            rows = (np.arange(k0, k0 + lk),)
        for h in range(wl.hq):
            kh = h // g
            a, bk, bv = attention_backward_one_head(_f64(wl.q[q0:q0 + lq, h]), kk[:, kh], vv[:, kh], m, wl.scale,
                                                    dout[q0:q0 + lq, h],
                                                    None if dlse is None else dlse[q0:q0 + lq, h])
            dq[q0:q0 + lq, h] = a
            np.add.at(dk, rows + (kh,), bk)
            np.add.at(dv, rows + (kh,), bv)
    return dq, dk, dv


def sampled_backward(wl, spec, dout, q_samples, k_samples, row_block: int = 1024):
    """Gradients at sampled places of a contiguous workload, for full-size problems.

    q_samples: (b, h, i) -> dq[token of row i of sequence b, h]
    k_samples: (b, kh, j) -> dk, dv[key j of sequence b, kh] (summed over kh's query heads)
    Every value follows the definitions of this module; a dq row needs its own row of p and
    dp, a dk / dv row needs column j of p and ds over every query row of every query head
    of kh (computed in blocks of rows). Returns (dq [n_q, d], dk [n_k, d], dv [n_k, d])."""
    import torch
    dout = dout.to(torch.float64).numpy() if hasattr(dout, "numpy") else np.asarray(dout, np.float64)
    g = wl.hq // wl.hkv
    dq = np.zeros((len(q_samples), wl.d))
    for n, (b, h, i) in enumerate(q_samples):
        lq, lk = wl.lq(b), wl.lk(b)
        q0, k0 = int(wl.cu_seqlens_q[b]), int(wl.cu_seqlens_k[b])
        kk, vv = (_f64(t) for t in wl.kv_of_seq(b))
        m = dense_mask_rows(spec, b, lq, lk, i, i + 1)
        a, _, _ = attention_backward_one_head(_f64(wl.q[q0 + i:q0 + i + 1, h]), kk[:, h // g], vv[:, h // g], m,
                                              wl.scale, dout[q0 + i:q0 + i + 1, h])
        dq[n] = a[0]
    dk = np.zeros((len(k_samples), wl.d))
    dv = np.zeros((len(k_samples), wl.d))
    by_seq_head = {}
    for n, (b, kh, j) in enumerate(k_samples):
        by_seq_head.setdefault((b, kh), []).append((n, j))
    for (b, kh), lst in by_seq_head.items():
        lq, lk = wl.lq(b), wl.lk(b)
        q0 = int(wl.cu_seqlens_q[b])
        kk, vv = (_f64(t) for t in wl.kv_of_seq(b))
        kk, vv = kk[:, kh], vv[:, kh]
        cols = np.array([j for _, j in lst])
        for h in range(kh * g, (kh + 1) * g):
            for r0 in range(0, lq, row_block):
                r1 = min(lq, r0 + row_block)
                m = dense_mask_rows(spec, b, lq, lk, r0, r1)
                q = _f64(wl.q[q0 + r0:q0 + r1, h])
                do = dout[q0 + r0:q0 + r1, h]
                out, lse = attention_one_head(q, kk, vv, m, wl.scale)
                has = np.isfinite(lse)
                s = wl.scale * (q @ kk[cols].T)                       # rows x sampled keys
                mc = m[:, cols] & has[:, None]
                p = np.where(mc, np.exp(np.where(mc, s, 0.0) - np.where(has, lse, 0.0)[:, None]), 0.0)
                big_d = np.sum(do * out, axis=1)                      # D_i = dout_i . out_i
                ds = p * (do @ vv[cols].T - big_d[:, None])
                for c, (n, _) in enumerate(lst):
                    dk[n] += wl.scale * ds[:, c] @ q
                    dv[n] += p[:, c] @ do
    return dq, dk, dv
