"""fp64 masked attention (oracle; test infrastructure only).

For one sequence and one query head h (key/value head floor(h / (Hq/Hkv))):

    s_ij  = scale * sum_t q[i, t] * k[j, t]                (exact bf16 inputs, fp64)
    lse_i = m_i + ln( sum_{j: M[i,j]} exp(s_ij - m_i) ),   m_i = max_{j: M[i,j]} s_ij
    out_i = sum_{j: M[i,j]} exp(s_ij - lse_i) * v[j]

i.e. O = softmax(scale * Q K^T + mask) V with the natural-log row log-sum-exp
(scale included). A row with no visible key has out = 0 and lse = -inf.
The mask is the boolean dense mask of ``oracle.masks``; masked entries are
excluded outright, which equals the additive -1e30 mask of "feat: add Gemma2
sliding-window (local/global) attention" (Summary) on every row that keeps at
least one key.
"""
from __future__ import annotations

import numpy as np
import torch

from .masks import dense_mask_rows


def attention_one_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, mask: np.ndarray, scale: float):
    """q [n, d], k [L_k, d], v [L_k, d], mask bool [n, L_k]; all fp64. Returns (out [n, d], lse [n])."""
    s = scale * (q @ k.T)
    s = np.where(mask, s, -np.inf)
    m = s.max(axis=1) if s.shape[1] else np.full(s.shape[0], -np.inf)
    has = np.isfinite(m)
    m_safe = np.where(has, m, 0.0)
    e = np.exp(s - m_safe[:, None])              # exp(-inf) = 0 on masked entries
    z = e.sum(axis=1)
    lse = np.where(has, m_safe + np.log(np.where(has, z, 1.0)), -np.inf)
    p = np.exp(s - np.where(has, lse, 0.0)[:, None])
    out = np.where(has[:, None], p @ v, 0.0)
    return out, lse


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


def masked_attention(wl, spec, heads=None, row_block: int = 1024):
    """Full oracle over a workload: returns (out fp64 [total_q, Hq, d], lse fp64 [total_q, Hq]).
    ``heads`` restricts the computation to a subset of query heads (others left NaN)."""
    g = wl.hq // wl.hkv
    heads = list(range(wl.hq)) if heads is None else list(heads)
    total_q = int(wl.cu_seqlens_q[-1])
    out = np.full((total_q, wl.hq, wl.d), np.nan)
    lse = np.full((total_q, wl.hq), np.nan)
    for b in range(wl.batch):
        lq, lk = wl.lq(b), wl.lk(b)
        q0 = int(wl.cu_seqlens_q[b])
        kk, vv = wl.kv_of_seq(b)
        kk, vv = _f64(kk), _f64(vv)
        for r0 in range(0, lq, row_block):
            r1 = min(lq, r0 + row_block)
            m = dense_mask_rows(spec, b, lq, lk, r0, r1)
            for h in heads:
                qq = _f64(wl.q[q0 + r0:q0 + r1, h])
                o, l = attention_one_head(qq, kk[:, h // g], vv[:, h // g], m, wl.scale)
                out[q0 + r0:q0 + r1, h] = o
                lse[q0 + r0:q0 + r1, h] = l
    return out, lse


def sampled_attention(wl, spec, samples):
    """Oracle rows for a list of (sequence b, head h, local row i). Returns
    (out fp64 [n, d], lse fp64 [n]) in the order given."""
    g = wl.hq // wl.hkv
    out = np.zeros((len(samples), wl.d))
    lse = np.zeros(len(samples))
    cache = {}
    for n, (b, h, i) in enumerate(samples):
        lq, lk = wl.lq(b), wl.lk(b)
        if b not in cache:
            kk, vv = wl.kv_of_seq(b)
            cache = {b: (_f64(kk), _f64(vv))}
        kk, vv = cache[b]
        m = dense_mask_rows(spec, b, lq, lk, i, i + 1)
        qq = _f64(wl.q[int(wl.cu_seqlens_q[b]) + i, h][None, :])
        o, l = attention_one_head(qq, kk[:, h // g], vv[:, h // g], m, wl.scale)
        out[n], lse[n] = o[0], l[0]
    return out, lse
