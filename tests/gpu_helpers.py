"""Shared helpers of the GPU parity tests: run a workload through the C ABI and compare
with the oracle. Tolerances (out vs oracle: max-abs 2e-2, mean-abs 2e-3; lse: 1e-3
absolute) are the ones the benchmark suite states for bf16 inputs with fp32
accumulation."""
import numpy as np
import torch

import masked_flash_attention_attn_b200 as M
import oracle

OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
LSE_ABS = 1e-3


def noalloc_too_large_problem():
    """A problem whose plan exceeds the allocation-free entry's 32 MiB array: 16384 sequences
    of 128 tokens, 64 query and KV heads, FULL mask -- about a million 64-byte work items.
    Returns (cu_seqlens, keyword arguments)."""
    cq = (np.arange(16384 + 1) * 128).astype(np.int32)
    return cq, dict(hq=64, hkv=64, head_dim=128)


def device_inputs(wl, dev="cuda"):
    q = wl.q.to(dev)
    if wl.paged:
        return q, wl.k_cache.to(dev), wl.v_cache.to(dev)
    return q, wl.k.to(dev), wl.v.to(dev)


def make_plan(wl, spec, dev="cuda", stream=None, kv_splits=0):
    kw = dict(hq=wl.hq, hkv=wl.hkv, head_dim=wl.d, cu_seqlens_q=wl.cu_seqlens_q, mask=spec, scale=wl.scale,
              stream=stream, kv_splits=kv_splits)
    if wl.paged:
        kw.update(kv_lens=wl.kv_lens, page_table=torch.from_numpy(wl.page_table).to(dev),
                  page_size=wl.page_size, num_pages=wl.k_cache.shape[0])
    else:
        kw.update(cu_seqlens_k=wl.cu_seqlens_k)
    return M.attn_plan(**kw)


def run(wl, spec, inputs=None, extra_rows=0, canary=None, kv_splits=0):
    """Plan + forward; returns (out fp32 [total_q, hq, d], lse [total_q, hq], plan).
    ``extra_rows`` canary-filled rows follow the real ones in the output buffers."""
    q, k, v = inputs if inputs is not None else device_inputs(wl)
    plan = make_plan(wl, spec, kv_splits=kv_splits)
    tq = int(wl.cu_seqlens_q[-1])
    out = torch.empty(tq + extra_rows, wl.hq, wl.d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(tq + extra_rows, wl.hq, dtype=torch.float32, device="cuda")
    if canary is not None:
        out.fill_(canary)
        lse.fill_(canary)
    M.attn_masked_fwd(plan, q, k, v, out, lse)
    st = M.attn_plan_check_status(plan)
    assert st == 0, M.STATUS.get(st, st)
    return out.float().cpu(), lse.cpu(), plan


def compare(out, lse, ref_out, ref_lse, what=""):
    out = out.numpy().astype(np.float64) if isinstance(out, torch.Tensor) else out
    lse = lse.numpy().astype(np.float64) if isinstance(lse, torch.Tensor) else lse
    assert np.isfinite(out).all(), f"{what}: non-finite output"
    err = np.abs(out - ref_out)
    assert err.max() <= OUT_MAX_ABS, f"{what}: out max-abs {err.max():.3e}"
    assert err.mean() <= OUT_MEAN_ABS, f"{what}: out mean-abs {err.mean():.3e}"
    fin = np.isfinite(ref_lse)
    assert np.array_equal(fin, np.isfinite(lse)), f"{what}: -inf rows differ"
    assert np.all(lse[~fin] == -np.inf)
    if fin.any():
        le = np.abs(lse[fin] - ref_lse[fin])
        assert le.max() <= LSE_ABS, f"{what}: lse max-abs {le.max():.3e}"
    return float(err.max()), float(err.mean())


def lengths(wl):
    return [(wl.lq(b), wl.lk(b)) for b in range(wl.batch)]


def check_full(wl, spec, what="", kv_splits=0):
    """Whole-output comparison against the full oracle (small problems)."""
    out, lse, plan = run(wl, spec, kv_splits=kv_splits)
    ref_out, ref_lse = oracle.masked_attention(wl, spec)
    cls = M.attn_plan_get_tile_classes(plan)
    assert np.array_equal(cls, oracle.tile_classes(spec, lengths(wl))), f"{what}: tile classes"
    return compare(out, lse, ref_out, ref_lse, what)


def sample_rows(wl, n, seed):
    """Deterministic sample of (b, h, i) that always includes first/last rows of sequences."""
    rng = np.random.default_rng(seed)
    s = []
    for b in range(wl.batch):
        lq = wl.lq(b)
        if lq == 0:
            continue
        for i in {0, lq - 1, lq // 2}:
            s.append((b, int(rng.integers(0, wl.hq)), int(i)))
    while len(s) < n:
        b = int(rng.integers(0, wl.batch))
        if wl.lq(b) == 0:
            continue
        s.append((b, int(rng.integers(0, wl.hq)), int(rng.integers(0, wl.lq(b)))))
    return s


def check_sampled(wl, spec, out, lse, samples, what=""):
    ref_o, ref_l = oracle.sampled_attention(wl, spec, samples)
    got_o = np.stack([out[int(wl.cu_seqlens_q[b]) + i, h].numpy() for b, h, i in samples]).astype(np.float64)
    got_l = np.array([float(lse[int(wl.cu_seqlens_q[b]) + i, h]) for b, h, i in samples])
    return compare(got_o, got_l, ref_o, ref_l, what)
