"""GPU test of attn_masked_fwd_noalloc, the forward for callers that cannot allocate
device memory (for example a runtime that hands out every device buffer from its own
pool). It keeps its plan in a fixed array inside the library; this test calls it twice in
a row through the C ABI, on different problems, and checks each output against the
regular attn_plan + attn_masked_fwd path, with the tolerances of the other parity tests.
It lives in its own file so that it is collected last."""
import numpy as np
import pytest
import torch

import workloads as W
import masked_flash_attention_attn_b200 as M
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


def _noalloc(wl, spec):
    q, k, v = G.device_inputs(wl)
    tq = int(wl.cu_seqlens_q[-1])
    out = torch.full((tq, wl.hq, wl.d), 5.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((tq, wl.hq), 5.0, dtype=torch.float32, device="cuda")
    kw = dict(hq=wl.hq, hkv=wl.hkv, head_dim=wl.d, cu_seqlens_q=wl.cu_seqlens_q, mask=spec, scale=wl.scale,
              q=q, k=k, v=v, out=out, lse=lse)
    if wl.paged:
        kw.update(kv_lens=wl.kv_lens, page_table=torch.from_numpy(wl.page_table).cuda(), page_size=wl.page_size,
                  num_pages=wl.k_cache.shape[0])
    else:
        kw.update(cu_seqlens_k=wl.cu_seqlens_k)
    M.attn_masked_fwd_noalloc(**kw)
    torch.cuda.synchronize()
    return out.float().cpu(), lse.cpu(), (q, k, v)


def test_noalloc_matches_regular_entry_two_calls_in_a_row(attn_lib):
    assert torch.cuda.is_available()
    cases = [W.random_small(seed=61, kind="CHUNK_CAUSAL", batch=3, hq=4, hkv=2, d=128, lmin=100, lmax=600),
             W.random_small(seed=62, kind="SLIDING_WINDOW", batch=4, hq=8, hkv=2, d=256, lmin=1, lmax=500,
                            paged=True)]
    for wl in cases:
        out, lse, inputs = _noalloc(wl, wl.masks[0])
        ref_out, ref_lse, _ = G.run(wl, wl.masks[0], inputs)
        G.compare(out, lse, ref_out.numpy().astype(np.float64), ref_lse.numpy().astype(np.float64),
                  f"noalloc {wl.name}")


def test_noalloc_rejects_plans_beyond_its_scratch(attn_lib):
    # 16384 sequences of 128 tokens x 64 heads: about a million 64-byte work items (68 MiB,
    # see the CPU test of this premise), rejected before any device work (no tensors are touched)
    cq, kw = G.noalloc_too_large_problem()
    with pytest.raises(M.AttnError) as e:
        M.attn_masked_fwd_noalloc(cu_seqlens_q=cq, cu_seqlens_k=cq, mask=W.MaskSpec("FULL"), q=None, k=None,
                                  v=None, out=None, **kw)
    assert e.value.status == 7
    with pytest.raises(M.AttnError) as e:
        wl = W.random_small(seed=3, kind="CUSTOM", batch=2)
        _noalloc(wl, wl.masks[0])
    assert e.value.status == 2
