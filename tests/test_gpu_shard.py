"""GPU parity of the query-row shards (one long sequence over several GPUs): the ranks are
emulated one after the other on one GPU, each with its own plan over its query rows and
all of K/V, writing into one output buffer; together they must give the oracle's output,
and one shard alone must leave the other rows untouched."""
import numpy as np
import pytest
import torch

import workloads as W
import oracle
from masked_flash_attention_attn_b200 import sharding as S
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu
CANARY = -777.0


@pytest.fixture(scope="module", autouse=True)
def _lib(attn_lib):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return attn_lib


def _plan(wl, spec, rows):
    kw = dict(hq=wl.hq, hkv=wl.hkv, head_dim=wl.d, cu_seqlens_q=wl.cu_seqlens_q, cu_seqlens_k=wl.cu_seqlens_k,
              mask=spec, scale=wl.scale, q_rows=rows)
    return G.M.attn_plan(**kw)


@pytest.mark.parametrize("d,kind,world", [(128, "CAUSAL", 3), (128, "CUSTOM", 2), (256, "SLIDING_WINDOW", 3),
                                          (64, "RANGES", 4)])
def test_query_shards_together_equal_the_oracle(d, kind, world):
    wl = W.random_small(seed=40 + d + world, kind=kind, batch=2, hq=4, hkv=2, d=d, lmin=300, lmax=1100)
    spec = wl.masks[0]
    q, k, v = G.device_inputs(wl)
    tq = int(wl.cu_seqlens_q[-1])
    out = torch.full((tq, wl.hq, wl.d), CANARY, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((tq, wl.hq), CANARY, dtype=torch.float32, device="cuda")
    lmax = max(wl.lq(b) for b in range(wl.batch))
    for r in range(world):
        plan = _plan(wl, spec, S.query_shard(lmax, r, world))
        G.M.attn_masked_fwd(plan, q, k, v, out, lse)
        assert G.M.attn_plan_check_status(plan) == 0
    ref_o, ref_l = oracle.masked_attention(wl, spec)
    G.compare(out.float().cpu(), lse.cpu(), ref_o, ref_l, f"{world} shards {kind} d={d}")


def test_one_shard_leaves_other_rows():
    wl = W.random_small(seed=5, kind="CAUSAL", batch=2, hq=4, hkv=2, d=128, lmin=500, lmax=900)
    spec = wl.masks[0]
    q, k, v = G.device_inputs(wl)
    tq = int(wl.cu_seqlens_q[-1])
    out = torch.full((tq, wl.hq, wl.d), CANARY, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((tq, wl.hq), CANARY, dtype=torch.float32, device="cuda")
    rows = (256, 512)
    plan = _plan(wl, spec, rows)
    G.M.attn_masked_fwd(plan, q, k, v, out, lse)
    assert G.M.attn_plan_check_status(plan) == 0
    ref_o, ref_l = oracle.masked_attention(wl, spec)
    got, gl = out.float().cpu().numpy(), lse.cpu().numpy()
    for b in range(wl.batch):
        q0, lq = int(wl.cu_seqlens_q[b]), wl.lq(b)
        inside = np.zeros(lq, bool)
        inside[rows[0]:min(rows[1], lq)] = True
        sel = q0 + np.nonzero(inside)[0]
        G.compare(got[sel], gl[sel], ref_o[sel], ref_l[sel], f"shard rows seq {b}")
        # the plan's row blocks are whole 128-row (R-row) blocks: [256, 512) is exactly two
        rest = q0 + np.nonzero(~inside)[0]
        canary_bf16 = torch.tensor(CANARY, dtype=torch.bfloat16).item()   # -777 rounds to -776 in bf16
        assert np.all(got[rest] == canary_bf16) and np.all(gl[rest] == CANARY)
