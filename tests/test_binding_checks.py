"""CPU tests of the binding's tensor checks: the C ABI takes bare pointers, so the binding
refuses, before any library call, tensors of the wrong type, layout or size and tensors
that are not on a CUDA device."""
import pytest
import torch

import masked_flash_attention_attn_b200 as M


def _plan():
    # a plan object without a library handle: only its sizes are used by the checks
    return M.Plan(None, None, hq=4, head_dim=64, total_q=10, hkv=2, kv_rows=12)


def _good():
    bf = torch.bfloat16
    return dict(q=torch.zeros(10, 4, 64, dtype=bf), k=torch.zeros(12, 2, 64, dtype=bf),
                v=torch.zeros(12, 2, 64, dtype=bf), out=torch.zeros(10, 4, 64, dtype=bf),
                lse=torch.zeros(10, 4, dtype=torch.float32))


def _fwd(**kw):
    a = _good()
    a.update(kw)
    M.attn_masked_fwd(_plan(), a["q"], a["k"], a["v"], a["out"], a["lse"])


def test_right_tensors_fail_only_for_not_being_on_a_gpu():
    with pytest.raises(ValueError, match="CUDA"):
        _fwd()


@pytest.mark.parametrize("name", ["q", "k", "v", "out"])
def test_wrong_dtype(name):
    t = _good()[name].float()
    with pytest.raises(TypeError, match=name):
        _fwd(**{name: t})


def test_lse_dtype_and_optional():
    with pytest.raises(TypeError, match="lse"):
        _fwd(lse=torch.zeros(10, 4, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="CUDA"):   # lse may be omitted
        _fwd(lse=None)


@pytest.mark.parametrize("name,shape", [("q", (9, 4, 64)), ("k", (11, 2, 64)), ("v", (12, 2, 32)),
                                        ("out", (10, 3, 64)), ("lse", (10, 3))])
def test_too_small(name, shape):
    dt = torch.float32 if name == "lse" else torch.bfloat16
    with pytest.raises(ValueError, match=name):
        _fwd(**{name: torch.zeros(*shape, dtype=dt)})


def test_not_contiguous_and_not_a_tensor():
    with pytest.raises(ValueError, match="contiguous"):
        _fwd(q=torch.zeros(64, 4, 10, dtype=torch.bfloat16).transpose(0, 2))
    with pytest.raises(TypeError, match="torch tensor"):
        _fwd(k=[0.0] * 10)
    with pytest.raises(ValueError, match="required"):
        _fwd(out=None)


def test_backward_checks_every_tensor():
    a = _good()
    g = dict(dout=a["out"].clone(), dq=a["q"].clone(), dk=a["k"].clone(), dv=a["v"].clone())
    with pytest.raises(ValueError, match="CUDA"):
        M.attn_masked_bwd(_plan(), a["q"], a["k"], a["v"], a["out"], a["lse"], g["dout"], g["dq"], g["dk"], g["dv"])
    with pytest.raises(ValueError, match="dk"):
        M.attn_masked_bwd(_plan(), a["q"], a["k"], a["v"], a["out"], a["lse"], g["dout"], g["dq"],
                          a["k"][:5].clone(), g["dv"])
    with pytest.raises(ValueError, match="lse is required"):
        M.attn_masked_bwd(_plan(), a["q"], a["k"], a["v"], a["out"], None, g["dout"], g["dq"], g["dk"], g["dv"])
    with pytest.raises(TypeError, match="dlse"):
        M.attn_masked_bwd(_plan(), a["q"], a["k"], a["v"], a["out"], a["lse"], g["dout"], g["dq"], g["dk"], g["dv"],
                          dlse=a["lse"].double())


def test_e4m3_inputs_are_bytes():
    z = torch.zeros(64, dtype=torch.uint8)
    out = torch.zeros(10, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(TypeError, match="q8"):
        M.attn_masked_fwd_fp8(_plan(), z.float(), z, z, 16, 1.0, 1.0, 1.0, out)
    with pytest.raises(ValueError, match="CUDA"):
        M.attn_masked_fwd_fp8(_plan(), z, z.view(torch.float8_e4m3fn), z, 16, 1.0, 1.0, 1.0, out)


def test_noalloc_checks_the_tensors_it_is_given():
    import numpy as np
    import workloads as W
    a = _good()
    cq, ck = np.array([0, 10], np.int32), np.array([0, 12], np.int32)
    kw = dict(hq=4, hkv=2, head_dim=64, cu_seqlens_q=cq, cu_seqlens_k=ck, mask=W.MaskSpec("CAUSAL"))
    with pytest.raises(ValueError, match="CUDA"):
        M.attn_masked_fwd_noalloc(**kw, **a)
    with pytest.raises(ValueError, match="v has"):
        M.attn_masked_fwd_noalloc(**kw, **dict(a, v=a["v"][:3].clone()))


def test_ranges_with_the_wrong_number_of_fields_are_refused(attn_lib):
    import numpy as np
    import workloads as W
    cq = np.array([0, 12], np.int32)
    bad = W.MaskSpec("RANGES", ranges=[[(0, 12, 0, 12, 1)] * 6])   # five fields: 30 numbers = 5 x 6
    with pytest.raises(ValueError, match="six fields"):
        attn_lib.attn_classify_host(hq=1, hkv=1, head_dim=64, cu_seqlens_q=cq, cu_seqlens_k=cq, mask=bad)


def test_mask_host_arrays_checked_against_the_batch(attn_lib):
    import numpy as np
    import workloads as W
    cq = np.array([0, 100, 300], np.int32)
    kw = dict(hq=1, hkv=1, head_dim=64, cu_seqlens_q=cq, cu_seqlens_k=cq)
    cases = [W.MaskSpec("PREFIX_LM", prefix_lens=np.array([4], np.int32)),
             W.MaskSpec("RANGES", ranges=[[(0, 10, 0, 10, 0, 0)]]),
             W.MaskSpec("BLOCK_SPARSE", block_q=64, block_k=64, bsr_row_ptr=np.zeros(5, np.int32),
                        bsr_col_idx=np.zeros(0, np.int32)),   # 2 + 4 block rows need 7 entries
             W.MaskSpec("BLOCK_SPARSE", block_q=64, block_k=64, bsr_row_ptr=np.full(7, 3, np.int32),
                        bsr_col_idx=np.zeros(2, np.int32))]
    for spec in cases:
        with pytest.raises(ValueError):
            attn_lib.attn_classify_host(mask=spec, **kw)
        with pytest.raises(ValueError):
            attn_lib.attn_plan_dry_run(mask=spec, **kw)


def test_page_table_checked():
    import numpy as np
    import workloads as W
    cq = np.array([0, 10, 20], np.int32)
    kw = dict(hq=1, hkv=1, head_dim=64, cu_seqlens_q=cq, kv_lens=np.array([10, 10], np.int32), page_size=16,
              num_pages=4, mask=W.MaskSpec("CAUSAL"))
    with pytest.raises(TypeError, match="page_table"):
        M.attn_plan(page_table=torch.zeros(2, 1, dtype=torch.int64), **kw)
    with pytest.raises(ValueError, match="rows"):
        M.attn_plan(page_table=torch.zeros(1, 1, dtype=torch.int32), **kw)
    with pytest.raises(ValueError, match="CUDA"):
        M.attn_plan(page_table=torch.zeros(2, 1, dtype=torch.int32), **kw)


def test_device_mask_bits_checked():
    import numpy as np
    import workloads as W
    cq = np.array([0, 40], np.int32)
    off = np.array([0, 80], np.int64)
    kw = dict(hq=1, hkv=1, head_dim=64, cu_seqlens_q=cq, cu_seqlens_k=cq)
    with pytest.raises(TypeError, match="mask.bits"):
        M.attn_plan(mask=W.MaskSpec("CUSTOM", bits=torch.zeros(80, dtype=torch.int64), word_offsets=off), **kw)
    with pytest.raises(ValueError, match="CUDA"):
        M.attn_plan(mask=W.MaskSpec("CUSTOM", bits=torch.zeros(80, dtype=torch.int32), word_offsets=off), **kw)
