"""B200 (sm_100a) masked attention: forward, backward and e4m3 forward.

Thin Python binding over the C ABI declared in ``include/attn.h``: every function
here only marshals arguments (torch tensors supply device memory and streams);
all of the computation happens in ``libattn_b200.so``. Importing succeeds without a
GPU; calls that need one fail with a RuntimeError. If the library has not been
built, every call raises instead of falling back to anything else.

Typical use (q [total_q, hq, d], k / v [total_k, hkv, d] bf16 CUDA tensors)::

    from masked_flash_attention_attn_b200 import mask as masks
    plan = attn_plan(hq=16, hkv=8, head_dim=256, cu_seqlens_q=cu, cu_seqlens_k=cu,
                     mask=masks.sliding_window(4096))  # masks.causal(), .ranges(...), .custom(...)
    out, lse = forward(plan, q, k, v)                # every layer can reuse the plan

    plan = attn_plan(..., backward=True)             # also the dQ / dK / dV work lists
    out, lse = forward(plan, q, k, v)
    dq, dk, dv = backward(plan, q, k, v, out, lse, dout)

    attn_fp8_transpose_v(plan, v8, vt8, ldv)         # e4m3 inputs (uint8 tensors)
    attn_masked_fwd_fp8(plan, q8, k8, vt8, ldv, q_scale, k_scale, v_scale, out, lse)

``kv_splits`` (split-KV) and ``q_rows`` (a query-row shard, see ``sharding``) are
further attn_plan() arguments; attn_plan_dry_run() gives the plan statistics without
a GPU.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libattn_b200.so")

ATTN_OK = 0
STATUS = {0: "ATTN_OK", 1: "ATTN_ERR_INVALID_ARG", 2: "ATTN_ERR_UNSUPPORTED", 3: "ATTN_ERR_MASK_TOO_SMALL",
          4: "ATTN_ERR_OOM", 5: "ATTN_ERR_CUDA", 6: "ATTN_ERR_TIMEOUT", 7: "ATTN_ERR_TOO_LARGE"}
NOALLOC_SCRATCH_BYTES = 32 << 20
MASK_KIND = {"FULL": 0, "CAUSAL": 1, "SLIDING_WINDOW": 2, "PREFIX_LM": 3, "CHUNK_CAUSAL": 4, "RANGES": 5,
             "CUSTOM": 6, "BLOCK_SPARSE": 7}
RANGE_FULL, RANGE_CAUSAL, RANGE_INV_CAUSAL, RANGE_BI_CAUSAL, RANGE_CHUNK_CAUSAL = 0, 1, 2, 3, 4

# every symbol include/attn.h declares
EXPORTS = ("attn_plan", "attn_masked_fwd", "attn_plan_get_tile_classes", "attn_plan_get_stats",
           "attn_plan_check_status", "attn_plan_set_debug", "attn_plan_destroy", "attn_classify_host",
           "attn_status_string", "attn_masked_fwd_noalloc", "attn_test_exp2_poly", "attn_plan_dry_run",
           "attn_plan_bwd", "attn_masked_bwd", "attn_masked_fwd_fp8", "attn_fp8_transpose_v",
           "attn_test_transpose_mask_tile", "attn_test_noalloc_debug", "attn_plan_bwd_dry_run")


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class attn_range_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("q_start", "q_end", "k_start", "k_end", "type", "chunk_size")]


class attn_mask_desc_t(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("window", ctypes.c_int32), ("prefix_len", ctypes.c_int32),
                ("prefix_lens", ctypes.c_void_p), ("chunk", attn_range_t), ("ranges", ctypes.c_void_p),
                ("cu_ranges", ctypes.c_void_p), ("mask_bits", ctypes.c_void_p),
                ("mask_word_offsets", ctypes.c_void_p), ("mask_words_total", ctypes.c_int64),
                ("block_q", ctypes.c_int32), ("block_k", ctypes.c_int32), ("bsr_row_ptr", ctypes.c_void_p),
                ("bsr_col_idx", ctypes.c_void_p)]


class attn_problem_t(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("hq", ctypes.c_int32), ("hkv", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("scale", ctypes.c_float), ("cu_seqlens_q", ctypes.c_void_p),
                ("cu_seqlens_k", ctypes.c_void_p), ("kv_lens", ctypes.c_void_p), ("page_table", ctypes.c_void_p),
                ("page_size", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("kv_splits", ctypes.c_int32), ("q_begin", ctypes.c_int32), ("q_end", ctypes.c_int32)]


class attn_bwd_stats_t(ctypes.Structure):
    _fields_ = [("dq_items", ctypes.c_int64), ("dq_jobs", ctypes.c_int64), ("dkv_items", ctypes.c_int64),
                ("dkv_jobs", ctypes.c_int64), ("mask_tiles", ctypes.c_int64), ("dq_ctas", ctypes.c_int32),
                ("dkv_ctas", ctypes.c_int32), ("dq_cost", ctypes.c_int64), ("dkv_cost", ctypes.c_int64),
                ("dq_max_cta_cost", ctypes.c_int64), ("dkv_max_cta_cost", ctypes.c_int64),
                ("dq_max_item_cost", ctypes.c_int64), ("dkv_max_item_cost", ctypes.c_int64)]


class attn_plan_stats_t(ctypes.Structure):
    _fields_ = [("unmasked_pairs", ctypes.c_int64), ("tiles_empty", ctypes.c_int64), ("tiles_full", ctypes.c_int64),
                ("tiles_partial", ctypes.c_int64), ("mask_tiles", ctypes.c_int64), ("work_items", ctypes.c_int64),
                ("jobs", ctypes.c_int64), ("mask_tile_reads", ctypes.c_int64), ("ctas", ctypes.c_int32), ("heads_per_tile", ctypes.c_int32),
                ("tiles_per_cta", ctypes.c_int32), ("cluster_size", ctypes.c_int32),
                ("kv_splits_max", ctypes.c_int32), ("merge_tiles", ctypes.c_int32), ("vt_keys", ctypes.c_int64),
                ("workspace_bytes", ctypes.c_int64)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it was not built (no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                               "`python -m masked_flash_attention_attn_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        L.attn_plan.argtypes = [ctypes.POINTER(attn_problem_t), ctypes.POINTER(attn_mask_desc_t), vp,
                                ctypes.POINTER(vp)]
        L.attn_masked_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp]
        L.attn_plan_get_tile_classes.argtypes = [vp, vp, sz, ctypes.POINTER(sz)]
        L.attn_plan_get_stats.argtypes = [vp, ctypes.POINTER(attn_plan_stats_t)]
        L.attn_plan_check_status.argtypes = [vp, vp]
        L.attn_plan_set_debug.argtypes = [vp, i32, i64]
        L.attn_plan_destroy.argtypes = [vp]
        L.attn_classify_host.argtypes = [ctypes.POINTER(attn_problem_t), ctypes.POINTER(attn_mask_desc_t), vp, sz,
                                         ctypes.POINTER(sz), ctypes.POINTER(i64)]
        L.attn_status_string.argtypes = [i32]
        L.attn_status_string.restype = ctypes.c_char_p
        L.attn_test_exp2_poly.argtypes = [vp, vp, i64, vp]
        L.attn_plan_bwd.argtypes = [ctypes.POINTER(attn_problem_t), ctypes.POINTER(attn_mask_desc_t), vp,
                                    ctypes.POINTER(vp)]
        L.attn_masked_bwd.argtypes = [vp] * 12
        L.attn_masked_fwd_fp8.argtypes = [vp, vp, vp, vp, i64, ctypes.c_float, ctypes.c_float, ctypes.c_float, vp, vp,
                                          vp]
        L.attn_fp8_transpose_v.argtypes = [vp, vp, vp, i64, vp]
        L.attn_test_transpose_mask_tile.argtypes = [vp, vp]
        L.attn_plan_dry_run.argtypes = [ctypes.POINTER(attn_problem_t), ctypes.POINTER(attn_mask_desc_t), i32,
                                        ctypes.POINTER(attn_plan_stats_t)]
        L.attn_plan_bwd_dry_run.argtypes = [ctypes.POINTER(attn_problem_t), ctypes.POINTER(attn_mask_desc_t), i32,
                                            ctypes.POINTER(attn_bwd_stats_t)]
        L.attn_masked_fwd_noalloc.argtypes = [ctypes.POINTER(attn_problem_t), ctypes.POINTER(attn_mask_desc_t),
                                              vp, vp, vp, vp, vp, vp]
        L.attn_test_noalloc_debug.argtypes = [i32, i64]
        for n in EXPORTS:
            if n != "attn_status_string":
                getattr(L, n).restype = i32
        _lib = L
    return _lib


def _check(st: int, where: str):
    if st != ATTN_OK:
        raise AttnError(st, where)


def _ptr(a) -> Optional[int]:
    if a is None:
        return None
    if isinstance(a, np.ndarray):
        return a.ctypes.data
    return a.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return getattr(stream, "cuda_stream", stream)


class _Marshal:
    """Host arrays of one call, kept alive while the C side reads them."""

    def __init__(self):
        self.keep = []

    def arr(self, x, dtype):
        if x is None:
            return None
        a = np.ascontiguousarray(np.asarray(x, dtype=dtype))
        self.keep.append(a)
        return a.ctypes.data


def _problem(m: _Marshal, *, hq, hkv, head_dim, cu_seqlens_q, cu_seqlens_k=None, kv_lens=None, page_table=None,
             page_size=0, num_pages=0, scale=0.0, kv_splits=0, q_rows=None):
    cq = np.asarray(cu_seqlens_q, dtype=np.int32)
    pr = attn_problem_t()
    pr.batch = len(cq) - 1
    pr.hq, pr.hkv, pr.head_dim, pr.scale = hq, hkv, head_dim, float(scale)
    pr.kv_splits = int(kv_splits)
    if q_rows is not None:
        pr.q_begin, pr.q_end = int(q_rows[0]), int(q_rows[1])
    pr.cu_seqlens_q = m.arr(cq, np.int32)
    pr.cu_seqlens_k = m.arr(cu_seqlens_k, np.int32)
    pr.kv_lens = m.arr(kv_lens, np.int32)
    if page_table is not None:
        pr.page_table = _ptr(page_table)
        pr.max_pages_per_seq = int(page_table.shape[1])
        pr.page_size, pr.num_pages = int(page_size), int(num_pages)
    return pr


def _check_page_table(page_table, cu_seqlens_q):
    """The kernels read page_table[b][p] for every sequence b: a device int32 [batch,
    max_pages] tensor with a row per sequence."""
    if page_table is None:
        return
    import torch
    batch = len(np.asarray(cu_seqlens_q)) - 1
    if isinstance(page_table, torch.Tensor) and (page_table.dim() != 2 or page_table.shape[0] < batch):
        raise ValueError(f"page_table must be [batch, max_pages] with at least {batch} rows")
    _tensors((page_table, "page_table", (torch.int32,), None, False))


def _check_mask_arrays(mask, cu_seqlens_q):
    """The C side reads the mask's host arrays at indices the lengths imply and cannot see
    their sizes: check them here."""
    lq = np.diff(np.asarray(cu_seqlens_q, dtype=np.int64))
    batch = len(lq)
    pl = getattr(mask, "prefix_lens", None)
    if mask.kind == "PREFIX_LM" and pl is not None and len(pl) < batch:
        raise ValueError(f"prefix_lens has {len(pl)} entries for {batch} sequences")
    if mask.kind == "RANGES" and len(mask.ranges) < batch:
        raise ValueError(f"ranges has {len(mask.ranges)} sequences for {batch}")
    if mask.kind == "CUSTOM" and len(mask.word_offsets) < batch + 1:
        raise ValueError(f"word_offsets has {len(mask.word_offsets)} entries for {batch} sequences (needs B + 1)")
    if mask.kind == "BLOCK_SPARSE":
        bq = int(mask.block_q)
        if bq < 1:
            raise ValueError("block_q must be >= 1")
        rows = int(((lq + bq - 1) // bq).sum())
        ptr = np.asarray(mask.bsr_row_ptr, dtype=np.int64)
        if len(ptr) < rows + 1:
            raise ValueError(f"bsr_row_ptr has {len(ptr)} entries for {rows} block rows (needs rows + 1)")
        if len(mask.bsr_col_idx) < ptr[rows]:
            raise ValueError(f"bsr_col_idx has {len(mask.bsr_col_idx)} entries; bsr_row_ptr needs {ptr[rows]}")


def _mask_desc(m: _Marshal, mask, device_bits=None, cu_seqlens_q=None):
    """``mask``: an object with the attributes kind, window, prefix_len, prefix_lens, chunk,
    ranges (per-sequence lists of 6-tuples), bits, word_offsets, block_q, block_k,
    bsr_row_ptr, bsr_col_idx (see include/attn.h). With ``cu_seqlens_q`` the host arrays
    are checked against the batch first."""
    if cu_seqlens_q is not None:
        _check_mask_arrays(mask, cu_seqlens_q)
    d = attn_mask_desc_t()
    d.kind = MASK_KIND[mask.kind]
    d.window = int(getattr(mask, "window", 0) or 0)
    d.prefix_len = int(getattr(mask, "prefix_len", 0) or 0)
    d.prefix_lens = m.arr(getattr(mask, "prefix_lens", None), np.int32)
    ch = getattr(mask, "chunk", None)
    if ch is not None:
        d.chunk = attn_range_t(*[int(x) for x in ch])
    rs = getattr(mask, "ranges", None)
    if rs is not None:
        # attn_range_t is six int32 fields: an [n, 6] int32 array has its layout
        counts = [len(per) for per in rs]
        flat = np.zeros((max(1, sum(counts)), 6), np.int32)
        parts = [np.asarray(per, dtype=np.int64) for per in rs if len(per)]
        if any(a.ndim != 2 or a.shape[1] != 6 for a in parts):
            raise ValueError("each range has six fields (q_start, q_end, k_start, k_end, type, chunk_size)")
        if parts:
            flat[:sum(counts)] = np.concatenate(parts)
        cu = np.zeros(len(rs) + 1, np.int32)
        cu[1:] = np.cumsum(counts)
        d.ranges = m.arr(flat, np.int32)
        d.cu_ranges = m.arr(cu, np.int32)
    if mask.kind == "BLOCK_SPARSE":
        d.block_q, d.block_k = int(mask.block_q), int(mask.block_k)
        d.bsr_row_ptr = m.arr(mask.bsr_row_ptr, np.int32)
        d.bsr_col_idx = m.arr(mask.bsr_col_idx if len(mask.bsr_col_idx) else np.zeros(1), np.int32)
    if mask.kind == "CUSTOM":
        d.mask_word_offsets = m.arr(mask.word_offsets, np.int64)
        d.mask_bits = _ptr(device_bits)
        d.mask_words_total = int(device_bits.numel()) if device_bits is not None else 0
    return d


class Plan:
    """Owns an attn_plan_t. Keeps the device page table (read by every forward) alive and
    remembers the sizes the tensors of its calls must have."""

    def __init__(self, handle, page_table, hq, head_dim, total_q, hkv=None, kv_rows=None):
        self.handle = handle
        self._page_table = page_table
        self.hq, self.head_dim, self.total_q = hq, head_dim, total_q
        self.hkv, self.kv_rows = hkv, kv_rows   # kv_rows: total keys, or pages x page size

    def __del__(self):
        if getattr(self, "handle", None):
            try:
                attn_plan_destroy(self)
            except Exception:
                pass

    @property
    def stats(self) -> dict:
        return attn_plan_get_stats(self)


def attn_plan(*, hq: int, hkv: int, head_dim: int, cu_seqlens_q, mask, cu_seqlens_k=None, kv_lens=None,
              page_table=None, page_size: int = 0, num_pages: int = 0, scale: float = 0.0, kv_splits: int = 0,
              stream=None, backward: bool = False, q_rows=None) -> Plan:
    """attn_plan(): validate, classify tiles, build the work list. ``page_table`` is a device
    int32 tensor [batch, max_pages]; CUSTOM ``mask.bits`` may be host (numpy) or device words;
    ``kv_splits``: 0 automatic, 1 never, N >= 2 at most N key ranges per query tile."""
    import torch
    _check_page_table(page_table, cu_seqlens_q)
    m = _Marshal()
    pr = _problem(m, hq=hq, hkv=hkv, head_dim=head_dim, cu_seqlens_q=cu_seqlens_q, cu_seqlens_k=cu_seqlens_k,
                  kv_lens=kv_lens, page_table=page_table, page_size=page_size, num_pages=num_pages, scale=scale,
                  kv_splits=kv_splits, q_rows=q_rows)
    dev_bits = None
    if mask.kind == "CUSTOM":
        b = mask.bits
        if isinstance(b, np.ndarray):
            dev_bits = torch.from_numpy(np.ascontiguousarray(b.astype(np.uint32).view(np.int32))).cuda()
        else:   # device words: 32-bit, contiguous, on the GPU
            _tensors((b, "mask.bits", (torch.int32, torch.uint32), None, False))
            dev_bits = b
    d = _mask_desc(m, mask, dev_bits, cu_seqlens_q)
    h = ctypes.c_void_p()
    if backward:   # attn_plan_bwd(): forward and backward work lists
        _check(lib().attn_plan_bwd(ctypes.byref(pr), ctypes.byref(d), _stream(stream), ctypes.byref(h)),
               "attn_plan_bwd")
    else:
        _check(lib().attn_plan(ctypes.byref(pr), ctypes.byref(d), _stream(stream), ctypes.byref(h)), "attn_plan")
    total_q = int(np.asarray(cu_seqlens_q)[-1])
    kv_rows = int(np.asarray(cu_seqlens_k)[-1]) if cu_seqlens_k is not None else int(num_pages) * int(page_size)
    return Plan(h.value, page_table, hq, head_dim, total_q, hkv=hkv, kv_rows=kv_rows)


def _tensors(*specs):
    """Device pointers of tensor arguments after checking them. Each spec is (tensor, name,
    dtypes, least numel or None, optional): a torch tensor of one of ``dtypes``, contiguous,
    with at least that many elements; then every one must be on a CUDA device. The C ABI
    takes bare pointers and cannot see sizes; a wrong tensor would be read or written out
    of bounds, so it is refused here."""
    import torch
    for t, name, dtypes, numel, optional in specs:
        if t is None:
            if optional:
                continue
            raise ValueError(f"{name} is required")
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch tensor")
        if t.dtype not in dtypes:
            raise TypeError(f"{name} must be {' or '.join(str(d) for d in dtypes)}, not {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if numel is not None and t.numel() < numel:
            raise ValueError(f"{name} has {t.numel()} elements; the plan needs {numel}")
    for t, name, *_ in specs:
        if t is not None and not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
    return [None if t is None else t.data_ptr() for t, *_ in specs]


def _bf16():
    import torch
    return (torch.bfloat16,)


def _f32():
    import torch
    return (torch.float32,)


def _bytes():
    import torch
    return (torch.uint8, torch.float8_e4m3fn)


def _sizes(plan: Plan):
    """(q / out elements, k / v elements, lse elements) of a plan; None where unknown."""
    qn = plan.total_q * plan.hq * plan.head_dim
    kn = plan.kv_rows * plan.hkv * plan.head_dim if plan.kv_rows is not None and plan.hkv else None
    return qn, kn, plan.total_q * plan.hq


def attn_masked_fwd(plan: Plan, q, k, v, out, lse=None, stream=None) -> None:
    """attn_masked_fwd(): enqueue the forward on ``stream`` (default: torch's current stream).
    q, out: bf16 [total_q, hq, d]; k, v: bf16 [total_k, hkv, d] or paged caches; lse: fp32
    [total_q, hq] or None."""
    qn, kn, ln = _sizes(plan)
    b, f = _bf16(), _f32()
    args = _tensors((q, "q", b, qn, False), (k, "k", b, kn, False), (v, "v", b, kn, False),
                    (out, "out", b, qn, False), (lse, "lse", f, ln, True))
    _check(lib().attn_masked_fwd(plan.handle, *args, _stream(stream)), "attn_masked_fwd")


def attn_masked_bwd(plan: Plan, q, k, v, out, lse, dout, dq, dk, dv, stream=None, dlse=None) -> None:
    """attn_masked_bwd(): enqueue dq, dk, dv for the gradient dout of out and, optionally,
    dlse of lse (plan from attn_plan(..., backward=True)). Shapes as in attn_masked_fwd;
    dq like q, dk / dv like k / v, dout like out, dlse like lse."""
    qn, kn, ln = _sizes(plan)
    b, f = _bf16(), _f32()
    args = _tensors((q, "q", b, qn, False), (k, "k", b, kn, False), (v, "v", b, kn, False),
                    (out, "out", b, qn, False), (lse, "lse", f, ln, False), (dout, "dout", b, qn, False),
                    (dlse, "dlse", f, ln, True), (dq, "dq", b, qn, False), (dk, "dk", b, kn, False),
                    (dv, "dv", b, kn, False))
    _check(lib().attn_masked_bwd(plan.handle, *args, _stream(stream)), "attn_masked_bwd")


def attn_plan_get_tile_classes(plan: Plan) -> np.ndarray:
    n = ctypes.c_size_t()
    _check(lib().attn_plan_get_tile_classes(plan.handle, None, 0, ctypes.byref(n)), "attn_plan_get_tile_classes")
    out = np.zeros(n.value, dtype=np.uint8)
    _check(lib().attn_plan_get_tile_classes(plan.handle, out.ctypes.data, n.value, None),
           "attn_plan_get_tile_classes")
    return out


def attn_plan_get_stats(plan: Plan) -> dict:
    s = attn_plan_stats_t()
    _check(lib().attn_plan_get_stats(plan.handle, ctypes.byref(s)), "attn_plan_get_stats")
    return {n: getattr(s, n) for n, _ in attn_plan_stats_t._fields_}


def attn_plan_check_status(plan: Plan, stream=None) -> int:
    """Synchronises the stream; returns the status code (0 ok, 6 a bounded wait expired)."""
    return int(lib().attn_plan_check_status(plan.handle, _stream(stream)))


def attn_plan_set_debug(plan: Plan, flags: int, timeout_ns: int = 0) -> None:
    _check(lib().attn_plan_set_debug(plan.handle, int(flags), int(timeout_ns)), "attn_plan_set_debug")


def attn_plan_destroy(plan: Plan) -> None:
    if plan.handle:
        h, plan.handle = plan.handle, None
        _check(lib().attn_plan_destroy(h), "attn_plan_destroy")


def attn_plan_dry_run(*, hq: int, hkv: int, head_dim: int, cu_seqlens_q, mask, num_sms: int = 148,
                      cu_seqlens_k=None, kv_lens=None, page_size: int = 0, max_pages_per_seq: int = 0,
                      num_pages: int = 0, kv_splits: int = 0, q_rows=None) -> dict:
    """Host-only attn_plan() (analytic kinds) for a GPU of ``num_sms`` SMs: the plan statistics."""
    m = _Marshal()
    pr = _problem(m, hq=hq, hkv=hkv, head_dim=head_dim, cu_seqlens_q=cu_seqlens_q, cu_seqlens_k=cu_seqlens_k,
                  kv_lens=kv_lens, kv_splits=kv_splits, q_rows=q_rows)
    if kv_lens is not None:
        pr.page_size, pr.max_pages_per_seq, pr.num_pages = page_size, max_pages_per_seq, num_pages
    d = _mask_desc(m, mask, cu_seqlens_q=cu_seqlens_q)
    st = attn_plan_stats_t()
    _check(lib().attn_plan_dry_run(ctypes.byref(pr), ctypes.byref(d), int(num_sms), ctypes.byref(st)),
           "attn_plan_dry_run")
    return {n: getattr(st, n) for n, _ in attn_plan_stats_t._fields_}


def attn_plan_bwd_dry_run(*, hq: int, hkv: int, head_dim: int, cu_seqlens_q, mask, num_sms: int = 148,
                          cu_seqlens_k=None, kv_lens=None, page_size: int = 0, max_pages_per_seq: int = 0,
                          num_pages: int = 0) -> dict:
    """Host-only attn_plan_bwd() work lists (analytic kinds) for a GPU of ``num_sms`` SMs: their statistics."""
    m = _Marshal()
    pr = _problem(m, hq=hq, hkv=hkv, head_dim=head_dim, cu_seqlens_q=cu_seqlens_q, cu_seqlens_k=cu_seqlens_k,
                  kv_lens=kv_lens)
    if kv_lens is not None:
        pr.page_size, pr.max_pages_per_seq, pr.num_pages = page_size, max_pages_per_seq, num_pages
    d = _mask_desc(m, mask, cu_seqlens_q=cu_seqlens_q)
    st = attn_bwd_stats_t()
    _check(lib().attn_plan_bwd_dry_run(ctypes.byref(pr), ctypes.byref(d), int(num_sms), ctypes.byref(st)),
           "attn_plan_bwd_dry_run")
    return {n: getattr(st, n) for n, _ in attn_bwd_stats_t._fields_}


def attn_classify_host(*, hq: int, hkv: int, head_dim: int, cu_seqlens_q, mask, cu_seqlens_k=None, kv_lens=None,
                       page_size: int = 0, max_pages_per_seq: int = 0, num_pages: int = 0, kv_splits: int = 0):
    """Host-only tile classes (analytic kinds). Returns (classes uint8, unmasked pairs per head)."""
    m = _Marshal()
    pr = _problem(m, hq=hq, hkv=hkv, head_dim=head_dim, cu_seqlens_q=cu_seqlens_q, cu_seqlens_k=cu_seqlens_k,
                  kv_lens=kv_lens, kv_splits=kv_splits)
    if kv_lens is not None:
        pr.page_size, pr.max_pages_per_seq, pr.num_pages = page_size, max_pages_per_seq, num_pages
    d = _mask_desc(m, mask, cu_seqlens_q=cu_seqlens_q)
    n, pairs = ctypes.c_size_t(), ctypes.c_int64()
    _check(lib().attn_classify_host(ctypes.byref(pr), ctypes.byref(d), None, 0, ctypes.byref(n), ctypes.byref(pairs)),
           "attn_classify_host")
    out = np.zeros(n.value, dtype=np.uint8)
    _check(lib().attn_classify_host(ctypes.byref(pr), ctypes.byref(d), out.ctypes.data, n.value, None, None),
           "attn_classify_host")
    return out, int(pairs.value)


def attn_masked_fwd_noalloc(*, hq: int, hkv: int, head_dim: int, cu_seqlens_q, mask, q, k, v, out, lse=None,
                            cu_seqlens_k=None, kv_lens=None, page_table=None, page_size: int = 0,
                            num_pages: int = 0, scale: float = 0.0, stream=None) -> None:
    """attn_masked_fwd_noalloc(): plan + forward in one call without any device allocation.

    For callers that may not allocate device memory (e.g. a runtime that owns every device
    allocation through its own pool): the plan goes into a fixed 32 MiB array inside the
    library instead of a cudaMalloc'd workspace. Calls that overlap on the GPU race on that
    array; keep them on one stream. CUSTOM masks are not accepted here. An in-kernel wait
    that expires leaves the rows it did not compute with lse = NaN (lse is filled with NaN
    first); pass lse to see it."""
    _check_page_table(page_table, cu_seqlens_q)
    m = _Marshal()
    pr = _problem(m, hq=hq, hkv=hkv, head_dim=head_dim, cu_seqlens_q=cu_seqlens_q, cu_seqlens_k=cu_seqlens_k,
                  kv_lens=kv_lens, page_table=page_table, page_size=page_size, num_pages=num_pages, scale=scale)
    d = _mask_desc(m, mask, cu_seqlens_q=cu_seqlens_q)
    total_q = int(np.asarray(cu_seqlens_q)[-1])
    kv_rows = int(np.asarray(cu_seqlens_k)[-1]) if cu_seqlens_k is not None else int(num_pages) * int(page_size)
    qn, kn = total_q * hq * head_dim, kv_rows * hkv * head_dim
    b = _bf16()
    # a missing tensor is left to the C side, which reports it after its own size limit
    args = _tensors((q, "q", b, qn, True), (k, "k", b, kn, True), (v, "v", b, kn, True), (out, "out", b, qn, True),
                    (lse, "lse", _f32(), total_q * hq, True))
    _check(lib().attn_masked_fwd_noalloc(ctypes.byref(pr), ctypes.byref(d), *args, _stream(stream)),
           "attn_masked_fwd_noalloc")


def attn_test_noalloc_debug(flags: int, timeout_ns: int) -> None:
    """Test hook: debug flags / wait limit of the following attn_masked_fwd_noalloc() calls."""
    _check(lib().attn_test_noalloc_debug(int(flags), int(timeout_ns)), "attn_test_noalloc_debug")


def attn_test_exp2_poly(x, y, stream=None) -> None:
    """Test hook: y = 2^x by the forward kernel's polynomial exp2 (device fp32 tensors)."""
    _check(lib().attn_test_exp2_poly(_ptr(x), _ptr(y), int(x.numel()), _stream(stream)), "attn_test_exp2_poly")


def attn_status_string(status: int) -> str:
    return lib().attn_status_string(int(status)).decode()


def forward(plan: Plan, q, k, v, stream=None):
    """Allocate out / lse with torch and run attn_masked_fwd (convenience)."""
    import torch
    out = torch.empty(q.shape[0], plan.hq, plan.head_dim, dtype=torch.bfloat16, device=q.device)
    lse = torch.empty(q.shape[0], plan.hq, dtype=torch.float32, device=q.device)
    attn_masked_fwd(plan, q, k, v, out, lse, stream)
    return out, lse


def backward(plan: Plan, q, k, v, out, lse, dout, stream=None, dlse=None):
    """Allocate dq / dk / dv with torch and run attn_masked_bwd (convenience)."""
    import torch
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    attn_masked_bwd(plan, q, k, v, out, lse, dout, dq, dk, dv, stream, dlse=dlse)
    return dq, dk, dv


def attn_fp8_transpose_v(plan: Plan, v8, vt8, ldv: int, stream=None) -> None:
    """attn_fp8_transpose_v(): e4m3 V [total_k, hkv, d] -> vt [hkv, d, ldv] (uint8 tensors)."""
    by = _bytes()
    pv, pvt = _tensors((v8, "v8", by, None, False), (vt8, "vt8", by, None, False))
    _check(lib().attn_fp8_transpose_v(plan.handle, pv, pvt, int(ldv), _stream(stream)), "attn_fp8_transpose_v")


def attn_masked_fwd_fp8(plan: Plan, q8, k8, vt8, ldv: int, q_scale: float, k_scale: float, v_scale: float, out,
                        lse=None, stream=None) -> None:
    """attn_masked_fwd_fp8(): e4m3 q, k (uint8 tensors) and transposed v with per-tensor scales."""
    by = _bytes()
    pq, pk, pvt, po, pl = _tensors((q8, "q8", by, None, False), (k8, "k8", by, None, False),
                                   (vt8, "vt8", by, None, False), (out, "out", _bf16(), None, False),
                                   (lse, "lse", _f32(), None, True))
    _check(lib().attn_masked_fwd_fp8(plan.handle, pq, pk, pvt, int(ldv), float(q_scale), float(k_scale),
                                     float(v_scale), po, pl, _stream(stream)), "attn_masked_fwd_fp8")


def attn_test_transpose_mask_tile(tile_words: np.ndarray) -> np.ndarray:
    """Test hook: the planner's transposition of one 2 KiB mask tile (512 uint32 words)."""
    src = np.ascontiguousarray(tile_words, dtype=np.uint32).reshape(512)
    dst = np.zeros(512, dtype=np.uint32)
    _check(lib().attn_test_transpose_mask_tile(src.ctypes.data, dst.ctypes.data), "attn_test_transpose_mask_tile")
    return dst
