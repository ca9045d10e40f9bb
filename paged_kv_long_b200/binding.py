"""ctypes binding of ``libpa.so`` — argument marshalling only.

Every step of the attention runs in the library's CUDA kernels; this module checks the
torch tensors it is given (device, dtype, shape, contiguity) and passes their device pointers
and the caller's current CUDA stream across the C ABI declared in ``include/pa.h``. There is
no CPU fallback: if the library is missing or a tensor is not on a CUDA device, it raises.
"""
from __future__ import annotations

import ctypes
import math
import os

PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(PKG, "libpa.so")

PA_F16, PA_BF16 = 0, 1
POLICIES = {"makespan": 0, "cores": 1, "legacy": 2, "balanced": 3}
PA_POLICY_BALANCED = 3
STATUS = {0: "PA_OK", -1: "PA_ERR_INVALID_ARG", -2: "PA_ERR_UNSUPPORTED", -3: "PA_ERR_WORKSPACE",
          -4: "PA_ERR_CUDA", -5: "PA_ERR_TIMEOUT", -6: "PA_ERR_PAGE_INDEX"}
EXPORTED = ("pa_plan", "pa_prefill", "pa_combine", "pa_prefill_noalloc", "pa_device_error",
            "pa_set_wait_timeout_ns",
            "pa_selftest_timeout", "pa_status_string", "pa_cores_policy_splits",
            "pa_legacy_policy_splits", "pa_schedule_items", "pa_kv_append", "pa_pieces",
            "pa_decode_plan", "pa_decode", "pa_batch_plan", "pa_batch_prefill",
            "pa_batch_combine", "pa_batch_schedule_items", "pa_kv_publish")


class PaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class Plan(ctypes.Structure):
    """Mirror of ``pa_plan_t``."""
    _fields_ = [
        ("num_sms", ctypes.c_int32), ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32), ("group", ctypes.c_int32),
        ("chunk_rows", ctypes.c_int32), ("q_tiles", ctypes.c_int32), ("splits", ctypes.c_int32),
        ("paged", ctypes.c_int32), ("dtype", ctypes.c_int32), ("policy", ctypes.c_int32),
        ("ctas_per_unit", ctypes.c_int32), ("batch", ctypes.c_int32), ("hist_len", ctypes.c_int64),
        ("units", ctypes.c_int64), ("scale", ctypes.c_float),
        ("est_us", ctypes.c_float), ("ws_bytes", ctypes.c_uint64),
    ]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


_lib = None


def lib_path() -> str:
    return _LIB_PATH


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load libpa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or _LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"libpa.so not built at {p}: run `python -m paged_kv_long_b200.build`")
    lib = ctypes.CDLL(p)
    vp, i32, i64, u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64
    lib.pa_plan.argtypes = [i32, i32, i32, i32, i32, i32, i64, i32, ctypes.c_float, i32, i32, i32,
                            ctypes.POINTER(Plan)]
    lib.pa_plan.restype = i32
    lib.pa_prefill.argtypes = [ctypes.POINTER(Plan), vp, vp, vp, vp, i64, i64, i32, vp, vp, u64, vp]
    lib.pa_prefill.restype = i32
    lib.pa_combine.argtypes = [ctypes.POINTER(Plan), vp, u64, vp, vp]
    lib.pa_combine.restype = i32
    lib.pa_prefill_noalloc.argtypes = [ctypes.POINTER(Plan), vp, vp, vp, vp, i64, i64, i32, vp, vp]
    lib.pa_prefill_noalloc.restype = i32
    lib.pa_device_error.argtypes = [ctypes.POINTER(ctypes.c_int), i32]
    lib.pa_device_error.restype = i32
    lib.pa_set_wait_timeout_ns.argtypes = [u64]
    lib.pa_set_wait_timeout_ns.restype = None
    lib.pa_selftest_timeout.argtypes = [u64, vp]
    lib.pa_selftest_timeout.restype = i32
    lib.pa_status_string.argtypes = [i32]
    lib.pa_status_string.restype = ctypes.c_char_p
    lib.pa_cores_policy_splits.argtypes = [i32, i32, i32]
    lib.pa_cores_policy_splits.restype = i32
    lib.pa_legacy_policy_splits.argtypes = [i32, i32]
    lib.pa_legacy_policy_splits.restype = i32
    lib.pa_schedule_items.argtypes = [ctypes.POINTER(Plan), ctypes.POINTER(ctypes.c_int32), i32]
    lib.pa_schedule_items.restype = i32
    lib.pa_kv_append.argtypes = [i32, i32, i32, i32, vp, vp, vp, vp, vp, i64, i64, i32, vp]
    lib.pa_kv_append.restype = i32
    lib.pa_pieces.argtypes = [i32, i64, i32, ctypes.POINTER(ctypes.c_int32), i32]
    lib.pa_pieces.restype = i32
    lib.pa_decode_plan.argtypes = [i32, i32, i32, i32, i32, i32, i64, i32, ctypes.c_float, i32,
                                   ctypes.POINTER(Plan)]
    lib.pa_decode_plan.restype = i32
    lib.pa_decode.argtypes = [ctypes.POINTER(Plan), vp, vp, vp, vp, i32, vp, i64, vp, vp, u64, vp]
    lib.pa_decode.restype = i32
    lib.pa_batch_plan.argtypes = [i32, i32, i32, i32, i32, i32, vp, vp, i32, ctypes.c_float,
                                  ctypes.POINTER(Plan)]
    lib.pa_batch_plan.restype = i32
    lib.pa_batch_prefill.argtypes = [ctypes.POINTER(Plan), vp, vp, vp, vp, vp, vp, i32, i64, vp,
                                     vp, u64, vp]
    lib.pa_batch_prefill.restype = i32
    lib.pa_batch_combine.argtypes = [ctypes.POINTER(Plan), vp, vp, vp, u64, vp, vp]
    lib.pa_batch_combine.restype = i32
    lib.pa_batch_schedule_items.argtypes = [ctypes.POINTER(Plan), vp, vp,
                                            ctypes.POINTER(ctypes.c_int32), i32]
    lib.pa_batch_schedule_items.restype = i32
    lib.pa_kv_publish.argtypes = [i32, i32, i32, i32, vp, vp, vp, vp, vp, i64, i64, i32, vp]
    lib.pa_kv_publish.restype = i32
    if path is None:
        _lib = lib
    return lib


def _check(status: int, where: str):
    if status != 0:
        raise PaError(status, where)


def _dtype_code(dtype) -> int:
    import torch
    if dtype in ("f16", torch.float16):
        return PA_F16
    if dtype in ("bf16", torch.bfloat16):
        return PA_BF16
    raise ValueError(f"unsupported dtype {dtype}")


def plan(n_q_heads: int, n_kv_heads: int, head_dim: int, page_size: int, chunk_rows: int,
         hist_len: int, dtype="bf16", scale: float = 0.0, splits: int = 0,
         policy: str = "makespan", paged: bool = True, num_sms: int | None = None) -> Plan:
    """pa_plan: split count and workspace for one piece (host only)."""
    if num_sms is None:
        import torch
        num_sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    p = Plan()
    st = load_library().pa_plan(num_sms, n_q_heads, n_kv_heads, head_dim, page_size, chunk_rows,
                                hist_len, _dtype_code(dtype), scale, splits, POLICIES[policy],
                                1 if paged else 0, ctypes.byref(p))
    _check(st, "pa_plan")
    return p


def schedule_items(p: Plan):
    """pa_schedule_items: the work items of a balanced plan as an int32 array [n, 4] of
    (row block, kt0, kt1, workspace slot or -1); empty for other plans."""
    import numpy as np
    lib = load_library()
    n = lib.pa_schedule_items(ctypes.byref(p), None, 0)
    _check(0 if n >= 0 else n, "pa_schedule_items")
    buf = (ctypes.c_int32 * max(4 * n, 1))()
    lib.pa_schedule_items(ctypes.byref(p), buf, n)
    return np.frombuffer(buf, dtype=np.int32)[:4 * n].reshape(n, 4).copy()


def pieces(chunk_rows: int, hist_len: int, log2_budget: int = 25) -> list[int]:
    """pa_pieces: the pages' cut of a chunk into pieces (rows of each, in order)."""
    lib = load_library()
    n = lib.pa_pieces(chunk_rows, hist_len, log2_budget, None, 0)
    _check(0 if n >= 0 else n, "pa_pieces")
    buf = (ctypes.c_int32 * max(n, 1))()
    lib.pa_pieces(chunk_rows, hist_len, log2_budget, buf, n)
    return list(buf)[:n]


def kv_append(k_new, v_new, k_pool, v_pool, page_table, hist_len: int, stream=None):
    """pa_kv_append: write the chunk's K/V rows [R, Hkv, D] into the page pools
    [num_pages, PS, Hkv, D] at positions hist_len.. through page_table (see include/pa.h)."""
    import torch
    if k_new.dtype not in (torch.float16, torch.bfloat16):
        raise TypeError("k_new must be float16 or bfloat16")
    dt = k_new.dtype
    _require_cuda(k_new, "k_new", dt)
    if k_new.dim() != 3:
        raise ValueError("k_new must be [R, Hkv, D]")
    R, Hkv, D = k_new.shape
    _require_cuda(v_new, "v_new", dt, (R, Hkv, D))
    _require_cuda(k_pool, "k_pool", dt)
    if k_pool.dim() != 4 or tuple(k_pool.shape[2:]) != (Hkv, D):
        raise ValueError("k_pool must be [num_pages, page_size, Hkv, D]")
    _require_cuda(v_pool, "v_pool", dt, tuple(k_pool.shape))
    _require_cuda(page_table, "page_table", torch.int32)
    PS = k_pool.shape[1]
    if page_table.numel() < math.ceil((hist_len + R) / PS):
        raise ValueError("page_table is shorter than ceil((hist_len+R)/page_size)")
    st = load_library().pa_kv_append(Hkv, D, PS, _dtype_code(dt), k_new.data_ptr(),
                                     v_new.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(),
                                     page_table.data_ptr(), k_pool.shape[0], hist_len, R,
                                     _stream_ptr(stream))
    _check(st, "pa_kv_append")


def kv_publish(k_staged, v_staged, k_pool, v_pool, page_table, first_pos: int, rows: int,
               stream=None):
    """pa_kv_publish: copy staged rows [first_pos, first_pos + rows) of the contiguous staging
    buffers [T, Hkv, D] to their pages (see include/pa.h)."""
    import torch
    if k_staged.dtype not in (torch.float16, torch.bfloat16):
        raise TypeError("k_staged must be float16 or bfloat16")
    dt = k_staged.dtype
    _require_cuda(k_staged, "k_staged", dt)
    if k_staged.dim() != 3:
        raise ValueError("k_staged must be [T, Hkv, D]")
    T, Hkv, D = k_staged.shape
    if first_pos < 0 or rows < 0 or first_pos + rows > T:
        raise ValueError("rows [first_pos, first_pos + rows) must lie in the staging buffer")
    _require_cuda(v_staged, "v_staged", dt, (T, Hkv, D))
    _require_cuda(k_pool, "k_pool", dt)
    if k_pool.dim() != 4 or tuple(k_pool.shape[2:]) != (Hkv, D):
        raise ValueError("k_pool must be [num_pages, page_size, Hkv, D]")
    _require_cuda(v_pool, "v_pool", dt, tuple(k_pool.shape))
    _require_cuda(page_table, "page_table", torch.int32)
    PS = k_pool.shape[1]
    if page_table.numel() < math.ceil((first_pos + rows) / PS):
        raise ValueError("page_table is shorter than ceil((first_pos+rows)/page_size)")
    st = load_library().pa_kv_publish(Hkv, D, PS, _dtype_code(dt), k_staged.data_ptr(),
                                      v_staged.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(),
                                      page_table.data_ptr(), k_pool.shape[0], first_pos, rows,
                                      _stream_ptr(stream))
    _check(st, "pa_kv_publish")


def _stream_ptr(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _require_cuda(t, name, dtype=None, shape=None):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _torch_dtype(p: Plan):
    import torch
    return torch.bfloat16 if p.dtype == PA_BF16 else torch.float16


def workspace(p: Plan, device=None):
    """A workspace tensor of plan.ws_bytes (fp32), or None when no split is used."""
    import torch
    if p.ws_bytes == 0:
        return None
    return torch.empty(p.ws_bytes // 4, dtype=torch.float32, device=device or "cuda")


def prefill(p: Plan, q, k_pool, v_pool, page_table, out, ws=None, stream=None):
    """pa_prefill on torch tensors (see include/pa.h for layouts)."""
    import torch
    dt = _torch_dtype(p)
    R, Hq, Hkv, D = p.chunk_rows, p.n_q_heads, p.n_kv_heads, p.head_dim
    _require_cuda(q, "q", dt, (R, Hq, D))
    _require_cuda(k_pool, "k_pool", dt)
    _require_cuda(v_pool, "v_pool", dt, tuple(k_pool.shape))
    if p.paged:
        if k_pool.dim() != 4 or tuple(k_pool.shape[1:]) != (p.page_size, Hkv, D):
            raise ValueError("k_pool must be [num_pages, page_size, Hkv, D]")
        _require_cuda(page_table, "page_table", torch.int32)
        if page_table.numel() < math.ceil((p.hist_len + R) / p.page_size):
            raise ValueError("page_table is shorter than ceil((H+R)/page_size)")
        num_pages, tab = k_pool.shape[0], page_table.data_ptr()
    else:
        if k_pool.dim() != 3 or tuple(k_pool.shape) != (p.hist_len + R, Hkv, D):
            raise ValueError("contiguous k/v must be [H+R, Hkv, D]")
        num_pages, tab = 0, None
    out_ptr, ws_ptr, ws_bytes = None, None, 0
    if p.splits == 1 or p.policy == PA_POLICY_BALANCED:
        _require_cuda(out, "out", torch.float32, (R, Hq, D))
        out_ptr = out.data_ptr()
    if p.ws_bytes > 0:
        _require_cuda(ws, "ws", torch.float32)
        ws_ptr, ws_bytes = ws.data_ptr(), ws.numel() * 4
    st = load_library().pa_prefill(ctypes.byref(p), q.data_ptr(), k_pool.data_ptr(),
                                   v_pool.data_ptr(), tab, num_pages, p.hist_len, R, out_ptr,
                                   ws_ptr, ws_bytes, _stream_ptr(stream))
    _check(st, "pa_prefill")


def combine(p: Plan, ws, out, stream=None):
    """pa_combine: merge split partials into out (no-op when there are none)."""
    import torch
    if p.ws_bytes == 0:
        return
    _require_cuda(ws, "ws", torch.float32)
    _require_cuda(out, "out", torch.float32, (p.chunk_rows, p.n_q_heads, p.head_dim))
    st = load_library().pa_combine(ctypes.byref(p), ws.data_ptr(), ws.numel() * 4, out.data_ptr(),
                                   _stream_ptr(stream))
    _check(st, "pa_combine")


def prefill_combine(p: Plan, q, k_pool, v_pool, page_table, out=None, ws=None, stream=None):
    """pa_prefill followed by pa_combine; allocates out / ws with torch when not given."""
    import torch
    if out is None:
        out = torch.empty((p.chunk_rows, p.n_q_heads, p.head_dim), dtype=torch.float32,
                          device=q.device)
    if p.ws_bytes > 0 and ws is None:
        ws = workspace(p, q.device)
    prefill(p, q, k_pool, v_pool, page_table, out, ws, stream)
    combine(p, ws, out, stream)
    return out


def prefill_noalloc(p: Plan, q, k_pool, v_pool, page_table, out, stream=None):
    """pa_prefill_noalloc: prefill + combine with the library's own device scratch (for
    callers that cannot allocate device memory; see include/pa.h)."""
    import torch
    dt = _torch_dtype(p)
    R, Hq, D = p.chunk_rows, p.n_q_heads, p.head_dim
    _require_cuda(q, "q", dt, (R, Hq, D))
    _require_cuda(k_pool, "k_pool", dt)
    _require_cuda(v_pool, "v_pool", dt, tuple(k_pool.shape))
    _require_cuda(out, "out", torch.float32, (R, Hq, D))
    if p.paged:
        _require_cuda(page_table, "page_table", torch.int32)
        num_pages, tab = k_pool.shape[0], page_table.data_ptr()
    else:
        num_pages, tab = 0, None
    st = load_library().pa_prefill_noalloc(ctypes.byref(p), q.data_ptr(), k_pool.data_ptr(),
                                           v_pool.data_ptr(), tab, num_pages, p.hist_len, R,
                                           out.data_ptr(), _stream_ptr(stream))
    _check(st, "pa_prefill_noalloc")


def decode_plan(n_q_heads: int, n_kv_heads: int, head_dim: int, page_size: int, batch: int,
                max_seq_len: int, dtype="bf16", scale: float = 0.0, splits: int = 0,
                num_sms: int | None = None) -> Plan:
    """pa_decode_plan: split count and workspace for one batched decode step (host only)."""
    if num_sms is None:
        import torch
        num_sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    p = Plan()
    st = load_library().pa_decode_plan(num_sms, n_q_heads, n_kv_heads, head_dim, page_size, batch,
                                       max_seq_len, _dtype_code(dtype), scale, splits,
                                       ctypes.byref(p))
    _check(st, "pa_decode_plan")
    return p


def decode(p: Plan, q, k_pool, v_pool, block_table, seq_lens, out=None, ws=None, stream=None):
    """pa_decode followed by pa_combine: one query token per sequence against that sequence's
    paged keys. q [B, Hq, D]; block_table int32 [B, max_pages]; seq_lens int32 [B] (keys of
    each sequence, the new token's included). Returns out fp32 [B, Hq, D]."""
    import torch
    dt = _torch_dtype(p)
    B, Hq, Hkv, D, PS = p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim, p.page_size
    _require_cuda(q, "q", dt, (B, Hq, D))
    _require_cuda(k_pool, "k_pool", dt)
    _require_cuda(v_pool, "v_pool", dt, tuple(k_pool.shape))
    if k_pool.dim() != 4 or tuple(k_pool.shape[1:]) != (PS, Hkv, D):
        raise ValueError("k_pool must be [num_pages, page_size, Hkv, D]")
    _require_cuda(block_table, "block_table", torch.int32)
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be [batch, max_pages]")
    _require_cuda(seq_lens, "seq_lens", torch.int32, (B,))
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
    _require_cuda(out, "out", torch.float32, (B, Hq, D))
    ws_ptr, ws_bytes = None, 0
    if p.ws_bytes > 0:
        if ws is None:
            ws = workspace(p, q.device)
        _require_cuda(ws, "ws", torch.float32)
        ws_ptr, ws_bytes = ws.data_ptr(), ws.numel() * 4
    lib = load_library()
    st = lib.pa_decode(ctypes.byref(p), q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(),
                       block_table.data_ptr(), block_table.stride(0), seq_lens.data_ptr(),
                       k_pool.shape[0], out.data_ptr(), ws_ptr, ws_bytes, _stream_ptr(stream))
    _check(st, "pa_decode")
    if p.ws_bytes > 0:
        _check(lib.pa_combine(ctypes.byref(p), ws_ptr, ws_bytes, out.data_ptr(),
                              _stream_ptr(stream)), "pa_combine")
    return out


class BatchPlan:
    """A batched plan with the host length arrays it was made from (pa_batch_plan)."""

    def __init__(self, plan: Plan, q_lens, hist_lens):
        import numpy as np
        self.plan = plan
        self.q_lens = np.ascontiguousarray(q_lens, dtype=np.int32)
        self.hist_lens = np.ascontiguousarray(hist_lens, dtype=np.int64)

    def _arrays(self):
        return self.q_lens.ctypes.data, self.hist_lens.ctypes.data


def batch_plan(n_q_heads: int, n_kv_heads: int, head_dim: int, page_size: int, q_lens,
               hist_lens, dtype="bf16", scale: float = 0.0,
               num_sms: int | None = None) -> BatchPlan:
    """pa_batch_plan: the balanced schedule of a batch of chunks (host only)."""
    import numpy as np
    if num_sms is None:
        import torch
        num_sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    q_lens = np.ascontiguousarray(q_lens, dtype=np.int32)
    hist_lens = np.ascontiguousarray(hist_lens, dtype=np.int64)
    if q_lens.shape != hist_lens.shape or q_lens.ndim != 1:
        raise ValueError("q_lens and hist_lens must be 1-D of the same length")
    p = Plan()
    st = load_library().pa_batch_plan(num_sms, n_q_heads, n_kv_heads, head_dim, page_size,
                                      len(q_lens), q_lens.ctypes.data, hist_lens.ctypes.data,
                                      _dtype_code(dtype), scale, ctypes.byref(p))
    _check(st, "pa_batch_plan")
    return BatchPlan(p, q_lens, hist_lens)


def batch_schedule_items(bp: BatchPlan):
    """pa_batch_schedule_items: int32 [n, 4] of (global row block, kt0, kt1, slot or -1)."""
    import numpy as np
    lib = load_library()
    ql, hl = bp._arrays()
    n = lib.pa_batch_schedule_items(ctypes.byref(bp.plan), ql, hl, None, 0)
    if n < 0:
        raise PaError(n, "pa_batch_schedule_items")
    out = np.zeros((max(n, 1), 4), dtype=np.int32)
    lib.pa_batch_schedule_items(ctypes.byref(bp.plan), ql, hl,
                                out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), n)
    return out[:n]


def batch_prefill(bp: BatchPlan, q, k_pool, v_pool, block_table, out=None, ws=None,
                  stream=None):
    """pa_batch_prefill followed by pa_batch_combine. q [sum q_lens, Hq, D] (the sequences'
    chunks packed in order); block_table int32 [batch, max_pages]. Returns out fp32
    [sum q_lens, Hq, D]."""
    import torch
    p = bp.plan
    dt = _torch_dtype(p)
    rows, Hq, Hkv, D, PS = p.chunk_rows, p.n_q_heads, p.n_kv_heads, p.head_dim, p.page_size
    _require_cuda(q, "q", dt, (rows, Hq, D))
    _require_cuda(k_pool, "k_pool", dt)
    _require_cuda(v_pool, "v_pool", dt, tuple(k_pool.shape))
    if k_pool.dim() != 4 or tuple(k_pool.shape[1:]) != (PS, Hkv, D):
        raise ValueError("k_pool must be [num_pages, page_size, Hkv, D]")
    _require_cuda(block_table, "block_table", torch.int32)
    if block_table.dim() != 2 or block_table.shape[0] != p.batch:
        raise ValueError("block_table must be [batch, max_pages]")
    if out is None:
        out = torch.empty((rows, Hq, D), dtype=torch.float32, device=q.device)
    _require_cuda(out, "out", torch.float32, (rows, Hq, D))
    ws_ptr, ws_bytes = None, 0
    if p.ws_bytes > 0:
        if ws is None:
            ws = workspace(p, q.device)
        _require_cuda(ws, "ws", torch.float32)
        ws_ptr, ws_bytes = ws.data_ptr(), ws.numel() * 4
    ql, hl = bp._arrays()
    lib = load_library()
    st = lib.pa_batch_prefill(ctypes.byref(p), ql, hl, q.data_ptr(), k_pool.data_ptr(),
                              v_pool.data_ptr(), block_table.data_ptr(), block_table.stride(0),
                              k_pool.shape[0], out.data_ptr(), ws_ptr, ws_bytes,
                              _stream_ptr(stream))
    _check(st, "pa_batch_prefill")
    _check(lib.pa_batch_combine(ctypes.byref(p), ql, hl, ws_ptr, ws_bytes, out.data_ptr(),
                                _stream_ptr(stream)), "pa_batch_combine")
    return out


def device_error(reset: bool = True) -> tuple[int, int]:
    """(status, flags) of the library's device-side error word (synchronises the device)."""
    flags = ctypes.c_int(0)
    st = load_library().pa_device_error(ctypes.byref(flags), 1 if reset else 0)
    return st, flags.value


def set_wait_timeout_ns(ns: int):
    load_library().pa_set_wait_timeout_ns(ns)


def selftest_timeout(timeout_ns: int, stream=None):
    _check(load_library().pa_selftest_timeout(timeout_ns, _stream_ptr(stream)), "pa_selftest_timeout")
