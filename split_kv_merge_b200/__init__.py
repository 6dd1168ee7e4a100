"""Python binding of libsplitkv (paged attention + split-KV + exact LSE merge on B200).

Argument marshalling only: every step of the attention path runs in the CUDA kernels of
``libsplitkv.so``.  Device buffers are torch CUDA tensors (PyTorch is used for memory and
streams); host arrays are numpy.  Importing this package without the built library raises --
there is no fallback path.

Functions mirror the C ABI in include/splitkv.h:
``plan_paged``, ``paged_attn_fwd``, ``pod_attn_fwd``, ``plan_mla``, ``mla_decode_fwd``, ``merge_states``,
``paged_kv_gather``, ``mla_splice``, ``mla_fold_ratio``, ``status_str``, ``version``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsplitkv.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libsplitkv.so not built at {_LIB_PATH}: run `python split_kv_merge_b200/build.py`")
_lib = ctypes.CDLL(_LIB_PATH)

# ----------------------------------------------------------------------------- constants
OK, ERR_INVALID, ERR_UNSUPPORTED, ERR_ALIGNMENT, ERR_WORKSPACE, ERR_CUDA = range(6)
DEV_OK, DEV_TIMEOUT, DEV_PAGE_OOB, DEV_PLAN_BAD = 0, 16, 17, 18
BF16, F32, E4M3 = 0, 1, 2
ROPE_INTERLEAVED, ROPE_HALVES = 0, 1
_ROPE = {"interleaved": ROPE_INTERLEAVED, "halves": ROPE_HALVES}
SPLIT_NONE, SPLIT_FIXED, SPLIT_BALANCED, SPLIT_EXPLICIT = 0, 1, 2, 3
_POLICY = {"none": SPLIT_NONE, "fixed": SPLIT_FIXED, "balanced": SPLIT_BALANCED, "explicit": SPLIT_EXPLICIT}

_i32p = ctypes.POINTER(ctypes.c_int32)
_vp = ctypes.c_void_p


class PlanInfo(ctypes.Structure):
    _fields_ = [("num_work", ctypes.c_int32), ("num_partial_rows", ctypes.c_int32),
                ("num_merge_rows", ctypes.c_int32), ("kernel", ctypes.c_int32),
                ("q_tile", ctypes.c_int32), ("plan_words", ctypes.c_int32),
                ("max_splits", ctypes.c_int32), ("total_splits", ctypes.c_int32),
                ("num_ctas", ctypes.c_int32), ("cta_offset", ctypes.c_int32)]

    def as_dict(self) -> dict:
        return {k: getattr(self, k) for k, _ in self._fields_}


class PagedParams(ctypes.Structure):
    _fields_ = [("q", _vp), ("k_cache", _vp), ("v_cache", _vp),
                ("k_stride", ctypes.c_int64 * 3), ("v_stride", ctypes.c_int64 * 3),
                ("kv_indptr", _vp), ("kv_indices", _vp), ("kv_last_page_len", _vp),
                ("batch", ctypes.c_int32), ("total_q", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("num_qo_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("sm_scale", ctypes.c_float),
                ("o", _vp), ("o_dtype", ctypes.c_int32), ("lse", _vp), ("o_part", _vp), ("lse_part", _vp),
                ("status", _vp), ("kv_dtype", ctypes.c_int32), ("kv_scale", ctypes.c_float)]


class MlaParams(ctypes.Structure):
    _fields_ = [("q_nope", _vp), ("q_pe", _vp), ("ckv", _vp), ("kpe", _vp),
                ("ckv_stride", ctypes.c_int64 * 2), ("kpe_stride", ctypes.c_int64 * 2),
                ("kv_dtype", ctypes.c_int32), ("kv_scale", ctypes.c_float),
                ("kv_indptr", _vp), ("kv_indices", _vp), ("kv_last_page_len", _vp),
                ("batch", ctypes.c_int32), ("q_len", ctypes.c_int32), ("num_heads", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("page_size", ctypes.c_int32), ("sm_scale", ctypes.c_float),
                ("o", _vp), ("o_dtype", ctypes.c_int32), ("lse", _vp), ("o_part", _vp), ("lse_part", _vp),
                ("status", _vp)]


class SpliceParams(ctypes.Structure):
    _fields_ = [("src_ckv", _vp), ("src_kpe", _vp),
                ("src_ckv_stride", ctypes.c_int64 * 2), ("src_kpe_stride", ctypes.c_int64 * 2),
                ("src_pages", _vp), ("src_num_pages", ctypes.c_int32), ("src_page_size", ctypes.c_int32),
                ("dst_ckv", _vp), ("dst_kpe", _vp),
                ("dst_ckv_stride", ctypes.c_int64 * 2), ("dst_kpe_stride", ctypes.c_int64 * 2),
                ("dst_pages", _vp), ("dst_num_pages", ctypes.c_int32), ("dst_page_size", ctypes.c_int32),
                ("rope_theta", ctypes.c_float), ("rope_layout", ctypes.c_int32), ("inv_freq", _vp),
                ("kv_dtype", ctypes.c_int32), ("status", _vp)]


class SpliceChunk(ctypes.Structure):
    _fields_ = [("src_start", ctypes.c_int64), ("dst_start", ctypes.c_int64), ("n_tokens", ctypes.c_int64),
                ("delta_pos", ctypes.c_int64)]


def _proto(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


_plan_paged = _proto("skv_plan_paged", ctypes.c_int, [ctypes.c_int32, _i32p, _i32p, _i32p, ctypes.c_int32,
                                                       ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                                       ctypes.c_int32, ctypes.c_int32, _i32p, _i32p, _i32p,
                                                       ctypes.c_int64, ctypes.POINTER(PlanInfo)])
_plan_subset = _proto("skv_plan_paged_subset", ctypes.c_int, [ctypes.c_int32, _i32p, _i32p, _i32p, ctypes.c_int32,
                                                             ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                                             ctypes.c_int32, ctypes.c_int32, _i32p, ctypes.c_int32,
                                                             _i32p, ctypes.c_int64, ctypes.POINTER(PlanInfo)])
_plan_mla = _proto("skv_plan_mla", ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, _i32p, _i32p, ctypes.c_int32,
                                                   ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                                   _i32p, _i32p, _i32p, ctypes.c_int64, ctypes.POINTER(PlanInfo)])
_paged_fwd = _proto("skv_paged_attn_fwd", ctypes.c_int, [ctypes.POINTER(PagedParams), _vp,
                                                          ctypes.POINTER(PlanInfo), _vp])
_mla_fwd = _proto("skv_mla_decode_fwd", ctypes.c_int, [ctypes.POINTER(MlaParams), _vp,
                                                        ctypes.POINTER(PlanInfo), _vp])
_paged_partial = _proto("skv_paged_attn_partial", ctypes.c_int, [ctypes.POINTER(PagedParams), _vp,
                                                                  ctypes.POINTER(PlanInfo), _vp])
_mla_partial = _proto("skv_mla_decode_partial", ctypes.c_int, [ctypes.POINTER(MlaParams), _vp,
                                                                ctypes.POINTER(PlanInfo), _vp])
_paged_static = _proto("skv_paged_attn_fwd_static_scratch", ctypes.c_int, [ctypes.POINTER(PagedParams), _vp,
                                                                          ctypes.POINTER(PlanInfo), _vp])
_pod_fwd = _proto("skv_pod_attn_fwd", ctypes.c_int, [ctypes.POINTER(PagedParams), _vp, ctypes.POINTER(PlanInfo), _vp,
                                                     ctypes.POINTER(PlanInfo), _vp, _vp, _vp])
_merge_plan = _proto("skv_merge_plan", ctypes.c_int, [_vp, _vp, _vp, ctypes.POINTER(PlanInfo), ctypes.c_int32,
                                                       ctypes.c_int32, _vp, ctypes.c_int32, _vp, _vp])
_merge = _proto("skv_merge_states", ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32,
                                                    ctypes.c_int32, _vp, ctypes.c_int32, _vp, _vp])
_gather = _proto("skv_paged_kv_gather", ctypes.c_int, [ctypes.POINTER(PagedParams), _vp, ctypes.c_int64, _vp,
                                                        _vp, _vp])
_splice = _proto("skv_mla_splice", ctypes.c_int, [ctypes.POINTER(SpliceParams), ctypes.POINTER(SpliceChunk),
                                                   ctypes.c_int32, _vp])
_causal = _proto("skv_causal_tables", ctypes.c_int, [ctypes.c_int32, _i32p, _i32p, _i32p, _i32p, ctypes.c_int32,
                                                     _i32p, _i32p, _i32p, _i32p, _i32p, _i32p, ctypes.c_int64,
                                                     ctypes.POINTER(ctypes.c_int64)])
_wait_timeout = _proto("skv_test_wait_timeout", ctypes.c_int, [_vp, ctypes.c_int64, _vp])
_fold = _proto("skv_mla_fold_ratio", ctypes.c_int32, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32])
_status_str = _proto("skv_status_str", ctypes.c_char_p, [ctypes.c_int32])
_version = _proto("skv_version", ctypes.c_int32, [])

SYMBOLS = ["skv_plan_paged", "skv_paged_attn_fwd", "skv_paged_attn_partial", "skv_merge_plan", "skv_plan_mla",
           "skv_mla_decode_fwd", "skv_mla_decode_partial", "skv_merge_states", "skv_paged_kv_gather",
           "skv_mla_fold_ratio", "skv_status_str", "skv_version", "skv_paged_attn_fwd_static_scratch",
           "skv_test_wait_timeout", "skv_mla_splice", "skv_causal_tables", "skv_plan_paged_subset",
           "skv_pod_attn_fwd"]


class SkvError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {status_str(code)} (status {code})")
        self.code = code


def status_str(code: int) -> str:
    return _status_str(int(code)).decode()


def version() -> int:
    return int(_version())


def mla_fold_ratio(num_heads: int, q_len: int, tile_m: int = 128) -> int:
    return int(_fold(num_heads, q_len, tile_m))


def _check(code: int, where: str) -> None:
    if code != OK:
        raise SkvError(code, where)


# ----------------------------------------------------------------------------- helpers
def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _ptr_i32(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(_i32p)


def _dptr(t) -> Optional[int]:
    """Device pointer of a torch tensor (None passes NULL)."""
    return None if t is None else int(t.data_ptr())


_PLACEHOLDER = {}


def _index_ptr(t) -> Optional[int]:
    """Pointer of an int32 index tensor; an empty one (no page of any request) is passed as a small
    zero buffer on its device, since torch gives empty tensors no storage and the library rejects
    a NULL page list.  The kernels read no page id of a request without pages."""
    if t is None or t.numel() > 0:
        return _dptr(t)
    import torch
    key = str(t.device)
    if key not in _PLACEHOLDER:
        _PLACEHOLDER[key] = torch.zeros(4, dtype=torch.int32, device=t.device)
    return _dptr(_PLACEHOLDER[key])


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t) -> int:
    import torch
    return {torch.bfloat16: BF16, torch.float32: F32, torch.float8_e4m3fn: E4M3, torch.uint8: E4M3}[t.dtype]


def _split_args(policy, split_page_start):
    if policy != SPLIT_EXPLICIT:
        return None, None
    sizes = [len(b) - 1 for b in split_page_start]
    indptr = _i32(np.concatenate([[0], np.cumsum(sizes)]))
    bounds = _i32(np.concatenate([np.asarray(b, np.int64) for b in split_page_start]))
    return indptr, bounds


@dataclass
class Plan:
    """Host plan words, its summary, and (after ``to``) the device copy."""
    words: np.ndarray
    info: PlanInfo
    device: Optional[object] = None

    def to(self, device, non_blocking: bool = False):
        import torch
        src = torch.from_numpy(self.words)
        if non_blocking:
            src = src.pin_memory()
        self.device = src.to(device, non_blocking=non_blocking)
        return self


def _plan(fn, args, policy, split_page_start, where):
    pol = _POLICY[policy] if isinstance(policy, str) else int(policy)
    si, sb = _split_args(pol, split_page_start)
    info = PlanInfo()
    cap = 0
    code = fn(*args(pol), _ptr_i32(si), _ptr_i32(sb), None, 0, ctypes.byref(info))
    if code not in (OK, ERR_WORKSPACE):
        _check(code, where)
    words = np.zeros(max(1, info.plan_words), dtype=np.int32)
    cap = words.size
    _check(fn(*args(pol), _ptr_i32(si), _ptr_i32(sb), _ptr_i32(words), cap, ctypes.byref(info)), where)
    return Plan(words[: info.plan_words] if info.plan_words else words[:0], info)


# ----------------------------------------------------------------------------- planners
def plan_paged(qo_indptr, kv_indptr, kv_last_page_len, page_size: int, num_qo_heads: int,
               num_kv_heads: int, head_dim: int, policy="balanced", param: int = 0,
               split_page_start: Optional[Sequence[Sequence[int]]] = None) -> Plan:
    """Host planner (skv_plan_paged).  Host int arrays in, Plan out."""
    qo, ki, la = _i32(qo_indptr), _i32(kv_indptr), _i32(kv_last_page_len)
    b = len(ki) - 1
    return _plan(_plan_paged, lambda pol: (b, _ptr_i32(qo), _ptr_i32(ki), _ptr_i32(la), page_size, num_qo_heads,
                                           num_kv_heads, head_dim, pol, param),
                 policy, split_page_start, "skv_plan_paged")


def plan_paged_subset(qo_indptr, kv_indptr, kv_last_page_len, page_size: int, num_qo_heads: int,
                      num_kv_heads: int, head_dim: int, requests, policy="balanced", param: int = 0) -> Plan:
    """Host planner for the listed requests of a batch only (skv_plan_paged_subset)."""
    qo, ki, la, rq = _i32(qo_indptr), _i32(kv_indptr), _i32(kv_last_page_len), _i32(requests)
    b = len(ki) - 1
    pol = _POLICY[policy] if isinstance(policy, str) else int(policy)
    info = PlanInfo()
    args = (b, _ptr_i32(qo), _ptr_i32(ki), _ptr_i32(la), page_size, num_qo_heads, num_kv_heads, head_dim, pol,
            param, _ptr_i32(rq), len(rq))
    code = _plan_subset(*args, None, 0, ctypes.byref(info))
    if code not in (OK, ERR_WORKSPACE):
        _check(code, "skv_plan_paged_subset")
    words = np.zeros(max(1, info.plan_words), dtype=np.int32)
    _check(_plan_subset(*args, _ptr_i32(words), words.size, ctypes.byref(info)), "skv_plan_paged_subset")
    return Plan(words[: info.plan_words] if info.plan_words else words[:0], info)


def plan_mla(batch_q_len: int, kv_indptr, kv_last_page_len, page_size: int, num_heads: int,
             policy="balanced", param: int = 0,
             split_page_start: Optional[Sequence[Sequence[int]]] = None, kv_dtype="bf16") -> Plan:
    """Host planner (skv_plan_mla).  ``batch_q_len`` is the query length of every request;
    ``kv_dtype`` the latent cache type ("bf16" / "e4m3") the plan will run on."""
    ki, la = _i32(kv_indptr), _i32(kv_last_page_len)
    b = len(ki) - 1
    kd = {"bf16": BF16, "e4m3": E4M3}[kv_dtype] if isinstance(kv_dtype, str) else int(kv_dtype)
    return _plan(_plan_mla, lambda pol: (b, batch_q_len, _ptr_i32(ki), _ptr_i32(la), page_size, num_heads, kd,
                                         pol, param),
                 policy, split_page_start, "skv_plan_mla")


# ----------------------------------------------------------------------------- launches
def _paged_params(q, k_cache, v_cache, kv_indptr, kv_indices, kv_last_page_len, o, lse, o_part, lse_part,
                  status, sm_scale, num_pages, page_size=None, kv_scale: float = 1.0):
    if k_cache.stride(-1) != 1 or v_cache.stride(-1) != 1:
        raise ValueError("the innermost (head_dim) stride of K and V must be 1")
    p = PagedParams()
    p.q, p.k_cache, p.v_cache = _dptr(q), _dptr(k_cache), _dptr(v_cache)
    for i in range(3):
        p.k_stride[i] = k_cache.stride(i)
        p.v_stride[i] = v_cache.stride(i)
    p.kv_indptr, p.kv_indices, p.kv_last_page_len = _dptr(kv_indptr), _index_ptr(kv_indices), _dptr(kv_last_page_len)
    p.batch = kv_indptr.shape[0] - 1
    p.total_q = q.shape[0] if q is not None else 0
    p.num_pages = k_cache.shape[0] if num_pages is None else num_pages
    p.page_size = k_cache.shape[1] if page_size is None else page_size
    p.num_qo_heads = q.shape[1] if q is not None else k_cache.shape[2]
    p.num_kv_heads = k_cache.shape[2]
    p.head_dim = k_cache.shape[3]
    p.sm_scale = float(p.head_dim ** -0.5 if sm_scale is None else sm_scale)
    p.o = _dptr(o)
    p.o_dtype = _dtype_code(o) if o is not None else F32
    p.lse, p.o_part, p.lse_part, p.status = _dptr(lse), _dptr(o_part), _dptr(lse_part), _dptr(status)
    p.kv_dtype = _dtype_code(k_cache)
    if _dtype_code(v_cache) != p.kv_dtype:
        raise ValueError("K and V caches must have the same dtype")
    p.kv_scale = float(kv_scale)
    return p


def paged_attn_fwd(q, k_cache, v_cache, kv_indptr, kv_indices, kv_last_page_len, plan: Plan, o, lse=None,
                   o_part=None, lse_part=None, status=None, sm_scale: Optional[float] = None,
                   num_pages: Optional[int] = None, stream=None, phase: str = "all", kv_scale: float = 1.0) -> None:
    """skv_paged_attn_fwd.  q [total_q, Hq, D] bf16; k_cache / v_cache [num_pages, P, Hk, D] bf16,
    or e4m3 codes (float8_e4m3fn / uint8) with the per-tensor ``kv_scale``, views (any page/slot/head
    strides, head_dim contiguous); page-table tensors int32 on the device; o [total_q, Hq, D]
    f32|bf16; lse [total_q, Hq] f32; o_part / lse_part sized by ``plan.info.num_partial_rows``
    when the plan splits."""
    p = _paged_params(q, k_cache, v_cache, kv_indptr, kv_indices, kv_last_page_len, o, lse, o_part, lse_part,
                      status, sm_scale, num_pages, kv_scale=kv_scale)
    fn = {"all": _paged_fwd, "partial": _paged_partial}[phase]
    _check(fn(ctypes.byref(p), _dptr(plan.device), ctypes.byref(plan.info), _stream_ptr(stream)),
           "skv_paged_attn_fwd" if phase == "all" else "skv_paged_attn_partial")


def pod_attn_fwd(q, k_cache, v_cache, kv_indptr, kv_indices, kv_last_page_len, decode_plan: Plan, prefill_plan: Plan,
                 o, lse=None, decode_o_part=None, decode_lse_part=None, prefill_o_part=None, prefill_lse_part=None,
                 status=None, sm_scale: Optional[float] = None, num_pages: Optional[int] = None, stream=None) -> None:
    """skv_pod_attn_fwd: the decode subset plan (all-KV-heads kernel) and the prefill subset plan
    (128-row kernel) of one batch in one attention launch, then both plans' merge passes.  Each
    plan's split partials go to its own o_part / lse_part."""
    p = _paged_params(q, k_cache, v_cache, kv_indptr, kv_indices, kv_last_page_len, o, lse, decode_o_part,
                      decode_lse_part, status, sm_scale, num_pages)
    _check(_pod_fwd(ctypes.byref(p), _dptr(decode_plan.device), ctypes.byref(decode_plan.info),
                    _dptr(prefill_plan.device), ctypes.byref(prefill_plan.info), _dptr(prefill_o_part),
                    _dptr(prefill_lse_part), _stream_ptr(stream)), "skv_pod_attn_fwd")


def paged_attn_fwd_static_scratch(q, k_cache, v_cache, kv_indptr, kv_indices, kv_last_page_len, plan: Plan, o,
                                  lse=None, status=None, sm_scale: Optional[float] = None,
                                  num_pages: Optional[int] = None, stream=None) -> None:
    """skv_paged_attn_fwd_static_scratch: paged_attn_fwd with the split partials kept in the
    library's own fixed 32 MiB device array, for callers that cannot allocate device memory."""
    p = _paged_params(q, k_cache, v_cache, kv_indptr, kv_indices, kv_last_page_len, o, lse, None, None,
                      status, sm_scale, num_pages)
    _check(_paged_static(ctypes.byref(p), _dptr(plan.device), ctypes.byref(plan.info), _stream_ptr(stream)),
           "skv_paged_attn_fwd_static_scratch")


def mla_decode_fwd(q_nope, q_pe, ckv, kpe, kv_indptr, kv_indices, kv_last_page_len, plan: Plan, o, lse=None,
                   o_part=None, lse_part=None, status=None, sm_scale: Optional[float] = None,
                   kv_scale: float = 1.0, num_pages: Optional[int] = None, stream=None, phase: str = "all") -> None:
    """skv_mla_decode_fwd.  q_nope [B, q_len, H, 512], q_pe [B, q_len, H, 64] bf16; ckv
    [num_pages, P, 512], kpe [num_pages, P, 64] views (bf16, or uint8 / float8_e4m3fn codes);
    o [B, q_len, H, 512]; lse [B, q_len, H]."""
    if ckv.stride(-1) != 1 or kpe.stride(-1) != 1:
        raise ValueError("the innermost stride of ckv and kpe must be 1")
    p = MlaParams()
    p.q_nope, p.q_pe, p.ckv, p.kpe = _dptr(q_nope), _dptr(q_pe), _dptr(ckv), _dptr(kpe)
    for i in range(2):
        p.ckv_stride[i] = ckv.stride(i)
        p.kpe_stride[i] = kpe.stride(i)
    p.kv_dtype = _dtype_code(ckv)
    p.kv_scale = float(kv_scale)
    p.kv_indptr, p.kv_indices, p.kv_last_page_len = _dptr(kv_indptr), _index_ptr(kv_indices), _dptr(kv_last_page_len)
    p.batch = kv_indptr.shape[0] - 1
    p.q_len = q_nope.shape[1]
    p.num_heads = q_nope.shape[2]
    p.num_pages = ckv.shape[0] if num_pages is None else num_pages
    p.page_size = ckv.shape[1]
    p.sm_scale = float(192.0 ** -0.5 if sm_scale is None else sm_scale)
    p.o, p.o_dtype = _dptr(o), _dtype_code(o)
    p.lse, p.o_part, p.lse_part, p.status = _dptr(lse), _dptr(o_part), _dptr(lse_part), _dptr(status)
    fn = {"all": _mla_fwd, "partial": _mla_partial}[phase]
    _check(fn(ctypes.byref(p), _dptr(plan.device), ctypes.byref(plan.info), _stream_ptr(stream)),
           "skv_mla_decode_fwd" if phase == "all" else "skv_mla_decode_partial")


def merge_plan(o_part, lse_part, plan: Plan, num_heads: int, head_dim: int, o, lse=None, stream=None) -> None:
    """skv_merge_plan: the plan's merge pass (second phase of paged_attn_fwd / mla_decode_fwd)."""
    _check(_merge_plan(_dptr(o_part), _dptr(lse_part), _dptr(plan.device), ctypes.byref(plan.info), num_heads,
                       head_dim, _dptr(o), _dtype_code(o), _dptr(lse), _stream_ptr(stream)), "skv_merge_plan")


def merge_states(o_states, lse_states, o_out, lse_out=None, state_indptr=None, num_states: int = 0,
                 stream=None) -> None:
    """skv_merge_states.  With ``state_indptr`` (device int32 [rows+1]): o_states [*, H, D],
    lse_states [*, H].  Without: state-major o_states [S, rows, H, D], lse_states [S, rows, H]."""
    if state_indptr is None:
        num_states = o_states.shape[0]
        rows, H, D = o_states.shape[1], o_states.shape[2], o_states.shape[3]
    else:
        rows, H, D = state_indptr.shape[0] - 1, o_states.shape[-2], o_states.shape[-1]
    _check(_merge(_dptr(o_states), _dptr(lse_states), _dptr(state_indptr), num_states, rows, H, D, _dptr(o_out),
                  _dtype_code(o_out), _dptr(lse_out), _stream_ptr(stream)), "skv_merge_states")


def paged_kv_gather(k_cache, v_cache, kv_indptr, kv_indices, kv_last_page_len, token_indptr, total_tokens: int,
                    k_out, v_out, status=None, num_pages: Optional[int] = None, stream=None) -> None:
    """skv_paged_kv_gather (test hook): dense copies of every request's logical K and V."""
    p = _paged_params(None, k_cache, v_cache, kv_indptr, kv_indices, kv_last_page_len, None, None, None, None,
                      status, None, num_pages)
    _check(_gather(ctypes.byref(p), _dptr(token_indptr), total_tokens, _dptr(k_out), _dptr(v_out),
                   _stream_ptr(stream)), "skv_paged_kv_gather")


def mla_splice(src_ckv, src_kpe, src_pages, dst_ckv, dst_kpe, dst_pages, chunks, rope_theta: float = 10000.0,
               rope_layout: str = "interleaved", inv_freq=None, status=None, src_num_pages: Optional[int] = None,
               dst_num_pages: Optional[int] = None, stream=None) -> None:
    """skv_mla_splice (fetch primitive, local compute).  src/dst ckv [pages, P, 512] and kpe
    [pages, P, 64] bf16 views; src_pages / dst_pages device int32 page lists; ``chunks`` a sequence
    of (src_start, dst_start, n_tokens, delta_pos): token t of a chunk moves from logical position
    src_start + t to dst_start + t and its rope pairs turn by delta_pos * theta_i."""
    p = splice_params(src_ckv, src_kpe, src_pages, dst_ckv, dst_kpe, dst_pages, rope_theta, rope_layout, inv_freq,
                      status, src_num_pages, dst_num_pages)
    splice_launch(p, splice_chunks(chunks), stream)


def splice_chunks(chunks) -> "ctypes.Array":
    """Host array of skv_splice_chunk from (src_start, dst_start, n_tokens, delta_pos) rows."""
    rows = np.asarray(chunks, dtype=np.int64).reshape(-1, 4)
    arr = (SpliceChunk * max(1, len(rows)))()
    for i, (s0, d0, n, dl) in enumerate(rows):
        arr[i].src_start, arr[i].dst_start, arr[i].n_tokens, arr[i].delta_pos = int(s0), int(d0), int(n), int(dl)
    arr._n = len(rows)
    return arr


def splice_launch(p: "SpliceParams", chunks: "ctypes.Array", stream=None) -> None:
    """Launch skv_mla_splice on prepared arguments (``splice_params``, ``splice_chunks``)."""
    _check(_splice(ctypes.byref(p), chunks, chunks._n, _stream_ptr(stream)), "skv_mla_splice")


def splice_params(src_ckv, src_kpe, src_pages, dst_ckv, dst_kpe, dst_pages, rope_theta: float = 10000.0,
                  rope_layout: str = "interleaved", inv_freq=None, status=None, src_num_pages: Optional[int] = None,
                  dst_num_pages: Optional[int] = None) -> "SpliceParams":
    """The skv_splice_params of an mla_splice call, for repeated launches."""
    for t in (src_ckv, src_kpe, dst_ckv, dst_kpe):
        if t.stride(-1) != 1:
            raise ValueError("the innermost stride of every cache view must be 1")
    p = SpliceParams()
    p.src_ckv, p.src_kpe, p.dst_ckv, p.dst_kpe = _dptr(src_ckv), _dptr(src_kpe), _dptr(dst_ckv), _dptr(dst_kpe)
    for i in range(2):
        p.src_ckv_stride[i], p.src_kpe_stride[i] = src_ckv.stride(i), src_kpe.stride(i)
        p.dst_ckv_stride[i], p.dst_kpe_stride[i] = dst_ckv.stride(i), dst_kpe.stride(i)
    p.src_pages, p.dst_pages = _dptr(src_pages), _dptr(dst_pages)
    p.src_num_pages = src_ckv.shape[0] if src_num_pages is None else src_num_pages
    p.dst_num_pages = dst_ckv.shape[0] if dst_num_pages is None else dst_num_pages
    p.src_page_size, p.dst_page_size = src_ckv.shape[1], dst_ckv.shape[1]
    p.rope_theta, p.rope_layout = float(rope_theta), _ROPE[rope_layout]
    p.inv_freq, p.kv_dtype, p.status = _dptr(inv_freq), _dtype_code(src_ckv), _dptr(status)
    if _dtype_code(dst_ckv) != p.kv_dtype:
        raise ValueError("source and destination caches must have the same dtype")
    return p


def causal_tables(qo_indptr, kv_indptr, kv_indices, kv_last_page_len, page_size: int) -> dict:
    """skv_causal_tables on host arrays: {"prefix": (kv_indptr, kv_indices, kv_last_page_len),
    "diag": (kv_indptr, token rows, kv_last_page_len)}, int32 numpy arrays."""
    qo, ip, ix, la = _i32(qo_indptr), _i32(kv_indptr), _i32(kv_indices), _i32(kv_last_page_len)
    B, total_q = len(ip) - 1, int(qo[-1])
    pre_ip, pre_ix, pre_la = (np.zeros(B + 1, np.int32), np.zeros(max(1, int(ip[-1])), np.int32),
                              np.zeros(max(1, B), np.int32))
    d_ip, d_la = np.zeros(total_q + 1, np.int32), np.zeros(max(1, total_q), np.int32)
    need = ctypes.c_int64(0)
    args = lambda rows, cap: (B, _ptr_i32(qo), _ptr_i32(ip), _ptr_i32(ix), _ptr_i32(la), int(page_size),
                              _ptr_i32(pre_ip), _ptr_i32(pre_ix), _ptr_i32(pre_la), _ptr_i32(d_ip), _ptr_i32(rows),
                              _ptr_i32(d_la), cap, ctypes.byref(need))
    code = _causal(*args(None, 0))
    if code == ERR_WORKSPACE:
        rows = np.zeros(int(need.value), np.int32)
        code = _causal(*args(rows, int(need.value)))
    else:
        rows = np.zeros(0, np.int32)
    _check(code, "skv_causal_tables")
    return {"prefix": (pre_ip, pre_ix[:int(pre_ip[-1])], pre_la[:B]),
            "diag": (d_ip, rows, d_la[:total_q])}


def test_wait_timeout(status, limit_ns: int, stream=None) -> None:
    """skv_test_wait_timeout (failure-detection test hook)."""
    _check(_wait_timeout(_dptr(status), int(limit_ns), _stream_ptr(stream)), "skv_test_wait_timeout")


def library_path() -> str:
    return _LIB_PATH


from .runner import (CausalMlaDecode, PagedDecodePipeline, PodAttention, RouteMerge, mla_decode,  # noqa: E402,F401
                     paged_attention, pod_attention, pod_decode_sms)
