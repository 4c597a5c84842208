"""Python binding of the SegPagedAttention C ABI (include/segpaged.h), with the same names.

Argument marshalling only: torch tensors become raw pointers, numpy arrays become host pointers,
the current CUDA stream is passed through, and negative return codes raise SegPagedError. Every
step of the computation runs in libsegpaged.so; if the library is missing the import fails.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsegpaged.so")
UNIT_FIELDS = 32
MASS_ITEM_FIELDS = 16

STATUS_PAGE_ID = 1
STATUS_TABLE = 2
STATUS_TIMEOUT = 4
STATUS_UNIT = 8

# Every function include/segpaged.h declares.
EXPORTS = ("segpaged_error_string", "segpaged_pages_bytes", "segpaged_rope_cos_sin", "segpaged_build",
           "segpaged_prefill_plan", "segpaged_prefill_workspace_bytes", "segpaged_attn_prefill",
           "segpaged_attn_prefill_rope", "segpaged_rope_realign", "segpaged_prefill_plan_append", "segpaged_attn_prefill_append",
           "segpaged_attn_prefill_noalloc", "segpaged_mass_plan", "segpaged_mass_workspace_bytes",
           "segpaged_token_mass", "segpaged_select_topk")


class SegPagedError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {error_string(code)} (code {code})")
        self.code = code


class _PlanInfo(ctypes.Structure):
    _fields_ = [("num_units", ctypes.c_int64), ("num_groups", ctypes.c_int64), ("num_partials", ctypes.c_int64),
                ("num_half_units", ctypes.c_int64), ("combine_row_blocks", ctypes.c_int64),
                ("total_q", ctypes.c_int64), ("page_table_len", ctypes.c_int64), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32)]


PLAN_INFO_FIELDS = tuple(name for name, _ in _PlanInfo._fields_)


class _Dims(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32), ("num_pages", ctypes.c_int32)]


@dataclass
class Dims:
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    num_pages: int = 0

    def c(self) -> _Dims:
        return _Dims(self.num_seqs, self.num_q_heads, self.num_kv_heads, self.head_dim, self.page_size, self.num_pages)


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libsegpaged.so not built at {LIB_PATH}; run head_sparse_paged_b200/build_ext.py")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    dp = ctypes.POINTER(_Dims)
    lib.segpaged_error_string.restype = ctypes.c_char_p
    lib.segpaged_error_string.argtypes = [ctypes.c_int]
    lib.segpaged_pages_bytes.restype = i64
    lib.segpaged_pages_bytes.argtypes = [dp, vp, vp, vp, vp, vp]
    lib.segpaged_rope_cos_sin.restype = ctypes.c_int
    lib.segpaged_rope_cos_sin.argtypes = [ctypes.c_double, vp, i32, i32, vp]
    lib.segpaged_build.restype = ctypes.c_int
    lib.segpaged_build.argtypes = [dp] + [vp] * 12
    ip = ctypes.POINTER(_PlanInfo)
    lib.segpaged_prefill_plan.restype = i64
    lib.segpaged_prefill_plan.argtypes = [dp, vp, vp, vp, vp, i32, vp, i64, ip]
    lib.segpaged_rope_realign.restype = ctypes.c_int
    lib.segpaged_rope_realign.argtypes = [dp] + [vp] * 12
    lib.segpaged_prefill_plan_append.restype = i64
    lib.segpaged_prefill_plan_append.argtypes = [dp, vp, vp, vp, vp, i32, vp, i64, ip]
    lib.segpaged_attn_prefill_append.restype = ctypes.c_int
    lib.segpaged_attn_prefill_append.argtypes = [dp, vp, i32, vp, vp, vp, vp, vp, i64, vp, ip, ctypes.c_float, vp, vp, vp,
                                                 ctypes.c_size_t, vp, vp]
    lib.segpaged_prefill_workspace_bytes.restype = ctypes.c_size_t
    lib.segpaged_prefill_workspace_bytes.argtypes = [dp, ip]
    lib.segpaged_attn_prefill.restype = ctypes.c_int
    lib.segpaged_attn_prefill.argtypes = [dp, vp, i32, vp, vp, vp, i64, vp, ip, ctypes.c_float, vp, vp, vp,
                                          ctypes.c_size_t, vp, vp]
    lib.segpaged_attn_prefill_rope.restype = ctypes.c_int
    lib.segpaged_attn_prefill_rope.argtypes = [dp, vp, i32, vp, vp, vp, i64, vp, ip, ctypes.c_float, vp, vp, vp, vp, vp, vp,
                                               ctypes.c_size_t, vp, vp]
    lib.segpaged_attn_prefill_noalloc.restype = ctypes.c_int
    lib.segpaged_attn_prefill_noalloc.argtypes = [dp, vp, i32, vp, vp, vp, i64, vp, i64, ctypes.c_float, vp, vp, vp, vp]
    lib.segpaged_mass_plan.restype = i64
    lib.segpaged_mass_plan.argtypes = [dp, vp, vp, vp, vp, vp, i64]
    lib.segpaged_mass_workspace_bytes.restype = ctypes.c_size_t
    lib.segpaged_mass_workspace_bytes.argtypes = [dp, i32]
    lib.segpaged_token_mass.restype = ctypes.c_int
    lib.segpaged_token_mass.argtypes = [dp, vp, i32, vp, vp, i64, vp, i64, vp, ctypes.c_float, vp, vp, vp, vp, vp,
                                        ctypes.c_size_t, vp, vp]
    lib.segpaged_select_topk.restype = ctypes.c_int
    lib.segpaged_select_topk.argtypes = [i32, vp, vp, vp, vp, vp]
    return lib


_lib = _load()


def library():
    return _lib


def error_string(code: int) -> str:
    return _lib.segpaged_error_string(int(code)).decode()


segpaged_error_string = error_string


def _host_i32(a, n=None):
    a = np.ascontiguousarray(np.asarray(a, dtype=np.int32))
    if n is not None and a.size != n:
        raise ValueError(f"expected {n} int32 values, got {a.size}")
    return a


def _hp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dev(t: torch.Tensor | None, dtype=None, what=""):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{what}: expected a CUDA tensor")
    # the library launches on, and encodes its tensor maps for, the current device
    cur = torch.cuda.current_device()
    if t.device.index is not None and t.device.index != cur:
        raise ValueError(f"{what}: tensor on {t.device}, but the current device is cuda:{cur}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{what}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{what}: expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def segpaged_pages_bytes(dims: Dims, ctx_len, q_len, cls):
    """(stored K+V bytes, dense K+V bytes, stored pages per (b, k) as int32 [B*Hkv]). Host only."""
    B, H = dims.num_seqs, dims.num_kv_heads
    L, Lq, c = _host_i32(ctx_len, B), _host_i32(q_len, B), _host_i32(cls, B * H * 3)
    dense = ctypes.c_int64(0)
    per = np.zeros(B * H, np.int32)
    r = _lib.segpaged_pages_bytes(ctypes.byref(dims.c()), _hp(L), _hp(Lq), _hp(c), ctypes.byref(dense), _hp(per))
    if r < 0:
        raise SegPagedError(int(r), "segpaged_pages_bytes")
    return int(r), int(dense.value), per


def segpaged_rope_cos_sin(theta: float, deltas, head_dim: int) -> np.ndarray:
    """[B, D/2, 2] float32 (cos, sin) table of delta_b * theta^(-2d/D)."""
    d = _host_i32(deltas)
    out = np.zeros((d.size, head_dim // 2, 2), np.float32)
    r = _lib.segpaged_rope_cos_sin(float(theta), _hp(d), d.size, head_dim, _hp(out))
    if r < 0:
        raise SegPagedError(r, "segpaged_rope_cos_sin")
    return out


def prepare_build(dims: Dims, k_dense, v_dense, cu_seqlens_k, q_len, cls, page_table, page_table_offs, rope_cos_sin,
                  k_pool, v_pool, status=None) -> PreparedCall:
    """segpaged_build with its arguments checked and marshalled once (see PreparedCall)."""
    bf = torch.bfloat16
    d = dims.c()
    args = (ctypes.byref(d), _dev(k_dense, bf, "k_dense"), _dev(v_dense, bf, "v_dense"),
            _dev(cu_seqlens_k, torch.int32, "cu_seqlens_k"), _dev(q_len, torch.int32, "q_len"),
            _dev(cls, torch.int32, "cls"), _dev(page_table, torch.int32, "page_table"),
            _dev(page_table_offs, torch.int32, "page_table_offs"), _dev(rope_cos_sin, torch.float32, "rope_cos_sin"),
            _dev(k_pool, bf, "k_pool"), _dev(v_pool, bf, "v_pool"), _dev(status, torch.int32, "status"))
    return PreparedCall(_lib.segpaged_build, "segpaged_build", args,
                        (d, k_dense, v_dense, cu_seqlens_k, q_len, cls, page_table, page_table_offs, rope_cos_sin,
                         k_pool, v_pool, status))


def segpaged_build(dims: Dims, k_dense, v_dense, cu_seqlens_k, q_len, cls, page_table, page_table_offs,
                   rope_cos_sin, k_pool, v_pool, status=None, stream=None):
    """Scatter dense K/V [sum L, Hkv, D] (bf16, CUDA) into k_pool/v_pool [num_pages, P, D]."""
    prepare_build(dims, k_dense, v_dense, cu_seqlens_k, q_len, cls, page_table, page_table_offs, rope_cos_sin, k_pool,
                  v_pool, status)(stream)


def _info(d: dict) -> _PlanInfo:
    """The C struct of a plan-info dict as segpaged_prefill_plan returns it (every field required)."""
    return _PlanInfo(*(int(d[name]) for name in PLAN_INFO_FIELDS))


def _plan(fn, name, dims: Dims, ctx_len, q_len, cls, page_table_offs, split_ctas):
    B, H = dims.num_seqs, dims.num_kv_heads
    L, Lq = _host_i32(ctx_len, B), _host_i32(q_len, B)
    c, offs = _host_i32(cls, B * H * 3), _host_i32(page_table_offs, B * H + 1)
    d = dims.c()
    info = _PlanInfo()
    n = fn(ctypes.byref(d), _hp(L), _hp(Lq), _hp(c), _hp(offs), int(split_ctas), None, 0, ctypes.byref(info))
    if n < 0:
        raise SegPagedError(int(n), name)
    units = np.zeros((max(n, 1), UNIT_FIELDS), np.int32)
    n2 = fn(ctypes.byref(d), _hp(L), _hp(Lq), _hp(c), _hp(offs), int(split_ctas), _hp(units), n, ctypes.byref(info))
    if n2 < 0:
        raise SegPagedError(int(n2), name)
    return units[:n], {name: int(getattr(info, name)) for name in PLAN_INFO_FIELDS}


def segpaged_prefill_plan(dims: Dims, ctx_len, q_len, cls, page_table_offs, split_ctas: int = 0):
    """(records int32 [n, 32], info dict). Records [0, num_units) are work units (longest first by cost
    bucket), the rest combine records of split units. split_ctas > 0 lets long units be split across that
    many concurrent CTAs (the SM count); 0 never splits. Host only."""
    return _plan(_lib.segpaged_prefill_plan, "segpaged_prefill_plan", dims, ctx_len, q_len, cls, page_table_offs,
                 split_ctas)


def segpaged_prefill_plan_append(dims: Dims, ctx_len, q_len, cls, page_table_offs, split_ctas: int = 0):
    """Plan of the fused append-and-attend call, same form as segpaged_prefill_plan. Host only."""
    return _plan(_lib.segpaged_prefill_plan_append, "segpaged_prefill_plan_append", dims, ctx_len, q_len, cls,
                 page_table_offs, split_ctas)


def segpaged_prefill_workspace_bytes(dims: Dims, info: dict) -> int:
    return int(_lib.segpaged_prefill_workspace_bytes(ctypes.byref(dims.c()), ctypes.byref(_info(info))))


class PreparedCall:
    """A C-ABI call whose arguments were checked and marshalled once, for callers that repeat it (a serving loop
    runs the same layer's prefill every step). The tensors it was prepared with must stay allocated, with the same
    shape, dtype, device and storage, while it is used; their contents may change between calls. Calling it passes
    the given CUDA stream (default: the current one) and raises SegPagedError on a negative return code."""

    __slots__ = ("_fn", "_name", "_args", "_keep")

    def __init__(self, fn, name: str, args: tuple, keep: tuple):
        self._fn, self._name, self._args, self._keep = fn, name, args, keep

    def __call__(self, stream=None):
        r = self._fn(*self._args, _stream(stream))
        if r < 0:
            raise SegPagedError(r, self._name)


def prepare_attn_prefill(dims: Dims, q, k_pool, v_pool, page_table, plan, info: dict, softmax_scale, o, lse, workspace,
                         status=None) -> PreparedCall:
    """segpaged_attn_prefill with its arguments checked and marshalled once (see PreparedCall)."""
    bf = torch.bfloat16
    d, inf = dims.c(), _info(info)
    args = (ctypes.byref(d), _dev(q, bf, "q"), int(q.shape[0]), _dev(k_pool, bf, "k_pool"), _dev(v_pool, bf, "v_pool"),
            _dev(page_table, torch.int32, "page_table"), int(page_table.numel()), _dev(plan, torch.int32, "plan"),
            ctypes.byref(inf), float(softmax_scale), _dev(o, bf, "o"), _dev(lse, torch.float32, "lse"),
            _dev(workspace, None, "workspace"), int(workspace.numel() * workspace.element_size()),
            _dev(status, torch.int32, "status"))
    return PreparedCall(_lib.segpaged_attn_prefill, "segpaged_attn_prefill", args,
                        (d, inf, q, k_pool, v_pool, page_table, plan, o, lse, workspace, status))


def segpaged_attn_prefill(dims: Dims, q, k_pool, v_pool, page_table, plan, info: dict, softmax_scale, o, lse, workspace,
                          status=None, stream=None):
    """O [total_q, Hq, D] bf16 and LSE [Hq, total_q] float32, written in place (CUDA tensors).
    plan: the plan's records on the device; info: the dict segpaged_prefill_plan returned."""
    prepare_attn_prefill(dims, q, k_pool, v_pool, page_table, plan, info, softmax_scale, o, lse, workspace, status)(stream)


def segpaged_attn_prefill_append(dims: Dims, q, k_new, v_new, k_pool, v_pool, page_table, plan, info: dict,
                                 softmax_scale, o, lse, workspace, status=None, stream=None):
    """Fused append-and-attend: writes the query rows' new keys/values (k_new, v_new [total_q, Hkv, D] bf16)
    into their pool pages and computes O / LSE over the pool before the query range and the new rows from it."""
    bf = torch.bfloat16
    r = _lib.segpaged_attn_prefill_append(ctypes.byref(dims.c()), _dev(q, bf, "q"), int(q.shape[0]),
                                          _dev(k_new, bf, "k_new"), _dev(v_new, bf, "v_new"), _dev(k_pool, bf, "k_pool"),
                                          _dev(v_pool, bf, "v_pool"), _dev(page_table, torch.int32, "page_table"),
                                          int(page_table.numel()), _dev(plan, torch.int32, "plan"),
                                          ctypes.byref(_info(info)), float(softmax_scale), _dev(o, bf, "o"),
                                          _dev(lse, torch.float32, "lse"), _dev(workspace, None, "workspace"),
                                          int(workspace.numel() * workspace.element_size()),
                                          _dev(status, torch.int32, "status"), _stream(stream))
    if r < 0:
        raise SegPagedError(r, "segpaged_attn_prefill_append")


def segpaged_rope_realign(dims: Dims, cu_seqlens_k, q_len, cls, page_table, page_table_offs, frag_offs, frag_start,
                          frag_cos_sin, k_pool, k_pool_out, status=None, stream=None):
    """Copy one layer's stored K pages into k_pool_out (same ids) with per-fragment RoPE re-alignment."""
    bf = torch.bfloat16
    r = _lib.segpaged_rope_realign(ctypes.byref(dims.c()), _dev(cu_seqlens_k, torch.int32, "cu_seqlens_k"),
                                   _dev(q_len, torch.int32, "q_len"), _dev(cls, torch.int32, "cls"),
                                   _dev(page_table, torch.int32, "page_table"),
                                   _dev(page_table_offs, torch.int32, "page_table_offs"),
                                   _dev(frag_offs, torch.int32, "frag_offs"), _dev(frag_start, torch.int32, "frag_start"),
                                   _dev(frag_cos_sin, torch.float32, "frag_cos_sin"), _dev(k_pool, bf, "k_pool"),
                                   _dev(k_pool_out, bf, "k_pool_out"), _dev(status, torch.int32, "status"),
                                   _stream(stream))
    if r < 0:
        raise SegPagedError(r, "segpaged_rope_realign")


def segpaged_attn_prefill_rope(dims: Dims, q, k_pool, v_pool, page_table, plan, info: dict, softmax_scale, frag_offs,
                               frag_start, frag_cos_sin, o, lse, workspace, status=None, stream=None):
    """segpaged_attn_prefill with gather-time RoPE re-alignment per sequence fragment. frag_offs int32 [B+1],
    frag_start int32 [F], frag_cos_sin float32 [F, D/2, 2] (CUDA tensors)."""
    bf = torch.bfloat16
    r = _lib.segpaged_attn_prefill_rope(ctypes.byref(dims.c()), _dev(q, bf, "q"), int(q.shape[0]),
                                        _dev(k_pool, bf, "k_pool"), _dev(v_pool, bf, "v_pool"),
                                        _dev(page_table, torch.int32, "page_table"), int(page_table.numel()),
                                        _dev(plan, torch.int32, "plan"), ctypes.byref(_info(info)), float(softmax_scale),
                                        _dev(frag_offs, torch.int32, "frag_offs"),
                                        _dev(frag_start, torch.int32, "frag_start"),
                                        _dev(frag_cos_sin, torch.float32, "frag_cos_sin"), _dev(o, bf, "o"),
                                        _dev(lse, torch.float32, "lse"), _dev(workspace, None, "workspace"),
                                        int(workspace.numel() * workspace.element_size()),
                                        _dev(status, torch.int32, "status"), _stream(stream))
    if r < 0:
        raise SegPagedError(r, "segpaged_attn_prefill_rope")


NOALLOC_MAX_UNITS = 16384


def segpaged_attn_prefill_noalloc(dims: Dims, q, k_pool, v_pool, page_table, units_host, softmax_scale, o, lse,
                                  status=None, stream=None):
    """segpaged_attn_prefill for callers that cannot allocate device memory: the plan comes straight from
    the host (int32 [n, 32] records from segpaged_prefill_plan) and the library's own static device array
    holds it and the work counter. At most NOALLOC_MAX_UNITS units, from a plan made with split_ctas = 0;
    calls that overlap on the GPU race."""
    bf = torch.bfloat16
    units = np.ascontiguousarray(np.asarray(units_host, dtype=np.int32).reshape(-1, UNIT_FIELDS))
    r = _lib.segpaged_attn_prefill_noalloc(ctypes.byref(dims.c()), _dev(q, bf, "q"), int(q.shape[0]),
                                           _dev(k_pool, bf, "k_pool"), _dev(v_pool, bf, "v_pool"),
                                           _dev(page_table, torch.int32, "page_table"), int(page_table.numel()),
                                           _hp(units), int(units.shape[0]), float(softmax_scale), _dev(o, bf, "o"),
                                           _dev(lse, torch.float32, "lse"), _dev(status, torch.int32, "status"),
                                           _stream(stream))
    if r < 0:
        raise SegPagedError(r, "segpaged_attn_prefill_noalloc")


def segpaged_mass_plan(dims: Dims, ctx_len, q_len, cls, page_table_offs) -> np.ndarray:
    """Work items (int32 [n, 16]) of segpaged_token_mass, longest first. Host only."""
    B, H = dims.num_seqs, dims.num_kv_heads
    L, Lq = _host_i32(ctx_len, B), _host_i32(q_len, B)
    c, offs = _host_i32(cls, B * H * 3), _host_i32(page_table_offs, B * H + 1)
    d = dims.c()
    n = _lib.segpaged_mass_plan(ctypes.byref(d), _hp(L), _hp(Lq), _hp(c), _hp(offs), None, 0)
    if n < 0:
        raise SegPagedError(int(n), "segpaged_mass_plan")
    items = np.zeros((max(n, 1), MASS_ITEM_FIELDS), np.int32)
    n2 = _lib.segpaged_mass_plan(ctypes.byref(d), _hp(L), _hp(Lq), _hp(c), _hp(offs), _hp(items), n)
    if n2 < 0:
        raise SegPagedError(int(n2), "segpaged_mass_plan")
    return items[:n]


def segpaged_mass_workspace_bytes(dims: Dims, total_q: int) -> int:
    return int(_lib.segpaged_mass_workspace_bytes(ctypes.byref(dims.c()), int(total_q)))


def segpaged_token_mass(dims: Dims, q, k_pool, page_table, items, lse, softmax_scale, mass, workspace, status=None,
                        stream=None, frags=None):
    """mass [total_q] float32 (CUDA), written in place: the attention mass each query row's token receives.
    items: the mass plan on the device; lse: the prefill's LSE [Hq, total_q] for the same inputs; frags:
    (frag_offs, frag_start, frag_cos_sin) of a gather-time RoPE prefill, or None."""
    bf = torch.bfloat16
    fo, fs, fc = frags if frags is not None else (None, None, None)
    r = _lib.segpaged_token_mass(ctypes.byref(dims.c()), _dev(q, bf, "q"), int(q.shape[0]), _dev(k_pool, bf, "k_pool"),
                                 _dev(page_table, torch.int32, "page_table"), int(page_table.numel()),
                                 _dev(items, torch.int32, "items"), int(items.shape[0]), _dev(lse, torch.float32, "lse"),
                                 float(softmax_scale), _dev(fo, torch.int32, "frag_offs"),
                                 _dev(fs, torch.int32, "frag_start"), _dev(fc, torch.float32, "frag_cos_sin"),
                                 _dev(mass, torch.float32, "mass"),
                                 _dev(workspace, None, "workspace"), int(workspace.numel() * workspace.element_size()),
                                 _dev(status, torch.int32, "status"), _stream(stream))
    if r < 0:
        raise SegPagedError(r, "segpaged_token_mass")


def segpaged_select_topk(mass, cu_seqlens_q, k_per_seq, selected, stream=None):
    """Top-k rows per sequence by mass into `selected` (int32, CUDA), ascending within each sequence."""
    r = _lib.segpaged_select_topk(int(cu_seqlens_q.numel()) - 1, _dev(mass, torch.float32, "mass"),
                                  _dev(cu_seqlens_q, torch.int32, "cu_seqlens_q"),
                                  _dev(k_per_seq, torch.int32, "k_per_seq"), _dev(selected, torch.int32, "selected"),
                                  _stream(stream))
    if r < 0:
        raise SegPagedError(r, "segpaged_select_topk")
