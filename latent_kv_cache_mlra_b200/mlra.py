"""ctypes binding of libmlra.so (declared in include/mlra.h).

Argument marshalling only: every step of the decode runs in the library's CUDA kernels.
PyTorch provides device memory and the current stream.  There is no fallback: if the
library is missing, loading it raises.
"""
from __future__ import annotations

import ctypes
import math
import pathlib
from typing import Optional

import torch

LIB_PATH = pathlib.Path(__file__).resolve().parent / "libmlra.so"

MLRA_OK, MLRA_ERR_INVALID_ARG, MLRA_ERR_UNSUPPORTED, MLRA_ERR_CUDA = 0, 1, 2, 3
MLRA_ERR_TIMEOUT, MLRA_ERR_WORKSPACE, MLRA_ERR_BAD_PAGE, MLRA_ERR_BAD_LENGTH = 4, 5, 6, 7
MLRA_ERR_SCRATCH_LIMIT = 8
STATIC_SCRATCH_BYTES = 16 * 1024 * 1024
MLRA_BF16, MLRA_F32 = 0, 1
MLRA_OUT_BRANCHES, MLRA_OUT_SUMMED = 0, 1
FLAG_TIMEOUT, FLAG_BAD_PAGE, FLAG_BAD_LENGTH = 0x1, 0x2, 0x4

# Every entry point of include/mlra.h.
EXPORTS = ("mlra_workspace_size", "mlra_decode", "mlra_decode_profiled", "mlra_query_plan",
           "mlra_decode_static_scratch",
           "mlra_read_status", "mlra_debug_resolve_rows", "mlra_plan_host",
           "mlra_plan_segments_host", "mlra_project", "mlra_pack_wuv", "mlra_absorb",
           "mlra_pack_wuk", "mlra_rope_append", "mlra_decode_multi", "mlra_workspace_size_multi",
           "mlra_decode_project", "mlra_workspace_size_project", "mlra_status_string",
           "mlra_version")


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("heads", ctypes.c_int), ("num_branches", ctypes.c_int),
                ("d_latent", ctypes.c_int), ("d_rope", ctypes.c_int), ("page_size", ctypes.c_int),
                ("max_pages_per_seq", ctypes.c_int), ("max_seq_len", ctypes.c_int),
                ("cache_rows", ctypes.c_longlong), ("c_row_stride", ctypes.c_longlong),
                ("kr_row_stride", ctypes.c_longlong), ("dtype", ctypes.c_int),
                ("out_mode", ctypes.c_int), ("num_ranges", ctypes.c_int)]


class Scales(ctypes.Structure):
    _fields_ = [("softmax_scale", ctypes.c_float), ("branch_scale", ctypes.c_float)]


class PlanInfo(ctypes.Structure):
    _fields_ = [("repack", ctypes.c_int), ("launches", ctypes.c_int), ("num_ranges", ctypes.c_int),
                ("ctas", ctypes.c_int), ("kernel_branch_width", ctypes.c_int),
                ("branches_per_cta", ctypes.c_int), ("tile", ctypes.c_int),
                ("partial_slots", ctypes.c_longlong), ("segment_cost_tiles", ctypes.c_int),
                ("workspace_bytes", ctypes.c_size_t)]


class MlraError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises ImportError when it has not been built."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m latent_kv_cache_mlra_b200.build` (needs nvcc)")
        L = ctypes.CDLL(str(LIB_PATH))
        vp, i32p, i64p, u32p = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32), \
            ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_uint32)
        L.mlra_workspace_size.argtypes = [ctypes.POINTER(Dims), ctypes.POINTER(ctypes.c_size_t)]
        L.mlra_decode.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_int, ctypes.POINTER(Scales),
                                  vp, vp, ctypes.POINTER(Dims), vp, ctypes.c_size_t, vp]
        L.mlra_decode_profiled.argtypes = L.mlra_decode.argtypes + [vp, vp]
        L.mlra_query_plan.argtypes = [ctypes.POINTER(Dims), ctypes.POINTER(PlanInfo)]
        L.mlra_decode_static_scratch.argtypes = L.mlra_decode.argtypes[:11] + [vp]
        L.mlra_read_status.argtypes = [vp, vp, u32p]
        L.mlra_debug_resolve_rows.argtypes = [vp, vp, ctypes.POINTER(Dims), vp, ctypes.c_int, vp]
        L.mlra_plan_host.argtypes = [i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, i32p, i32p]
        L.mlra_plan_segments_host.argtypes = [i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, i32p,
                                              i32p, i32p, i32p, ctypes.c_int,
                                              ctypes.POINTER(ctypes.c_int)]
        L.mlra_project.argtypes = [vp, vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   vp, vp]
        L.mlra_pack_wuv.argtypes = [vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp]
        L.mlra_absorb.argtypes = L.mlra_project.argtypes
        L.mlra_pack_wuk.argtypes = L.mlra_pack_wuv.argtypes
        L.mlra_rope_append.argtypes = [vp, vp, vp, vp, vp, ctypes.POINTER(Dims), vp, vp, vp,
                                       ctypes.c_double, vp, vp]
        L.mlra_decode_multi.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_int, ctypes.c_int,
                                        ctypes.POINTER(Scales), vp, vp, ctypes.POINTER(Dims), vp,
                                        ctypes.c_size_t, vp]
        L.mlra_workspace_size_multi.argtypes = [ctypes.POINTER(Dims), ctypes.c_int,
                                                ctypes.POINTER(ctypes.c_size_t)]
        L.mlra_workspace_size_project.argtypes = [ctypes.POINTER(Dims), ctypes.POINTER(ctypes.c_size_t)]
        L.mlra_decode_project.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_int, ctypes.POINTER(Scales),
                                          vp, ctypes.c_int, vp, ctypes.POINTER(Dims), vp,
                                          ctypes.c_size_t, vp]
        L.mlra_status_string.argtypes = [ctypes.c_int]
        L.mlra_status_string.restype = ctypes.c_char_p
        L.mlra_version.argtypes = []
        for f in ("mlra_workspace_size", "mlra_decode", "mlra_decode_profiled", "mlra_query_plan",
                  "mlra_decode_static_scratch",
                  "mlra_read_status", "mlra_debug_resolve_rows", "mlra_plan_host",
                  "mlra_plan_segments_host", "mlra_project", "mlra_pack_wuv", "mlra_absorb",
                  "mlra_pack_wuk", "mlra_rope_append", "mlra_decode_multi",
                  "mlra_workspace_size_multi", "mlra_decode_project", "mlra_workspace_size_project"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().mlra_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != MLRA_OK:
        raise MlraError(status, what)


def make_dims(*, batch, heads, num_branches, d_latent, d_rope, max_seq_len, cache_rows,
              c_row_stride=None, kr_row_stride=None, page_size=0, max_pages_per_seq=0,
              dtype="bf16", out_mode="branches", num_ranges=0) -> Dims:
    return Dims(batch, heads, num_branches, d_latent, d_rope, page_size, max_pages_per_seq,
                max_seq_len, cache_rows, c_row_stride if c_row_stride is not None else d_latent,
                kr_row_stride if kr_row_stride is not None else d_rope,
                MLRA_BF16 if dtype == "bf16" else MLRA_F32,
                MLRA_OUT_BRANCHES if out_mode == "branches" else MLRA_OUT_SUMMED, num_ranges)


def workspace_size(dims: Dims) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().mlra_workspace_size(ctypes.byref(dims), ctypes.byref(n)), "mlra_workspace_size")
    return int(n.value)


def query_plan(dims: Dims) -> PlanInfo:
    info = PlanInfo()
    _check(lib().mlra_query_plan(ctypes.byref(dims), ctypes.byref(info)), "mlra_query_plan")
    return info


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def dims_for(q_lat, q_rope, c_kv, k_rope, seq_lens, page_table, num_branches, *, max_seq_len=None,
             page_size=0, out_mode="branches", num_ranges=0) -> Dims:
    """mlra_dims from tensor shapes/strides (q tensors contiguous, cache rows strided)."""
    N, H, d_c = q_lat.shape
    d_R = q_rope.shape[-1]
    if c_kv.stride(-1) != 1 or k_rope.stride(-1) != 1:
        raise ValueError("cache rows must be contiguous in their last dimension")
    dtype = {torch.bfloat16: "bf16", torch.float32: "f32"}[q_lat.dtype]
    if page_table is None:
        if max_seq_len is None:
            max_seq_len = c_kv.shape[0] // N
        return make_dims(batch=N, heads=H, num_branches=num_branches, d_latent=d_c, d_rope=d_R,
                         max_seq_len=max_seq_len, cache_rows=c_kv.shape[0],
                         c_row_stride=c_kv.stride(0), kr_row_stride=k_rope.stride(0), dtype=dtype,
                         out_mode=out_mode, num_ranges=num_ranges)
    max_pages = page_table.shape[1]
    return make_dims(batch=N, heads=H, num_branches=num_branches, d_latent=d_c, d_rope=d_R,
                     max_seq_len=max_seq_len if max_seq_len is not None else max_pages * page_size,
                     cache_rows=c_kv.shape[0], c_row_stride=c_kv.stride(0),
                     kr_row_stride=k_rope.stride(0), page_size=page_size,
                     max_pages_per_seq=max_pages, dtype=dtype, out_mode=out_mode,
                     num_ranges=num_ranges)


def pack_wuv(w_uv: torch.Tensor, stream=None) -> torch.Tensor:
    """Packs the step-3 weights (bf16 [H, d_head, d_latent]) for ``project`` through
    ``mlra_pack_wuv``; the result has the same shape and dtype, packed content."""
    if w_uv.dtype != torch.bfloat16 or w_uv.dim() != 3 or not w_uv.is_contiguous():
        raise ValueError("pack_wuv: contiguous bf16 [H, d_head, d_latent] expected")
    H, d_head, d_latent = w_uv.shape
    packed = torch.empty_like(w_uv)
    st = stream if stream is not None else torch.cuda.current_stream(w_uv.device).cuda_stream
    _check(lib().mlra_pack_wuv(_ptr(w_uv), _ptr(packed), H, d_latent, d_head, ctypes.c_void_p(st)),
           "mlra_pack_wuv")
    return packed


def project(o: torch.Tensor, w_packed: torch.Tensor, y: Optional[torch.Tensor] = None, status=None,
            stream=None) -> torch.Tensor:
    """Step 3 through ``mlra_project``: y[s, h] = W_h @ o[s, h] with o fp32 [N, H, d_latent] from
    ``decode`` in branch mode and ``w_packed`` from ``pack_wuv`` (shape [H, d_head, d_latent]);
    returns y fp32 [N, H, d_head]."""
    N, H, d_latent = o.shape
    d_head = w_packed.shape[1]
    if (o.dtype != torch.float32 or w_packed.dtype != torch.bfloat16
            or w_packed.shape != (H, d_head, d_latent)):
        raise ValueError("project: o fp32 [N, H, d_latent], w_packed bf16 [H, d_head, d_latent]")
    if not (o.is_contiguous() and w_packed.is_contiguous()):
        raise ValueError("project: contiguous tensors expected")
    if y is None:
        y = torch.empty(N, H, d_head, dtype=torch.float32, device=o.device)
    st = stream if stream is not None else torch.cuda.current_stream(o.device).cuda_stream
    _check(lib().mlra_project(_ptr(o), _ptr(w_packed), _ptr(y), N, H, d_latent, d_head,
                              _ptr(status), ctypes.c_void_p(st)), "mlra_project")
    return y


def pack_wuk(w_uk: torch.Tensor, stream=None) -> torch.Tensor:
    """Packs the step-1 weights (bf16 [H, d_head, d_latent], head h's W^UK_{h,b} side by side)
    for ``absorb`` through ``mlra_pack_wuk``; the result has the same shape, packed content."""
    if w_uk.dtype != torch.bfloat16 or w_uk.dim() != 3 or not w_uk.is_contiguous():
        raise ValueError("pack_wuk: contiguous bf16 [H, d_head, d_latent] expected")
    H, d_head, d_latent = w_uk.shape
    packed = torch.empty_like(w_uk)
    st = stream if stream is not None else torch.cuda.current_stream(w_uk.device).cuda_stream
    _check(lib().mlra_pack_wuk(_ptr(w_uk), _ptr(packed), H, d_head, d_latent, ctypes.c_void_p(st)),
           "mlra_pack_wuk")
    return packed


def absorb(q_nope: torch.Tensor, w_packed: torch.Tensor, q_lat: Optional[torch.Tensor] = None,
           status=None, stream=None) -> torch.Tensor:
    """Step 1 through ``mlra_absorb``: q_lat[s, h, b-block] = W^UK_{h,b}^T q_nope[s, h] with
    q_nope fp32 [N, H, d_head] and ``w_packed`` from ``pack_wuk``; returns bf16 [N, H, d_latent]."""
    N, H, d_head = q_nope.shape
    d_latent = w_packed.shape[2]
    if (q_nope.dtype != torch.float32 or w_packed.dtype != torch.bfloat16
            or w_packed.shape != (H, d_head, d_latent) or not q_nope.is_contiguous()):
        raise ValueError("absorb: q_nope fp32 [N, H, d_head], w_packed bf16 [H, d_head, d_latent]")
    if q_lat is None:
        q_lat = torch.empty(N, H, d_latent, dtype=torch.bfloat16, device=q_nope.device)
    st = stream if stream is not None else torch.cuda.current_stream(q_nope.device).cuda_stream
    _check(lib().mlra_absorb(_ptr(q_nope), _ptr(w_packed), _ptr(q_lat), N, H, d_head, d_latent,
                             _ptr(status), ctypes.c_void_p(st)), "mlra_absorb")
    return q_lat


def rope_append(q_rope_in, kr_new, c_new, seq_lens, page_table, c_kv, k_rope, *, max_seq_len=None,
                page_size=0, rope_base=10000.0, q_rope_out=None, status=None, stream=None):
    """RoPE of the new token's query and key and its append to the (bf16) cache at position
    seq_lens[s], through ``mlra_rope_append``; returns the rotated query bf16 [N, H, d_rope]."""
    N, H, d_rope = q_rope_in.shape
    d_latent = c_new.shape[1]
    q_lat_like = torch.empty(N, H, d_latent, dtype=torch.bfloat16, device=c_kv.device)
    q_rope_like = torch.empty(N, H, d_rope, dtype=torch.bfloat16, device=c_kv.device)
    dims = dims_for(q_lat_like, q_rope_like, c_kv, k_rope, seq_lens, page_table, 1,
                    max_seq_len=max_seq_len, page_size=page_size)
    if q_rope_out is None:
        q_rope_out = q_rope_like
    st = stream if stream is not None else torch.cuda.current_stream(c_kv.device).cuda_stream
    _check(lib().mlra_rope_append(_ptr(q_rope_in), _ptr(kr_new), _ptr(c_new), _ptr(seq_lens),
                                  _ptr(page_table), ctypes.byref(dims), _ptr(c_kv), _ptr(k_rope),
                                  _ptr(q_rope_out), float(rope_base), _ptr(status),
                                  ctypes.c_void_p(st)), "mlra_rope_append")
    return q_rope_out


def decode(q_lat, q_rope, c_kv, k_rope, seq_lens, page_table=None, *, num_branches: int,
           softmax_scale: float, branch_scale: Optional[float] = None, out_mode="branches",
           max_seq_len=None, page_size=0, with_lse=False, out=None, lse=None, workspace=None,
           num_ranges=0, stream=None):
    """MLRA step-2 decode attention through ``mlra_decode``.  Returns (out, lse or None).

    q_lat [N, H, d_c], q_rope [N, H, d_R] contiguous; c_kv [rows, >=d_c], k_rope [rows, >=d_R]
    with unit inner stride (may be two column ranges of one tensor); seq_lens int32 [N];
    page_table int32 [N, max_pages] or None.  All on the same CUDA device.
    """
    gamma = 1.0 / num_branches if branch_scale is None else branch_scale
    dims = dims_for(q_lat, q_rope, c_kv, k_rope, seq_lens, page_table, num_branches,
                    max_seq_len=max_seq_len, page_size=page_size, out_mode=out_mode,
                    num_ranges=num_ranges)
    N, H, d_c = q_lat.shape
    width = d_c if out_mode == "branches" else d_c // num_branches
    dev = q_lat.device
    if out is None:
        out = torch.empty(N, H, width, dtype=torch.float32, device=dev)
    if with_lse and lse is None:
        lse = torch.empty(N, H, num_branches, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(workspace_size(dims), dtype=torch.uint8, device=dev)
    st = stream if stream is not None else torch.cuda.current_stream(dev).cuda_stream
    scales = Scales(softmax_scale, gamma)
    _check(lib().mlra_decode(_ptr(q_lat), _ptr(q_rope), _ptr(c_kv), _ptr(k_rope), _ptr(seq_lens),
                             _ptr(page_table), num_branches, ctypes.byref(scales), _ptr(out),
                             _ptr(lse), ctypes.byref(dims), _ptr(workspace), workspace.numel(),
                             ctypes.c_void_p(st)), "mlra_decode")
    return out, lse


def workspace_size_multi(dims: Dims, q_len: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().mlra_workspace_size_multi(ctypes.byref(dims), q_len, ctypes.byref(n)),
           "mlra_workspace_size_multi")
    return n.value


def decode_multi(q_lat, q_rope, c_kv, k_rope, seq_lens, page_table=None, *, num_branches: int,
                 softmax_scale: float, branch_scale: Optional[float] = None, out_mode="branches",
                 max_seq_len=None, page_size=0, with_lse=False, out=None, lse=None,
                 workspace=None, num_ranges=0, stream=None):
    """Decode for the q newest tokens of every sequence through ``mlra_decode_multi``.

    q_lat [N, q, H, d_c], q_rope [N, q, H, d_R] contiguous: token t of sequence s sits at position
    seq_lens[s] - q + t (all q tokens already in the cache) and attends positions up to its own.
    Returns (out [N, q, H, width], lse [N, q, H, B] or None)."""
    N, q, H, d_c = q_lat.shape
    gamma = 1.0 / num_branches if branch_scale is None else branch_scale
    dims = dims_for(q_lat[:, 0], q_rope[:, 0], c_kv, k_rope, seq_lens, page_table, num_branches,
                    max_seq_len=max_seq_len, page_size=page_size, out_mode=out_mode,
                    num_ranges=num_ranges)
    if not (q_lat.is_contiguous() and q_rope.is_contiguous()):
        raise ValueError("decode_multi: contiguous queries expected")
    width = d_c if out_mode == "branches" else d_c // num_branches
    dev = q_lat.device
    if out is None:
        out = torch.empty(N, q, H, width, dtype=torch.float32, device=dev)
    if with_lse and lse is None:
        lse = torch.empty(N, q, H, num_branches, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(workspace_size_multi(dims, q), dtype=torch.uint8, device=dev)
    st = stream if stream is not None else torch.cuda.current_stream(dev).cuda_stream
    scales = Scales(softmax_scale, gamma)
    _check(lib().mlra_decode_multi(_ptr(q_lat), _ptr(q_rope), _ptr(c_kv), _ptr(k_rope),
                                   _ptr(seq_lens), _ptr(page_table), q, num_branches,
                                   ctypes.byref(scales), _ptr(out), _ptr(lse), ctypes.byref(dims),
                                   _ptr(workspace), workspace.numel(), ctypes.c_void_p(st)),
           "mlra_decode_multi")
    return out, lse


def workspace_size_project(dims: Dims) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().mlra_workspace_size_project(ctypes.byref(dims), ctypes.byref(n)),
           "mlra_workspace_size_project")
    return n.value


def decode_project(q_lat, q_rope, c_kv, k_rope, seq_lens, page_table, w_packed, *,
                   num_branches: int, softmax_scale: float, d_head: int = 128,
                   branch_scale: Optional[float] = None, max_seq_len=None, page_size=0, y=None,
                   workspace=None, num_ranges=0, stream=None):
    """``mlra_decode_project``: steps 2 and 3 of one layer in one call (the attention kernel, then
    the step-3 product that merges split sequences itself).  ``w_packed`` from ``pack_wuv``.
    Returns y [N, H, d_head] fp32."""
    gamma = 1.0 / num_branches if branch_scale is None else branch_scale
    dims = dims_for(q_lat, q_rope, c_kv, k_rope, seq_lens, page_table, num_branches,
                    max_seq_len=max_seq_len, page_size=page_size, num_ranges=num_ranges)
    N, H, _ = q_lat.shape
    dev = q_lat.device
    if y is None:
        y = torch.empty(N, H, d_head, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(workspace_size_project(dims), dtype=torch.uint8, device=dev)
    st = stream if stream is not None else torch.cuda.current_stream(dev).cuda_stream
    scales = Scales(softmax_scale, gamma)
    _check(lib().mlra_decode_project(_ptr(q_lat), _ptr(q_rope), _ptr(c_kv), _ptr(k_rope),
                                     _ptr(seq_lens), _ptr(page_table), num_branches,
                                     ctypes.byref(scales), _ptr(w_packed), d_head, _ptr(y),
                                     ctypes.byref(dims), _ptr(workspace), workspace.numel(),
                                     ctypes.c_void_p(st)), "mlra_decode_project")
    return y


def decode_static_scratch(q_lat, q_rope, c_kv, k_rope, seq_lens, page_table=None, *,
                          num_branches: int, softmax_scale: float,
                          branch_scale: Optional[float] = None, out_mode="branches",
                          max_seq_len=None, page_size=0, out=None, lse=None, num_ranges=0,
                          stream=None):
    """``mlra_decode_static_scratch``: the decode without a workspace argument; the library uses
    its built-in scratch array.  ``out`` is allocated here when not given (the C entry point itself
    allocates nothing); ``lse`` is written only when the caller passes an fp32 [N, H, B] tensor,
    else no LSE is computed.  Returns (out, lse or None)."""
    gamma = 1.0 / num_branches if branch_scale is None else branch_scale
    dims = dims_for(q_lat, q_rope, c_kv, k_rope, seq_lens, page_table, num_branches,
                    max_seq_len=max_seq_len, page_size=page_size, out_mode=out_mode,
                    num_ranges=num_ranges)
    N, H, d_c = q_lat.shape
    width = d_c if out_mode == "branches" else d_c // num_branches
    if out is None:
        out = torch.empty(N, H, width, dtype=torch.float32, device=q_lat.device)
    st = stream if stream is not None else torch.cuda.current_stream(q_lat.device).cuda_stream
    scales = Scales(softmax_scale, gamma)
    _check(lib().mlra_decode_static_scratch(
        _ptr(q_lat), _ptr(q_rope), _ptr(c_kv), _ptr(k_rope), _ptr(seq_lens), _ptr(page_table),
        num_branches, ctypes.byref(scales), _ptr(out), _ptr(lse), ctypes.byref(dims),
        ctypes.c_void_p(st)), "mlra_decode_static_scratch")
    return out, lse


class Decoder:
    """Holds the dims, a workspace and outputs for repeated decode calls on fixed shapes."""

    def __init__(self, q_lat, q_rope, c_kv, k_rope, seq_lens, page_table=None, *, num_branches,
                 softmax_scale, branch_scale=None, out_mode="branches", max_seq_len=None,
                 page_size=0, with_lse=False, num_ranges=0):
        self.num_branches = num_branches
        self.scales = Scales(softmax_scale, 1.0 / num_branches if branch_scale is None else branch_scale)
        self.dims = dims_for(q_lat, q_rope, c_kv, k_rope, seq_lens, page_table, num_branches,
                             max_seq_len=max_seq_len, page_size=page_size, out_mode=out_mode,
                             num_ranges=num_ranges)
        N, H, d_c = q_lat.shape
        width = d_c if out_mode == "branches" else d_c // num_branches
        dev = q_lat.device
        self.out = torch.empty(N, H, width, dtype=torch.float32, device=dev)
        self.lse = torch.empty(N, H, num_branches, dtype=torch.float32, device=dev) if with_lse else None
        self.workspace = torch.empty(workspace_size(self.dims), dtype=torch.uint8, device=dev)
        self.args = (q_lat, q_rope, c_kv, k_rope, seq_lens, page_table)

        self.plan = query_plan(self.dims)

    def __call__(self, stream=None, args=None, k1_events=None):
        """One decode call.  ``k1_events`` = (begin, end) torch.cuda.Event pair recorded around
        the attention kernel on the launch stream."""
        q_lat, q_rope, c_kv, k_rope, seq_lens, page_table = self.args if args is None else args
        st = stream if stream is not None else torch.cuda.current_stream(q_lat.device).cuda_stream
        common = (_ptr(q_lat), _ptr(q_rope), _ptr(c_kv), _ptr(k_rope), _ptr(seq_lens),
                  _ptr(page_table), self.num_branches, ctypes.byref(self.scales), _ptr(self.out),
                  _ptr(self.lse), ctypes.byref(self.dims), _ptr(self.workspace),
                  self.workspace.numel(), ctypes.c_void_p(st))
        if k1_events is None:
            _check(lib().mlra_decode(*common), "mlra_decode")
        else:
            _check(lib().mlra_decode_profiled(*common, ctypes.c_void_p(k1_events[0].cuda_event),
                                              ctypes.c_void_p(k1_events[1].cuda_event)),
                   "mlra_decode_profiled")
        return self.out

    def status(self, stream=None):
        """(status code, flag bits) left by the last call; synchronises the stream."""
        flags = ctypes.c_uint32(0)
        st = stream if stream is not None else torch.cuda.current_stream(self.out.device).cuda_stream
        rc = lib().mlra_read_status(_ptr(self.workspace), ctypes.c_void_p(st), ctypes.byref(flags))
        return rc, flags.value


def read_status(workspace: torch.Tensor, stream=None):
    flags = ctypes.c_uint32(0)
    st = stream if stream is not None else torch.cuda.current_stream(workspace.device).cuda_stream
    rc = lib().mlra_read_status(_ptr(workspace), ctypes.c_void_p(st), ctypes.byref(flags))
    return rc, flags.value


def resolve_rows(seq_lens, page_table, dims: Dims, row_pitch: int, stream=None) -> torch.Tensor:
    """Test hook: cache row of every position, computed by the decode kernel's addressing."""
    N = dims.batch
    rows = torch.full((N, row_pitch), -1, dtype=torch.int64, device=seq_lens.device)
    st = stream if stream is not None else torch.cuda.current_stream(seq_lens.device).cuda_stream
    _check(lib().mlra_debug_resolve_rows(_ptr(seq_lens), _ptr(page_table), ctypes.byref(dims),
                                         _ptr(rows), row_pitch, ctypes.c_void_p(st)),
           "mlra_debug_resolve_rows")
    return rows


def plan_host(tiles, num_ranges: int, seg_cost: int = 0):
    """Host replica of the split plan: (first range, number of parts) per sequence."""
    n = len(tiles)
    arr = (ctypes.c_int32 * n)(*[int(t) for t in tiles])
    first, parts = (ctypes.c_int32 * n)(), (ctypes.c_int32 * n)()
    _check(lib().mlra_plan_host(arr, n, num_ranges, seg_cost, first, parts), "mlra_plan_host")
    return list(first), list(parts)


def plan_segments_host(tiles, num_ranges: int, seg_cost: int = 0):
    """Host replica of the kernel's per-CTA segment walk: list of (range, seq, tile0, ntiles)."""
    n = len(tiles)
    arr = (ctypes.c_int32 * n)(*[int(t) for t in tiles])
    count = ctypes.c_int(0)
    _check(lib().mlra_plan_segments_host(arr, n, num_ranges, seg_cost, None, None, None, None, 0,
                                         ctypes.byref(count)), "mlra_plan_segments_host")
    m = count.value
    bufs = [(ctypes.c_int32 * max(m, 1))() for _ in range(4)]
    _check(lib().mlra_plan_segments_host(arr, n, num_ranges, seg_cost, *bufs, m,
                                         ctypes.byref(count)), "mlra_plan_segments_host")
    return [tuple(b[i] for b in bufs) for i in range(m)]


def default_scales(num_branches: int, d_rope: int, head_dim: int = 128):
    """(sigma, gamma) = (1/sqrt(d_h + d_R), 1/B)."""
    return 1.0 / math.sqrt(head_dim + d_rope), 1.0 / num_branches
