"""Python binding over the C ABI in include/mla_decode.h.

Argument marshalling only: torch supplies device memory and the current CUDA
stream; every step of the decode runs in the library's kernels.  There is no
fallback: if the compiled library is missing the import of this module fails,
and on a machine without a CUDA device the compute calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

D_QK = 576
D_V = 512
PAGE = 64
MD_STRIDE = 8

MLA_OK = 0
MLA_ERR_INVALID_ARG = 1
MLA_ERR_UNSUPPORTED = 2
MLA_ERR_CUDA = 3
MLA_ERR_DEVICE_TIMEOUT = 4
MLA_ERR_DEVICE_CHECK = 5
MLA_ERR_SCRATCH_LIMIT = 6
MLA_ERR_NO_FREE_PAGES = 7
STATIC_SCRATCH_BYTES = 48 << 20

EXPORTS = ("mla_metadata_shape", "mla_get_metadata", "mla_workspace_size", "mla_decode_kvcache",
           "mla_decode_kvcache_static_scratch", "mla_append_latent", "mla_release_pages",
           "mla_append_latent_fp8", "mla_decode_kvcache_fp8", "mla_sparse_workspace_size",
           "mla_decode_sparse", "mla_merge_partials", "mla_set_wait_limit_ns",
           "mla_debug_set_stall_flag",
           "mla_error_string", "mla_version")


class MLAError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {error_string(code)}")
        self.code = code


def _load() -> ctypes.CDLL:
    path = os.environ.get("MLA_DECODE_LIB", _build.LIB_PATH)
    if not os.path.exists(path):
        raise ImportError(f"libmla_decode.so not built ({path}); run "
                          "`python -m mla_paged_latent_decode_b200.build`")
    lib = ctypes.CDLL(path)
    p, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                            ctypes.c_size_t)
    ip = ctypes.POINTER(ctypes.c_int)
    lib.mla_metadata_shape.argtypes = [i32, i32, i32, ip, ip]
    lib.mla_metadata_shape.restype = i32
    lib.mla_get_metadata.argtypes = [p, i32, i32, i32, p, p, i32, p]
    lib.mla_get_metadata.restype = i32
    lib.mla_workspace_size.argtypes = [i32, i32, i32, i32, i32]
    lib.mla_workspace_size.restype = sz
    lib.mla_decode_kvcache.argtypes = [p, p, i64, p, i32, p, i32, i32, i32, i32, i32, f32, i32,
                                       p, p, i32, p, sz, p, p, p, p]
    lib.mla_decode_kvcache.restype = i32
    lib.mla_decode_kvcache_static_scratch.argtypes = [p, p, i64, p, i32, p, i32, i32, i32, i32, i32,
                                                      f32, i32, p, p, i32, p, p, p, p]
    lib.mla_decode_kvcache_static_scratch.restype = i32
    lib.mla_append_latent.argtypes = [p, i32, p, i64, p, i32, p, i32, p, i32, p, p, p]
    lib.mla_append_latent.restype = i32
    lib.mla_append_latent_fp8.argtypes = [p, i32, p, p, i64, p, i32, p, i32, p, i32, p, p, p]
    lib.mla_append_latent_fp8.restype = i32
    lib.mla_decode_kvcache_fp8.argtypes = [p, p, p, i64, p, i32, p, i32, i32, i32, i32, i32, f32,
                                           i32, p, p, i32, p, sz, p, p, p, p]
    lib.mla_decode_kvcache_fp8.restype = i32
    lib.mla_sparse_workspace_size.argtypes = [i32, i32, i32, i32, i32]
    lib.mla_sparse_workspace_size.restype = sz
    lib.mla_decode_sparse.argtypes = [p, p, i64, p, i32, p, i32, i32, i32, i32, i32, p, i32, f32,
                                      i32, i32, p, sz, p, p, p, p]
    lib.mla_decode_sparse.restype = i32
    lib.mla_release_pages.argtypes = [p, p, i32, p, i32, p, i32, p, p, p]
    lib.mla_release_pages.restype = i32
    lib.mla_error_string.argtypes = [i32]
    lib.mla_error_string.restype = ctypes.c_char_p
    lib.mla_merge_partials.argtypes = [p, p, i32, i32, i32, i32, p, p, p]
    lib.mla_merge_partials.restype = i32
    lib.mla_debug_set_stall_flag.argtypes = [p]
    lib.mla_debug_set_stall_flag.restype = p
    lib.mla_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.mla_set_wait_limit_ns.restype = ctypes.c_uint64
    lib.mla_version.argtypes = []
    lib.mla_version.restype = ctypes.c_char_p
    return lib


lib = _load()
LIB_PATH = lib._name


def error_string(code: int) -> str:
    return lib.mla_error_string(int(code)).decode()


def version() -> str:
    return lib.mla_version().decode()


def debug_set_stall_flag(flag: torch.Tensor | None):
    """Test hook of the timeout path: the PV issuer of every decode CTA waits for
    flag (a device int32) to become non-zero before its first PV.  None = off."""
    if flag is not None:
        _require(flag.is_cuda and flag.dtype == torch.int32 and flag.numel() >= 1,
                 "flag must be a device int32")
    lib.mla_debug_set_stall_flag(_ptr(flag))


def set_wait_limit_ns(ns: int) -> int:
    """Limit of each bounded wait inside the decode kernels (0 = the 2 s default).
    Returns the previous limit."""
    return int(lib.mla_set_wait_limit_ns(int(ns)))


def _check(code: int, what: str):
    if code != MLA_OK:
        raise MLAError(code, what)


def _require(ok: bool, what: str):
    """Argument check that stays on under `python -O` (unlike assert)."""
    if not ok:
        raise ValueError(f"invalid argument: {what}")


def _shape(t: torch.Tensor, shape, dtype, what: str):
    """t must be a contiguous `dtype` tensor of exactly `shape`."""
    _require(t.dtype == dtype, f"{what} must be {dtype}")
    _require(tuple(t.shape) == tuple(shape), f"{what} must have shape {tuple(shape)}, "
             f"got {tuple(t.shape)}")
    _require(t.is_contiguous(), f"{what} must be contiguous")


def _check_decode_args(q, block_table, cache_seqlens, tile_md, num_splits, out, lse, workspace,
                       device_status, dv, extra=()):
    """Shapes, dtypes and devices of the decode's tensors.  The C ABI sees only
    pointers, so a tensor of the wrong extent would be read or written past its
    end on the device: every extent the kernels rely on is checked here."""
    _require(q.dim() == 4 and q.shape[3] == D_QK, "q must be [batch, s_q, h_q, 576]")
    b, s_q, h_q, _ = q.shape
    _require(q.dtype == torch.bfloat16 and q.is_contiguous(), "q must be contiguous bf16")
    _require(block_table.dim() == 2 and block_table.shape[0] == b and block_table.shape[1] >= 1,
             "block_table must be [batch, max_pages]")
    _require(block_table.dtype == torch.int32 and block_table.is_contiguous(),
             "block_table must be contiguous int32")
    _shape(cache_seqlens, (b,), torch.int32, "cache_seqlens")
    if tile_md is not None:
        _require(tile_md.dim() == 2 and tile_md.shape[1] == MD_STRIDE and tile_md.shape[0] >= 1,
                 "tile_md must be [num_workers, 8]")
        _shape(tile_md, tuple(tile_md.shape), torch.int32, "tile_md")
        _shape(num_splits, (b + 1,), torch.int32, "num_splits")
    if out is not None:
        _shape(out, (b, s_q, h_q, dv), torch.bfloat16, "out")
    if lse is not None:
        _shape(lse, (b, h_q, s_q), torch.float32, "lse")
    if workspace is not None:
        _require(workspace.dtype == torch.uint8 and workspace.dim() == 1 and
                 workspace.is_contiguous(), "workspace must be a contiguous 1-D uint8 tensor")
    if device_status is not None:
        _require(device_status.dtype == torch.int32 and device_status.numel() >= 1 and
                 device_status.is_contiguous(), "device_status must hold one int32")
    dev = q.device
    for t in (block_table, cache_seqlens, tile_md, num_splits, out, lse, workspace,
              device_status, *extra):
        if t is not None:
            _require(t.device == dev, "every tensor must be on q's device")
    return b, s_q, h_q


def _ptr(t: torch.Tensor | None):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream_handle(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def metadata_shape(batch: int, h_q: int, s_q: int) -> tuple[int, int]:
    """(num_workers, md_stride) for the current CUDA device."""
    nw, st = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib.mla_metadata_shape(batch, h_q, s_q, ctypes.byref(nw), ctypes.byref(st)),
           "mla_metadata_shape")
    return nw.value, st.value


def workspace_size(batch: int, s_q: int, h_q: int, num_workers: int, dv: int = D_V) -> int:
    return int(lib.mla_workspace_size(batch, s_q, h_q, dv, num_workers))


def get_mla_metadata(cache_seqlens: torch.Tensor, h_q: int, s_q: int,
                     num_workers: int | None = None):
    """Split-KV tile scheduler.  Returns (tile_md [W, 8] int32, num_splits [b + 1] int32),
    both on cache_seqlens' device, produced on the current stream."""
    _require(cache_seqlens.is_cuda and cache_seqlens.dtype == torch.int32,
             "cache_seqlens must be int32 on a CUDA device")
    _require(cache_seqlens.dim() == 1 and cache_seqlens.is_contiguous(),
             "cache_seqlens must be 1-D and contiguous")
    dev = cache_seqlens.device
    b = cache_seqlens.numel()
    with torch.cuda.device(dev):
        if num_workers is None:
            num_workers, _ = metadata_shape(b, h_q, s_q)
        tile_md = torch.empty((num_workers, MD_STRIDE), dtype=torch.int32, device=dev)
        num_splits = torch.empty((b + 1,), dtype=torch.int32, device=dev)
        _check(lib.mla_get_metadata(_ptr(cache_seqlens), b, h_q, s_q, _ptr(tile_md),
                                    _ptr(num_splits), num_workers, _stream_handle(dev)),
               "mla_get_metadata")
    return tile_md, num_splits


def mla_decode_kvcache(q: torch.Tensor, kcache: torch.Tensor, block_table: torch.Tensor,
                       cache_seqlens: torch.Tensor, dv: int, tile_md: torch.Tensor,
                       num_splits: torch.Tensor, softmax_scale: float, causal: bool = False,
                       out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                       workspace: torch.Tensor | None = None,
                       device_status: torch.Tensor | None = None):
    """Paged MLA decode.  Returns (out [b, s_q, h_q, 512] bf16, lse [b, h_q, s_q] fp32)."""
    b, s_q, h_q = _check_decode_args(q, block_table, cache_seqlens, tile_md, num_splits, out, lse,
                                     workspace, device_status, dv, extra=(kcache,))
    d = D_QK
    dev = q.device
    _require(kcache.dtype == torch.bfloat16 and kcache.is_contiguous(),
             "kcache must be contiguous bf16")
    _require(kcache.dim() == 3 and kcache.shape[1] == PAGE and kcache.shape[2] == d,
             "kcache must be [num_blocks, 64, 576]")
    _require(q.is_cuda, "q must be on a CUDA device")
    num_workers = tile_md.shape[0]
    with torch.cuda.device(dev):
        if out is None:
            out = torch.empty((b, s_q, h_q, dv), dtype=torch.bfloat16, device=dev)
        if lse is None:
            lse = torch.empty((b, h_q, s_q), dtype=torch.float32, device=dev)
        need = workspace_size(b, s_q, h_q, num_workers, dv)
        if workspace is None:
            workspace = torch.empty((max(need, 256),), dtype=torch.uint8, device=dev)
        rc = lib.mla_decode_kvcache(
            _ptr(q), _ptr(kcache), kcache.shape[0], _ptr(block_table), block_table.shape[1],
            _ptr(cache_seqlens), b, s_q, h_q, d, dv, float(softmax_scale), int(bool(causal)),
            _ptr(tile_md), _ptr(num_splits), num_workers, _ptr(workspace), workspace.numel(),
            _ptr(out), _ptr(lse), _ptr(device_status), _stream_handle(dev))
        _check(rc, "mla_decode_kvcache")
    return out, lse


def _check_state(block_table, cache_seqlens, free_pages, free_count, dev, device_status=None):
    for t in (block_table, cache_seqlens, free_pages, free_count):
        _require(t.is_cuda and t.device == dev and t.is_contiguous() and t.dtype == torch.int32,
                 "page-state tensors must be contiguous int32 on one CUDA device")
    _require(block_table.dim() == 2 and block_table.shape[0] == cache_seqlens.numel(),
             "block_table must be [batch, max_pages]")
    _require(free_count.numel() == 1, "free_count must hold one int32")
    if device_status is not None:
        _require(device_status.dtype == torch.int32 and device_status.numel() >= 1 and
                 device_status.is_contiguous() and device_status.device == dev,
                 "device_status must hold one int32 on the cache's device")


def append_latent(rows: torch.Tensor, kcache: torch.Tensor, block_table: torch.Tensor,
                  cache_seqlens: torch.Tensor, free_pages: torch.Tensor, free_count: torch.Tensor,
                  device_status: torch.Tensor | None = None):
    """Append rows [b, s_new, 576] bf16 as the next s_new tokens of every sequence, taking
    64-token pages off the free stack free_pages[:free_count].  Updates kcache, block_table,
    cache_seqlens and free_count in place, on the current stream."""
    b, s_new, d = rows.shape
    dev = rows.device
    _require(rows.dtype == torch.bfloat16 and kcache.dtype == torch.bfloat16,
             "rows and kcache must be bf16")
    _require(rows.is_contiguous() and kcache.is_contiguous() and kcache.device == dev,
             "rows and kcache must be contiguous on one device")
    _require(kcache.dim() == 3 and kcache.shape[1] == PAGE and kcache.shape[2] == d == D_QK,
             "kcache must be [num_blocks, 64, 576] and rows [batch, s_new, 576]")
    _check_state(block_table, cache_seqlens, free_pages, free_count, dev, device_status)
    _require(cache_seqlens.numel() == b, "cache_seqlens must have one entry per sequence")
    with torch.cuda.device(dev):
        _check(lib.mla_append_latent(_ptr(rows), s_new, _ptr(kcache), kcache.shape[0],
                                     _ptr(block_table), block_table.shape[1], _ptr(cache_seqlens),
                                     b, _ptr(free_pages), free_pages.numel(), _ptr(free_count),
                                     _ptr(device_status), _stream_handle(dev)),
               "mla_append_latent")


def release_pages(release_mask: torch.Tensor, block_table: torch.Tensor,
                  cache_seqlens: torch.Tensor, free_pages: torch.Tensor, free_count: torch.Tensor,
                  device_status: torch.Tensor | None = None):
    """Push the pages of every sequence with release_mask[i] != 0 back onto the free stack and
    set its length to 0 (in place, on the current stream)."""
    dev = cache_seqlens.device
    _check_state(block_table, cache_seqlens, free_pages, free_count, dev, device_status)
    _require(release_mask.dtype == torch.int32 and release_mask.device == dev,
             "release_mask must be int32 on the cache's device")
    _require(release_mask.is_contiguous() and release_mask.numel() == cache_seqlens.numel(),
             "release_mask must be contiguous, one entry per sequence")
    with torch.cuda.device(dev):
        _check(lib.mla_release_pages(_ptr(release_mask), _ptr(block_table), block_table.shape[1],
                                     _ptr(cache_seqlens), cache_seqlens.numel(), _ptr(free_pages),
                                     free_pages.numel(), _ptr(free_count), _ptr(device_status),
                                     _stream_handle(dev)),
               "mla_release_pages")


def append_latent_fp8(rows: torch.Tensor, kcache8: torch.Tensor, kscale: torch.Tensor,
                      block_table: torch.Tensor, cache_seqlens: torch.Tensor,
                      free_pages: torch.Tensor, free_count: torch.Tensor,
                      device_status: torch.Tensor | None = None):
    """append_latent for an FP8 cache: rows [b, s_new, 576] bf16 are encoded into E4M3
    codes (kcache8 [nblk, 64, 576] uint8) and per-token scales (kscale [nblk, 64] fp32)."""
    b, s_new, d = rows.shape
    dev = rows.device
    _require(rows.dtype == torch.bfloat16 and rows.is_contiguous() and d == D_QK,
             "rows must be contiguous bf16 [batch, s_new, 576]")
    _require(kcache8.dtype == torch.uint8 and kcache8.is_contiguous() and kcache8.device == dev,
             "kcache8 must be contiguous uint8 on the rows' device")
    _require(kcache8.dim() == 3 and kcache8.shape[1] == PAGE and kcache8.shape[2] == D_QK,
             "kcache8 must be [num_blocks, 64, 576]")
    _require(kscale.dtype == torch.float32 and kscale.is_contiguous() and kscale.device == dev,
             "kscale must be contiguous fp32 on the rows' device")
    _require(tuple(kscale.shape) == tuple(kcache8.shape[:2]), "kscale must be [num_blocks, 64]")
    _check_state(block_table, cache_seqlens, free_pages, free_count, dev, device_status)
    _require(cache_seqlens.numel() == b, "cache_seqlens must have one entry per sequence")
    with torch.cuda.device(dev):
        _check(lib.mla_append_latent_fp8(_ptr(rows), s_new, _ptr(kcache8), _ptr(kscale),
                                         kcache8.shape[0], _ptr(block_table), block_table.shape[1],
                                         _ptr(cache_seqlens), b, _ptr(free_pages),
                                         free_pages.numel(), _ptr(free_count),
                                         _ptr(device_status), _stream_handle(dev)),
               "mla_append_latent_fp8")


def mla_decode_kvcache_fp8(q: torch.Tensor, kcache8: torch.Tensor, kscale: torch.Tensor,
                           block_table: torch.Tensor, cache_seqlens: torch.Tensor, dv: int,
                           tile_md: torch.Tensor, num_splits: torch.Tensor,
                           softmax_scale: float, causal: bool = False,
                           out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                           workspace: torch.Tensor | None = None,
                           device_status: torch.Tensor | None = None):
    """Paged MLA decode over an FP8 cache (codes kcache8 [nblk, 64, 576] uint8 and per-token
    scales kscale [nblk, 64] fp32).  Returns (out [b, s_q, h_q, 512] bf16, lse [b, h_q, s_q])."""
    b, s_q, h_q = _check_decode_args(q, block_table, cache_seqlens, tile_md, num_splits, out, lse,
                                     workspace, device_status, dv, extra=(kcache8, kscale))
    d = D_QK
    dev = q.device
    _require(kcache8.dtype == torch.uint8 and kcache8.is_contiguous(),
             "kcache8 must be contiguous uint8")
    _require(kcache8.dim() == 3 and kcache8.shape[1] == PAGE and kcache8.shape[2] == d,
             "kcache8 must be [num_blocks, 64, 576]")
    _shape(kscale, tuple(kcache8.shape[:2]), torch.float32, "kscale")
    _require(q.is_cuda, "q must be on a CUDA device")
    num_workers = tile_md.shape[0]
    with torch.cuda.device(dev):
        if out is None:
            out = torch.empty((b, s_q, h_q, dv), dtype=torch.bfloat16, device=dev)
        if lse is None:
            lse = torch.empty((b, h_q, s_q), dtype=torch.float32, device=dev)
        need = workspace_size(b, s_q, h_q, num_workers, dv)
        if workspace is None:
            workspace = torch.empty((max(need, 256),), dtype=torch.uint8, device=dev)
        rc = lib.mla_decode_kvcache_fp8(
            _ptr(q), _ptr(kcache8), _ptr(kscale), kcache8.shape[0], _ptr(block_table),
            block_table.shape[1], _ptr(cache_seqlens), b, s_q, h_q, d, dv, float(softmax_scale),
            int(bool(causal)), _ptr(tile_md), _ptr(num_splits), num_workers, _ptr(workspace),
            workspace.numel(), _ptr(out), _ptr(lse), _ptr(device_status), _stream_handle(dev))
        _check(rc, "mla_decode_kvcache_fp8")
    return out, lse


def mla_decode_sparse(q: torch.Tensor, kcache: torch.Tensor, block_table: torch.Tensor,
                      cache_seqlens: torch.Tensor, indices: torch.Tensor, softmax_scale: float,
                      causal: bool = False, dv: int = D_V, out: torch.Tensor | None = None,
                      lse: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                      device_status: torch.Tensor | None = None):
    """Sparse decode: each query position attends to the cached tokens listed in
    indices [b, s_q, topk] int32 (entries outside the sequence, or past the causal
    limit, are skipped).  Returns (out [b, s_q, h_q, 512] bf16, lse [b, h_q, s_q])."""
    b, s_q, h_q = _check_decode_args(q, block_table, cache_seqlens, None, None, out, lse,
                                     workspace, device_status, dv, extra=(kcache, indices))
    d = D_QK
    dev = q.device
    _require(kcache.dtype == torch.bfloat16 and kcache.is_contiguous(),
             "kcache must be contiguous bf16")
    _require(kcache.dim() == 3 and kcache.shape[1] == PAGE and kcache.shape[2] == d,
             "kcache must be [num_blocks, 64, 576]")
    _require(indices.dtype == torch.int32 and indices.dim() == 3 and indices.is_contiguous(),
             "indices must be contiguous int32 [batch, s_q, topk]")
    _require(indices.shape[0] == b and indices.shape[1] == s_q and indices.shape[2] >= 1,
             "indices must be [batch, s_q, topk]")
    _require(q.is_cuda, "q must be on a CUDA device")
    topk = indices.shape[2]
    with torch.cuda.device(dev):
        num_workers, _ = metadata_shape(b * s_q, h_q, 1)
        if out is None:
            out = torch.empty((b, s_q, h_q, dv), dtype=torch.bfloat16, device=dev)
        if lse is None:
            lse = torch.empty((b, h_q, s_q), dtype=torch.float32, device=dev)
        need = int(lib.mla_sparse_workspace_size(b, s_q, h_q, topk, num_workers))
        if need == 0:
            raise MLAError(MLA_ERR_INVALID_ARG, "mla_sparse_workspace_size")
        if workspace is None:
            workspace = torch.empty((need,), dtype=torch.uint8, device=dev)
        rc = lib.mla_decode_sparse(
            _ptr(q), _ptr(kcache), kcache.shape[0], _ptr(block_table), block_table.shape[1],
            _ptr(cache_seqlens), b, s_q, h_q, d, dv, _ptr(indices), topk, float(softmax_scale),
            int(bool(causal)), num_workers, _ptr(workspace), workspace.numel(), _ptr(out),
            _ptr(lse), _ptr(device_status), _stream_handle(dev))
        _check(rc, "mla_decode_sparse")
    return out, lse


def merge_partials(outs: torch.Tensor, lses: torch.Tensor, out: torch.Tensor | None = None,
                   lse: torch.Tensor | None = None):
    """Merge decode results over disjoint parts of the cache by log-sum-exp.
    outs [R, b, s_q, h_q, 512] bf16, lses [R, b, h_q, s_q] fp32 (one entry per part).
    Returns (out [b, s_q, h_q, 512] bf16, lse [b, h_q, s_q] fp32)."""
    _require(outs.dim() == 5 and outs.shape[4] == D_V, "outs must be [parts, b, s_q, h_q, 512]")
    R, b, s_q, h_q, _ = outs.shape
    _shape(outs, (R, b, s_q, h_q, D_V), torch.bfloat16, "outs")
    _shape(lses, (R, b, h_q, s_q), torch.float32, "lses")
    dev = outs.device
    if out is not None:
        _shape(out, (b, s_q, h_q, D_V), torch.bfloat16, "out")
    if lse is not None:
        _shape(lse, (b, h_q, s_q), torch.float32, "lse")
    for t in (lses, out, lse):
        if t is not None:
            _require(t.device == dev, "every tensor must be on outs' device")
    _require(outs.is_cuda, "outs must be on a CUDA device")
    with torch.cuda.device(dev):
        if out is None:
            out = torch.empty((b, s_q, h_q, D_V), dtype=torch.bfloat16, device=dev)
        if lse is None:
            lse = torch.empty((b, h_q, s_q), dtype=torch.float32, device=dev)
        _check(lib.mla_merge_partials(_ptr(outs), _ptr(lses), R, b, s_q, h_q, _ptr(out), _ptr(lse),
                                      _stream_handle(dev)), "mla_merge_partials")
    return out, lse
