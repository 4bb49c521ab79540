"""Paged decode attention for B200 (sm_100a): Python binding of ``libpa_b200.so``.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels; torch supplies device memory and the current stream.  There is no
CPU fallback: if the library is missing or no GPU is present the calls raise.

* :func:`write_kv` -- slot-mapped scatter of a step's new K/V rows into the
  block pool ("4. vLLM核心机制", section 4.3 with the page layout of 4.2).
* :func:`decode`   -- single-token attention over the block-paged cache through
  per-sequence block tables ("4. vLLM核心机制", section 4.2;
  "vLLM：大型语言模型推理优化的革命性突破", section 2.1).
* :func:`decode_cascade` -- the same attention for batches whose tables share
  leading blocks, each shared tile read once per group ("4. vLLM核心机制",
  section 4.2), with :func:`find_prefix_groups` and :func:`cascade_plan` on the host.

Caches are ``[num_blocks, num_kv_heads, block_size, head_dim]`` float16 or
bfloat16 tensors; ``block_tables`` int32 ``[S, max_blocks]``; ``context_lens``
int32 ``[S]`` (each counts the token written in the same step);
``slot_mapping`` int64 ``[T]`` (negative = skip).
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = [
    "PagedAttentionError", "write_kv", "decode", "decode_workspace_size", "copy_blocks", "swap_blocks", "prefill",
    "device_status", "launch_count", "debug_wait_timeout", "read_bandwidth_probe", "library_path", "load_library", "EXPORTED_SYMBOLS",
    "DEV_ERR_BLOCK_ID", "DEV_ERR_CONTEXT", "DEV_ERR_CONTEXT_HINT", "DEV_ERR_SLOT", "DEV_ERR_TIMEOUT",
    "DEV_ERR_INTERNAL", "BUILD_DEBUG", "build_flags",
    "BlockManager", "BlockManagerError", "DecodeStepPlan", "PrefillStepPlan",
    "DEV_ERR_PLAN", "find_prefix_groups", "cascade_plan", "cascade_workspace_size", "decode_cascade", "PrefixGroups",
    "CascadePlan",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libpa_b200.so")
_lock = threading.Lock()
_lib = None

DEV_ERR_BLOCK_ID = 0x1
DEV_ERR_CONTEXT = 0x2
DEV_ERR_CONTEXT_HINT = 0x4
DEV_ERR_SLOT = 0x8
DEV_ERR_TIMEOUT = 0x10
DEV_ERR_INTERNAL = 0x20
DEV_ERR_PLAN = 0x40
BUILD_DEBUG = 0x1

_DTYPES = {torch.float16: 1, torch.bfloat16: 2}

EXPORTED_SYMBOLS = (
    "pa_write_kv", "pa_decode_workspace_size", "pa_decode",
    "pa_get_device_status", "pa_status_string", "pa_last_cuda_error", "pa_launch_count",
    "pa_debug_wait_timeout", "pa_version", "pa_decode_static_workspace", "pa_copy_blocks", "pa_swap_blocks",
    "pa_bm_create", "pa_bm_destroy", "pa_bm_num_free_device_blocks", "pa_bm_num_free_host_blocks",
    "pa_bm_ref_count", "pa_bm_add_sequence", "pa_bm_fork", "pa_bm_free_sequence", "pa_bm_num_tokens",
    "pa_bm_is_swapped", "pa_bm_block_table", "pa_bm_slots", "pa_bm_append_slot", "pa_bm_build_decode_step", "pa_bm_build_prefill_step", "pa_bm_step_needs",
    "pa_bm_swap_out", "pa_bm_swap_in", "pa_prefill", "pa_read_bandwidth_probe", "pa_build_flags",
    "pa_find_prefix_groups", "pa_cascade_plan", "pa_cascade_workspace_size", "pa_decode_cascade",
)


class PagedAttentionError(RuntimeError):
    pass


def library_path() -> str:
    """The library this process loads: ``PA_B200_LIBRARY`` if set (e.g. the PA_DEBUG build,
    ``libpa_b200_debug.so``), else the in-tree release build."""
    return os.environ.get("PA_B200_LIBRARY") or _LIB_PATH


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load (once) and type the C ABI.  Raises if the library has not been built."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or library_path()
        if not os.path.exists(p):
            raise PagedAttentionError(
                f"CUDA library {p} is missing; build it with `python -m paged_kv_cache_457_b200.build_lib`")
        lib = ctypes.CDLL(p)
        vp, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        lib.pa_write_kv.restype = ctypes.c_int
        lib.pa_write_kv.argtypes = [vp, vp, vp, vp, vp, i64, i32, i32, i32, i64, i64, i64, i32, vp]
        lib.pa_decode_workspace_size.restype = sz
        lib.pa_decode_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32, i32]
        lib.pa_decode.restype = ctypes.c_int
        lib.pa_decode.argtypes = [vp, vp, vp, vp, vp, f32, vp, i32, i32, i32, i32, i32, i64, i32, i32, i64, i64,
                                  i32, i32, vp, sz, vp]
        lib.pa_get_device_status.restype = ctypes.c_int
        lib.pa_get_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint32), i32, vp]
        lib.pa_status_string.restype = ctypes.c_char_p
        lib.pa_status_string.argtypes = [i32]
        lib.pa_last_cuda_error.restype = ctypes.c_char_p
        lib.pa_last_cuda_error.argtypes = []
        lib.pa_launch_count.restype = ctypes.c_uint64
        lib.pa_launch_count.argtypes = []
        lib.pa_debug_wait_timeout.restype = ctypes.c_int
        lib.pa_debug_wait_timeout.argtypes = [i64, vp]
        lib.pa_decode_static_workspace.restype = ctypes.c_int
        lib.pa_decode_static_workspace.argtypes = [vp, vp, vp, vp, vp, f32, vp, i32, i32, i32, i32, i32, i64, i32,
                                                   i32, i64, i64, i32, i32, vp]
        lib.pa_copy_blocks.restype = ctypes.c_int
        lib.pa_copy_blocks.argtypes = [vp, vp, vp, i64, i32, i32, i32, i64, vp]
        lib.pa_swap_blocks.restype = ctypes.c_int
        lib.pa_swap_blocks.argtypes = [vp, vp, vp, vp, vp, i64, i32, i32, i32, i64, i64, vp]
        lib.pa_prefill.restype = ctypes.c_int
        lib.pa_prefill.argtypes = [vp, vp, vp, vp, vp, vp, f32, vp, i32, i64, i32, i32, i32, i32, i64, i32, i32, i64,
                                   i64, i32, vp]
        lib.pa_read_bandwidth_probe.restype = ctypes.c_int
        lib.pa_read_bandwidth_probe.argtypes = [vp, i64, vp, vp]
        lib.pa_build_flags.restype = ctypes.c_uint32
        lib.pa_build_flags.argtypes = []
        lib.pa_version.restype = i32
        lib.pa_version.argtypes = []
        from .block_manager import bind as _bind_block_manager
        from .cascade import bind as _bind_cascade
        _bind_block_manager(lib)
        _bind_cascade(lib)
        if path is None:
            _lib = lib
        return lib


def _check(rc: int, what: str) -> None:
    if rc != 0:
        lib = load_library()
        msg = lib.pa_status_string(rc).decode()
        if rc == -9:
            msg += ": " + lib.pa_last_cuda_error().decode()
        raise PagedAttentionError(f"{what} failed ({rc}): {msg}")


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _need_cuda(name: str, t: torch.Tensor, device=None) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise PagedAttentionError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise PagedAttentionError(f"{name} is on {t.device}, expected {device}")


def _cache_geometry(k_cache: torch.Tensor, v_cache: torch.Tensor):
    if k_cache.dim() != 4 or k_cache.shape != v_cache.shape:
        raise PagedAttentionError("k_cache/v_cache must both be [num_blocks, num_kv_heads, block_size, head_dim]")
    if not (k_cache.is_contiguous() and v_cache.is_contiguous()):
        raise PagedAttentionError("caches must be contiguous")
    if k_cache.dtype not in _DTYPES or v_cache.dtype != k_cache.dtype:
        raise PagedAttentionError("caches must be float16 or bfloat16 (same dtype)")
    return tuple(int(x) for x in k_cache.shape)


def write_kv(k: torch.Tensor, v: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
             slot_mapping: torch.Tensor) -> None:
    """Store k[t], v[t] ([T, Hkv, d], heads contiguous) at slot_mapping[t] of the caches, in place."""
    dev = k_cache.device
    for name, t in (("k", k), ("v", v), ("k_cache", k_cache), ("v_cache", v_cache), ("slot_mapping", slot_mapping)):
        _need_cuda(name, t, dev)
    nb, hkv, bs, d = _cache_geometry(k_cache, v_cache)
    T = int(slot_mapping.shape[0])
    if slot_mapping.dtype != torch.int64 or slot_mapping.dim() != 1 or not slot_mapping.is_contiguous():
        raise PagedAttentionError("slot_mapping must be a contiguous int64 [T] tensor")
    for name, t in (("k", k), ("v", v)):
        if t.dtype != k_cache.dtype or t.dim() != 3 or tuple(t.shape) != (T, hkv, d):
            raise PagedAttentionError(f"{name} must be [T, Hkv, d] with the caches' dtype")
        if t.stride(2) != 1 or t.stride(1) != d:
            raise PagedAttentionError(f"{name}: heads and dims must be contiguous within a token")
    lib = load_library()
    rc = lib.pa_write_kv(k.data_ptr(), v.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), slot_mapping.data_ptr(),
                         T, hkv, d, bs, nb, k.stride(0) if T else hkv * d, v.stride(0) if T else hkv * d,
                         _DTYPES[k_cache.dtype], _stream(dev))
    _check(rc, "pa_write_kv")


_workspaces: dict = {}


def decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len,
                          partition_tokens: int = 0) -> int:
    return int(load_library().pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                                       max_context_len, partition_tokens))


def _workspace(dev: torch.device, stream: int, nbytes: int) -> torch.Tensor | None:
    if nbytes == 0:
        return None
    key = (dev.index, stream)
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        _workspaces[key] = ws
    return ws


def decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_tables: torch.Tensor,
           context_lens: torch.Tensor, scale: float, max_context_len: int | None = None,
           out: torch.Tensor | None = None, partition_tokens: int = 0,
           workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Attention of q ([S, Hq, d]) over each sequence's paged K/V; returns out ([S, Hq, d], q's dtype).

    ``max_context_len`` is a host-side bound of ``context_lens`` (it sizes the split along
    the context); when omitted it is read from the device, which synchronises.
    """
    dev = k_cache.device
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("block_tables", block_tables),
                    ("context_lens", context_lens)):
        _need_cuda(name, t, dev)
    nb, hkv, bs, d = _cache_geometry(k_cache, v_cache)
    if q.dim() != 3 or q.dtype != k_cache.dtype or q.shape[2] != d or q.stride(2) != 1 or q.stride(1) != d:
        raise PagedAttentionError("q must be [S, Hq, d] with the caches' dtype, heads and dims contiguous")
    S, hq = int(q.shape[0]), int(q.shape[1])
    if block_tables.dtype != torch.int32 or block_tables.dim() != 2 or block_tables.shape[0] != S \
            or block_tables.stride(1) != 1:
        raise PagedAttentionError("block_tables must be int32 [S, max_blocks] with contiguous rows")
    if context_lens.dtype != torch.int32 or tuple(context_lens.shape) != (S,) or not context_lens.is_contiguous():
        raise PagedAttentionError("context_lens must be a contiguous int32 [S] tensor")
    if out is None:
        out = torch.empty((S, hq, d), dtype=q.dtype, device=dev)
    else:
        _need_cuda("out", out, dev)
        if out.dtype != q.dtype or tuple(out.shape) != (S, hq, d) or out.stride(2) != 1 or out.stride(1) != d:
            raise PagedAttentionError("out must be [S, Hq, d] with q's dtype, heads and dims contiguous")
    if max_context_len is None:
        max_context_len = int(context_lens.max().item()) if S else 0
    stream = _stream(dev)
    lib = load_library()
    need = int(lib.pa_decode_workspace_size(S, hq, hkv, d, bs, int(max_context_len), int(partition_tokens)))
    if workspace is None:
        workspace = _workspace(dev, stream, need)
    rc = lib.pa_decode(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), block_tables.data_ptr(),
                       context_lens.data_ptr(), float(scale), out.data_ptr(), S, hq, hkv, d, bs, nb,
                       int(block_tables.stride(0)) if S else 1, int(max_context_len), q.stride(0) if S else hq * d,
                       out.stride(0) if S else hq * d, int(partition_tokens), _DTYPES[q.dtype],
                       workspace.data_ptr() if workspace is not None else None,
                       workspace.numel() * workspace.element_size() if workspace is not None else 0, stream)
    _check(rc, "pa_decode")
    return out


def prefill(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_tables: torch.Tensor,
            query_start: torch.Tensor, context_lens: torch.Tensor, scale: float, max_query_len: int,
            out: torch.Tensor | None = None) -> torch.Tensor:
    """Causal attention of each sequence's new tokens over its paged context (K/V already written).

    q: [N, Hq, d] (token rows of all sequences, back to back); query_start: int32 [S + 1];
    context_lens: int32 [S] (new tokens included); max_query_len >= every sequence's new tokens.
    """
    dev = k_cache.device
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("block_tables", block_tables),
                    ("query_start", query_start), ("context_lens", context_lens)):
        _need_cuda(name, t, dev)
    nb, hkv, bs, d = _cache_geometry(k_cache, v_cache)
    if q.dim() != 3 or q.shape[2] != d or q.dtype != k_cache.dtype or q.stride(2) != 1 or q.stride(1) != d:
        raise PagedAttentionError("q must be [N, Hq, head_dim] with contiguous heads, same dtype as the caches")
    S = int(context_lens.shape[0])
    for name, t, shape in (("query_start", query_start, (S + 1,)), ("context_lens", context_lens, (S,))):
        if t.dtype != torch.int32 or tuple(t.shape) != shape or not t.is_contiguous():
            raise PagedAttentionError(f"{name} must be a contiguous int32 tensor of shape {shape}")
    if block_tables.dtype != torch.int32 or block_tables.dim() != 2 or block_tables.shape[0] != S \
            or block_tables.stride(1) != 1:
        raise PagedAttentionError("block_tables must be int32 [S, max_blocks] with unit column stride")
    N, hq = int(q.shape[0]), int(q.shape[1])
    if out is None:
        out = torch.empty((N, hq, d), dtype=q.dtype, device=dev)
    else:
        _need_cuda("out", out, dev)
        if tuple(out.shape) != (N, hq, d) or out.dtype != q.dtype or out.stride(2) != 1 or out.stride(1) != d:
            raise PagedAttentionError("out must match q's shape and dtype, heads contiguous")
    rc = load_library().pa_prefill(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), block_tables.data_ptr(),
                                   query_start.data_ptr(), context_lens.data_ptr(), float(scale), out.data_ptr(), S, N,
                                   hq, hkv, d, bs, nb, int(block_tables.stride(0)), int(max_query_len),
                                   int(q.stride(0)), int(out.stride(0)), _DTYPES[k_cache.dtype], _stream(dev))
    _check(rc, "pa_prefill")
    return out


def _mapping(block_mapping: torch.Tensor, device: torch.device) -> torch.Tensor:
    if block_mapping.dtype != torch.int64 or block_mapping.dim() != 2 or block_mapping.shape[1] != 2 \
            or not block_mapping.is_contiguous():
        raise PagedAttentionError("block_mapping must be a contiguous int64 [n, 2] tensor")
    if not block_mapping.is_cuda and not block_mapping.is_pinned():
        raise PagedAttentionError("block_mapping must be on the GPU or in pinned host memory")
    return block_mapping


def copy_blocks(k_cache: torch.Tensor, v_cache: torch.Tensor, block_mapping: torch.Tensor) -> None:
    """Copy block block_mapping[i, 0] to block block_mapping[i, 1] inside the caches (copy-on-write)."""
    dev = k_cache.device
    _need_cuda("k_cache", k_cache, dev)
    _need_cuda("v_cache", v_cache, dev)
    nb, hkv, bs, d = _cache_geometry(k_cache, v_cache)
    m = _mapping(block_mapping, dev)
    rc = load_library().pa_copy_blocks(k_cache.data_ptr(), v_cache.data_ptr(), m.data_ptr(), int(m.shape[0]), hkv, d,
                                       bs, nb, _stream(dev))
    _check(rc, "pa_copy_blocks")


def swap_blocks(src_k: torch.Tensor, src_v: torch.Tensor, dst_k: torch.Tensor, dst_v: torch.Tensor,
                block_mapping: torch.Tensor, device: torch.device | None = None) -> None:
    """Copy blocks between two pools of the same layout; either may be pinned host memory."""
    for name, t in (("src_k", src_k), ("src_v", src_v), ("dst_k", dst_k), ("dst_v", dst_v)):
        if not (t.is_cuda or t.is_pinned()):
            raise PagedAttentionError(f"{name} must be on the GPU or in pinned host memory")
    dev = device or next((t.device for t in (src_k, dst_k) if t.is_cuda), torch.device("cuda", torch.cuda.current_device()))
    snb, hkv, bs, d = _cache_geometry(src_k, src_v)
    dnb = _cache_geometry(dst_k, dst_v)
    if dnb[1:] != (hkv, bs, d) or src_k.dtype != dst_k.dtype:
        raise PagedAttentionError("pools must share heads, block size, head dim and dtype")
    m = _mapping(block_mapping, dev)
    rc = load_library().pa_swap_blocks(src_k.data_ptr(), src_v.data_ptr(), dst_k.data_ptr(), dst_v.data_ptr(),
                                       m.data_ptr(), int(m.shape[0]), hkv, d, bs, snb, dnb[0], _stream(dev))
    _check(rc, "pa_swap_blocks")


def device_status(clear: bool = True, device: torch.device | None = None) -> int:
    """Synchronise the current stream and return (and by default clear) the device status bits."""
    dev = device or torch.device("cuda", torch.cuda.current_device())
    val = ctypes.c_uint32(0)
    _check(load_library().pa_get_device_status(ctypes.byref(val), 1 if clear else 0, _stream(dev)),
           "pa_get_device_status")
    return int(val.value)


def read_bandwidth_probe(buf: torch.Tensor, sink: torch.Tensor) -> None:
    """Stream every byte of ``buf`` (a contiguous CUDA tensor) through the SMs once, read-only;
    ``sink`` is a one-element int32 CUDA tensor the kernel folds the data into."""
    _need_cuda("buf", buf)
    _need_cuda("sink", sink, buf.device)
    if not buf.is_contiguous() or sink.dtype != torch.int32 or sink.numel() < 1:
        raise PagedAttentionError("buf must be contiguous and sink an int32 tensor")
    nbytes = buf.numel() * buf.element_size() // 16 * 16
    _check(load_library().pa_read_bandwidth_probe(buf.data_ptr(), nbytes, sink.data_ptr(), _stream(buf.device)),
           "pa_read_bandwidth_probe")


def build_flags() -> int:
    """BUILD_* bits of the loaded library (BUILD_DEBUG: the PA_DEBUG build)."""
    return int(load_library().pa_build_flags())


def launch_count() -> int:
    return int(load_library().pa_launch_count())


def debug_wait_timeout(limit_ns: int = 10_000_000) -> None:
    dev = torch.device("cuda", torch.cuda.current_device())
    _check(load_library().pa_debug_wait_timeout(int(limit_ns), _stream(dev)), "pa_debug_wait_timeout")


from .block_manager import BlockManager, BlockManagerError, DecodeStepPlan, PrefillStepPlan  # noqa: E402
from .cascade import (CascadePlan, PrefixGroups, cascade_plan, cascade_workspace_size,  # noqa: E402
                      decode_cascade, find_prefix_groups)
