"""Cascade decode: the attention of :func:`decode` for batches whose sequences share leading
blocks, with each shared K/V tile read once per group ("4. vLLM核心机制", section 4.2: the blocks
of a shared prefix are named by several block tables).

Argument marshalling only.  The grouping (``pa_find_prefix_groups``) and the work plan
(``pa_cascade_plan``) are computed by the library's host C++; the attention runs in its CUDA
kernels (``pa_decode_cascade``).  A plan depends on the groups, head counts, block size and
``max_context_len`` only, so one plan serves every step until a group changes.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import numpy as np
import torch


class CascadeInfo(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("max_context_len", ctypes.c_int32), ("num_jobs", ctypes.c_int32),
                ("num_prefix_jobs", ctypes.c_int32),
                ("num_members", ctypes.c_int32), ("num_pieces", ctypes.c_int32), ("rows_per_head", ctypes.c_int32),
                ("plan_ints", ctypes.c_int64)]


def bind(lib: ctypes.CDLL) -> None:
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    pinfo = ctypes.POINTER(CascadeInfo)
    sig = {
        "pa_find_prefix_groups": (ctypes.c_int, [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp]),
        "pa_cascade_plan": (ctypes.c_int, [i32, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, i64, pinfo]),
        "pa_cascade_workspace_size": (ctypes.c_size_t, [pinfo, i32]),
        "pa_decode_cascade": (ctypes.c_int, [vp, vp, vp, vp, vp, ctypes.c_float, vp, i32, i64, i32, i64, i64, i32,
                                             vp, pinfo, vp, ctypes.c_size_t, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


@dataclass
class PrefixGroups:
    """Groups of sequences sharing leading blocks: group g is ``members[offsets[g]:offsets[g+1]]``
    (increasing sequence indices) sharing ``prefix_blocks[g]`` blocks."""
    offsets: np.ndarray
    members: np.ndarray
    prefix_blocks: np.ndarray

    @property
    def num_groups(self) -> int:
        return int(self.prefix_blocks.shape[0])


@dataclass
class CascadePlan:
    """A host-built plan: ``plan`` (int32, to be copied to the device) and its sizes ``info``."""
    plan: np.ndarray
    info: CascadeInfo

    def to(self, device) -> torch.Tensor:
        return torch.from_numpy(self.plan).to(device)


def find_prefix_groups(block_tables, context_lens, block_size: int, min_prefix_blocks: int = 1) -> PrefixGroups:
    """Groups of a batch by shared leading blocks, from host copies of its tables and lengths."""
    from . import _check, load_library
    tables = _i32(block_tables)
    lens = _i32(context_lens)
    if tables.ndim != 2 or lens.ndim != 1 or tables.shape[0] != lens.shape[0]:
        raise ValueError("block_tables must be [S, W] and context_lens [S]")
    S, W = tables.shape
    offsets = np.zeros(S + 1, np.int32)
    members = np.zeros(max(S, 1), np.int32)
    prefix = np.zeros(max(S, 1), np.int32)
    ng = ctypes.c_int32(0)
    rc = load_library().pa_find_prefix_groups(tables.ctypes.data, lens.ctypes.data, S, max(W, 1), int(block_size),
                                              int(min_prefix_blocks), offsets.ctypes.data, members.ctypes.data,
                                              prefix.ctypes.data, ctypes.addressof(ng))
    _check(rc, "pa_find_prefix_groups")
    n = ng.value
    return PrefixGroups(offsets[:n + 1].copy(), members[:offsets[n]].copy(), prefix[:n].copy())


def cascade_plan(num_seqs: int, num_q_heads: int, num_kv_heads: int, block_size: int, max_context_len: int,
                 groups: PrefixGroups | None = None, chunk_tokens: int = 0) -> CascadePlan:
    """The work plan of :func:`decode_cascade` for these sizes and groups (host only)."""
    from . import _check, load_library
    lib = load_library()
    if groups is None:
        groups = PrefixGroups(np.zeros(1, np.int32), np.zeros(0, np.int32), np.zeros(0, np.int32))
    off, mem, pre = _i32(groups.offsets), _i32(groups.members), _i32(groups.prefix_blocks)
    ng = int(pre.shape[0])
    info = CascadeInfo()
    args = (int(num_seqs), int(num_q_heads), int(num_kv_heads), int(block_size), int(max_context_len),
            int(chunk_tokens), ng, off.ctypes.data, mem.ctypes.data if mem.size else None, pre.ctypes.data)
    _check(lib.pa_cascade_plan(*args, None, 0, ctypes.byref(info)), "pa_cascade_plan")
    plan = np.zeros(int(info.plan_ints), np.int32)
    _check(lib.pa_cascade_plan(*args, plan.ctypes.data, plan.size, ctypes.byref(info)), "pa_cascade_plan")
    return CascadePlan(plan, info)


def cascade_workspace_size(plan: CascadePlan, head_dim: int) -> int:
    from . import load_library
    return int(load_library().pa_cascade_workspace_size(ctypes.byref(plan.info), int(head_dim)))


def decode_cascade(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_tables: torch.Tensor,
                   context_lens: torch.Tensor, scale: float, plan: CascadePlan, plan_device: torch.Tensor,
                   out: torch.Tensor | None = None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """:func:`decode` through a cascade plan; ``plan_device`` is ``plan.plan`` in device memory."""
    from . import (PagedAttentionError, _DTYPES, _cache_geometry, _check, _need_cuda, _stream, _workspace,
                   load_library)
    dev = k_cache.device
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("block_tables", block_tables),
                    ("context_lens", context_lens), ("plan_device", plan_device)):
        _need_cuda(name, t, dev)
    nb, hkv, bs, d = _cache_geometry(k_cache, v_cache)
    info = plan.info
    S, hq = info.num_seqs, info.num_q_heads
    if q.dim() != 3 or q.dtype != k_cache.dtype or tuple(q.shape) != (S, hq, d) or q.stride(2) != 1 \
            or q.stride(1) != d:
        raise PagedAttentionError("q must be [S, Hq, d] as planned, with the caches' dtype, heads and dims contiguous")
    if info.num_kv_heads != hkv or info.block_size != bs:
        raise PagedAttentionError("the plan was built for other kv heads or block size than the caches have")
    if block_tables.dtype != torch.int32 or block_tables.dim() != 2 or block_tables.shape[0] != S \
            or block_tables.stride(1) != 1:
        raise PagedAttentionError("block_tables must be int32 [S, max_blocks] with contiguous rows")
    if context_lens.dtype != torch.int32 or tuple(context_lens.shape) != (S,) or not context_lens.is_contiguous():
        raise PagedAttentionError("context_lens must be a contiguous int32 [S] tensor")
    if plan_device.dtype != torch.int32 or plan_device.numel() != info.plan_ints or not plan_device.is_contiguous():
        raise PagedAttentionError("plan_device must be the plan's int32 array on the caches' device")
    if out is None:
        out = torch.empty((S, hq, d), dtype=q.dtype, device=dev)
    else:
        _need_cuda("out", out, dev)
        if out.dtype != q.dtype or tuple(out.shape) != (S, hq, d) or out.stride(2) != 1 or out.stride(1) != d:
            raise PagedAttentionError("out must be [S, Hq, d] with q's dtype, heads and dims contiguous")
    lib = load_library()
    stream = _stream(dev)
    if workspace is None:
        workspace = _workspace(dev, stream, int(lib.pa_cascade_workspace_size(ctypes.byref(info), d)))
    rc = lib.pa_decode_cascade(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), block_tables.data_ptr(),
                               context_lens.data_ptr(), float(scale), out.data_ptr(), d, nb,
                               int(block_tables.stride(0)) if S else 1, q.stride(0) if S else hq * d,
                               out.stride(0) if S else hq * d, _DTYPES[q.dtype], plan_device.data_ptr(),
                               ctypes.byref(info), workspace.data_ptr() if workspace is not None else None,
                               workspace.numel() * workspace.element_size() if workspace is not None else 0, stream)
    _check(rc, "pa_decode_cascade")
    return out
