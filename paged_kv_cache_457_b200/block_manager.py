"""Python view of the native page pool (``include/pa_block_manager.h``).

Argument marshalling only: the free lists, reference counts, copy-on-write
decisions, swap plans and step tables are all computed by the C++ manager
inside ``libpa_b200.so``.  Arrays are numpy (host) arrays; the caller moves
them to the device and applies the copies with ``copy_blocks`` /
``swap_blocks`` before the step's ``write_kv``.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import numpy as np

ERRORS = {
    -20: "bad argument", -21: "not enough free pages", -22: "unknown sequence", -23: "sequence exists",
    -24: "sequence is in the other pool", -25: "output array or table stride too small",
    -26: "host memory for the bookkeeping ran out",
}
NO_SPACE = -21


class BlockManagerError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {ERRORS.get(code, code)} ({code})")
        self.code = code


def bind(lib: ctypes.CDLL) -> None:
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    p64 = ctypes.POINTER(ctypes.c_int64)
    sig = {
        "pa_bm_create": (vp, [i32, i64, i64]),
        "pa_bm_destroy": (None, [vp]),
        "pa_bm_num_free_device_blocks": (i64, [vp]),
        "pa_bm_num_free_host_blocks": (i64, [vp]),
        "pa_bm_ref_count": (i32, [vp, i32, i64]),
        "pa_bm_add_sequence": (ctypes.c_int, [vp, i64, i64]),
        "pa_bm_fork": (ctypes.c_int, [vp, i64, i64]),
        "pa_bm_free_sequence": (ctypes.c_int, [vp, i64]),
        "pa_bm_num_tokens": (i64, [vp, i64]),
        "pa_bm_is_swapped": (ctypes.c_int, [vp, i64]),
        "pa_bm_block_table": (ctypes.c_int, [vp, i64, vp, i64, p64]),
        "pa_bm_slots": (ctypes.c_int, [vp, i64, i64, i64, vp]),
        "pa_bm_append_slot": (ctypes.c_int, [vp, i64, p64, p64, p64]),
        "pa_bm_build_decode_step": (ctypes.c_int, [vp, vp, i64, i64, vp, vp, vp, vp, i64, p64]),
        "pa_bm_build_prefill_step": (ctypes.c_int, [vp, vp, vp, i64, i64, vp, vp, vp, vp, i64, vp, i64, p64]),
        "pa_bm_step_needs": (ctypes.c_int, [vp, vp, vp, i64, p64, p64]),
        "pa_bm_swap_out": (ctypes.c_int, [vp, vp, i64, vp, i64, p64]),
        "pa_bm_swap_in": (ctypes.c_int, [vp, vp, i64, vp, i64, p64]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args


@dataclass
class DecodeStepPlan:
    """Host arrays of one decode step, as the kernels take them."""
    block_tables: np.ndarray   # int32 [S, table_stride], -1 padded
    context_lens: np.ndarray   # int32 [S], including the new token
    slot_mapping: np.ndarray   # int64 [S], the new token's slot
    copy_pairs: np.ndarray     # int64 [n, 2], copy-on-write pairs to apply first


@dataclass
class PrefillStepPlan:
    """Host arrays of one prefill (or chunked-prefill) step, as pa_write_kv and pa_prefill take them."""
    block_tables: np.ndarray   # int32 [S, table_stride], -1 padded
    query_start: np.ndarray    # int32 [S + 1], prefix sum of the new tokens
    context_lens: np.ndarray   # int32 [S], including the new tokens
    slot_mapping: np.ndarray   # int64 [total new tokens], row order
    copy_pairs: np.ndarray     # int64 [n, 2], copy-on-write pairs to apply first


def _p(a: np.ndarray):
    return a.ctypes.data if a.size else None


class BlockManager:
    """Reference-counted page pool over a device pool and a host (swap) pool."""

    def __init__(self, block_size: int, num_device_blocks: int, num_host_blocks: int = 0):
        from . import load_library
        self._lib = load_library()
        self._h = self._lib.pa_bm_create(int(block_size), int(num_device_blocks), int(num_host_blocks))
        if not self._h:
            raise BlockManagerError(-20, "pa_bm_create")
        self.block_size = int(block_size)
        self.num_device_blocks = int(num_device_blocks)
        self.num_host_blocks = int(num_host_blocks)

    def close(self) -> None:
        if getattr(self, "_h", None):
            self._lib.pa_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    def _check(self, rc: int, what: str) -> None:
        if rc != 0:
            raise BlockManagerError(rc, what)

    # ---- state
    @property
    def num_free_device_blocks(self) -> int:
        return int(self._lib.pa_bm_num_free_device_blocks(self._h))

    @property
    def num_free_host_blocks(self) -> int:
        return int(self._lib.pa_bm_num_free_host_blocks(self._h))

    def ref_count(self, block: int, host: bool = False) -> int:
        return int(self._lib.pa_bm_ref_count(self._h, int(bool(host)), int(block)))

    def num_tokens(self, seq_id: int) -> int:
        n = int(self._lib.pa_bm_num_tokens(self._h, int(seq_id)))
        self._check(min(n, 0), "pa_bm_num_tokens")
        return n

    def is_swapped(self, seq_id: int) -> bool:
        r = int(self._lib.pa_bm_is_swapped(self._h, int(seq_id)))
        self._check(min(r, 0), "pa_bm_is_swapped")
        return bool(r)

    def block_table(self, seq_id: int) -> np.ndarray:
        n = ctypes.c_int64(0)
        rc = self._lib.pa_bm_block_table(self._h, int(seq_id), None, 0, ctypes.byref(n))
        if rc not in (0, -25):
            self._check(rc, "pa_bm_block_table")
        out = np.empty(n.value, dtype=np.int32)
        self._check(self._lib.pa_bm_block_table(self._h, int(seq_id), _p(out), n.value, ctypes.byref(n)),
                    "pa_bm_block_table")
        return out

    def slots(self, seq_id: int, first: int, count: int) -> np.ndarray:
        out = np.empty(int(count), dtype=np.int64)
        self._check(self._lib.pa_bm_slots(self._h, int(seq_id), int(first), int(count), _p(out)), "pa_bm_slots")
        return out

    # ---- lifecycle
    def add_sequence(self, seq_id: int, num_tokens: int) -> None:
        self._check(self._lib.pa_bm_add_sequence(self._h, int(seq_id), int(num_tokens)), "pa_bm_add_sequence")

    def fork(self, parent_id: int, child_id: int) -> None:
        self._check(self._lib.pa_bm_fork(self._h, int(parent_id), int(child_id)), "pa_bm_fork")

    def free_sequence(self, seq_id: int) -> None:
        self._check(self._lib.pa_bm_free_sequence(self._h, int(seq_id)), "pa_bm_free_sequence")

    def append_slot(self, seq_id: int):
        """Reserve the next token's slot; returns (slot, (copy_src, copy_dst) or None)."""
        slot, src, dst = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        self._check(self._lib.pa_bm_append_slot(self._h, int(seq_id), ctypes.byref(slot), ctypes.byref(src),
                                                ctypes.byref(dst)), "pa_bm_append_slot")
        return slot.value, ((src.value, dst.value) if src.value >= 0 else None)

    def build_decode_step(self, seq_ids, table_stride: int) -> DecodeStepPlan:
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        S = len(ids)
        tables = np.empty((S, int(table_stride)), dtype=np.int32)
        lens = np.empty(S, dtype=np.int32)
        slots = np.empty(S, dtype=np.int64)
        pairs = np.empty((S, 2), dtype=np.int64)
        n = ctypes.c_int64(0)
        self._check(self._lib.pa_bm_build_decode_step(self._h, _p(ids), S, int(table_stride), _p(tables), _p(lens),
                                                      _p(slots), _p(pairs), S, ctypes.byref(n)),
                    "pa_bm_build_decode_step")
        return DecodeStepPlan(tables, lens, slots, pairs[: n.value].copy())

    def build_prefill_step(self, seq_ids, new_tokens, table_stride: int) -> PrefillStepPlan:
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n_new = np.ascontiguousarray(new_tokens, dtype=np.int64)
        S = len(ids)
        if len(n_new) != S:
            raise BlockManagerError(-20, "pa_bm_build_prefill_step")
        total = int(n_new.sum()) if S else 0
        tables = np.empty((S, int(table_stride)), dtype=np.int32)
        qs = np.empty(S + 1, dtype=np.int32)
        lens = np.empty(S, dtype=np.int32)
        slots = np.empty(max(total, 0), dtype=np.int64)
        pairs = np.empty((S, 2), dtype=np.int64)
        n = ctypes.c_int64(0)
        self._check(self._lib.pa_bm_build_prefill_step(self._h, _p(ids), _p(n_new), S, int(table_stride), _p(tables),
                                                       _p(qs), _p(lens), _p(slots), slots.size, _p(pairs), S,
                                                       ctypes.byref(n)),
                    "pa_bm_build_prefill_step")
        return PrefillStepPlan(tables, qs, lens, slots, pairs[: n.value].copy())

    def step_needs(self, seq_ids, new_tokens) -> tuple:
        """(fresh device pages, copy-on-write pairs) a step would take; nothing changes."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n_new = np.ascontiguousarray(new_tokens, dtype=np.int64)
        if len(n_new) != len(ids):
            raise BlockManagerError(-20, "pa_bm_step_needs")
        pages, copies = ctypes.c_int64(0), ctypes.c_int64(0)
        self._check(self._lib.pa_bm_step_needs(self._h, _p(ids), _p(n_new), len(ids), ctypes.byref(pages),
                                               ctypes.byref(copies)), "pa_bm_step_needs")
        return pages.value, copies.value

    def _move(self, fn, seq_ids, what):
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ctypes.c_int64(0)
        cap = sum(len(self.block_table(int(i))) for i in ids) if len(ids) else 0
        mapping = np.empty((max(cap, 0), 2), dtype=np.int64)
        self._check(fn(self._h, _p(ids), len(ids), _p(mapping), cap, ctypes.byref(n)), what)
        return mapping[: n.value].copy()

    def swap_out(self, seq_ids) -> np.ndarray:
        """Move sequences to the host pool; returns the (device, host) page pairs to copy."""
        return self._move(self._lib.pa_bm_swap_out, seq_ids, "pa_bm_swap_out")

    def swap_in(self, seq_ids) -> np.ndarray:
        """Bring sequences back; returns the (host, device) page pairs to copy."""
        return self._move(self._lib.pa_bm_swap_in, seq_ids, "pa_bm_swap_in")
