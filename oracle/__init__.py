"""fp64 CPU oracle for paged decode attention and the slot-mapped KV write.

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline leg may call it; the product package never imports it.
It shares no code with the CUDA library: the arithmetic lives in
``pa_oracle.c`` (plain C, double precision), compiled here with gcc and called
through ctypes.  Every function follows the pages on vLLM / PagedAttention
cited in ``pa_oracle.c``:

* ``write_kv``  -- "4. vLLM核心机制", section 4.3 (each iteration yields the
  updated KV cache) with the page layout of section 4.2;
* ``copy_blocks`` -- "4. vLLM核心机制", section 4.2 (a private copy of a shared
  page before a sequence appends to it) and section 4.4 (pages moved to a CPU-side
  pool and back on preemption);
* ``decode``    -- "4. vLLM核心机制", section 4.2 (page table lookup, pages
  anywhere in the pool) and "vLLM：大型语言模型推理优化的革命性突破",
  section 2.1 (no copy, no padding: plain attention over the logical tokens);
* ``prefill``   -- "4. vLLM核心机制", section 4.3 (the prompt enters the cache
  before decoding, possibly in pieces): causal attention of several new
  tokens per sequence over the paged context.

All pins (closed forms, invariants, library special cases, the page-table
worked example) live in ``tests/test_oracle_pins.py``; no function here is
left unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libpa_oracle.so")
_OMP_LIB_PATH = os.path.join(_HERE, "libpa_oracle_omp.so")
_lock = threading.Lock()
_lib = None
_omp_lib = None

DTYPE_CODES = {"fp16": 1, "bf16": 2}

ERRORS = {
    -1: "bad argument",
    -2: "block id out of range",
    -3: "slot out of range",
    -4: "context length out of range",
    -5: "out of memory",
}


def build(src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the C oracle into a shared library (IEEE semantics, no fast-math)."""
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math", "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def build_parallel(src: str = _SRC, out: str = _OMP_LIB_PATH) -> str:
    """Compile the same source with OpenMP: only ``oracle_decode_parallel`` changes, from one
    thread to all the host's cores; its arithmetic per (sequence, query head) is unchanged."""
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math", "-fopenmp", "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _load_parallel() -> ctypes.CDLL:
    global _omp_lib
    with _lock:
        if _omp_lib is None:
            if (not os.path.exists(_OMP_LIB_PATH)) or os.path.getmtime(_OMP_LIB_PATH) < os.path.getmtime(_SRC):
                build_parallel()
            _omp_lib = _bind(ctypes.CDLL(_OMP_LIB_PATH))
        return _omp_lib


def _load(path: str | None = None) -> ctypes.CDLL:
    global _lib
    with _lock:
        if path is not None:
            return _bind(ctypes.CDLL(path))
        if _lib is None:
            if (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
                build()
            _lib = _bind(ctypes.CDLL(_LIB_PATH))
        return _lib


def _bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    p = ctypes.c_void_p
    i64 = ctypes.c_int64
    lib.oracle_write_kv.restype = ctypes.c_int
    lib.oracle_write_kv.argtypes = [p, p, p, p, p, i64, i64, i64, i64, i64]
    lib.oracle_decode.restype = ctypes.c_int
    lib.oracle_decode.argtypes = [p, p, p, p, i64, p, i64, i64, i64, i64, i64, i64, ctypes.c_int,
                                  ctypes.c_double, p]
    lib.oracle_decode_parallel.restype = ctypes.c_int
    lib.oracle_decode_parallel.argtypes = lib.oracle_decode.argtypes
    lib.oracle_parallel_threads.restype = ctypes.c_int
    lib.oracle_parallel_threads.argtypes = []
    lib.oracle_prefill.restype = ctypes.c_int
    lib.oracle_prefill.argtypes = [p, p, p, p, i64, p, p, i64, i64, i64, i64, i64, i64, ctypes.c_int,
                                   ctypes.c_double, p]
    lib.oracle_copy_blocks.restype = ctypes.c_int
    lib.oracle_copy_blocks.argtypes = [p, p, p, p, p, i64, i64, i64, i64, i64, i64]
    lib.oracle_half_to_double.restype = ctypes.c_double
    lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_to_double.restype = ctypes.c_double
    lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
    return lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _u16(a: np.ndarray, name: str) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"{name} must hold uint16 storage bit patterns, got {a.dtype}")
    return np.ascontiguousarray(a)


def widen(bits: int, dtype: str, lib_path: str | None = None) -> float:
    """Value of one fp16/bf16 storage pattern, as the oracle reads it."""
    lib = _load(lib_path)
    if dtype == "fp16":
        return lib.oracle_half_to_double(int(bits))
    return lib.oracle_bf16_to_double(int(bits))


def write_kv(k, v, k_cache, v_cache, slot_mapping, block_size: int, lib_path: str | None = None):
    """Scatter new K/V rows into copies of the caches; returns (k_cache', v_cache').

    k, v: uint16 [T, Hkv, d]; caches: uint16 [NB, Hkv, bs, d]; slot_mapping: int64 [T].
    """
    lib = _load(lib_path)
    k = _u16(k, "k")
    v = _u16(v, "v")
    kc = _u16(k_cache, "k_cache").copy()
    vc = _u16(v_cache, "v_cache").copy()
    slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    T = slots.shape[0]
    nb, hkv, bs, d = kc.shape
    if bs != block_size:
        raise ValueError("cache block dimension does not match block_size")
    if T:
        if k.shape != (T, hkv, d) or v.shape != (T, hkv, d):
            raise ValueError("k/v must be [T, Hkv, d]")
    rc = lib.oracle_write_kv(_ptr(k) if T else None, _ptr(v) if T else None, _ptr(kc), _ptr(vc),
                             _ptr(slots) if T else None, T, hkv, d, bs, nb)
    if rc != 0:
        raise ValueError(f"oracle_write_kv: {ERRORS.get(rc, rc)}")
    return kc, vc


def decode(q, k_cache, v_cache, block_tables, context_lens, scale: float, dtype: str,
           lib_path: str | None = None, parallel: bool = False) -> np.ndarray:
    """Exact (fp64) paged decode attention; returns float64 [S, Hq, d].

    ``parallel=True`` runs the OpenMP build over all host cores (same arithmetic, same bits);
    it exists to time the oracle on every core."""
    lib = _load_parallel() if parallel else _load(lib_path)
    fn = lib.oracle_decode_parallel if parallel else lib.oracle_decode
    q = _u16(q, "q")
    kc = _u16(k_cache, "k_cache")
    vc = _u16(v_cache, "v_cache")
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    S, hq, d = q.shape
    nb, hkv, bs, d2 = kc.shape
    if d2 != d or vc.shape != kc.shape:
        raise ValueError("cache shapes do not match q")
    if bt.ndim != 2 or bt.shape[0] != S or cl.shape != (S,):
        raise ValueError("block_tables must be [S, MB] and context_lens [S]")
    out = np.zeros((S, hq, d), dtype=np.float64)
    if S == 0:
        return out
    rc = fn(_ptr(q), _ptr(kc), _ptr(vc), _ptr(bt), bt.shape[1], _ptr(cl), S, hq, hkv, d, bs,
            nb, DTYPE_CODES[dtype], float(scale), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_decode: {ERRORS.get(rc, rc)}")
    return out


def parallel_threads() -> int:
    """Threads the OpenMP build of the decode uses on this host."""
    return int(_load_parallel().oracle_parallel_threads())


def copy_blocks(src_k, src_v, dst_k, dst_v, mapping, lib_path: str | None = None):
    """Copy whole blocks (all heads, rows, dims) from the source pools to the destination pools.

    mapping: int64 [n, 2] (source block, destination block); negative entries skip the pair.
    Returns new destination arrays (the source and destination may be the same arrays: pairs
    are applied in order, reading the pools as updated so far).
    """
    lib = _load(lib_path)
    sk, sv = _u16(src_k, "src_k"), _u16(src_v, "src_v")
    same = src_k is dst_k
    dk, dv = _u16(dst_k, "dst_k").copy(), _u16(dst_v, "dst_v").copy()
    if same:
        sk, sv = dk, dv
    m = np.ascontiguousarray(mapping, dtype=np.int64).reshape(-1, 2)
    if sk.shape[1:] != dk.shape[1:]:
        raise ValueError("pools differ in heads, block size or head dim")
    nb_s, hkv, bs, d = sk.shape
    rc = lib.oracle_copy_blocks(_ptr(sk), _ptr(sv), _ptr(dk), _ptr(dv), _ptr(m) if len(m) else None, len(m), hkv,
                                bs, d, nb_s, dk.shape[0])
    if rc != 0:
        raise ValueError(f"oracle_copy_blocks: {ERRORS.get(rc, rc)}")
    return dk, dv


def prefill(q, k_cache, v_cache, block_tables, query_start, context_lens, scale: float, dtype: str,
            lib_path: str | None = None) -> np.ndarray:
    """Exact (fp64) causal attention of each sequence's new tokens over its paged context.

    q: uint16 [N, Hq, d] (N = query_start[-1]); query_start: int32 [S + 1], query_start[0] = 0;
    context_lens: int32 [S], every token of the sequence including the new ones.  Returns
    float64 [N, Hq, d].
    """
    lib = _load(lib_path)
    q = _u16(q, "q")
    kc = _u16(k_cache, "k_cache")
    vc = _u16(v_cache, "v_cache")
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    qs = np.ascontiguousarray(query_start, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    S = cl.shape[0]
    N, hq, d = q.shape
    nb, hkv, bs, d2 = kc.shape
    if d2 != d or vc.shape != kc.shape:
        raise ValueError("cache shapes do not match q")
    if qs.shape != (S + 1,) or bt.ndim != 2 or bt.shape[0] != S or int(qs[-1]) != N:
        raise ValueError("query_start must be [S + 1] ending at the number of query rows; block_tables [S, MB]")
    out = np.zeros((N, hq, d), dtype=np.float64)
    if S == 0 or N == 0:
        return out
    rc = lib.oracle_prefill(_ptr(q), _ptr(kc), _ptr(vc), _ptr(bt), bt.shape[1], _ptr(qs), _ptr(cl), S, hq, hkv, d,
                            bs, nb, DTYPE_CODES[dtype], float(scale), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_prefill: {ERRORS.get(rc, rc)}")
    return out
