"""Helpers shared by the GPU parity tests: device upload, one decode step, comparison."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import paged_kv_cache_457_b200 as pa
from oracle_pins import from_bits, to_bits

TORCH_DT = {"fp16": torch.float16, "bf16": torch.bfloat16}

# Tolerances on the attention output (fp16/bf16 storage, fp32 accumulation),
# both against the exact fp64 oracle value: max |gpu - exact| <= 1e-2 over all
# elements and mean |gpu - exact| <= 1e-3.  As an extra diagnostic the mean
# distance to the exact value rounded once to the output's storage type is
# held to the same 1e-3 (it isolates the kernel's own error from the format's).
MAX_ABS = 1e-2
MEAN_ABS = 1e-3


def require_gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    pa.load_library()


def to_dev(bits: np.ndarray, dtype: str) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(TORCH_DT[dtype])


def to_dev_index(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class DeviceState:
    """The workload's caches on the device, stepped by the CUDA library."""

    def __init__(self, wl):
        self.wl = wl
        self.k_cache = to_dev(wl.k_cache, wl.dtype)
        self.v_cache = to_dev(wl.v_cache, wl.dtype)

    def write(self, step):
        wl = self.wl
        pa.write_kv(to_dev(step.k_new, wl.dtype), to_dev(step.v_new, wl.dtype), self.k_cache, self.v_cache,
                    to_dev_index(step.slot_mapping))

    def decode(self, step, partition_tokens=0, max_context_len=None, q=None, tables=None, lens=None):
        wl = self.wl
        q = to_dev(step.q if q is None else q, wl.dtype)
        tables = to_dev_index(step.block_tables if tables is None else tables)
        lens = to_dev_index(step.context_lens if lens is None else lens)
        mcl = step.max_context_len if max_context_len is None else max_context_len
        out = pa.decode(q, self.k_cache, self.v_cache, tables, lens, wl.scale, max_context_len=mcl,
                        partition_tokens=partition_tokens)
        return host_bits(out)


def oracle_step(wl, k_cache, v_cache, step, seqs=None):
    """Apply the step's write to host caches and return (k', v', exact output of the selected seqs)."""
    kc, vc = oracle.write_kv(step.k_new, step.v_new, k_cache, v_cache, step.slot_mapping, wl.block_size)
    sel = slice(None) if seqs is None else seqs
    ref = oracle.decode(step.q[sel], kc, vc, step.block_tables[sel], step.context_lens[sel], wl.scale, wl.dtype)
    return kc, vc, ref


def compare(out_bits: np.ndarray, ref: np.ndarray, dtype: str, max_abs=MAX_ABS, mean_abs=MEAN_ABS, what=""):
    got = from_bits(out_bits, dtype)
    assert got.shape == ref.shape, f"{what}: shape {got.shape} vs {ref.shape}"
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    rounded = from_bits(to_bits(ref, dtype), dtype)
    err_r = np.abs(got - rounded)
    stats = {"max_abs": float(err.max(initial=0.0)), "mean_abs": float(err.mean()) if err.size else 0.0,
             "mean_abs_vs_rounded": float(err_r.mean()) if err_r.size else 0.0,
             "max_abs_vs_rounded": float(err_r.max(initial=0.0))}
    print(f"[parity] {what}: max_abs {stats['max_abs']:.3e} mean_abs {stats['mean_abs']:.3e} "
          f"mean_abs_vs_rounded {stats['mean_abs_vs_rounded']:.3e}")
    assert stats["max_abs"] <= max_abs, f"{what}: {stats}"
    assert stats["mean_abs"] <= mean_abs, f"{what}: {stats}"
    assert stats["mean_abs_vs_rounded"] <= mean_abs, f"{what}: {stats}"
    return stats
