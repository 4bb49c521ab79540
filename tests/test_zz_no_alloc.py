"""pa_decode_static_workspace: decode for callers that cannot allocate device memory (B200).

Some users run this library inside a host framework that owns every device allocation, or
in a server whose memory budget is fixed at start-up, and may not call cudaMalloc during a
step; they cannot hand pa_decode a workspace.  The static-workspace entry point uses a
fixed 32 MiB scratch array compiled into the library instead.  These tests call it through
the C ABI and check, twice in a row (the array keeps the previous call's contents), that it
gives exactly pa_decode's bytes (both run the same kernels with the same work split, so
nothing else is acceptable) and that those bytes are within the oracle's tolerance of the
exact fp64 attention; and that a problem too large for the array is refused.

This file is named to be collected last, so a failure here never hides another test.
"""
import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_457_b200 as pa
import workloads as W
from gpu_util import compare, host_bits, oracle_step, require_gpu, to_dev, to_dev_index

pytestmark = pytest.mark.gpu

PA_ERR_STATIC_WORKSPACE = -10
STATIC_BYTES = 32 * 1024 * 1024


def _call_static(lib, q, kc, vc, tables, lens, scale, out, hkv, bs, max_ctx, part, dtype_code):
    S, hq, d = q.shape
    return lib.pa_decode_static_workspace(
        q.data_ptr(), kc.data_ptr(), vc.data_ptr(), tables.data_ptr(), lens.data_ptr(), ctypes.c_float(scale),
        out.data_ptr(), S, hq, hkv, d, bs, kc.shape[0], tables.stride(0), max_ctx, q.stride(0), out.stride(0), part,
        dtype_code, torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("dtype,part", [("bf16", 64), ("fp16", 0)])
def test_static_workspace_matches_pa_decode_twice(dtype, part):
    require_gpu()
    lib = pa.load_library()
    lens = [1, 17, 300, 1500, 2048, 777, 64, 1025]
    wl = W.custom(seed=31, num_seqs=len(lens), num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                  lens=lens, dtype=dtype)
    st = wl.steps[0]
    kc, vc = to_dev(wl.k_cache, dtype), to_dev(wl.v_cache, dtype)
    pa.write_kv(to_dev(st.k_new, dtype), to_dev(st.v_new, dtype), kc, vc, to_dev_index(st.slot_mapping))
    q = to_dev(st.q, dtype)
    tables = to_dev_index(st.block_tables)
    ctx = to_dev_index(st.context_lens)
    max_ctx = st.max_context_len
    need = pa.decode_workspace_size(len(lens), 32, 8, 128, 16, max_ctx, part)
    assert 0 < need <= STATIC_BYTES, "the case must use split-context scratch that fits the array"
    ref = host_bits(pa.decode(q, kc, vc, tables, ctx, wl.scale, max_context_len=max_ctx, partition_tokens=part))
    _, _, exact = oracle_step(wl, wl.k_cache, wl.v_cache, st)
    compare(ref, exact, dtype, what="pa_decode")
    code = 2 if dtype == "bf16" else 1
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        rc = _call_static(lib, q, kc, vc, tables, ctx, wl.scale, out, 8, 16, max_ctx, part, code)
        assert rc == 0, lib.pa_status_string(rc)
        got = host_bits(out)
        assert np.array_equal(got, ref), f"call {call}: static-workspace output differs from pa_decode's"
        compare(got, exact, dtype, what=f"static workspace, call {call}")
    assert pa.device_status() == 0


def test_static_workspace_refuses_oversized_problems():
    require_gpu()
    lib = pa.load_library()
    # 256 seqs x 32 heads x 64 partitions x (128 + 2) floats = 272 MB of scratch: beyond the array
    S, hq, hkv, d, bs = 256, 32, 8, 128, 16
    assert pa.decode_workspace_size(S, hq, hkv, d, bs, 8192, 128) > STATIC_BYTES
    q = torch.zeros((S, hq, d), dtype=torch.float16, device="cuda")
    kc = torch.zeros((4, hkv, bs, d), dtype=torch.float16, device="cuda")
    tables = torch.zeros((S, 512), dtype=torch.int32, device="cuda")
    ctx = torch.ones((S,), dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    n0 = pa.launch_count()
    rc = _call_static(lib, q, kc, kc, tables, ctx, 0.1, out, hkv, bs, 8192, 128, 1)
    assert rc == PA_ERR_STATIC_WORKSPACE
    assert b"32 MiB" in lib.pa_status_string(rc)
    assert pa.launch_count() == n0
