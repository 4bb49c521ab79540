"""The C ABI library on a machine without a GPU: it builds, loads, exports every symbol the
header declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import glob
import os
import re

import pytest

import paged_kv_cache_457_b200 as pa
from paged_kv_cache_457_b200 import build_lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _has_gpu():
    import torch
    return torch.cuda.is_available()


@pytest.fixture(scope="module")
def lib():
    build_lib.build()
    return pa.load_library()


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        with open(h) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("pa_write_kv", "pa_decode", "pa_decode_workspace_size", "pa_get_device_status"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert names
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, f"not exported: {missing}"
    assert set(names) == set(pa.EXPORTED_SYMBOLS)


def test_version_and_status_strings(lib):
    assert lib.pa_version() == 100
    assert lib.pa_build_flags() == 0  # the release build; libpa_b200_debug.so reports PA_BUILD_DEBUG
    assert lib.pa_status_string(0) == b"ok"
    for code in range(-9, 0):
        assert lib.pa_status_string(code) != b"unknown status"


def _decode(lib, **over):
    args = dict(q=16, k=16, v=16, bt=16, cl=16, scale=0.1, out=16, S=2, hq=4, hkv=2, d=128, bs=16, nb=10, mb=4,
                mcl=40, qs=512, os_=512, part=0, dtype=1, ws=None, wsb=0, stream=None)
    args.update(over)
    return lib.pa_decode(args["q"], args["k"], args["v"], args["bt"], args["cl"], args["scale"], args["out"],
                         args["S"], args["hq"], args["hkv"], args["d"], args["bs"], args["nb"], args["mb"],
                         args["mcl"], args["qs"], args["os_"], args["part"], args["dtype"], args["ws"], args["wsb"],
                         args["stream"])


def test_host_validation_of_decode(lib):
    assert _decode(lib, d=96) == -5
    assert _decode(lib, bs=8) == -5
    assert _decode(lib, hq=6, hkv=4) == -6
    assert _decode(lib, dtype=3) == -2
    assert _decode(lib, S=-1) == -3
    assert _decode(lib, mcl=-1) == -3
    assert _decode(lib, qs=100) == -3
    assert _decode(lib, q=None) == -1
    assert _decode(lib, q=24) == -4  # misaligned pointer
    assert _decode(lib, qs=516) == -4  # stride not a multiple of 8
    if not _has_gpu():  # never launch on the fake pointers used here
        assert _decode(lib) == -9  # valid arguments reach CUDA, absent here: reported, not thrown
    assert _decode(lib, S=0) == 0  # empty batch: nothing to do, no CUDA call


def test_host_validation_of_write(lib):
    w = lib.pa_write_kv
    # every call below fails validation (or has no tokens) before any CUDA call
    assert w(16, 16, 16, 16, 16, 4, 2, 128, 16, 10, 256, 256, 5, None) == -2
    assert w(16, 16, 16, 16, 16, 4, 2, 96, 16, 10, 256, 256, 1, None) == -5
    assert w(16, 16, 16, 16, None, 4, 2, 128, 16, 10, 256, 256, 1, None) == -1
    assert w(16, 16, 16, 16, 16, 4, 2, 128, 16, 10, 100, 256, 1, None) == -3
    assert w(16, 16, 16, 20, 16, 4, 2, 128, 16, 10, 256, 256, 1, None) == -4
    assert w(16, 16, 16, 16, 16, 0, 2, 128, 16, 10, 256, 256, 1, None) == 0


def test_library_is_sm100a_only():
    cmd = build_lib.command()
    assert "arch=compute_100a,code=sm_100a" in cmd
    assert not any("sm_90" in c or "compute_90" in c for c in cmd)


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(2, 4, 128, dtype=torch.float16)
    with pytest.raises(pa.PagedAttentionError):
        pa.decode(x, x, x, torch.zeros(2, 1, dtype=torch.int32), torch.zeros(2, dtype=torch.int32), 0.1,
                  max_context_len=1)


def _prefill(lib, **over):
    args = dict(q=16, k=16, v=16, bt=16, qs=16, cl=16, scale=0.1, out=16, S=2, N=40, hq=4, hkv=2, d=128, bs=16,
                nb=10, mb=4, mql=32, qts=512, ots=512, dtype=1, stream=None)
    args.update(over)
    return lib.pa_prefill(args["q"], args["k"], args["v"], args["bt"], args["qs"], args["cl"], args["scale"],
                          args["out"], args["S"], args["N"], args["hq"], args["hkv"], args["d"], args["bs"],
                          args["nb"], args["mb"], args["mql"], args["qts"], args["ots"], args["dtype"], args["stream"])


def test_host_validation_of_prefill(lib):
    assert _prefill(lib, d=96) == -5
    assert _prefill(lib, bs=8) == -5
    assert _prefill(lib, hq=6, hkv=4) == -6
    assert _prefill(lib, dtype=0) == -2
    assert _prefill(lib, S=-1) == -3
    assert _prefill(lib, mql=-1) == -3
    assert _prefill(lib, qts=100) == -3  # token stride shorter than a token's heads
    assert _prefill(lib, scale=float("nan")) == -3
    assert _prefill(lib, out=None) == -1
    assert _prefill(lib, q=24) == -4
    assert _prefill(lib, ots=516) == -4
    assert _prefill(lib, nb=0) == -3  # an empty pool has no rows for the tensor maps
    assert _prefill(lib, S=0) == 0 and _prefill(lib, N=0) == 0 and _prefill(lib, mql=0) == 0


def test_host_validation_of_block_copies(lib):
    c = lib.pa_copy_blocks
    # (k, v, mapping, n, hkv, d, bs, nb, stream)
    assert c(16, 16, 16, 3, 4, 96, 16, 10, None) == -5
    assert c(16, 16, 16, 3, 4, 128, 8, 10, None) == -5
    assert c(16, 16, 16, -1, 4, 128, 16, 10, None) == -3
    assert c(16, 16, 16, 3, 0, 128, 16, 10, None) == -3
    assert c(None, 16, 16, 3, 4, 128, 16, 10, None) == -1
    assert c(16, 16, None, 3, 4, 128, 16, 10, None) == -1
    assert c(24, 16, 16, 3, 4, 128, 16, 10, None) == -4
    assert c(16, 16, 20, 3, 4, 128, 16, 10, None) == -4  # mapping must be 8-byte aligned
    assert c(16, 16, 16, 0, 4, 128, 16, 10, None) == 0  # nothing to copy: no CUDA call
    s = lib.pa_swap_blocks
    # (src_k, src_v, dst_k, dst_v, mapping, n, hkv, d, bs, src_nb, dst_nb, stream)
    assert s(16, 16, 16, 16, 16, 2, 4, 128, 16, 10, 0, None) == -3
    assert s(16, 16, 16, 16, 16, 2, 4, 64, 32, 10, 10, None) != -5  # d 64 and bs 32 are supported
    assert s(16, 16, 16, 16, 16, 0, 4, 64, 32, 10, 10, None) == 0
    if not _has_gpu():
        # valid arguments reach the pointer check, which needs the CUDA runtime: reported, not thrown
        assert s(16, 16, 16, 16, 16, 2, 4, 64, 32, 10, 10, None) in (-9, -11)


def test_status_strings_cover_new_codes(lib):
    for code in (-10, -11):
        assert lib.pa_status_string(code) != b"unknown status"


def _cascade(lib, info_over=None, **over):
    """pa_decode_cascade on fake aligned pointers with a consistent host-built plan (2 sequences, 4 query /
    2 kv heads, block 16, max_context_len 40, no groups); `info_over` edits the plan's sizes."""
    import ctypes
    from paged_kv_cache_457_b200.cascade import CascadeInfo
    plan = pa.cascade_plan(2, 4, 2, 16, 40)
    info = CascadeInfo.from_buffer_copy(plan.info)
    for k, v in (info_over or {}).items():
        setattr(info, k, v)
    args = dict(q=16, k=16, v=16, bt=16, cl=16, scale=0.1, out=16, d=128, nb=10, mb=4, qs=512, os_=512, dtype=1,
                plan=16, ws=256, wsb=1 << 20, stream=None)
    args.update(over)
    return lib.pa_decode_cascade(args["q"], args["k"], args["v"], args["bt"], args["cl"], args["scale"], args["out"],
                                 args["d"], args["nb"], args["mb"], args["qs"], args["os_"], args["dtype"], args["plan"],
                                 ctypes.byref(info), args["ws"], args["wsb"], args["stream"])


def test_host_validation_of_cascade_decode(lib):
    # every call below fails validation (or has no sequences) before any CUDA call
    assert _cascade(lib, d=96) == -5
    assert _cascade(lib, dtype=3) == -2
    assert _cascade(lib, info_over={"num_q_heads": 5}) == -6
    assert _cascade(lib, info_over={"num_q_heads": 18}) == -5  # 9 query heads per kv head
    assert _cascade(lib, info_over={"block_size": 8}) == -5
    assert _cascade(lib, info_over={"max_context_len": -1}) == -3
    assert _cascade(lib, info_over={"plan_ints": 3}) == -3  # sizes that do not add up to the plan
    assert _cascade(lib, info_over={"num_prefix_jobs": 99}) == -3
    assert _cascade(lib, nb=0) == -3
    assert _cascade(lib, qs=100) == -3
    assert _cascade(lib, scale=float("inf")) == -3
    assert _cascade(lib, q=None) == -1
    assert _cascade(lib, plan=None) == -1
    assert _cascade(lib, q=24) == -4
    assert _cascade(lib, os_=516) == -4
    assert _cascade(lib, ws=None) == -7
    assert _cascade(lib, wsb=16) == -7
    assert _cascade(lib, ws=264) == -7  # misaligned workspace
    assert _cascade(lib, info_over={"num_seqs": 0, "plan_ints": 1, "num_jobs": 0, "num_members": 0,
                                    "num_pieces": 0, "num_prefix_jobs": 0}) == 0
    if not _has_gpu():  # never launch on the fake pointers used here
        assert _cascade(lib) == -9


def test_cascade_workspace_size_refuses_bad_input(lib):
    plan = pa.cascade_plan(2, 4, 2, 16, 40)
    assert pa.cascade_workspace_size(plan, 128) >= 256
    assert pa.cascade_workspace_size(plan, 96) == 0
