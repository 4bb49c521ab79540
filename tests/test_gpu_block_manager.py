"""The native page pool driving the CUDA kernels: forks, copy-on-write, preemption to a pinned
host pool and back, each decode step compared with the oracle's attention over every
sequence's own tokens laid out contiguously."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_457_b200 as pa
from gpu_util import TORCH_DT, compare, host_bits, require_gpu, to_dev, to_dev_index
from oracle_pins import to_bits

pytestmark = pytest.mark.gpu


def _contiguous(lk, lv, bs):
    L = len(lk)
    nblk = -(-L // bs)
    hkv, d = lk.shape[1:]
    ck = np.zeros((nblk, bs, hkv, d), dtype=np.uint16)
    cv = np.zeros_like(ck)
    ck.reshape(-1, hkv, d)[:L] = lk
    cv.reshape(-1, hkv, d)[:L] = lv
    return np.ascontiguousarray(ck.transpose(0, 2, 1, 3)), np.ascontiguousarray(cv.transpose(0, 2, 1, 3))


@pytest.mark.parametrize("dtype,hq,hkv,d,bs", [("fp16", 8, 8, 128, 16), ("bf16", 32, 4, 128, 32),
                                                ("fp16", 16, 2, 64, 16)])
def test_manager_driven_steps_match_oracle(dtype, hq, hkv, d, bs):
    require_gpu()
    rng = np.random.default_rng(hq + hkv + d + bs)
    nb, nh = 96, 32
    bm = pa.BlockManager(bs, nb, nh)
    tdt = TORCH_DT[dtype]
    kc = torch.zeros((nb, hkv, bs, d), dtype=tdt, device="cuda")
    vc = torch.zeros_like(kc)
    hk = torch.zeros((nh, hkv, bs, d), dtype=tdt, pin_memory=True)
    hv = torch.zeros((nh, hkv, bs, d), dtype=tdt, pin_memory=True)
    logical = {}
    for sid, n in enumerate([3 * bs + 5, bs, 7, 2 * bs - 1]):
        bm.add_sequence(sid, n)
        k = to_bits(rng.standard_normal((n, hkv, d)), dtype)
        v = to_bits(rng.standard_normal((n, hkv, d)), dtype)
        pa.write_kv(to_dev(k, dtype), to_dev(v, dtype), kc, vc, to_dev_index(bm.slots(sid, 0, n)))
        logical[sid] = (k, v)
    # parallel sampling: two children share sequence 0's pages, including its partly filled last page
    for child in (10, 11):
        bm.fork(0, child)
        logical[child] = logical[0]
    running = [0, 1, 2, 3, 10, 11]
    swapped = []
    table_stride = 12
    scale = 1.0 / np.sqrt(d)
    copies = 0
    for step in range(24):
        if step == 6:  # preempt two sequences, one of which shares pages with a running one
            out = [3, 11]
            m = bm.swap_out(out)
            pa.swap_blocks(kc, vc, hk, hv, to_dev_index(m))
            running = [s for s in running if s not in out]
            swapped = out
        if step == 12:  # bring them back into whatever device pages are free now
            m = bm.swap_in(swapped)
            pa.swap_blocks(hk, hv, kc, vc, to_dev_index(m), device=kc.device)
            running += swapped
            swapped = []
        plan = bm.build_decode_step(running, table_stride)
        if len(plan.copy_pairs):
            copies += len(plan.copy_pairs)
            pa.copy_blocks(kc, vc, to_dev_index(plan.copy_pairs))
        k = to_bits(rng.standard_normal((len(running), hkv, d)), dtype)
        v = to_bits(rng.standard_normal((len(running), hkv, d)), dtype)
        pa.write_kv(to_dev(k, dtype), to_dev(v, dtype), kc, vc, to_dev_index(plan.slot_mapping))
        for i, sid in enumerate(running):
            lk, lv = logical[sid]
            logical[sid] = (np.concatenate([lk, k[i:i + 1]]), np.concatenate([lv, v[i:i + 1]]))
        q = to_bits(rng.standard_normal((len(running), hq, d)), dtype)
        out_bits = host_bits(pa.decode(to_dev(q, dtype), kc, vc, to_dev_index(plan.block_tables),
                                       to_dev_index(plan.context_lens), scale,
                                       max_context_len=int(plan.context_lens.max())))
        ref = np.empty((len(running), hq, d))
        for i, sid in enumerate(running):
            ck, cv = _contiguous(*logical[sid], bs)
            L = len(logical[sid][0])
            ref[i] = oracle.decode(q[i:i + 1], ck, cv, np.arange(len(ck), dtype=np.int32)[None],
                                   np.array([L], np.int32), scale, dtype)[0]
        compare(out_bits, ref, dtype, what=f"step {step}")
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    assert copies >= 2  # both children split sequence 0's shared partial page
    for sid in list(logical):
        bm.free_sequence(sid)
    assert bm.num_free_device_blocks == nb and bm.num_free_host_blocks == nh


def test_manager_driven_chunked_prefill_matches_oracle():
    """Chunked prefill steps planned by the native pool (a forked pair sharing a partly full page,
    ragged chunks, idle sequences) through copy_blocks, write_kv and the tensor-core prefill, each
    sequence's rows compared with the oracle over its own tokens laid out contiguously."""
    require_gpu()
    dtype, hq, hkv, d, bs = "fp16", 8, 2, 128, 16
    rng = np.random.default_rng(17)
    nb = 64
    bm = pa.BlockManager(bs, nb, 0)
    tdt = TORCH_DT[dtype]
    kc = torch.zeros((nb, hkv, bs, d), dtype=tdt, device="cuda")
    vc = torch.zeros_like(kc)
    logical = {}
    for sid, n in ((0, 29), (1, 16)):
        bm.add_sequence(sid, n)
        k = to_bits(rng.standard_normal((n, hkv, d)), dtype)
        v = to_bits(rng.standard_normal((n, hkv, d)), dtype)
        pa.write_kv(to_dev(k, dtype), to_dev(v, dtype), kc, vc, to_dev_index(bm.slots(sid, 0, n)))
        logical[sid] = (k, v)
    bm.fork(0, 2)
    logical[2] = logical[0]
    ids = [0, 1, 2]
    scale = 1.0 / np.sqrt(d)
    copies = 0
    for step in range(5):
        chunk = [int(rng.integers(1, 40))] + [int(x) for x in rng.integers(0, 40, size=len(ids) - 1)]
        plan = bm.build_prefill_step(ids, chunk, 16)
        if len(plan.copy_pairs):
            copies += len(plan.copy_pairs)
            pa.copy_blocks(kc, vc, to_dev_index(plan.copy_pairs))
        total = int(sum(chunk))
        k = to_bits(rng.standard_normal((total, hkv, d)), dtype)
        v = to_bits(rng.standard_normal((total, hkv, d)), dtype)
        pa.write_kv(to_dev(k, dtype), to_dev(v, dtype), kc, vc, to_dev_index(plan.slot_mapping))
        for i, sid in enumerate(ids):
            a, b = int(plan.query_start[i]), int(plan.query_start[i + 1])
            lk, lv = logical[sid]
            logical[sid] = (np.concatenate([lk, k[a:b]]), np.concatenate([lv, v[a:b]]))
        q = to_bits(rng.standard_normal((total, hq, d)), dtype)
        out_bits = host_bits(pa.prefill(to_dev(q, dtype), kc, vc, to_dev_index(plan.block_tables),
                                        to_dev_index(plan.query_start), to_dev_index(plan.context_lens), scale,
                                        max(chunk)))
        for i, sid in enumerate(ids):
            a, b = int(plan.query_start[i]), int(plan.query_start[i + 1])
            if a == b:
                continue
            ck, cv = _contiguous(*logical[sid], bs)
            L = len(logical[sid][0])
            ref = oracle.prefill(q[a:b], ck, cv, np.arange(len(ck), dtype=np.int32)[None],
                                 np.array([0, b - a], np.int32), np.array([L], np.int32), scale, dtype)
            compare(out_bits[a:b], ref, dtype, what=f"step {step} sequence {sid}")
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    assert copies >= 1  # the first of the forked pair to append split the shared partial page
