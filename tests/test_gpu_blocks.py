"""Block copy (copy-on-write) and swap through the C ABI against the oracle.

Copies are bit-exact: the device pools are compared as raw 16-bit patterns
with the oracle's copy applied to host copies of the same pools.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_457_b200 as pa
import workloads
from gpu_util import TORCH_DT, compare, host_bits, require_gpu, to_dev, to_dev_index
from oracle_pins import to_bits

pytestmark = pytest.mark.gpu


def _pool(rng, nb, hkv, bs, d):
    bits = rng.integers(0, 1 << 16, size=(nb, hkv, bs, d), dtype=np.uint16)
    return bits, rng.integers(0, 1 << 16, size=(nb, hkv, bs, d), dtype=np.uint16)


def _pairs(rng, n, src_blocks, dst_blocks, same_pool):
    """n pairs with distinct destinations, none of which is another pair's source."""
    if same_pool:
        ids = rng.permutation(src_blocks)[: 2 * n]
        return np.stack([ids[:n], ids[n:]], axis=1).astype(np.int64)
    return np.stack([rng.choice(src_blocks, n, replace=False), rng.choice(dst_blocks, n, replace=False)],
                    axis=1).astype(np.int64)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("hkv,bs,d", [(1, 16, 64), (4, 32, 128), (8, 16, 128), (3, 32, 64)])
@pytest.mark.parametrize("n", [0, 1, 7, 100])
def test_copy_blocks_matches_oracle(dtype, hkv, bs, d, n):
    require_gpu()
    rng = np.random.default_rng(1000 + hkv * 31 + bs + d + n)
    nb = 256
    kb, vb = _pool(rng, nb, hkv, bs, d)
    m = _pairs(rng, n, nb, nb, True)
    if n >= 7:
        m[3, 0] = -1  # skipped pairs
        m[5, 1] = -1
    kc, vc = to_dev(kb, dtype), to_dev(vb, dtype)
    pa.copy_blocks(kc, vc, to_dev_index(m))
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    ek, ev = oracle.copy_blocks(kb, vb, kb, vb, m)
    assert np.array_equal(host_bits(kc), ek)
    assert np.array_equal(host_bits(vc), ev)


def test_copy_blocks_out_of_range_is_flagged_and_skipped():
    require_gpu()
    rng = np.random.default_rng(7)
    nb, hkv, bs, d = 64, 2, 16, 128
    kb, vb = _pool(rng, nb, hkv, bs, d)
    m = _pairs(rng, 6, nb, nb, True)
    bad = m.copy()
    bad[2, 1] = nb  # destination past the pool
    bad[4, 0] = nb + 100  # source past the pool
    kc, vc = to_dev(kb, "fp16"), to_dev(vb, "fp16")
    pa.device_status(clear=True)
    pa.copy_blocks(kc, vc, to_dev_index(bad))
    torch.cuda.synchronize()
    assert pa.device_status() & pa.DEV_ERR_BLOCK_ID
    keep = np.delete(bad, [2, 4], axis=0)
    ek, ev = oracle.copy_blocks(kb, vb, kb, vb, keep)
    assert np.array_equal(host_bits(kc), ek)
    assert np.array_equal(host_bits(vc), ev)


def test_copy_blocks_mapping_in_pinned_host_memory():
    require_gpu()
    rng = np.random.default_rng(8)
    nb, hkv, bs, d = 128, 4, 16, 128
    kb, vb = _pool(rng, nb, hkv, bs, d)
    m = _pairs(rng, 20, nb, nb, True)
    kc, vc = to_dev(kb, "bf16"), to_dev(vb, "bf16")
    pa.copy_blocks(kc, vc, torch.from_numpy(m).pin_memory())
    torch.cuda.synchronize()
    ek, ev = oracle.copy_blocks(kb, vb, kb, vb, m)
    assert np.array_equal(host_bits(kc), ek) and np.array_equal(host_bits(vc), ev)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_swap_out_and_in_round_trip(dtype):
    """Device pool -> pinned host pool -> other device blocks, each leg against the oracle."""
    require_gpu()
    rng = np.random.default_rng(11)
    nb, cpu_nb, hkv, bs, d = 300, 64, 4, 16, 128
    kb, vb = _pool(rng, nb, hkv, bs, d)
    hk, hv = _pool(rng, cpu_nb, hkv, bs, d)
    out_map = _pairs(rng, 40, nb, cpu_nb, False)
    kc, vc = to_dev(kb, dtype), to_dev(vb, dtype)
    host_k = torch.from_numpy(hk.view(np.int16)).view(TORCH_DT[dtype]).pin_memory()
    host_v = torch.from_numpy(hv.view(np.int16)).view(TORCH_DT[dtype]).pin_memory()
    pa.swap_blocks(kc, vc, host_k, host_v, to_dev_index(out_map))
    torch.cuda.synchronize()
    ehk, ehv = oracle.copy_blocks(kb, vb, hk, hv, out_map)
    assert np.array_equal(host_bits(host_k), ehk) and np.array_equal(host_bits(host_v), ehv)

    in_map = np.stack([out_map[:, 1], rng.permutation(nb)[:40]], axis=1).astype(np.int64)
    pa.swap_blocks(host_k, host_v, kc, vc, torch.from_numpy(in_map).pin_memory(), device=kc.device)
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    ek, ev = oracle.copy_blocks(ehk, ehv, kb, vb, in_map)
    assert np.array_equal(host_bits(kc), ek) and np.array_equal(host_bits(vc), ev)


def test_swapped_sequence_decodes_like_before():
    """Preempt one batch's sequences to a host pool, restore them to fresh blocks, decode again."""
    require_gpu()
    wl = workloads.tiny(seed=5)
    step = wl.steps[0]
    kc, vc = to_dev(wl.k_cache, wl.dtype), to_dev(wl.v_cache, wl.dtype)
    pa.write_kv(to_dev(step.k_new, wl.dtype), to_dev(step.v_new, wl.dtype), kc, vc, to_dev_index(step.slot_mapping))
    q, lens = to_dev(step.q, wl.dtype), to_dev_index(step.context_lens)
    before = host_bits(pa.decode(q, kc, vc, to_dev_index(step.block_tables), lens, wl.scale,
                                 max_context_len=step.max_context_len))
    tables = step.block_tables
    used = np.unique(tables[tables >= 0]).astype(np.int64)
    nb = kc.shape[0]
    host_k = torch.empty((len(used),) + tuple(kc.shape[1:]), dtype=kc.dtype, pin_memory=True)
    host_v = torch.empty((len(used),) + tuple(kc.shape[1:]), dtype=kc.dtype, pin_memory=True)
    pa.swap_blocks(kc, vc, host_k, host_v, to_dev_index(np.stack([used, np.arange(len(used))], 1).astype(np.int64)))
    # Overwrite the originals, then restore into blocks the batch did not use.
    kc[torch.from_numpy(used).cuda()] = 0
    vc[torch.from_numpy(used).cuda()] = 0
    free = np.setdiff1d(np.arange(nb), used)
    assert len(free) >= len(used)
    new_ids = np.random.default_rng(3).permutation(free)[: len(used)]
    pa.swap_blocks(host_k, host_v, kc, vc,
                   to_dev_index(np.stack([np.arange(len(used)), new_ids], 1).astype(np.int64)), device=kc.device)
    remap = np.full(nb, -1, dtype=np.int64)
    remap[used] = new_ids
    new_tables = np.where(tables >= 0, remap[np.maximum(tables, 0)], tables).astype(np.int32)
    after = host_bits(pa.decode(q, kc, vc, to_dev_index(new_tables), lens, wl.scale,
                                max_context_len=step.max_context_len))
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    # Same data in the same logical order: the same arithmetic, bit for bit.
    assert np.array_equal(before, after)
    kh = host_bits(kc)
    vh = host_bits(vc)
    ref = oracle.decode(step.q, kh, vh, new_tables, step.context_lens, wl.scale, wl.dtype)
    compare(after, ref, wl.dtype, what="after swap-in")


def test_copy_on_write_then_append():
    """Two sequences share a partly filled last block; one copies it before appending its token."""
    require_gpu()
    rng = np.random.default_rng(21)
    dtype, nb, hkv, hq, bs, d = "fp16", 32, 2, 8, 16, 128
    # Values in a tame range so the decode compares on attention, not on garbage bits.
    kb = to_bits(rng.standard_normal((nb, hkv, bs, d)), dtype)
    vb = to_bits(rng.standard_normal((nb, hkv, bs, d)), dtype)
    shared = [4, 9, 17]  # 2 full blocks + block 17 holding 5 tokens
    prefix = 2 * bs + 5
    private = 23
    tables = np.array([shared, [4, 9, private]], dtype=np.int32)
    m = np.array([[17, private]], dtype=np.int64)
    knew = to_bits(rng.standard_normal((2, hkv, d)), dtype)
    vnew = to_bits(rng.standard_normal((2, hkv, d)), dtype)
    slots = np.array([17 * bs + 5, private * bs + 5], dtype=np.int64)
    q = to_bits(rng.standard_normal((2, hq, d)), dtype)
    lens = np.array([prefix + 1, prefix + 1], dtype=np.int32)
    scale = 1.0 / np.sqrt(d)

    kc, vc = to_dev(kb, dtype), to_dev(vb, dtype)
    pa.copy_blocks(kc, vc, to_dev_index(m))
    pa.write_kv(to_dev(knew, dtype), to_dev(vnew, dtype), kc, vc, to_dev_index(slots))
    out = host_bits(pa.decode(to_dev(q, dtype), kc, vc, to_dev_index(tables), to_dev_index(lens), scale,
                              max_context_len=prefix + 1))
    torch.cuda.synchronize()
    assert pa.device_status() == 0

    ok, ov = oracle.copy_blocks(kb, vb, kb, vb, m)
    ok, ov = oracle.write_kv(knew, vnew, ok, ov, slots, bs)
    assert np.array_equal(host_bits(kc), ok) and np.array_equal(host_bits(vc), ov)
    ref = oracle.decode(q, ok, ov, tables, lens, scale, dtype)
    compare(out, ref, dtype, what="copy-on-write decode")


def test_full_size_copy_blocks_llama2_7b_pool():
    """A Llama-2-7B-shaped pool (32 kv heads, 16-token blocks, d=128): 1024 pairs, sampled against the oracle."""
    require_gpu()
    rng = np.random.default_rng(99)
    nb, hkv, bs, d = 4096, 32, 16, 128
    kc = torch.randint(-32768, 32767, (nb, hkv, bs, d), dtype=torch.int16, device="cuda").view(torch.float16)
    vc = torch.randint(-32768, 32767, (nb, hkv, bs, d), dtype=torch.int16, device="cuda").view(torch.float16)
    m = _pairs(rng, 1024, nb, nb, True)
    k0, v0 = kc.clone(), vc.clone()
    pa.copy_blocks(kc, vc, to_dev_index(m))
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    # Sampled pairs through the oracle, on the pool's own blocks.
    for i in rng.choice(len(m), 16, replace=False):
        s, t = int(m[i, 0]), int(m[i, 1])
        src_k, src_v = host_bits(k0[s:s + 1]), host_bits(v0[s:s + 1])
        dst_k, dst_v = host_bits(k0[t:t + 1]), host_bits(v0[t:t + 1])
        ek, ev = oracle.copy_blocks(src_k, src_v, dst_k, dst_v, np.array([[0, 0]], dtype=np.int64))
        assert np.array_equal(host_bits(kc[t:t + 1]), ek) and np.array_equal(host_bits(vc[t:t + 1]), ev)
    # Every block not named as a destination is unchanged.
    untouched = torch.ones(nb, dtype=torch.bool, device="cuda")
    untouched[torch.from_numpy(m[:, 1]).cuda()] = False
    assert torch.equal(kc.view(torch.int16)[untouched], k0.view(torch.int16)[untouched])
    assert torch.equal(vc.view(torch.int16)[untouched], v0.view(torch.int16)[untouched])


def test_pageable_host_pool_is_refused_before_launch():
    require_gpu()
    lib = pa.load_library()
    nb, hkv, bs, d = 4, 1, 16, 64
    dev_k = torch.zeros((nb, hkv, bs, d), dtype=torch.float16, device="cuda")
    dev_v = torch.zeros_like(dev_k)
    pageable = np.zeros((nb, hkv, bs, d), dtype=np.uint16)
    m = to_dev_index(np.array([[0, 1]], dtype=np.int64))
    before = pa.launch_count()
    rc = lib.pa_swap_blocks(dev_k.data_ptr(), dev_v.data_ptr(), pageable.ctypes.data, pageable.ctypes.data,
                            m.data_ptr(), 1, hkv, d, bs, nb, nb, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == -11
    assert pa.launch_count() == before
