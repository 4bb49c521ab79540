"""Properties of the CUDA path that hold exactly (bitwise), needing no tolerance (B200)."""
import numpy as np
import pytest
import torch

import paged_kv_cache_457_b200 as pa
import workloads as W
from gpu_util import DeviceState, compare, host_bits, oracle_step, require_gpu, to_dev, to_dev_index

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


@pytest.mark.parametrize("dtype,d,bs", [("fp16", 128, 16), ("bf16", 64, 32)])
def test_single_token_returns_v_row_exactly(dtype, d, bs):
    """L = 1: the weight is exactly 1, so the output is the written V row, bit for bit."""
    wl = W.custom(seed=5, num_seqs=6, num_q_heads=8, num_kv_heads=2, head_dim=d, block_size=bs, lens=[1] * 6,
                  dtype=dtype)
    st = wl.steps[0]
    dev = DeviceState(wl)
    dev.write(st)
    out = dev.decode(st)
    want = np.repeat(st.v_new, 4, axis=1)  # q head hq reads kv head hq // 4
    assert np.array_equal(out, want)


def test_placement_permutation_is_bit_identical():
    """Moving every block to another physical id (tables rewritten) gives identical bits."""
    wl = W.custom(seed=7, num_seqs=5, num_q_heads=8, num_kv_heads=4, head_dim=128, block_size=16,
                  lens=[40, 333, 1, 700, 129], dtype="bf16")
    st = wl.steps[0]
    dev = DeviceState(wl)
    dev.write(st)
    base = dev.decode(st, partition_tokens=64)
    nb = wl.num_blocks
    perm = np.random.default_rng(1).permutation(nb)
    kc = host_bits(dev.k_cache)
    vc = host_bits(dev.v_cache)
    kc2 = np.empty_like(kc)
    vc2 = np.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    tables = np.where(st.block_tables >= 0, perm[np.clip(st.block_tables, 0, None)], -1).astype(np.int32)
    dev.k_cache = to_dev(kc2, wl.dtype)
    dev.v_cache = to_dev(vc2, wl.dtype)
    moved = dev.decode(st, partition_tokens=64, tables=tables)
    assert np.array_equal(base, moved)


def test_shared_prefix_equals_private_copies():
    """Tables naming shared prefix blocks give the same bits as tables with private copies,
    and the shared blocks' bytes are unchanged by the step's writes."""
    wl = W.shared_prefix(num_steps=2)
    st = wl.steps[0]
    dev = DeviceState(wl)
    prefix_ids = np.unique(st.block_tables[:8, :64])
    assert prefix_ids.size == 64
    before = host_bits(dev.k_cache)[prefix_ids]
    dev.write(st)
    after = host_bits(dev.k_cache)[prefix_ids]
    assert np.array_equal(before, after), "a step's writes must not touch shared prefix blocks"
    shared = dev.decode(st)
    # give sequences 1..7 of group 0 private copies of the prefix
    kc = host_bits(dev.k_cache)
    vc = host_bits(dev.v_cache)
    used = set(np.unique(st.block_tables[st.block_tables >= 0]).tolist())
    free = [b for b in range(wl.num_blocks) if b not in used]
    tables = st.block_tables.copy()
    for s in range(1, 8):
        for i in range(64):
            nid = free.pop()
            kc[nid] = kc[tables[s, i]]
            vc[nid] = vc[tables[s, i]]
            tables[s, i] = nid
    dev.k_cache = to_dev(kc, wl.dtype)
    dev.v_cache = to_dev(vc, wl.dtype)
    private = dev.decode(st, tables=tables)
    assert np.array_equal(shared, private)


def test_deterministic_run_to_run():
    wl = W.custom(seed=8, num_seqs=7, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                  lens=[3000, 17, 800, 1, 2048, 999, 64], dtype="bf16")
    st = wl.steps[0]
    dev = DeviceState(wl)
    dev.write(st)
    a = dev.decode(st)
    b = dev.decode(st)
    c = dev.decode(st, partition_tokens=128)
    d = dev.decode(st, partition_tokens=128)
    assert np.array_equal(a, b) and np.array_equal(c, d)


def test_partition_sizes_agree():
    """Every chunk length of the tile stream agrees with the oracle (4096 tokens: no cut at all)."""
    wl = W.custom(seed=9, num_seqs=3, num_q_heads=4, num_kv_heads=4, head_dim=128, block_size=32,
                  lens=[1024, 1000, 33], dtype="fp16", key_boost_frac=0.01, key_boost=8.0)
    st = wl.steps[0]
    dev = DeviceState(wl)
    dev.write(st)
    _, _, ref = oracle_step(wl, wl.k_cache, wl.v_cache, st)
    outs = {}
    for part in (16, 32, 64, 96, 128, 256, 512, 1024, 4096):
        outs[part] = dev.decode(st, partition_tokens=part)
        compare(outs[part], ref, "fp16", what=f"partition {part}")


def test_full_table_and_maximum_context():
    """Context length equal to the table's capacity (every entry used), at the largest partition."""
    lens = [32 * 64, 32 * 64 - 1, 16]
    wl = W.custom(seed=10, num_seqs=3, num_q_heads=8, num_kv_heads=8, head_dim=64, block_size=32, lens=lens,
                  dtype="bf16", table_width=64)
    st = wl.steps[0]
    dev = DeviceState(wl)
    dev.write(st)
    _, _, ref = oracle_step(wl, wl.k_cache, wl.v_cache, st)
    for part in (0, 1024):
        compare(dev.decode(st, partition_tokens=part), ref, "bf16", what=f"full table part {part}")
    assert pa.device_status() == 0


def test_zero_length_and_empty_batch():
    wl = W.custom(seed=11, num_seqs=3, num_q_heads=4, num_kv_heads=4, head_dim=64, block_size=16, lens=[0, 20, 0],
                  dtype="fp16")
    st = wl.steps[0]
    dev = DeviceState(wl)
    dev.write(st)
    out = dev.decode(st, partition_tokens=16)
    _, _, ref = oracle_step(wl, wl.k_cache, wl.v_cache, st)
    assert np.all(out[0] == 0) and np.all(out[2] == 0)
    compare(out, ref, "fp16", what="zero-length rows")
    # empty batch and empty write launch nothing and succeed
    n0 = pa.launch_count()
    empty_q = torch.empty((0, 4, 64), dtype=torch.float16, device="cuda")
    res = pa.decode(empty_q, dev.k_cache, dev.v_cache, torch.empty((0, 2), dtype=torch.int32, device="cuda"),
                    torch.empty((0,), dtype=torch.int32, device="cuda"), 0.125, max_context_len=0)
    assert res.shape == (0, 4, 64)
    e = torch.empty((0, 4, 64), dtype=torch.float16, device="cuda")
    pa.write_kv(e, e, dev.k_cache, dev.v_cache, torch.empty((0,), dtype=torch.int64, device="cuda"))
    assert pa.launch_count() == n0
    assert pa.device_status() == 0


def test_write_kv_strided_and_padding_slots():
    """k/v as views into a wider per-token buffer (fused projection layout); slot -1 is skipped."""
    rng = np.random.default_rng(12)
    nb, hkv, bs, d, T = 20, 4, 16, 128, 50
    kc = rng.integers(0, 65536, size=(nb, hkv, bs, d), dtype=np.uint16)
    vc = rng.integers(0, 65536, size=(nb, hkv, bs, d), dtype=np.uint16)
    fused = rng.integers(0, 65536, size=(T, 3 * hkv * d), dtype=np.uint16)
    slots = rng.permutation(nb * bs)[:T].astype(np.int64)
    slots[::5] = -1
    import oracle
    k_np = fused[:, hkv * d:2 * hkv * d].reshape(T, hkv, d)
    v_np = fused[:, 2 * hkv * d:].reshape(T, hkv, d)
    want_k, want_v = oracle.write_kv(k_np, v_np, kc, vc, slots, bs)
    dk = to_dev(kc, "bf16")
    dv = to_dev(vc, "bf16")
    f = to_dev(fused, "bf16")
    pa.write_kv(f[:, hkv * d:2 * hkv * d].view(T, hkv, d), f[:, 2 * hkv * d:].view(T, hkv, d), dk, dv,
                to_dev_index(slots))
    assert np.array_equal(host_bits(dk), want_k) and np.array_equal(host_bits(dv), want_v)
