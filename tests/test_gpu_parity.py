"""CUDA path against the fp64 oracle, element by element (needs a B200)."""
import gc
import json

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from gpu_util import DeviceState, compare, host_bits, oracle_step, require_gpu

pytestmark = pytest.mark.gpu


def _free():
    gc.collect()
    torch.cuda.empty_cache()


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    yield
    _free()


@pytest.mark.parametrize("name", ["tiny_decode", "llama2_7b_decode", "gqa_llama3_decode", "long_context_splitk"])
def test_full_config_write_and_decode(name):
    """Full-size single-step workloads: the KV write is bit-exact over the whole pool and every
    output element is within tolerance of the oracle, in the launch configuration the bench times."""
    wl = W.NAMED[name]()
    st = wl.steps[0]
    dev = DeviceState(wl)
    dev.write(st)
    out = dev.decode(st)
    torch.cuda.synchronize()
    import paged_kv_cache_457_b200 as pa
    assert pa.device_status() == 0
    kc, vc, ref = oracle_step(wl, wl.k_cache, wl.v_cache, st)
    assert np.array_equal(host_bits(dev.k_cache), kc), "k_cache differs from the oracle's scatter"
    assert np.array_equal(host_bits(dev.v_cache), vc), "v_cache differs from the oracle's scatter"
    stats = compare(out, ref, wl.dtype, what=name)
    print(name, json.dumps(stats))
    del dev, kc, vc
    _free()


def test_shared_prefix_steps():
    """16 continuous-batching steps over shared-prefix groups (retire + join after step 8):
    every step's cache is bit-exact; outputs are checked in full on steps 0, 8 and 15 and on
    eight sampled sequences on the others."""
    wl = W.shared_prefix()
    dev = DeviceState(wl)
    kc, vc = wl.k_cache, wl.v_cache
    rng = np.random.default_rng(0)
    for i, st in enumerate(wl.steps):
        dev.write(st)
        out = dev.decode(st)
        seqs = None if i in (0, 8, 15) else np.sort(rng.choice(st.num_seqs, 8, replace=False))
        kc, vc, ref = oracle_step(wl, kc, vc, st, seqs)
        got = out if seqs is None else out[seqs]
        compare(got, ref, wl.dtype, what=f"step {i}")
        if i in (0, 8, 15):
            assert np.array_equal(host_bits(dev.k_cache), kc), f"k_cache differs at step {i}"
            assert np.array_equal(host_bits(dev.v_cache), vc), f"v_cache differs at step {i}"
    import paged_kv_cache_457_b200 as pa
    assert pa.device_status() == 0


SMALL = [  # (hq, hkv, d, bs, dtype)
    (4, 4, 64, 16, "fp16"),
    (8, 8, 128, 16, "bf16"),
    (8, 2, 128, 32, "fp16"),
    (8, 1, 64, 32, "bf16"),
    (6, 2, 128, 16, "bf16"),
    (12, 4, 64, 16, "fp16"),
    (16, 2, 128, 16, "bf16"),
    (2, 2, 128, 32, "bf16"),
    (4, 2, 64, 16, "bf16"),     # group 2
    (10, 2, 128, 16, "fp16"),   # group 5
    (12, 2, 64, 32, "bf16"),    # group 6
    (14, 2, 128, 16, "bf16"),   # group 7
    (24, 2, 128, 16, "fp16"),   # group 12: two chunks of 6 heads per kv head
    (32, 2, 64, 16, "bf16"),    # group 16: two chunks of 8 heads per kv head
]
LENS = [1, 2, 15, 16, 17, 31, 33, 100, 257, 512, 513, 777, 1024, 1025]


@pytest.mark.parametrize("hq,hkv,d,bs,dtype", SMALL)
@pytest.mark.parametrize("partition", [0, 16, 48, 512])
def test_small_shapes(hq, hkv, d, bs, dtype, partition):
    """Every supported head dim / block size / group size / dtype, ragged lengths spanning
    several tiles, with the balanced split and with fixed chunks of 1, 3 and 32 tiles (so
    sequences are cut at every kind of offset and pieces straddle sequence boundaries)."""
    wl = W.custom(seed=hq * 1000 + hkv * 100 + d + bs, num_seqs=len(LENS), num_q_heads=hq, num_kv_heads=hkv,
                  head_dim=d, block_size=bs, lens=LENS, dtype=dtype)
    st = wl.steps[0]
    dev = DeviceState(wl)
    dev.write(st)
    out = dev.decode(st, partition_tokens=partition)
    _, _, ref = oracle_step(wl, wl.k_cache, wl.v_cache, st)
    compare(out, ref, dtype, what=f"{hq}/{hkv} d{d} bs{bs} {dtype} part {partition}")


@pytest.mark.parametrize("hq,hkv,dtype", [(32, 8, "fp16"), (8, 8, "fp16")])
def test_many_short_sequences(hq, hkv, dtype):
    """3000 sequences of 1 to 32 tokens and six of 1000 (tensor-core and CUDA-core paths).  The split
    kernels' tile prefix then takes 12 KB of shared memory per block (fewer blocks per SM), each thread
    of its scan covers 24 sequences, most chunks hold many whole segments and the long ones are cut
    across chunks: every output row against the oracle.  fp16 storage: contexts this short give outputs
    up to about 4 in magnitude, where one bf16 ulp (2^-6) is already above the 1e-2 bound."""
    rng = np.random.default_rng(77)
    lens = rng.integers(1, 33, size=3000)
    lens[::500] = 1000
    wl = W.custom(seed=78, num_seqs=len(lens), num_q_heads=hq, num_kv_heads=hkv, head_dim=128, block_size=16,
                  lens=lens, dtype=dtype)
    st = wl.steps[0]
    dev = DeviceState(wl)
    dev.write(st)
    out = dev.decode(st)
    import paged_kv_cache_457_b200 as pa
    assert pa.device_status() == 0
    _, _, ref = oracle_step(wl, wl.k_cache, wl.v_cache, st)
    compare(out, ref, dtype, what=f"3006 seqs {hq}/{hkv} {dtype}")
    del dev
    _free()


SEGMENT_SHAPES = [  # (hq, hkv, d, bs, dtype): CUDA-core groups of 1 and 2 heads
    (8, 8, 64, 16, "fp16"),
    (8, 8, 128, 32, "bf16"),
    (8, 4, 128, 16, "bf16"),
    (4, 2, 64, 32, "fp16"),
]
SEGMENT_LENS = [0, 1, 2, 15, 16, 17, 31, 33, 100, 255, 256, 257, 400, 511, 512]


@pytest.mark.parametrize("hq,hkv,d,bs,dtype", SEGMENT_SHAPES)
def test_small_batch_segment_path(hq, hkv, d, bs, dtype):
    """Small batches with short contexts take the per-segment kernel (one block per (sequence, head
    chunk), no workspace, no merge kernel): checked against the oracle, with an empty sequence and
    ragged lengths up to 32 tiles, and against the split path (fixed chunks of one tile) on the same
    inputs."""
    import paged_kv_cache_457_b200 as pa
    wl = W.custom(seed=500 + hq + hkv + d + bs, num_seqs=len(SEGMENT_LENS), num_q_heads=hq, num_kv_heads=hkv,
                  head_dim=d, block_size=bs, lens=SEGMENT_LENS, dtype=dtype)
    st = wl.steps[0]
    assert pa.decode_workspace_size(st.num_seqs, hq, hkv, d, bs, st.max_context_len, 0) == 0, \
        "expected the per-segment path (it needs no workspace)"
    dev = DeviceState(wl)
    dev.write(st)
    seg = dev.decode(st, partition_tokens=0)
    split = dev.decode(st, partition_tokens=16)
    assert pa.device_status() == 0
    _, _, ref = oracle_step(wl, wl.k_cache, wl.v_cache, st)
    compare(seg, ref, dtype, what=f"segment path {hq}/{hkv} d{d} bs{bs} {dtype}")
    compare(split, ref, dtype, what=f"split path {hq}/{hkv} d{d} bs{bs} {dtype}")
    assert not np.any(seg[0])  # the empty sequence's rows are zero
    assert np.array_equal(seg, dev.decode(st, partition_tokens=0)), "not deterministic"


def test_small_batch_segment_path_one_full_wave():
    """As many segments as the per-segment kernel takes in one wave of blocks (and one more, which
    falls back to the split path), checked against the oracle on sampled sequences."""
    import paged_kv_cache_457_b200 as pa
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    rng = np.random.default_rng(7)
    for extra in (0, 1):
        S = None
        # the largest batch of 8-head sequences the segment path accepts: S * 8 segments in one wave
        for cand in range(sms * 4, 0, -1):
            if pa.decode_workspace_size(cand, 8, 8, 64, 16, 200, 0) == 0:
                S = cand
                break
        assert S is not None
        S += extra
        lens = [int(x) for x in rng.integers(1, 201, size=S)]
        wl = W.custom(seed=600 + extra, num_seqs=S, num_q_heads=8, num_kv_heads=8, head_dim=64, block_size=16,
                      lens=lens, dtype="fp16")
        st = wl.steps[0]
        assert (pa.decode_workspace_size(S, 8, 8, 64, 16, st.max_context_len, 0) == 0) == (extra == 0)
        dev = DeviceState(wl)
        dev.write(st)
        out = dev.decode(st)
        assert pa.device_status() == 0
        seqs = np.sort(rng.choice(S, 12, replace=False))
        _, _, ref = oracle_step(wl, wl.k_cache, wl.v_cache, st, seqs)
        compare(out[seqs], ref, "fp16", what=f"{S} sequences")


PAIR_SHAPES = [  # (hq, hkv, d, bs, dtype): tensor-core groups of 3 and 4 heads
    (8, 2, 128, 16, "bf16"),
    (8, 2, 64, 32, "fp16"),
    (6, 2, 128, 32, "fp16"),
    (12, 4, 64, 16, "bf16"),
]
# (L0, L1, blocks of the first sequence's table the second one names too: a prefix they share)
PAIR_LENS = [(1040, 1040, 64), (300, 520, 10), (17, 900, 1), (900, 17, 1), (0, 50, 0), (70, 0, 0), (256, 256, 15),
             (33, 2000, 2), (1, 1, 0), (640, 333, 0), (129, 129, 8), (47, 0, 0), (5000, 4000, 200)]


def _paired_case(hq, hkv, d, bs, dtype, seed):
    lens = [x for L0, L1, _ in PAIR_LENS for x in (L0, L1)] + [613]  # an odd batch: the last unit has one sequence
    wl = W.custom(seed=seed, num_seqs=len(lens), num_q_heads=hq, num_kv_heads=hkv, head_dim=d, block_size=bs,
                  lens=lens, dtype=dtype)
    st = wl.steps[0]
    tables = st.block_tables.copy()
    for i, (L0, L1, blocks) in enumerate(PAIR_LENS):
        # name the first sequence's leading blocks in the second one's table (a shared prefix); the new tokens
        # written by the step stay in unshared blocks
        share = min(blocks * 16 // bs, max(0, (min(L0, L1) - 1) // bs))
        tables[2 * i + 1, :share] = tables[2 * i, :share]
    return wl, st, tables


@pytest.mark.parametrize("hq,hkv,d,bs,dtype", PAIR_SHAPES)
@pytest.mark.parametrize("partition", [0, 16, 48])
def test_shared_prefix_tables(hq, hkv, d, bs, dtype, partition):
    """Consecutive sequences whose tables name the same leading blocks (shared prefixes of every length:
    long, short, one block, none), an empty sequence on either side of such a pair, and an odd batch, on
    the tensor-core path, against the oracle through the same tables, with the balanced split and with
    chunks of 1 and 3 tiles (pieces cut inside the shared blocks and inside each sequence's own)."""
    import paged_kv_cache_457_b200 as pa
    wl, st, tables = _paired_case(hq, hkv, d, bs, dtype, seed=700 + hq + d + bs)
    dev = DeviceState(wl)
    dev.write(st)
    out = dev.decode(st, partition_tokens=partition, tables=tables)
    assert pa.device_status() == 0
    kc, vc = oracle.write_kv(st.k_new, st.v_new, wl.k_cache, wl.v_cache, st.slot_mapping, wl.block_size)
    ref = oracle.decode(st.q, kc, vc, tables, st.context_lens, wl.scale, wl.dtype)
    compare(out, ref, dtype, what=f"shared prefixes {hq}/{hkv} d{d} bs{bs} {dtype} part {partition}")
    for s, L in enumerate(st.context_lens):
        if L == 0:
            assert not np.any(out[s]), f"sequence {s} (empty) not zero"


def test_shared_prefix_bad_block_zeroes_only_its_sequence():
    """A table entry outside the pool in one of two sequences that share their first blocks zeroes that
    sequence's rows only (and sets the status bit); its partner and the rest are exact."""
    import paged_kv_cache_457_b200 as pa
    wl, st, tables = _paired_case(8, 2, 128, 16, "bf16", seed=77)
    tables[3, 25] = wl.num_blocks + 3  # sequence 3 (pair 1: 300 / 520 tokens, 10 shared blocks), its own part
    dev = DeviceState(wl)
    dev.write(st)
    for part in (0, 48):
        out = dev.decode(st, partition_tokens=part, tables=tables)
        assert pa.device_status() == pa.DEV_ERR_BLOCK_ID
        assert not np.any(out[3])
        good = [s for s in range(st.num_seqs) if s != 3]
        kc, vc = oracle.write_kv(st.k_new, st.v_new, wl.k_cache, wl.v_cache, st.slot_mapping, wl.block_size)
        ref = oracle.decode(st.q[good], kc, vc, tables[good], st.context_lens[good], wl.scale, wl.dtype)
        compare(out[good], ref, "bf16", what=f"the other sequences, part {part}")
