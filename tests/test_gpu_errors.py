"""Error paths: host-side rejections, device status bits, the bounded wait (B200).

Nothing here faults or hangs the GPU: bad table entries and slots are caught by the
kernels' own bounds checks before any access, and the timeout self-test waits on a
shared-memory barrier with a 10 ms limit.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_457_b200 as pa
import workloads as W
from gpu_util import DeviceState, compare, oracle_step, require_gpu, to_dev, to_dev_index

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    pa.device_status(clear=True)


def _case(lens, **kw):
    args = dict(seed=21, num_seqs=len(lens), num_q_heads=4, num_kv_heads=2, head_dim=128, block_size=16, lens=lens,
                dtype="fp16")
    args.update(kw)
    wl = W.custom(**args)
    st = wl.steps[0]
    dev = DeviceState(wl)
    dev.write(st)
    return wl, st, dev


def test_block_id_out_of_range_zeroes_only_that_sequence():
    wl, st, dev = _case([40, 300, 90])
    tables = st.block_tables.copy()
    tables[1, 2] = wl.num_blocks + 5  # past the pool: never dereferenced
    for part in (0, 64):
        out = dev.decode(st, tables=tables, partition_tokens=part)
        assert pa.device_status() == pa.DEV_ERR_BLOCK_ID
        assert np.all(out[1] == 0)
        _, _, ref = oracle_step(wl, wl.k_cache, wl.v_cache, st, seqs=[0, 2])
        compare(out[[0, 2]], ref, "fp16", what="neighbours of a bad table")
    tables[1, 2] = -3
    dev.decode(st, tables=tables)
    assert pa.device_status() == pa.DEV_ERR_BLOCK_ID


def test_context_longer_than_table_or_hint():
    wl, st, dev = _case([40, 60])
    lens = st.context_lens.copy()
    lens[0] = st.block_tables.shape[1] * 16 + 1  # beyond the table's capacity
    out = dev.decode(st, lens=lens, max_context_len=int(lens.max()))
    assert pa.device_status() & pa.DEV_ERR_CONTEXT
    assert np.all(out[0] == 0)
    lens = st.context_lens.copy()
    out = dev.decode(st, lens=lens, max_context_len=int(lens.max()) - 1)  # hint too small for seq 1
    assert pa.device_status() == pa.DEV_ERR_CONTEXT_HINT
    assert np.all(out[1] == 0)


def test_slot_out_of_range_is_skipped_and_flagged():
    wl, st, dev = _case([10, 20])
    k = to_dev(st.k_new, "fp16")
    before = dev.k_cache.clone()
    bad = to_dev_index(np.array([wl.num_blocks * 16, -1], dtype=np.int64))
    pa.write_kv(k, k, dev.k_cache, dev.v_cache, bad)
    assert pa.device_status() == pa.DEV_ERR_SLOT
    assert torch.equal(before.view(torch.int16), dev.k_cache.view(torch.int16))  # bits: the pool holds NaN


def test_bounded_wait_times_out_with_status():
    pa.debug_wait_timeout(10_000_000)
    assert pa.device_status() == pa.DEV_ERR_TIMEOUT
    # the context is still usable afterwards
    wl, st, dev = _case([5])
    dev.decode(st)
    assert pa.device_status() == 0


def test_host_rejections_launch_nothing():
    wl, st, dev = _case([30])
    q = to_dev(st.q, "fp16")
    tables = to_dev_index(st.block_tables)
    lens = to_dev_index(st.context_lens)
    n0 = pa.launch_count()
    with pytest.raises(pa.PagedAttentionError):
        pa.decode(q, dev.k_cache, dev.v_cache, tables, lens, 0.1, max_context_len=30, partition_tokens=24)
    with pytest.raises(pa.PagedAttentionError):
        pa.decode(q, dev.k_cache, dev.v_cache, tables, lens, 0.1, max_context_len=30,
                  workspace=torch.empty(0, dtype=torch.uint8, device="cuda"), partition_tokens=16)
    with pytest.raises(pa.PagedAttentionError):
        pa.decode(q.float(), dev.k_cache, dev.v_cache, tables, lens, 0.1, max_context_len=30)
    with pytest.raises(pa.PagedAttentionError):
        pa.decode(q, dev.k_cache, dev.v_cache, tables.long(), lens, 0.1, max_context_len=30)
    assert pa.launch_count() == n0
