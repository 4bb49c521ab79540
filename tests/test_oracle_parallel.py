"""The OpenMP build of the oracle's decode (used only to time the oracle on every host core)
gives the single-thread oracle's results bit for bit: it runs the same gather-then-attend steps
per (sequence, query head), only on several threads."""
import numpy as np
import pytest

import oracle
import workloads as W


@pytest.mark.parametrize("hq,hkv,d,bs,dtype", [(8, 8, 64, 16, "fp16"), (32, 8, 128, 16, "bf16"),
                                               (8, 2, 128, 32, "fp16")])
def test_parallel_decode_equals_serial(hq, hkv, d, bs, dtype):
    lens = [0, 1, 15, 16, 17, 100, 333, 700]
    wl = W.custom(seed=hq + hkv + d + bs, num_seqs=len(lens), num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                  block_size=bs, lens=lens, dtype=dtype)
    st = wl.steps[0]
    kc, vc = oracle.write_kv(st.k_new, st.v_new, wl.k_cache, wl.v_cache, st.slot_mapping, wl.block_size)
    serial = oracle.decode(st.q, kc, vc, st.block_tables, st.context_lens, wl.scale, wl.dtype)
    par = oracle.decode(st.q, kc, vc, st.block_tables, st.context_lens, wl.scale, wl.dtype, parallel=True)
    assert np.array_equal(serial, par)
    assert not np.any(par[0])  # the empty sequence's rows are zero


def test_parallel_decode_refuses_what_the_serial_one_refuses():
    wl = W.custom(seed=3, num_seqs=2, num_q_heads=4, num_kv_heads=4, head_dim=64, block_size=16, lens=[20, 40],
                  dtype="fp16")
    st = wl.steps[0]
    bt = st.block_tables.copy()
    bt[1, 1] = wl.num_blocks  # outside the pool
    for par in (False, True):
        with pytest.raises(ValueError, match="block id"):
            oracle.decode(st.q, wl.k_cache, wl.v_cache, bt, st.context_lens, wl.scale, wl.dtype, parallel=par)


def test_thread_count_is_reported():
    assert oracle.parallel_threads() >= 1
