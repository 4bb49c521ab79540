"""The seeded workload generators produce what the decode step assumes (CPU only)."""
import numpy as np
import pytest

import workloads as W


def _check_step(wl, st, shared_ok=False):
    S = st.num_seqs
    assert st.block_tables.shape[0] == S and st.q.shape == (S, wl.num_q_heads, wl.head_dim)
    used = []
    for s in range(S):
        L = int(st.context_lens[s])
        nblk = -(-L // wl.block_size)
        row = st.block_tables[s]
        assert np.all((row[:nblk] >= 0) & (row[:nblk] < wl.num_blocks)), "table entries inside the pool"
        assert np.all(row[nblk:] == W.TABLE_PAD), "entries past the end are padding"
        used.extend(row[:nblk].tolist())
    if not shared_ok:
        assert len(used) == len(set(used)), "independent sequences never share a block"
    # the step writes token L-1 of every sequence into its own slot
    for s in range(S):
        L = int(st.context_lens[s])
        blk = st.block_tables[s, (L - 1) // wl.block_size]
        assert st.slot_mapping[-S + s] == blk * wl.block_size + (L - 1) % wl.block_size
    assert len(set(st.slot_mapping.tolist())) == len(st.slot_mapping), "slots are distinct"


def test_tiny_matches_its_description():
    wl = W.tiny()
    st = wl.steps[0]
    assert (wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block_size, wl.num_blocks, wl.dtype) == \
        (8, 8, 64, 16, 64, "fp16")
    assert st.num_seqs == 4 and np.all((st.context_lens >= 1) & (st.context_lens <= 200))
    _check_step(wl, st)


def test_llama2_shape_small():
    wl = W.llama2_7b(num_seqs=6, num_blocks=1024)
    st = wl.steps[0]
    assert (wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block_size, wl.dtype) == (32, 32, 128, 16, "fp16")
    assert np.all((st.context_lens >= 128) & (st.context_lens <= 2048))
    assert wl.scale == pytest.approx(1 / np.sqrt(128))
    _check_step(wl, st)


def test_unowned_slots_hold_nan_and_owned_rows_do_not():
    wl = W.custom(seed=3, num_seqs=3, num_q_heads=2, num_kv_heads=2, head_dim=64, block_size=16,
                  lens=[1, 17, 40])
    st = wl.steps[0]
    nan = W.NAN_BITS["fp16"]
    for s, L in enumerate(st.context_lens):
        for j in range(-(-int(L) // 16) * 16):
            blk, row = st.block_tables[s, j // 16], j % 16
            cell = wl.k_cache[blk, :, row, :]
            if j < L - 1:
                assert not np.all(cell == nan), "rows before the new token hold data"
            else:
                assert np.all(cell == nan), "the new token's slot and the rows after it are empty"
    assert st.k_new.shape == (3, 2, 64)


def test_long_context_key_boost():
    wl = W.long_context(num_seqs=1, num_blocks=80, lo=2000, hi=2500)
    st = wl.steps[0]
    L = int(st.context_lens[0])
    k = np.array([wl.k_cache[st.block_tables[0, j // 32], 0, j % 32, :] for j in range(L - 1)])
    mag = np.abs(k.view(np.uint16).astype(np.uint32) << 16).view(np.float32).max(axis=1)
    boosted = np.sum(mag > 5.0)  # N(0,1) rows almost never exceed 5; boosted rows (x8) usually do
    assert 0.5 * 0.01 * L <= boosted <= 2 * 0.01 * L + 2


def test_gqa_lengths_are_lognormal_and_clipped():
    wl = W.gqa_llama3(num_seqs=64, num_blocks=8192)
    L = wl.steps[0].context_lens
    assert L.min() >= 16 and L.max() <= 8192
    assert 300 < np.median(L) < 900


def test_shared_prefix_session():
    wl = W.shared_prefix(num_steps=10, retire_after=5)
    assert len(wl.steps) == 10
    for i, st in enumerate(wl.steps):
        assert st.num_seqs == 64
        _check_step(wl, st, shared_ok=True)
        for g in range(8):  # each group's 8 tables name the same 64 prefix blocks
            pre = st.block_tables[8 * g:8 * g + 8, :64]
            assert np.all(pre == pre[0])
        # no write ever lands in a shared prefix block
        prefix_blocks = set(st.block_tables[:, :64].ravel().tolist())
        assert not (set((st.slot_mapping // 16).tolist()) & prefix_blocks) or i == 5
    # after the retire step, blocks of the retired group are reused by the newcomers
    before = set(wl.steps[4].block_tables[:8].ravel().tolist()) - {W.TABLE_PAD}
    after = set(wl.steps[5].block_tables[56:].ravel().tolist()) - {W.TABLE_PAD}
    assert before & after


def test_generators_are_deterministic():
    a = W.custom(seed=9, num_seqs=2, num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=32, lens=[50, 3])
    b = W.custom(seed=9, num_seqs=2, num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=32, lens=[50, 3])
    assert np.array_equal(a.k_cache, b.k_cache) and np.array_equal(a.steps[0].q, b.steps[0].q)
    assert np.array_equal(a.steps[0].block_tables, b.steps[0].block_tables)


def test_unique_and_logical_bytes():
    wl = W.shared_prefix(num_steps=1)
    st = wl.steps[0]
    logical = W.kv_bytes(st, 8, 128)
    unique = W.unique_kv_bytes(st, 8, 128, 16)
    assert unique < logical
    # the eight 64-block prefixes are counted once in the unique figure
    assert logical - unique >= 7 * 8 * 1024 * 8 * 128 * 2 * 2


def test_prefill_case_structure():
    shape = [(1, 1), (40, 8), (300, 129), (16, 0), (64, 64)]
    c = W.prefill_case(3, shape, 8, 2, 64, 16, "bf16")
    assert c.query_start.tolist() == [0, 1, 9, 138, 138, 202]
    assert c.context_lens.tolist() == [1, 40, 300, 16, 64]
    assert c.q.shape == (202, 8, 64) and c.q.dtype == np.uint16
    assert c.max_query_len == 129
    # attended (query, key) pairs: n (L - n) + n (n + 1) / 2 per sequence
    assert c.attended_pairs == sum(n * (L - n) + n * (n + 1) // 2 for L, n in shape)
    # every table entry a sequence needs is a distinct block of the pool; the rest is padding
    used = []
    for s, (L, _) in enumerate(shape):
        nblk = -(-L // 16)
        row = c.block_tables[s]
        assert (row[:nblk] >= 0).all() and (row[:nblk] < c.num_blocks).all()
        assert (row[nblk:] == W.TABLE_PAD).all()
        used += row[:nblk].tolist()
    assert len(used) == len(set(used))
    # slots no sequence owns hold NaN; owned slots hold finite draws
    owned = np.zeros((c.num_blocks, 16), dtype=bool)
    for s, (L, _) in enumerate(shape):
        for j in range(L):
            owned[c.block_tables[s, j // 16], j % 16] = True
    kc = c.k_cache.transpose(0, 2, 1, 3)  # [NB, bs, Hkv, d]
    assert (kc[~owned] == W.NAN_BITS["bf16"]).all()
    vals = (kc[owned].astype(np.uint32) << 16).view(np.float32)
    assert np.isfinite(vals).all()


def test_named_prefill_workloads_are_deterministic():
    for name, make in W.PREFILL_NAMED.items():
        a, b = make(), make()
        assert a.name == name
        assert np.array_equal(a.q, b.q) and np.array_equal(a.block_tables, b.block_tables)
        assert np.array_equal(a.query_start, b.query_start) and np.array_equal(a.context_lens, b.context_lens)
        assert (a.context_lens >= np.diff(a.query_start)).all()
        assert a.max_query_len <= 2048
