"""The native page pool on the host: lifecycle, copy-on-write, swap plans, step tables.

A random driver applies the manager's plans to label pools (one label per
token slot, moved the way the kernels move K/V) and checks after every call
that each sequence still reads its own tokens through its table, that the
reference counts equal the number of tables naming each page, and that a
failed call changed nothing.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import paged_kv_cache_457_b200 as pa
from paged_kv_cache_457_b200 import build_lib
from paged_kv_cache_457_b200.block_manager import BlockManagerError


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build_lib.build()
    pa.load_library()


def test_prompt_pages_and_slots():
    bm = pa.BlockManager(16, 10)
    bm.add_sequence(7, 33)
    t = bm.block_table(7)
    assert list(t) == [0, 1, 2]  # a fresh pool hands out ascending ids
    assert bm.num_free_device_blocks == 7
    assert list(bm.slots(7, 30, 3)) == [1 * 16 + 14, 1 * 16 + 15, 2 * 16 + 0]
    bm.add_sequence(8, 0)
    assert len(bm.block_table(8)) == 0
    slot, cow = bm.append_slot(8)
    assert cow is None and slot == int(bm.block_table(8)[0]) * 16
    with pytest.raises(BlockManagerError) as e:
        bm.add_sequence(7, 1)
    assert e.value.code == -23
    with pytest.raises(BlockManagerError) as e:
        bm.add_sequence(9, 16 * 7 + 1)  # 8 pages, 6 free
    assert e.value.code == -21
    with pytest.raises(BlockManagerError) as e:
        bm.slots(7, 30, 4)  # token 33 has no page yet
    assert e.value.code == -20


def test_fork_shares_and_copy_on_write_splits_a_partial_page():
    bm = pa.BlockManager(16, 8)
    bm.add_sequence(1, 21)  # pages 0 (full), 1 (5 tokens)
    bm.fork(1, 2)
    assert bm.ref_count(0) == 2 and bm.ref_count(1) == 2
    slot, cow = bm.append_slot(2)  # writes into shared page 1 -> private copy
    assert cow == (1, 2)
    assert list(bm.block_table(2)) == [0, 2] and list(bm.block_table(1)) == [0, 1]
    assert slot == 2 * 16 + 5
    assert bm.ref_count(1) == 1 and bm.ref_count(2) == 1 and bm.ref_count(0) == 2
    slot, cow = bm.append_slot(1)  # page 1 is now private to seq 1: in place
    assert cow is None and slot == 1 * 16 + 5


def test_full_shared_page_is_not_copied():
    bm = pa.BlockManager(16, 8)
    bm.add_sequence(1, 32)
    bm.fork(1, 2)
    slot, cow = bm.append_slot(2)
    assert cow is None and list(bm.block_table(2)) == [0, 1, 2] and slot == 32
    assert bm.ref_count(0) == 2 and bm.ref_count(1) == 2


def test_decode_step_copies_once_per_sharing_sequence():
    """Three forks of a partly filled page: two copies, the last writer keeps the original."""
    bm = pa.BlockManager(16, 16)
    bm.add_sequence(0, 20)
    bm.fork(0, 1)
    bm.fork(0, 2)
    plan = bm.build_decode_step([0, 1, 2], 4)
    assert plan.copy_pairs.tolist() == [[1, 2], [1, 3]]
    assert plan.block_tables[:, :2].tolist() == [[0, 2], [0, 3], [0, 1]]
    assert (plan.block_tables[:, 2:] == -1).all()
    assert plan.context_lens.tolist() == [21, 21, 21]
    assert plan.slot_mapping.tolist() == [2 * 16 + 4, 3 * 16 + 4, 1 * 16 + 4]
    assert [bm.ref_count(b) for b in range(4)] == [3, 1, 1, 1]


def test_step_is_all_or_nothing():
    bm = pa.BlockManager(16, 3)
    bm.add_sequence(0, 16)
    bm.add_sequence(1, 16)
    bm.add_sequence(2, 15)
    before = [bm.block_table(i).tolist() for i in range(3)], bm.num_free_device_blocks
    with pytest.raises(BlockManagerError) as e:
        bm.build_decode_step([2, 0, 1], 4)  # 0 and 1 need a page each, none free
    assert e.value.code == -21
    assert ([bm.block_table(i).tolist() for i in range(3)], bm.num_free_device_blocks) == before
    assert [bm.num_tokens(i) for i in range(3)] == [16, 16, 15]
    with pytest.raises(BlockManagerError) as e:
        bm.build_decode_step([2], 0)  # table stride too small
    assert e.value.code == -25
    with pytest.raises(BlockManagerError) as e:
        bm.build_decode_step([2, 2], 4)  # repeated id
    assert e.value.code == -20
    assert bm.num_tokens(2) == 15


def test_swap_keeps_sharing_and_refuses_when_full():
    bm = pa.BlockManager(16, 8, num_host_blocks=3)
    bm.add_sequence(1, 40)  # 3 pages
    bm.fork(1, 2)
    m = bm.swap_out([1, 2])
    assert m.tolist() == [[0, 0], [1, 1], [2, 2]]  # each shared page crosses once
    assert bm.num_free_device_blocks == 8 and bm.num_free_host_blocks == 0
    assert [bm.ref_count(b, host=True) for b in range(3)] == [2, 2, 2]
    assert bm.is_swapped(1) and bm.is_swapped(2)
    with pytest.raises(BlockManagerError) as e:
        bm.append_slot(1)
    assert e.value.code == -24
    bm.add_sequence(3, 16 * 6)
    with pytest.raises(BlockManagerError) as e:
        bm.swap_in([1])  # 3 pages needed, 2 free
    assert e.value.code == -21
    assert bm.is_swapped(1)
    bm.free_sequence(3)
    m = bm.swap_in([2])
    assert sorted(m[:, 0].tolist()) == [0, 1, 2]
    assert [bm.ref_count(b, host=True) for b in range(3)] == [1, 1, 1]  # seq 1 still holds them
    bm.add_sequence(4, 1)
    with pytest.raises(BlockManagerError) as e:
        bm.swap_out([4])  # host pool is full
    assert e.value.code == -21


def test_bad_arguments():
    with pytest.raises(BlockManagerError):
        pa.BlockManager(0, 4)
    with pytest.raises(BlockManagerError):
        pa.BlockManager(16, -1)
    bm = pa.BlockManager(16, 4)
    for call in (lambda: bm.free_sequence(5), lambda: bm.fork(5, 6), lambda: bm.append_slot(5),
                 lambda: bm.block_table(5), lambda: bm.swap_out([5])):
        with pytest.raises(BlockManagerError) as e:
            call()
        assert e.value.code == -22
    lib = pa.load_library()
    assert lib.pa_bm_num_free_device_blocks(None) == -20
    assert lib.pa_bm_add_sequence(None, 1, 1) == -20
    assert lib.pa_bm_ref_count(bm._h, 0, 4) == -1


class LabelWorld:
    """The manager plus label pools moved the way the kernels move K/V."""

    def __init__(self, rng, bs, nd, nh):
        self.bm = pa.BlockManager(bs, nd, nh)
        self.bs, self.nd, self.nh = bs, nd, nh
        self.dev = np.full((nd, bs), -1, dtype=np.int64)
        self.host = np.full((nh, bs), -1, dtype=np.int64)
        self.tokens = {}  # seq -> list of labels
        self.rng = rng
        self.next_label = 0

    def label(self):
        self.next_label += 1
        return self.next_label

    def write(self, slot, lab):
        self.dev[slot // self.bs, slot % self.bs] = lab

    def snapshot(self):
        bm = self.bm
        return ({s: (bm.block_table(s).tolist(), bm.num_tokens(s), bm.is_swapped(s)) for s in self.tokens},
                bm.num_free_device_blocks, bm.num_free_host_blocks,
                [bm.ref_count(b) for b in range(self.nd)], [bm.ref_count(b, True) for b in range(self.nh)])

    def check(self):
        bm = self.bm
        refs_d = np.zeros(self.nd, dtype=np.int64)
        refs_h = np.zeros(self.nh, dtype=np.int64)
        for s, labs in self.tokens.items():
            t = bm.block_table(s)
            assert bm.num_tokens(s) == len(labs)
            assert len(t) == -(-len(labs) // self.bs)
            assert len(set(t.tolist())) == len(t)
            pool, refs = (self.host, refs_h) if bm.is_swapped(s) else (self.dev, refs_d)
            np.add.at(refs, t, 1)
            got = pool[t].reshape(-1)[: len(labs)]
            assert got.tolist() == labs, f"sequence {s} reads other tokens"
        assert [bm.ref_count(b) for b in range(self.nd)] == refs_d.tolist()
        assert [bm.ref_count(b, True) for b in range(self.nh)] == refs_h.tolist()
        assert bm.num_free_device_blocks == int((refs_d == 0).sum())
        assert bm.num_free_host_blocks == int((refs_h == 0).sum())

    # Each op returns True if the manager accepted it.
    def op_add(self, sid):
        n = int(self.rng.integers(0, 3 * self.bs))
        try:
            self.bm.add_sequence(sid, n)
        except BlockManagerError as e:
            assert e.code == -21
            return False
        labs = [self.label() for _ in range(n)]
        for slot, lab in zip(self.bm.slots(sid, 0, n), labs):
            self.write(int(slot), lab)
        self.tokens[sid] = labs
        return True

    def op_fork(self, parent, child):
        try:
            self.bm.fork(parent, child)
        except BlockManagerError as e:
            assert e.code == -24
            return False
        self.tokens[child] = list(self.tokens[parent])
        return True

    def op_step(self, ids, stride):
        try:
            plan = self.bm.build_decode_step(ids, stride)
        except BlockManagerError as e:
            assert e.code in (-21, -24, -25)
            return False
        src, dst = plan.copy_pairs[:, 0], plan.copy_pairs[:, 1]
        assert len(set(dst.tolist())) == len(dst) and not set(dst.tolist()) & set(src.tolist())
        self.dev[dst] = self.dev[src]  # copy-on-write before the write
        for sid, slot, ln, row in zip(ids, plan.slot_mapping, plan.context_lens, plan.block_tables):
            lab = self.label()
            self.write(int(slot), lab)
            self.tokens[sid].append(lab)
            assert ln == len(self.tokens[sid])
            assert row[: -(-ln // self.bs)].tolist() == self.bm.block_table(sid).tolist()
        assert len(set(plan.slot_mapping.tolist())) == len(ids)
        return True

    def op_swap(self, ids, out):
        try:
            m = self.bm.swap_out(ids) if out else self.bm.swap_in(ids)
        except BlockManagerError as e:
            assert e.code in (-21, -24)
            return False
        if len(m):
            if out:
                self.host[m[:, 1]] = self.dev[m[:, 0]]
            else:
                self.dev[m[:, 1]] = self.host[m[:, 0]]
        return True

    def op_free(self, sid):
        self.bm.free_sequence(sid)
        del self.tokens[sid]
        return True


@pytest.mark.parametrize("seed", range(6))
def test_random_lifecycle_keeps_every_sequence_intact(seed):
    rng = np.random.default_rng(seed)
    bs = [16, 32][seed % 2]
    w = LabelWorld(rng, bs, nd=24, nh=12)
    next_id = 0
    for it in range(400):
        live = sorted(w.tokens)
        on_dev = [s for s in live if not w.bm.is_swapped(s)]
        swapped = [s for s in live if w.bm.is_swapped(s)]
        r = rng.random()
        before = w.snapshot()
        if r < 0.15 or not live:
            ok = w.op_add(next_id)
            next_id += 1
        elif r < 0.25:
            ok = w.op_fork(int(rng.choice(live)), next_id)
            next_id += ok
        elif r < 0.65 and on_dev:
            k = int(rng.integers(1, len(on_dev) + 1))
            ids = [int(x) for x in rng.permutation(on_dev)[:k]]
            ok = w.op_step(ids, int(rng.choice([2, 8])))
        elif r < 0.75 and on_dev:
            ok = w.op_swap([int(x) for x in rng.permutation(on_dev)[: int(rng.integers(1, 3))]], True)
        elif r < 0.85 and swapped:
            ok = w.op_swap([int(x) for x in rng.permutation(swapped)[: int(rng.integers(1, 3))]], False)
        else:
            ok = w.op_free(int(rng.choice(live)))
        if not ok:
            assert w.snapshot() == before, f"failed call changed state at iteration {it}"
        w.check()


def test_manager_plans_through_the_oracle_decode():
    """The manager's tables, copies and slots, applied with the oracle's write / copy, give the
    same attention as the oracle over each sequence's tokens laid out contiguously."""
    rng = np.random.default_rng(3)
    dtype, hkv, hq, d, bs, nb = "fp16", 2, 4, 64, 16, 40
    from oracle_pins import to_bits
    bm = pa.BlockManager(bs, nb, 0)
    kc = np.zeros((nb, hkv, bs, d), dtype=np.uint16)
    vc = np.zeros_like(kc)
    logical = {}
    for sid, n in ((0, 37), (1, 16), (2, 5)):
        bm.add_sequence(sid, n)
        k = to_bits(rng.standard_normal((n, hkv, d)), dtype)
        v = to_bits(rng.standard_normal((n, hkv, d)), dtype)
        kc, vc = oracle.write_kv(k, v, kc, vc, bm.slots(sid, 0, n), bs)
        logical[sid] = (k, v)
    bm.fork(0, 3)
    logical[3] = logical[0]
    ids = [0, 1, 2, 3]
    for _ in range(20):
        plan = bm.build_decode_step(ids, 8)
        if len(plan.copy_pairs):
            kc, vc = oracle.copy_blocks(kc, vc, kc, vc, plan.copy_pairs)
        k = to_bits(rng.standard_normal((len(ids), hkv, d)), dtype)
        v = to_bits(rng.standard_normal((len(ids), hkv, d)), dtype)
        kc, vc = oracle.write_kv(k, v, kc, vc, plan.slot_mapping, bs)
        for i, sid in enumerate(ids):
            lk, lv = logical[sid]
            logical[sid] = (np.concatenate([lk, k[i:i + 1]]), np.concatenate([lv, v[i:i + 1]]))
        q = to_bits(rng.standard_normal((len(ids), hq, d)), dtype)
        got = oracle.decode(q, kc, vc, plan.block_tables, plan.context_lens, 0.125, dtype)
        for i, sid in enumerate(ids):
            lk, lv = logical[sid]
            L = len(lk)
            nblk = -(-L // bs)
            ck = np.zeros((nblk, hkv, bs, d), dtype=np.uint16)
            cv = np.zeros_like(ck)
            ck.reshape(nblk, hkv, bs, d)[:] = 0
            for j in range(L):
                ck[j // bs, :, j % bs] = lk[j]
                cv[j // bs, :, j % bs] = lv[j]
            want = oracle.decode(q[i:i + 1], ck, cv, np.arange(nblk, dtype=np.int32)[None], np.array([L], np.int32),
                                 0.125, dtype)
            assert np.array_equal(got[i:i + 1], want), f"sequence {sid}"


def test_concurrent_calls_keep_the_pool_consistent():
    """Calls on one manager from several host threads are serialised: after a storm of adds, forks,
    appends, prefill chunks and frees the reference counts still equal the tables that name each page."""
    import threading
    bm = pa.BlockManager(16, 4096)
    errors = []

    def worker(base):
        rng = np.random.default_rng(base)
        mine = []
        for i in range(300):
            sid = base * 100000 + i
            r = rng.random()
            try:
                if r < 0.4 or not mine:
                    bm.add_sequence(sid, int(rng.integers(0, 80)))
                    mine.append(sid)
                elif r < 0.6:
                    bm.fork(int(rng.choice(mine)), sid)
                    mine.append(sid)
                elif r < 0.75:
                    bm.append_slot(int(rng.choice(mine)))
                elif r < 0.85:  # a chunk for a few of this thread's sequences
                    pick = [int(x) for x in rng.choice(mine, size=min(3, len(mine)), replace=False)]
                    chunk = [int(x) for x in rng.integers(0, 40, size=len(pick))]
                    # the copies a step needs depend only on pages this thread's own sequences share
                    # (each thread forks only its own), so the prediction holds under contention
                    _, copies = bm.step_needs(pick, chunk)
                    plan = bm.build_prefill_step(pick, chunk, 256)
                    if len(plan.copy_pairs) != copies:
                        errors.append(AssertionError(f"step_needs said {copies} copies, the step made "
                                                     f"{len(plan.copy_pairs)}"))
                else:
                    victim = int(rng.choice(mine))
                    bm.free_sequence(victim)
                    mine.remove(victim)
            except BlockManagerError as e:
                # running out of pages is allowed under contention (that operation changed nothing, and
                # the thread goes on); anything else is not
                if e.code != -21:
                    errors.append(e)
        return mine

    results = {}
    threads = [threading.Thread(target=lambda b=b: results.__setitem__(b, worker(b))) for b in range(1, 7)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors
    refs = np.zeros(4096, dtype=np.int64)
    for mine in results.values():
        for sid in mine:
            t = bm.block_table(sid)
            assert len(t) == -(-bm.num_tokens(sid) // 16)
            np.add.at(refs, t, 1)
    assert [bm.ref_count(b) for b in range(4096)] == refs.tolist()
    assert bm.num_free_device_blocks == int((refs == 0).sum())


def test_prefill_step_reserves_a_chunk_per_sequence():
    """A chunk of new tokens per sequence: slots continue each sequence, pages are taken at page
    boundaries, query_start is the prefix sum, and a sequence with no new tokens keeps its state."""
    bm = pa.BlockManager(16, 64, 0)
    bm.add_sequence(0, 100)   # 7 pages, 4 rows used in the last
    bm.add_sequence(1, 32)    # 2 full pages
    bm.add_sequence(2, 5)
    free0 = bm.num_free_device_blocks
    plan = bm.build_prefill_step([0, 1, 2], [50, 1, 0], 12)
    assert isinstance(plan, pa.PrefillStepPlan)
    assert plan.query_start.tolist() == [0, 50, 51, 51]
    assert plan.context_lens.tolist() == [150, 33, 5]
    assert len(plan.slot_mapping) == 51 and len(plan.copy_pairs) == 0
    assert np.array_equal(plan.slot_mapping[:50], bm.slots(0, 100, 50))
    assert plan.slot_mapping[50] == bm.slots(1, 32, 1)[0]
    assert bm.num_free_device_blocks == free0 - (3 + 1)   # pages 8-10 of sequence 0, page 3 of sequence 1
    for i, sid in enumerate([0, 1, 2]):
        t = bm.block_table(sid)
        assert np.array_equal(plan.block_tables[i, :len(t)], t) and np.all(plan.block_tables[i, len(t):] == -1)


def test_prefill_step_copies_a_shared_partial_page_once():
    """Two sequences share a partly full last page: the first to append gets a private copy, after
    which the second is the page's only owner and appends in place."""
    bm = pa.BlockManager(16, 32, 0)
    bm.add_sequence(0, 37)
    bm.fork(0, 1)
    last = int(bm.block_table(0)[-1])
    assert bm.ref_count(last) == 2
    plan = bm.build_prefill_step([0, 1], [20, 3], 8)
    assert plan.copy_pairs.shape == (1, 2) and plan.copy_pairs[0, 0] == last
    assert int(bm.block_table(0)[2]) == plan.copy_pairs[0, 1]
    assert int(bm.block_table(1)[2]) == last and bm.ref_count(last) == 1
    assert plan.context_lens.tolist() == [57, 40]


def test_prefill_step_is_all_or_nothing():
    bm = pa.BlockManager(16, 6, 0)
    bm.add_sequence(0, 20)
    bm.add_sequence(1, 30)
    before = (bm.num_free_device_blocks, bm.block_table(0).tolist(), bm.block_table(1).tolist(),
              bm.num_tokens(0), bm.num_tokens(1))

    def state():
        return (bm.num_free_device_blocks, bm.block_table(0).tolist(), bm.block_table(1).tolist(),
                bm.num_tokens(0), bm.num_tokens(1))

    with pytest.raises(pa.BlockManagerError) as e:   # 2 + 1 pages needed, 2 free
        bm.build_prefill_step([0, 1], [40, 20], 8)
    assert e.value.code == -21 and state() == before
    with pytest.raises(pa.BlockManagerError) as e:   # the table of sequence 0 would need 3 entries
        bm.build_prefill_step([0, 1], [20, 1], 2)
    assert e.value.code == -25 and state() == before
    for bad in ([0, 0], [0, 99]):
        with pytest.raises(pa.BlockManagerError):
            bm.build_prefill_step(bad, [1, 1], 8)
        assert state() == before
    with pytest.raises(pa.BlockManagerError):
        bm.build_prefill_step([0, 1], [1, -1], 8)
    with pytest.raises(pa.BlockManagerError):
        bm.build_prefill_step([0, 1], [1], 8)
    assert state() == before


def test_manager_plans_through_the_oracle_prefill():
    """Chunked prefill steps planned by the manager (forked sequences, ragged chunks, idle
    sequences), applied with the oracle's copy and write, give the same causal attention as the
    oracle over each sequence's tokens laid out contiguously."""
    rng = np.random.default_rng(5)
    dtype, hkv, hq, d, bs, nb = "bf16", 2, 4, 64, 16, 64
    from oracle_pins import to_bits
    bm = pa.BlockManager(bs, nb, 0)
    kc = np.zeros((nb, hkv, bs, d), dtype=np.uint16)
    vc = np.zeros_like(kc)
    logical = {}
    for sid, n in ((0, 29), (1, 16)):
        bm.add_sequence(sid, n)
        k = to_bits(rng.standard_normal((n, hkv, d)), dtype)
        v = to_bits(rng.standard_normal((n, hkv, d)), dtype)
        kc, vc = oracle.write_kv(k, v, kc, vc, bm.slots(sid, 0, n), bs)
        logical[sid] = (k, v)
    bm.fork(0, 2)
    logical[2] = logical[0]
    ids = [0, 1, 2]
    for step in range(6):
        chunk = [int(x) for x in rng.integers(0, 40, size=len(ids))]
        plan = bm.build_prefill_step(ids, chunk, 16)
        if len(plan.copy_pairs):
            kc, vc = oracle.copy_blocks(kc, vc, kc, vc, plan.copy_pairs)
        total = int(sum(chunk))
        k = to_bits(rng.standard_normal((total, hkv, d)), dtype)
        v = to_bits(rng.standard_normal((total, hkv, d)), dtype)
        kc, vc = oracle.write_kv(k, v, kc, vc, plan.slot_mapping, bs)
        for i, sid in enumerate(ids):
            a, b = plan.query_start[i], plan.query_start[i + 1]
            lk, lv = logical[sid]
            logical[sid] = (np.concatenate([lk, k[a:b]]), np.concatenate([lv, v[a:b]]))
        q = to_bits(rng.standard_normal((total, hq, d)), dtype)
        got = oracle.prefill(q, kc, vc, plan.block_tables, plan.query_start, plan.context_lens, 0.125, dtype)
        for i, sid in enumerate(ids):
            a, b = int(plan.query_start[i]), int(plan.query_start[i + 1])
            if a == b:
                continue
            lk, lv = logical[sid]
            L = len(lk)
            assert L == plan.context_lens[i]
            nblk = -(-L // bs)
            ck = np.zeros((nblk, hkv, bs, d), dtype=np.uint16)
            cv = np.zeros_like(ck)
            for j in range(L):
                ck[j // bs, :, j % bs] = lk[j]
                cv[j // bs, :, j % bs] = lv[j]
            want = oracle.prefill(q[a:b], ck, cv, np.arange(nblk, dtype=np.int32)[None], np.array([0, b - a], np.int32),
                                  np.array([L], np.int32), 0.125, dtype)
            assert np.array_equal(got[a:b], want), f"step {step} sequence {sid}"


def test_step_needs_predicts_every_step_without_changing_anything():
    """step_needs gives the pages and copies that the next step then takes, for prefill chunks and
    decode steps over forked sequences, and leaves the pool as it was."""
    rng = np.random.default_rng(9)
    bm = pa.BlockManager(16, 200, 0)
    bm.add_sequence(0, 37)
    bm.add_sequence(1, 48)
    bm.fork(0, 2)
    bm.fork(2, 3)
    ids = [0, 1, 2, 3]
    for step in range(30):
        decode = step % 3 == 2
        chunk = [1] * len(ids) if decode else [int(x) for x in rng.integers(0, 30, size=len(ids))]
        tables = [bm.block_table(i).tolist() for i in ids]
        free = bm.num_free_device_blocks
        pages, copies = bm.step_needs(ids, chunk)
        assert bm.num_free_device_blocks == free and [bm.block_table(i).tolist() for i in ids] == tables
        plan = bm.build_decode_step(ids, 64) if decode else bm.build_prefill_step(ids, chunk, 64)
        assert free - bm.num_free_device_blocks == pages, f"step {step}"
        assert len(plan.copy_pairs) == copies, f"step {step}"
    with pytest.raises(pa.BlockManagerError):
        bm.step_needs([0, 0], [1, 1])
    with pytest.raises(pa.BlockManagerError):
        bm.step_needs([0, 7], [1, 1])
