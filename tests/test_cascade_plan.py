"""Host side of cascade decode (no GPU): the prefix grouping against a brute-force restatement, and the
work plan against the property that makes the attention exact -- every (sequence, tile) below the call's
bound is covered by exactly one of the sequence's pieces, in increasing order, read through a table row
that names the sequence's own blocks ("4. vLLM核心机制", section 4.2: shared prefix blocks are named by
several tables, so the blocks one table names are the blocks the other reads)."""
import numpy as np
import pytest

import paged_kv_cache_457_b200 as pa

CJ = 8  # ints per job: seq, t0, t1, member offset, members, row, kind, split
PREFIX, SUFFIX = 0, 1


def brute_groups(tables, lens, bs, min_blocks=1):
    """Sequences with a full first block grouped by that block; prefix = longest run of leading entries
    all members share, over full blocks only; groups of >= 2 members with prefix >= max(1, min_blocks),
    in order of first member."""
    S = len(lens)
    keys = {}
    for s in range(S):
        if lens[s] // bs >= 1:
            keys.setdefault(int(tables[s, 0]), []).append(s)
    out = []
    for mem in sorted(keys.values(), key=lambda m: m[0]):
        if len(mem) < 2:
            continue
        P = min(int(lens[m]) // bs for m in mem)
        j = 0
        while j < P and all(tables[m, j] == tables[mem[0], j] for m in mem):
            j += 1
        if j >= max(1, min_blocks):
            out.append((mem, j))
    return out


def forked_batch(rng, S, bs, width):
    """Tables with planted sharing: some sequences copy a leading run of an earlier one's entries."""
    tables = rng.permutation(S * width * 2)[:S * width].reshape(S, width).astype(np.int32)
    lens = rng.integers(0, width * bs + 1, size=S).astype(np.int32)
    for s in range(1, S):
        if rng.random() < 0.6:
            src = int(rng.integers(0, s))
            k = int(rng.integers(0, width + 1))
            tables[s, :k] = tables[src, :k]
    return tables, lens


@pytest.mark.parametrize("seed", range(12))
@pytest.mark.parametrize("bs", [16, 32])
def test_find_prefix_groups_matches_brute_force(seed, bs):
    rng = np.random.default_rng(seed)
    S, width = int(rng.integers(1, 40)), int(rng.integers(1, 12))
    tables, lens = forked_batch(rng, S, bs, width)
    for min_blocks in (0, 1, 3):
        g = pa.find_prefix_groups(tables, lens, bs, min_prefix_blocks=min_blocks)
        got = [(list(g.members[g.offsets[i]:g.offsets[i + 1]]), int(g.prefix_blocks[i])) for i in range(g.num_groups)]
        assert got == brute_groups(tables, lens, bs, min_blocks)


def test_find_prefix_groups_cases():
    bs = 16
    t = np.array([[5, 6, 7, 9], [5, 6, 7, 10], [5, 6, 8, 11], [1, 2, 3, 4], [5, 6, 7, 12], [1, 9, 9, 9]], np.int32)
    lens = np.array([64, 60, 50, 64, 33, 15], np.int32)  # sequence 5 has no full block
    g = pa.find_prefix_groups(t, lens, bs)
    assert list(g.offsets) == [0, 4] and list(g.members) == [0, 1, 2, 4] and list(g.prefix_blocks) == [2]
    lens[5] = 16  # now it shares block 1 with sequence 3: a second group, one block
    g = pa.find_prefix_groups(t, lens, bs)
    assert list(g.offsets) == [0, 4, 6] and list(g.members) == [0, 1, 2, 4, 3, 5] and list(g.prefix_blocks) == [2, 1]
    assert pa.find_prefix_groups(t, lens, bs, min_prefix_blocks=2).num_groups == 1
    assert pa.find_prefix_groups(np.zeros((0, 4), np.int32), np.zeros(0, np.int32), bs).num_groups == 0
    with pytest.raises(pa.PagedAttentionError):
        pa.find_prefix_groups(t, np.array([64, 60, 50, 64, 33, 65], np.int32), bs)  # beyond the table row


def pieces_of(plan, S):
    info = plan.info
    p = plan.plan
    J = info.num_jobs
    jobs = p[:J * CJ].reshape(J, CJ)
    members = p[J * CJ:J * CJ + info.num_members]
    offs = p[J * CJ + info.num_members:J * CJ + info.num_members + S + 1]
    rows = p[J * CJ + info.num_members + S + 1:]
    assert rows.shape[0] == info.num_pieces == offs[-1]
    return jobs, members, offs, rows


def check_plan(plan, S, G, bs, mcl, prefix_of, lead_of, chunk):
    """Coverage, order, row uniqueness and job shapes of a plan (prefix_of[s]: shared tiles of s's group,
    lead_of[s]: the sequence whose table the group's prefix jobs read)."""
    jobs, members, offs, rows = pieces_of(plan, S)
    info = plan.info
    max_tiles = -(-mcl // 16)
    kinds = list(jobs[:, 6])
    assert kinds == sorted(kinds) and kinds.count(PREFIX) == info.num_prefix_jobs, "prefix jobs come first"
    row_owner = {}
    for j, (seq, t0, t1, mfirst, nm, row, kind, split) in enumerate(jobs):
        assert kind in (PREFIX, SUFFIX) and 0 <= t0 < t1 and t1 - t0 <= chunk // 16
        if kind == SUFFIX:
            assert nm == 1 and split == 1
        else:
            n_rt = -(-nm // (16 // G))  # row tiles of 16 (member, head) rows
            assert 1 <= nm <= 4 * (16 // G) and split == {1: 4, 2: 2}.get(n_rt, 1) and n_rt * split <= 4
        assert 0 <= mfirst and mfirst + nm <= info.num_members
        assert 0 <= row and row + nm * G * split <= info.rows_per_head
        for sp in range(split):
            for i in range(nm):
                m = int(members[mfirst + i])
                for h in range(G):
                    r = row + (sp * nm + i) * G + h
                    assert r not in row_owner, "partial rows overlap"
                    row_owner[r] = (j, m, sp)
                if kind == SUFFIX:
                    assert m == seq
                else:
                    assert lead_of[m] == seq and t1 <= prefix_of[m]
    assert len(row_owner) == info.rows_per_head
    for s in range(S):
        covered = []
        for r in rows[offs[s]:offs[s + 1]]:
            j, m, sp = row_owner[int(r)]
            assert m == s, "a piece row of another sequence"
            covered += list(range(jobs[j][1] + sp, jobs[j][2], jobs[j][7]))
        assert sorted(covered) == list(range(max(max_tiles, prefix_of[s]))), f"sequence {s}: tiles {covered}"


@pytest.mark.parametrize("hq,hkv", [(32, 8), (8, 8), (16, 8), (24, 8), (8, 1), (6, 2)])
@pytest.mark.parametrize("chunk", [0, 16, 48, 512])
@pytest.mark.parametrize("seed", range(3))
def test_cascade_plan_covers_every_tile_once(hq, hkv, chunk, seed):
    rng = np.random.default_rng(seed * 31 + hq)
    bs = 16 if seed % 2 else 32
    S, width = int(rng.integers(1, 70)), int(rng.integers(2, 20))
    tables, lens = forked_batch(rng, S, bs, width)
    g = pa.find_prefix_groups(tables, lens, bs)
    mcl = int(lens.max(initial=0))
    plan = pa.cascade_plan(S, hq, hkv, bs, mcl, g, chunk_tokens=chunk)
    prefix_of, lead_of = [0] * S, list(range(S))
    for i in range(g.num_groups):
        mem = g.members[g.offsets[i]:g.offsets[i + 1]]
        for m in mem:
            prefix_of[m] = int(g.prefix_blocks[i]) * bs // 16
            lead_of[m] = int(mem[0])
    check_plan(plan, S, hq // hkv, bs, mcl, prefix_of, lead_of, chunk or 320)
    assert plan.info.num_seqs == S and plan.info.max_context_len == mcl


def test_cascade_plan_large_group_splits_columns():
    """A group of 70 members with 4 heads per kv head: jobs of 16 members (4 row tiles of 4 members x 4 heads,
    no split) and one of 6 (2 row tiles, its tiles dealt to 2 warp sets)."""
    S, bs = 70, 16
    g = pa.PrefixGroups(np.array([0, S], np.int32), np.arange(S, dtype=np.int32), np.array([40], np.int32))
    plan = pa.cascade_plan(S, 32, 8, bs, 700, g, chunk_tokens=256)
    jobs, *_ = pieces_of(plan, S)
    pre = jobs[jobs[:, 6] == PREFIX]
    assert sorted(set(pre[:, 4].tolist())) == [6, 16]
    assert sorted(set(zip(pre[:, 4].tolist(), pre[:, 7].tolist()))) == [(6, 2), (16, 1)]
    assert pre.shape[0] == 5 * 3  # 40 blocks = 40 tiles: chunks of 16, 16, 8
    check_plan(plan, S, 4, bs, 700, [40] * S, [0] * S, 256)


def test_cascade_plan_without_groups_is_per_sequence():
    plan = pa.cascade_plan(3, 8, 2, 16, 100, None, chunk_tokens=64)
    jobs, members, offs, rows = pieces_of(plan, 3)
    assert (jobs[:, 6] == SUFFIX).all() and plan.info.num_jobs == 3 * 2  # 7 tiles in chunks of 4
    assert list(offs) == [0, 2, 4, 6]


def test_cascade_plan_rejects_bad_input():
    g = lambda off, mem, pre: pa.PrefixGroups(np.array(off, np.int32), np.array(mem, np.int32), np.array(pre, np.int32))
    ok = g([0, 2], [0, 1], [2])
    pa.cascade_plan(4, 8, 2, 16, 64, ok)
    with pytest.raises(pa.PagedAttentionError):
        pa.cascade_plan(4, 8, 2, 16, 64, g([0, 2, 4], [0, 1, 1, 2], [1, 1]))  # a sequence in two groups
    with pytest.raises(pa.PagedAttentionError):
        pa.cascade_plan(4, 8, 2, 16, 64, g([0, 2], [0, 4], [1]))  # member out of range
    with pytest.raises(pa.PagedAttentionError):
        pa.cascade_plan(4, 8, 2, 16, 16, ok)  # prefix beyond max_context_len
    with pytest.raises(pa.PagedAttentionError):
        pa.cascade_plan(4, 8, 2, 16, 64, g([0, 0], [], [1]))  # empty group
    with pytest.raises(pa.PagedAttentionError):
        pa.cascade_plan(4, 32, 2, 16, 64, ok)  # 16 heads per kv head
    with pytest.raises(pa.PagedAttentionError):
        pa.cascade_plan(4, 8, 2, 16, 64, ok, chunk_tokens=40)
    with pytest.raises(pa.PagedAttentionError):
        pa.cascade_plan(4, 8, 2, 24, 64, ok)


def test_cascade_plan_capacity_and_workspace(lib=None):
    import ctypes
    lib = pa.load_library()
    info = pa.cascade.CascadeInfo()
    off, mem, pre = np.array([0, 2], np.int32), np.array([0, 1], np.int32), np.array([2], np.int32)
    rc = lib.pa_cascade_plan(4, 8, 2, 16, 64, 0, 1, off.ctypes.data, mem.ctypes.data, pre.ctypes.data, None, 0,
                             ctypes.byref(info))
    assert rc == 0 and info.plan_ints > 0
    small = np.zeros(int(info.plan_ints) - 1, np.int32)
    rc = lib.pa_cascade_plan(4, 8, 2, 16, 64, 0, 1, off.ctypes.data, mem.ctypes.data, pre.ctypes.data,
                             small.ctypes.data, small.size, ctypes.byref(info))
    assert rc == -7  # PA_ERR_WORKSPACE
    assert lib.pa_cascade_workspace_size(ctypes.byref(info), 128) >= 2 * info.rows_per_head * (8 + 512)
    assert lib.pa_cascade_workspace_size(ctypes.byref(info), 96) == 0
    assert lib.pa_cascade_workspace_size(None, 128) == 0
