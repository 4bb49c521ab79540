"""Cascade decode on the GPU against the fp64 oracle (needs a B200).  The cascade path computes the same
attention as pa_decode ("4. vLLM核心机制", section 4.2, with shared prefix blocks named by several tables),
so the oracle is the plain decode definition applied through the very tables the kernels read."""
import gc

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from gpu_util import DeviceState, compare, host_bits, oracle_step, require_gpu, to_dev, to_dev_index

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    yield
    gc.collect()
    torch.cuda.empty_cache()


def run_cascade(dev, st, tables=None, lens=None, groups=None, chunk=0, max_context_len=None, q=None):
    import paged_kv_cache_457_b200 as pa
    wl = dev.wl
    tables = st.block_tables if tables is None else tables
    lens = st.context_lens if lens is None else lens
    mcl = int(st.max_context_len if max_context_len is None else max_context_len)
    if groups is None:
        groups = pa.find_prefix_groups(tables, lens, wl.block_size)
    plan = pa.cascade_plan(len(lens), wl.num_q_heads, wl.num_kv_heads, wl.block_size, mcl, groups,
                           chunk_tokens=chunk)
    out = pa.decode_cascade(to_dev(st.q if q is None else q, wl.dtype), dev.k_cache, dev.v_cache,
                            to_dev_index(tables), to_dev_index(lens), wl.scale, plan, plan.to("cuda"))
    return host_bits(out), groups


def test_cascade_shared_prefix_steps():
    """The 16 continuous-batching steps of the shared-prefix workload (8 groups x 8 sequences, 1024 shared
    tokens; group 0 retires and a new group joins after step 8): groups found from the host tables, every
    step's output against the oracle (in full on steps 0, 8 and 15, eight sampled sequences otherwise)."""
    import paged_kv_cache_457_b200 as pa
    wl = W.shared_prefix()
    dev = DeviceState(wl)
    kc, vc = wl.k_cache, wl.v_cache
    rng = np.random.default_rng(1)
    for i, st in enumerate(wl.steps):
        dev.write(st)
        out, g = run_cascade(dev, st)
        assert g.num_groups == 8 and list(np.diff(g.offsets)) == [8] * 8 and list(g.prefix_blocks) == [64] * 8
        seqs = None if i in (0, 8, 15) else np.sort(rng.choice(st.num_seqs, 8, replace=False))
        kc, vc, ref = oracle_step(wl, kc, vc, st, seqs)
        compare(out if seqs is None else out[seqs], ref, wl.dtype, what=f"cascade step {i}")
    assert pa.device_status() == 0


def grouped_case(hq, hkv, d, bs, dtype, seed):
    """A batch with planted groups: 20 members sharing 40 blocks' worth of tokens (more members than one
    block's columns hold), a pair sharing one block, a trio whose shortest member ends one token past the
    prefix, singletons, an empty sequence and one-token sequences.  Returns (workload, step, tables,
    expected groups as (members, blocks))."""
    tok = 640
    lens, groups = [], []

    def add_group(ls, shared_tokens):
        first = len(lens)
        lens.extend(ls)
        groups.append((list(range(first, first + len(ls))), shared_tokens))

    r = np.random.default_rng(seed)
    add_group([tok + int(x) for x in r.integers(1, 300, size=20)], tok)
    add_group([33, 900], 16)
    add_group([321, 257, 600], 256)
    lens += [0, 1, 17, 513, 1]
    wl = W.custom(seed=seed, num_seqs=len(lens), num_q_heads=hq, num_kv_heads=hkv, head_dim=d, block_size=bs,
                  lens=lens, dtype=dtype)
    st = wl.steps[0]
    tables = st.block_tables.copy()
    expect = []
    for mem, shared in groups:
        # name the first member's leading blocks in the others' tables; every member's newly written token
        # stays in a block of its own
        nb = min(shared // bs, min((lens[m] - 1) // bs for m in mem))
        for m in mem[1:]:
            tables[m, :nb] = tables[mem[0], :nb]
        if nb >= 1:
            expect.append((mem, nb))
    return wl, st, tables, expect


SHAPES = [  # (hq, hkv, d, bs, dtype): 4, 8, 1, 2 and 3 heads per kv head
    (32, 8, 128, 16, "bf16"),
    (16, 2, 64, 32, "fp16"),
    (8, 8, 128, 32, "fp16"),
    (8, 4, 64, 16, "bf16"),
    (6, 2, 128, 16, "fp16"),
]


@pytest.mark.parametrize("hq,hkv,d,bs,dtype", SHAPES)
@pytest.mark.parametrize("chunk", [0, 16, 48])
def test_cascade_planted_groups(hq, hkv, d, bs, dtype, chunk):
    """Planted groups are found exactly, and every output element is within tolerance of the oracle for
    the default chunks and for chunks of 1 and 3 tiles (prefix and suffix cut at every offset; more than
    32 pieces per sequence with 1-tile chunks)."""
    import paged_kv_cache_457_b200 as pa
    wl, st, tables, expect = grouped_case(hq, hkv, d, bs, dtype, seed=900 + hq + d + bs)
    dev = DeviceState(wl)
    dev.write(st)
    out, g = run_cascade(dev, st, tables=tables, chunk=chunk)
    got = [(list(g.members[g.offsets[i]:g.offsets[i + 1]]), int(g.prefix_blocks[i])) for i in range(g.num_groups)]
    assert got == expect
    assert pa.device_status() == 0
    kc, vc = oracle.write_kv(st.k_new, st.v_new, wl.k_cache, wl.v_cache, st.slot_mapping, wl.block_size)
    ref = oracle.decode(st.q, kc, vc, tables, st.context_lens, wl.scale, wl.dtype)
    compare(out, ref, dtype, what=f"cascade {hq}/{hkv} d{d} bs{bs} {dtype} chunk {chunk}")
    assert not np.any(out[st.context_lens == 0])


def test_cascade_matches_decode_without_groups():
    """With no groups every sequence is its own suffix job; the result agrees with the oracle as pa_decode's."""
    wl, st, tables, _ = grouped_case(32, 8, 128, 16, "bf16", seed=5)
    dev = DeviceState(wl)
    dev.write(st)
    import paged_kv_cache_457_b200 as pa
    empty = pa.PrefixGroups(np.zeros(1, np.int32), np.zeros(0, np.int32), np.zeros(0, np.int32))
    out, _ = run_cascade(dev, st, tables=tables, groups=empty)
    kc, vc = oracle.write_kv(st.k_new, st.v_new, wl.k_cache, wl.v_cache, st.slot_mapping, wl.block_size)
    ref = oracle.decode(st.q, kc, vc, tables, st.context_lens, wl.scale, wl.dtype)
    compare(out, ref, "bf16", what="cascade, no groups")
    compare(dev.decode(st, tables=tables), ref, "bf16", what="pa_decode, same tables")


def test_cascade_deterministic_and_graph_replay():
    """Two calls give identical bits, and a CUDA graph of the call replays to the same bits."""
    import paged_kv_cache_457_b200 as pa
    wl, st, tables, _ = grouped_case(32, 8, 128, 16, "bf16", seed=8)
    dev = DeviceState(wl)
    dev.write(st)
    g = pa.find_prefix_groups(tables, st.context_lens, wl.block_size)
    plan = pa.cascade_plan(st.num_seqs, 32, 8, 16, st.max_context_len, g)
    args = (to_dev(st.q, "bf16"), dev.k_cache, dev.v_cache, to_dev_index(tables), to_dev_index(st.context_lens),
            wl.scale, plan, plan.to("cuda"))
    out = torch.empty_like(args[0])
    ws = torch.empty(pa.cascade_workspace_size(plan, 128), dtype=torch.uint8, device="cuda")
    pa.decode_cascade(*args, out=out, workspace=ws)
    a = host_bits(out)
    pa.decode_cascade(*args, out=out, workspace=ws)
    assert np.array_equal(a, host_bits(out))
    out.zero_()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            pa.decode_cascade(*args, out=out, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    graph.replay()
    torch.cuda.synchronize()
    assert np.array_equal(a, host_bits(out))
    assert pa.device_status() == 0


def test_cascade_device_checks():
    """A plan that no longer fits the tables: a member whose table differs on one shared block, and a member
    whose context ends inside the prefix, get zero rows and PA_DEV_ERR_PLAN; a table entry outside the pool
    in a sequence's own part gives it a zero row and PA_DEV_ERR_BLOCK_ID; a context above max_context_len
    a zero row and PA_DEV_ERR_CONTEXT_HINT.  Every other sequence stays exact."""
    import paged_kv_cache_457_b200 as pa
    wl, st, tables, expect = grouped_case(32, 8, 128, 16, "bf16", seed=11)
    dev = DeviceState(wl)
    dev.write(st)
    g = pa.find_prefix_groups(tables, st.context_lens, wl.block_size)
    kc, vc = oracle.write_kv(st.k_new, st.v_new, wl.k_cache, wl.v_cache, st.slot_mapping, wl.block_size)
    S = st.num_seqs

    def check(bad_seqs, bit, tables_used, lens_used, mcl=None):
        out, _ = run_cascade(dev, st, tables=tables_used, lens=lens_used, groups=g, max_context_len=mcl)
        assert pa.device_status() == bit
        for s in bad_seqs:
            assert not np.any(out[s]), f"sequence {s} not zeroed"
        good = [s for s in range(S) if s not in bad_seqs]
        ref = oracle.decode(st.q[good], kc, vc, tables_used[good], lens_used[good], wl.scale, wl.dtype)
        compare(out[good], ref, "bf16", what=f"the other sequences (bit {bit})")

    t = tables.copy()
    t[5, 3] = t[5, 3] + 1 if t[5, 3] + 1 < wl.num_blocks else t[5, 3] - 1  # member 5 of group 0: block 3 differs
    check([5], pa.DEV_ERR_PLAN, t, st.context_lens)
    lens = st.context_lens.copy()
    lens[7] = 500  # member 7 of group 0 (640 shared tokens) now ends inside the prefix
    check([7], pa.DEV_ERR_PLAN, tables, lens)
    t = tables.copy()
    s_own = expect[1][0][1]  # the pair's second member: its own blocks start after the one shared block
    t[s_own, 1] = wl.num_blocks + 5
    check([s_own], pa.DEV_ERR_BLOCK_ID, t, st.context_lens)
    lens = st.context_lens.copy()
    lens[19] = st.max_context_len + 1  # a member of group 0 (not its first) above the call's bound
    assert lens[19] <= tables.shape[1] * wl.block_size
    check([19], pa.DEV_ERR_CONTEXT_HINT, tables, lens, mcl=st.max_context_len)


def test_cascade_without_jobs_runs_the_combine_alone():
    """A call bounded at max_context_len 0 has no jobs, so the combine kernel runs alone, right behind the
    kernel that wrote the lengths (it waits for that kernel before reading them).  Empty contexts give zero
    rows and no status bit; a context above the bound gives a zero row and PA_DEV_ERR_CONTEXT_HINT."""
    import paged_kv_cache_457_b200 as pa
    wl = W.custom(seed=3, num_seqs=4, num_q_heads=8, num_kv_heads=2, head_dim=64, block_size=16, lens=[5, 1, 9, 3],
                  dtype="fp16")
    st = wl.steps[0]
    dev = DeviceState(wl)
    plan = pa.cascade_plan(4, 8, 2, 16, 0)
    assert plan.info.num_jobs == 0
    q = to_dev(st.q, "fp16")
    tables = to_dev_index(st.block_tables)
    plan_dev = plan.to("cuda")
    lens = torch.full((4,), 7, dtype=torch.int32, device="cuda")
    out = torch.full_like(q, float("nan"))
    pa.device_status()
    lens.zero_()  # the kernel just before the call writes the lengths
    pa.decode_cascade(q, dev.k_cache, dev.v_cache, tables, lens, wl.scale, plan, plan_dev, out=out)
    assert pa.device_status() == 0
    assert not np.any(host_bits(out))
    lens.copy_(torch.tensor([0, 3, 0, 0], dtype=torch.int32))
    out.fill_(float("nan"))
    pa.decode_cascade(q, dev.k_cache, dev.v_cache, tables, lens, wl.scale, plan, plan_dev, out=out)
    assert pa.device_status() == pa.DEV_ERR_CONTEXT_HINT
    assert not np.any(host_bits(out))
