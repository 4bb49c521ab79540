"""Paged causal prefill on the tensor cores against the fp64 oracle.

Cases span one query tile and several, ragged last tiles (1, 5, 127, 128, 129,
300 new tokens), whole prompts and chunks over a cached prefix, MHA and
grouped heads, d 64 and 128, 16- and 32-token pages, both storage types.
Every unowned slot of the pool holds NaN, so a kernel that lets a row past
the context into the sums shows up.
"""
from __future__ import annotations

import zlib

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_457_b200 as pa
import workloads as W
from gpu_util import compare, host_bits, require_gpu, to_dev, to_dev_index

pytestmark = pytest.mark.gpu


def run(case, max_query_len=None, tables=None, lens=None):
    kc, vc = to_dev(case.k_cache, case.dtype), to_dev(case.v_cache, case.dtype)
    out = pa.prefill(to_dev(case.q, case.dtype), kc, vc, to_dev_index(case.block_tables if tables is None else tables),
                     to_dev_index(case.query_start), to_dev_index(case.context_lens if lens is None else lens),
                     case.scale, case.max_query_len if max_query_len is None else max_query_len)
    return host_bits(out)


def expect(case):
    return oracle.prefill(case.q, case.k_cache, case.v_cache, case.block_tables, case.query_start, case.context_lens,
                          case.scale, case.dtype)


SHAPES = {
    "prompts": [(1, 1), (5, 5), (127, 127), (128, 128), (129, 129), (300, 300)],
    "chunks": [(700, 200), (1000, 1), (257, 256), (130, 2), (64, 64), (513, 129)],
}


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("hq,hkv,d,bs", [(4, 4, 128, 16), (8, 2, 128, 32), (4, 1, 64, 16), (6, 3, 64, 32)])
@pytest.mark.parametrize("kind", sorted(SHAPES))
def test_prefill_matches_oracle(dtype, hq, hkv, d, bs, kind):
    require_gpu()
    case = W.prefill_case(zlib.crc32(repr((dtype, hq, hkv, d, bs, kind)).encode()) % 1000, SHAPES[kind], hq, hkv,
                          d, bs, dtype)
    got = run(case)
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    compare(got, expect(case), dtype, what=f"prefill {kind}")


def test_one_new_token_matches_decode_path():
    """n = 1 for every sequence is a decode step: prefill agrees with the oracle and with pa_decode."""
    require_gpu()
    case = W.prefill_case(11, [(37, 1), (64, 1), (200, 1), (1, 1)], 8, 2, 128, 16, "fp16")
    got = run(case)
    ref = expect(case)
    compare(got, ref, "fp16", what="prefill n=1")
    kc, vc = to_dev(case.k_cache, "fp16"), to_dev(case.v_cache, "fp16")
    dec = host_bits(pa.decode(to_dev(case.q, "fp16"), kc, vc, to_dev_index(case.block_tables),
                              to_dev_index(case.context_lens), case.scale, max_context_len=200))
    compare(dec, ref, "fp16", what="decode on the same inputs")


def test_empty_sequences_and_larger_grid():
    """Sequences with no new tokens write nothing; max_query_len above the real maximum is harmless."""
    require_gpu()
    case = W.prefill_case(12, [(40, 0), (90, 33), (16, 0), (17, 17)], 4, 4, 64, 16, "bf16")
    got = run(case, max_query_len=400)
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    compare(got, expect(case), "bf16", what="empty sequences")


def test_bad_page_and_bad_context_zero_their_rows():
    require_gpu()
    case = W.prefill_case(13, [(50, 50), (40, 20), (33, 3)], 4, 2, 64, 16, "fp16")
    tables = case.block_tables.copy()
    tables[0, 1] = case.num_blocks + 5  # outside the pool
    lens = case.context_lens.copy()
    lens[1] = 10  # fewer context tokens than new tokens
    pa.device_status(clear=True)
    got = run(case, tables=tables, lens=lens)
    torch.cuda.synchronize()
    st = pa.device_status()
    assert st & pa.DEV_ERR_BLOCK_ID and st & pa.DEV_ERR_CONTEXT
    qs = case.query_start
    assert not got[qs[0]:qs[2]].any()  # rows of sequences 0 and 1 are zero
    ok = W.PrefillCase(**{**case.__dict__, "q": case.q[qs[2]:], "query_start": (qs[2:] - qs[2]).astype(np.int32),
                          "context_lens": case.context_lens[2:], "block_tables": case.block_tables[2:]})
    compare(got[qs[2]:], expect(ok), "fp16", what="untouched sequence")


def test_max_query_len_too_small_is_flagged():
    require_gpu()
    case = W.prefill_case(17, [(600, 600), (40, 40)], 4, 4, 64, 16, "fp16")
    pa.device_status(clear=True)
    got = run(case, max_query_len=200)  # covers 256 rows: sequence 0's rows 256.. are left unwritten
    torch.cuda.synchronize()
    assert pa.device_status() & pa.DEV_ERR_CONTEXT_HINT
    ref = expect(case)
    compare(got[:256], ref[:256], "fp16", what="rows the grid covers")
    compare(got[600:], ref[600:], "fp16", what="the other sequence")


def test_chunked_equals_whole_prompt():
    """A prompt processed as two chunks (the second over the cached first) gives the one-pass rows."""
    require_gpu()
    whole = W.prefill_case(14, [(400, 400)], 8, 8, 128, 16, "bf16")
    a = run(whole)
    first = W.PrefillCase(**{**whole.__dict__, "q": whole.q[:250], "query_start": np.array([0, 250], np.int32),
                             "context_lens": np.array([250], np.int32)})
    second = W.PrefillCase(**{**whole.__dict__, "q": whole.q[250:], "query_start": np.array([0, 150], np.int32),
                              "context_lens": np.array([400], np.int32)})
    b = np.concatenate([run(first), run(second)])
    compare(a, expect(whole), "bf16", what="one pass")
    compare(b, expect(whole), "bf16", what="two chunks")


@pytest.mark.parametrize("name", sorted(W.PREFILL_NAMED))
def test_full_size_sampled(name):
    """The measured configurations at full size, in the launch the bench times; the two shortest
    sequences checked row by row against the oracle, and the first and last 64 rows of the longest
    one (its lightest and heaviest rows: the last ones attend to the whole context); every row checked
    finite."""
    require_gpu()
    case = W.PREFILL_NAMED[name]()
    got = run(case)
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    assert np.all(np.isfinite(got.view(np.float16) if case.dtype == "fp16" else
                              (got.astype(np.uint32) << 16).view(np.float32)))
    qs, lens = case.query_start, case.context_lens
    order = np.argsort(lens)
    for s in (int(order[0]), int(order[1])):  # the two shortest contexts keep the fp64 oracle to seconds
        sub = W.PrefillCase(**{**case.__dict__, "q": case.q[qs[s]:qs[s + 1]],
                               "query_start": np.array([0, qs[s + 1] - qs[s]], np.int32),
                               "context_lens": lens[s:s + 1], "block_tables": case.block_tables[s:s + 1]})
        compare(got[qs[s]:qs[s + 1]], expect(sub), case.dtype, what=f"{name} sequence {s}")
    s = int(order[-1])
    n, L = int(qs[s + 1] - qs[s]), int(lens[s])
    k = min(64, n)
    # the last k new tokens sit at positions L - k .. L - 1: a sub-case with k new tokens and the same context
    last = W.PrefillCase(**{**case.__dict__, "q": case.q[qs[s + 1] - k:qs[s + 1]],
                            "query_start": np.array([0, k], np.int32), "context_lens": lens[s:s + 1],
                            "block_tables": case.block_tables[s:s + 1]})
    compare(got[qs[s + 1] - k:qs[s + 1]], expect(last), case.dtype, what=f"{name} longest sequence, last rows")
    # the first k new tokens sit at positions L - n .. L - n + k - 1: context L - n + k
    first = W.PrefillCase(**{**case.__dict__, "q": case.q[qs[s]:qs[s] + k],
                             "query_start": np.array([0, k], np.int32),
                             "context_lens": np.array([L - n + k], np.int32),
                             "block_tables": case.block_tables[s:s + 1]})
    compare(got[qs[s]:qs[s] + k], expect(first), case.dtype, what=f"{name} longest sequence, first rows")


def test_skewed_batch_one_long_prompt_among_decode_steps():
    """A chunked-prefill batch: one long prompt and many one-token sequences (exact), and one prompt among
    thousands of sequences with no new token, whose empty (query tile, sequence, head) items cost little."""
    require_gpu()
    shape = [(int(L), 1) for L in np.random.default_rng(15).integers(1, 300, size=120)] + [(2000, 2000)]
    case = W.prefill_case(15, shape, 8, 2, 128, 16, "bf16")
    got = run(case)
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    compare(got[:120], expect(W.PrefillCase(**{**case.__dict__, "q": case.q[:120],
                                                 "query_start": case.query_start[:121],
                                                 "context_lens": case.context_lens[:120],
                                                 "block_tables": case.block_tables[:120]})), "bf16",
            what="one-token sequences")
    last = W.PrefillCase(**{**case.__dict__, "q": case.q[120:], "query_start": np.array([0, 2000], np.int32),
                            "context_lens": case.context_lens[120:], "block_tables": case.block_tables[120:]})
    compare(got[120:], expect(last), "bf16", what="long prompt")
    # empty items are cheap but not free: 4000 cached sequences that bring no new token and one 1000-token
    # prompt, 8 query heads: 4 * 4001 * 8 items, all but 32 of them empty (about 0.7 ms on a B200; the bound
    # catches a schedule that would spend a full item's pipeline on each)
    big_shape = [(int(L), 0) for L in np.random.default_rng(16).integers(1, 64, size=4000)] + [(1000, 1000)]
    big = W.prefill_case(16, big_shape, 8, 2, 128, 16, "bf16")
    kc, vc = to_dev(big.k_cache, "bf16"), to_dev(big.v_cache, "bf16")
    args = (to_dev(big.q, "bf16"), kc, vc, to_dev_index(big.block_tables), to_dev_index(big.query_start),
            to_dev_index(big.context_lens), big.scale, big.max_query_len)
    out = pa.prefill(*args)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(5):
        pa.prefill(*args)
    e1.record()
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    assert e0.elapsed_time(e1) / 5 < 2.0
    got_big = host_bits(out)
    sub = W.PrefillCase(**{**big.__dict__, "query_start": np.array([0, 1000], np.int32),
                           "context_lens": big.context_lens[-1:], "block_tables": big.block_tables[-1:]})
    compare(got_big, expect(sub), "bf16", what="the prompt among empty sequences")
