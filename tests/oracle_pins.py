"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each ``pin_*`` function takes an optional path to an oracle shared library
(the default build, or a deliberately broken copy in the mutation tests) and
raises ``AssertionError`` when the oracle disagrees with:

* the page-table worked example of "4. vLLM核心机制" section 4.2 (golden fixture);
* a library routine on a special case (torch's fp64 scaled-dot-product
  attention on the contiguous logical rows, scipy's softmax, numpy's fp16 and
  float32 decoders);
* closed forms (one token, zero query, constant V, a hand-worked two-token case);
* invariants the pages fix (any physical placement, any block size, shared
  prefix pages, head grouping, unread slots never matter).
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import scipy.special
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "page_table_example.json")


# ----------------------------------------------------------------- test-side helpers
def to_bits(x, dtype: str) -> np.ndarray:
    """Round float values once to the storage type; return uint16 bit patterns."""
    t = torch.as_tensor(np.asarray(x, dtype=np.float32))
    t = t.to(torch.float16 if dtype == "fp16" else torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def from_bits(bits, dtype: str) -> np.ndarray:
    """Decode storage bits with numpy (independent of the oracle's own decoder)."""
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype == "fp16":
        return bits.view(np.float16).astype(np.float64)
    with np.errstate(invalid="ignore"):  # signalling-NaN patterns widen to NaN, which is the point
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def paged(logical, bs, num_blocks, rng, nan_fill=True, dtype="fp16", shared=None):
    """Place per-sequence logical rows ([L, Hkv, d] uint16) into a random block pool.

    ``shared`` optionally maps a sequence index to (other sequence, n_blocks): its first
    n_blocks table entries reuse the other's physical blocks.
    Returns (cache [NB, Hkv, bs, d], tables [S, MB]).
    """
    hkv, d = logical[0].shape[1], logical[0].shape[2]
    fill = 0x7E00 if dtype == "fp16" else 0x7FC0
    cache = np.full((num_blocks, hkv, bs, d), fill if nan_fill else 0, dtype=np.uint16)
    width = max(1, max(-(-x.shape[0] // bs) for x in logical))
    tables = np.full((len(logical), width), -1, dtype=np.int32)
    free = list(rng.permutation(num_blocks))
    for s, rows in enumerate(logical):
        L = rows.shape[0]
        n = -(-L // bs)
        first = 0
        if shared and s in shared:
            other, nshare = shared[s]
            tables[s, :nshare] = tables[other, :nshare]
            first = nshare
        for i in range(first, n):
            tables[s, i] = free.pop(0)
        for j in range(first * bs, L):
            cache[tables[s, j // bs], :, j % bs, :] = rows[j]
    return cache, tables


def sdpa_reference(q_bits, k_rows, v_rows, scale, dtype):
    """torch fp64 scaled-dot-product attention over contiguous logical rows of one sequence.

    q_bits [Hq, d]; k_rows/v_rows [L, Hkv, d]; heads grouped consecutively.
    """
    hq = q_bits.shape[0]
    hkv = k_rows.shape[1]
    q = torch.from_numpy(from_bits(q_bits, dtype)).reshape(1, hq, 1, -1)
    k = torch.from_numpy(from_bits(k_rows, dtype)).permute(1, 0, 2).unsqueeze(0)
    v = torch.from_numpy(from_bits(v_rows, dtype)).permute(1, 0, 2).unsqueeze(0)
    k = k.repeat_interleave(hq // hkv, dim=1)
    v = v.repeat_interleave(hq // hkv, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=scale)
    return o.reshape(hq, -1).numpy()


def random_case(rng, lens, hq, hkv, d, dtype, boost=None):
    logical_k, logical_v = [], []
    for L in lens:
        k = rng.standard_normal((L, hkv, d))
        if boost is not None and L:
            idx = rng.choice(L, size=max(1, L // 50), replace=False)
            k[idx] *= boost
        logical_k.append(to_bits(k, dtype))
        logical_v.append(to_bits(rng.standard_normal((L, hkv, d)), dtype))
    q = to_bits(rng.standard_normal((len(lens), hq, d)), dtype)
    return q, logical_k, logical_v


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol, f"{what}: max abs diff {err:.3e} > {tol:.1e}"


# ----------------------------------------------------------------- pins
def pin_widen_fp16(lib=None):
    """The oracle's binary16 decoder equals numpy's on every finite pattern (and on inf)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    for b in list(range(0, 65536, 7)) + [0x0001, 0x03FF, 0x0400, 0x3C00, 0x7BFF, 0x7C00, 0x8001, 0xFBFF, 0xFC00]:
        got = oracle.widen(b, "fp16", lib)
        r = ref[b]
        if math.isnan(r):
            assert math.isnan(got), f"fp16 {b:#06x}: expected NaN"
        else:
            assert got == r, f"fp16 {b:#06x}: {got!r} != {r!r}"


def pin_widen_bf16(lib=None):
    """The oracle's bfloat16 decoder equals the float32 with the same upper 16 bits."""
    for b in list(range(0, 65536, 5)) + [0x0001, 0x007F, 0x0080, 0x3F80, 0x7F7F, 0x7F80, 0xFF80]:
        r = float(from_bits(np.array([b], dtype=np.uint16), "bf16")[0])
        got = oracle.widen(b, "bf16", lib)
        if math.isnan(r):
            assert math.isnan(got)
        else:
            assert got == r, f"bf16 {b:#06x}: {got!r} != {r!r}"


def pin_page_table_example(lib=None):
    """Section 4.2's figure: A -> physical 7,2,5; B -> two free pages; q = 0 gives plain means."""
    with open(GOLDEN) as f:
        g = json.load(f)
    bs, nb = g["block_size"], g["num_blocks"]
    u = g["uniform_attention"]
    d = u["head_dim"]
    tables = np.full((2, 3), -1, dtype=np.int32)
    tables[0, :3] = g["request_A"]["logical_to_physical"]
    tables[1, :2] = g["request_B"]["logical_to_physical"]
    lens = np.array([g["request_A"]["context_len"], g["request_B"]["context_len"]], dtype=np.int32)
    kc = np.full((nb, 1, bs, d), 0x7E00, dtype=np.uint16)
    vc = kc.copy()
    slots = np.array(g["expected_slots_A"] + g["expected_slots_B"], dtype=np.int64)
    v_rows = np.array(u["v_rows_A"] + u["v_rows_B"], dtype=np.float64).reshape(-1, 1, d)
    k_rows = np.arange(v_rows.size, dtype=np.float64).reshape(-1, 1, d) / 8.0
    kc, vc = oracle.write_kv(to_bits(k_rows, "fp16"), to_bits(v_rows, "fp16"), kc, vc, slots, bs, lib)
    # the written rows sit exactly where the figure's mapping puts them
    for tok, slot in enumerate(slots):
        assert np.array_equal(vc[slot // bs, 0, slot % bs], to_bits(v_rows[tok, 0], "fp16")), f"slot {slot}"
    used = {int(s) // bs for s in slots}
    assert used == {7, 2, 5, 0, 1}
    for p in set(range(nb)) - used:
        assert np.all(vc[p] == 0x7E00), f"physical page {p} should be untouched"
    q = np.zeros((2, 1, d), dtype=np.uint16)
    out = oracle.decode(q, kc, vc, tables, lens, 1.0, "fp16", lib)
    _close(out[0, 0], u["expected_out_A"], 1e-12, "request A mean")
    _close(out[1, 0], u["expected_out_B"], 1e-12, "request B mean")
    # and with a non-zero query the gathered rows are A's and B's logical rows in order
    rng = np.random.default_rng(0)
    qr = to_bits(rng.standard_normal((2, 1, d)), "fp16")
    out = oracle.decode(qr, kc, vc, tables, lens, 0.7, "fp16", lib)
    kb = to_bits(k_rows, "fp16")
    vb = to_bits(v_rows, "fp16")
    _close(out[0], sdpa_reference(qr[0], kb[:12], vb[:12], 0.7, "fp16"), 1e-12, "A vs sdpa")
    _close(out[1], sdpa_reference(qr[1], kb[12:], vb[12:], 0.7, "fp16"), 1e-12, "B vs sdpa")


def pin_two_token_closed_form(lib=None):
    """Two tokens with scaled logits 1 and 0: weights sigmoid(1), sigmoid(-1)."""
    # q = (1, 0), k0 = (2, 0), k1 = (0, 5), scale 0.5 -> logits 1 and 0.
    # out = s * v0 + (1 - s) * v1 with s = e / (1 + e) = 0.7310585786300049.
    q = to_bits([[[1.0, 0.0]]], "fp16")
    k = to_bits([[[2.0, 0.0]], [[0.0, 5.0]]], "fp16")
    v = to_bits([[[4.0, -2.0]], [[0.0, 6.0]]], "fp16")
    kc = np.zeros((3, 1, 1, 2), dtype=np.uint16)
    vc = kc.copy()
    kc[2, 0, 0], kc[0, 0, 0] = k[0, 0], k[1, 0]
    vc[2, 0, 0], vc[0, 0, 0] = v[0, 0], v[1, 0]
    tables = np.array([[2, 0]], dtype=np.int32)
    out = oracle.decode(q, kc, vc, tables, np.array([2], np.int32), 0.5, "fp16", lib)
    s = 0.7310585786300049
    _close(out[0, 0], [4.0 * s, -2.0 * s + 6.0 * (1 - s)], 1e-14, "two-token closed form")


def pin_single_token(lib=None):
    """L = 1: the only weight is 1, the output is that V row exactly."""
    rng = np.random.default_rng(1)
    for dtype in ("fp16", "bf16"):
        q, lk, lv = random_case(rng, [1, 1, 1], 4, 2, 64, dtype)
        kc, tables = paged(lk, 16, 9, np.random.default_rng(2), dtype=dtype)
        vc, _ = paged(lv, 16, 9, np.random.default_rng(2), dtype=dtype)
        out = oracle.decode(q, kc, vc, tables, np.array([1, 1, 1], np.int32), 0.125, dtype, lib)
        for s in range(3):
            want = from_bits(lv[s][0], dtype).repeat(2, axis=0)
            assert np.array_equal(out[s], want), f"L=1 must return the V row ({dtype})"


def pin_zero_query_mean(lib=None):
    """q = 0: all logits equal, the output is the mean of the V rows."""
    rng = np.random.default_rng(3)
    lens = [5, 16, 33]
    _, lk, lv = random_case(rng, lens, 2, 2, 64, "bf16")
    kc, tables = paged(lk, 16, 8, np.random.default_rng(4), dtype="bf16")
    vc, _ = paged(lv, 16, 8, np.random.default_rng(4), dtype="bf16")
    q = np.zeros((3, 2, 64), dtype=np.uint16)
    out = oracle.decode(q, kc, vc, tables, np.array(lens, np.int32), 0.125, "bf16", lib)
    for s in range(3):
        _close(out[s], from_bits(lv[s], "bf16").mean(axis=0), 1e-12, "zero-query mean")


def pin_constant_v(lib=None):
    """Every V row equal to c gives c whatever the weights (they sum to 1)."""
    rng = np.random.default_rng(5)
    lens = [7, 40]
    q, lk, _ = random_case(rng, lens, 4, 4, 64, "fp16")
    c = to_bits(rng.standard_normal((4, 64)), "fp16")
    lv = [np.broadcast_to(c, (L, 4, 64)).copy() for L in lens]
    kc, tables = paged(lk, 16, 6, np.random.default_rng(6))
    vc, _ = paged(lv, 16, 6, np.random.default_rng(6))
    out = oracle.decode(q, kc, vc, tables, np.array(lens, np.int32), 0.3, "fp16", lib)
    for s in range(2):
        _close(out[s], from_bits(c, "fp16"), 1e-12, "constant V")


def pin_one_hot_v_softmax(lib=None):
    """V row j = e_j: the output is the weight vector, equal to scipy's softmax of the logits."""
    rng = np.random.default_rng(7)
    L, d = 50, 64
    kf = rng.standard_normal((L, 1, d))
    k = to_bits(kf, "fp16")
    v = np.zeros((L, 1, d))
    v[np.arange(L), 0, np.arange(L)] = 1.0
    v = to_bits(v, "fp16")
    q = to_bits(rng.standard_normal((1, 1, d)), "fp16")
    kc, tables = paged([k], 16, 7, np.random.default_rng(8))
    vc, _ = paged([v], 16, 7, np.random.default_rng(8))
    scale = 1.0 / 8.0
    out = oracle.decode(q, kc, vc, tables, np.array([L], np.int32), scale, "fp16", lib)[0, 0]
    logits = scale * (from_bits(k[:, 0], "fp16") @ from_bits(q[0, 0], "fp16"))
    _close(out[:L], scipy.special.softmax(logits), 1e-14, "one-hot V vs scipy softmax")
    assert abs(out[:L].sum() - 1.0) < 1e-12
    assert np.all(out[L:] == 0.0)


def pin_matches_library_attention(lib=None):
    """Random cases against torch fp64 SDPA on the contiguous logical rows."""
    rng = np.random.default_rng(9)
    cases = [  # lens, hq, hkv, d, bs, dtype
        ([1, 2, 15, 16, 17, 100], 4, 4, 64, 16, "fp16"),
        ([31, 32, 33, 129], 8, 2, 128, 32, "bf16"),
        ([3, 70], 6, 3, 64, 16, "bf16"),
    ]
    for lens, hq, hkv, d, bs, dtype in cases:
        q, lk, lv = random_case(rng, lens, hq, hkv, d, dtype)
        nb = sum(-(-L // bs) for L in lens) + 5
        kc, tables = paged(lk, bs, nb, np.random.default_rng(10), dtype=dtype)
        vc, _ = paged(lv, bs, nb, np.random.default_rng(10), dtype=dtype)
        scale = 1.0 / math.sqrt(d)
        out = oracle.decode(q, kc, vc, tables, np.array(lens, np.int32), scale, dtype, lib)
        for s in range(len(lens)):
            _close(out[s], sdpa_reference(q[s], lk[s], lv[s], scale, dtype), 1e-12, f"sdpa L={lens[s]}")


def pin_large_logits(lib=None):
    """Keys scaled by 8 (logits of tens): the output stays finite and equals SDPA."""
    rng = np.random.default_rng(11)
    lens = [300, 517]
    q, lk, lv = random_case(rng, lens, 2, 2, 128, "bf16", boost=8.0)
    kc, tables = paged(lk, 32, 30, np.random.default_rng(12), dtype="bf16")
    vc, _ = paged(lv, 32, 30, np.random.default_rng(12), dtype="bf16")
    out = oracle.decode(q, kc, vc, tables, np.array(lens, np.int32), 1.0, "bf16", lib)
    assert np.all(np.isfinite(out))
    for s in range(2):
        _close(out[s], sdpa_reference(q[s], lk[s], lv[s], 1.0, "bf16"), 1e-11, "large logits vs sdpa")


def pin_huge_logits_no_overflow(lib=None):
    """Logits in the thousands (far past exp's range) still give SDPA's finite answer."""
    rng = np.random.default_rng(29)
    lens = [40, 70]
    q, lk, lv = random_case(rng, lens, 2, 1, 64, "fp16")
    kc, tables = paged(lk, 16, 8, np.random.default_rng(30))
    vc, _ = paged(lv, 16, 8, np.random.default_rng(30))
    scale = 400.0  # |logit| up to several thousand
    out = oracle.decode(q, kc, vc, tables, np.array(lens, np.int32), scale, "fp16", lib)
    assert np.all(np.isfinite(out))
    for s in range(2):
        _close(out[s], sdpa_reference(q[s], lk[s], lv[s], scale, "fp16"), 1e-9, "huge logits vs sdpa")


def pin_placement_invariance(lib=None):
    """Moving blocks to other physical ids (and rewriting the tables) changes nothing."""
    rng = np.random.default_rng(13)
    lens = [20, 45, 64]
    q, lk, lv = random_case(rng, lens, 4, 2, 64, "fp16")
    nb = 16
    kc, tables = paged(lk, 16, nb, np.random.default_rng(14))
    vc, _ = paged(lv, 16, nb, np.random.default_rng(14))
    base = oracle.decode(q, kc, vc, tables, np.array(lens, np.int32), 0.125, "fp16", lib)
    perm = np.random.default_rng(15).permutation(nb)  # physical p moves to perm[p]
    kc2 = np.empty_like(kc)
    vc2 = np.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    t2 = np.where(tables >= 0, perm[np.clip(tables, 0, None)], -1).astype(np.int32)
    moved = oracle.decode(q, kc2, vc2, t2, np.array(lens, np.int32), 0.125, "fp16", lib)
    assert np.array_equal(base, moved), "placement must not change the result"


def pin_block_size_independence(lib=None):
    """The same logical rows stored with block_size 16 and 32 give the same output."""
    rng = np.random.default_rng(16)
    lens = [1, 33, 96]
    q, lk, lv = random_case(rng, lens, 2, 2, 64, "bf16")
    outs = []
    for bs in (16, 32, 5):
        nb = sum(-(-L // bs) for L in lens) + 2
        kc, tables = paged(lk, bs, nb, np.random.default_rng(17), dtype="bf16")
        vc, _ = paged(lv, bs, nb, np.random.default_rng(17), dtype="bf16")
        outs.append(oracle.decode(q, kc, vc, tables, np.array(lens, np.int32), 0.125, "bf16", lib))
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])


def pin_shared_prefix(lib=None):
    """Tables that name the same prefix blocks equal tables with private copies."""
    rng = np.random.default_rng(18)
    hkv, d, bs = 2, 64, 16
    prefix_k = to_bits(rng.standard_normal((48, hkv, d)), "fp16")
    prefix_v = to_bits(rng.standard_normal((48, hkv, d)), "fp16")
    lk, lv, lens = [], [], []
    for L in (48, 50, 61, 80):
        sk = to_bits(rng.standard_normal((L - 48, hkv, d)), "fp16")
        sv = to_bits(rng.standard_normal((L - 48, hkv, d)), "fp16")
        lk.append(np.concatenate([prefix_k, sk]))
        lv.append(np.concatenate([prefix_v, sv]))
        lens.append(L)
    q = to_bits(rng.standard_normal((4, 4, d)), "fp16")
    share = {1: (0, 3), 2: (0, 3), 3: (0, 3)}
    kc, t_shared = paged(lk, bs, 24, np.random.default_rng(19), shared=share)
    vc, _ = paged(lv, bs, 24, np.random.default_rng(19), shared=share)
    assert len(set(t_shared[:, :3].ravel().tolist())) == 3, "prefix blocks must be shared"
    kp, t_priv = paged(lk, bs, 24, np.random.default_rng(20))
    vp, _ = paged(lv, bs, 24, np.random.default_rng(20))
    a = oracle.decode(q, kc, vc, t_shared, np.array(lens, np.int32), 0.125, "fp16", lib)
    b = oracle.decode(q, kp, vp, t_priv, np.array(lens, np.int32), 0.125, "fp16", lib)
    assert np.array_equal(a, b)


def pin_gqa_is_repeated_mha(lib=None):
    """Grouped heads equal ordinary multi-head attention with each KV head repeated."""
    rng = np.random.default_rng(21)
    lens = [9, 40]
    q, lk, lv = random_case(rng, lens, 8, 2, 64, "bf16")
    kc, tables = paged(lk, 16, 6, np.random.default_rng(22), dtype="bf16")
    vc, _ = paged(lv, 16, 6, np.random.default_rng(22), dtype="bf16")
    a = oracle.decode(q, kc, vc, tables, np.array(lens, np.int32), 0.125, "bf16", lib)
    rk = [x.repeat(4, axis=1) for x in lk]
    rv = [x.repeat(4, axis=1) for x in lv]
    kc2, t2 = paged(rk, 16, 6, np.random.default_rng(22), dtype="bf16")
    vc2, _ = paged(rv, 16, 6, np.random.default_rng(22), dtype="bf16")
    b = oracle.decode(q, kc2, vc2, t2, np.array(lens, np.int32), 0.125, "bf16", lib)
    assert np.array_equal(a, b)


def pin_unread_slots_ignored(lib=None):
    """NaN in every slot and table entry past a sequence's end leaves the result unchanged."""
    rng = np.random.default_rng(23)
    lens = [17, 30]
    q, lk, lv = random_case(rng, lens, 2, 2, 64, "fp16")
    kz, tables = paged(lk, 16, 8, np.random.default_rng(24), nan_fill=False)
    vz, _ = paged(lv, 16, 8, np.random.default_rng(24), nan_fill=False)
    kn, _ = paged(lk, 16, 8, np.random.default_rng(24), nan_fill=True)
    vn, _ = paged(lv, 16, 8, np.random.default_rng(24), nan_fill=True)
    wide = np.full((2, 6), 1 << 30, dtype=np.int32)  # garbage past the used entries
    wide[:, :tables.shape[1]] = np.where(tables >= 0, tables, 1 << 30)
    a = oracle.decode(q, kz, vz, tables, np.array(lens, np.int32), 0.125, "fp16", lib)
    b = oracle.decode(q, kn, vn, wide, np.array(lens, np.int32), 0.125, "fp16", lib)
    assert np.all(np.isfinite(b)) and np.array_equal(a, b)


def pin_write_kv_scatter(lib=None):
    """Each written row lands at (slot / bs, slot % bs); negative slots write nothing;
    every other byte of the pool is untouched."""
    rng = np.random.default_rng(25)
    nb, hkv, bs, d, T = 10, 3, 16, 64, 40
    kc = rng.integers(0, 65536, size=(nb, hkv, bs, d), dtype=np.uint16)
    vc = rng.integers(0, 65536, size=(nb, hkv, bs, d), dtype=np.uint16)
    k = rng.integers(0, 65536, size=(T, hkv, d), dtype=np.uint16)
    v = rng.integers(0, 65536, size=(T, hkv, d), dtype=np.uint16)
    slots = rng.permutation(nb * bs)[:T].astype(np.int64)
    slots[::7] = -1
    k2, v2 = oracle.write_kv(k, v, kc, vc, slots, bs, lib)
    touched = np.zeros((nb, bs), dtype=bool)
    for t, s in enumerate(slots):
        if s < 0:
            continue
        blk, row = divmod(int(s), bs)
        touched[blk, row] = True
        assert np.array_equal(k2[blk, :, row], k[t]) and np.array_equal(v2[blk, :, row], v[t])
    keep = ~touched
    assert np.array_equal(k2.transpose(0, 2, 1, 3)[keep], kc.transpose(0, 2, 1, 3)[keep])
    assert np.array_equal(v2.transpose(0, 2, 1, 3)[keep], vc.transpose(0, 2, 1, 3)[keep])


def pin_write_then_decode_single(lib=None):
    """A step that writes token 0 of fresh sequences and attends over L = 1 returns the new V."""
    rng = np.random.default_rng(26)
    nb, hkv, bs, d = 4, 2, 16, 128
    kc = np.full((nb, hkv, bs, d), 0x7FC0, dtype=np.uint16)
    vc = kc.copy()
    k = to_bits(rng.standard_normal((2, hkv, d)), "bf16")
    v = to_bits(rng.standard_normal((2, hkv, d)), "bf16")
    tables = np.array([[3], [1]], dtype=np.int32)
    kc, vc = oracle.write_kv(k, v, kc, vc, np.array([48, 16], np.int64), bs, lib)
    q = to_bits(rng.standard_normal((2, 4, d)), "bf16")
    out = oracle.decode(q, kc, vc, tables, np.array([1, 1], np.int32), 0.1, "bf16", lib)
    for s in range(2):
        assert np.array_equal(out[s], from_bits(v[s], "bf16").repeat(2, axis=0))


def pin_zero_length(lib=None):
    """A sequence of length 0 yields zeros and does not disturb its neighbours."""
    rng = np.random.default_rng(27)
    q, lk, lv = random_case(rng, [0, 12], 2, 2, 64, "fp16")
    kc, tables = paged(lk, 16, 3, np.random.default_rng(28))
    vc, _ = paged(lv, 16, 3, np.random.default_rng(28))
    out = oracle.decode(q, kc, vc, tables, np.array([0, 12], np.int32), 0.125, "fp16", lib)
    assert np.all(out[0] == 0.0)
    _close(out[1], sdpa_reference(q[1], lk[1], lv[1], 0.125, "fp16"), 1e-12, "neighbour of L=0")


def pin_copy_blocks_is_fancy_indexing(lib=None):
    """Block copies equal numpy's fancy-index assignment (pairs with distinct destinations, none of
    which is another pair's source); untouched blocks and skipped pairs change nothing."""
    rng = np.random.default_rng(31)
    nb, hkv, bs, d = 12, 3, 16, 64
    k = rng.integers(0, 65536, size=(nb, hkv, bs, d), dtype=np.uint16)
    v = rng.integers(0, 65536, size=(nb, hkv, bs, d), dtype=np.uint16)
    pairs = np.array([[1, 7], [4, 2], [-1, 3], [9, 11], [5, -1]], dtype=np.int64)
    k2, v2 = oracle.copy_blocks(k, v, k, v, pairs, lib)
    want_k, want_v = k.copy(), v.copy()
    live = pairs[(pairs >= 0).all(axis=1)]
    want_k[live[:, 1]] = k[live[:, 0]]
    want_v[live[:, 1]] = v[live[:, 0]]
    assert np.array_equal(k2, want_k) and np.array_equal(v2, want_v)


def pin_swap_round_trip(lib=None):
    """Swapping blocks out to a second pool and back restores them bit for bit."""
    rng = np.random.default_rng(32)
    dev_k = rng.integers(0, 65536, size=(10, 2, 32, 128), dtype=np.uint16)
    dev_v = rng.integers(0, 65536, size=(10, 2, 32, 128), dtype=np.uint16)
    host_k = np.zeros((6, 2, 32, 128), dtype=np.uint16)
    host_v = host_k.copy()
    out_pairs = np.array([[3, 0], [8, 5], [0, 2]], dtype=np.int64)
    host_k, host_v = oracle.copy_blocks(dev_k, dev_v, host_k, host_v, out_pairs, lib)
    for s_, d_ in out_pairs:
        assert np.array_equal(host_k[d_], dev_k[s_]) and np.array_equal(host_v[d_], dev_v[s_])
    wiped_k, wiped_v = dev_k.copy(), dev_v.copy()
    wiped_k[[3, 8, 0]] = 0
    wiped_v[[3, 8, 0]] = 0
    back_k, back_v = oracle.copy_blocks(host_k, host_v, wiped_k, wiped_v, out_pairs[:, ::-1].copy(), lib)
    assert np.array_equal(back_k, dev_k) and np.array_equal(back_v, dev_v)


def pin_copy_on_write_decode(lib=None):
    """A sequence that reads a private copy of a shared block decodes exactly as through the shared one."""
    rng = np.random.default_rng(33)
    q, lk, lv = random_case(rng, [40], 4, 2, 64, "fp16")
    kc, tables = paged(lk, 16, 8, np.random.default_rng(34))
    vc, _ = paged(lv, 16, 8, np.random.default_rng(34))
    used = set(tables[0, :3].tolist())
    spare = next(b for b in range(8) if b not in used)
    kc2, vc2 = oracle.copy_blocks(kc, vc, kc, vc, np.array([[tables[0, 2], spare]], np.int64), lib)
    t2 = tables.copy()
    t2[0, 2] = spare
    a = oracle.decode(q, kc, vc, tables, np.array([40], np.int32), 0.125, "fp16", lib)
    b = oracle.decode(q, kc2, vc2, t2, np.array([40], np.int32), 0.125, "fp16", lib)
    assert np.array_equal(a, b)


def causal_reference(q_bits, k_rows, v_rows, scale, dtype):
    """torch fp64 SDPA of n new tokens (q_bits [n, Hq, d]) over L contiguous rows ([L, Hkv, d]).

    The new tokens are the last n of the L; token t may see rows 0..L-n+t (an explicit mask:
    the causal diagonal ends at the bottom-right corner).
    """
    n, hq, _ = q_bits.shape
    L, hkv, _ = k_rows.shape
    q = torch.from_numpy(from_bits(q_bits, dtype)).permute(1, 0, 2).unsqueeze(0)
    k = torch.from_numpy(from_bits(k_rows, dtype)).permute(1, 0, 2).unsqueeze(0).repeat_interleave(hq // hkv, 1)
    v = torch.from_numpy(from_bits(v_rows, dtype)).permute(1, 0, 2).unsqueeze(0).repeat_interleave(hq // hkv, 1)
    mask = torch.arange(L)[None, :] <= (L - n + torch.arange(n))[:, None]
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale)
    return o[0].permute(1, 0, 2).numpy()


def prefill_case(rng, shape, hq, hkv, d, bs, dtype, nb_extra=4):
    """shape: [(L, n)] per sequence.  Returns q [N, Hq, d], logical rows, caches, tables, query_start, lens."""
    lens = [L for L, _ in shape]
    logical_k = [to_bits(rng.standard_normal((L, hkv, d)), dtype) for L in lens]
    logical_v = [to_bits(rng.standard_normal((L, hkv, d)), dtype) for L in lens]
    qs = np.concatenate([[0], np.cumsum([n for _, n in shape])]).astype(np.int32)
    q = to_bits(rng.standard_normal((int(qs[-1]), hq, d)), dtype)
    nb = sum(-(-L // bs) for L in lens) + nb_extra
    kc, tables = paged(logical_k, bs, nb, np.random.default_rng(50), dtype=dtype)
    vc, _ = paged(logical_v, bs, nb, np.random.default_rng(50), dtype=dtype)
    return q, logical_k, logical_v, kc, vc, tables, qs, np.array(lens, np.int32)


def pin_prefill_matches_library_causal(lib=None):
    """Prompt and chunked-prompt rows of several sequences against torch fp64 SDPA with the causal mask."""
    rng = np.random.default_rng(41)
    cases = [  # [(L, n)], hq, hkv, d, bs, dtype
        ([(1, 1), (16, 16), (17, 17), (40, 8), (100, 1), (70, 33)], 8, 2, 64, 16, "fp16"),
        ([(33, 33), (64, 20), (5, 2)], 4, 4, 128, 32, "bf16"),
    ]
    for shape, hq, hkv, d, bs, dtype in cases:
        q, lk, lv, kc, vc, tables, qs, lens = prefill_case(rng, shape, hq, hkv, d, bs, dtype)
        scale = 1.0 / math.sqrt(d)
        out = oracle.prefill(q, kc, vc, tables, qs, lens, scale, dtype, lib)
        for s in range(len(shape)):
            rows = slice(qs[s], qs[s + 1])
            _close(out[rows], causal_reference(q[rows], lk[s], lv[s], scale, dtype), 1e-12,
                   f"prefill (L, n) = {shape[s]}")


def pin_prefill_first_token_is_v0(lib=None):
    """A whole prompt: the token at position 0 sees only itself, so its output is V[0] exactly."""
    rng = np.random.default_rng(42)
    q, lk, lv, kc, vc, tables, qs, lens = prefill_case(rng, [(23, 23), (9, 9)], 6, 3, 64, 16, "fp16")
    out = oracle.prefill(q, kc, vc, tables, qs, lens, 0.3, "fp16", lib)
    for s in range(2):
        want = from_bits(lv[s][0], "fp16").repeat(2, axis=0)  # 2 query heads per kv head
        assert np.array_equal(out[qs[s]], want)


def pin_prefill_chunked_equals_whole(lib=None):
    """A prompt processed in two chunks (the second one over the cached first) equals one pass."""
    rng = np.random.default_rng(43)
    q, lk, lv, kc, vc, tables, qs, lens = prefill_case(rng, [(50, 50)], 4, 2, 64, 16, "bf16")
    whole = oracle.prefill(q, kc, vc, tables, qs, lens, 0.125, "bf16", lib)
    first = oracle.prefill(q[:30], kc, vc, tables, np.array([0, 30], np.int32), np.array([30], np.int32), 0.125,
                           "bf16", lib)
    second = oracle.prefill(q[30:], kc, vc, tables, np.array([0, 20], np.int32), np.array([50], np.int32), 0.125,
                            "bf16", lib)
    assert np.array_equal(np.concatenate([first, second]), whole)


def pin_prefill_is_causal(lib=None):
    """Rewriting the K/V rows after position p leaves the outputs of positions <= p unchanged."""
    rng = np.random.default_rng(44)
    q, lk, lv, kc, vc, tables, qs, lens = prefill_case(rng, [(48, 48)], 2, 2, 64, 16, "fp16")
    a = oracle.prefill(q, kc, vc, tables, qs, lens, 0.125, "fp16", lib)
    p = 29
    lk2, lv2 = lk[0].copy(), lv[0].copy()
    lk2[p + 1:] = to_bits(rng.standard_normal(lk2[p + 1:].shape), "fp16")
    lv2[p + 1:] = to_bits(rng.standard_normal(lv2[p + 1:].shape), "fp16")
    kc2, _ = paged([lk2], 16, tables.size + 4, np.random.default_rng(50))
    vc2, _ = paged([lv2], 16, tables.size + 4, np.random.default_rng(50))
    b = oracle.prefill(q, kc2, vc2, tables, qs, lens, 0.125, "fp16", lib)
    assert np.array_equal(a[:p + 1], b[:p + 1])
    assert not np.array_equal(a[p + 1:], b[p + 1:])


def pin_prefill_one_new_token_is_decode(lib=None):
    """One new token per sequence is the decode step: equal to the decode function bit for bit."""
    rng = np.random.default_rng(45)
    shape = [(1, 1), (37, 1), (64, 1), (65, 1)]
    q, lk, lv, kc, vc, tables, qs, lens = prefill_case(rng, shape, 8, 2, 128, 32, "fp16")
    a = oracle.prefill(q, kc, vc, tables, qs, lens, 0.1, "fp16", lib)
    b = oracle.decode(q, kc, vc, tables, lens, 0.1, "fp16", lib)
    assert np.array_equal(a, b)


ALL_PINS = [
    pin_widen_fp16,
    pin_widen_bf16,
    pin_page_table_example,
    pin_two_token_closed_form,
    pin_single_token,
    pin_zero_query_mean,
    pin_constant_v,
    pin_one_hot_v_softmax,
    pin_matches_library_attention,
    pin_large_logits,
    pin_huge_logits_no_overflow,
    pin_placement_invariance,
    pin_block_size_independence,
    pin_shared_prefix,
    pin_gqa_is_repeated_mha,
    pin_unread_slots_ignored,
    pin_write_kv_scatter,
    pin_write_then_decode_single,
    pin_zero_length,
    pin_copy_blocks_is_fancy_indexing,
    pin_swap_round_trip,
    pin_copy_on_write_decode,
    pin_prefill_matches_library_causal,
    pin_prefill_first_token_is_v0,
    pin_prefill_chunked_equals_whole,
    pin_prefill_is_causal,
    pin_prefill_one_new_token_is_decode,
]
