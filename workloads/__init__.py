"""Seeded synthetic inputs for paged decode attention.

This module is shared by the tests, the bench and the smoke check.  It holds
none of the method's arithmetic: it only draws random numbers, rounds them
once to the storage type, allocates physical blocks from a shuffled free list
and lays the drawn rows into the block pool.  Both the CUDA path and the CPU
oracle consume what it produces.

Storage types are carried as uint16 bit patterns so that neither side has to
trust the other's conversions.  Layouts:

* caches   ``[num_blocks, num_kv_heads, block_size, head_dim]``
* q        ``[S, Hq, d]``
* k/v new  ``[T, Hkv, d]``
* tables   int32 ``[S, max_blocks]`` (entries past a sequence's last block hold ``TABLE_PAD``)
* lengths  int32 ``[S]``; ``slot_mapping`` int64 ``[T]``

Semantics: ``context_lens[s]`` counts the token written in the same step, so
a step writes token ``L-1`` of every live sequence and then attends over
``L`` tokens.  Every slot that no sequence owns holds a NaN pattern, so a
kernel that reads past the end of a sequence shows up in the output.

The five named workloads follow the synthetic decode configurations used for
measurement (sizes in their docstrings); ``custom`` builds small cases for the
parity tests.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

NAN_BITS = {"fp16": 0x7E00, "bf16": 0x7FC0}
TABLE_PAD = -1
TILE = 16


@dataclass
class Step:
    """One decode step: write the step's new K/V rows, then attend."""

    q: np.ndarray  # uint16 [S, Hq, d]
    block_tables: np.ndarray  # int32 [S, MB]
    context_lens: np.ndarray  # int32 [S]
    k_new: np.ndarray  # uint16 [T, Hkv, d]
    v_new: np.ndarray  # uint16 [T, Hkv, d]
    slot_mapping: np.ndarray  # int64 [T]

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.context_lens.size else 0


@dataclass
class Workload:
    name: str
    dtype: str  # "fp16" | "bf16"
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    scale: float
    k_cache: np.ndarray  # uint16 [NB, Hkv, bs, d], contents before the first step
    v_cache: np.ndarray
    steps: list = field(default_factory=list)
    description: str = ""

    @property
    def max_context_len(self) -> int:
        return max((s.max_context_len for s in self.steps), default=0)

    @property
    def table_width(self) -> int:
        return max(s.block_tables.shape[1] for s in self.steps)


class _Draw:
    """Seeded generators: numpy PCG64 for structure, torch CPU for bulk normals."""

    def __init__(self, seed: int):
        self.np = np.random.Generator(np.random.PCG64(seed))
        self.torch = torch.Generator().manual_seed(seed)

    def normal_bits(self, shape, dtype: str, scale_rows: np.ndarray | None = None) -> np.ndarray:
        """N(0,1) draws rounded once (RNE) to the storage type, as uint16 bits.

        ``scale_rows`` optionally multiplies leading-axis rows before rounding.
        """
        x = torch.randn(*shape, generator=self.torch, dtype=torch.float32)
        if scale_rows is not None:
            x *= torch.from_numpy(scale_rows.astype(np.float32)).reshape((-1,) + (1,) * (len(shape) - 1))
        tdt = torch.float16 if dtype == "fp16" else torch.bfloat16
        return x.to(tdt).view(torch.int16).numpy().view(np.uint16)


def _nan_pool(num_blocks, hkv, bs, d, dtype):
    return np.full((num_blocks, hkv, bs, d), NAN_BITS[dtype], dtype=np.uint16)


def _place(cache, table_row, first_token, rows, bs):
    """Lay ``rows`` ([n, Hkv, d]) at logical positions first_token.. of one table."""
    n = rows.shape[0]
    if n == 0:
        return
    pos = np.arange(first_token, first_token + n)
    blocks = table_row[pos // bs]
    cache[blocks, :, pos % bs, :] = rows


def _slots(table_row, positions, bs):
    positions = np.asarray(positions, dtype=np.int64)
    return table_row[positions // bs].astype(np.int64) * bs + positions % bs


def _fill_sequences(draw, name, dtype, lens, hq, hkv, d, bs, nb, table_width, free_list,
                    key_boost_frac=0.0, key_boost=1.0, chunk_tokens=8192, description=""):
    """Independent sequences: tokens 0..L-2 in the cache, token L-1 as this step's write."""
    S = len(lens)
    k_cache = _nan_pool(nb, hkv, bs, d, dtype)
    v_cache = _nan_pool(nb, hkv, bs, d, dtype)
    tables = np.full((S, table_width), TABLE_PAD, dtype=np.int32)
    cursor = 0
    for s, L in enumerate(lens):
        nblk = -(-int(L) // bs)
        if cursor + nblk > nb:
            raise ValueError(f"{name}: pool of {nb} blocks exhausted")
        tables[s, :nblk] = free_list[cursor:cursor + nblk]
        cursor += nblk
    k_new = np.empty((S, hkv, d), dtype=np.uint16)
    v_new = np.empty((S, hkv, d), dtype=np.uint16)
    for s, L in enumerate(lens):
        L = int(L)
        boost = None
        if key_boost_frac > 0.0:
            nb_boost = int(round(key_boost_frac * L))
            boost = np.ones(L, dtype=np.float64)
            boost[draw.np.choice(L, size=nb_boost, replace=False)] = key_boost
        for t0 in range(0, L, chunk_tokens):
            t1 = min(L, t0 + chunk_tokens)
            kr = draw.normal_bits((t1 - t0, hkv, d), dtype, None if boost is None else boost[t0:t1])
            vr = draw.normal_bits((t1 - t0, hkv, d), dtype)
            old = min(t1, L - 1)  # rows already in the cache before this step
            _place(k_cache, tables[s], t0, kr[:max(0, old - t0)], bs)
            _place(v_cache, tables[s], t0, vr[:max(0, old - t0)], bs)
            if t1 == L:
                k_new[s] = kr[-1]
                v_new[s] = vr[-1]
    q = draw.normal_bits((S, hq, d), dtype)
    lens32 = np.asarray(lens, dtype=np.int32)
    slot_mapping = np.array([_slots(tables[s], [int(L) - 1], bs)[0] for s, L in enumerate(lens)],
                            dtype=np.int64)
    step = Step(q=q, block_tables=tables, context_lens=lens32, k_new=k_new, v_new=v_new,
                slot_mapping=slot_mapping)
    return Workload(name=name, dtype=dtype, num_q_heads=hq, num_kv_heads=hkv, head_dim=d, block_size=bs,
                    num_blocks=nb, scale=1.0 / math.sqrt(d), k_cache=k_cache, v_cache=v_cache, steps=[step],
                    description=description)


def tiny(seed: int = 1) -> Workload:
    """4 seqs, 8 heads (MHA), d=64, bs=16, fp16; L ~ U{1..200}; 64-block pool, random permutation."""
    draw = _Draw(seed)
    lens = draw.np.integers(1, 201, size=4)
    free = draw.np.permutation(64).astype(np.int32)
    return _fill_sequences(draw, "tiny_decode", "fp16", lens, 8, 8, 64, 16, 64, 13, free,
                           description="4 seqs, 8 heads MHA, d64, bs16, fp16, L~U[1,200], 64-block pool")


def llama2_7b(seed: int = 2, num_seqs: int = 64, num_blocks: int = 8192) -> Workload:
    """Llama-2-7B-shaped decode: 64 seqs, 32 heads, d=128, bs=16, fp16; L ~ U{128..2048};
    8192-block pool with shuffled free-list allocation."""
    draw = _Draw(seed)
    lens = draw.np.integers(128, 2049, size=num_seqs)
    free = draw.np.permutation(num_blocks).astype(np.int32)
    return _fill_sequences(draw, "llama2_7b_decode", "fp16", lens, 32, 32, 128, 16, num_blocks, 128, free,
                           description=f"{num_seqs} seqs, 32 heads, d128, bs16, fp16, L~U[128,2048], "
                                       f"{num_blocks}-block shuffled pool")


def gqa_llama3(seed: int = 3, num_seqs: int = 256, num_blocks: int = 65536) -> Workload:
    """GQA decode: 256 seqs, 32 q / 8 kv heads, d=128, bs=16, bf16; L lognormal with median 512
    (sigma 1 in log space), rounded and clipped to [16, 8192]; 65536-block pool, random placement."""
    draw = _Draw(seed)
    lens = np.clip(np.rint(np.exp(draw.np.normal(math.log(512.0), 1.0, size=num_seqs))), 16, 8192)
    lens = lens.astype(np.int64)
    free = draw.np.permutation(num_blocks).astype(np.int32)
    return _fill_sequences(draw, "gqa_llama3_decode", "bf16", lens, 32, 8, 128, 16, num_blocks, 512, free,
                           description=f"{num_seqs} seqs, 32q/8kv heads, d128, bs16, bf16, L lognormal "
                                       f"median 512 clip [16,8192], {num_blocks}-block pool")


def long_context(seed: int = 4, num_seqs: int = 8, num_blocks: int = 8192,
                 lo: int = 16384, hi: int = 32768) -> Workload:
    """Long-context split-K: 8 seqs, 32 heads, d=128, bs=32, bf16; L ~ U{16384..32768};
    1% of key rows (all heads) scaled by 8 before rounding; 8192-block pool, random placement."""
    draw = _Draw(seed)
    lens = draw.np.integers(lo, hi + 1, size=num_seqs)
    free = draw.np.permutation(num_blocks).astype(np.int32)
    width = -(-hi // 32)
    return _fill_sequences(draw, "long_context_splitk", "bf16", lens, 32, 32, 128, 32, num_blocks, width, free,
                           key_boost_frac=0.01, key_boost=8.0,
                           description=f"{num_seqs} seqs, 32 heads, d128, bs32, bf16, L~U[{lo},{hi}], "
                                       f"1% keys x8, {num_blocks}-block pool")


def custom(seed: int, num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int, block_size: int,
           lens, dtype: str = "fp16", num_blocks: int | None = None, table_width: int | None = None,
           key_boost_frac: float = 0.0, key_boost: float = 1.0) -> Workload:
    """A small single-step case with explicit context lengths (randomly placed blocks)."""
    draw = _Draw(seed)
    lens = np.asarray(lens, dtype=np.int64)
    assert lens.shape == (num_seqs,)
    need = int(sum(-(-int(L) // block_size) for L in lens))
    nb = num_blocks if num_blocks is not None else max(1, need + 3)
    free = draw.np.permutation(nb).astype(np.int32)
    width = table_width if table_width is not None else max(1, -(-int(lens.max(initial=1)) // block_size))
    w = _fill_sequences(draw, "custom", dtype, [int(x) for x in lens], num_q_heads, num_kv_heads, head_dim,
                        block_size, nb, width, free, key_boost_frac=key_boost_frac, key_boost=key_boost)
    # a zero-length sequence has nothing to write this step
    st = w.steps[0]
    keep = lens > 0
    if not keep.all():
        st.k_new, st.v_new, st.slot_mapping = st.k_new[keep], st.v_new[keep], st.slot_mapping[keep]
    return w


def shared_prefix(seed: int = 5, num_steps: int = 16, groups: int = 8, seqs_per_group: int = 8,
                  prefix_tokens: int = 1024, max_suffix: int = 256, num_blocks: int = 4096,
                  retire_after: int = 8) -> Workload:
    """Parallel sampling with a shared prefix plus continuous batching.

    8 groups x 8 seqs, 32 q / 8 kv heads, d=128, bs=16, bf16.  Each group's 8
    tables name the same 64 physical prefix blocks (1024 tokens); each sequence
    adds a private suffix of U{0..256} tokens.  Every step appends one token per
    live sequence (allocating a block when it starts a new one), writes it, and
    decodes.  After ``retire_after`` steps group 0 retires (its blocks go back
    to the front of the free list, so they are reused at once) and a new group
    joins; its prefix and suffixes are written by that step's KV write.
    """
    dtype, hq, hkv, d, bs = "bf16", 32, 8, 128, 16
    assert prefix_tokens % bs == 0, "the shared prefix must end on a block boundary (no copy-on-write)"
    draw = _Draw(seed)
    free = list(draw.np.permutation(num_blocks).astype(np.int32))
    k_cache = _nan_pool(num_blocks, hkv, bs, d, dtype)
    v_cache = _nan_pool(num_blocks, hkv, bs, d, dtype)
    width = -(-(prefix_tokens + max_suffix + num_steps + 1) // bs)

    def alloc(n):
        out = free[:n]
        del free[:n]
        if len(out) < n:
            raise ValueError("shared_prefix: pool exhausted")
        return out

    def new_group():
        """Returns (seqs, pending writes) for one group: tables, lengths and rows to write."""
        prefix_blocks = alloc(prefix_tokens // bs)
        pk = draw.normal_bits((prefix_tokens, hkv, d), dtype)
        pv = draw.normal_bits((prefix_tokens, hkv, d), dtype)
        seqs = []
        for _ in range(seqs_per_group):
            suffix = int(draw.np.integers(0, max_suffix + 1))
            seqs.append({"blocks": list(prefix_blocks), "len": prefix_tokens, "suffix": suffix,
                         "prefix": prefix_blocks})
        return seqs, pk, pv

    def extend_blocks(seq, new_len):
        need = -(-new_len // bs)
        if need > len(seq["blocks"]):
            seq["blocks"].extend(alloc(need - len(seq["blocks"])))

    def table_of(seq):
        row = np.full(width, TABLE_PAD, dtype=np.int32)
        row[:len(seq["blocks"])] = seq["blocks"]
        return row

    # initial state: groups laid directly into the cache (prefix + suffix), like the other workloads
    live = []
    for _g in range(groups):
        seqs, pk, pv = new_group()
        row0 = table_of(seqs[0])
        _place(k_cache, row0, 0, pk, bs)
        _place(v_cache, row0, 0, pv, bs)
        for seq in seqs:
            extend_blocks(seq, prefix_tokens + seq["suffix"])
            sk = draw.normal_bits((seq["suffix"], hkv, d), dtype)
            sv = draw.normal_bits((seq["suffix"], hkv, d), dtype)
            _place(k_cache, table_of(seq), prefix_tokens, sk, bs)
            _place(v_cache, table_of(seq), prefix_tokens, sv, bs)
            seq["len"] = prefix_tokens + seq["suffix"]
        live.append(seqs)

    steps = []
    for step_idx in range(num_steps):
        ks, vs, slots = [], [], []
        if step_idx == retire_after:
            gone = live.pop(0)
            returned = []
            for seq in gone:
                returned.extend(b for b in seq["blocks"] if b not in seq["prefix"])
            returned.extend(gone[0]["prefix"])
            free[:0] = returned  # reused first
            seqs, pk, pv = new_group()
            row0 = table_of(seqs[0])
            ks.append(pk); vs.append(pv); slots.append(_slots(row0, np.arange(prefix_tokens), bs))
            for seq in seqs:
                extend_blocks(seq, prefix_tokens + seq["suffix"])
                sk = draw.normal_bits((seq["suffix"], hkv, d), dtype)
                sv = draw.normal_bits((seq["suffix"], hkv, d), dtype)
                ks.append(sk); vs.append(sv)
                slots.append(_slots(table_of(seq), np.arange(prefix_tokens, prefix_tokens + seq["suffix"]), bs))
                seq["len"] = prefix_tokens + seq["suffix"]
            live.append(seqs)
        flat = [seq for grp in live for seq in grp]
        for seq in flat:
            pos = seq["len"]
            extend_blocks(seq, pos + 1)
            seq["len"] = pos + 1
            ks.append(draw.normal_bits((1, hkv, d), dtype))
            vs.append(draw.normal_bits((1, hkv, d), dtype))
            slots.append(_slots(table_of(seq), [pos], bs))
        tables = np.stack([table_of(seq) for seq in flat])
        lens = np.array([seq["len"] for seq in flat], dtype=np.int32)
        q = draw.normal_bits((len(flat), hq, d), dtype)
        steps.append(Step(q=q, block_tables=tables, context_lens=lens, k_new=np.concatenate(ks),
                          v_new=np.concatenate(vs), slot_mapping=np.concatenate(slots).astype(np.int64)))
    return Workload(name="shared_prefix_step", dtype=dtype, num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                    block_size=bs, num_blocks=num_blocks, scale=1.0 / math.sqrt(d), k_cache=k_cache,
                    v_cache=v_cache, steps=steps,
                    description=f"{groups}x{seqs_per_group} seqs sharing {prefix_tokens}-token prefixes, "
                                f"suffix U[0,{max_suffix}], 32q/8kv, d128, bs16, bf16, {num_steps} steps, "
                                f"group 0 retires after step {retire_after}")


@dataclass
class PrefillCase:
    """Causal prefill of new tokens over a paged context whose K/V rows (the new tokens' included)
    are already in the pool: sequence s brings query rows query_start[s]..query_start[s+1]-1, the
    last n_s of its context_lens[s] tokens."""

    name: str
    dtype: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    scale: float
    k_cache: np.ndarray  # uint16 [NB, Hkv, bs, d]
    v_cache: np.ndarray
    q: np.ndarray  # uint16 [N, Hq, d]
    query_start: np.ndarray  # int32 [S + 1]
    context_lens: np.ndarray  # int32 [S]
    block_tables: np.ndarray  # int32 [S, MB]
    description: str = ""

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def query_lens(self) -> np.ndarray:
        return np.diff(self.query_start)

    @property
    def max_query_len(self) -> int:
        return int(self.query_lens.max(initial=0))

    @property
    def attended_pairs(self) -> int:
        """Sum over new tokens of the keys each attends to (causal)."""
        total = 0
        for L, n in zip(self.context_lens.astype(np.int64), self.query_lens.astype(np.int64)):
            total += int(n * (L - n) + n * (n + 1) // 2)
        return total


def prefill_case(seed: int, shape, num_q_heads: int, num_kv_heads: int, head_dim: int, block_size: int,
                 dtype: str = "fp16", num_blocks: int | None = None, table_width: int | None = None,
                 name: str = "custom_prefill", description: str = "") -> PrefillCase:
    """shape: [(L, n)] per sequence (context length, new tokens).  Blocks come from a shuffled free
    list; unowned slots hold NaN."""
    draw = _Draw(seed)
    lens = [int(L) for L, _ in shape]
    ns = [int(n) for _, n in shape]
    assert all(0 <= n <= L for L, n in zip(lens, ns))
    bs = block_size
    need = sum(-(-L // bs) for L in lens)
    nb = num_blocks if num_blocks is not None else need + 3
    if need > nb:
        raise ValueError(f"{name}: pool of {nb} blocks too small for {need}")
    width = table_width if table_width is not None else max(1, max((-(-L // bs) for L in lens), default=1))
    free = draw.np.permutation(nb).astype(np.int32)
    k_cache = _nan_pool(nb, num_kv_heads, bs, head_dim, dtype)
    v_cache = _nan_pool(nb, num_kv_heads, bs, head_dim, dtype)
    tables = np.full((len(lens), width), TABLE_PAD, dtype=np.int32)
    cursor = 0
    for s, L in enumerate(lens):
        nblk = -(-L // bs)
        tables[s, :nblk] = free[cursor:cursor + nblk]
        cursor += nblk
        for t0 in range(0, L, 8192):
            t1 = min(L, t0 + 8192)
            _place(k_cache, tables[s], t0, draw.normal_bits((t1 - t0, num_kv_heads, head_dim), dtype), bs)
            _place(v_cache, tables[s], t0, draw.normal_bits((t1 - t0, num_kv_heads, head_dim), dtype), bs)
    qs = np.concatenate([[0], np.cumsum(ns)]).astype(np.int32)
    q = draw.normal_bits((int(qs[-1]), num_q_heads, head_dim), dtype)
    return PrefillCase(name=name, dtype=dtype, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
                       head_dim=head_dim, block_size=bs, num_blocks=nb, scale=1.0 / math.sqrt(head_dim),
                       k_cache=k_cache, v_cache=v_cache, q=q, query_start=qs,
                       context_lens=np.asarray(lens, dtype=np.int32), block_tables=tables, description=description)


def prefill_llama2_7b(seed: int = 6, num_seqs: int = 16, num_blocks: int = 4096) -> PrefillCase:
    """Llama-2-7B-shaped prompt prefill: 16 prompts of U{512..2048} tokens, 32 heads, d=128, bs=16,
    fp16, whole prompt in one pass; 4096-block shuffled pool."""
    rng = np.random.Generator(np.random.PCG64(seed + 1000))
    lens = rng.integers(512, 2049, size=num_seqs)
    return prefill_case(seed, [(int(L), int(L)) for L in lens], 32, 32, 128, 16, "fp16", num_blocks, 128,
                        name="llama2_7b_prefill",
                        description=f"{num_seqs} prompts, L~U[512,2048], 32 heads, d128, bs16, fp16, "
                                    f"{num_blocks}-block pool")


def chunked_prefill_gqa(seed: int = 7, num_seqs: int = 32, chunk: int = 512, num_blocks: int = 16384) -> PrefillCase:
    """Chunked prefill, GQA 32 q / 8 kv heads, d=128, bs=16, bf16: each sequence has a cached prefix
    of U{0..3584} tokens and brings the next chunk of 512; 16384-block pool."""
    rng = np.random.Generator(np.random.PCG64(seed + 1000))
    prefix = rng.integers(0, 3585, size=num_seqs)
    return prefill_case(seed, [(int(p) + chunk, chunk) for p in prefix], 32, 8, 128, 16, "bf16", num_blocks, 256,
                        name="gqa_chunked_prefill",
                        description=f"{num_seqs} seqs, cached prefix U[0,3584] + chunk {chunk}, 32q/8kv heads, "
                                    f"d128, bs16, bf16, {num_blocks}-block pool")


PREFILL_NAMED = {
    "llama2_7b_prefill": prefill_llama2_7b,
    "gqa_chunked_prefill": chunked_prefill_gqa,
}


NAMED = {
    "tiny_decode": tiny,
    "llama2_7b_decode": llama2_7b,
    "gqa_llama3_decode": gqa_llama3,
    "long_context_splitk": long_context,
    "shared_prefix_step": shared_prefix,
}


def kv_bytes(step: Step, num_kv_heads: int, head_dim: int, elem: int = 2) -> int:
    """K and V bytes of exactly the live tokens (no partial-block slack)."""
    return int(step.context_lens.astype(np.int64).sum()) * num_kv_heads * head_dim * 2 * elem


def unique_kv_bytes(step: Step, num_kv_heads: int, head_dim: int, block_size: int, elem: int = 2) -> int:
    """K and V bytes of the distinct physical rows the step reads: a block named by several
    tables counts once (with the most rows any reader uses)."""
    rows_of = {}
    for s in range(step.num_seqs):
        L = int(step.context_lens[s])
        for i in range(-(-L // block_size)):
            p = int(step.block_tables[s, i])
            rows_of[p] = max(rows_of.get(p, 0), min(block_size, L - i * block_size))
    return sum(rows_of.values()) * num_kv_heads * head_dim * 2 * elem
