"""Launch configuration depends on the batch size: calls of different sizes, in any order,
must all launch (regression: a smaller batch once lowered a kernel's shared-memory limit
below what a later, larger batch needed)."""
import numpy as np
import pytest

import workloads as W
from gpu_util import DeviceState, compare, oracle_step, require_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2)])
def test_alternating_batch_sizes(hq, hkv):
    require_gpu()
    big = W.custom(seed=41, num_seqs=300, num_q_heads=hq, num_kv_heads=hkv, head_dim=64, block_size=16,
                   lens=np.random.default_rng(1).integers(1, 90, size=300), dtype="fp16")
    small = W.custom(seed=42, num_seqs=3, num_q_heads=hq, num_kv_heads=hkv, head_dim=64, block_size=16,
                     lens=[5, 70, 33], dtype="fp16")
    states = {id(w): DeviceState(w) for w in (big, small)}
    for w in (big, small):
        states[id(w)].write(w.steps[0])
    for w in (big, small, big, small):
        st = w.steps[0]
        out = states[id(w)].decode(st)
        _, _, ref = oracle_step(w, w.k_cache, w.v_cache, st)
        compare(out, ref, "fp16", what=f"S={st.num_seqs}")
