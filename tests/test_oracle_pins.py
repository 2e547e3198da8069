"""The fp64 oracle against facts that do not come from it (see tests/oracle_pins.py)."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(orc, pin):
    pin(orc)


def test_oracle_rejects_bad_schedule(orc):
    import torch
    from paged_kv_attention_39_b200 import workloads as W
    wl = W.make_gqa("bad", 1, [20], [1], 2, 1, 8, 8, 8, torch.float32)
    bt = wl.sched.block_tables.clone()
    bt[0, 1] = wl.sched.num_pages  # outside the pool
    with pytest.raises(ValueError):
        orc.attention(wl.q, wl.k_cache, wl.v_cache, wl.sched.seq_lens, wl.sched.query_offsets, bt, 8,
                      wl.scale)
    with pytest.raises(ValueError):  # more queries than keys
        orc.attention(wl.q, wl.k_cache, wl.v_cache, torch.tensor([0]), wl.sched.query_offsets,
                      wl.sched.block_tables, 8, wl.scale)
