"""The seeded input module: determinism, layout and poisoning of everything no key may read."""
import math

import torch

from paged_kv_attention_39_b200 import workloads as W


def test_deterministic_and_seed_sensitive():
    a = W.make_gqa("a", 5, [40, 7], [3, 7], 4, 2, 16, 16, 8, torch.bfloat16)
    b = W.make_gqa("a", 5, [40, 7], [3, 7], 4, 2, 16, 16, 8, torch.bfloat16)
    c = W.make_gqa("a", 6, [40, 7], [3, 7], 4, 2, 16, 16, 8, torch.bfloat16)
    assert torch.equal(a.q, b.q) and torch.equal(a.k_cache.nan_to_num(7), b.k_cache.nan_to_num(7))
    assert torch.equal(a.sched.block_tables, b.sched.block_tables)
    assert not torch.equal(a.q, c.q)


def test_large_draw_is_chunk_parallel_deterministic():
    x = W.randn((3, W._CHUNK + 17), 9, 1, torch.float32)
    y = W.randn((3, W._CHUNK + 17), 9, 1, torch.float32)
    assert torch.equal(x, y)
    assert abs(float(x.mean())) < 0.01 and abs(float(x.std()) - 1) < 0.01


def test_pool_layout_and_poison():
    wl = W.make_gqa("p", 3, [37, 100, 16], [1, 1, 16], 4, 2, 8, 8, 16, torch.float32)
    s = wl.sched
    need = [3, 7, 1]
    assert s.num_pages == sum(need) + math.ceil(sum(need) * 0.1)
    used = []
    for i, k in enumerate(need):
        assert (s.block_tables[i, :k] >= 0).all() and (s.block_tables[i, k:] == -1).all()
        used += s.block_tables[i, :k].tolist()
    assert len(set(used)) == len(used)  # no page shared
    for p in range(s.num_pages):
        assert bool(torch.isnan(wl.k_cache[p]).all()) == (p not in used)
    last = int(s.block_tables[0, 2])  # L = 37 -> slots 5.. of the third page are past the end
    assert torch.isnan(wl.k_cache[last, 5:]).all() and not torch.isnan(wl.k_cache[last, :5]).any()
    assert s.query_offsets.tolist() == [0, 1, 2, 18]


def test_tiny_config_shape():
    wl = W.c1_tiny_fp32_decode(0)
    assert wl.sched.num_pages == 16 and int(wl.sched.owned.sum()) == 10
    assert wl.q.shape == (2, 4, 64) and wl.k_cache.shape == (16, 16, 2, 64)
    assert wl.scale == 0.125 and wl.causal and wl.window == 0


def test_algorithmic_counts():
    wl = W.make_gqa("c", 1, [10, 20], [1, 4], 4, 2, 8, 8, 8, torch.bfloat16, window=3)
    # seq 0: one query at p=9 sees keys 7..9; seq 1: queries at 16..19 see 14..19
    assert W.algorithmic_kv_bytes(wl) == (3 + 6) * 2 * (8 + 8) * 2
    assert W.visible_pairs(wl) == 3 + 4 * 3


def test_next_row_work_counts():
    """The append, GQA backward and MLA backward numerators against per-pair brute force."""
    wl = W.make_gqa("w", 5, [10, 6], [4, 6], 8, 2, 16, 8, 4, torch.bfloat16, causal=True, window=3)
    s = wl.sched
    pairs = 0
    for i in range(s.num_seqs):
        L, n = int(s.seq_lens[i]), int(s.query_offsets[i + 1] - s.query_offsets[i])
        for j in range(n):
            p = L - n + j
            pairs += sum(1 for t in range(L) if t <= p and t + 3 > p)
    assert W.backward_flops(wl) == pairs * 8 * 2 * (3 * 16 + 2 * 8)
    assert W.append_bytes(wl) == 2 * s.num_queries * 2 * (16 + 8) * 2
    ml = W.make_mla("m", 6, [9, 5], [2, 5], 4, 32, 8, 4, torch.float16, causal=False)
    sm = ml.sched
    mpairs = sum(int(sm.seq_lens[i]) * int(sm.query_offsets[i + 1] - sm.query_offsets[i]) for i in range(sm.num_seqs))
    assert W.mla_backward_flops(ml) == mpairs * 4 * 2 * (3 * (32 + 8) + 2 * 32)
    wb, d_out = W.backward_chunk(0, batch=2, hmax=64, chunk=16)
    assert d_out.shape == (wb.sched.num_queries, 32, 128) and d_out.dtype == torch.bfloat16
    wa, nk, nv = W.append_chunk(0)
    assert nk.shape == (wa.sched.num_queries, 8, 128) and nv.shape == nk.shape
