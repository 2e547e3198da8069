"""GPU parity of the tensor-core chunked-prefill path (tcgen05 + TMEM + TMA) against the fp64
oracle, through the C ABI: ragged query tiles, GQA packing of 128-row tiles, pages of 16 to
256 keys, sliding windows, decode and prefill sequences in one call."""
import pytest
import torch

import oracle_pins
import paged_kv_attention_39_b200 as pa
from gpu_helpers import check, run_gqa, sample_rows, visible_count
from paged_kv_attention_39_b200 import workloads as W

pytestmark = pytest.mark.gpu


def prefill_wl(seed, hq=32, hkv=8, d=128, ps=64, dtype=torch.bfloat16, hist=(0, 700), chunk=200, batch=3,
               window=0, causal=True):
    hs = W._uniform_ints(seed, 77, batch, hist[0], hist[1])
    lens = [h + chunk for h in hs]
    return W.make_gqa("small_prefill", seed, lens, [chunk] * batch, hq, hkv, d, d, ps, dtype, causal=causal,
                      window=window)


def status_ok(wl):
    return True


def on_tensor_cores(plan):
    """The last call ran the tcgen05 prefill kernel and no CUDA-core kernel."""
    k = pa.pa_plan_get_info(plan)["last_kernels"]
    return bool(k & pa.PA_KERNEL_PREFILL_TC) and not (k & pa.PA_KERNEL_SIMT)


def test_prefill_basic(orc):
    wl = prefill_wl(1)
    ref = orc.run(wl)
    plan = pa.plan_for(wl)
    out, lse = run_gqa(wl, plan=plan)
    assert pa.pa_plan_get_info(plan)["last_launches"] == 1
    assert on_tensor_cores(plan)
    assert pa.pa_plan_device_status(plan) == 0
    plan.close()
    check(wl, out, lse, *ref, tag="prefill basic")


@pytest.mark.parametrize("dtype,hq,hkv,ps,window,causal", [
    (torch.bfloat16, 32, 8, 64, 0, True),
    (torch.float16, 32, 8, 64, 0, True),
    (torch.bfloat16, 8, 8, 16, 0, True),      # G 1, pages of 16: four boxes per 64-key tile
    (torch.bfloat16, 16, 8, 32, 100, True),   # G 2, sliding window
    (torch.bfloat16, 64, 4, 128, 0, False),   # G 16, not causal, two tiles per page
    (torch.float16, 32, 4, 256, 300, True),   # G 8, pages of 256, window
    (torch.bfloat16, 32, 8, 64, 1, True),     # window 1: each row sees itself only
])
def test_prefill_head_dim_256(orc, dtype, hq, hkv, ps, window, causal):
    """D = 256 on the tcgen05 prefill kernel (64-key tiles): ragged query tiles and histories from
    empty to 700 keys, against the oracle element by element."""
    wl = prefill_wl(11, hq=hq, hkv=hkv, d=256, ps=ps, dtype=dtype, hist=(0, 700), chunk=150, window=window,
                    causal=causal)
    ref = orc.run(wl)
    plan = pa.plan_for(wl)
    out, lse = run_gqa(wl, plan=plan)
    assert on_tensor_cores(plan)
    assert pa.pa_plan_device_status(plan) == 0
    plan.close()
    check(wl, out, lse, *ref, tag=f"d256 {dtype} G{hq // hkv} ps{ps} w{window} c{causal}")


def test_prefill_head_dim_256_many_units_and_decode_rows(orc):
    """Several hundred D = 256 tiles walked by each persistent CTA in turn, plus decode rows (the
    D = 256 split-KV decode kernel) in the same call."""
    hs = W._uniform_ints(12, 78, 40, 0, 600)
    lens = [h + 70 for h in hs] + [3000, 1500]
    qs = [70] * 40 + [1, 1]
    wl = W.make_gqa("d256_many", 12, lens, qs, 16, 4, 256, 256, 64, torch.bfloat16, causal=True, window=0)
    ref = orc.run(wl)
    plan = pa.plan_for(wl)
    out, lse = run_gqa(wl, plan=plan)
    k = pa.pa_plan_get_info(plan)["last_kernels"]
    assert k & pa.PA_KERNEL_PREFILL_TC and k & pa.PA_KERNEL_DECODE_TC and not k & pa.PA_KERNEL_SIMT
    assert pa.pa_plan_device_status(plan) == 0
    plan.close()
    check(wl, out, lse, *ref, tag="d256 many units + decode")


def test_prefill_head_dim_256_mask_bit_exact_by_counts():
    for window, causal in ((0, True), (70, True), (33, False)):
        wl = W.make_gqa("pmask256", 13, [200, 450, 64], [200, 130, 64], 16, 4, 256, 256, 64, torch.bfloat16,
                        causal=causal, window=window)
        wl.q.zero_()
        out, lse = run_gqa(wl)
        s = wl.sched
        for si in range(s.num_seqs):
            L = int(s.seq_lens[si]); q0 = int(s.query_offsets[si]); n = int(s.query_offsets[si + 1]) - q0
            cnt = torch.tensor([visible_count(L, n, j, causal, window)[0] for j in range(n)])
            got = torch.exp(lse[q0:q0 + n].double()).round().long()
            assert bool((got == cnt.view(-1, 1)).all()), (window, causal, si)


@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 8), (64, 8), (32, 2), (128, 1)])
def test_prefill_groups(orc, hq, hkv):
    wl = prefill_wl(2, hq=hq, hkv=hkv, chunk=150)
    ref = orc.run(wl)
    out, lse = run_gqa(wl)
    check(wl, out, lse, *ref, tag=f"G{hq // hkv}")


@pytest.mark.parametrize("ps", [16, 32, 128, 256])
def test_prefill_page_sizes(orc, ps):
    wl = prefill_wl(3, ps=ps, hist=(1, 900), chunk=97)
    ref = orc.run(wl)
    out, lse = run_gqa(wl)
    check(wl, out, lse, *ref, tag=f"ps{ps}")


@pytest.mark.parametrize("dtype,d", [(torch.float16, 128), (torch.bfloat16, 64), (torch.float16, 64)])
def test_prefill_dtypes_and_head_dims(orc, dtype, d):
    wl = prefill_wl(4, dtype=dtype, d=d, chunk=130)
    ref = orc.run(wl)
    out, lse = run_gqa(wl)
    check(wl, out, lse, *ref, tag=f"{dtype} d{d}")


@pytest.mark.parametrize("window,causal", [(1, True), (50, True), (300, True), (5000, True), (0, False), (77, False)])
def test_prefill_masks(orc, window, causal):
    wl = prefill_wl(5, window=window, causal=causal, hist=(0, 500), chunk=180)
    ref = orc.run(wl)
    out, lse = run_gqa(wl)
    check(wl, out, lse, *ref, tag=f"window {window} causal {causal}")


@pytest.mark.parametrize("d,dtype,window,causal,ps", [(64, torch.bfloat16, 0, True, 64), (128, torch.float16, 100, True, 16),
                                                    (128, torch.bfloat16, 0, False, 128)])
def test_prefill_many_units_per_cta(orc, d, dtype, window, causal, ps):
    """Several hundred 128-row tiles, so that each CTA of the persistent kernel runs one unit after
    another (stage indices and barrier phases carried across units, Q reloaded per unit), with
    ragged last tiles and histories from empty to 600 keys."""
    wl = prefill_wl(8, hq=16, hkv=4, d=d, ps=ps, dtype=dtype, hist=(0, 600), chunk=70, batch=48,
                    window=window, causal=causal)
    ref = orc.run(wl)
    plan = pa.plan_for(wl)
    out, lse = run_gqa(wl, plan=plan)
    assert pa.pa_plan_get_info(plan)["last_launches"] == 1
    assert pa.pa_plan_device_status(plan) == 0
    plan.close()
    check(wl, out, lse, *ref, tag=f"many units d{d} {dtype} w{window} c{causal} ps{ps}")


def test_prefill_without_history_and_single_query_tiles(orc):
    wl = W.make_gqa("p0", 6, [1, 33, 128, 129, 300], [1, 33, 128, 129, 300], 32, 8, 128, 128, 64,
                    torch.bfloat16, causal=True)
    ref = orc.run(wl)
    out, lse = run_gqa(wl)
    check(wl, out, lse, *ref, tag="no history")


def test_mixed_decode_and_prefill_one_call(orc):
    """Decode rows (tensor-core split-KV decode kernel) and prefill chunks (tcgen05 kernel) in
    one pa_forward, sliding window, Hq 64 / Hkv 8."""
    lens = [3000, 5000, 777, 2100 + 300, 900 + 256]
    qs = [1, 1, 1, 300, 256]
    wl = W.make_gqa("mixed", 7, lens, qs, 64, 8, 128, 128, 64, torch.bfloat16, causal=True, window=1000)
    ref = orc.run(wl)
    plan = pa.plan_for(wl)
    out, lse = run_gqa(wl, plan=plan)
    assert pa.pa_plan_get_info(plan)["last_launches"] >= 2
    plan.close()
    check(wl, out, lse, *ref, tag="mixed")


def test_prefill_mask_bit_exact_by_counts():
    for window, causal in ((0, True), (70, True), (33, False)):
        wl = W.make_gqa("pmask", 8, [200, 450, 64], [200, 130, 64], 16, 4, 128, 128, 64, torch.bfloat16,
                        causal=causal, window=window)
        wl.q.zero_()
        out, lse = run_gqa(wl)
        s = wl.sched
        for si in range(s.num_seqs):
            L = int(s.seq_lens[si]); q0 = int(s.query_offsets[si]); n = int(s.query_offsets[si + 1]) - q0
            cnt = torch.tensor([visible_count(L, n, j, causal, window)[0] for j in range(n)])
            got = torch.exp(lse[q0:q0 + n].double()).round().long()
            assert bool((got == cnt.view(-1, 1)).all()), (window, causal, si)


def test_prefill_block_table_indexing_bit_exact():
    wl = W.make_gqa("pidx", 9, [300, 190], [100, 70], 16, 4, 128, 128, 64, torch.float32, causal=True, window=150)
    target = oracle_pins.select_target_queries(wl, 6, margin=120.0)
    wl.q = wl.q.to(torch.bfloat16); wl.k_cache = wl.k_cache.to(torch.bfloat16); wl.v_cache = wl.v_cache.to(torch.bfloat16)
    out, lse = run_gqa(wl)
    s = wl.sched
    for (qi, h), (si, ts) in target.items():
        page = int(s.block_tables[si, ts // s.page_size])
        assert torch.equal(out[qi, h], wl.v_cache[page, ts % s.page_size, h // 4]), (qi, h, si, ts)


def test_chunked_equals_one_shot_on_gpu(orc):
    hist, na, nb = 333, 160, 190
    wl = W.make_gqa("chunks", 10, [hist + na + nb], [na + nb], 32, 8, 128, 128, 64, torch.bfloat16)
    s = wl.sched
    out, lse = run_gqa(wl)
    pa_ = pa.pa_plan_create([hist + na], [0, na], s.block_tables, 64, s.num_pages)
    pb_ = pa.pa_plan_create([hist + na + nb], [0, nb], s.block_tables, 64, s.num_pages)
    oa, la = run_gqa(wl, plan=pa_, q=wl.q[:na])
    ob, lb = run_gqa(wl, plan=pb_, q=wl.q[na:])
    pa_.close(); pb_.close()
    assert float((torch.cat([oa, ob]).float() - out.float()).abs().max()) <= 1e-2
    assert float((torch.cat([la, lb]) - lse).abs().max()) <= 2e-3


@pytest.mark.slow
def test_full_size_chunked_prefill_sampled(orc):
    wl = W.c3_chunked_prefill(0)
    rows = sample_rows(wl, 256, seed=2)
    ref = orc.run(wl, rows=rows)
    out, lse = run_gqa(wl)
    check(wl, out, lse, *ref, rows=rows, tag="full prefill")


@pytest.mark.slow
def test_full_size_window_mixed_sampled(orc):
    wl = W.c4_window_mixed(0)
    rows = sample_rows(wl, 256, seed=3)
    ref = orc.run(wl, rows=rows)
    out, lse = run_gqa(wl)
    check(wl, out, lse, *ref, rows=rows, tag="full mixed")
