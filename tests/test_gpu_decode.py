"""GPU parity of the decode paths (CUDA-core kernel, tensor-core split-KV kernel, combine)
against the fp64 oracle, element by element on seeded inputs, through the C ABI."""
import math

import pytest
import torch

import oracle_pins
import paged_kv_attention_39_b200 as pa
from gpu_helpers import check, run, run_gqa, sample_rows, visible_count
from paged_kv_attention_39_b200 import workloads as W

pytestmark = pytest.mark.gpu

SIMT = pa.PA_PATH_SIMT


@pytest.mark.parametrize("seed", range(10))
@pytest.mark.parametrize("kv_chunk", [0, -1, 16, 23, 64])
def test_tiny_fp32_decode(orc, seed, kv_chunk):
    """2 sequences (37 and 100 keys), Hq 4, Hkv 2, D 64, pages of 16 shuffled in a 16-page pool
    with 6 NaN pages; forced splits cut 100 keys into 1..7 parts."""
    wl = W.c1_tiny_fp32_decode(seed)
    ref = orc.run(wl)
    out, lse = run_gqa(wl, kv_chunk=kv_chunk)
    check(wl, out, lse, *ref, tag=f"seed {seed} chunk {kv_chunk}")


def small_decode(seed, dtype=torch.bfloat16, hq=32, hkv=8, d=128, batch=8, lmin=17, lmax=600, ps=16,
                 window=0, qn=1):
    lens = W._uniform_ints(seed, 99, batch, lmin, lmax)
    return W.make_gqa("small_decode", seed, lens, [qn] * batch, hq, hkv, d, d, ps, dtype, window=window)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("kv_chunk", [0, -1, 48, 100])
def test_small_decode_tensor_core(orc, dtype, d, kv_chunk):
    wl = small_decode(1, dtype=dtype, d=d)
    ref = orc.run(wl)
    out, lse = run_gqa(wl, kv_chunk=kv_chunk)
    check(wl, out, lse, *ref, tag=f"{dtype} d{d} chunk {kv_chunk}")


@pytest.mark.parametrize("hq,hkv,qn", [(8, 8, 1), (16, 2, 1), (16, 1, 1), (8, 2, 3), (4, 2, 8), (6, 2, 5)])
def test_decode_groups_and_multi_query(orc, hq, hkv, qn):
    """G from 1 to 16 and several queries per sequence (speculative-decode shapes): up to 16
    rows share one KV head; per-element causal masks at right-aligned positions."""
    wl = small_decode(2, hq=hq, hkv=hkv, qn=qn, window=0, lmin=qn, lmax=300)
    ref = orc.run(wl)
    for kv_chunk in (0, 32):
        out, lse = run_gqa(wl, kv_chunk=kv_chunk)
        check(wl, out, lse, *ref, tag=f"G{hq // hkv} n{qn} chunk {kv_chunk}")


@pytest.mark.parametrize("hq,hkv,qn", [(16, 1, 1), (8, 2, 4), (4, 4, 1), (32, 8, 1)])
def test_decode_head_dim_64(orc, hq, hkv, qn):
    """head_dim 64 (32-key warp tiles) with 1 to 16 rows per KV head, parts that start off the
    32-key grid (chunk 100) and ragged lengths."""
    wl = small_decode(5, hq=hq, hkv=hkv, d=64, qn=qn, lmin=qn, lmax=700)
    ref = orc.run(wl)
    for kv_chunk in (0, 100, -1):
        out, lse = run_gqa(wl, kv_chunk=kv_chunk)
        check(wl, out, lse, *ref, tag=f"d64 G{hq // hkv} n{qn} chunk {kv_chunk}")


@pytest.mark.parametrize("hq,hkv,qn", [(16, 1, 1), (8, 2, 4), (4, 4, 1)])
def test_decode_head_dim_256(orc, hq, hkv, qn):
    """head_dim 256 on the tensor-core decode kernel, up to 16 rows per KV head (two n-tiles)."""
    wl = small_decode(3, hq=hq, hkv=hkv, d=256, qn=qn, lmin=qn, lmax=400)
    ref = orc.run(wl)
    for kv_chunk in (0, 64):
        out, lse = run_gqa(wl, kv_chunk=kv_chunk)
        check(wl, out, lse, *ref, tag=f"d256 G{hq // hkv} n{qn} chunk {kv_chunk}")


def test_split_rows_plan_reused(orc):
    """One plan, five calls with other queries and split sizes (the workspace, the cached work lists
    and the merge counters reused across calls), each against the oracle; the tensor-core decode
    kernel merges its own split rows (no merge launch)."""
    wl = small_decode(5, batch=12, lmin=200, lmax=3000)
    s = wl.sched
    plan = pa.plan_for(wl)
    for i, kv_chunk in enumerate((64, 64, 100, 0, 64)):
        q = W.randn(tuple(wl.q.shape), 100 + i, 1, wl.q.dtype)
        ref = orc.attention(q, wl.k_cache, wl.v_cache, s.seq_lens, s.query_offsets, s.block_tables, s.page_size,
                            wl.scale, wl.causal, wl.window)
        out, lse = run_gqa(wl, kv_chunk=kv_chunk, plan=plan, q=q)
        k = pa.pa_plan_get_info(plan)["last_kernels"]
        assert k & pa.PA_KERNEL_DECODE_TC and not k & pa.PA_KERNEL_MERGE, k
        check(wl, out, lse, *ref, tag=f"call {i} chunk {kv_chunk}")
    assert pa.pa_plan_device_status(plan) == 0
    plan.close()


def test_plan_memory_recycled_across_steps(orc):
    """Forty decode steps, each with a new plan (other lengths, so other work lists, part counts and
    workspace sizes) created on an upload stream and released as soon as its forward is queued,
    without synchronising: the library may hand a released plan's device memory to a later plan
    only once the work queued before the release has completed. Every step matches the oracle."""
    up = torch.cuda.Stream()
    main = torch.cuda.current_stream()
    steps = []
    for i in range(40):
        wl = small_decode(200 + i, batch=3 + i % 6, lmin=17, lmax=300 + 60 * i)
        plan = pa.plan_for(wl, device=0, stream=up)
        pa.pa_plan_prepare(plan, wl.q.dtype, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.v_head_dim,
                           wl.causal, wl.window, stream=up)
        main.wait_stream(up)
        qd, kd, vd = wl.q.to("cuda"), wl.k_cache.to("cuda"), wl.v_cache.to("cuda")
        out = torch.full((qd.shape[0], wl.num_q_heads, wl.v_head_dim), float("nan"), dtype=qd.dtype, device="cuda")
        lse = torch.full((qd.shape[0], wl.num_q_heads), float("nan"), dtype=torch.float32, device="cuda")
        pa.pa_forward(plan, qd, kd, vd, out, lse, wl.scale, wl.causal, wl.window, kv_chunk=64 if i % 2 else 0)
        plan.close()
        steps.append((wl, (qd, kd, vd), out, lse))
    torch.cuda.synchronize()
    for i, (wl, _, out, lse) in enumerate(steps):
        check(wl, out.cpu(), lse.cpu(), *orc.run(wl), tag=f"step {i}")


def test_split_rows_of_both_decode_kernels_in_one_call(orc):
    """Rows of the tensor-core decode kernel and of the CUDA-core kernel (5 queries x 4 heads per
    KV head, pages of 48 that the tcgen05 prefill kernel does not take) split in the same call and
    merged by one merge launch."""
    lens = [700, 1300, 450, 900, 1000]
    qs = [1, 5, 1, 5, 1]
    wl = W.make_gqa("two_merges", 6, lens, qs, 32, 8, 128, 128, 48, torch.bfloat16)
    ref = orc.run(wl)
    plan = pa.plan_for(wl)
    out, lse = run_gqa(wl, kv_chunk=96, plan=plan)
    k = pa.pa_plan_get_info(plan)["last_kernels"]
    assert k & pa.PA_KERNEL_DECODE_TC and k & pa.PA_KERNEL_SIMT and k & pa.PA_KERNEL_MERGE, k
    plan.close()
    check(wl, out, lse, *ref, tag="tensor-core and CUDA-core splits")


@pytest.mark.parametrize("window", [1, 7, 100, 5000])
def test_decode_window(orc, window):
    wl = small_decode(3, window=window, qn=2, hq=16, hkv=4, lmin=2, lmax=900)
    ref = orc.run(wl)
    for path in (pa.PA_PATH_AUTO, SIMT):
        out, lse = run_gqa(wl, kv_chunk=64, path=path)
        check(wl, out, lse, *ref, tag=f"window {window} path {path}")


def test_simt_path_matches_oracle_bf16(orc):
    wl = small_decode(4, d=128)
    ref = orc.run(wl)
    out, lse = run_gqa(wl, path=SIMT)
    check(wl, out, lse, *ref, tag="simt bf16")


def test_non_causal_and_edges(orc):
    """L = 1, a sequence with no queries between two others, non-causal scores."""
    wl = W.make_gqa("edges", 5, [1, 40, 300, 2], [1, 0, 1, 2], 8, 2, 128, 128, 16, torch.bfloat16,
                    causal=False, window=0)
    ref = orc.run(wl)
    for kv_chunk in (0, 16):
        out, lse = run_gqa(wl, kv_chunk=kv_chunk)
        check(wl, out, lse, *ref, tag=f"edges {kv_chunk}")


def test_empty_batch():
    wl = W.make_gqa("empty", 6, [10, 20], [0, 0], 8, 2, 128, 128, 16, torch.bfloat16)
    plan = pa.plan_for(wl)
    q = torch.empty(0, 8, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(0, 8, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(0, 8, dtype=torch.float32, device="cuda")
    pa.pa_forward(plan, q, wl.k_cache.cuda(), wl.v_cache.cuda(), out, lse, wl.scale)
    torch.cuda.synchronize()


@pytest.mark.parametrize("path", [pa.PA_PATH_AUTO, SIMT])
@pytest.mark.parametrize("kv_chunk", [0, 32])
def test_mask_bit_exact_by_counts(path, kv_chunk):
    """Q = 0 gives every visible key weight 1, so exp(lse) counts the visible keys exactly:
    the closed-form count for each row's absolute position, causal flag and window."""
    for window, causal in ((0, True), (37, True), (5, False)):
        wl = W.make_gqa("mask", 7, [1, 57, 130, 333], [1, 3, 1, 4], 8, 2, 128, 128, 16, torch.bfloat16,
                        causal=causal, window=window)
        wl.q.zero_()
        out, lse = run_gqa(wl, kv_chunk=kv_chunk, path=path)
        s = wl.sched
        for si in range(s.num_seqs):
            L = int(s.seq_lens[si]); q0 = int(s.query_offsets[si]); n = int(s.query_offsets[si + 1]) - q0
            for j in range(n):
                cnt, _, _ = visible_count(L, n, j, causal, window)
                got = torch.exp(lse[q0 + j].double()).round().long()
                assert bool((got == cnt).all()), (window, causal, si, j, got.tolist(), cnt)


@pytest.mark.parametrize("dtype,path", [(torch.float32, pa.PA_PATH_AUTO), (torch.bfloat16, pa.PA_PATH_AUTO),
                                        (torch.bfloat16, SIMT), (torch.float16, pa.PA_PATH_AUTO)])
def test_block_table_indexing_bit_exact(dtype, path):
    """Each row's query is a large multiple of one visible key: its output must be exactly that
    key's value row, read through the shuffled block table (NaN pages all around)."""
    wl = W.make_gqa("idx", 8, [70, 33, 129, 500], [1, 2, 1, 1], 8, 2, 128, 128, 16, torch.float32,
                    causal=True, window=300)
    target = oracle_pins.select_target_queries(wl, 5, margin=120.0)
    wl.q = wl.q.to(dtype); wl.k_cache = wl.k_cache.to(dtype); wl.v_cache = wl.v_cache.to(dtype)
    # recheck after rounding to dtype that the target still dominates by a wide margin
    out, lse = run_gqa(wl, kv_chunk=48, path=path)
    s = wl.sched
    for (qi, h), (si, ts) in target.items():
        page = int(s.block_tables[si, ts // s.page_size])
        want = wl.v_cache[page, ts % s.page_size, h // 4]
        assert torch.equal(out[qi, h], want), (qi, h, si, ts)


def test_page_permutation_invariance():
    wl = small_decode(9, lmin=100, lmax=700)
    out, lse = run_gqa(wl, kv_chunk=64)
    P = wl.sched.num_pages
    pi = torch.randperm(P, generator=torch.Generator().manual_seed(2))
    k2 = torch.empty_like(wl.k_cache); k2[pi] = wl.k_cache
    v2 = torch.empty_like(wl.v_cache); v2[pi] = wl.v_cache
    bt = wl.sched.block_tables.clone(); m = bt >= 0
    bt[m] = pi[bt[m].long()].to(torch.int32)
    wl.k_cache, wl.v_cache = k2, v2
    wl.sched.block_tables = bt
    out2, lse2 = run_gqa(wl, kv_chunk=64)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


def test_split_equals_unsplit_within_tolerance(orc):
    wl = small_decode(10, lmin=500, lmax=3000)
    ref = orc.run(wl)
    base, lbase = run_gqa(wl, kv_chunk=-1)
    for kv_chunk in (16, 112, 1000):
        out, lse = run_gqa(wl, kv_chunk=kv_chunk)
        check(wl, out, lse, *ref, tag=f"chunk {kv_chunk}")
        assert float((out.float() - base.float()).abs().max()) < 1e-2
        assert float((lse - lbase).abs().max()) < 1e-3


def test_plan_reuse_and_workspace_growth(orc):
    wl = small_decode(11, lmin=400, lmax=2000)
    ref = orc.run(wl)
    plan = pa.plan_for(wl)
    for kv_chunk in (256, 64, 16, 64):
        out, lse = run_gqa(wl, kv_chunk=kv_chunk, plan=plan)
        check(wl, out, lse, *ref, tag=f"reuse {kv_chunk}")
    assert pa.pa_plan_get_info(plan)["workspace_bytes"] > 0
    plan.close()


def test_forward_replayed_from_a_cuda_graph(orc):
    """pa_forward on decode rows (parts merged by the decode kernel's last CTA) and a prefill chunk
    (two launches, the decode kernel on the library's side stream, forked from and joined back into
    the captured stream), captured into a CUDA graph after a first call has built the plan's work list
    and workspace, then replayed with three other sets of queries written into the captured input
    buffer: every replay matches the oracle on its own queries (the merge counters are back at
    zero after each replay)."""
    wl = W.make_gqa("graph", 41, [3000, 700, 1400, 900], [1, 1, 200, 1], 32, 8, 128, 128, 64, torch.bfloat16)
    s = wl.sched
    plan = pa.plan_for(wl)
    qd, kd, vd = wl.q.to("cuda"), wl.k_cache.to("cuda"), wl.v_cache.to("cuda")
    out = torch.empty((qd.shape[0], wl.num_q_heads, wl.v_head_dim), dtype=qd.dtype, device="cuda")
    lse = torch.empty((qd.shape[0], wl.num_q_heads), dtype=torch.float32, device="cuda")
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        pa.pa_forward(plan, qd, kd, vd, out, lse, wl.scale, wl.causal, wl.window, kv_chunk=256)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        pa.pa_forward(plan, qd, kd, vd, out, lse, wl.scale, wl.causal, wl.window, kv_chunk=256)
    kernels = pa.pa_plan_get_info(plan)["last_kernels"]
    assert kernels & pa.PA_KERNEL_DECODE_TC and kernels & pa.PA_KERNEL_PREFILL_TC, kernels
    for i in range(3):
        q = W.randn(tuple(wl.q.shape), 300 + i, 1, wl.q.dtype)
        qd.copy_(q.to("cuda"))
        graph.replay()
        torch.cuda.synchronize()
        ref = orc.attention(q, wl.k_cache, wl.v_cache, s.seq_lens, s.query_offsets, s.block_tables, s.page_size,
                            wl.scale, wl.causal, wl.window)
        check(wl, out.cpu(), lse.cpu(), *ref, tag=f"graph replay {i}")
    assert pa.pa_plan_device_status(plan) == 0
    del graph
    plan.close()


@pytest.mark.slow
def test_full_size_bf16_decode_sampled(orc):
    """The full decode workload (batch 64, context U[512, 8192], Hq 32, Hkv 8, D 128, pages of
    16) in the benchmark's launch configuration, checked on sampled rows."""
    wl = W.c2_bf16_decode(0)
    rows = sample_rows(wl, 192, seed=1)
    ref = orc.run(wl, rows=rows)
    out, lse = run_gqa(wl)
    check(wl, out, lse, *ref, rows=rows, tag="full decode")
