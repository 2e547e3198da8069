"""Sparse top-K block attention on the GPU (pa_sparse_select + pa_sparse_forward) against the
fp64 oracle (alice-llm `llama3_sparse_attention`: proxy block scores, top-K selection,
attention over the selected blocks, logsumexp merge).

Where floating point decides the selection, the two sides are compared as follows:
  * proxy scores: float32 dot products of the stored values against the fp64 oracle, within
    1e-4 * (1 + |ref|); -inf (no visible key) must match exactly;
  * selection on integer-valued inputs with a power-of-two scale: every score is exact on both
    sides, so the selection (ties included) must match bit for bit;
  * selection on random inputs: rows whose oracle scores separate the k-th from the (k+1)-th
    block by more than 1e-3 must match exactly; every row must be a valid top-k of the oracle
    scores within 1e-3 (nothing unselected scores clearly above something selected);
  * attention with the oracle's own selection: elementwise, the tolerances of the dense path.
"""
import math

import pytest
import torch

import paged_kv_attention_39_b200 as pa
from paged_kv_attention_39_b200 import workloads as W
from gpu_helpers import check, sample_rows, to_dev

pytestmark = pytest.mark.gpu


def gpu_select(wl, bs, topk, plan=None, width=None, with_scores=True):
    own = plan is None
    if own:
        plan = pa.plan_for(wl)
    s = wl.sched
    nbs = (s.seq_lens.long() + bs - 1) // bs
    nb_max = int(nbs.max()) if nbs.numel() else 0
    if width is None:
        width = topk if topk > 0 else nb_max
    q, k = to_dev(wl.q), to_dev(wl.k_cache)
    sel = torch.full((s.num_queries, wl.num_kv_heads, width), -9, dtype=torch.int32, device="cuda")
    sc = torch.full((s.num_queries, wl.num_kv_heads, nb_max), float("nan"), device="cuda") if with_scores else None
    pa.pa_sparse_select(plan, q, k, sel, wl.scale, bs, topk, wl.causal, wl.window, block_scores=sc)
    torch.cuda.synchronize()
    if own:
        plan.close()
    return (sc.cpu() if sc is not None else None), sel.cpu()


def gpu_sparse_forward(wl, bs, sel, plan=None, kv_chunk=0, path=pa.PA_PATH_AUTO):
    own = plan is None
    if own:
        plan = pa.plan_for(wl)
    q, k, v = to_dev(wl.q), to_dev(wl.k_cache), to_dev(wl.v_cache)
    out = torch.full((q.shape[0], wl.num_q_heads, wl.v_head_dim), float("nan"), dtype=q.dtype, device="cuda")
    lse = torch.full((q.shape[0], wl.num_q_heads), float("nan"), dtype=torch.float32, device="cuda")
    pa.pa_sparse_forward(plan, q, k, v, sel.to(torch.int32).cuda().contiguous(), out, lse, wl.scale, bs, wl.causal,
                         wl.window, kv_chunk=kv_chunk, path=path)
    torch.cuda.synchronize()
    status = pa.pa_plan_device_status(plan)
    if own:
        plan.close()
    return out.cpu(), lse.cpu(), status


def check_scores(sc, ref, tag):
    ninf = torch.isinf(ref) & (ref < 0)
    assert torch.equal(torch.isinf(sc) & (sc < 0), ninf), f"{tag}: -inf pattern differs"
    d = (sc.double()[~ninf] - ref[~ninf]).abs()
    tol = 1e-4 * (1 + ref[~ninf].abs())
    assert bool((d <= tol).all()), f"{tag}: score err {float(d.max()) if d.numel() else 0}"


def valid_topk(sel_row, scores_row, k, nb, eps=1e-3):
    """sel_row is a valid top-k of scores_row (fp64) within eps: ascending, distinct, k entries
    in range then -1, and no unselected block scores more than eps above a selected one."""
    got = [b for b in sel_row if b >= 0]
    if got != sorted(set(got)) or len(got) != k or any(b >= nb for b in got):
        return False
    if sel_row[len(got):] and any(b != -1 for b in sel_row[len(got):]):
        return False
    chosen = set(got)
    lo = min((float(scores_row[b]) for b in got), default=math.inf)
    hi = max((float(scores_row[b]) for b in range(nb) if b not in chosen), default=-math.inf)
    return hi <= lo + eps or (math.isinf(hi) and hi < 0)


def compare_selection(wl, bs, topk, sel, ref_scores, ref_sel, max_mismatch_frac=0.01):
    s = wl.sched
    rows = mism = 0
    for seq in range(s.num_seqs):
        nb = (int(s.seq_lens[seq]) + bs - 1) // bs
        k = nb if (topk == 0 or topk >= nb) else topk
        for qi in range(int(s.query_offsets[seq]), int(s.query_offsets[seq + 1])):
            for h in range(wl.num_kv_heads):
                rows += 1
                g, r = sel[qi, h].tolist(), ref_sel[qi, h].tolist()
                assert valid_topk(g, ref_scores[qi, h], k, nb), (seq, qi, h, g, r)
                if g != r:
                    mism += 1
                    sc = sorted((float(x) for x in ref_scores[qi, h, :nb]), reverse=True)
                    gap = sc[k - 1] - sc[k] if k < nb else math.inf
                    assert gap <= 1e-3, (seq, qi, h, g, r, gap)
    assert mism <= max_mismatch_frac * max(rows, 1), (mism, rows)
    return mism


def sparse_cases():
    return [
        ("bf16_decode_tc", W.make_gqa("sp1", 61, [300, 1000, 64, 17, 513], [1] * 5, 32, 8, 128, 128, 16,
                                      torch.bfloat16), 64, 4),
        ("bf16_decode_d64_g2", W.make_gqa("sp2", 62, [200, 777], [1, 1], 8, 4, 64, 64, 32, torch.bfloat16), 32, 3),
        ("f16_prefill_causal", W.make_gqa("sp3", 63, [150, 90], [20, 90], 8, 2, 64, 64, 16, torch.float16), 16, 2),
        ("fp32_window_simt", W.make_gqa("sp4", 64, [400, 120], [3, 1], 4, 2, 32, 48, 8, torch.float32,
                                        window=100), 16, 5),
        ("bf16_noncausal_g16", W.make_gqa("sp5", 65, [260], [2], 16, 1, 128, 128, 16, torch.bfloat16,
                                          causal=False), 32, 3),
        # 16 KV heads of 256-byte rows: the proxy pass on the tensor cores, warps over (head, keys)
        ("bf16_hkv16_mma_proxy", W.make_gqa("sp6", 67, [333, 70], [1, 1], 32, 16, 128, 128, 16,
                                            torch.bfloat16), 32, 3),
        # slots wider than one warp's 32 lanes x 64 bytes (16 KV heads of 512-byte float32 rows):
        # the proxy pass scores one (query, KV head) row per warp
        ("fp32_hkv16_row_proxy", W.make_gqa("sp8", 70, [200, 90], [1, 1], 16, 16, 128, 128, 16,
                                            torch.float32), 32, 3),
        # head dim 256: the tensor-core proxy with two fragment rows per piece
        ("bf16_d256_mma_proxy", W.make_gqa("sp9", 71, [300, 513], [1, 1], 16, 4, 256, 256, 16,
                                           torch.bfloat16), 64, 3),
        # rows of 80 bytes: the proxy pass's scalar kernel
        ("bf16_d40_scalar_proxy", W.make_gqa("sp7", 68, [150, 77], [1, 2], 4, 2, 40, 40, 16, torch.bfloat16),
         16, 2),
        # more than 256 blocks in a row, and k above 32: the top-K kernel's shared-memory sort (the
        # other cases take its warp-per-row form)
        ("bf16_313_blocks_sorted_topk", W.make_gqa("sp10", 72, [5000, 300], [1, 1], 8, 2, 64, 64, 16,
                                                   torch.bfloat16), 16, 5),
        ("bf16_k40_sorted_topk", W.make_gqa("sp11", 73, [3000, 800], [1, 1], 8, 2, 128, 128, 16, torch.bfloat16),
         32, 40),
        # 256-key blocks: eight 32-key pieces per KV head in the tensor-core proxy pass; 2048-key
        # blocks: beyond its 1024 keys, so the CUDA-core slot kernel scores them
        ("bf16_bs256_mma_proxy", W.make_gqa("sp12", 74, [3000, 700, 90], [1, 1, 1], 16, 4, 128, 128, 16,
                                            torch.bfloat16), 256, 3),
        ("bf16_bs2048_slot_proxy", W.make_gqa("sp13", 75, [5000, 300], [1, 1], 8, 2, 128, 128, 64, torch.bfloat16),
         2048, 1),
    ]


@pytest.mark.parametrize("name,wl,bs,topk", sparse_cases(), ids=[c[0] for c in sparse_cases()])
def test_select_scores_and_topk(orc, name, wl, bs, topk):
    sc, sel = gpu_select(wl, bs, topk)
    s = wl.sched
    ref_sc = orc.sparse_block_scores(wl.q, wl.k_cache, s.seq_lens, s.query_offsets, s.block_tables, s.page_size,
                                     wl.scale, bs, wl.causal, wl.window)
    check_scores(sc, ref_sc, name)
    ref_sel = orc.sparse_topk(ref_sc, s.seq_lens, s.query_offsets, bs, topk, width=sel.shape[2])
    compare_selection(wl, bs, topk, sel, ref_sc, ref_sel)


def test_select_more_rows_than_a_grid_dimension_holds(orc):
    """4200 queries x 16 KV heads = 67200 (query, KV head) rows, more than the 65535 a grid's second
    dimension holds (the proxy kernels put rows on the first): scores and selection against the
    oracle."""
    wl = W.make_gqa("rows", 69, [2200, 2150], [2100, 2100], 16, 16, 128, 128, 64, torch.bfloat16)
    s = wl.sched
    sc, sel = gpu_select(wl, 64, 4)
    ref_sc = orc.sparse_block_scores(wl.q, wl.k_cache, s.seq_lens, s.query_offsets, s.block_tables, s.page_size,
                                     wl.scale, 64, wl.causal, wl.window)
    check_scores(sc, ref_sc, "67200 rows")
    ref_sel = orc.sparse_topk(ref_sc, s.seq_lens, s.query_offsets, 64, 4, width=sel.shape[2])
    compare_selection(wl, 64, 4, sel, ref_sc, ref_sel)


@pytest.mark.parametrize("topk", [1, 3, 0])
def test_select_exact_on_integer_inputs(orc, topk):
    """Small-integer Q and K with scale 1/8: exact scores, so ties decide alike on both sides."""
    wl = W.make_gqa("ints", 66, [257, 96, 33], [1, 4, 1], 8, 2, 64, 64, 16, torch.bfloat16, scale=0.125, window=70)
    g = torch.Generator().manual_seed(3)
    wl.q.copy_(torch.randint(-1, 2, wl.q.shape, generator=g).to(torch.bfloat16))
    kk = torch.randint(-1, 2, wl.k_cache.shape, generator=g).to(torch.bfloat16)
    wl.k_cache.copy_(torch.where(torch.isnan(wl.k_cache), wl.k_cache, kk))
    sc, sel = gpu_select(wl, 16, topk)
    s = wl.sched
    ref_sc = orc.sparse_block_scores(wl.q, wl.k_cache, s.seq_lens, s.query_offsets, s.block_tables, s.page_size,
                                     wl.scale, 16, wl.causal, wl.window)
    assert torch.equal(sc.double(), ref_sc)
    ref_sel = orc.sparse_topk(ref_sc, s.seq_lens, s.query_offsets, 16, topk, width=sel.shape[2])
    assert torch.equal(sel, ref_sel)


@pytest.mark.parametrize("name,wl,bs,topk", sparse_cases(), ids=[c[0] for c in sparse_cases()])
def test_forward_with_oracle_selection(orc, name, wl, bs, topk):
    s = wl.sched
    ref_sc = orc.sparse_block_scores(wl.q, wl.k_cache, s.seq_lens, s.query_offsets, s.block_tables, s.page_size,
                                     wl.scale, bs, wl.causal, wl.window)
    ref_sel = orc.sparse_topk(ref_sc, s.seq_lens, s.query_offsets, bs, topk)
    out, lse, status = gpu_sparse_forward(wl, bs, ref_sel)
    assert status == 0
    ref_out, ref_lse = orc.sparse_attention(wl.q, wl.k_cache, wl.v_cache, s.seq_lens, s.query_offsets,
                                            s.block_tables, s.page_size, wl.scale, bs, ref_sel, wl.causal, wl.window)
    check(wl, out, lse, ref_out, ref_lse, tag=name)


def test_forward_selection_order_and_padding(orc):
    """Entries in any order with -1 gaps give the same result as the ascending selection."""
    name, wl, bs, topk = sparse_cases()[0]
    s = wl.sched
    ref_sc = orc.sparse_block_scores(wl.q, wl.k_cache, s.seq_lens, s.query_offsets, s.block_tables, s.page_size,
                                     wl.scale, bs, wl.causal, wl.window)
    ref_sel = orc.sparse_topk(ref_sc, s.seq_lens, s.query_offsets, bs, topk)
    shuffled = torch.full((ref_sel.shape[0], ref_sel.shape[1], 2 * topk + 1), -1, dtype=torch.int32)
    shuffled[:, :, 1::2] = ref_sel.flip(-1)
    out, lse, status = gpu_sparse_forward(wl, bs, shuffled)
    assert status == 0
    ref_out, ref_lse = orc.sparse_attention(wl.q, wl.k_cache, wl.v_cache, s.seq_lens, s.query_offsets,
                                            s.block_tables, s.page_size, wl.scale, bs, ref_sel, wl.causal, wl.window)
    check(wl, out, lse, ref_out, ref_lse, tag="shuffled")


def test_end_to_end_select_then_forward(orc):
    name, wl, bs, topk = sparse_cases()[0]
    plan = pa.plan_for(wl)
    _, sel = gpu_select(wl, bs, topk, plan=plan, with_scores=False)
    out, lse, status = gpu_sparse_forward(wl, bs, sel, plan=plan)
    plan.close()
    assert status == 0
    ref_sc, ref_sel, ref_out, ref_lse = orc.sparse(wl, bs, topk)
    compare_selection(wl, bs, topk, sel, ref_sc, ref_sel)
    G = wl.num_q_heads // wl.num_kv_heads
    same = [r for r in range(wl.sched.num_queries * wl.num_q_heads)
            if torch.equal(sel[r // wl.num_q_heads, (r % wl.num_q_heads) // G],
                           ref_sel[r // wl.num_q_heads, (r % wl.num_q_heads) // G])]
    check(wl, out, lse, ref_out, ref_lse, rows=same, tag="end-to-end")


@pytest.mark.parametrize("name,wl,bs,topk", sparse_cases()[:3], ids=[c[0] for c in sparse_cases()[:3]])
def test_topk_zero_is_dense(orc, name, wl, bs, topk):
    """Every block selected: the sparse path equals dense attention (and the dense GPU path)."""
    _, sel = gpu_select(wl, bs, 0, with_scores=False)
    out, lse, status = gpu_sparse_forward(wl, bs, sel)
    assert status == 0
    ref_out, ref_lse = orc.run(wl)
    check(wl, out, lse, ref_out, ref_lse, tag=name + " dense")


def test_empty_and_all_unused_selection(orc):
    """Width 0, or a row of -1 only, leaves no key: out = 0 and lse = -inf."""
    name, wl, bs, topk = sparse_cases()[1]
    for width in (0, 3):
        sel = torch.full((wl.sched.num_queries, wl.num_kv_heads, width), -1, dtype=torch.int32)
        out, lse, status = gpu_sparse_forward(wl, bs, sel)
        assert status == 0
        assert bool((out == 0).all()) and bool(torch.isinf(lse).all()) and bool((lse < 0).all())


def test_bad_selection_sets_device_error(orc):
    """An entry past the sequence's blocks, or a repeated block, is reported (code 64) and skipped."""
    name, wl, bs, topk = sparse_cases()[1]
    s = wl.sched
    nb0 = (int(s.seq_lens[0]) + bs - 1) // bs
    good = torch.tensor([[[0, 1, -1]] * wl.num_kv_heads] * s.num_queries, dtype=torch.int32)
    _, _, status = gpu_sparse_forward(wl, bs, good)
    assert status == 0
    for bad_entry in ([nb0, 0, 1], [1, 1, 0], [-5, 0, 1]):
        bad = good.clone()
        bad[0, 0] = torch.tensor(bad_entry, dtype=torch.int32)
        out, lse, status = gpu_sparse_forward(wl, bs, bad)
        assert status == 64, (bad_entry, status)
        assert bool(torch.isfinite(out).all())


def test_full_size_sparse_decode_sampled(orc):
    """The benchmarked configuration (64 decode sequences, context U[512, 8192], blocks of 64,
    top-16) in the bench's launch configuration, on sampled rows."""
    wl, bs, topk = W.sparse_bf16_decode(0)
    plan = pa.plan_for(wl)
    _, sel = gpu_select(wl, bs, topk, plan=plan, with_scores=False)
    out, lse, status = gpu_sparse_forward(wl, bs, sel, plan=plan)
    plan.close()
    assert status == 0
    s = wl.sched
    ref_sc = orc.sparse_block_scores(wl.q, wl.k_cache, s.seq_lens, s.query_offsets, s.block_tables, s.page_size,
                                     wl.scale, bs, wl.causal, wl.window)
    ref_sel = orc.sparse_topk(ref_sc, s.seq_lens, s.query_offsets, bs, topk)
    compare_selection(wl, bs, topk, sel, ref_sc, ref_sel)
    rows = sample_rows(wl, 256, seed=7)
    G = wl.num_q_heads // wl.num_kv_heads
    rows = [r for r in rows if torch.equal(sel[r // wl.num_q_heads, (r % wl.num_q_heads) // G],
                                           ref_sel[r // wl.num_q_heads, (r % wl.num_q_heads) // G])]
    ref_out, ref_lse = orc.sparse_attention(wl.q, wl.k_cache, wl.v_cache, s.seq_lens, s.query_offsets,
                                            s.block_tables, s.page_size, wl.scale, bs, ref_sel, wl.causal, wl.window,
                                            rows=rows)
    check(wl, out, lse, ref_out, ref_lse, rows=rows, tag="full-size sparse")


@pytest.mark.parametrize("kv_chunk,path", [(-1, pa.PA_PATH_AUTO), (16, pa.PA_PATH_AUTO), (40, pa.PA_PATH_AUTO),
                                           (0, pa.PA_PATH_SIMT), (24, pa.PA_PATH_SIMT)])
def test_forward_split_and_path(orc, kv_chunk, path):
    """Any split of the selected keys into parts (rounded to 16 keys), and the CUDA-core path."""
    name, wl, bs, topk = sparse_cases()[0]
    s = wl.sched
    ref_sc = orc.sparse_block_scores(wl.q, wl.k_cache, s.seq_lens, s.query_offsets, s.block_tables, s.page_size,
                                     wl.scale, bs, wl.causal, wl.window)
    ref_sel = orc.sparse_topk(ref_sc, s.seq_lens, s.query_offsets, bs, topk)
    out, lse, status = gpu_sparse_forward(wl, bs, ref_sel, kv_chunk=kv_chunk, path=path)
    assert status == 0
    ref_out, ref_lse = orc.sparse_attention(wl.q, wl.k_cache, wl.v_cache, s.seq_lens, s.query_offsets,
                                            s.block_tables, s.page_size, wl.scale, bs, ref_sel, wl.causal, wl.window)
    check(wl, out, lse, ref_out, ref_lse, tag=f"chunk {kv_chunk} path {path}")
