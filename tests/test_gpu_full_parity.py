"""Whole-batch parity of the full-size configurations: every (query, head) row of the benchmarked
batches compared with the fp64 oracle, which runs on all host cores, in the launch configuration
bench.py times (automatic split sizes, default path).

  tiny fp32 decode            2 sequences, Hq 4 / Hkv 2, D 64, pages of 16
  bf16 decode (the headline)  64 sequences, context U[512, 8192], Hq 32 / Hkv 8, D 128, pages of 16
  chunked prefill             8 x (history U[0, 4096] + 512 queries), Hq 32 / Hkv 8, D 128, pages of 64
  chunked prefill, D 256      the same batch at head size 256 (64-key tiles)
  window + mixed              16 decode rows at 32768 + 4 x (8192 + 1024), window 4096, Hq 64 / Hkv 8
  MLA decode                  32 sequences, context U[1024, 16384], 128 heads, latent 512, rope 64
  sparse top-K decode         the bf16 decode batch, blocks of 64 keys, top 16

The sampled-row tests elsewhere check the same batches on a few hundred rows; these check all of
them (minutes of oracle time on the host cores in total).
"""
import pytest
import torch

import paged_kv_attention_39_b200 as pa
from paged_kv_attention_39_b200 import workloads as W
from gpu_helpers import check, run_gqa, run_mla
from test_gpu_sparse import compare_selection, gpu_select, gpu_sparse_forward

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def whole(orc, wl, tag):
    out, lse = run_mla(wl) if wl.kind == "mla" else run_gqa(wl)
    ref_out, ref_lse = orc.run(wl)
    check(wl, out, lse, ref_out, ref_lse, tag=tag)


def test_tiny_fp32_decode_whole_batch(orc):
    whole(orc, W.c1_tiny_fp32_decode(0), "C1 tiny fp32 decode")


def test_bf16_decode_whole_batch(orc):
    whole(orc, W.c2_bf16_decode(0), "C2 bf16 decode")


def test_chunked_prefill_whole_batch(orc):
    whole(orc, W.c3_chunked_prefill(0), "C3 chunked prefill")


def test_chunked_prefill_d256_whole_batch(orc):
    whole(orc, W.c3_prefill_variant(0, torch.bfloat16, 256), "C3 chunked prefill D256")


def test_window_mixed_whole_batch(orc):
    whole(orc, W.c4_window_mixed(0), "C4 window + mixed")


def test_mla_decode_whole_batch(orc):
    whole(orc, W.c5_mla_decode(0), "C5 MLA decode")


def test_sparse_topk_decode_whole_batch(orc):
    """The GPU's selection must be a valid top-k of the oracle's proxy scores on every row (equal
    wherever the k-th and (k+1)-th scores are apart); attention over the oracle's selection must
    match the oracle on every row."""
    wl, bs, topk = W.sparse_bf16_decode(0)
    s = wl.sched
    plan = pa.plan_for(wl)
    _, sel = gpu_select(wl, bs, topk, plan=plan, with_scores=False)
    ref_sc = orc.sparse_block_scores(wl.q, wl.k_cache, s.seq_lens, s.query_offsets, s.block_tables, s.page_size,
                                     wl.scale, bs, wl.causal, wl.window)
    ref_sel = orc.sparse_topk(ref_sc, s.seq_lens, s.query_offsets, bs, topk)
    compare_selection(wl, bs, topk, sel, ref_sc, ref_sel)
    out, lse, status = gpu_sparse_forward(wl, bs, ref_sel, plan=plan)
    plan.close()
    assert status == 0
    ref_out, ref_lse = orc.sparse_attention(wl.q, wl.k_cache, wl.v_cache, s.seq_lens, s.query_offsets,
                                            s.block_tables, s.page_size, wl.scale, bs, ref_sel, wl.causal,
                                            wl.window)
    check(wl, out, lse, ref_out, ref_lse, tag="sparse top-16 decode")
