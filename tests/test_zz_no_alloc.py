"""pa_forward_static_workspace: the split-KV decode entry point that allocates nothing.

It is for callers that cannot allocate device memory while attention runs (a decode loop that
must not stall on the allocator, a fixed memory budget, a host runtime that forbids cudaMalloc
in plugins). It keeps its work list and split parts in the library's fixed device array and
must give the same results as pa_forward, and both must match the fp64 oracle.

The file name sorts last on purpose, so that a run stopping at its first failure has already
run every other test when one of these fails. Nothing here depends on that order: each test
builds its own plans and inputs, and each passes alone in a fresh process as well.
"""
import pytest
import torch

import paged_kv_attention_39_b200 as pa
from paged_kv_attention_39_b200 import workloads as W
from gpu_helpers import check

pytestmark = pytest.mark.gpu


def decode_batch(seed, hq=32, hkv=8, d=128, dtype=torch.bfloat16, lmin=300, lmax=6000, batch=24, qn=1, window=0):
    lens = W._uniform_ints(seed, 123, batch, lmin, lmax)
    return W.make_gqa("noalloc", seed, lens, [qn] * batch, hq, hkv, d, d, 16, dtype, window=window)


def run_both(wl, kv_chunk):
    """pa_forward and the fixed-workspace call on the same plan and inputs."""
    q, k, v = wl.q.cuda(), wl.k_cache.cuda(), wl.v_cache.cuda()
    nq, hq, _ = q.shape
    plan = pa.plan_for(wl)
    ref_o = torch.empty(nq, hq, wl.v_head_dim, dtype=q.dtype, device="cuda")
    ref_l = torch.empty(nq, hq, dtype=torch.float32, device="cuda")
    got_o = torch.full_like(ref_o, float("nan"))
    got_l = torch.full_like(ref_l, float("nan"))
    before = pa.pa_plan_get_info(plan)
    pa.pa_forward_static_workspace(plan, q, k, v, got_o, got_l, wl.scale, wl.causal, wl.window, kv_chunk=kv_chunk)
    torch.cuda.synchronize()
    after = pa.pa_plan_get_info(plan)
    # the plan gained no workspace and uploaded nothing: the call used the fixed array only
    assert after["workspace_bytes"] == 0 and after["uploaded_bytes"] == before["uploaded_bytes"]
    pa.pa_forward(plan, q, k, v, ref_o, ref_l, wl.scale, wl.causal, wl.window, kv_chunk=kv_chunk)
    torch.cuda.synchronize()
    assert pa.pa_plan_device_status(plan) == 0
    plan.close()
    return got_o.cpu(), got_l.cpu(), ref_o.cpu(), ref_l.cpu()


def close(got_o, got_l, ref_o, ref_l):
    o, r = got_o.double(), ref_o.double()
    assert torch.isfinite(o).all() and torch.isfinite(got_l).all()
    assert not bool(((o - r).abs() > 1e-2 + 2e-2 * r.abs()).any()), float((o - r).abs().max())
    assert float((got_l - ref_l).abs().max()) <= 2e-3


def both_and_oracle(orc, wl, kv_chunk, tag):
    got_o, got_l, ref_o, ref_l = run_both(wl, kv_chunk)
    close(got_o, got_l, ref_o, ref_l)
    oo, ol = orc.run(wl)
    check(wl, got_o, got_l, oo, ol, tag=tag + " (fixed workspace vs oracle)")
    check(wl, ref_o, ref_l, oo, ol, tag=tag + " (pa_forward vs oracle)")


def test_two_calls_in_a_row_match_pa_forward_and_the_oracle(orc):
    # first call: splits across CTAs; second call: another batch and split size, so that any
    # state the first call left in the shared array would show
    wl1 = decode_batch(1)
    both_and_oracle(orc, wl1, 0, "first call")
    wl2 = decode_batch(2, hq=16, hkv=4, d=64, dtype=torch.float16, lmin=17, lmax=2500, batch=40, qn=2, window=700)
    both_and_oracle(orc, wl2, 96, "second call")


def test_unsplit_and_forced_split_match(orc):
    wl = decode_batch(3, batch=8)
    for kv_chunk in (-1, 64):
        both_and_oracle(orc, wl, kv_chunk, f"kv_chunk {kv_chunk}")


def test_more_than_1024_parts_requested_are_capped(orc):
    # 16 keys per part on a 32768-key context asks for 2048 parts; the merge kernel takes 1024
    # per row, so the call (like pa_forward) cuts 1024 parts of 32 keys instead
    wl = W.make_gqa("noalloc_cap", 6, [32768, 900], [1, 1], 4, 4, 64, 64, 16, torch.bfloat16)
    both_and_oracle(orc, wl, 16, "capped parts")


def test_rejects_batches_beyond_the_fixed_size():
    wl = decode_batch(4, batch=64, lmin=8000, lmax=8192)
    q, k, v = wl.q.cuda(), wl.k_cache.cuda(), wl.v_cache.cuda()
    plan = pa.plan_for(wl)
    o = torch.empty(q.shape, dtype=q.dtype, device="cuda")
    l = torch.empty(q.shape[:2], dtype=torch.float32, device="cuda")
    # 16 keys per part -> ~500 parts per sequence: far more split parts than the array holds
    with pytest.raises(pa.PaError) as ei:
        pa.pa_forward_static_workspace(plan, q, k, v, o, l, wl.scale, kv_chunk=16)
    assert ei.value.name == "PA_ERR_BOUNDS" and "split parts" in str(ei.value)
    # unsupported shapes are refused, not approximated
    wf = decode_batch(5, dtype=torch.float32, batch=2)
    pf = pa.plan_for(wf)
    of = torch.empty(wf.q.shape, dtype=torch.float32, device="cuda")
    lf = torch.empty(wf.q.shape[:2], dtype=torch.float32, device="cuda")
    with pytest.raises(pa.PaError) as ei:
        pa.pa_forward_static_workspace(pf, wf.q.cuda(), wf.k_cache.cuda(), wf.v_cache.cuda(), of, lf, wf.scale)
    assert ei.value.name == "PA_ERR_UNSUPPORTED"
    plan.close(); pf.close()


def _refused(wl, kv_chunk):
    q, k, v = wl.q.cuda(), wl.k_cache.cuda(), wl.v_cache.cuda()
    plan = pa.plan_for(wl)
    o = torch.full((q.shape[0], q.shape[1], wl.v_head_dim), 7.0, dtype=q.dtype, device="cuda")
    l = torch.full(q.shape[:2], 7.0, dtype=torch.float32, device="cuda")
    with pytest.raises(pa.PaError) as ei:
        pa.pa_forward_static_workspace(plan, q, k, v, o, l, wl.scale, wl.causal, wl.window, kv_chunk=kv_chunk)
    torch.cuda.synchronize()
    # refused before any launch: the outputs are untouched
    assert bool((o == 7.0).all()) and bool((l == 7.0).all())
    plan.close()
    return ei.value


def test_rejects_more_work_units_than_the_array_holds():
    # 33000 one-query sequences, never split: one work unit each, above the 32768 the array holds
    wl = W.make_gqa("noalloc_units", 7, [16] * 33000, [1] * 33000, 1, 1, 64, 64, 16, torch.bfloat16)
    err = _refused(wl, -1)
    assert err.name == "PA_ERR_BOUNDS" and "work units" in str(err)


def test_rejects_more_split_rows_than_the_array_holds():
    # 1100 sequences x 16 queries (G = 1), 64 keys cut into 2 parts: 17600 split query rows to
    # merge, above the 16384 merge units the array holds (the parts themselves would fit)
    wl = W.make_gqa("noalloc_merge", 8, [64] * 1100, [16] * 1100, 1, 1, 64, 64, 16, torch.bfloat16)
    err = _refused(wl, 32)
    assert err.name == "PA_ERR_BOUNDS" and "merge units" in str(err)
