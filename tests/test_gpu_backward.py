"""GPU backward against the fp64 oracle's backward: the tensor-core path (bf16 / fp16, D in {64, 128},
G dividing 128; deterministic dK/dV) and the float32 CUDA-core kernel (other shapes)."""
import pytest
import torch

import paged_kv_attention_39_b200 as pa
from paged_kv_attention_39_b200 import workloads as W

pytestmark = pytest.mark.gpu


def run_backward(wl, g):
    s = wl.sched
    q, k, v = wl.q.cuda(), wl.k_cache.cuda(), wl.v_cache.cuda()
    nq, hq, d = q.shape
    dout = torch.randn(nq, hq, wl.v_head_dim, generator=g).to(q.dtype)
    plan = pa.plan_for(wl)
    out = torch.empty(nq, hq, wl.v_head_dim, dtype=q.dtype, device="cuda")
    lse = torch.empty(nq, hq, dtype=torch.float32, device="cuda")
    pa.pa_forward(plan, q, k, v, out, lse, wl.scale, wl.causal, wl.window)
    dq = torch.full((nq, hq, d), float("nan"), dtype=torch.float32, device="cuda")
    dk = torch.zeros(k.shape, dtype=torch.float32, device="cuda")
    dv = torch.zeros(v.shape, dtype=torch.float32, device="cuda")
    pa.pa_backward(plan, q, k, v, out, lse, dout.cuda(), dq, dk, dv, wl.scale, wl.causal, wl.window)
    torch.cuda.synchronize()
    plan.close()
    return dout, dq.cpu(), dk.cpu(), dv.cpu()


# Tolerances. float32: the CUDA-core kernel computes in float32 throughout (1e-4 of the largest
# gradient element). bf16 / fp16: the tensor-core path rounds P and dS to the 16-bit input type
# before the dV, dK and dQ products (as the forward rounds P before P V). With unit roundoff u
# (2^-8 bf16, 2^-11 fp16) an element summed over N keys is off by about u * sqrt(N) * |term|,
# which does not shrink where the terms cancel, so the bound is set against the largest element:
# an fp64 emulation of exactly that rounding on the 1000-key shape below gives 0.34 % of the
# largest |dQ|; the bounds leave about three times that.
TOL_MAX = {torch.bfloat16: 1e-2, torch.float16: 2.5e-3}
TOL_REL = {torch.bfloat16: 2e-2, torch.float16: 1e-2}


def close(got, ref, dtype, tag):
    got, ref = got.double(), ref.double()
    owned = torch.isfinite(ref)
    scale = float(ref[owned].abs().max())
    if dtype == torch.float32:
        tol = 1e-4 * scale
        assert float((got - ref)[owned].abs().max()) <= tol, (tag, float((got - ref)[owned].abs().max()), tol)
    else:
        bad = (got - ref).abs() > TOL_MAX[dtype] * scale + TOL_REL[dtype] * ref.abs()
        assert not bool(bad[owned].any()), (tag, float((got - ref)[owned].abs().max()), scale)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("causal,window", [(True, 0), (True, 33), (False, 0)])
def test_backward_matches_oracle(orc, dtype, causal, window):
    wl = W.make_gqa("bwd", 3, [70, 130, 9, 200], [1, 40, 9, 3], 8, 2, 64, 64, 16, dtype, causal=causal,
                    window=window)
    g = torch.Generator().manual_seed(7)
    dout, dq, dk, dv = run_backward(wl, g)
    s = wl.sched
    rq, rk, rv = orc.attention_backward(wl.q, wl.k_cache, wl.v_cache, dout, s.seq_lens, s.query_offsets,
                                        s.block_tables, s.page_size, wl.scale, causal, window)
    close(dq, rq, dtype, "dq")
    close(dk, rk, dtype, "dk")
    close(dv, rv, dtype, "dv")


def test_backward_shared_prefix_page_accumulates(orc):
    """Two sequences whose tables share their first pages: the shared slots get both gradients."""
    wl = W.make_gqa("share", 4, [40, 40], [2, 2], 4, 2, 64, 64, 16, torch.float32)
    s = wl.sched
    s.block_tables[1, :2] = s.block_tables[0, :2]  # keys 0..31 shared
    g = torch.Generator().manual_seed(8)
    dout, dq, dk, dv = run_backward(wl, g)
    rq, rk, rv = orc.attention_backward(wl.q, wl.k_cache, wl.v_cache, dout, s.seq_lens, s.query_offsets,
                                        s.block_tables, 16, wl.scale, True, 0)
    close(dq, rq, torch.float32, "dq")
    close(dk, rk, torch.float32, "dk")
    close(dv, rv, torch.float32, "dv")


@pytest.mark.parametrize("hq,hkv,d,ps,causal,window,dtype", [
    (32, 8, 128, 64, True, 0, torch.bfloat16),
    (16, 16, 128, 16, True, 0, torch.float16),   # one head per group
    (16, 1, 64, 32, True, 100, torch.bfloat16),  # sixteen heads per group, window
    (8, 2, 128, 16, False, 0, torch.bfloat16),
    (8, 4, 64, 128, True, 0, torch.float16),
    (32, 1, 64, 16, True, 0, torch.bfloat16),   # 32 heads per group: 4 queries per 128-row block
    (8, 2, 128, 256, True, 0, torch.bfloat16),  # pages longer than a key tile: boxes inside a page
])
def test_backward_tensor_core_shapes(orc, hq, hkv, d, ps, causal, window, dtype):
    """The tensor-core backward (key-major dK/dV, query-major dQ, both on tcgen05): chunked prefills
    with history, a prefill from empty history, many 128-key tiles and 128-row blocks, ragged ends."""
    wl = W.make_gqa("bwd_tc", 5, [300, 513, 64, 1000], [100, 200, 64, 17], hq, hkv, d, d, ps, dtype,
                    causal=causal, window=window)
    g = torch.Generator().manual_seed(11)
    dout, dq, dk, dv = run_backward(wl, g)
    s = wl.sched
    rq, rk, rv = orc.attention_backward(wl.q, wl.k_cache, wl.v_cache, dout, s.seq_lens, s.query_offsets,
                                        s.block_tables, s.page_size, wl.scale, causal, window)
    tag = f"hq{hq} hkv{hkv} d{d} ps{ps} c{causal} w{window}"
    close(dq, rq, dtype, "dq " + tag)
    close(dk, rk, dtype, "dk " + tag)
    close(dv, rv, dtype, "dv " + tag)


@pytest.mark.parametrize("name,hq,hkv,d,dv,ps,dtype,path", [
    ("d256", 16, 4, 256, 256, 16, torch.bfloat16, "simt"),         # head dim beyond the tensor-core kernels
    ("d192v128", 8, 2, 192, 128, 16, torch.bfloat16, "simt"),      # key and value widths differ
    ("d512f32", 8, 2, 512, 512, 16, torch.float32, "simt"),        # float32, wide rows
    ("g128", 128, 1, 128, 128, 64, torch.bfloat16, "tc"),          # 128 heads on one KV head: one query per block
])
def test_backward_limits(orc, name, hq, hkv, d, dv, ps, dtype, path):
    """The backward at the edges of its shapes, each against the oracle, on the kernel the shape is
    meant for (the CUDA-core kernel for head dims outside {64, 128}, unequal widths and float32; the
    tensor-core kernels for a 128-head group)."""
    wl = W.make_gqa("bwd_lim_" + name, 71, [300, 45, 700], [60, 9, 3], hq, hkv, d, dv, ps, dtype)
    s = wl.sched
    g = torch.Generator().manual_seed(17)
    q, k, v = wl.q.cuda(), wl.k_cache.cuda(), wl.v_cache.cuda()
    nq = q.shape[0]
    dout = torch.randn(nq, hq, dv, generator=g).to(dtype)
    plan = pa.plan_for(wl)
    out = torch.empty(nq, hq, dv, dtype=dtype, device="cuda")
    lse = torch.empty(nq, hq, dtype=torch.float32, device="cuda")
    pa.pa_forward(plan, q, k, v, out, lse, wl.scale, True, 0)
    dq = torch.full((nq, hq, d), float("nan"), dtype=torch.float32, device="cuda")
    dk = torch.zeros(k.shape, dtype=torch.float32, device="cuda")
    dv_ = torch.zeros(v.shape, dtype=torch.float32, device="cuda")
    pa.pa_backward(plan, q, k, v, out, lse, dout.cuda(), dq, dk, dv_, wl.scale, True, 0)
    kernels = pa.pa_plan_get_info(plan)["last_kernels"]
    torch.cuda.synchronize()
    plan.close()
    expect = pa.PA_KERNEL_BACKWARD_SIMT if path == "simt" else pa.PA_KERNEL_BACKWARD_TC
    assert kernels == expect, (name, kernels)
    rq, rk, rv = orc.attention_backward(wl.q, wl.k_cache, wl.v_cache, dout, s.seq_lens, s.query_offsets,
                                        s.block_tables, ps, wl.scale, True, 0)
    close(dq.cpu(), rq, dtype, "dq " + name)
    close(dk.cpu(), rk, dtype, "dk " + name)
    close(dv_.cpu(), rv, dtype, "dv " + name)


def test_backward_page_size_outside_the_box_layout_runs_the_cuda_core_kernel(orc):
    """A page of 48 rows neither divides the 128-key tile nor is a multiple of it, so the tensor-core
    kernels (one TMA box per page) do not take it: the CUDA-core kernel does, and matches."""
    wl = W.make_gqa("bwd_ps48", 9, [300, 100], [40, 5], 8, 2, 64, 64, 48, torch.bfloat16)
    g = torch.Generator().manual_seed(13)
    s = wl.sched
    q, k, v = wl.q.cuda(), wl.k_cache.cuda(), wl.v_cache.cuda()
    nq, hq, d = q.shape
    dout = torch.randn(nq, hq, d, generator=g).to(q.dtype)
    plan = pa.plan_for(wl)
    out = torch.empty(nq, hq, d, dtype=q.dtype, device="cuda")
    lse = torch.empty(nq, hq, dtype=torch.float32, device="cuda")
    pa.pa_forward(plan, q, k, v, out, lse, wl.scale, True, 0)
    dq = torch.empty((nq, hq, d), dtype=torch.float32, device="cuda")
    dk = torch.zeros(k.shape, dtype=torch.float32, device="cuda")
    dv = torch.zeros(v.shape, dtype=torch.float32, device="cuda")
    pa.pa_backward(plan, q, k, v, out, lse, dout.cuda(), dq, dk, dv, wl.scale, True, 0)
    assert pa.pa_plan_get_info(plan)["last_kernels"] == pa.PA_KERNEL_BACKWARD_SIMT
    torch.cuda.synchronize()
    plan.close()
    rq, rk, rv = orc.attention_backward(wl.q, wl.k_cache, wl.v_cache, dout, s.seq_lens, s.query_offsets,
                                        s.block_tables, 48, wl.scale, True, 0)
    close(dq.cpu(), rq, torch.bfloat16, "dq")
    close(dk.cpu(), rk, torch.bfloat16, "dk")
    close(dv.cpu(), rv, torch.bfloat16, "dv")


def test_backward_tensor_core_shared_pages_and_launches(orc):
    """bf16 on the tensor-core path with two sequences sharing their first pages: the key tiles that
    touch the shared pages hand their rows to the ordered pass, which adds each shared slot's rows
    in sequence order, so the shared slots receive both sequences' gradients. The path runs four
    kernels (Drow, dK/dV, the ordered pass, dQ)."""
    wl = W.make_gqa("share_tc", 6, [150, 150], [30, 30], 8, 2, 64, 64, 16, torch.bfloat16)
    s = wl.sched
    s.block_tables[1, :3] = s.block_tables[0, :3]  # keys 0..47 shared
    g = torch.Generator().manual_seed(12)
    q, k, v = wl.q.cuda(), wl.k_cache.cuda(), wl.v_cache.cuda()
    nq, hq, d = q.shape
    dout = torch.randn(nq, hq, d, generator=g).to(q.dtype)
    plan = pa.plan_for(wl)
    out = torch.empty(nq, hq, d, dtype=q.dtype, device="cuda")
    lse = torch.empty(nq, hq, dtype=torch.float32, device="cuda")
    pa.pa_forward(plan, q, k, v, out, lse, wl.scale, True, 0)
    dq = torch.empty((nq, hq, d), dtype=torch.float32, device="cuda")
    dk = torch.zeros(k.shape, dtype=torch.float32, device="cuda")
    dv = torch.zeros(v.shape, dtype=torch.float32, device="cuda")
    pa.pa_backward(plan, q, k, v, out, lse, dout.cuda(), dq, dk, dv, wl.scale, True, 0)
    assert pa.pa_plan_get_info(plan)["last_launches"] == 4
    torch.cuda.synchronize()
    plan.close()
    rq, rk, rv = orc.attention_backward(wl.q, wl.k_cache, wl.v_cache, dout, s.seq_lens, s.query_offsets,
                                        s.block_tables, 16, wl.scale, True, 0)
    close(dq.cpu(), rq, torch.bfloat16, "dq")
    close(dk.cpu(), rk, torch.bfloat16, "dk")
    close(dv.cpu(), rv, torch.bfloat16, "dv")


@pytest.mark.parametrize("ps,shared_pages", [(16, 5), (64, 2), (128, 1)])
def test_backward_tensor_core_shared_pages_same_bits(orc, ps, shared_pages):
    """Three sequences share a prefix of pages (a common prompt) and one more lists a page twice:
    every shared cache slot is summed by the ordered pass in sequence order, so two runs give the
    same bits, and the gradients match the oracle."""
    wl = W.make_gqa("share_bits", 8, [400, 260, 333, 200], [60, 130, 1, 40], 16, 4, 128, 128, ps, torch.bfloat16)
    s = wl.sched
    for j in (1, 2):
        s.block_tables[j, :shared_pages] = s.block_tables[0, :shared_pages]
    used = (200 + ps - 1) // ps
    if used >= 2:
        s.block_tables[3, used - 1] = s.block_tables[3, 0]  # keys of its first and last page share slots
    runs = [run_backward(wl, torch.Generator().manual_seed(21)) for _ in range(2)]
    for a, b in zip(runs[0][1:], runs[1][1:]):
        assert torch.equal(torch.nan_to_num(a, nan=0.0), torch.nan_to_num(b, nan=0.0))
    dout, dq, dk, dv = runs[0]
    rq, rk, rv = orc.attention_backward(wl.q, wl.k_cache, wl.v_cache, dout, s.seq_lens, s.query_offsets,
                                        s.block_tables, ps, wl.scale, True, 0)
    close(dq, rq, torch.bfloat16, f"dq ps{ps}")
    close(dk, rk, torch.bfloat16, f"dk ps{ps}")
    close(dv, rv, torch.bfloat16, f"dv ps{ps}")


def test_backward_tensor_core_deterministic():
    """Without shared pages every gradient element is summed by one CTA in a fixed order: two runs
    give the same bits."""
    wl = W.make_gqa("det", 7, [400, 260], [60, 260], 16, 4, 128, 128, 64, torch.bfloat16)
    runs = [run_backward(wl, torch.Generator().manual_seed(13)) for _ in range(2)]
    for a, b in zip(runs[0][1:], runs[1][1:]):
        assert torch.equal(torch.nan_to_num(a, nan=0.0), torch.nan_to_num(b, nan=0.0))


@pytest.mark.parametrize("h,r,pr,ps,dtype,causal,window", [
    (8, 64, 16, 16, torch.float32, True, 0),
    (16, 512, 64, 64, torch.bfloat16, True, 0),
    (4, 96, 32, 32, torch.float16, True, 40),
    (8, 128, 64, 16, torch.bfloat16, False, 0),
])
def test_mla_backward_matches_oracle(orc, h, r, pr, ps, dtype, causal, window):
    """pa_mla_backward against the oracle (the GQA backward on the key [latent | rope] with the latent
    as value, the latent's key and value gradients summed), decode and chunked rows, ragged pages."""
    wl = W.make_mla("mla_bwd", 9, [70, 200, 9, 130], [1, 40, 9, 3], h, r, pr, ps, dtype, causal=causal,
                    window=window)
    s = wl.sched
    g = torch.Generator().manual_seed(15)
    nq = s.num_queries
    dout = torch.randn(nq, h, r, generator=g).to(dtype)
    ql, qr = wl.q_latent.cuda(), wl.q_rope.cuda()
    lat, rope = wl.latent_cache.cuda(), wl.rope_cache.cuda()
    plan = pa.plan_for(wl)
    out = torch.empty(nq, h, r, dtype=dtype, device="cuda")
    lse = torch.empty(nq, h, dtype=torch.float32, device="cuda")
    pa.pa_mla_forward(plan, ql, qr, lat, rope, out, lse, wl.scale, causal, window)
    dql = torch.full((nq, h, r), float("nan"), dtype=torch.float32, device="cuda")
    dqr = torch.full((nq, h, pr), float("nan"), dtype=torch.float32, device="cuda")
    dlat = torch.zeros(lat.shape, dtype=torch.float32, device="cuda")
    drope = torch.zeros(rope.shape, dtype=torch.float32, device="cuda")
    pa.pa_mla_backward(plan, ql, qr, lat, rope, out, lse, dout.cuda(), dql, dqr, dlat, drope, wl.scale, causal,
                       window)
    torch.cuda.synchronize()
    assert pa.pa_plan_device_status(plan) == 0
    plan.close()
    ref = orc.mla_backward(wl.q_latent, wl.q_rope, wl.latent_cache, wl.rope_cache, dout, s.seq_lens,
                           s.query_offsets, s.block_tables, ps, wl.scale, causal, window)
    tag = f"mla h{h} r{r} pr{pr} {dtype}"
    for got, want, name in zip((dql, dqr, dlat, drope), ref, ("dq_latent", "dq_rope", "d_latent", "d_rope")):
        close(got.cpu(), want, dtype, f"{name} {tag}")


def _mla_backward_run(wl, causal, window, seed):
    s = wl.sched
    g = torch.Generator().manual_seed(seed)
    nq, h, r, pr = s.num_queries, wl.num_heads, wl.latent_dim, wl.rope_dim
    dtype = wl.q_latent.dtype
    dout = torch.randn(nq, h, r, generator=g).to(dtype)
    ql, qr = wl.q_latent.cuda(), wl.q_rope.cuda()
    lat, rope = wl.latent_cache.cuda(), wl.rope_cache.cuda()
    plan = pa.plan_for(wl)
    out = torch.empty(nq, h, r, dtype=dtype, device="cuda")
    lse = torch.empty(nq, h, dtype=torch.float32, device="cuda")
    pa.pa_mla_forward(plan, ql, qr, lat, rope, out, lse, wl.scale, causal, window)
    dql = torch.full((nq, h, r), float("nan"), dtype=torch.float32, device="cuda")
    dqr = torch.full((nq, h, pr), float("nan"), dtype=torch.float32, device="cuda")
    dlat = torch.zeros(lat.shape, dtype=torch.float32, device="cuda")
    drope = torch.zeros(rope.shape, dtype=torch.float32, device="cuda")
    pa.pa_mla_backward(plan, ql, qr, lat, rope, out, lse, dout.cuda(), dql, dqr, dlat, drope, wl.scale, causal,
                       window)
    torch.cuda.synchronize()
    assert pa.pa_plan_device_status(plan) == 0
    kernels = pa.pa_plan_get_info(plan)["last_kernels"]
    plan.close()
    return dout, (dql.cpu(), dqr.cpu(), dlat.cpu(), drope.cpu()), kernels


@pytest.mark.parametrize("h,lens,qs,ps,dtype,causal,window", [
    (128, [700, 2000, 130, 4100], [1, 1, 1, 1], 64, torch.bfloat16, True, 0),   # decode, many key tiles
    (16, [300, 513, 64, 1000], [8, 3, 1, 5], 16, torch.float16, True, 300),     # 16 heads x up to 8 queries, window
    (128, [90, 1500, 257], [1, 1, 1], 128, torch.bfloat16, False, 0),           # a tile shorter than 128 keys
    (64, [1024, 777], [2, 1], 32, torch.bfloat16, True, 0),                     # 2 queries x 64 heads = 128 rows
])
def test_mla_backward_tensor_core(orc, h, lens, qs, ps, dtype, causal, window):
    """The tensor-core MLA backward (latent 512, rope 64, every sequence's rows within one block of
    128): key tiles in CTA pairs over the latent's column halves, dQ per 64-column chunk; against the
    oracle, and on the tensor-core path."""
    wl = W.make_mla("mla_bwd_tc", 19, lens, qs, h, 512, 64, ps, dtype, causal=causal, window=window)
    dout, got, kernels = _mla_backward_run(wl, causal, window, 21)
    assert kernels == pa.PA_KERNEL_BACKWARD_TC, kernels
    s = wl.sched
    ref = orc.mla_backward(wl.q_latent, wl.q_rope, wl.latent_cache, wl.rope_cache, dout, s.seq_lens,
                           s.query_offsets, s.block_tables, ps, wl.scale, causal, window)
    tag = f"mla tc h{h} ps{ps} {dtype} c{causal} w{window}"
    for g, want, name in zip(got, ref, ("dq_latent", "dq_rope", "d_latent", "d_rope")):
        close(g, want, dtype, f"{name} {tag}")


def test_mla_backward_shared_pages_take_the_cuda_core_kernel(orc):
    """Sequences sharing a page would give its cache rows two writers: the CUDA-core kernel (float32
    atomics) takes such plans, and the shared slots get both sequences' gradients."""
    wl = W.make_mla("mla_bwd_share", 23, [200, 200], [1, 1], 128, 512, 64, 64, torch.bfloat16)
    s = wl.sched
    s.block_tables[1, :2] = s.block_tables[0, :2]  # keys 0..127 shared
    dout, got, kernels = _mla_backward_run(wl, True, 0, 24)
    assert kernels == pa.PA_KERNEL_BACKWARD_SIMT, kernels
    ref = orc.mla_backward(wl.q_latent, wl.q_rope, wl.latent_cache, wl.rope_cache, dout, s.seq_lens,
                           s.query_offsets, s.block_tables, 64, wl.scale, True, 0)
    for g, want, name in zip(got, ref, ("dq_latent", "dq_rope", "d_latent", "d_rope")):
        close(g, want, torch.bfloat16, f"{name} shared pages")


def test_mla_backward_tensor_core_deterministic():
    """Every cache row of the tensor-core MLA backward has one writer: two runs give the same bits."""
    wl = W.make_mla("mla_bwd_det", 25, [900, 300], [1, 1], 128, 512, 64, 64, torch.bfloat16)
    a = _mla_backward_run(wl, True, 0, 26)[1]
    b = _mla_backward_run(wl, True, 0, 26)[1]
    for x, y in zip(a, b):
        assert torch.equal(torch.nan_to_num(x, nan=0.0), torch.nan_to_num(y, nan=0.0))
