"""GPU backward (recompute-based, float32 atomics for dK/dV) against the fp64 oracle's backward."""
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


def close(got, ref, dtype, tag):
    got, ref = got.double(), ref.double()
    owned = torch.isfinite(ref)
    scale = float(ref[owned].abs().max())
    if dtype == torch.float32:
        tol = 1e-4 * scale
        assert float((got - ref)[owned].abs().max()) <= tol, (tag, float((got - ref)[owned].abs().max()), tol)
    else:
        bad = (got - ref).abs() > 2e-3 * scale + 2e-2 * ref.abs()
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
