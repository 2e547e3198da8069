"""Paged K/V append (ruDNN `DevicePlan::append`): bit-exact page scatter through the block table,
and append + attention chained chunk by chunk equal to one-shot prefill and to the oracle."""
import pytest
import torch

import paged_kv_attention_39_b200 as pa
from gpu_helpers import check, run_gqa
from paged_kv_attention_39_b200 import workloads as W

pytestmark = pytest.mark.gpu


def expected_after_append(cache, sched, new):
    """Host scatter by torch indexing: query j of s goes to position L - n + j."""
    out = cache.clone()
    for s in range(sched.num_seqs):
        L = int(sched.seq_lens[s]); q0 = int(sched.query_offsets[s]); n = int(sched.query_offsets[s + 1]) - q0
        for j in range(n):
            p = L - n + j
            out[int(sched.block_tables[s, p // sched.page_size]), p % sched.page_size] = new[q0 + j]
    return out


@pytest.mark.parametrize("dtype,d,dv,ps", [(torch.bfloat16, 128, 128, 16), (torch.float16, 64, 64, 64),
                                           (torch.float32, 64, 32, 32), (torch.bfloat16, 512, 64, 64)])
def test_append_scatter_bit_exact(dtype, d, dv, ps):
    hkv = 1 if d == 512 else 4
    wl = W.make_gqa("app", 1, [37, 100, 5, 300], [1, 7, 5, 64], 8 if hkv > 1 else 4, hkv, d, dv, ps, dtype)
    s = wl.sched
    g = torch.Generator().manual_seed(3)
    new_k = torch.randn(s.num_queries, hkv, d, generator=g).to(dtype)
    new_v = torch.randn(s.num_queries, hkv, dv, generator=g).to(dtype)
    kc, vc = wl.k_cache.cuda(), wl.v_cache.cuda()
    plan = pa.plan_for(wl)
    pa.pa_append(plan, new_k.cuda(), new_v.cuda(), kc, vc)
    torch.cuda.synchronize()
    ek = expected_after_append(wl.k_cache, s, new_k)
    ev = expected_after_append(wl.v_cache, s, new_v)
    assert torch.equal(kc.cpu().view(torch.int16 if dtype != torch.float32 else torch.int32),
                       ek.view(torch.int16 if dtype != torch.float32 else torch.int32))
    assert torch.equal(vc.cpu().view(torch.int16 if dtype != torch.float32 else torch.int32),
                       ev.view(torch.int16 if dtype != torch.float32 else torch.int32))
    plan.close()


def test_append_then_attend_chunk_by_chunk_equals_one_shot(orc):
    """History in the cache, then two prefill chunks appended and attended one after the other:
    the rows equal a one-shot prefill over both chunks (and the oracle on the final cache)."""
    hist, na, nb = [300, 90], [100, 37], [64, 120]
    full = [h + a + b for h, a, b in zip(hist, na, nb)]
    wl = W.make_gqa("chain", 2, full, [a + b for a, b in zip(na, nb)], 32, 8, 128, 128, 64, torch.bfloat16)
    s = wl.sched
    g = torch.Generator().manual_seed(5)
    new_k = torch.randn(s.num_queries, 8, 128, generator=g).to(torch.bfloat16)
    new_v = torch.randn(s.num_queries, 8, 128, generator=g).to(torch.bfloat16)
    kc, vc = wl.k_cache.cuda(), wl.v_cache.cuda()
    # chunk A of every sequence, then chunk B
    rows_a, rows_b = [], []
    for si in range(2):
        q0 = int(s.query_offsets[si])
        rows_a += list(range(q0, q0 + na[si]))
        rows_b += list(range(q0 + na[si], q0 + na[si] + nb[si]))
    ia, ib = torch.tensor(rows_a), torch.tensor(rows_b)
    plan_a = pa.pa_plan_create([h + a for h, a in zip(hist, na)], [0, na[0], na[0] + na[1]], s.block_tables, 64,
                               s.num_pages)
    plan_b = pa.pa_plan_create(full, [0, nb[0], nb[0] + nb[1]], s.block_tables, 64, s.num_pages)
    pa.pa_append(plan_a, new_k[ia].cuda(), new_v[ia].cuda(), kc, vc)
    wl.k_cache, wl.v_cache = kc.cpu(), vc.cpu()  # run_gqa uploads the workload's caches
    oa, la = run_gqa(wl, plan=plan_a, q=wl.q[ia])
    pa.pa_append(plan_b, new_k[ib].cuda(), new_v[ib].cuda(), kc, vc)
    wl.k_cache, wl.v_cache = kc.cpu(), vc.cpu()
    ob, lb = run_gqa(wl, plan=plan_b, q=wl.q[ib])
    # one shot over the final cache
    wl.k_cache, wl.v_cache = kc.cpu(), vc.cpu()
    ref = orc.run(wl)
    out, lse = run_gqa(wl)
    check(wl, out, lse, *ref, tag="one shot after append")
    o_chain = torch.empty_like(out); l_chain = torch.empty_like(lse)
    o_chain[ia], o_chain[ib] = oa, ob
    l_chain[ia], l_chain[ib] = la, lb
    check(wl, o_chain, l_chain, *ref, tag="chunk by chunk")
    plan_a.close(); plan_b.close()
