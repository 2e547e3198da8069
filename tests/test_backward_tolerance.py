"""Where the bf16 / fp16 backward tolerances come from, reproduced on the CPU.

The tensor-core backward computes in float32 but feeds 16-bit operands to its products: the
forward's output O arrives rounded to the input type (so Drow = dO . O carries that rounding),
P is rounded before dV += P^T dO, and dS = P (dP - Drow) is rounded before dK += dS^T Q and
dQ += dS K. This file emulates exactly those roundings in float64 (every other step exact) on the
inputs of each backward GPU test, measures how far the emulated gradients land from the exact
ones, and checks that the tolerances of tests/test_gpu_backward.py keep at least a factor of two
above that error everywhere:

    |emulated - exact| <= (TOL_MAX * max|exact| + TOL_REL * |exact|) / 2     for every element.

The emulation is a model of the kernels' rounding written from their description, not the
oracle: it gathers the paged K/V itself and uses torch float64 products.
"""
import pytest
import torch

from paged_kv_attention_39_b200 import workloads as W
from test_gpu_backward import TOL_MAX, TOL_REL

MARGIN = 2.0


def _gradients(wl, dout, rounded):
    """dQ [Nq, Hq, D], dK / dV in the cache layout (float64), exact or with the kernel's roundings."""
    s = wl.sched
    dt = wl.q.dtype
    rnd = (lambda x: x.to(dt).double()) if rounded else (lambda x: x)
    hq, hkv = wl.num_q_heads, wl.num_kv_heads
    G = hq // hkv
    ps = s.page_size
    q, k, v, do = wl.q.double(), wl.k_cache.double(), wl.v_cache.double(), dout.double()
    dq = torch.zeros_like(q)
    dk = torch.zeros(k.shape, dtype=torch.float64)
    dv = torch.zeros(v.shape, dtype=torch.float64)
    for si in range(s.num_seqs):
        L = int(s.seq_lens[si])
        q0, q1 = int(s.query_offsets[si]), int(s.query_offsets[si + 1])
        n = q1 - q0
        if n == 0:
            continue
        t = torch.arange(L)
        pages = s.block_tables[si, t // ps].long()
        slots = t % ps
        Ks = k[pages, slots].repeat_interleave(G, dim=1)   # [L, Hq, D]
        Vs = v[pages, slots].repeat_interleave(G, dim=1)   # [L, Hq, Dv]
        Qs, dOs = q[q0:q1], do[q0:q1]                      # [n, Hq, D]
        pos = L - n + torch.arange(n)
        vis = torch.ones(n, L, dtype=torch.bool)
        if wl.causal:
            vis &= t.view(1, -1) <= pos.view(-1, 1)
        if wl.window > 0:
            vis &= t.view(1, -1) + wl.window > pos.view(-1, 1)
        S = wl.scale * torch.einsum("jhd,thd->hjt", Qs, Ks)
        S = S.masked_fill(~vis.unsqueeze(0), float("-inf"))
        lse = torch.logsumexp(S, dim=-1, keepdim=True)
        P = torch.where(vis.unsqueeze(0), torch.exp(S - lse), torch.zeros((), dtype=torch.float64))
        O = torch.einsum("hjt,thd->jhd", P, Vs)
        Drow = (dOs * rnd(O)).sum(-1).transpose(0, 1).unsqueeze(-1)  # [Hq, n, 1]
        dP = torch.einsum("jhd,thd->hjt", dOs, Vs)
        dS = P * (dP - Drow)
        Pr, dSr = rnd(P), rnd(dS)
        dq[q0:q1] = wl.scale * torch.einsum("hjt,thd->jhd", dSr, Ks)
        dKs = wl.scale * torch.einsum("hjt,jhd->thd", dSr, Qs)   # [L, Hq, D]
        dVs = torch.einsum("hjt,jhd->thd", Pr, dOs)
        dKs = dKs.view(L, hkv, G, -1).sum(2)
        dVs = dVs.view(L, hkv, G, -1).sum(2)
        dk.index_put_((pages, slots), dKs, accumulate=True)
        dv.index_put_((pages, slots), dVs, accumulate=True)
    return dq, dk, dv


def _cases():
    """The inputs of every bf16 / fp16 backward comparison with the oracle on the GPU."""
    out = []
    for dtype in (torch.bfloat16, torch.float16):
        for causal, window in ((True, 0), (True, 33), (False, 0)):
            wl = W.make_gqa("bwd", 3, [70, 130, 9, 200], [1, 40, 9, 3], 8, 2, 64, 64, 16, dtype, causal=causal,
                            window=window)
            g = torch.Generator().manual_seed(7)
            dout = torch.randn(wl.sched.num_queries, 8, 64, generator=g).to(dtype)
            out.append((f"matches_oracle {dtype} c{causal} w{window}", wl, dout))
    for hq, hkv, d, ps, causal, window, dtype in [(32, 8, 128, 64, True, 0, torch.bfloat16),
                                                   (16, 16, 128, 16, True, 0, torch.float16),
                                                   (16, 1, 64, 32, True, 100, torch.bfloat16),
                                                   (8, 2, 128, 16, False, 0, torch.bfloat16),
                                                   (8, 4, 64, 128, True, 0, torch.float16),
                                                   (32, 1, 64, 16, True, 0, torch.bfloat16),
                                                   (8, 2, 128, 256, True, 0, torch.bfloat16)]:
        wl = W.make_gqa("bwd_tc", 5, [300, 513, 64, 1000], [100, 200, 64, 17], hq, hkv, d, d, ps, dtype,
                        causal=causal, window=window)
        g = torch.Generator().manual_seed(11)
        dout = torch.randn(wl.sched.num_queries, hq, d, generator=g).to(dtype)
        out.append((f"tensor_core_shapes hq{hq} hkv{hkv} d{d} ps{ps} c{causal} w{window}", wl, dout))
    # the tensor-core MLA backward's shapes, as the GQA backward they are: one KV head, the key
    # [latent | rope] (576 columns), the value the latent (512), every query head in the group
    for h, lens, qs, ps, dtype, causal, window in [
            (128, [700, 2000, 130, 4100], [1, 1, 1, 1], 64, torch.bfloat16, True, 0),
            (16, [300, 513, 64, 1000], [8, 3, 1, 5], 16, torch.float16, True, 300),
            (128, [90, 1500, 257], [1, 1, 1], 128, torch.bfloat16, False, 0),
            (64, [1024, 777], [2, 1], 32, torch.bfloat16, True, 0)]:
        m = W.make_mla("mla_bwd_tc", 19, lens, qs, h, 512, 64, ps, dtype, causal=causal, window=window)
        wl = W.GqaWorkload("mla_as_gqa", m.sched, torch.cat([m.q_latent, m.q_rope], dim=-1),
                           torch.cat([m.latent_cache, m.rope_cache], dim=-1), m.latent_cache, h, 1, 576, 512,
                           m.scale, causal, window)
        g = torch.Generator().manual_seed(21)
        dout = torch.randn(m.sched.num_queries, h, 512, generator=g).to(dtype)
        out.append((f"mla tensor core h{h} ps{ps} {dtype} c{causal} w{window}", wl, dout))
    # the bf16 shapes of test_backward_limits (CUDA-core kernel: no 16-bit rounding of P or dS, so
    # its error stays below this emulation's; the 128-head group on the tensor cores)
    for name, hq, hkv, d, dv, ps in [("d256", 16, 4, 256, 256, 16), ("d192v128", 8, 2, 192, 128, 16),
                                     ("g128", 128, 1, 128, 128, 64)]:
        wl = W.make_gqa("bwd_lim_" + name, 71, [300, 45, 700], [60, 9, 3], hq, hkv, d, dv, ps, torch.bfloat16)
        g = torch.Generator().manual_seed(17)
        out.append((f"limits {name}", wl, torch.randn(wl.sched.num_queries, hq, dv, generator=g).to(torch.bfloat16)))
    wl = W.make_gqa("share_tc", 6, [150, 150], [30, 30], 8, 2, 64, 64, 16, torch.bfloat16)
    wl.sched.block_tables[1, :3] = wl.sched.block_tables[0, :3]
    g = torch.Generator().manual_seed(12)
    out.append(("shared pages", wl, torch.randn(wl.sched.num_queries, 8, 64, generator=g).to(torch.bfloat16)))
    wl = W.make_gqa("smoke_bwd", 2, [90, 150], [20, 3], 8, 2, 64, 64, 16, torch.bfloat16)
    g = torch.Generator().manual_seed(3)
    out.append(("smoke", wl, torch.randn(wl.sched.num_queries, 8, 64, generator=g).to(torch.bfloat16)))
    return out


@pytest.mark.parametrize("tag,wl,dout", _cases(), ids=lambda x: x if isinstance(x, str) else "")
def test_tolerance_keeps_a_margin_over_the_emulated_rounding(tag, wl, dout):
    dt = wl.q.dtype
    exact = _gradients(wl, dout, rounded=False)
    emul = _gradients(wl, dout, rounded=True)
    for name, e, r in zip(("dq", "dk", "dv"), emul, exact):
        touched = r != 0
        scale = float(r.abs().max())
        bound = TOL_MAX[dt] * scale + TOL_REL[dt] * r.abs()
        ratio = float(((e - r).abs() / bound)[touched].max())
        frac = float((e - r).abs().max()) / scale
        print(f"{tag} {name}: emulated error {frac:.4%} of max|ref|, {ratio:.3f} of the bound")
        assert ratio * MARGIN <= 1.0, (tag, name, ratio, frac)


def test_the_emulation_sees_the_rounding():
    """The rounded emulation differs from the exact gradients (bf16 rounding is visible), and an
    emulation with float64 operands would not: the measurement above is not vacuous."""
    tag, wl, dout = _cases()[0]
    exact = _gradients(wl, dout, rounded=False)
    emul = _gradients(wl, dout, rounded=True)
    assert all(float((e - r).abs().max()) > 1e-6 * float(r.abs().max()) for e, r in zip(emul, exact))
