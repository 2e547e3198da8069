"""Pins for the fp64 oracle: checks against facts that do not come from the oracle itself.

Each pin takes an `Oracle` (the real one, or a compile-time mutant) and raises AssertionError
when the oracle disagrees with the fact it checks. Sources of truth:
  * torch's fp64 scaled_dot_product_attention / logsumexp on a densely gathered copy
    (boostr `standard_attention_fwd` says every fused kernel must match the dense result);
  * closed forms: a single key returns its value row and lse = scale * q.k; a constant value
    per KV head comes back unchanged for every query head of its group; with Q = 0 every
    visible key weighs the same, so exp(lse) is the visible-key count (closed form from the
    query's absolute position, the causal flag and the window) and out is their mean value;
    V[t] = t makes out the mean visible position; q = a large multiple of K[t*] selects t*;
  * invariances the definition implies: relabelling the page pool, splitting the keys and
    merging the parts (ruDNN "merge FP32 statistics"; alice-llm `lse_combine`), splitting a
    prefill chunk in two, a window wider than the context, GQA on a repeated cache, MLA as
    single-head attention on the concatenated key;
  * exact widening of bf16/fp16 inputs (same values given as fp32 give identical results);
  * sparse top-K (alice-llm `llama3_sparse_attention`): a torch restatement on tiny cases, every
    block selected == dense attention, a planted block wins top-1 and then equals attention
    restricted to its keys, Q = 0 makes all visible blocks tie (lowest indices win, uniform
    weights), and the page's own bridge tests on `fixture_gqa`.
"""
from __future__ import annotations

import math

import numpy as np
import torch
import torch.nn.functional as F

from paged_kv_attention_39_b200 import workloads as W


def _dense_kv(cache: torch.Tensor, bt: torch.Tensor, s: int, L: int, ps: int) -> torch.Tensor:
    """Gather sequence s's first L rows as [L, heads, dim] via torch indexing."""
    t = torch.arange(L)
    pages = bt[s, (t // ps)].long()
    return cache[pages, t % ps].double()


def _counts(L: int, n: int, causal: bool, window: int):
    """Closed-form visible range [lo, hi] per query of a sequence (right-aligned positions)."""
    res = []
    for j in range(n):
        p = L - n + j
        hi = p if causal else L - 1
        lo = max(0, p - window + 1) if window > 0 else 0
        res.append((lo, hi))
    return res


def _small_cases():
    """Tiny GQA workloads spanning decode, prefill chunks, windows, page sizes and dtypes."""
    return [
        W.make_gqa("t1", 1, [5, 17, 33], [1, 3, 33], 4, 2, 8, 8, 4, torch.float32, causal=True),
        W.make_gqa("t2", 2, [40, 9], [7, 9], 6, 3, 16, 8, 8, torch.float32, causal=True, window=5),
        W.make_gqa("t3", 3, [30, 12, 1], [4, 12, 1], 4, 1, 8, 12, 16, torch.bfloat16, causal=False),
        W.make_gqa("t4", 4, [23, 64], [23, 2], 8, 8, 8, 8, 4, torch.float16, causal=False, window=7),
        W.make_gqa("t5", 5, [50], [20], 4, 2, 8, 8, 16, torch.float32, causal=True, window=1),
    ]


def pin_sdpa_bruteforce(orc):
    for wl in _small_cases():
        s_ = wl.sched
        out, lse = orc.run(wl)
        G = wl.num_q_heads // wl.num_kv_heads
        for s in range(s_.num_seqs):
            L = int(s_.seq_lens[s]); q0 = int(s_.query_offsets[s]); n = int(s_.query_offsets[s + 1]) - q0
            if n == 0:
                continue
            K = _dense_kv(wl.k_cache, s_.block_tables, s, L, s_.page_size).repeat_interleave(G, dim=1)
            V = _dense_kv(wl.v_cache, s_.block_tables, s, L, s_.page_size).repeat_interleave(G, dim=1)
            Q = wl.q[q0:q0 + n].double()
            pos = torch.arange(L - n, L).view(n, 1)
            t = torch.arange(L).view(1, L)
            keep = torch.ones(n, L, dtype=torch.bool)
            if wl.causal:
                keep &= t <= pos
            if wl.window > 0:
                keep &= t + wl.window > pos
            qh, kh, vh = Q.transpose(0, 1), K.transpose(0, 1), V.transpose(0, 1)
            ref = F.scaled_dot_product_attention(qh, kh, vh, attn_mask=keep, scale=wl.scale)
            sc = (qh @ kh.transpose(1, 2)) * wl.scale
            ref_lse = torch.logsumexp(sc.masked_fill(~keep, float("-inf")), dim=-1)
            got = out[q0:q0 + n].transpose(0, 1)
            assert torch.allclose(got, ref, rtol=1e-11, atol=1e-12), (wl.name, s, (got - ref).abs().max())
            assert torch.allclose(lse[q0:q0 + n].transpose(0, 1), ref_lse, rtol=1e-12, atol=1e-12), (wl.name, s)


def alice_fixture():
    """alice-llm `fixture_gqa`: tq=3, hq=4, hkv=2, head_dim=8, seq_len=12, values sin/cos of
    the flat index; dense [seq, hkv, d] K/V placed in pages of 4 with an identity table."""
    tq, hq, hkv, d, L, ps = 3, 4, 2, 8, 12, 4
    q = torch.tensor([math.sin(i * 0.05) for i in range(tq * hq * d)], dtype=torch.float32).view(tq, hq, d)
    k = torch.tensor([math.cos(i * 0.07) for i in range(L * hkv * d)], dtype=torch.float32).view(L // ps, ps, hkv, d)
    v = torch.tensor([math.sin(i * 0.03) for i in range(L * hkv * d)], dtype=torch.float32).view(L // ps, ps, hkv, d)
    sl = torch.tensor([L], dtype=torch.int32)
    qo = torch.tensor([0, tq], dtype=torch.int32)
    bt = torch.arange(L // ps, dtype=torch.int32).view(1, -1)
    return q, k, v, sl, qo, bt, ps, 1.0 / math.sqrt(d)


def pin_alice_fixture_dense(orc):
    q, k, v, sl, qo, bt, ps, scale = alice_fixture()
    out, lse = orc.attention(q, k, v, sl, qo, bt, ps, scale, causal=False, window=0)
    G = 2
    K = k.reshape(-1, 2, 8).double().repeat_interleave(G, 1).transpose(0, 1)
    V = v.reshape(-1, 2, 8).double().repeat_interleave(G, 1).transpose(0, 1)
    Q = q.double().transpose(0, 1)
    ref = F.scaled_dot_product_attention(Q, K, V, scale=scale).transpose(0, 1)
    rel = ((out - ref).abs() / ref.abs().clamp_min(1e-6)).max()
    assert rel < 1e-12, rel


def pin_single_key(orc):
    for dt in (torch.float32, torch.bfloat16):
        wl = W.make_gqa("one", 7, [1, 1, 1], [1, 1, 1], 6, 2, 16, 8, 4, dt, causal=True)
        out, lse = orc.run(wl)
        s_ = wl.sched
        G = 3
        for s in range(3):
            page = int(s_.block_tables[s, 0])
            for h in range(6):
                kv = h // G
                assert torch.equal(out[s, h], wl.v_cache[page, 0, kv].double())
                qk = math.fsum(float(a) * float(b) for a, b in zip(wl.q[s, h].double(), wl.k_cache[page, 0, kv].double()))
                assert abs(float(lse[s, h]) - wl.scale * qk) <= 1e-12 * max(1.0, abs(wl.scale * qk))


def pin_constant_v_per_kv_head(orc):
    wl = W.make_gqa("cv", 8, [19, 40, 7], [3, 1, 7], 8, 2, 8, 6, 8, torch.float32, causal=True, window=9)
    c = torch.randn(2, 6, generator=torch.Generator().manual_seed(1))
    wl.v_cache[:] = c.view(1, 1, 2, 6)
    out, _ = orc.run(wl)
    G = 4
    for h in range(8):
        ref = c[h // G].double().view(1, 6)
        assert torch.allclose(out[:, h], ref.expand_as(out[:, h]), rtol=0, atol=1e-14), h


def pin_q_zero_counts_and_mean(orc):
    cases = [
        W.make_gqa("z1", 9, [37, 100, 64, 5], [1, 1, 13, 5], 4, 2, 8, 8, 16, torch.float32, causal=True),
        W.make_gqa("z2", 10, [37, 100, 64], [1, 9, 13], 4, 2, 8, 8, 16, torch.float32, causal=True, window=6),
        W.make_gqa("z3", 11, [37, 60], [2, 9], 4, 4, 8, 8, 8, torch.float32, causal=False, window=11),
        W.make_gqa("z4", 12, [37, 60], [2, 9], 2, 1, 8, 8, 8, torch.float32, causal=False),
    ]
    for wl in cases:
        wl.q.zero_()
        out, lse = orc.run(wl)
        s_ = wl.sched
        G = wl.num_q_heads // wl.num_kv_heads
        for s in range(s_.num_seqs):
            L = int(s_.seq_lens[s]); q0 = int(s_.query_offsets[s]); n = int(s_.query_offsets[s + 1]) - q0
            V = _dense_kv(wl.v_cache, s_.block_tables, s, L, s_.page_size)
            for j, (lo, hi) in enumerate(_counts(L, n, wl.causal, wl.window)):
                cnt = hi - lo + 1
                for h in range(wl.num_q_heads):
                    got = float(lse[q0 + j, h])
                    assert round(math.exp(got)) == cnt, (wl.name, s, j, h, math.exp(got), cnt)
                    assert abs(got - math.log(cnt)) <= 1e-12
                    ref = V[lo:hi + 1, h // G].mean(0)
                    assert torch.allclose(out[q0 + j, h], ref, rtol=1e-12, atol=1e-13), (wl.name, s, j, h)


def pin_position_probe(orc):
    """V[t, :, 0] = t (exact in fp32), Q = 0: out[..., 0] is the mean visible position."""
    wl = W.make_gqa("pp", 13, [100, 37, 250], [1, 5, 30], 4, 2, 8, 8, 16, torch.float32, causal=True, window=40)
    wl.q.zero_()
    s_ = wl.sched
    for s in range(s_.num_seqs):
        L = int(s_.seq_lens[s])
        t = torch.arange(L)
        wl.v_cache[s_.block_tables[s, t // s_.page_size].long(), t % s_.page_size, :, 0] = t.float().view(-1, 1)
    out, _ = orc.run(wl)
    for s in range(s_.num_seqs):
        L = int(s_.seq_lens[s]); q0 = int(s_.query_offsets[s]); n = int(s_.query_offsets[s + 1]) - q0
        for j, (lo, hi) in enumerate(_counts(L, n, True, 40)):
            assert torch.allclose(out[q0 + j, :, 0], torch.full((4,), (lo + hi) / 2.0, dtype=torch.float64),
                                  rtol=0, atol=1e-10), (s, j)


def select_target_queries(wl, seed: int, margin: float = 80.0):
    """Rewrite Q so that each (query, head) row puts all its weight on one visible key t*.

    q = alpha * K[t*] with t* a visible key whose self-score beats every other visible key's
    score by a positive gap, and alpha chosen so the scaled gap is `margin`: every other
    weight is below exp(-margin). Returns {(query, head): (sequence, t*)}.
    """
    s_ = wl.sched
    g = torch.Generator().manual_seed(seed)
    G = wl.num_q_heads // wl.num_kv_heads
    target = {}
    for s in range(s_.num_seqs):
        L = int(s_.seq_lens[s]); q0 = int(s_.query_offsets[s]); n = int(s_.query_offsets[s + 1]) - q0
        K = _dense_kv(wl.k_cache, s_.block_tables, s, L, s_.page_size)
        for j, (lo, hi) in enumerate(_counts(L, n, wl.causal, wl.window)):
            for h in range(wl.num_q_heads):
                Kh = K[lo:hi + 1, h // G]
                cand = torch.randperm(hi - lo + 1, generator=g)[:8].tolist() + [int(Kh.norm(dim=1).argmax())]
                for c in cand:
                    dots = Kh @ Kh[c]
                    own = float(dots[c])
                    dots[c] = float("-inf")
                    gap = own - (float(dots.max()) if hi > lo else own - 1.0)
                    if gap > 1e-3 * max(own, 1e-30):
                        break
                alpha = margin / (wl.scale * gap)
                wl.q[q0 + j, h] = (alpha * Kh[c]).to(wl.q.dtype)
                target[(q0 + j, h)] = (s, lo + c)
    return target


def pin_large_score_selects_target(orc):
    """q = alpha * K[t*] for a visible t*: every other weight underflows, out == V[t*]."""
    wl = W.make_gqa("ls", 14, [70, 33, 129], [1, 6, 2], 4, 2, 16, 8, 8, torch.float32, causal=True, window=50)
    s_ = wl.sched
    target = select_target_queries(wl, 3)
    out, _ = orc.run(wl)
    G = 2
    for (qi, h), (s, ts) in target.items():
        V = _dense_kv(wl.v_cache, s_.block_tables, s, int(s_.seq_lens[s]), s_.page_size)
        assert torch.allclose(out[qi, h], V[ts, h // G], rtol=0, atol=1e-12), (qi, h, s, ts)


def pin_page_permutation_invariance(orc):
    wl = W.make_gqa("perm", 15, [45, 90, 3], [2, 1, 3], 4, 2, 8, 8, 8, torch.bfloat16, causal=True, window=20)
    out, lse = orc.run(wl)
    P = wl.sched.num_pages
    pi = torch.randperm(P, generator=torch.Generator().manual_seed(4))
    k2 = torch.empty_like(wl.k_cache); k2[pi] = wl.k_cache
    v2 = torch.empty_like(wl.v_cache); v2[pi] = wl.v_cache
    bt = wl.sched.block_tables.clone()
    m = bt >= 0
    bt[m] = pi[bt[m].long()].to(torch.int32)
    out2, lse2 = orc.attention(wl.q, k2, v2, wl.sched.seq_lens, wl.sched.query_offsets, bt,
                               wl.sched.page_size, wl.scale, wl.causal, wl.window)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


def pin_split_equals_unsplit(orc):
    wl = W.make_gqa("split", 16, [77, 130, 20], [1, 4, 20], 4, 2, 8, 8, 16, torch.float32, causal=True, window=60)
    out, lse = orc.run(wl)
    L = wl.sched.seq_lens
    nparts = 5
    o_parts, l_parts = [], []
    for i in range(nparts):
        kb = (L.long() * i // nparts).to(torch.int32)
        ke = (L.long() * (i + 1) // nparts).to(torch.int32)
        o, l = orc.run(wl, key_begin=kb, key_end=ke)
        o_parts.append(o.reshape(-1, o.shape[-1])); l_parts.append(l.reshape(-1))
    mo, ml = orc.lse_combine(torch.stack(o_parts), torch.stack(l_parts))
    assert torch.allclose(mo.view_as(out), out, rtol=1e-12, atol=1e-13)
    assert torch.allclose(ml.view_as(lse), lse, rtol=1e-12, atol=1e-13)


def pin_chunked_equals_oneshot(orc):
    hist, nA, nB = 45, 13, 22
    for causal, window in ((True, 0), (True, 17)):
        wl = W.make_gqa("chunk", 17, [hist + nA + nB], [nA + nB], 4, 2, 8, 8, 8, torch.float32, causal=causal, window=window)
        s_ = wl.sched
        out, lse = orc.run(wl)
        oa, la = orc.attention(wl.q[:nA], wl.k_cache, wl.v_cache, torch.tensor([hist + nA]),
                               torch.tensor([0, nA]), s_.block_tables, s_.page_size, wl.scale, causal, window)
        ob, lb = orc.attention(wl.q[nA:], wl.k_cache, wl.v_cache, torch.tensor([hist + nA + nB]),
                               torch.tensor([0, nB]), s_.block_tables, s_.page_size, wl.scale, causal, window)
        assert torch.equal(torch.cat([oa, ob]), out) and torch.equal(torch.cat([la, lb]), lse)


def pin_window_cases(orc):
    wl = W.make_gqa("win", 18, [60, 31], [5, 31], 4, 2, 8, 8, 8, torch.float32, causal=True)
    out0, lse0 = orc.run(wl)
    big, lbig = orc.attention(wl.q, wl.k_cache, wl.v_cache, wl.sched.seq_lens, wl.sched.query_offsets,
                              wl.sched.block_tables, 8, wl.scale, True, 61)
    assert torch.equal(out0, big) and torch.equal(lse0, lbig)
    one, _ = orc.attention(wl.q, wl.k_cache, wl.v_cache, wl.sched.seq_lens, wl.sched.query_offsets,
                           wl.sched.block_tables, 8, wl.scale, True, 1)
    s_ = wl.sched
    for s in range(2):
        L = int(s_.seq_lens[s]); q0 = int(s_.query_offsets[s]); n = int(s_.query_offsets[s + 1]) - q0
        V = _dense_kv(wl.v_cache, s_.block_tables, s, L, 8)
        for j in range(n):
            p = L - n + j
            for h in range(4):
                assert torch.equal(one[q0 + j, h], V[p, h // 2])


def pin_gqa_equals_mha_repeated(orc):
    wl = W.make_gqa("rep", 19, [33, 70], [3, 1], 8, 2, 8, 8, 8, torch.bfloat16, causal=True, window=25)
    out, lse = orc.run(wl)
    k = wl.k_cache.repeat_interleave(4, dim=2)
    v = wl.v_cache.repeat_interleave(4, dim=2)
    out2, lse2 = orc.attention(wl.q, k, v, wl.sched.seq_lens, wl.sched.query_offsets, wl.sched.block_tables,
                               8, wl.scale, True, 25)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


def pin_mla_equals_gqa_concat(orc):
    wl = W.make_mla("mla", 20, [40, 9, 77], [1, 9, 3], 8, 32, 8, 8, torch.float32, causal=True, window=30)
    out, lse = orc.run(wl)
    q = torch.cat([wl.q_latent, wl.q_rope], dim=-1)
    k = torch.cat([wl.latent_cache, wl.rope_cache], dim=-1)
    out2, lse2 = orc.attention(q, k, wl.latent_cache, wl.sched.seq_lens, wl.sched.query_offsets,
                               wl.sched.block_tables, 8, wl.scale, True, 30)
    assert torch.allclose(out, out2, rtol=1e-12, atol=1e-13)
    assert torch.allclose(lse, lse2, rtol=1e-12, atol=1e-13)


def pin_half_precision_widening(orc):
    for dt in (torch.bfloat16, torch.float16):
        wl = W.make_gqa("wid", 21, [29, 50], [2, 1], 4, 2, 16, 8, 8, dt, causal=True)
        out, lse = orc.run(wl)
        out2, lse2 = orc.attention(wl.q.float(), wl.k_cache.float(), wl.v_cache.float(), wl.sched.seq_lens,
                                   wl.sched.query_offsets, wl.sched.block_tables, 8, wl.scale, True, 0)
        assert torch.equal(out, out2) and torch.equal(lse, lse2)
    # every fp16 bit pattern (finite ones) widens to the value torch assigns it
    bits = torch.from_numpy(np.arange(1 << 16, dtype=np.uint16).view(np.float16).copy())
    finite = bits[torch.isfinite(bits)]
    n = finite.numel() // 8 * 8
    vals = finite[:n].view(-1, 1, 1, 8)  # pages of one slot, one head, eight dims
    P = vals.shape[0]
    q = torch.zeros(1, 1, 8, dtype=torch.float16)
    q[0, 0, 0] = 1.0
    sl = torch.tensor([1], dtype=torch.int32)
    qo = torch.tensor([0, 1], dtype=torch.int32)
    for page in (0, P // 3, P - 1):
        bt = torch.tensor([[page]], dtype=torch.int32)
        o, _ = orc.attention(q, vals, vals, sl, qo, bt, 1, 1.0, True, 0)
        assert torch.equal(o[0, 0], vals[page, 0, 0].double())


def _backward_cases():
    return [
        W.make_gqa("b1", 31, [9, 20], [3, 20], 4, 2, 8, 8, 4, torch.float32, causal=True),
        W.make_gqa("b2", 32, [25, 6], [4, 2], 6, 3, 8, 4, 8, torch.float32, causal=True, window=5),
        W.make_gqa("b3", 33, [12], [5], 2, 2, 8, 8, 4, torch.float32, causal=False, window=4),
    ]


def pin_backward_vs_autograd(orc):
    """dq, dk, dv against torch autograd of fp64 SDPA on the dense gather (GQA by repeat_interleave,
    whose backward sums the group), scattered back to the cache slots through the block table."""
    for wl in _backward_cases():
        s_ = wl.sched
        g = torch.Generator().manual_seed(9)
        dout = torch.randn(wl.q.shape[0], wl.num_q_heads, wl.v_head_dim, generator=g).to(wl.q.dtype)
        dq, dk, dv = orc.attention_backward(wl.q, wl.k_cache, wl.v_cache, dout, s_.seq_lens, s_.query_offsets,
                                            s_.block_tables, s_.page_size, wl.scale, wl.causal, wl.window)
        G = wl.num_q_heads // wl.num_kv_heads
        ref_dk = torch.zeros_like(dk)
        ref_dv = torch.zeros_like(dv)
        for s in range(s_.num_seqs):
            L = int(s_.seq_lens[s]); q0 = int(s_.query_offsets[s]); n = int(s_.query_offsets[s + 1]) - q0
            t = torch.arange(L)
            pages = s_.block_tables[s, t // s_.page_size].long()
            K = wl.k_cache[pages, t % s_.page_size].double().requires_grad_(True)
            V = wl.v_cache[pages, t % s_.page_size].double().requires_grad_(True)
            Q = wl.q[q0:q0 + n].double().requires_grad_(True)
            pos = torch.arange(L - n, L).view(n, 1)
            keep = torch.ones(n, L, dtype=torch.bool)
            if wl.causal:
                keep &= t.view(1, L) <= pos
            if wl.window > 0:
                keep &= t.view(1, L) + wl.window > pos
            o = F.scaled_dot_product_attention(Q.transpose(0, 1), K.repeat_interleave(G, 1).transpose(0, 1),
                                               V.repeat_interleave(G, 1).transpose(0, 1), attn_mask=keep,
                                               scale=wl.scale)
            (o * dout[q0:q0 + n].double().transpose(0, 1)).sum().backward()
            assert torch.allclose(dq[q0:q0 + n], Q.grad, rtol=1e-10, atol=1e-12), (wl.name, s)
            ref_dk.index_put_((pages, t % s_.page_size), K.grad, accumulate=True)
            ref_dv.index_put_((pages, t % s_.page_size), V.grad, accumulate=True)
        assert torch.allclose(dk, ref_dk, rtol=1e-10, atol=1e-12), wl.name
        assert torch.allclose(dv, ref_dv, rtol=1e-10, atol=1e-12), wl.name


def pin_backward_finite_differences(orc):
    """Central differences of L = sum(out * dO) (forward oracle) at a few entries of q, k, v."""
    wl = W.make_gqa("fd", 34, [10, 7], [4, 2], 4, 2, 8, 8, 4, torch.float32, causal=True, window=6)
    s_ = wl.sched
    g = torch.Generator().manual_seed(10)
    dout = torch.randn(wl.q.shape[0], 4, 8, generator=g).to(torch.float32)
    dq, dk, dv = orc.attention_backward(wl.q, wl.k_cache, wl.v_cache, dout, s_.seq_lens, s_.query_offsets,
                                        s_.block_tables, 4, wl.scale, True, 6)

    def loss(q, k, v):
        out, _ = orc.attention(q, k, v, s_.seq_lens, s_.query_offsets, s_.block_tables, 4, wl.scale, True, 6)
        return float((out * dout.double()).sum())

    probes = [("q", (1, 2, 3)), ("q", (5, 0, 7)), ("k", (int(s_.block_tables[0, 1]), 2, 1, 4)),
              ("v", (int(s_.block_tables[1, 0]), 3, 0, 6)), ("v", (int(s_.block_tables[0, 2]), 1, 1, 0))]
    for name, idx in probes:
        base = {"q": wl.q, "k": wl.k_cache, "v": wl.v_cache}[name]
        plus, minus = base.clone(), base.clone()
        plus[idx] += 1e-2
        minus[idx] -= 1e-2
        h2 = float(plus[idx]) - float(minus[idx])
        args_p = {"q": wl.q, "k": wl.k_cache, "v": wl.v_cache}; args_p[name] = plus
        args_m = {"q": wl.q, "k": wl.k_cache, "v": wl.v_cache}; args_m[name] = minus
        fd = (loss(args_p["q"], args_p["k"], args_p["v"]) - loss(args_m["q"], args_m["k"], args_m["v"])) / h2
        an = float({"q": dq, "k": dk, "v": dv}[name][idx])
        assert abs(fd - an) <= 1e-4 * max(1.0, abs(an)), (name, idx, fd, an)


def pin_mla_backward_finite_differences(orc):
    """Central differences of L = sum(out * dO) (MLA forward oracle) at entries of q_latent, q_rope,
    the latent cache (a key and a value at once) and the rope cache."""
    wl = W.make_mla("fdm", 35, [9, 6], [3, 2], 3, 8, 4, 4, torch.float32, causal=True, window=5)
    s_ = wl.sched
    g = torch.Generator().manual_seed(14)
    dout = torch.randn(wl.q_latent.shape[0], 3, 8, generator=g).to(torch.float32)
    dql, dqr, dlat, drope = orc.mla_backward(wl.q_latent, wl.q_rope, wl.latent_cache, wl.rope_cache, dout,
                                             s_.seq_lens, s_.query_offsets, s_.block_tables, 4, wl.scale, True, 5)
    names = ("ql", "qr", "lat", "rope")
    base = {"ql": wl.q_latent, "qr": wl.q_rope, "lat": wl.latent_cache, "rope": wl.rope_cache}

    def loss(a):
        out, _ = orc.mla(a["ql"], a["qr"], a["lat"], a["rope"], s_.seq_lens, s_.query_offsets, s_.block_tables, 4,
                         wl.scale, True, 5)
        return float((out * dout.double()).sum())

    probes = [("ql", (1, 2, 3)), ("ql", (4, 0, 7)), ("qr", (0, 1, 2)), ("qr", (3, 2, 0)),
              ("lat", (int(s_.block_tables[0, 1]), 1, 0, 5)), ("lat", (int(s_.block_tables[1, 0]), 2, 0, 0)),
              ("rope", (int(s_.block_tables[0, 0]), 3, 0, 1)), ("rope", (int(s_.block_tables[1, 1]), 0, 0, 3))]
    grads = {"ql": dql, "qr": dqr, "lat": dlat, "rope": drope}
    for name, idx in probes:
        plus, minus = base[name].clone(), base[name].clone()
        plus[idx] += 1e-2
        minus[idx] -= 1e-2
        h2 = float(plus[idx]) - float(minus[idx])
        ap = dict(base); ap[name] = plus
        am = dict(base); am[name] = minus
        fd = (loss(ap) - loss(am)) / h2
        an = float(grads[name][idx])
        assert abs(fd - an) <= 1e-4 * max(1.0, abs(an)), (name, idx, fd, an)
    assert names  # every input has at least one probe


# ---- sparse top-K block selection (alice-llm `llama3_sparse_attention`) -------------------------

def _sparse_cases():
    """(workload, block_size) pairs: decode and prefill chunks, windows, ragged last blocks."""
    return [
        (W.make_gqa("s1", 21, [37, 100, 64], [1, 1, 1], 4, 2, 8, 8, 4, torch.float32, causal=True), 8),
        (W.make_gqa("s2", 22, [45, 30], [9, 30], 6, 3, 16, 8, 8, torch.float32, causal=True, window=13), 8),
        (W.make_gqa("s3", 23, [50, 19], [5, 19], 4, 1, 8, 12, 4, torch.bfloat16, causal=False), 12),
        (W.make_gqa("s4", 24, [70], [16], 8, 2, 8, 8, 16, torch.float32, causal=True), 16),
    ]


def _brute_sparse(wl, bs, topk):
    """Proxy scores, selection and attention restated with torch on the dense gather."""
    s_ = wl.sched
    G = wl.num_q_heads // wl.num_kv_heads
    nq = s_.num_queries
    nb_max = max(1, max((int(L) + bs - 1) // bs for L in s_.seq_lens))
    scores = torch.full((nq, wl.num_kv_heads, nb_max), float("-inf"), dtype=torch.float64)
    width = topk if topk > 0 else nb_max
    sel = torch.full((nq, wl.num_kv_heads, width), -1, dtype=torch.int32)
    out = torch.zeros(nq, wl.num_q_heads, wl.v_head_dim, dtype=torch.float64)
    lse = torch.full((nq, wl.num_q_heads), float("-inf"), dtype=torch.float64)
    for s in range(s_.num_seqs):
        L = int(s_.seq_lens[s]); q0 = int(s_.query_offsets[s]); n = int(s_.query_offsets[s + 1]) - q0
        if n == 0:
            continue
        nb = (L + bs - 1) // bs
        k = nb if (topk == 0 or topk >= nb) else topk
        K = _dense_kv(wl.k_cache, s_.block_tables, s, L, s_.page_size)
        V = _dense_kv(wl.v_cache, s_.block_tables, s, L, s_.page_size)
        for j in range(n):
            p = L - n + j
            t = torch.arange(L)
            vis = torch.ones(L, dtype=torch.bool)
            if wl.causal:
                vis &= t <= p
            if wl.window > 0:
                vis &= t + wl.window > p
            for kvh in range(wl.num_kv_heads):
                qp = wl.q[q0 + j, kvh * G].double()
                sc = (K[:, kvh] @ qp) * wl.scale
                blk = []
                for b in range(nb):
                    m = sc[b * bs:(b + 1) * bs][vis[b * bs:(b + 1) * bs]]
                    blk.append(float(m.max()) if m.numel() else float("-inf"))
                scores[q0 + j, kvh, :nb] = torch.tensor(blk, dtype=torch.float64)
                chosen = sorted(sorted(range(nb), key=lambda b: (-blk[b], b))[:k])
                sel[q0 + j, kvh, :k] = torch.tensor(chosen, dtype=torch.int32)
                keep = vis & torch.isin(t // bs, torch.tensor(chosen, dtype=torch.int64))
                for g in range(G):
                    h = kvh * G + g
                    x = (K[:, kvh] @ wl.q[q0 + j, h].double()) * wl.scale
                    if keep.any():
                        w = torch.softmax(x[keep], dim=0)
                        out[q0 + j, h] = w @ V[keep, kvh]
                        lse[q0 + j, h] = torch.logsumexp(x[keep], dim=0)
    return scores, sel, out, lse


def pin_sparse_bruteforce(orc):
    """Scores, the exact selection and the output against a torch restatement, for top-k below,
    at and above the block count."""
    for wl, bs in _sparse_cases():
        for topk in (1, 2, 3, 0):
            rs, rsel, rout, rlse = _brute_sparse(wl, bs, topk)
            sc, sel, out, lse = orc.sparse(wl, bs, topk)
            assert sc.shape == rs.shape and torch.allclose(sc, rs, rtol=1e-12, atol=1e-12, equal_nan=False), wl.name
            assert torch.equal(sel, rsel), (wl.name, topk)
            assert torch.allclose(out, rout, rtol=1e-11, atol=1e-12), (wl.name, topk, (out - rout).abs().max())
            assert torch.allclose(lse, rlse, rtol=1e-12, atol=1e-12), (wl.name, topk)


def pin_sparse_dense_fallback(orc):
    """Every block selected (top-k 0, equal to or above the block count) is dense attention: the
    selection is 0 .. nb-1 and out/lse equal the dense oracle's."""
    for wl, bs in _sparse_cases():
        dout, dlse = orc.run(wl)
        s_ = wl.sched
        nbs = orc.num_blocks(s_.seq_lens, bs)
        for topk in (0, int(nbs.max()), int(nbs.max()) + 5):
            sc, sel, out, lse = orc.sparse(wl, bs, topk)
            for s in range(s_.num_seqs):
                nb = int(nbs[s])
                rows = sel[int(s_.query_offsets[s]):int(s_.query_offsets[s + 1])]
                assert torch.equal(rows[..., :nb], torch.arange(nb, dtype=torch.int32).expand_as(rows[..., :nb]))
                assert bool((rows[..., nb:] == -1).all())
            assert torch.allclose(out, dout, rtol=1e-13, atol=1e-14), (wl.name, topk)
            assert torch.allclose(lse, dlse, rtol=1e-13, atol=1e-14), (wl.name, topk)


def pin_sparse_planted_block(orc):
    """Decode: one key of block b*_s is a large multiple of the proxy query of every KV head, so a
    top-1 selection is b*_s for all heads, and the output equals dense attention restricted to
    the keys of b*_s (key_begin/key_end)."""
    bs = 8
    wl = W.make_gqa("plant", 31, [37, 100, 64, 8], [1, 1, 1, 1], 4, 2, 8, 8, 4, torch.float32, causal=True)
    s_ = wl.sched
    G = 2
    gen = torch.Generator().manual_seed(5)
    kb, ke = [], []
    for s in range(s_.num_seqs):
        L = int(s_.seq_lens[s])
        nb = (L + bs - 1) // bs
        b = int(torch.randint(0, nb, (1,), generator=gen))
        t = min(L - 1, b * bs + int(torch.randint(0, bs, (1,), generator=gen)))
        page = int(s_.block_tables[s, t // s_.page_size])
        for kvh in range(wl.num_kv_heads):
            wl.k_cache[page, t % s_.page_size, kvh] = 40.0 * wl.q[int(s_.query_offsets[s]), kvh * G]
        kb.append(b * bs)
        ke.append(min(L, (b + 1) * bs))
    sc, sel, out, lse = orc.sparse(wl, bs, 1)
    for s in range(s_.num_seqs):
        assert bool((sel[s, :, 0] == kb[s] // bs).all()), (s, sel[s])
    kb_t = torch.tensor(kb, dtype=torch.int32)
    ke_t = torch.tensor(ke, dtype=torch.int32)
    rout, rlse = orc.attention(wl.q, wl.k_cache, wl.v_cache, s_.seq_lens, s_.query_offsets, s_.block_tables,
                               s_.page_size, wl.scale, True, 0, key_begin=kb_t, key_end=ke_t)
    assert torch.equal(out, rout) and torch.equal(lse, rlse)


def pin_sparse_ties_lower_index(orc):
    """Q = 0: every visible block scores exactly 0 and blocks without a visible key -inf, so the
    selection is the lowest-indexed k visible blocks; the output is the mean of V over their
    visible keys and exp(lse) their count."""
    bs = 4
    wl = W.make_gqa("ties", 41, [30, 23, 40], [1, 6, 1], 4, 2, 8, 8, 4, torch.float32, causal=True, window=11)
    wl.q.zero_()
    s_ = wl.sched
    topk = 2
    sc, sel, out, lse = orc.sparse(wl, bs, topk)
    for s in range(s_.num_seqs):
        L = int(s_.seq_lens[s]); q0 = int(s_.query_offsets[s]); n = int(s_.query_offsets[s + 1]) - q0
        V = _dense_kv(wl.v_cache, s_.block_tables, s, L, s_.page_size)
        for j in range(n):
            p = L - n + j
            lo = max(0, p - wl.window + 1)
            first = lo // bs
            want = [first, first + 1] if first + 1 <= p // bs else [first]
            for kvh in range(wl.num_kv_heads):
                got = [b for b in sel[q0 + j, kvh].tolist() if b >= 0]
                assert got == want, (s, j, got, want)
                keys = [t for t in range(lo, p + 1) if t // bs in want]
                ref = V[keys, kvh].mean(dim=0)
                for g in range(2):
                    h = kvh * 2 + g
                    assert torch.allclose(out[q0 + j, h], ref, rtol=1e-13, atol=1e-14)
                    assert abs(math.exp(float(lse[q0 + j, h])) - len(keys)) < 1e-9 * len(keys)


def pin_sparse_alice_fixture(orc):
    """alice-llm bridge tests on `fixture_gqa` (blocks and pages of 4 keys, non-causal): top-k 0
    and top-k 3 (= the block count) match dense attention; top-2 of 3 gives finite values."""
    q, k, v, sl, qo, bt, ps, scale = alice_fixture()
    dout, _ = orc.attention(q, k, v, sl, qo, bt, ps, scale, causal=False, window=0)
    for topk in (0, 3, 2):
        sc = orc.sparse_block_scores(q, k, sl, qo, bt, ps, scale, 4, causal=False)
        sel = orc.sparse_topk(sc, sl, qo, 4, topk)
        out, _ = orc.sparse_attention(q, k, v, sl, qo, bt, ps, scale, 4, sel, causal=False)
        if topk == 2:
            assert bool(torch.isfinite(out).all()) and bool((sel >= 0).sum(-1).eq(2).all())
        else:
            rel = ((out - dout).abs() / dout.abs().clamp_min(1e-6)).max()
            assert rel < 1e-12, (topk, rel)


ALL_PINS = [
    pin_sdpa_bruteforce, pin_alice_fixture_dense, pin_single_key, pin_constant_v_per_kv_head,
    pin_q_zero_counts_and_mean, pin_position_probe, pin_large_score_selects_target,
    pin_page_permutation_invariance, pin_split_equals_unsplit, pin_chunked_equals_oneshot,
    pin_window_cases, pin_gqa_equals_mha_repeated, pin_mla_equals_gqa_concat,
    pin_half_precision_widening, pin_backward_vs_autograd, pin_backward_finite_differences,
    pin_mla_backward_finite_differences,
    pin_sparse_bruteforce, pin_sparse_dense_fallback, pin_sparse_planted_block, pin_sparse_ties_lower_index,
    pin_sparse_alice_fixture,
]
