"""GPU parity of the MLA absorbed-latent path (tensor-core decode kernel; CUDA-core kernel for
other shapes) against the fp64 oracle, through the C ABI."""
import math

import pytest
import torch

import paged_kv_attention_39_b200 as pa
from gpu_helpers import check, run_mla, sample_rows, visible_count
from paged_kv_attention_39_b200 import workloads as W

pytestmark = pytest.mark.gpu


def mla_wl(seed, h=128, dtype=torch.bfloat16, batch=6, lmin=1, lmax=3000, ps=64, window=0, qn=1, r=512, pr=64):
    lens = W._uniform_ints(seed, 55, batch, max(lmin, qn), lmax)
    return W.make_mla("small_mla", seed, lens, [qn] * batch, h, r, pr, ps, dtype,
                      scale=1.0 / math.sqrt(r + pr), window=window)


@pytest.mark.parametrize("kv_chunk", [0, -1, 64, 100, 1000])
def test_mla_decode(orc, kv_chunk):
    wl = mla_wl(1)
    ref = orc.run(wl)
    out, lse = run_mla(wl, kv_chunk=kv_chunk)
    check(wl, out, lse, *ref, tag=f"mla chunk {kv_chunk}")


@pytest.mark.parametrize("h", [1, 16, 64, 100])
def test_mla_fewer_heads(orc, h):
    wl = mla_wl(2, h=h)
    ref = orc.run(wl)
    out, lse = run_mla(wl)
    check(wl, out, lse, *ref, tag=f"mla H{h}")


@pytest.mark.parametrize("ps", [16, 32, 128, 256])
def test_mla_page_sizes(orc, ps):
    wl = mla_wl(3, ps=ps, lmax=1500)
    ref = orc.run(wl)
    out, lse = run_mla(wl, kv_chunk=96)
    check(wl, out, lse, *ref, tag=f"mla ps{ps}")


def test_mla_fp16_and_window(orc):
    wl = mla_wl(4, dtype=torch.float16, window=333)
    ref = orc.run(wl)
    out, lse = run_mla(wl, kv_chunk=128)
    check(wl, out, lse, *ref, tag="mla fp16 window")


def test_mla_other_shapes_on_cuda_cores(orc):
    """Several queries per sequence, a rope width other than 64, fp32: the CUDA-core kernel."""
    for wl in (mla_wl(5, h=16, qn=3, lmax=400), mla_wl(6, h=8, r=256, pr=32, lmax=300),
               mla_wl(7, h=8, dtype=torch.float32, lmax=300)):
        ref = orc.run(wl)
        out, lse = run_mla(wl)
        check(wl, out, lse, *ref, tag=f"mla other {wl.q_latent.dtype} {wl.latent_dim}/{wl.rope_dim}")


def test_mla_mask_bit_exact_by_counts():
    for window in (0, 77):
        wl = mla_wl(8, window=window, lmax=2000)
        wl.q_latent.zero_(); wl.q_rope.zero_()
        out, lse = run_mla(wl, kv_chunk=160)
        s = wl.sched
        for si in range(s.num_seqs):
            L = int(s.seq_lens[si]); q0 = int(s.query_offsets[si])
            cnt = visible_count(L, 1, 0, True, window)[0]
            got = torch.exp(lse[q0].double()).round().long()
            assert bool((got == cnt).all()), (window, si, got[:4].tolist(), cnt)


def test_mla_indexing_bit_exact():
    """q_lat / q_rope = a large multiple of one visible key's latent / rope rows: out must equal
    that latent row exactly (read through the shuffled table, NaN pages around)."""
    wl = mla_wl(9, lmax=1200, dtype=torch.float32)
    s = wl.sched
    g = torch.Generator().manual_seed(4)
    targets = {}
    for si in range(s.num_seqs):
        L = int(s.seq_lens[si]); q0 = int(s.query_offsets[si])
        t = torch.arange(L)
        lat = wl.latent_cache[s.block_tables[si, t // s.page_size].long(), t % s.page_size, 0].double()
        rope = wl.rope_cache[s.block_tables[si, t // s.page_size].long(), t % s.page_size, 0].double()
        kcat = torch.cat([lat, rope], dim=1)
        for h in range(wl.num_heads):
            for _ in range(8):
                ts = int(torch.randint(0, L, (1,), generator=g))
                dots = kcat @ kcat[ts]
                own = float(dots[ts]); dots[ts] = float("-inf")
                gap = own - (float(dots.max()) if L > 1 else own - 1.0)
                if gap > 1e-3 * own:
                    break
            alpha = 120.0 / (wl.scale * gap)
            wl.q_latent[q0, h] = (alpha * lat[ts]).float()
            wl.q_rope[q0, h] = (alpha * rope[ts]).float()
            targets[(q0, h)] = (si, ts)
    for name in ("q_latent", "q_rope", "latent_cache", "rope_cache"):
        setattr(wl, name, getattr(wl, name).to(torch.bfloat16))
    out, lse = run_mla(wl, kv_chunk=256)
    for (qi, h), (si, ts) in targets.items():
        page = int(s.block_tables[si, ts // s.page_size])
        assert torch.equal(out[qi, h], wl.latent_cache[page, ts % s.page_size, 0]), (qi, h, si, ts)


@pytest.mark.slow
def test_full_size_mla_decode_sampled(orc):
    """The full MLA workload (batch 32, context U[1024, 16384], 128 heads, R 512, rope 64,
    pages of 64) in the benchmark's launch configuration, on sampled rows."""
    wl = W.c5_mla_decode(0)
    rows = sample_rows(wl, 256, seed=5)
    ref = orc.run(wl, rows=rows)
    out, lse = run_mla(wl)
    check(wl, out, lse, *ref, rows=rows, tag="full mla")
