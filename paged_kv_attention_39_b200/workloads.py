"""Seeded synthetic inputs for paged attention: shapes, page pools, block tables, values.

This module holds no attention arithmetic. It only draws numbers and lays them out, and it
is the one piece shared by the CUDA path's tests/bench and by the fp64 oracle's tests: both
receive the very same host tensors.

Recipe (every config):
  * values ~ N(0, 1) drawn in fp32 by torch's CPU generator, in fixed-size chunks each seeded
    from (seed, stream, chunk) so that the result does not depend on thread scheduling, then
    rounded once to the config dtype (round-to-nearest-even, torch's float->bf16/f16 cast);
  * every sequence gets ceil(L_s / page_size) pages drawn without replacement from a pool
    that holds 10% spare pages; the pool order is a seeded random permutation, so the pages
    of one sequence are scattered over the pool;
  * pool pages that no sequence owns, and slots past L_s in a sequence's last page, are
    filled with NaN, and block-table entries past ceil(L_s / page_size) are -1: a kernel
    that reads any of them produces NaN or faults the bounds check, which the parity tests
    would see.

Paged layout (ruDNN `DevicePlan::attention` doc comment): K cache [pages, page_size, Hkv, D],
V cache [pages, page_size, Hkv, Dv], packed Q [queries, Hq, D]. Query j of sequence s sits at
absolute position L_s - n_s + j (right-aligned, L_s counts the sequence's own new keys).
MLA (ruDNN `DevicePlan::mla`): absorbed Q [queries, H, R], position Q [queries, H, P], latent
cache [pages, page_size, 1, R], rope cache [pages, page_size, 1, P].
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from typing import Optional

import torch

_CHUNK = 1 << 22  # elements drawn per independently seeded generator


def _mix(*xs: int) -> int:
    """64-bit mixing of integers into a generator seed (splitmix64 finaliser steps)."""
    h = 0x9E3779B97F4A7C15
    for x in xs:
        h = (h ^ (x & 0xFFFFFFFFFFFFFFFF)) & 0xFFFFFFFFFFFFFFFF
        h = (h * 0xBF58476D1CE4E5B9) & 0xFFFFFFFFFFFFFFFF
        h ^= h >> 31
        h = (h * 0x94D049BB133111EB) & 0xFFFFFFFFFFFFFFFF
        h ^= h >> 29
    return h & 0x7FFFFFFFFFFFFFFF


def randn(shape, seed: int, stream: int, dtype: torch.dtype, out: Optional[torch.Tensor] = None,
          pin: bool = False) -> torch.Tensor:
    """N(0,1) values of `shape`, deterministic in (seed, stream), rounded once to `dtype`."""
    n = 1
    for s in shape:
        n *= int(s)
    if out is None:
        out = torch.empty(n, dtype=dtype, pin_memory=pin and torch.cuda.is_available())
    flat = out.view(-1)
    nchunks = (n + _CHUNK - 1) // _CHUNK

    def fill(c: int) -> None:
        lo = c * _CHUNK
        hi = min(n, lo + _CHUNK)
        g = torch.Generator().manual_seed(_mix(seed, stream, c))
        flat[lo:hi] = torch.randn(hi - lo, generator=g, dtype=torch.float32).to(dtype)

    if nchunks <= 1:
        for c in range(nchunks):
            fill(c)
    else:
        with ThreadPoolExecutor(max_workers=min(16, nchunks)) as ex:
            list(ex.map(fill, range(nchunks)))
    return out.view(*shape)


@dataclass
class Schedule:
    """Per-sequence lengths, packed-query offsets and the page pool's block tables."""
    seq_lens: torch.Tensor        # [S] int32, L_s (includes the sequence's new keys)
    query_offsets: torch.Tensor   # [S+1] int32, prefix sums of n_s
    block_tables: torch.Tensor    # [S, table_width] int32, -1 past the used entries
    page_size: int
    num_pages: int
    owned: torch.Tensor           # [num_pages] bool, page belongs to some sequence

    @property
    def num_seqs(self) -> int:
        return int(self.seq_lens.numel())

    @property
    def num_queries(self) -> int:
        return int(self.query_offsets[-1])

    @property
    def table_width(self) -> int:
        return int(self.block_tables.shape[1])


def make_schedule(seed: int, seq_lens, q_counts, page_size: int, spare_frac: float = 0.10,
                  table_width: Optional[int] = None, min_spare: int = 0) -> Schedule:
    seq_lens = [int(x) for x in seq_lens]
    q_counts = [int(x) for x in q_counts]
    assert len(seq_lens) == len(q_counts)
    for L, n in zip(seq_lens, q_counts):
        assert 0 <= n <= L, (n, L)
    need = [(L + page_size - 1) // page_size for L in seq_lens]
    used = sum(need)
    num_pages = used + max(min_spare, int(math.ceil(used * spare_frac)))
    num_pages = max(num_pages, 1)
    g = torch.Generator().manual_seed(_mix(seed, 0xB10C))
    perm = torch.randperm(num_pages, generator=g).to(torch.int32)
    tw = max(need + [1]) if table_width is None else table_width
    assert tw >= max(need + [0])
    bt = torch.full((len(seq_lens), tw), -1, dtype=torch.int32)
    owned = torch.zeros(num_pages, dtype=torch.bool)
    pos = 0
    for s, k in enumerate(need):
        ids = perm[pos:pos + k]
        bt[s, :k] = ids
        owned[ids.long()] = True
        pos += k
    qo = torch.zeros(len(seq_lens) + 1, dtype=torch.int32)
    if q_counts:
        qo[1:] = torch.cumsum(torch.tensor(q_counts, dtype=torch.int64), 0).to(torch.int32)
    return Schedule(torch.tensor(seq_lens, dtype=torch.int32), qo, bt, page_size, num_pages, owned)


def poison_unused(cache: torch.Tensor, sched: Schedule) -> None:
    """NaN-fill pages no sequence owns and slots past L_s in each sequence's last page."""
    if cache.dtype not in (torch.float32, torch.float16, torch.bfloat16):
        return
    cache[~sched.owned] = float("nan")
    ps = sched.page_size
    for s in range(sched.num_seqs):
        L = int(sched.seq_lens[s])
        k = (L + ps - 1) // ps
        if k and L % ps:
            cache[int(sched.block_tables[s, k - 1]), L % ps:] = float("nan")


@dataclass
class GqaWorkload:
    name: str
    sched: Schedule
    q: torch.Tensor          # [N_q, Hq, D]
    k_cache: torch.Tensor    # [P, ps, Hkv, D]
    v_cache: torch.Tensor    # [P, ps, Hkv, Dv]
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    v_head_dim: int
    scale: float
    causal: bool
    window: int
    kind: str = "gqa"
    note: str = ""


@dataclass
class MlaWorkload:
    name: str
    sched: Schedule
    q_latent: torch.Tensor   # [N_q, H, R]
    q_rope: torch.Tensor     # [N_q, H, P]
    latent_cache: torch.Tensor  # [pages, ps, 1, R]
    rope_cache: torch.Tensor    # [pages, ps, 1, P]
    num_heads: int
    latent_dim: int
    rope_dim: int
    scale: float
    causal: bool
    window: int
    kind: str = "mla"
    note: str = ""


def make_gqa(name: str, seed: int, seq_lens, q_counts, hq: int, hkv: int, d: int, dv: int,
             page_size: int, dtype: torch.dtype, scale: Optional[float] = None,
             causal: bool = True, window: int = 0, spare_frac: float = 0.10,
             pin: bool = False, min_spare: int = 0) -> GqaWorkload:
    sched = make_schedule(seed, seq_lens, q_counts, page_size, spare_frac, min_spare=min_spare)
    nq = sched.num_queries
    q = randn((nq, hq, d), seed, 1, dtype, pin=pin)
    k = randn((sched.num_pages, page_size, hkv, d), seed, 2, dtype, pin=pin)
    v = randn((sched.num_pages, page_size, hkv, dv), seed, 3, dtype, pin=pin)
    poison_unused(k, sched)
    poison_unused(v, sched)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    return GqaWorkload(name, sched, q, k, v, hq, hkv, d, dv, float(scale), bool(causal), int(window))


def make_mla(name: str, seed: int, seq_lens, q_counts, h: int, r: int, pr: int, page_size: int,
             dtype: torch.dtype, scale: Optional[float] = None, causal: bool = True,
             window: int = 0, spare_frac: float = 0.10, pin: bool = False) -> MlaWorkload:
    sched = make_schedule(seed, seq_lens, q_counts, page_size, spare_frac)
    nq = sched.num_queries
    ql = randn((nq, h, r), seed, 11, dtype, pin=pin)
    qr = randn((nq, h, pr), seed, 12, dtype, pin=pin)
    lat = randn((sched.num_pages, page_size, 1, r), seed, 13, dtype, pin=pin)
    rope = randn((sched.num_pages, page_size, 1, pr), seed, 14, dtype, pin=pin)
    poison_unused(lat, sched)
    poison_unused(rope, sched)
    if scale is None:
        scale = 1.0 / math.sqrt(r + pr)
    return MlaWorkload(name, sched, ql, qr, lat, rope, h, r, pr, float(scale), bool(causal), int(window))


def _uniform_ints(seed: int, stream: int, n: int, lo: int, hi: int):
    """n integers uniform in [lo, hi] (inclusive)."""
    g = torch.Generator().manual_seed(_mix(seed, stream))
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g)]


# --- the five workload configurations --------------------------------------------------

def c1_tiny_fp32_decode(seed: int = 0) -> GqaWorkload:
    """2 sequences (context 37 and 100), 1 query each, Hq=4, Hkv=2, D=64, page 16, fp32,
    scale 1/8, causal, no window; a 16-page pool (10 owned, 6 NaN) in random order."""
    sched_lens = [37, 100]
    need = sum((L + 15) // 16 for L in sched_lens)
    wl = make_gqa("tiny_fp32_decode", seed, sched_lens, [1, 1], 4, 2, 64, 64, 16, torch.float32,
                  scale=1.0 / 8.0, causal=True, window=0, spare_frac=0.0, min_spare=16 - need)
    assert wl.sched.num_pages == 16
    return wl


def c2_bf16_decode(seed: int = 0, batch: int = 64, lmin: int = 512, lmax: int = 8192,
                   pin: bool = False) -> GqaWorkload:
    """Batch of decode sequences, context U[lmin, lmax], Hq=32, Hkv=8, D=128, page 16, bf16."""
    lens = _uniform_ints(seed, 0xC2, batch, lmin, lmax)
    return make_gqa(f"bf16_decode_b{batch}_L{lmin}-{lmax}", seed, lens, [1] * batch, 32, 8, 128,
                    128, 16, torch.bfloat16, causal=True, window=0, pin=pin)


def c3_chunked_prefill(seed: int = 0, batch: int = 8, hmax: int = 4096, chunk: int = 512,
                       pin: bool = False) -> GqaWorkload:
    """8 sequences with history U[0, hmax] plus a `chunk`-query chunk, Hq=32, Hkv=8, D=128,
    page 64, bf16, causal at absolute positions."""
    hist = _uniform_ints(seed, 0xC3, batch, 0, hmax)
    lens = [h + chunk for h in hist]
    return make_gqa(f"bf16_chunked_prefill_b{batch}_h0-{hmax}_n{chunk}", seed, lens,
                    [chunk] * batch, 32, 8, 128, 128, 64, torch.bfloat16, causal=True, window=0,
                    pin=pin)


def c4_window_mixed(seed: int = 0, n_decode: int = 16, ctx: int = 32768, n_prefill: int = 4,
                    hist: int = 8192, chunk: int = 1024, window: int = 4096,
                    pin: bool = False) -> GqaWorkload:
    """Decode sequences (context ctx) plus prefill chunks (history hist, `chunk` queries) in one
    batch, Hq=64, Hkv=8, D=128, page 64, sliding window, causal, bf16."""
    lens = [ctx] * n_decode + [hist + chunk] * n_prefill
    qs = [1] * n_decode + [chunk] * n_prefill
    return make_gqa(f"bf16_window{window}_mixed_{n_decode}x{ctx}+{n_prefill}x{hist}+{chunk}",
                    seed, lens, qs, 64, 8, 128, 128, 64, torch.bfloat16, causal=True,
                    window=window, pin=pin)


def c4_decode_part(seed: int = 0, n_decode: int = 16, ctx: int = 32768, window: int = 4096,
                   pin: bool = False) -> GqaWorkload:
    """The decode sub-batch of the window + mixed batch alone: n_decode sequences of context ctx,
    one query each, Hq=64, Hkv=8, D=128, page 64, window, causal, bf16."""
    return make_gqa(f"bf16_window{window}_decode_{n_decode}x{ctx}", seed, [ctx] * n_decode, [1] * n_decode, 64, 8,
                    128, 128, 64, torch.bfloat16, causal=True, window=window, pin=pin)


def c4_prefill_part(seed: int = 0, n_prefill: int = 4, hist: int = 8192, chunk: int = 1024, window: int = 4096,
                    pin: bool = False) -> GqaWorkload:
    """The prefill sub-batch of the window + mixed batch alone: n_prefill chunks of `chunk` queries
    after `hist` keys of history, Hq=64, Hkv=8, D=128, page 64, window, causal, bf16."""
    return make_gqa(f"bf16_window{window}_prefill_{n_prefill}x{hist}+{chunk}", seed, [hist + chunk] * n_prefill,
                    [chunk] * n_prefill, 64, 8, 128, 128, 64, torch.bfloat16, causal=True, window=window, pin=pin)


def c5_mla_decode(seed: int = 0, batch: int = 32, lmin: int = 1024, lmax: int = 16384,
                  pin: bool = False) -> MlaWorkload:
    """MLA absorbed-latent decode: batch, context U[lmin, lmax], H=128, R=512, rope 64,
    page 64, bf16, scale 1/sqrt(576), causal."""
    lens = _uniform_ints(seed, 0xC5, batch, lmin, lmax)
    return make_mla(f"bf16_mla_decode_b{batch}_L{lmin}-{lmax}", seed, lens, [1] * batch, 128,
                    512, 64, 64, torch.bfloat16, scale=1.0 / math.sqrt(576.0), causal=True,
                    pin=pin)


def c2_decode_variant(seed: int = 0, dtype: torch.dtype = torch.float16, d: int = 128, batch: int = 64,
                      pin: bool = False) -> GqaWorkload:
    """The bf16 decode batch's shape (64 sequences, context U[512, 8192], Hq=32, Hkv=8, page 16)
    in another element type or head size (D = Dv = d)."""
    lens = _uniform_ints(seed, 0xC2, batch, 512, 8192)
    tag = {torch.float16: "fp16", torch.bfloat16: "bf16", torch.float32: "fp32"}[dtype]
    return make_gqa(f"{tag}_decode_d{d}_b{batch}", seed, lens, [1] * batch, 32, 8, d, d, 16, dtype,
                    causal=True, window=0, pin=pin)


def c3_prefill_variant(seed: int = 0, dtype: torch.dtype = torch.bfloat16, d: int = 256, batch: int = 8,
                       pin: bool = False) -> GqaWorkload:
    """The chunked-prefill batch's shape (8 sequences, history U[0, 4096] plus a 512-query chunk,
    Hq=32, Hkv=8, page 64, causal) in another element type or head size (D = Dv = d)."""
    hist = _uniform_ints(seed, 0xC3, batch, 0, 4096)
    lens = [h + 512 for h in hist]
    tag = {torch.float16: "fp16", torch.bfloat16: "bf16", torch.float32: "fp32"}[dtype]
    return make_gqa(f"{tag}_chunked_prefill_d{d}_b{batch}", seed, lens, [512] * batch, 32, 8, d, d, 64, dtype,
                    causal=True, window=0, pin=pin)


def append_chunk(seed: int = 0):
    """Paged append of the chunked-prefill batch's new rows (8 sequences x 512 queries, Hkv=8,
    D=Dv=128, pages of 64, bf16): (workload, new_k [Nq, Hkv, D], new_v [Nq, Hkv, Dv])."""
    wl = c3_chunked_prefill(seed)
    nq = wl.sched.num_queries
    new_k = randn((nq, wl.num_kv_heads, wl.head_dim), seed, 21, wl.k_cache.dtype)
    new_v = randn((nq, wl.num_kv_heads, wl.v_head_dim), seed, 22, wl.v_cache.dtype)
    return wl, new_k, new_v


def append_bytes(wl) -> int:
    """Algorithmic HBM bytes of one append: every new K/V row read once and written once."""
    esz = wl.k_cache.element_size()
    return 2 * wl.sched.num_queries * wl.num_kv_heads * (wl.head_dim + wl.v_head_dim) * esz


def backward_chunk(seed: int = 0, batch: int = 4, hmax: int = 2048, chunk: int = 256):
    """Backward of a chunked-prefill batch (history U[0, hmax] plus `chunk` queries, Hq=32,
    Hkv=8, D=128, pages of 64, bf16, causal): (workload, d_out [Nq, Hq, Dv])."""
    wl = c3_chunked_prefill(seed, batch=batch, hmax=hmax, chunk=chunk)
    d_out = randn((wl.sched.num_queries, wl.num_q_heads, wl.v_head_dim), seed, 23, wl.q.dtype)
    return wl, d_out


def backward_flops(wl) -> int:
    """2 flops per multiply-add of the recompute-based backward over visible pairs, every query
    head: the scores q.k (D), dP = dO.v (Dv), dV += P dO (Dv), dQ += dS k (D), dK += dS q (D)."""
    return visible_pairs(wl) * wl.num_q_heads * 2 * (3 * wl.head_dim + 2 * wl.v_head_dim)


def mla_backward_small(seed: int = 0, batch: int = 4, lmin: int = 256, lmax: int = 1024):
    """Backward of a small MLA decode batch (128 heads, latent 512, rope 64, pages of 64, bf16):
    (workload, d_out [Nq, H, R])."""
    lens = _uniform_ints(seed, 0xB5, batch, lmin, lmax)
    wl = make_mla(f"bf16_mla_backward_b{batch}", seed, lens, [1] * batch, 128, 512, 64, 64, torch.bfloat16)
    d_out = randn((wl.sched.num_queries, 128, 512), seed, 24, torch.bfloat16)
    return wl, d_out


def mla_backward_decode_batch(seed: int = 0):
    """Backward of the MLA decode batch (32 sequences, context U[1024, 16384], 128 heads, latent
    512, rope 64, pages of 64, bf16): (workload, d_out [Nq, H, R])."""
    wl = c5_mla_decode(seed)
    d_out = randn((wl.sched.num_queries, 128, 512), seed, 25, torch.bfloat16)
    return wl, d_out


def mla_backward_flops(wl) -> int:
    """2 flops per multiply-add over visible pairs, every head: scores (R + Pr), dP (R), dV (R),
    dQ (R + Pr) and dK (R + Pr)."""
    k = wl.latent_dim + wl.rope_dim
    return visible_pairs(wl) * wl.num_heads * 2 * (3 * k + 2 * wl.latent_dim)


def sparse_bf16_decode(seed: int = 0, block_size: int = 64, topk: int = 16, pin: bool = False):
    """The bf16 decode batch (64 sequences, context U[512, 8192], Hq=32, Hkv=8, D=128, page 16)
    with sparse top-K attention over blocks of `block_size` keys: (workload, block_size, topk).
    Blocks of 64 and a handful of them per query follow the page's bridge (blocks of 64 keys)."""
    return c2_bf16_decode(seed, pin=pin), block_size, topk


def sparse_bytes(wl, block_size: int, selection) -> int:
    """Algorithmic HBM bytes of one sparse step: the proxy pass reads the K row of every key a
    query sees once per (query, KV head); attention reads the K and V rows of the keys it sees in
    the selected blocks (selection [Nq, Hkv, width], -1 = unused)."""
    sched = wl.sched
    esz = wl.k_cache.element_size()
    krow, kvrow = wl.head_dim * esz, (wl.head_dim + wl.v_head_dim) * esz
    sel = selection.cpu()
    total = 0
    W = wl.window
    for s in range(sched.num_seqs):
        L = int(sched.seq_lens[s])
        q0, q1 = int(sched.query_offsets[s]), int(sched.query_offsets[s + 1])
        for qi in range(q0, q1):
            p = L - (q1 - q0) + (qi - q0)
            hi = p + 1 if wl.causal else L
            lo = max(0, p - W + 1) if W > 0 else 0
            total += max(0, hi - lo) * krow * wl.num_kv_heads
            for h in range(wl.num_kv_heads):
                for b in sel[qi, h].tolist():
                    if b < 0:
                        continue
                    a, e = max(lo, b * block_size), min(hi, (b + 1) * block_size)
                    total += max(0, e - a) * kvrow
    return total


FULL_CONFIGS = {
    "tiny_fp32_decode": c1_tiny_fp32_decode,
    "bf16_decode": c2_bf16_decode,
    "bf16_chunked_prefill": c3_chunked_prefill,
    "bf16_window_mixed": c4_window_mixed,
    "bf16_mla_decode": c5_mla_decode,
}


def algorithmic_kv_bytes(wl) -> int:
    """Bytes of K/V (or latent/rope) rows that the mask lets some query of a sequence see.

    Each visible (token, kv head) row is counted once per sequence, whatever number of query
    heads or queries read it: that is the minimum a kernel must bring in from HBM.
    """
    sched = wl.sched
    total = 0
    if wl.kind == "gqa":
        esz = wl.k_cache.element_size()
        per_tok = wl.num_kv_heads * (wl.head_dim + wl.v_head_dim) * esz
    else:
        esz = wl.latent_cache.element_size()
        per_tok = (wl.latent_dim + wl.rope_dim) * esz
    for s in range(sched.num_seqs):
        L = int(sched.seq_lens[s])
        n = int(sched.query_offsets[s + 1] - sched.query_offsets[s])
        if n == 0:
            continue
        p_first, p_last = L - n, L - 1
        lo = max(0, p_first - wl.window + 1) if wl.window > 0 else 0
        hi = p_last + 1 if wl.causal else L
        total += max(0, hi - lo) * per_tok
    return total


def visible_pairs(wl) -> int:
    """Number of (query, key) pairs the mask keeps, summed over sequences (per query head)."""
    sched = wl.sched
    total = 0
    W = wl.window
    for s in range(sched.num_seqs):
        L = int(sched.seq_lens[s])
        n = int(sched.query_offsets[s + 1] - sched.query_offsets[s])
        for j in range(n):
            p = L - n + j
            hi = p if wl.causal else L - 1
            lo = max(0, p - W + 1) if W > 0 else 0
            total += max(0, hi - lo + 1)
    return total


def algorithmic_flops(wl) -> int:
    """2 flops per multiply-add of QK^T and PV over visible pairs, every query head."""
    pairs = visible_pairs(wl)
    if wl.kind == "gqa":
        return pairs * wl.num_q_heads * 2 * (wl.head_dim + wl.v_head_dim)
    return pairs * wl.num_heads * 2 * (wl.latent_dim + wl.rope_dim + wl.latent_dim)
