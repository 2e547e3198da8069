"""fp64 CPU oracle for paged attention (ctypes front end of oracle/pa_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU-baseline leg are
the only callers. The CUDA library neither imports nor links it, and this module imports
nothing from the CUDA package.

Every function returns float64 tensors. Inputs are CPU torch tensors holding the exact
values the GPU sees (fp32, bf16 or fp16); the C code widens them to double.

Pins (tests/test_oracle_pins.py): brute force against torch's fp64 SDPA/logsumexp on tiny
dense cases, closed forms (single key, constant V, Q = 0 -> exp(lse) counts the visible keys,
W = 1 -> own value row, position probe), invariances (page permutation, split == unsplit,
chunked == one-shot prefill, window >= context == no window, GQA == MHA on a repeated cache,
MLA == single-head GQA on a concatenated key), sparse top-K pins (every block selected ==
dense attention, a planted block wins a top-1 selection and then equals attention restricted to
that block, integer-valued scores fix ties exactly, a brute-force restatement on tiny cases), and
compile-time mutants of the C file that the pins must reject.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

from . import build as _build

_DT = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}
_P = ctypes.c_void_p
_I = ctypes.c_int32


class Oracle:
    """One loaded copy of the oracle library (the real one, or a test mutant)."""

    def __init__(self, path: Optional[str] = None):
        if path is None:
            path = _build.build()
        self.path = path
        lib = ctypes.CDLL(path)
        lib.pao_paged_attention.restype = ctypes.c_int
        lib.pao_paged_attention.argtypes = [_P, _P, _P, ctypes.c_int, _P, _P, _I, _P, _I, _I, _I,
                                            _I, _I, _I, _I, ctypes.c_double, ctypes.c_int, _I, _P,
                                            _P, _P, _P, _P, ctypes.c_int]
        lib.pao_mla_attention.restype = ctypes.c_int
        lib.pao_mla_attention.argtypes = [_P, _P, _P, _P, ctypes.c_int, _P, _P, _I, _P, _I, _I, _I,
                                          _I, _I, _I, ctypes.c_double, ctypes.c_int, _I, _P, _P,
                                          _P, _P, _P, ctypes.c_int]
        lib.pao_paged_attention_backward.restype = ctypes.c_int
        lib.pao_paged_attention_backward.argtypes = [_P, _P, _P, _P, ctypes.c_int, _P, _P, _I, _P, _I, _I, _I, _I, _I,
                                                     _I, _I, ctypes.c_double, ctypes.c_int, _I, _P, _P, _P,
                                                     ctypes.c_int]
        lib.pao_sparse_block_scores.restype = ctypes.c_int
        lib.pao_sparse_block_scores.argtypes = [_P, _P, ctypes.c_int, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I,
                                                ctypes.c_double, ctypes.c_int, _I, _I, _I, _P, ctypes.c_int]
        lib.pao_sparse_topk.restype = ctypes.c_int
        lib.pao_sparse_topk.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P]
        lib.pao_sparse_attention.restype = ctypes.c_int
        lib.pao_sparse_attention.argtypes = [_P, _P, _P, ctypes.c_int, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I,
                                             _I, ctypes.c_double, ctypes.c_int, _I, _I, _P, _I, _P, _P, _P,
                                             ctypes.c_int]
        lib.pao_lse_combine.restype = None
        lib.pao_lse_combine.argtypes = [_P, _P, ctypes.c_int64, ctypes.c_int64, _I, _P, _P]
        self.lib = lib

    # -- helpers ---------------------------------------------------------------------------
    @staticmethod
    def _c(t: torch.Tensor, dtype=None) -> torch.Tensor:
        t = t.detach().cpu()
        if dtype is not None:
            t = t.to(dtype)
        return t.contiguous()

    @staticmethod
    def _want(num_rows: int, rows: Optional[Sequence[int]]):
        if rows is None:
            return None
        w = torch.zeros(num_rows, dtype=torch.uint8)
        w[torch.as_tensor(rows, dtype=torch.int64)] = 1
        return w

    @staticmethod
    def _threads(nthreads: Optional[int]) -> int:
        return nthreads if nthreads else (os.cpu_count() or 1)

    # -- paged GQA attention ---------------------------------------------------------------
    def attention(self, q, k_cache, v_cache, seq_lens, query_offsets, block_tables, page_size,
                  scale, causal=True, window=0, key_begin=None, key_end=None, rows=None,
                  nthreads=None):
        """out [Nq, Hq, Dv] float64, lse [Nq, Hq] float64 (rows not asked for stay NaN)."""
        dt = q.dtype
        assert k_cache.dtype == dt and v_cache.dtype == dt and dt in _DT
        q, k_cache, v_cache = self._c(q), self._c(k_cache), self._c(v_cache)
        nq, hq, d = q.shape
        num_pages, ps, hkv, _ = k_cache.shape
        dv = v_cache.shape[3]
        assert ps == page_size
        sl = self._c(seq_lens, torch.int32)
        qo = self._c(query_offsets, torch.int32)
        bt = self._c(block_tables, torch.int32)
        kb = self._c(key_begin, torch.int32) if key_begin is not None else None
        ke = self._c(key_end, torch.int32) if key_end is not None else None
        want = self._want(nq * hq, rows)
        out = torch.full((nq, hq, dv), float("nan"), dtype=torch.float64)
        lse = torch.full((nq, hq), float("nan"), dtype=torch.float64)
        rc = self.lib.pao_paged_attention(
            q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), _DT[dt], sl.data_ptr(),
            qo.data_ptr(), sl.numel(), bt.data_ptr(), bt.shape[1] if bt.dim() == 2 else 0,
            page_size, num_pages, hq, hkv, d, dv, float(scale), int(bool(causal)), int(window),
            kb.data_ptr() if kb is not None else None, ke.data_ptr() if ke is not None else None,
            want.data_ptr() if want is not None else None, out.data_ptr(), lse.data_ptr(),
            self._threads(nthreads))
        if rc != 0:
            raise ValueError(f"oracle rejected the schedule (code {rc})")
        return out, lse

    # -- backward of paged GQA attention -----------------------------------------------------
    def attention_backward(self, q, k_cache, v_cache, d_out, seq_lens, query_offsets, block_tables, page_size,
                           scale, causal=True, window=0, nthreads=None):
        """(dq [Nq, Hq, D], dk [P, ps, Hkv, D], dv [P, ps, Hkv, Dv]) float64 for upstream d_out."""
        dt = q.dtype
        assert k_cache.dtype == dt and v_cache.dtype == dt and d_out.dtype == dt and dt in _DT
        q, k_cache, v_cache, d_out = self._c(q), self._c(k_cache), self._c(v_cache), self._c(d_out)
        nq, hq, d = q.shape
        num_pages, ps, hkv, _ = k_cache.shape
        dv = v_cache.shape[3]
        sl = self._c(seq_lens, torch.int32)
        qo = self._c(query_offsets, torch.int32)
        bt = self._c(block_tables, torch.int32)
        dq = torch.zeros((nq, hq, d), dtype=torch.float64)
        dk = torch.zeros((num_pages, ps, hkv, d), dtype=torch.float64)
        dvv = torch.zeros((num_pages, ps, hkv, dv), dtype=torch.float64)
        rc = self.lib.pao_paged_attention_backward(
            q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), d_out.data_ptr(), _DT[dt], sl.data_ptr(),
            qo.data_ptr(), sl.numel(), bt.data_ptr(), bt.shape[1], page_size, num_pages, hq, hkv, d, dv,
            float(scale), int(bool(causal)), int(window), dq.data_ptr(), dk.data_ptr(), dvv.data_ptr(),
            self._threads(nthreads))
        if rc != 0:
            raise ValueError(f"oracle rejected the schedule (code {rc})")
        return dq, dk, dvv

    # -- backward of MLA absorbed-latent attention ---------------------------------------------
    def mla_backward(self, q_latent, q_rope, latent_cache, rope_cache, d_out, seq_lens, query_offsets,
                     block_tables, page_size, scale, causal=True, window=0, nthreads=None):
        """(d_q_latent [Nq, H, R], d_q_rope [Nq, H, Pr], d_latent [P, ps, 1, R], d_rope [P, ps, 1, Pr])
        float64. MLA is single-head GQA with the key [latent | rope] and the value latent (ruDNN
        `mla` passes the latent as both K and V), so this is the GQA backward on the concatenated key
        and query, split back by columns; the latent's gradient is the sum of its key part and its
        value part."""
        r = q_latent.shape[2]
        q = torch.cat([q_latent, q_rope], dim=2)
        k = torch.cat([latent_cache, rope_cache], dim=3)
        dq, dk, dv = self.attention_backward(q, k, latent_cache, d_out, seq_lens, query_offsets, block_tables,
                                             page_size, scale, causal, window, nthreads)
        return dq[..., :r], dq[..., r:], dk[..., :r] + dv, dk[..., r:]

    # -- MLA absorbed-latent attention ------------------------------------------------------
    def mla(self, q_latent, q_rope, latent_cache, rope_cache, seq_lens, query_offsets,
            block_tables, page_size, scale, causal=True, window=0, key_begin=None, key_end=None,
            rows=None, nthreads=None):
        dt = q_latent.dtype
        q_latent, q_rope = self._c(q_latent), self._c(q_rope)
        latent_cache, rope_cache = self._c(latent_cache), self._c(rope_cache)
        nq, h, r = q_latent.shape
        pr = q_rope.shape[2]
        num_pages, ps = latent_cache.shape[0], latent_cache.shape[1]
        assert ps == page_size and latent_cache.shape[2] == 1
        sl = self._c(seq_lens, torch.int32)
        qo = self._c(query_offsets, torch.int32)
        bt = self._c(block_tables, torch.int32)
        kb = self._c(key_begin, torch.int32) if key_begin is not None else None
        ke = self._c(key_end, torch.int32) if key_end is not None else None
        want = self._want(nq * h, rows)
        out = torch.full((nq, h, r), float("nan"), dtype=torch.float64)
        lse = torch.full((nq, h), float("nan"), dtype=torch.float64)
        rc = self.lib.pao_mla_attention(
            q_latent.data_ptr(), q_rope.data_ptr(), latent_cache.data_ptr(), rope_cache.data_ptr(),
            _DT[dt], sl.data_ptr(), qo.data_ptr(), sl.numel(), bt.data_ptr(), bt.shape[1],
            page_size, num_pages, h, r, pr, float(scale), int(bool(causal)), int(window),
            kb.data_ptr() if kb is not None else None, ke.data_ptr() if ke is not None else None,
            want.data_ptr() if want is not None else None, out.data_ptr(), lse.data_ptr(),
            self._threads(nthreads))
        if rc != 0:
            raise ValueError(f"oracle rejected the schedule (code {rc})")
        return out, lse

    # -- sparse top-K block attention ---------------------------------------------------------
    @staticmethod
    def num_blocks(seq_lens, block_size: int) -> torch.Tensor:
        """Sparse blocks per sequence: ceil(L / block_size) (the last block may be partial)."""
        sl = torch.as_tensor(seq_lens, dtype=torch.int64)
        return (sl + block_size - 1) // block_size

    def sparse_block_scores(self, q, k_cache, seq_lens, query_offsets, block_tables, page_size, scale,
                            block_size, causal=True, window=0, max_blocks=None, nthreads=None):
        """Proxy block scores [Nq, Hkv, max_blocks] float64 (-inf past a sequence's blocks)."""
        dt = q.dtype
        assert k_cache.dtype == dt and dt in _DT
        q, k_cache = self._c(q), self._c(k_cache)
        nq, hq, d = q.shape
        num_pages, ps, hkv, _ = k_cache.shape
        sl = self._c(seq_lens, torch.int32)
        qo = self._c(query_offsets, torch.int32)
        bt = self._c(block_tables, torch.int32)
        if max_blocks is None:
            max_blocks = int(self.num_blocks(sl, block_size).max().item()) if sl.numel() else 0
        scores = torch.full((nq, hkv, max_blocks), float("nan"), dtype=torch.float64)
        rc = self.lib.pao_sparse_block_scores(
            q.data_ptr(), k_cache.data_ptr(), _DT[dt], sl.data_ptr(), qo.data_ptr(), sl.numel(), bt.data_ptr(),
            bt.shape[1], page_size, num_pages, hq, hkv, d, float(scale), int(bool(causal)), int(window),
            int(block_size), int(max_blocks), scores.data_ptr(), self._threads(nthreads))
        if rc != 0:
            raise ValueError(f"oracle rejected the arguments (code {rc})")
        return scores

    def sparse_topk(self, scores, seq_lens, query_offsets, block_size, topk, width=None):
        """Selected blocks [Nq, Hkv, width] int32, ascending, -1 past the row's count."""
        scores = self._c(scores, torch.float64)
        nq, hkv, max_blocks = scores.shape
        sl = self._c(seq_lens, torch.int32)
        qo = self._c(query_offsets, torch.int32)
        if width is None:
            width = topk if topk > 0 else max_blocks
        sel = torch.full((nq, hkv, width), -7, dtype=torch.int32)
        rc = self.lib.pao_sparse_topk(scores.data_ptr(), sl.data_ptr(), qo.data_ptr(), sl.numel(), hkv, max_blocks,
                                      int(block_size), int(topk), int(width), sel.data_ptr())
        if rc != 0:
            raise ValueError(f"oracle rejected the arguments (code {rc})")
        return sel

    def sparse_attention(self, q, k_cache, v_cache, seq_lens, query_offsets, block_tables, page_size, scale,
                         block_size, selection, causal=True, window=0, rows=None, nthreads=None):
        """Attention over the selected blocks: out [Nq, Hq, Dv], lse [Nq, Hq] float64."""
        dt = q.dtype
        assert k_cache.dtype == dt and v_cache.dtype == dt and dt in _DT
        q, k_cache, v_cache = self._c(q), self._c(k_cache), self._c(v_cache)
        nq, hq, d = q.shape
        num_pages, ps, hkv, _ = k_cache.shape
        dv = v_cache.shape[3]
        sl = self._c(seq_lens, torch.int32)
        qo = self._c(query_offsets, torch.int32)
        bt = self._c(block_tables, torch.int32)
        sel = self._c(selection, torch.int32)
        assert sel.shape[0] == nq and sel.shape[1] == hkv
        want = self._want(nq * hq, rows)
        out = torch.full((nq, hq, dv), float("nan"), dtype=torch.float64)
        lse = torch.full((nq, hq), float("nan"), dtype=torch.float64)
        rc = self.lib.pao_sparse_attention(
            q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), _DT[dt], sl.data_ptr(), qo.data_ptr(), sl.numel(),
            bt.data_ptr(), bt.shape[1], page_size, num_pages, hq, hkv, d, dv, float(scale), int(bool(causal)),
            int(window), int(block_size), sel.data_ptr(), sel.shape[2],
            want.data_ptr() if want is not None else None, out.data_ptr(), lse.data_ptr(), self._threads(nthreads))
        if rc == -4:
            raise ValueError("selection entry out of range or repeated")
        if rc != 0:
            raise ValueError(f"oracle rejected the arguments (code {rc})")
        return out, lse

    def sparse(self, wl, block_size, topk, rows=None, nthreads=None):
        """Proxy scores, selection and attention for a GQA workload: (scores, sel, out, lse)."""
        s = wl.sched
        scores = self.sparse_block_scores(wl.q, wl.k_cache, s.seq_lens, s.query_offsets, s.block_tables,
                                          s.page_size, wl.scale, block_size, wl.causal, wl.window,
                                          nthreads=nthreads)
        sel = self.sparse_topk(scores, s.seq_lens, s.query_offsets, block_size, topk)
        out, lse = self.sparse_attention(wl.q, wl.k_cache, wl.v_cache, s.seq_lens, s.query_offsets, s.block_tables,
                                         s.page_size, wl.scale, block_size, sel, wl.causal, wl.window, rows,
                                         nthreads)
        return scores, sel, out, lse

    # -- merge of partial results -------------------------------------------------------------
    def lse_combine(self, o_parts: torch.Tensor, lse_parts: torch.Tensor):
        """o_parts [nparts, rows, dv], lse_parts [nparts, rows] -> (out [rows, dv], lse [rows])."""
        o_parts = self._c(o_parts, torch.float64)
        lse_parts = self._c(lse_parts, torch.float64)
        nparts, rows, dv = o_parts.shape
        out = torch.empty((rows, dv), dtype=torch.float64)
        lse = torch.empty(rows, dtype=torch.float64)
        self.lib.pao_lse_combine(o_parts.data_ptr(), lse_parts.data_ptr(), nparts, rows, dv,
                                 out.data_ptr(), lse.data_ptr())
        return out, lse

    # -- workload conveniences ----------------------------------------------------------------
    def run(self, wl, rows=None, nthreads=None, key_begin=None, key_end=None):
        """Run the oracle on a workload object (GQA or MLA) from the seeded input module."""
        s = wl.sched
        if wl.kind == "mla":
            return self.mla(wl.q_latent, wl.q_rope, wl.latent_cache, wl.rope_cache, s.seq_lens,
                            s.query_offsets, s.block_tables, s.page_size, wl.scale, wl.causal,
                            wl.window, key_begin, key_end, rows, nthreads)
        return self.attention(wl.q, wl.k_cache, wl.v_cache, s.seq_lens, s.query_offsets,
                              s.block_tables, s.page_size, wl.scale, wl.causal, wl.window,
                              key_begin, key_end, rows, nthreads)


_default: Optional[Oracle] = None


def get() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default
