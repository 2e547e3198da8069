"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI and compare it
with the fp64 oracle on the same seeded inputs.

Tolerances (fixed for the path in the design notes, checked here):
  fp32 inputs : max |out - ref| <= 1e-5 * max|ref|   and  |lse - ref| <= 1e-5 * max(1, |ref|)
  bf16 / fp16 : |out - ref| <= 1e-2 + 2e-2 * |ref| elementwise, and |lse - ref| <= 2e-3
Rows the mask leaves empty must come back exactly as out = 0, lse = -inf.

Every comparison records its measured error (largest |out - ref|, the largest ratio of
|out - ref| to its allowed bound, largest lse error) in MARGINS; the session summary prints them
(tests/conftest.py), so that a passing run still shows how much room each case has.
"""
import math
import os

import torch

import paged_kv_attention_39_b200 as pa

# (tag, dtype, rows compared, max |dout|, max |dout| / allowed, max |dlse| (fp32: relative),
#  max |dlse| / allowed), one entry per check() call
MARGINS = []


def to_dev(t):
    return t.cuda() if t is not None else None


def run_gqa(wl, kv_chunk=0, path=pa.PA_PATH_AUTO, plan=None, q=None):
    s = wl.sched
    own = plan is None
    if own:
        plan = pa.plan_for(wl)
    qd = to_dev(wl.q if q is None else q)
    kd, vd = to_dev(wl.k_cache), to_dev(wl.v_cache)
    out = torch.full((qd.shape[0], wl.num_q_heads, wl.v_head_dim), float("nan"), dtype=qd.dtype, device="cuda")
    lse = torch.full((qd.shape[0], wl.num_q_heads), float("nan"), dtype=torch.float32, device="cuda")
    pa.pa_forward(plan, qd, kd, vd, out, lse, wl.scale, wl.causal, wl.window, kv_chunk=kv_chunk, path=path)
    torch.cuda.synchronize()
    if own:
        plan.close()
    return out.cpu(), lse.cpu()


def run_mla(wl, kv_chunk=0, path=pa.PA_PATH_AUTO):
    plan = pa.plan_for(wl)
    ql, qr = to_dev(wl.q_latent), to_dev(wl.q_rope)
    lat, rope = to_dev(wl.latent_cache), to_dev(wl.rope_cache)
    nq = ql.shape[0]
    out = torch.full((nq, wl.num_heads, wl.latent_dim), float("nan"), dtype=ql.dtype, device="cuda")
    lse = torch.full((nq, wl.num_heads), float("nan"), dtype=torch.float32, device="cuda")
    pa.pa_mla_forward(plan, ql, qr, lat, rope, out, lse, wl.scale, wl.causal, wl.window,
                      kv_chunk=kv_chunk, path=path)
    torch.cuda.synchronize()
    plan.close()
    return out.cpu(), lse.cpu()


def run(wl, **kw):
    return run_mla(wl, **kw) if wl.kind == "mla" else run_gqa(wl, **kw)


def check(wl, out, lse, ref_out, ref_lse, rows=None, tag=""):
    """Compare GPU results with the oracle on all rows (or the flat (query*H + head) rows)."""
    H = out.shape[1]
    o = out.double().reshape(-1, out.shape[-1])
    l = lse.double().reshape(-1)
    ro = ref_out.reshape(-1, ref_out.shape[-1])
    rl = ref_lse.reshape(-1)
    if rows is not None:
        idx = torch.as_tensor(rows, dtype=torch.int64)
        o, l, ro, rl = o[idx], l[idx], ro[idx], rl[idx]
    empty = torch.isinf(rl) & (rl < 0)
    assert torch.equal(l[empty], rl[empty]) and bool((o[empty] == 0).all()), f"{tag}: empty rows"
    o, l, ro, rl = o[~empty], l[~empty], ro[~empty], rl[~empty]
    assert torch.isfinite(o).all() and torch.isfinite(l).all(), f"{tag}: non-finite output"
    cur = os.environ.get("PYTEST_CURRENT_TEST", "")
    name = cur.split("::")[-1].split(" ")[0] if cur else ""
    tag = f"{name} {tag}".strip()
    dt = out.dtype
    diff = (o - ro).abs()
    err = float(diff.max()) if ro.numel() else 0.0
    if dt == torch.float32:
        scale = max(float(ro.abs().max()) if ro.numel() else 1.0, 1e-30)
        lrel = (l - rl).abs() / rl.abs().clamp_min(1.0)
        lerr = float(lrel.max()) if rl.numel() else 0.0
        MARGINS.append((tag, "fp32", int(o.shape[0]), err, err / (1e-5 * scale), lerr, lerr / 1e-5))
        assert err <= 1e-5 * scale, f"{tag}: out max err {err} > 1e-5 * {scale}"
        assert lerr <= 1e-5, f"{tag}: lse rel err {lerr}"
    else:
        bound = 1e-2 + 2e-2 * ro.abs()
        ratio = float((diff / bound).max()) if ro.numel() else 0.0
        lerr = float((l - rl).abs().max()) if rl.numel() else 0.0
        MARGINS.append((tag, str(dt).replace("torch.", ""), int(o.shape[0]), err, ratio, lerr, lerr / 2e-3))
        bad = diff > bound
        assert not bool(bad.any()), f"{tag}: out err {err} at {int(bad.sum())} elems"
        assert lerr <= 2e-3, f"{tag}: lse err {lerr}"
    return H


def visible_count(L, n, j, causal, window):
    p = L - n + j
    hi = p if causal else L - 1
    lo = max(0, p - window + 1) if window > 0 else 0
    return max(0, hi - lo + 1), lo, hi


def sample_rows(wl, k, seed=0):
    """k random flat (query * H + head) rows, always including the first and last."""
    nq = wl.sched.num_queries
    H = wl.num_q_heads if wl.kind == "gqa" else wl.num_heads
    g = torch.Generator().manual_seed(seed)
    rows = torch.randint(0, nq * H, (k,), generator=g).tolist()
    return sorted(set(rows + [0, nq * H - 1]))
