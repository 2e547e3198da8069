"""C ABI on the host (no GPU): the library loads, exports what include/pa.h declares, and
rejects bad arguments with the documented status before touching a device.

ruDNN's paged_attention/mod.rs validates every operand (`check_tensor`, `bounded`,
`execute_attention_into`) before any allocation or launch; these tests pin the same order
through host-only plans (device -1), which own no device memory.
"""
import ctypes
import os
import re

import pytest
import torch

import paged_kv_attention_39_b200 as pa
from paged_kv_attention_39_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from paged_kv_attention_39_b200 import build
    build.build()
    return pa.load_library()


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "pa.h")).read()
    return sorted(set(re.findall(r"^\s*(?:pa_status|const char\s*\*)\s*(pa_\w+)\s*\(", src, re.M)))


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(pa.SYMBOLS) == names


def test_status_strings(lib):
    for i, name in enumerate(pa.STATUS):
        assert pa.pa_status_string(i) == name
    assert pa.pa_version().count(".") == 2


def host_plan(**kw):
    wl = W.make_gqa("h", 1, [37, 100], [1, 5], 4, 2, 64, 64, 16, torch.bfloat16)
    s = wl.sched
    args = dict(seq_lens=s.seq_lens, query_offsets=s.query_offsets, block_tables=s.block_tables,
                page_size=s.page_size, num_pages=s.num_pages, device=-1)
    args.update(kw)
    return wl, pa.pa_plan_create(**args)


def expect(status_name, fn, *a, **k):
    with pytest.raises(pa.PaError) as ei:
        fn(*a, **k)
    assert ei.value.name == status_name, str(ei.value)


def test_plan_create_validation(lib):
    wl, plan = host_plan()
    info = pa.pa_plan_get_info(plan)
    assert info["num_queries"] == 6 and info["device"] == -1 and info["workspace_bytes"] == 0
    s = wl.sched
    bad = s.block_tables.clone(); bad[1, 3] = s.num_pages
    expect("PA_ERR_BOUNDS", pa.pa_plan_create, s.seq_lens, s.query_offsets, bad, 16, s.num_pages, device=-1)
    bad = s.block_tables.clone(); bad[0, 0] = -1
    expect("PA_ERR_BOUNDS", pa.pa_plan_create, s.seq_lens, s.query_offsets, bad, 16, s.num_pages, device=-1)
    expect("PA_ERR_BOUNDS", pa.pa_plan_create, s.seq_lens, s.query_offsets, s.block_tables[:, :2], 16,
           s.num_pages, device=-1)  # table too narrow for 37 keys in pages of 16
    expect("PA_ERR_INVALID_ARGUMENT", pa.pa_plan_create, [3, 100], [0, 5, 6], s.block_tables, 16,
           s.num_pages, device=-1)  # 5 queries but only 3 keys
    expect("PA_ERR_INVALID_ARGUMENT", pa.pa_plan_create, s.seq_lens, [1, 2, 3], s.block_tables, 16,
           s.num_pages, device=-1)
    expect("PA_ERR_INVALID_ARGUMENT", pa.pa_plan_create, s.seq_lens, [0, 3, 2], s.block_tables, 16,
           s.num_pages, device=-1)
    expect("PA_ERR_INVALID_ARGUMENT", pa.pa_plan_create, s.seq_lens, s.query_offsets, s.block_tables, 0,
           s.num_pages, device=-1)
    expect("PA_ERR_INVALID_ARGUMENT", pa.pa_plan_create, [-1, 100], [0, 0, 1], s.block_tables, 16,
           s.num_pages, device=-1)
    # entries past the used count are never read, so they may hold anything
    odd = s.block_tables.clone(); odd[0, 3:] = 123456
    pa.pa_plan_create(s.seq_lens, s.query_offsets, odd, 16, s.num_pages, device=-1).close()
    # an empty batch is a valid plan
    pa.pa_plan_create([], [0], torch.zeros(0, 0, dtype=torch.int32), 16, 0, device=-1).close()


def fake_ptrs(wl):
    """Disjoint, 256-byte aligned fake addresses standing in for device buffers."""
    base = 1 << 40
    sizes = [wl.q.numel() * 2, wl.k_cache.numel() * 2, wl.v_cache.numel() * 2,
             wl.q.shape[0] * wl.q.shape[1] * wl.v_head_dim * 2, wl.q.shape[0] * wl.q.shape[1] * 4]
    out = []
    for sz in sizes:
        out.append(base)
        base += (sz + 4095) // 4096 * 4096 + 4096
    return out


def call(lib, plan, ptrs, hq=4, hkv=2, d=64, dv=64, scale=0.125, causal=1, window=0, dtype=1, opts=None):
    q, k, v, o, l = ptrs
    st = lib.pa_forward_ex(plan.handle, q, k, v, dtype, hq, hkv, d, dv, ctypes.c_float(scale), causal,
                           window, o, l, None, opts)
    return pa.STATUS[st], pa.pa_last_error_message()


def test_forward_validation_order(lib):
    wl, plan = host_plan()
    p = fake_ptrs(wl)
    assert call(lib, plan, p)[0] == "PA_ERR_INVALID_ARGUMENT"  # all valid -> host-only plan refusal
    assert "host-only" in call(lib, plan, p)[1]
    assert call(lib, plan, p, hq=6, hkv=4)[0] == "PA_ERR_SHAPE"
    assert call(lib, plan, p, hq=0)[0] == "PA_ERR_SHAPE"
    assert call(lib, plan, p, d=0)[0] == "PA_ERR_SHAPE"
    assert call(lib, plan, p, d=2048)[0] == "PA_ERR_UNSUPPORTED"
    assert call(lib, plan, p, scale=0.0)[0] == "PA_ERR_INVALID_ARGUMENT"
    assert call(lib, plan, p, scale=float("nan"))[0] == "PA_ERR_INVALID_ARGUMENT"
    assert call(lib, plan, p, scale=-1.0)[0] == "PA_ERR_INVALID_ARGUMENT"
    assert call(lib, plan, p, window=-3)[0] == "PA_ERR_INVALID_ARGUMENT"
    assert call(lib, plan, p, causal=2)[0] == "PA_ERR_INVALID_ARGUMENT"
    assert call(lib, plan, p, dtype=7)[0] == "PA_ERR_DTYPE"
    q, k, v, o, l = p
    assert call(lib, plan, [q, k, v, q, l])[0] == "PA_ERR_ALIAS"          # out over q
    assert call(lib, plan, [q, k, v, o, k + 64])[0] == "PA_ERR_ALIAS"     # lse inside K
    assert call(lib, plan, [q, k, v, o, o + 32])[0] == "PA_ERR_ALIAS"     # lse inside out
    assert call(lib, plan, [q, k, v, o + 8, l])[0] == "PA_ERR_INVALID_ARGUMENT"  # misaligned
    assert call(lib, plan, [q, k, None, o, l])[0] == "PA_ERR_INVALID_ARGUMENT"
    assert call(lib, plan, p, opts=ctypes.byref(pa._Options(-5, 0, None)))[0] == "PA_ERR_INVALID_ARGUMENT"
    assert call(lib, plan, p, opts=ctypes.byref(pa._Options(0, 9, None)))[0] == "PA_ERR_INVALID_ARGUMENT"
    assert lib.pa_forward_ex(None, q, k, v, 1, 4, 2, 64, 64, ctypes.c_float(1.0), 1, 0, o, l, None, None) == 1


def test_mla_validation(lib):
    wl, plan = host_plan()
    q, k, v, o, l = fake_ptrs(wl)
    def mla(pr=64, r=512, h=4, scale=0.1):
        st = lib.pa_mla_forward_ex(plan.handle, q, k + (1 << 30), k, v, 1, h, r, pr, ctypes.c_float(scale), 1, 0,
                                   o + (1 << 31), l + (1 << 32), None, None)
        return pa.STATUS[st]
    assert mla() == "PA_ERR_INVALID_ARGUMENT"  # host-only plan
    assert mla(pr=0) == "PA_ERR_SHAPE"
    assert mla(pr=300) == "PA_ERR_SHAPE"
    assert mla(r=1500) == "PA_ERR_UNSUPPORTED"


def test_empty_batch_is_ok_without_launch(lib):
    plan = pa.pa_plan_create([5], [0, 0], torch.zeros(1, 1, dtype=torch.int32), 16, 1, device=-1)
    st = lib.pa_forward_ex(plan.handle, None, None, None, 1, 4, 2, 64, 64, ctypes.c_float(1.0), 1, 0,
                           None, None, None, None)
    assert pa.STATUS[st] == "PA_OK"


def test_binding_functions_compile_their_calls():
    """Every binding wrapper resolves the globals it loads (a typo would only show on a GPU)."""
    import builtins
    import dis
    names = [n for n in dir(pa) if n.startswith("pa_") and callable(getattr(pa, n))] + ["plan_for", "trace_events"]
    assert {"pa_backward", "pa_mla_backward", "pa_append", "pa_sparse_select", "pa_sparse_forward"} <= set(names)
    for name in names:
        fn = getattr(pa, name)
        for ins in dis.get_instructions(fn):
            if ins.opname == "LOAD_GLOBAL":
                g = ins.argval
                assert hasattr(pa, g) or hasattr(builtins, g), (name, g)
    # host-only plan: pa_plan_prepare reaches the library and is refused there
    plan = pa.pa_plan_create([5], [0, 1], torch.zeros(1, 1, dtype=torch.int32), 16, 1, device=-1)
    with pytest.raises(pa.PaError):
        pa.pa_plan_prepare(plan, torch.bfloat16, 4, 2, 64, 64)


def test_append_validation(lib):
    wl, plan = host_plan()
    q, k, v, o, l = fake_ptrs(wl)
    def app(nk=q, nv=q + 4096 * 64, kc=k, vc=v, hkv=2, d=64, dv=64, dtype=1, pl=plan):
        return pa.STATUS[lib.pa_append(pl.handle, nk, nv, kc, vc, dtype, hkv, d, dv, None)]
    assert app() == "PA_ERR_INVALID_ARGUMENT"          # host-only plan, after all checks
    assert app(kc=k, vc=k) == "PA_ERR_ALIAS"            # caches overlap
    assert app(nk=k) == "PA_ERR_ALIAS"                  # new rows inside a cache
    assert app(d=4) == "PA_ERR_UNSUPPORTED"             # 8-byte rows
    assert app(hkv=0) == "PA_ERR_SHAPE"
    assert app(dtype=9) == "PA_ERR_DTYPE"
    # two sequences that append into the same page slot
    bt = torch.tensor([[0, 1], [0, 1]], dtype=torch.int32)
    shared = pa.pa_plan_create([20, 20], [0, 1, 2], bt, 16, 4, device=-1)
    assert app(pl=shared) == "PA_ERR_ALIAS"


def test_sparse_validation(lib):
    """pa_sparse_select / pa_sparse_forward check every argument before the host-only refusal.
    Plan: L = 37 and 100 keys in pages of 16, so blocks of 16 keys give 3 and 7 blocks."""
    wl, plan = host_plan()
    q, k, v, o, l = fake_ptrs(wl)
    sel = l + (1 << 30)
    scores = sel + (1 << 30)
    def select(bs=16, topk=4, width=4, sc=None, scw=0, s=sel, hq=4, hkv=2, d=64, scale=0.125, causal=1, window=0):
        st = lib.pa_sparse_select(plan.handle, q, k, 1, hq, hkv, d, ctypes.c_float(scale), causal, window, bs, topk, s,
                                  width, sc, scw, None)
        return pa.STATUS[st]
    assert select() == "PA_ERR_INVALID_ARGUMENT"          # all valid -> host-only plan refusal
    assert "host-only" in pa.pa_last_error_message()
    assert select(bs=24) == "PA_ERR_SHAPE"                # not a multiple of the page size
    assert select(bs=0) == "PA_ERR_SHAPE"
    assert select(width=3) == "PA_ERR_SHAPE"              # the longer sequence keeps 4 blocks
    assert select(topk=0, width=6) == "PA_ERR_SHAPE"      # every block: 7 for the longer one
    assert select(topk=0, width=7) == "PA_ERR_INVALID_ARGUMENT"
    assert select(topk=9, width=7) == "PA_ERR_INVALID_ARGUMENT"  # topk above the block count: all 7
    assert select(sc=scores, scw=6) == "PA_ERR_SHAPE"     # scores need 7 columns
    assert select(sc=scores, scw=7) == "PA_ERR_INVALID_ARGUMENT"
    assert select(topk=-1) == "PA_ERR_INVALID_ARGUMENT"
    assert select(s=q) == "PA_ERR_ALIAS"                  # selection over q
    assert select(sc=k, scw=7) == "PA_ERR_ALIAS"          # scores inside K
    assert select(s=None) == "PA_ERR_INVALID_ARGUMENT"
    assert select(hq=5) == "PA_ERR_SHAPE"
    assert select(d=2048) == "PA_ERR_UNSUPPORTED"
    assert select(scale=0.0) == "PA_ERR_INVALID_ARGUMENT"
    def fwd(bs=16, width=4, s=sel, out=o, lse=l):
        st = lib.pa_sparse_forward(plan.handle, q, k, v, 1, 4, 2, 64, 64, ctypes.c_float(0.125), 1, 0, bs, s, width,
                                   out, lse, None)
        return pa.STATUS[st]
    assert fwd() == "PA_ERR_INVALID_ARGUMENT" and "host-only" in pa.pa_last_error_message()
    assert fwd(bs=24) == "PA_ERR_SHAPE"
    assert fwd(bs=0) == "PA_ERR_SHAPE"
    assert fwd(width=-1) == "PA_ERR_SHAPE"
    assert fwd(s=None) == "PA_ERR_INVALID_ARGUMENT"
    assert fwd(out=sel) == "PA_ERR_ALIAS"                  # out over the selection
    assert fwd(s=sel + 2) == "PA_ERR_INVALID_ARGUMENT"     # misaligned selection
    # more blocks than PA_SPARSE_MAX_BLOCKS in one sequence
    L = (pa.PA_SPARSE_MAX_BLOCKS + 1) * 16
    big = pa.pa_plan_create([L], [0, 1], torch.arange(L // 16, dtype=torch.int32).view(1, -1), 16, L // 16, device=-1)
    st = lib.pa_sparse_select(big.handle, q, k, 1, 4, 2, 64, ctypes.c_float(0.1), 1, 0, 16, 4, sel, 4, None, 0, None)
    assert pa.STATUS[st] == "PA_ERR_UNSUPPORTED"
    assert pa.STATUS[lib.pa_sparse_select(big.handle, q, k, 1, 4, 2, 64, ctypes.c_float(0.1), 1, 0, 32, 4, sel, 4,
                                          None, 0, None)] == "PA_ERR_INVALID_ARGUMENT"  # blocks of 32: fits


def test_mla_backward_validation(lib):
    """pa_mla_backward checks shapes, scalars, pointers and aliasing before the device: a host-only
    plan gets past every check only to be refused for having no device."""
    wl, plan = host_plan()
    base = 1 << 36
    ptr = [base + (i << 32) for i in range(11)]  # disjoint, 16-byte aligned fake ranges
    f = ctypes.c_float

    def call(r=512, pr=64, h=4, scale=0.1, causal=1, window=0, dt=1, p=None):
        a = list(ptr if p is None else p)
        st = lib.pa_mla_backward(plan.handle, a[0], a[1], a[2], a[3], a[4], a[5], a[6], dt, h, r, pr, f(scale), causal,
                                 window, a[7], a[8], a[9], a[10], None)
        return pa.STATUS[st]
    assert call() == "PA_ERR_INVALID_ARGUMENT"  # host-only plan: every check passed
    assert call(dt=7) == "PA_ERR_DTYPE"
    assert call(h=0) == "PA_ERR_SHAPE"
    assert call(r=2000) == "PA_ERR_UNSUPPORTED"
    assert call(pr=0) == "PA_ERR_UNSUPPORTED"
    assert call(pr=300) == "PA_ERR_UNSUPPORTED"
    assert call(scale=float("nan")) == "PA_ERR_INVALID_ARGUMENT"
    assert call(causal=2) == "PA_ERR_INVALID_ARGUMENT"
    assert call(window=-1) == "PA_ERR_INVALID_ARGUMENT"
    aliased = list(ptr)
    aliased[9] = aliased[7]  # d_latent_cache on top of d_q_latent
    assert call(p=aliased) == "PA_ERR_ALIAS"
    over_input = list(ptr)
    over_input[10] = over_input[2]  # d_rope_cache on the latent cache
    assert call(p=over_input) == "PA_ERR_ALIAS"
    misaligned = list(ptr)
    misaligned[8] += 4
    assert call(p=misaligned) == "PA_ERR_INVALID_ARGUMENT"
    null = list(ptr)
    null[6] = 0
    assert call(p=null) == "PA_ERR_INVALID_ARGUMENT"
    plan.close()


def test_backward_wrappers_marshal_to_the_library():
    """pa_backward / pa_mla_backward called through the Python binding with CPU tensors on a
    host-only plan: every argument reaches the C entry point (a wrong argument list would raise in
    ctypes), which passes its checks and refuses the plan for having no device."""
    wl, plan = host_plan()
    nq, hq, d = wl.q.shape
    f32 = torch.float32
    out = torch.zeros(nq, hq, d, dtype=wl.q.dtype)
    lse = torch.zeros(nq, hq, dtype=f32)
    with pytest.raises(pa.PaError) as ei:
        pa.pa_backward(plan, wl.q, wl.k_cache, wl.v_cache, out, lse, out.clone(), torch.zeros(nq, hq, d, dtype=f32),
                       torch.zeros(wl.k_cache.shape, dtype=f32), torch.zeros(wl.v_cache.shape, dtype=f32), 0.125)
    assert pa.STATUS[ei.value.status] == "PA_ERR_INVALID_ARGUMENT" and "host-only" in str(ei.value)
    h, r, pr = 4, 32, 16
    pages, ps = wl.k_cache.shape[0], wl.k_cache.shape[1]
    bf = torch.bfloat16
    with pytest.raises(pa.PaError) as ei:
        pa.pa_mla_backward(plan, torch.zeros(nq, h, r, dtype=bf), torch.zeros(nq, h, pr, dtype=bf),
                           torch.zeros(pages, ps, 1, r, dtype=bf), torch.zeros(pages, ps, 1, pr, dtype=bf),
                           torch.zeros(nq, h, r, dtype=bf), torch.zeros(nq, h, dtype=f32), torch.zeros(nq, h, r, dtype=bf),
                           torch.zeros(nq, h, r, dtype=f32), torch.zeros(nq, h, pr, dtype=f32),
                           torch.zeros(pages, ps, 1, r, dtype=f32), torch.zeros(pages, ps, 1, pr, dtype=f32), 0.1)
    assert pa.STATUS[ei.value.status] == "PA_ERR_INVALID_ARGUMENT" and "host-only" in str(ei.value)
    plan.close()


def test_missing_library_fails_loudly(tmp_path):
    """Without the built library the binding raises: there is no CPU or oracle fallback."""
    missing = str(tmp_path / "libpa_absent.so")
    with pytest.raises(RuntimeError) as ei:
        pa.load_library(missing)
    assert "no fallback" in str(ei.value)
    import paged_kv_attention_39_b200 as pkg
    src = open(pkg.__file__).read()
    assert "import oracle" not in src and "from oracle" not in src
