"""GPU parity at the limits of the forward path, against the fp64 oracle through the C ABI: the
largest head dim the pages allow (1024), unequal key and value widths, one-token pages and pages
wider than any tile, a sequence cut into more parts than the split cap (1024 per sequence), and
query groups far beyond the tensor-core decode kernel's 16 rows (MQA with 64 and 128 heads)."""
import pytest
import torch

import paged_kv_attention_39_b200 as pa
from gpu_helpers import check, run_gqa
from paged_kv_attention_39_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_head_dim_1024(orc, dtype):
    """D = Dv = 1024 (the CUDA-core path): decode rows and a short prefill chunk."""
    wl = W.make_gqa("d1024", 31, [90, 257, 33], [1, 17, 1], 8, 2, 1024, 1024, 16, dtype)
    ref = orc.run(wl)
    for kv_chunk in (0, 64):
        out, lse = run_gqa(wl, kv_chunk=kv_chunk)
        check(wl, out, lse, *ref, tag=f"d1024 {dtype} chunk {kv_chunk}")


def test_unequal_key_and_value_widths(orc):
    """D = 192 keys with Dv = 128 values (the CUDA-core path), window and causal masks."""
    wl = W.make_gqa("d192v128", 32, [300, 45, 700], [1, 9, 3], 16, 4, 192, 128, 16, torch.bfloat16, window=200)
    ref = orc.run(wl)
    out, lse = run_gqa(wl, kv_chunk=96)
    check(wl, out, lse, *ref, tag="d192 dv128")


@pytest.mark.parametrize("ps", [1, 8, 1024])
def test_extreme_page_sizes(orc, ps):
    """Pages of one token (every key through its own block-table entry), of 8 tokens (narrower than
    any TMA box), and of 1024 tokens (wider than every key tile): decode rows and prefill chunks."""
    wl = W.make_gqa(f"ps{ps}", 33, [1500, 70, 2100, 300], [1, 1, 130, 40], 32, 8, 128, 128, ps, torch.bfloat16)
    ref = orc.run(wl)
    for kv_chunk in (0, 128):
        out, lse = run_gqa(wl, kv_chunk=kv_chunk)
        check(wl, out, lse, *ref, tag=f"ps{ps} chunk {kv_chunk}")


def test_split_cap_of_1024_parts(orc):
    """A 40000-key sequence with 16-key parts asked for (2500 parts) is cut into at most 1024 parts;
    a short sequence beside it stays whole."""
    wl = W.make_gqa("cap", 34, [40000, 100], [1, 1], 8, 2, 128, 128, 64, torch.bfloat16)
    ref = orc.run(wl)
    plan = pa.plan_for(wl)
    out, lse = run_gqa(wl, kv_chunk=16, plan=plan)
    info = pa.pa_plan_get_info(plan)
    assert info["last_kernels"] & pa.PA_KERNEL_DECODE_TC, info
    assert pa.pa_plan_device_status(plan) == 0
    plan.close()
    check(wl, out, lse, *ref, tag="split cap")


@pytest.mark.parametrize("hq", [64, 128])
def test_mqa_large_groups(orc, hq):
    """One KV head shared by 64 or 128 query heads: decode rows of 64 / 128 heads (beyond the
    tensor-core decode kernel's 16 rows) and a prefill chunk, against the oracle."""
    wl = W.make_gqa(f"mqa{hq}", 35, [800, 2000, 150], [1, 1, 33], hq, 1, 128, 128, 16, torch.bfloat16)
    ref = orc.run(wl)
    for kv_chunk in (0, 256):
        out, lse = run_gqa(wl, kv_chunk=kv_chunk)
        check(wl, out, lse, *ref, tag=f"mqa {hq} chunk {kv_chunk}")
