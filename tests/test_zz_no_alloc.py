"""The no-allocation decode entry point (bdfp4_decode_noalloc).

Some callers cannot allocate device memory -- an operator that a host
framework hands only its inputs and outputs, or a serving loop that must not
call an allocator -- so the library offers a decode that keeps its split-KV
partials and query images in a scratch array compiled into the library
instead of a caller-provided workspace.  These tests check, through the C ABI,
that it gives exactly the output of bdfp4_decode with a workspace (the same
kernels on the same inputs), on two calls in a row (the second call reuses the
scratch the first one left behind), that its own automatic plan (chunk_tiles
<= 0) is bdfp4_decode's, that it matches the oracle, and that a plan too large
for the scratch is rejected.  This file is collected last.
"""
import pytest
import torch

from _util import assert_close, bf16_to_np, kv_params_gpu, oracle_calibration, quantize_both
from fp4_kv_cache_quant_b200 import bdfp4
from fp4_kv_cache_quant_b200.workloads import Workload, spec

pytestmark = pytest.mark.gpu

CASES = {
    # name: (spec, fmt)
    "g8_nv": (spec("qwen3_30b_a3b", B=4, ctx=("list", (1000, 77, 129, 513))), bdfp4.NVFP4),
    "g8_mx": (spec("qwen3_30b_a3b", B=4, ctx=("list", (1000, 77, 129, 513))), bdfp4.MXFP4),
    "mla16_nv": (spec("mla", B=2, H_q=16, ctx=("list", (700, 130))), bdfp4.NVFP4),
}


def _setup(name, seed=11):
    sp, fmt = CASES[name]
    wl = Workload(sp, seed=seed)
    kc, qc, vc = wl.calibration("cuda")
    kv = bdfp4.bdfp4_calibrate(kc, qc, vc, sp.H_q, sp.H_kv)
    cache = bdfp4.FP4Cache.empty(wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bdfp4.bdfp4_quantize_kv(wl.all_keys("cuda"), wl.all_values("cuda"), torch.from_numpy(wl.slot_mapping_all()).cuda(),
                            kv, cache, dev_status=status)
    bt = torch.from_numpy(wl.block_table).cuda()
    sl = torch.from_numpy(wl.seq_lens).cuda()
    return sp, wl, kv, cache, bt, sl, status


@pytest.mark.parametrize("chunk", [1, 3, "planned", 0])
@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_decode_equals_workspace_decode_twice(name, chunk):
    """chunk "planned": bdfp4_decode_plan_for's pick on the host lengths; 0: both entry
    points plan by themselves from max_pages_per_seq (the no-allocation call's own plan)."""
    sp, wl, kv, cache, bt, sl, status = _setup(name)
    if chunk == "planned":
        chunk = bdfp4.bdfp4_decode_plan_for(wl.seq_lens, sp.H_q, sp.H_kv, sp.d_k, sp.d_v,
                                            torch.cuda.get_device_properties(0).multi_processor_count)
    ws_chunk = chunk if chunk > 0 else 1   # a workspace large enough for any plan
    ws = bdfp4.workspace_for(sp.B, sp.H_q, sp.d_v, wl.max_pages, ws_chunk)
    for call in range(2):
        q = wl.queries("cuda", step=call)
        ref = torch.empty((sp.B, sp.H_q, sp.d_v), dtype=torch.bfloat16, device="cuda")
        bdfp4.bdfp4_decode(q, cache, bt, sl, kv, sp.sm_scale, chunk, ws, ref, dev_status=status)
        out = torch.full((sp.B, sp.H_q, sp.d_v), float("nan"), dtype=torch.bfloat16, device="cuda")
        bdfp4.bdfp4_decode_noalloc(q, cache, bt, sl, kv, sp.sm_scale, chunk, out, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(out, ref), (name, chunk, call)


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_decode_matches_oracle(ora, name):
    sp, fmt = CASES[name]
    wl = Workload(sp, seed=12)
    smooth, kg, vg = oracle_calibration(ora, wl)
    gcache, ocache = quantize_both(ora, wl, fmt, smooth, kg, vg)
    q = wl.queries("cpu")
    chunk = 2
    ref16, _ = ora.decode(q, ocache, wl.block_table, wl.seq_lens, sp.H_kv, sp.d_v, fmt, smooth, kg, vg, sp.sm_scale,
                          chunk, wl.num_pages)
    out = torch.empty((sp.B, sp.H_q, sp.d_v), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bdfp4.bdfp4_decode_noalloc(q.cuda(), gcache, torch.from_numpy(wl.block_table).cuda(),
                               torch.from_numpy(wl.seq_lens).cuda(), kv_params_gpu(smooth, kg, vg), sp.sm_scale, chunk,
                               out, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert_close(out.float().cpu().numpy(), bf16_to_np(ref16))


def test_noalloc_rejects_plans_beyond_the_scratch():
    sp, wl, kv, cache, bt, sl, status = _setup("g8_nv")
    q = wl.queries("cuda")
    out = torch.empty((sp.B, sp.H_q, sp.d_v), dtype=torch.bfloat16, device="cuda")
    # a block table claiming 65536 pages per sequence, one tile per split, needs
    # far more than the built-in scratch: refused before any launch
    big_bt = torch.zeros((sp.B, 65536), dtype=torch.int32, device="cuda")
    need = bdfp4.bdfp4_decode_workspace_size(sp.B, sp.H_q, sp.d_v, 65536, 1)
    assert need > bdfp4.NOALLOC_SCRATCH_BYTES
    with pytest.raises(bdfp4.BDFP4Error, match="workspace"):
        bdfp4.bdfp4_decode_noalloc(q, cache, big_bt, sl, kv, sp.sm_scale, 1, out, dev_status=status)
