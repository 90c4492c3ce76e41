"""The no-allocation decode entry point (bdfp4_decode_noalloc).

Some callers cannot allocate device memory -- an operator that a host
framework hands only its inputs and outputs, or a serving loop that must not
call an allocator -- so the library offers a decode that keeps its split-KV
partials in a scratch array compiled into the library instead of a
caller-provided workspace.  These tests check, through the C ABI, that it
gives the same output as bdfp4_decode with a workspace, on two calls in a row
(the second call reuses the scratch the first one left behind), and that a
plan too large for the scratch is rejected.  This file is collected last.
"""
import numpy as np
import pytest
import torch

from fp4_kv_cache_quant_b200 import bdfp4
from fp4_kv_cache_quant_b200.workloads import Workload, spec

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
REL_L2 = 5e-3


def _setup(seed=11):
    sp = spec("qwen3_30b_a3b", B=4, ctx=("list", (1000, 77, 129, 513)))
    wl = Workload(sp, seed=seed)
    kc, qc, vc = wl.calibration("cuda")
    kv = bdfp4.bdfp4_calibrate(kc, qc, vc, sp.H_q, sp.H_kv)
    cache = bdfp4.FP4Cache.empty(wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, bdfp4.NVFP4)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bdfp4.bdfp4_quantize_kv(wl.all_keys("cuda"), wl.all_values("cuda"), torch.from_numpy(wl.slot_mapping_all()).cuda(),
                            kv, cache, dev_status=status)
    bt = torch.from_numpy(wl.block_table).cuda()
    sl = torch.from_numpy(wl.seq_lens).cuda()
    return sp, wl, kv, cache, bt, sl, status


def _compare(a: torch.Tensor, b: torch.Tensor):
    x, y = a.float().cpu().numpy().astype(np.float64), b.float().cpu().numpy().astype(np.float64)
    return float(np.max(np.abs(x - y))), float(np.linalg.norm(x - y) / max(np.linalg.norm(y), 1e-30))


@pytest.mark.parametrize("chunk", [1, 3, 0])
def test_noalloc_decode_matches_workspace_decode_twice(chunk):
    sp, wl, kv, cache, bt, sl, status = _setup()
    if chunk <= 0:
        chunk = bdfp4.bdfp4_decode_plan(wl.seq_lens, sp.H_kv,
                                        torch.cuda.get_device_properties(0).multi_processor_count)
    ref = torch.empty((sp.B, sp.H_q, sp.d_v), dtype=torch.bfloat16, device="cuda")
    ws = bdfp4.workspace_for(sp.B, sp.H_q, sp.d_v, wl.max_pages, chunk)
    for call in range(2):
        q = wl.queries("cuda", step=call)
        bdfp4.bdfp4_decode(q, cache, bt, sl, kv, sp.sm_scale, chunk, ws, ref, dev_status=status)
        out = torch.full((sp.B, sp.H_q, sp.d_v), float("nan"), dtype=torch.bfloat16, device="cuda")
        bdfp4.bdfp4_decode_noalloc(q, cache, bt, sl, kv, sp.sm_scale, chunk, out, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        max_abs, rel = _compare(out, ref)
        assert max_abs <= MAX_ABS and rel <= REL_L2, (call, max_abs, rel)


def test_noalloc_rejects_plans_beyond_the_scratch():
    sp, wl, kv, cache, bt, sl, status = _setup()
    q = wl.queries("cuda")
    out = torch.empty((sp.B, sp.H_q, sp.d_v), dtype=torch.bfloat16, device="cuda")
    # a block table claiming 65536 pages per sequence, one tile per split, needs
    # far more than the built-in scratch: refused before any launch
    big_bt = torch.zeros((sp.B, 65536), dtype=torch.int32, device="cuda")
    need = bdfp4.bdfp4_decode_workspace_size(sp.B, sp.H_q, sp.d_v, 65536, 1)
    assert need > bdfp4.NOALLOC_SCRATCH_BYTES
    with pytest.raises(bdfp4.BDFP4Error, match="workspace"):
        bdfp4.bdfp4_decode_noalloc(q, cache, big_bt, sl, kv, sp.sm_scale, 1, out, dev_status=status)
