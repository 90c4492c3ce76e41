"""The bounded in-kernel waits of the d = 128 tensor-core decode, exercised
through the test hook of include/bdfp4_debug.h: every CTA withholds its first K
tile, so its MMA warp's wait runs out after a short bound (about a millisecond
of clock).  The CTA must unwind -- copies and tensor-core operations it started
finished, tensor memory freed -- report BDFP4_DEV_TIMEOUT, and leave the device
usable: the next normal decode on the same stream gives exactly the output it
gave before.  No fault is raised; the failure is a wait that nothing completes."""
import numpy as np
import pytest
import torch

from _util import assert_close, bf16_to_np, cache_from_np, kv_params_gpu, oracle_calibration, out_to_np
from fp4_kv_cache_quant_b200 import bdfp4
from fp4_kv_cache_quant_b200.workloads import Workload, spec

pytestmark = pytest.mark.gpu

SHORT_WAIT = 1 << 21   # clock cycles, about a millisecond


@pytest.mark.parametrize("chunk", [1, 8])
@pytest.mark.parametrize("fmt", [bdfp4.NVFP4, bdfp4.MXFP4])
def test_a_wait_that_runs_out_unwinds_and_reports(ora, fmt, chunk):
    sp = spec("qwen3_30b_a3b", B=4, ctx=("list", (1000, 77, 129, 513)))
    wl = Workload(sp, seed=16)
    smooth, kg, vg = oracle_calibration(ora, wl)
    ocache = ora.empty_cache(wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt)
    ora.quantize_kv(wl.all_keys(), wl.all_values(), wl.slot_mapping_all(), ocache, sp.H_kv, fmt, smooth, kg, vg,
                    wl.num_pages)
    gcache = cache_from_np(ocache, wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt)
    kvp = kv_params_gpu(smooth, kg, vg)
    q = wl.queries()
    qd = q.cuda()
    bt = torch.from_numpy(wl.block_table).cuda()
    sl = torch.from_numpy(wl.seq_lens).cuda()
    ws = bdfp4.workspace_for(sp.B, sp.H_q, sp.d_v, wl.max_pages, chunk)

    def normal():
        out = torch.empty((sp.B, sp.H_q, sp.d_v), dtype=torch.bfloat16, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        bdfp4.bdfp4_decode(qd, gcache, bt, sl, kvp, sp.sm_scale, chunk, ws, out, dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        return out

    before = normal()
    ref16, _ = ora.decode(q, ocache, wl.block_table, wl.seq_lens, sp.H_kv, sp.d_v, fmt, smooth, kg, vg, sp.sm_scale,
                          chunk, wl.num_pages)
    assert_close(out_to_np(before), bf16_to_np(ref16))

    # the short bound alone changes nothing in a run whose waits all complete
    out = torch.empty_like(before)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    bdfp4.bdfp4_debug_decode_wait_test(qd, gcache, bt, sl, kvp, sp.sm_scale, chunk, ws, out, SHORT_WAIT, False,
                                       dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and torch.equal(out, before)

    # every CTA's first K tile withheld: each CTA's wait runs out and it unwinds
    st.zero_()
    bdfp4.bdfp4_debug_decode_wait_test(qd, gcache, bt, sl, kvp, sp.sm_scale, chunk, ws, out, SHORT_WAIT, True,
                                       dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & bdfp4.DEV_TIMEOUT

    # the device is still usable: the same decode again, bit for bit
    assert torch.equal(normal(), before)


def test_the_hook_refuses_other_shapes(ora):
    sp = spec("tiny", B=1, ctx=("fixed", 64))   # four heads per KV head
    wl = Workload(sp, seed=16)
    cache = bdfp4.FP4Cache.empty(wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, bdfp4.NVFP4)
    smooth, kg, vg = oracle_calibration(ora, wl)
    out = torch.empty((sp.B, sp.H_q, sp.d_v), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bdfp4.BDFP4Error, match="compiled set"):
        bdfp4.bdfp4_debug_decode_wait_test(wl.queries().cuda(), cache, torch.from_numpy(wl.block_table).cuda(),
                                           torch.from_numpy(wl.seq_lens).cuda(), kv_params_gpu(smooth, kg, vg),
                                           sp.sm_scale, 1, None, out, SHORT_WAIT, True)
