"""GPU parity of the BF16-KV comparator (include/bdfp4_bf16.h).

The append's page bytes are compared with a numpy scatter written from the
header's layout description; the decode is compared with the oracle's fp64
softmax(q K^T * sm_scale) V on the same bf16 inputs (max-abs 1e-2, relative L2
5e-3).  Pages start filled with NaN bits, so slots no append wrote must not
leak into any output."""
import numpy as np
import pytest
import torch

from _util import assert_close, out_to_np
from fp4_kv_cache_quant_b200 import bdfp4
from fp4_kv_cache_quant_b200.workloads import Workload, spec

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": spec("tiny"),
    "ragged_g8": spec("qwen3_30b_a3b", B=4, ctx=("list", (1000, 77, 129, 513))),
    "g1": spec("tiny", H_q=2, H_kv=2, ctx=("fixed", 300)),
    "g2": spec("tiny", B=2, H_q=4, H_kv=2, ctx=("list", (64, 700))),
    "g16": spec("tiny", B=2, H_q=16, H_kv=1, ctx=("list", (200, 1))),
    "empty": spec("tiny", B=3, H_q=8, H_kv=2, ctx=("list", (0, 130, 5))),
}


def _u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _append(wl: Workload, fill: int) -> bdfp4.BF16Cache:
    sp = wl.spec
    cache = bdfp4.BF16Cache.empty(max(wl.num_pages, 1), sp.H_kv, sp.d_k)
    cache.k_pages.fill_(fill)
    cache.v_pages.fill_(fill)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bdfp4.bdfp4_bf16_append(wl.all_keys().cuda(), wl.all_values().cuda(),
                            torch.from_numpy(wl.slot_mapping_all()).cuda(), cache, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return cache


@pytest.mark.parametrize("name", ["tiny", "ragged_g8", "g2"])
def test_bf16_append_layout(name):
    wl = Workload(CASES[name], seed=11)
    sp = wl.spec
    d, P = sp.d_k, max(wl.num_pages, 1)
    cache = _append(wl, 0xAB)
    k, v, sm = _u16(wl.all_keys()), _u16(wl.all_values()), wl.slot_mapping_all()
    # K page: [slot/8][elem/8][slot%8][8 elements]; V page: [chan/8][slot/8][chan%8][8 slots]
    kexp = np.full((P, sp.H_kv, 8, d // 8, 8, 8), 0xABAB, np.uint16)
    vexp = np.full((P, sp.H_kv, d // 8, 8, 8, 8), 0xABAB, np.uint16)
    for t in range(k.shape[0]):
        page, slot = int(sm[t]) // 64, int(sm[t]) % 64
        for h in range(sp.H_kv):
            kexp[page, h, slot // 8, :, slot % 8, :] = k[t, h].reshape(d // 8, 8)
            vexp[page, h, :, slot // 8, :, slot % 8] = v[t, h].reshape(d // 8, 8)
    got_k = cache.k_pages.cpu().numpy().view(np.uint16).reshape(kexp.shape)
    got_v = cache.v_pages.cpu().numpy().view(np.uint16).reshape(vexp.shape)
    assert np.array_equal(got_k, kexp)
    assert np.array_equal(got_v, vexp)


@pytest.mark.parametrize("chunk", [0, 1, 3])
@pytest.mark.parametrize("name", list(CASES))
def test_bf16_decode_matches_oracle(ora, name, chunk):
    wl = Workload(CASES[name], seed=12)
    sp = wl.spec
    cache = _append(wl, 0xFF)   # bf16 0xFFFF is NaN: unwritten slots hold NaN
    q = wl.queries("cpu")
    if chunk <= 0:
        chunk = bdfp4.bdfp4_decode_plan(wl.seq_lens, sp.H_kv, torch.cuda.get_device_properties(0).multi_processor_count)
    bt = torch.from_numpy(wl.block_table).cuda()
    sl = torch.from_numpy(wl.seq_lens).cuda()
    out = torch.empty((sp.B, sp.H_q, sp.d_v), dtype=torch.bfloat16, device="cuda")
    ws = bdfp4.workspace_for(sp.B, sp.H_q, sp.d_v, bt.shape[1], chunk)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bdfp4.bdfp4_bf16_decode(q.cuda(), cache, bt, sl, sp.sm_scale, chunk, ws, out, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = out_to_np(out)
    ref = ora.attention_ref(q, wl.all_keys(), wl.all_values(), wl.cu_seqlens, sp.H_kv, sp.sm_scale)
    assert np.all(np.isfinite(got))
    assert_close(got, ref)
    for b, n in enumerate(wl.seq_lens):
        if n == 0:
            assert np.all(got[b] == 0)


def test_bf16_decode_full_size_sampled(ora):
    """Qwen3-4B shape (B=16, 32/8 heads, 32768 tokens each) in the bench's
    launch configuration; the oracle recomputes two sequences."""
    sp = spec("qwen3_4b")
    wl = Workload(sp, seed=13)
    cache = bdfp4.BF16Cache.empty(wl.num_pages, sp.H_kv, sp.d_k)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    checked = (0, sp.B - 1)   # drawn with the CPU generator, which the oracle sees
    for b in range(sp.B):
        k = wl.keys(b).cuda() if b in checked else wl.keys(b, "cuda")
        v = wl.values(b).cuda() if b in checked else wl.values(b, "cuda")
        bdfp4.bdfp4_bf16_append(k, v, torch.from_numpy(wl.slot_mapping(b)).cuda(), cache, dev_status=status)
    q = wl.queries("cpu")
    chunk = bdfp4.bdfp4_decode_plan(wl.seq_lens, sp.H_kv, torch.cuda.get_device_properties(0).multi_processor_count)
    bt = torch.from_numpy(wl.block_table).cuda()
    sl = torch.from_numpy(wl.seq_lens).cuda()
    out = torch.empty((sp.B, sp.H_q, sp.d_v), dtype=torch.bfloat16, device="cuda")
    ws = bdfp4.workspace_for(sp.B, sp.H_q, sp.d_v, bt.shape[1], chunk)
    bdfp4.bdfp4_bf16_decode(q.cuda(), cache, bt, sl, sp.sm_scale, chunk, ws, out, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = out_to_np(out)
    for b in checked:
        n = int(wl.seq_lens[b])
        ref = ora.attention_ref(q[b:b + 1], wl.keys(b), wl.values(b), np.array([0, n], np.int64), sp.H_kv,
                                sp.sm_scale)
        assert_close(got[b:b + 1], ref, b)
