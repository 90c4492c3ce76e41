"""GPU parity at the benchmark's full sizes and launch configuration.

Each case builds a whole serving batch of one workload (Qwen3-4B-shaped,
Qwen3-30B-A3B-shaped, the 131072-token underflow stress, MLA), prefills every
sequence but its newest token with bdfp4_quantize_kv, and runs one
bdfp4_decode_step (append + decode) at the split plan bdfp4_decode_plan_for
picks -- the call and the plan the benchmark times.  Sequences the oracle
recomputes (a seeded subset that always holds the longest) are drawn on the
CPU; the rest are drawn on the GPU, and three of their pages (the first, the
last, which the step appended into, and a seeded middle one) are copied back.

Checked against the oracle:
  * cache bytes, bit for bit: every page of the recomputed sequences and the
    sampled pages of every other sequence (keys are quantized per token and
    values per block of one page, so a page's bytes depend on its own tokens
    only);
  * the decode output of the recomputed sequences, within the decode bound;
  * bdfp4_decode over the updated cache equals the step's output bit for bit.
"""
import numpy as np
import pytest
import torch

from _util import assert_close, bf16_to_np, kv_params_gpu, oracle_calibration, out_to_np
from fp4_kv_cache_quant_b200 import bdfp4
from fp4_kv_cache_quant_b200.workloads import PAGE_SLOTS, Workload, spec

pytestmark = pytest.mark.gpu

NV, MX = 0, 1

FULL = {
    # name: (workload, fmt, sequences the oracle recomputes)
    "qwen3_4b_nv": ("qwen3_4b", NV, 2),
    "qwen3_4b_mx": ("qwen3_4b", MX, 2),
    "qwen3_30b_a3b_nv": ("qwen3_30b_a3b", NV, 4),
    "qwen3_30b_a3b_mx": ("qwen3_30b_a3b", MX, 4),
    "underflow_nv": ("underflow", NV, 2),
    "mla_nv": ("mla", NV, 2),
    "mla_mx": ("mla", MX, 2),
}

ARRAYS = ("k_pages", "k_scales", "v_pages", "v_scales")


def _page_view(t, num_pages: int) -> torch.Tensor:
    return t.view(num_pages, -1)


def _run_full(ora, name, flags=0, seed=21):
    cfg, fmt, n_checked = FULL[name]
    sp = spec(cfg)
    wl = Workload(sp, seed=seed)
    rng = np.random.default_rng(seed)
    longest = int(np.argmax(wl.seq_lens))
    others = [b for b in range(sp.B) if b != longest]
    checked = sorted({longest, *(int(x) for x in rng.choice(others, n_checked - 1, replace=False))})
    beta = 16 if fmt == NV else 32

    smooth, kg, vg = oracle_calibration(ora, wl)
    kvp = kv_params_gpu(smooth, kg, vg)
    gcache = bdfp4.FP4Cache.empty(wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    k_new = torch.zeros((sp.B, sp.H_kv, sp.d_k), dtype=torch.bfloat16, device="cuda")
    v_new = torch.zeros((sp.B, sp.H_kv, sp.d_v), dtype=torch.bfloat16, device="cuda")
    v_open = torch.zeros((sp.B, beta, sp.H_kv, sp.d_v), dtype=torch.bfloat16, device="cuda")
    ora_k, ora_v, ora_slots = [], [], []   # tokens the oracle quantizes (whole pages)
    pages_checked = []                      # page ids whose bytes are compared
    for b in range(sp.B):
        n = int(wl.seq_lens[b])
        dev = "cpu" if b in checked else "cuda"
        k, v = wl.keys(b, dev), wl.values(b, dev)
        kd, vd = k.cuda(), v.cuda()
        sm = wl.slot_mapping(b)
        if n > 1:
            bdfp4.bdfp4_quantize_kv(kd[:n - 1], vd[:n - 1], torch.from_numpy(sm[:n - 1]).cuda(), kvp, gcache,
                                    dev_status=status)
        last = (n - 1) % beta
        k_new[b] = kd[n - 1]
        v_new[b] = vd[n - 1]
        v_open[b, :last] = vd[n - 1 - last:n - 1]
        npg = (n + PAGE_SLOTS - 1) // PAGE_SLOTS
        if b in checked:
            pis = list(range(npg))
        else:
            pis = sorted({0, npg - 1, int(rng.integers(0, npg))})
        for pi in pis:
            t0, t1 = pi * PAGE_SLOTS, min(n, (pi + 1) * PAGE_SLOTS)
            ora_k.append(k[t0:t1].cpu())
            ora_v.append(v[t0:t1].cpu())
            ora_slots.append(sm[t0:t1])
            pages_checked.append(int(wl.block_table[b, pi]))
        del k, v, kd, vd
    torch.cuda.synchronize()
    assert int(status.item()) == 0

    num_sms = torch.cuda.get_device_properties(0).multi_processor_count
    chunk = bdfp4.bdfp4_decode_plan_for(wl.seq_lens, sp.H_q, sp.H_kv, sp.d_k, sp.d_v, num_sms)
    q = wl.queries("cpu")
    bt = torch.from_numpy(wl.block_table).cuda()
    sl = torch.from_numpy(wl.seq_lens).cuda()
    ws = bdfp4.workspace_for(sp.B, sp.H_q, sp.d_v, wl.max_pages, chunk)
    out = torch.empty((sp.B, sp.H_q, sp.d_v), dtype=torch.bfloat16, device="cuda")
    bdfp4.bdfp4_decode_step(q.cuda(), k_new, v_new, v_open, gcache, bt, sl, kvp, sp.sm_scale, chunk, ws, out,
                            flags=flags, dev_status=status)
    again = torch.empty_like(out)
    bdfp4.bdfp4_decode(q.cuda(), gcache, bt, sl, kvp, sp.sm_scale, chunk, ws, again, flags=flags, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(again, out), "bdfp4_decode on the updated cache differs from the step's output"

    # cache bytes of the sampled pages, against the oracle's quantization of those pages' tokens
    ocache = ora.empty_cache(wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt)
    ora.quantize_kv(torch.cat(ora_k), torch.cat(ora_v), np.concatenate(ora_slots), ocache, sp.H_kv, fmt, smooth, kg,
                    vg, wl.num_pages)
    idx = torch.tensor(pages_checked, dtype=torch.int64)
    for arr in ARRAYS:
        got = _page_view(getattr(gcache, arr), wl.num_pages)[idx.cuda()].cpu().numpy()
        exp = ocache[arr].reshape(wl.num_pages, -1)[idx.numpy()]
        bad = np.argwhere(got != exp)
        assert bad.size == 0, f"{arr}: {len(bad)} bytes differ, first (page row, byte) {bad[:4].tolist()}"

    # decode output of the recomputed sequences
    ref16, _ = ora.decode(q[checked], ocache, wl.block_table[checked], wl.seq_lens[checked], sp.H_kv, sp.d_v, fmt,
                          smooth, kg, vg, sp.sm_scale, chunk, wl.num_pages, flags=flags)
    got = out_to_np(out)
    assert np.isfinite(got).all()
    assert_close(got[checked], bf16_to_np(ref16), name, chunk, checked)
    return chunk


@pytest.mark.parametrize("name", list(FULL))
def test_full_size_step_matches_oracle(ora, name):
    _run_full(ora, name)


@pytest.mark.parametrize("name", ["qwen3_4b_nv", "underflow_nv"])
def test_full_size_step_dynamic_alpha_matches_oracle(ora, name):
    _run_full(ora, name, flags=bdfp4.FLAG_DYNAMIC_ALPHA)
