"""GPU parity of the multi-token decode (bdfp4_decode_multi): each sequence's
T_q newest tokens attend causally, and the (token, head) rows of a KV group
stack in one MMA operand.  Against the oracle's decode_multi (each query token
runs the single-token decode on its prefix, same tiles and splits)."""
import numpy as np
import pytest
import torch

from _util import assert_close, bf16_to_np, cache_from_np, kv_params_gpu, oracle_calibration, out_to_np
from fp4_kv_cache_quant_b200 import bdfp4
from fp4_kv_cache_quant_b200.workloads import Workload, spec

pytestmark = pytest.mark.gpu

NV, MX = 0, 1

CASES = {
    # name: (spec, fmt); G = 4 and G = 8 groups, ragged lengths across tile and page edges
    "g4_nv": (spec("tiny", B=3, H_q=8, H_kv=2, ctx=("list", (1000, 129, 64)), n_outlier=2), NV),
    "g4_mx": (spec("tiny", B=3, H_q=8, H_kv=2, ctx=("list", (1000, 129, 64)), n_outlier=2), MX),
    "g8_nv": (spec("qwen3_30b_a3b", B=3, ctx=("list", (700, 200, 128))), NV),
    "g8_mx": (spec("qwen3_30b_a3b", B=3, ctx=("list", (700, 200, 128))), MX),
    "mla16_nv": (spec("mla", B=2, H_q=16, ctx=("list", (300, 130))), NV),
}


def _queries(sp, T, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn((sp.B, T, sp.H_q, sp.d_k), generator=g).to(torch.bfloat16)


def _setup(ora, name, seed):
    sp, fmt = CASES[name]
    wl = Workload(sp, seed=seed)
    smooth, kg, vg = oracle_calibration(ora, wl)
    ocache = ora.empty_cache(wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt)
    ora.quantize_kv(wl.all_keys(), wl.all_values(), wl.slot_mapping_all(), ocache, sp.H_kv, fmt, smooth, kg, vg,
                    wl.num_pages)
    return sp, fmt, wl, smooth, kg, vg, ocache, cache_from_np(ocache, wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt)


def _run(wl, gcache, q, kvp, chunk, flags=0, seq_lens=None):
    sp = wl.spec
    B, T = q.shape[:2]
    sl = torch.from_numpy(np.asarray(wl.seq_lens if seq_lens is None else seq_lens, np.int32)).cuda()
    bt = torch.from_numpy(wl.block_table).cuda()
    out = torch.full((B, T, sp.H_q, sp.d_v), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = bdfp4.workspace_for(B * T, sp.H_q, sp.d_v, bt.shape[1], max(chunk, 1))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bdfp4.bdfp4_decode_multi(q.cuda(), gcache, bt, sl, kvp, sp.sm_scale, chunk, ws, out, flags=flags,
                             dev_status=status)
    torch.cuda.synchronize()
    return out, int(status.item())


@pytest.mark.parametrize("chunk", ["planned", 1])
@pytest.mark.parametrize("T", [1, 2, 4, 8])
@pytest.mark.parametrize("name", ["g4_nv", "g4_mx", "g8_nv", "g8_mx"])
def test_multi_token_decode_matches_oracle(ora, name, T, chunk):
    """G T stacked rows: up to 16 on the tensor-core decode (G = 4: T <= 4; G = 8: T <= 2),
    beyond on the CUDA-core decode."""
    sp, fmt, wl, smooth, kg, vg, ocache, gcache = _setup(ora, name, 31)
    if chunk == "planned":
        chunk = bdfp4.bdfp4_decode_multi_plan(wl.seq_lens, T, sp.H_q, sp.H_kv, sp.d_k, sp.d_v,
                                              torch.cuda.get_device_properties(0).multi_processor_count)
    q = _queries(sp, T, 32 + T)
    out, status = _run(wl, gcache, q, kv_params_gpu(smooth, kg, vg), chunk)
    assert status == 0
    ref16, _ = ora.decode_multi(q, ocache, wl.block_table, wl.seq_lens, sp.H_kv, sp.d_v, fmt, smooth, kg, vg,
                                sp.sm_scale, chunk, wl.num_pages)
    got = out_to_np(out)
    assert np.isfinite(got).all()
    assert_close(got, bf16_to_np(ref16), name, T, chunk)


@pytest.mark.parametrize("T", [2, 4])
@pytest.mark.parametrize("name", ["g4_nv", "g8_nv"])
def test_multi_token_decode_dynamic_alpha_matches_oracle(ora, name, T):
    sp, fmt, wl, smooth, kg, vg, ocache, gcache = _setup(ora, name, 33)
    q = _queries(sp, T, 34)
    out, status = _run(wl, gcache, q, kv_params_gpu(smooth, kg, vg), 2, flags=bdfp4.FLAG_DYNAMIC_ALPHA)
    assert status == 0
    ref16, _ = ora.decode_multi(q, ocache, wl.block_table, wl.seq_lens, sp.H_kv, sp.d_v, fmt, smooth, kg, vg,
                                sp.sm_scale, 2, wl.num_pages, flags=bdfp4.FLAG_DYNAMIC_ALPHA)
    assert_close(out_to_np(out), bf16_to_np(ref16), name, T)


@pytest.mark.parametrize("T", [2, 3])
def test_multi_token_decode_latent_geometry_matches_oracle(ora, T):
    sp, fmt, wl, smooth, kg, vg, ocache, gcache = _setup(ora, "mla16_nv", 35)
    q = _queries(sp, T, 36)
    out, status = _run(wl, gcache, q, kv_params_gpu(smooth, kg, vg), 1)
    assert status == 0
    ref16, _ = ora.decode_multi(q, ocache, wl.block_table, wl.seq_lens, sp.H_kv, sp.d_v, fmt, smooth, kg, vg,
                                sp.sm_scale, 1, wl.num_pages)
    assert_close(out_to_np(out), bf16_to_np(ref16), T)


@pytest.mark.parametrize("name", ["g4_nv", "g8_mx"])
def test_one_query_token_is_the_single_token_decode(ora, name):
    """T_q = 1 gives bdfp4_decode's output bit for bit."""
    sp, fmt, wl, smooth, kg, vg, ocache, gcache = _setup(ora, name, 37)
    q = _queries(sp, 1, 38)
    kvp = kv_params_gpu(smooth, kg, vg)
    out, status = _run(wl, gcache, q, kvp, 2)
    ref = torch.empty((sp.B, sp.H_q, sp.d_v), dtype=torch.bfloat16, device="cuda")
    ws = bdfp4.workspace_for(sp.B, sp.H_q, sp.d_v, wl.max_pages, 2)
    bdfp4.bdfp4_decode(q[:, 0].contiguous().cuda(), gcache, torch.from_numpy(wl.block_table).cuda(),
                       torch.from_numpy(wl.seq_lens).cuda(), kvp, sp.sm_scale, 2, ws, ref)
    torch.cuda.synchronize()
    assert status == 0 and torch.equal(out[:, 0], ref)


@pytest.mark.parametrize("T", [4, 8])
@pytest.mark.parametrize("name", ["g4_nv", "g8_nv"])
def test_sequence_shorter_than_its_query_tokens(ora, name, T):
    """0 < N_b < T_q is reported; query tokens that would see no key give zeros, the
    others see their prefixes; an empty sequence gives zeros."""
    sp, fmt, wl, smooth, kg, vg, ocache, gcache = _setup(ora, name, 39)
    q = _queries(sp, T, 40)
    lens = wl.seq_lens.copy()
    lens[1], lens[2] = T - 2, 0
    out, status = _run(wl, gcache, q, kv_params_gpu(smooth, kg, vg), 1, seq_lens=lens)
    assert status & bdfp4.DEV_BAD_SEQLEN
    got = out_to_np(out)
    assert np.isfinite(got).all()
    assert np.all(got[2] == 0) and np.all(got[1, :2] == 0)
    # the rows that see tokens: compare with the oracle on the prefixes they see
    ref16, _ = ora.decode_multi(q[:, 2:], ocache, wl.block_table, np.maximum(lens, T - 2), sp.H_kv, sp.d_v, fmt,
                                smooth, kg, vg, sp.sm_scale, 1, wl.num_pages)
    ref = bf16_to_np(ref16)
    assert_close(got[:2, 2:], ref[:2], name, T)
