"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Quantized bytes (cache, query codes, calibration) must match bit for bit;
decode outputs within max-abs 1e-2 and relative L2 5e-3 of the oracle run on
the same FP4 cache bytes."""
import math

import numpy as np
import pytest
import torch

from _util import (assert_bytes_equal, assert_close, bf16_to_np, cache_from_np, cache_to_np, kv_params_gpu,
                   oracle_calibration, out_to_np, quantize_both, run_gpu_decode)
from fp4_kv_cache_quant_b200 import bdfp4
from fp4_kv_cache_quant_b200.workloads import Workload, spec

pytestmark = pytest.mark.gpu

NV, MX = 0, 1

SMALL = {
    # name: (spec, fmt)
    "tiny_nv": (spec("tiny"), NV),
    "tiny_mx": (spec("tiny"), MX),
    "ragged_g8_nv": (spec("qwen3_30b_a3b", B=4, ctx=("list", (1000, 77, 129, 513))), NV),
    "ragged_g8_mx": (spec("qwen3_30b_a3b", B=4, ctx=("list", (1000, 77, 129, 513))), MX),
    "g1_nv": (spec("tiny", H_q=2, H_kv=2, ctx=("fixed", 300)), NV),
    "g16_nv": (spec("tiny", B=2, H_q=16, H_kv=1, ctx=("list", (200, 1)), n_outlier=2), NV),
    "mla_nv": (spec("mla", B=2, H_q=16, ctx=("list", (300, 130))), NV),
    "mla_mx": (spec("mla", B=2, H_q=16, ctx=("list", (300, 130))), MX),
    "mla128_nv": (spec("mla", B=2, ctx=("list", (300, 130))), NV),
    "mla128_mx": (spec("mla", B=2, ctx=("list", (300, 130))), MX),
    "mla64_nv": (spec("mla", B=2, H_q=64, ctx=("list", (1000, 77))), NV),
    "mla32_mx": (spec("mla", B=3, H_q=32, ctx=("list", (129, 0, 700))), MX),
    # shapes the tensor-core kernels do not take run the CUDA-core decode
    "g32_cuda_nv": (spec("tiny", B=2, H_q=32, H_kv=1, ctx=("list", (300, 77))), NV),
    "mla8_cuda_mx": (spec("mla", B=2, H_q=8, ctx=("list", (200, 65))), MX),
}


def planned_chunk(wl) -> int:
    """The split plan bdfp4_decode's kernel for this shape runs at (the bench's choice)."""
    sp = wl.spec
    return bdfp4.bdfp4_decode_plan_for(wl.seq_lens, sp.H_q, sp.H_kv, sp.d_k, sp.d_v,
                                       torch.cuda.get_device_properties(0).multi_processor_count)


@pytest.fixture(scope="module")
def lib():
    assert torch.cuda.is_available()
    bdfp4.load()
    return bdfp4


@pytest.mark.parametrize("name", list(SMALL))
def test_calibration_bit_exact(ora, lib, name):
    sp, fmt = SMALL[name]
    wl = Workload(sp, seed=1)
    smooth, kg, vg = oracle_calibration(ora, wl)
    kc, qc, vc = wl.calibration("cpu")
    kv = bdfp4.bdfp4_calibrate(kc.cuda(), qc.cuda(), vc.cuda(), sp.H_q, sp.H_kv)
    torch.cuda.synchronize()
    assert np.array_equal(kv.smooth.cpu().numpy(), smooth)
    assert np.array_equal(kv.k_gscale.cpu().numpy(), kg)
    assert np.array_equal(kv.v_gscale.cpu().numpy(), vg)


@pytest.mark.parametrize("flags", [0, bdfp4.FLAG_NO_HADAMARD | bdfp4.FLAG_NO_SCALE_SEARCH])
@pytest.mark.parametrize("name", list(SMALL))
def test_quantize_kv_bit_exact(ora, lib, name, flags):
    sp, fmt = SMALL[name]
    wl = Workload(sp, seed=2)
    smooth, kg, vg = oracle_calibration(ora, wl, flags)
    gcache, ocache = quantize_both(ora, wl, fmt, smooth, kg, vg, flags)
    assert_bytes_equal(cache_to_np(gcache), ocache)


@pytest.mark.parametrize("flags", [0, bdfp4.FLAG_NO_HADAMARD])
@pytest.mark.parametrize("name", list(SMALL))
def test_key_weights_bit_exact(ora, lib, name, flags):
    """Channel weights of the attention-aware key scale search (bdfp4_key_weights)."""
    sp, fmt = SMALL[name]
    wl = Workload(sp, seed=14)
    smooth, _, _ = oracle_calibration(ora, wl, flags)
    _, qc, _ = wl.calibration("cpu")
    ref = ora.key_weights(qc, sp.H_q, sp.H_kv, smooth, flags=flags)
    got = bdfp4.bdfp4_key_weights(qc.cuda(), sp.H_kv, torch.from_numpy(smooth).cuda(), flags=flags)
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy(), ref)


@pytest.mark.parametrize("flags", [0, bdfp4.FLAG_NO_HADAMARD])
@pytest.mark.parametrize("name", list(SMALL))
def test_quantize_kv_weighted_search_bit_exact(ora, lib, name, flags):
    """The attention-aware key scale search: the cache bytes equal the oracle's
    weighted quantization.  Without the rotation the calibration queries' energy
    is uneven across channels (smoothing moves it), so the weighted search must
    pick other codes than the plain one somewhere -- the path is exercised."""
    sp, fmt = SMALL[name]
    wl = Workload(sp, seed=15)
    smooth, kg, vg = oracle_calibration(ora, wl, flags)
    _, qc, _ = wl.calibration("cpu")
    w = ora.key_weights(qc, sp.H_q, sp.H_kv, smooth, flags=flags)
    k, v, sm = wl.all_keys(), wl.all_values(), wl.slot_mapping_all()
    ocache = ora.empty_cache(wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt)
    ora.quantize_kv(k, v, sm, ocache, sp.H_kv, fmt, smooth, kg, vg, wl.num_pages, flags=flags, k_weight=w)
    kvp = kv_params_gpu(smooth, kg, vg)
    kvp.k_weight = torch.from_numpy(w).cuda()
    gcache = bdfp4.FP4Cache.empty(wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bdfp4.bdfp4_quantize_kv(k.cuda(), v.cuda(), torch.from_numpy(sm).cuda(), kvp, gcache, flags=flags,
                            dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert_bytes_equal(cache_to_np(gcache), ocache)
    if flags & bdfp4.FLAG_NO_HADAMARD and fmt == NV:
        plain = ora.empty_cache(wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt)
        ora.quantize_kv(k, v, sm, plain, sp.H_kv, fmt, smooth, kg, vg, wl.num_pages, flags=flags)
        assert not np.array_equal(plain["k_scales"], ocache["k_scales"])


@pytest.mark.parametrize("name", ["tiny_nv", "tiny_mx", "ragged_g8_nv", "ragged_g8_mx", "mla_nv"])
def test_decode_step_append_matches_oracle(ora, lib, name):
    """Prefill all but the newest token with bdfp4_quantize_kv, then append the newest
    token's key with bdfp4_quantize_k and its open value block with bdfp4_quantize_v:
    the cache must equal the oracle's quantization of every token at once."""
    sp, fmt = SMALL[name]
    wl = Workload(sp, seed=7)
    smooth, kg, vg = oracle_calibration(ora, wl)
    ocache = ora.empty_cache(wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt)
    ora.quantize_kv(wl.all_keys(), wl.all_values(), wl.slot_mapping_all(), ocache, sp.H_kv, fmt, smooth, kg, vg,
                    wl.num_pages)
    kvp = kv_params_gpu(smooth, kg, vg)
    gcache = bdfp4.FP4Cache.empty(wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt)
    for name_ in ("k_pages", "k_scales", "v_pages", "v_scales"):
        getattr(gcache, name_).zero_()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    beta = 16 if fmt == NV else 32
    for b in range(sp.B):
        n = int(wl.seq_lens[b])
        if n == 0:
            continue
        k, v = wl.keys(b).cuda(), wl.values(b).cuda()
        sm = torch.from_numpy(wl.slot_mapping(b)).cuda()
        if n > 1:
            bdfp4.bdfp4_quantize_kv(k[:n - 1], v[:n - 1], sm[:n - 1], kvp, gcache, dev_status=status)
        bdfp4.bdfp4_quantize_k(k[n - 1:], sm[n - 1:], kvp, gcache, dev_status=status)
        r = (n - 1) % beta + 1   # the open block: the newest token and the earlier ones of its block
        bdfp4.bdfp4_quantize_v(v[n - r:], sm[n - r:], kvp, gcache)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert_bytes_equal(cache_to_np(gcache), ocache)


@pytest.mark.parametrize("chunk", [0, 1])
@pytest.mark.parametrize("name", ["tiny_nv", "tiny_mx", "ragged_g8_nv", "ragged_g8_mx", "g16_nv", "mla_nv", "mla_mx",
                                  "mla128_nv", "mla32_mx", "g32_cuda_nv", "mla8_cuda_mx"])
def test_decode_step_matches_oracle(ora, lib, name, chunk):
    """bdfp4_decode_step after a prefill of all but each sequence's newest token:
    the cache must equal the oracle's quantization of every token, the open
    value block must hold the new value, and the output must match the oracle's
    decode (and equal bdfp4_decode on the updated cache bit for bit).  Rows of
    the open block past the new token hold large noise the step must ignore."""
    _decode_step_case(ora, name, chunk, 0)


@pytest.mark.parametrize("chunk", [0, 1])
@pytest.mark.parametrize("name", ["tiny_nv", "ragged_g8_nv", "mla_nv"])
def test_decode_step_dynamic_alpha_matches_oracle(ora, lib, name, chunk):
    _decode_step_case(ora, name, chunk, bdfp4.FLAG_DYNAMIC_ALPHA)


@pytest.mark.parametrize("name", ["ragged_g8_nv", "ragged_g8_mx", "mla_nv", "mla8_cuda_mx"])
def test_decode_step_weighted_search_matches_oracle(ora, lib, name):
    """The step's key append takes the attention-aware search when the parameters carry weights."""
    _decode_step_case(ora, name, 1, 0, weighted=True)


def _decode_step_case(ora, name, chunk, flags, weighted=False):
    sp, fmt = SMALL[name]
    wl = Workload(sp, seed=8)
    smooth, kg, vg = oracle_calibration(ora, wl)
    w = None
    if weighted:
        _, qc, _ = wl.calibration("cpu")
        w = ora.key_weights(qc, sp.H_q, sp.H_kv, smooth)
    ocache = ora.empty_cache(wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt)
    ora.quantize_kv(wl.all_keys(), wl.all_values(), wl.slot_mapping_all(), ocache, sp.H_kv, fmt, smooth, kg, vg,
                    wl.num_pages, k_weight=w)
    kvp = kv_params_gpu(smooth, kg, vg)
    if weighted:
        kvp.k_weight = torch.from_numpy(w).cuda()
    gcache = bdfp4.FP4Cache.empty(wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt)
    for name_ in ("k_pages", "k_scales", "v_pages", "v_scales"):
        getattr(gcache, name_).zero_()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    beta = 16 if fmt == NV else 32
    gen = torch.Generator().manual_seed(9)
    k_new = torch.randn((sp.B, sp.H_kv, sp.d_k), generator=gen).to(torch.bfloat16)
    v_new = torch.randn((sp.B, sp.H_kv, sp.d_v), generator=gen).to(torch.bfloat16)
    v_open = (1e4 * torch.randn((sp.B, beta, sp.H_kv, sp.d_v), generator=gen)).to(torch.bfloat16)
    lasts = []
    for b in range(sp.B):
        n = int(wl.seq_lens[b])
        lasts.append((n - 1) % beta if n > 0 else -1)
        if n == 0:
            continue
        k, v = wl.keys(b), wl.values(b)
        if n > 1:
            sm = torch.from_numpy(wl.slot_mapping(b)).cuda()
            bdfp4.bdfp4_quantize_kv(k[:n - 1].cuda(), v[:n - 1].cuda(), sm[:n - 1], kvp, gcache, dev_status=status)
        last = lasts[-1]
        k_new[b] = k[n - 1]
        v_new[b] = v[n - 1]
        v_open[b, :last] = v[n - 1 - last:n - 1]
    q = wl.queries()
    if chunk <= 0:
        chunk = planned_chunk(wl)
    sl = torch.from_numpy(wl.seq_lens).cuda()
    bt = torch.from_numpy(wl.block_table).cuda()
    out = torch.empty((sp.B, sp.H_q, sp.d_v), dtype=torch.bfloat16, device="cuda")
    ws = bdfp4.workspace_for(sp.B, sp.H_q, sp.d_v, bt.shape[1], chunk)
    v_open_g = v_open.cuda()
    bdfp4.bdfp4_decode_step(q.cuda(), k_new.cuda(), v_new.cuda(), v_open_g, gcache, bt, sl, kvp, sp.sm_scale, chunk,
                            ws, out, flags=flags, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert_bytes_equal(cache_to_np(gcache), ocache)
    vo = v_open_g.cpu()
    for b, last in enumerate(lasts):
        if last >= 0:
            assert torch.equal(vo[b, last], v_new[b])
    ref16, _ = ora.decode(q, ocache, wl.block_table, wl.seq_lens, sp.H_kv, sp.d_v, fmt, smooth, kg, vg, sp.sm_scale,
                          chunk, wl.num_pages, flags=flags)
    got = out_to_np(out)
    assert_close(got, bf16_to_np(ref16))
    again, st2 = run_gpu_decode(wl, gcache, q, kvp, chunk, flags)
    assert st2 == 0 and torch.equal(again, out)


@pytest.mark.parametrize("fmt", [NV, MX])
def test_quantize_kv_adversarial_values(ora, lib, fmt):
    """Exact E2M1 midpoints (ties), zero blocks, tiny and huge values, runs
    that start mid-block, skipped tokens (-1), partial pages."""
    rng = np.random.default_rng(3)
    H_kv, d, T = 2, 128, 150
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0, 0.0])
    k = rng.choice(mids, size=(T, H_kv, d)) * rng.choice([-1, 1], size=(T, H_kv, d)) * 2.0 ** rng.integers(-3, 3, size=(T, H_kv, 1))
    v = rng.choice(mids, size=(T, H_kv, d)) * rng.choice([-1, 1], size=(T, H_kv, d)) * 2.0 ** rng.integers(-3, 3, size=(T, H_kv, 1))
    k[5] = 0.0
    v[20:40] = 0.0
    k[7] *= 1e-30
    v[9] *= 1e20
    k = torch.tensor(k, dtype=torch.float32).to(torch.bfloat16)
    v = torch.tensor(v, dtype=torch.float32).to(torch.bfloat16)
    # slots: a run starting mid-block, a skipped token, a run into a second page
    sm = np.concatenate([np.arange(3, 3 + 100), [-1], np.arange(64 * 2 + 10, 64 * 2 + 10 + 49)]).astype(np.int64)
    num_pages = 4
    for flags in (0, bdfp4.FLAG_NO_HADAMARD):
        smooth = (2.0 ** rng.integers(-2, 3, size=(H_kv, d))).astype(np.float32)
        kg = np.array([0.37, 0.011], np.float32)
        vg = np.array([0.05, 1.3], np.float32)
        ocache = ora.empty_cache(num_pages, H_kv, d, d, fmt)
        ora.quantize_kv(k, v, sm, ocache, H_kv, fmt, smooth, kg, vg, num_pages, flags=flags)
        gcache = bdfp4.FP4Cache.empty(num_pages, H_kv, d, d, fmt)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        bdfp4.bdfp4_quantize_kv(k.cuda(), v.cuda(), torch.from_numpy(sm).cuda(), kv_params_gpu(smooth, kg, vg), gcache,
                                flags=flags, dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert_bytes_equal(cache_to_np(gcache), ocache)


@pytest.mark.parametrize("flags", [0, bdfp4.FLAG_SINGLE_QUERY, bdfp4.FLAG_NO_HADAMARD])
@pytest.mark.parametrize("name", ["tiny_nv", "tiny_mx", "ragged_g8_nv", "mla_nv", "mla_mx"])
def test_quantize_q_bit_exact(ora, lib, name, flags):
    sp, fmt = SMALL[name]
    wl = Workload(sp, seed=4)
    smooth, _, _ = oracle_calibration(ora, wl, flags)
    q = wl.queries("cpu")
    ref = ora.quantize_q(q, sp.H_kv, fmt, smooth, flags=flags)
    got = bdfp4.bdfp4_quantize_q(q.cuda(), sp.H_kv, fmt, torch.from_numpy(smooth).cuda(), flags=flags)
    torch.cuda.synchronize()
    for key in ("q1_codes", "q1_scales", "q2_codes", "q2_scales", "g_q"):
        assert np.array_equal(got[key].cpu().numpy(), ref[key]), key


def _decode_case(ora, name, chunk_tiles, flags, seed=5):
    sp, fmt = SMALL[name]
    wl = Workload(sp, seed=seed)
    smooth, kg, vg = oracle_calibration(ora, wl, flags & bdfp4.FLAG_NO_HADAMARD)
    q = wl.queries("cpu")
    ocache = ora.empty_cache(wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt)
    ora.quantize_kv(wl.all_keys(), wl.all_values(), wl.slot_mapping_all(), ocache, sp.H_kv, fmt, smooth, kg, vg,
                    wl.num_pages, flags=flags & bdfp4.FLAG_NO_HADAMARD)
    if chunk_tiles <= 0:
        chunk_tiles = planned_chunk(wl)
    ref16, _ = ora.decode(q, ocache, wl.block_table, wl.seq_lens, sp.H_kv, sp.d_v, fmt, smooth, kg, vg, sp.sm_scale,
                          chunk_tiles, wl.num_pages, flags=flags)
    gcache = cache_from_np(ocache, wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt)
    out, status = run_gpu_decode(wl, gcache, q, kv_params_gpu(smooth, kg, vg), chunk_tiles, flags)
    assert status == 0
    return out_to_np(out), bf16_to_np(ref16), wl


@pytest.mark.parametrize("chunk", [0, 1, 3])
@pytest.mark.parametrize("name", list(SMALL))
def test_decode_matches_oracle(ora, lib, name, chunk):
    got, ref, wl = _decode_case(ora, name, chunk, 0)
    assert_close(got, ref)
    for b, n in enumerate(wl.seq_lens):
        if n == 0:
            assert np.all(got[b] == 0)


@pytest.mark.parametrize("flags", [bdfp4.FLAG_SINGLE_QUERY, bdfp4.FLAG_NO_UNDERFLOW, bdfp4.FLAG_NO_HADAMARD,
                                   bdfp4.FLAG_SINGLE_QUERY | bdfp4.FLAG_NO_UNDERFLOW])
@pytest.mark.parametrize("name", ["tiny_nv", "ragged_g8_nv", "ragged_g8_mx"])
def test_decode_ablation_flags_match_oracle(ora, lib, name, flags):
    got, ref, _ = _decode_case(ora, name, 2, flags)
    assert_close(got, ref)


@pytest.mark.parametrize("chunk", [0, 2])
@pytest.mark.parametrize("name", ["tiny_nv", "ragged_g8_nv", "g16_nv", "g32_cuda_nv", "mla_nv", "mla64_nv",
                                  "tiny_mx", "mla_mx"])
def test_decode_dynamic_alpha_matches_oracle(ora, lib, name, chunk):
    got, ref, _ = _decode_case(ora, name, chunk, bdfp4.FLAG_DYNAMIC_ALPHA)
    assert_close(got, ref)


@pytest.mark.parametrize("name", ["mla_nv", "mla64_nv", "mla128_nv"])
def test_dynamic_alpha_runs_on_the_mla_tensor_core_kernel(ora, lib, name):
    """MLA shapes with the per-tile pre-scale take the tensor-core kernel: it needs a
    workspace for its query images even with one split, which the CUDA-core decode
    does not, so a workspace-less single-split call is refused before any launch."""
    sp, fmt = SMALL[name]
    wl = Workload(sp, seed=5)
    smooth, kg, vg = oracle_calibration(ora, wl)
    gcache = bdfp4.FP4Cache.empty(wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt)
    one_split = (wl.max_pages * 64 + 127) // 128
    out = torch.empty((sp.B, sp.H_q, sp.d_v), dtype=torch.bfloat16, device="cuda")
    args = (wl.queries().cuda(), gcache, torch.from_numpy(wl.block_table).cuda(), torch.from_numpy(wl.seq_lens).cuda(),
            kv_params_gpu(smooth, kg, vg), sp.sm_scale, one_split, None, out)
    with pytest.raises(bdfp4.BDFP4Error, match="workspace"):
        bdfp4.bdfp4_decode(*args, flags=bdfp4.FLAG_DYNAMIC_ALPHA)
    # a shape the tensor-core kernels do not take runs without one
    sp8, _ = SMALL["mla8_cuda_mx"]
    wl8 = Workload(sp8, seed=5)
    s8, k8, v8 = oracle_calibration(ora, wl8)
    c8 = bdfp4.FP4Cache.empty(wl8.num_pages, sp8.H_kv, sp8.d_k, sp8.d_v, NV)
    o8 = torch.empty((sp8.B, sp8.H_q, sp8.d_v), dtype=torch.bfloat16, device="cuda")
    bdfp4.bdfp4_decode(wl8.queries().cuda(), c8, torch.from_numpy(wl8.block_table).cuda(),
                       torch.from_numpy(wl8.seq_lens).cuda(), kv_params_gpu(s8, k8, v8), sp8.sm_scale,
                       (wl8.max_pages * 64 + 127) // 128, None, o8, flags=bdfp4.FLAG_DYNAMIC_ALPHA)
    torch.cuda.synchronize()


@pytest.mark.parametrize("chunk", [0, 1])
@pytest.mark.parametrize("name", ["mla_nv", "mla128_nv"])
def test_decode_step_dynamic_alpha_mla_matches_oracle(ora, lib, name, chunk):
    _decode_step_case(ora, name, chunk, bdfp4.FLAG_DYNAMIC_ALPHA)


def test_dynamic_alpha_keeps_a_deep_sink_tail(ora, lib):
    """One key with logit 14 and 131071 with logit 0, one split: with alpha = 2^11
    every block without the sink collapses (E4M3(e^-14 2^11 / 6) = 0), a tenth of
    the attention mass; the per-tile pre-scale keeps it.  Both arms match the
    oracle; against the unquantized-P output both keep the sink block's own
    error (P^ = 1.03125 p on 90% of the mass, about 2.5%), and the static arm
    adds the lost tail (about 7% in all)."""
    N, H_kv, G, d = 131072, 1, 2, 128
    rng = np.random.default_rng(11)
    q = np.zeros((1, G, d), np.float32)
    q[0, :, 0] = 6.0
    k = np.zeros((N, H_kv, d), np.float32)
    k[0, 0, 0] = 6.0
    v = rng.uniform(0.5, 1.5, (N, H_kv, d)).astype(np.float32)
    npages = N // 64
    bt = rng.permutation(npages).astype(np.int32)[None, :]
    t = np.arange(N)
    slots = bt[0, t // 64].astype(np.int64) * 64 + t % 64
    ones = np.ones((H_kv, d), np.float32)
    g = np.ones(H_kv, np.float32)
    ocache = ora.empty_cache(npages, H_kv, d, d, NV)
    qb = torch.from_numpy(q).to(torch.bfloat16)
    ora.quantize_kv(torch.from_numpy(k).to(torch.bfloat16), torch.from_numpy(v).to(torch.bfloat16), slots, ocache,
                    H_kv, NV, ones, g, g, npages, flags=bdfp4.FLAG_NO_HADAMARD)
    gcache = cache_from_np(ocache, npages, H_kv, d, d, NV)
    sl = np.array([N], np.int32)
    sm_scale, chunk = 14.0 / 36.0, N // 128
    outs = {}
    for name, fl in (("static", 0), ("dynamic", bdfp4.FLAG_DYNAMIC_ALPHA)):
        fl |= bdfp4.FLAG_NO_HADAMARD
        ref16, _ = ora.decode(qb, ocache, bt, sl, H_kv, d, NV, ones, g, g, sm_scale, chunk, npages, flags=fl)
        out = torch.empty((1, G, d), dtype=torch.bfloat16, device="cuda")
        ws = bdfp4.workspace_for(1, G, d, npages, chunk)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        bdfp4.bdfp4_decode(qb.cuda(), gcache, torch.from_numpy(bt).cuda(), torch.from_numpy(sl).cuda(),
                           kv_params_gpu(ones, g, g), sm_scale, chunk, ws, out, flags=fl, dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        got = out_to_np(out)
        assert_close(got, bf16_to_np(ref16), name)
        outs[name] = got.astype(np.float64)
    _, exact = ora.decode(qb, ocache, bt, sl, H_kv, d, NV, ones, g, g, sm_scale, chunk, npages,
                          flags=bdfp4.FLAG_NO_HADAMARD | ora.FLAG_EXACT_P)
    err = {n: np.linalg.norm(o - exact) / np.linalg.norm(exact) for n, o in outs.items()}
    assert err["dynamic"] < 0.03 and err["static"] > err["dynamic"] + 0.04, err


def test_decode_empty_and_single_token(ora, lib):
    sp = spec("tiny", B=3, ctx=("list", (0, 1, 65)))
    SMALL["edge"] = (sp, NV)
    try:
        got, ref, wl = _decode_case(ora, "edge", 1, 0)
    finally:
        del SMALL["edge"]
    assert np.all(got[0] == 0)
    assert_close(got, ref)


def test_device_status_on_bad_block_table(ora, lib):
    """An out-of-range page id is reported through dev_status and skipped."""
    sp, fmt = SMALL["tiny_nv"]
    wl = Workload(sp, seed=6)
    smooth, kg, vg = oracle_calibration(ora, wl)
    gcache, _ = quantize_both(ora, wl, fmt, smooth, kg, vg)
    bt = wl.block_table.copy()
    bt[0, 3] = wl.num_pages + 100
    out, status = run_gpu_decode(wl, gcache, wl.queries(), kv_params_gpu(smooth, kg, vg), 2, block_table=bt)
    assert status & bdfp4.DEV_BAD_PAGE
    assert np.isfinite(out_to_np(out)).all()
    # a sequence longer than the table allows is reported too
    out, status = run_gpu_decode(wl, gcache, wl.queries(), kv_params_gpu(smooth, kg, vg), 2,
                                 seq_lens=[sp.ctx[1] + 10**6])
    assert status & bdfp4.DEV_BAD_SEQLEN


@pytest.mark.parametrize("name", ["ragged_g8_nv", "ragged_g8_mx", "mla32_mx", "mla128_nv"])
def test_bad_page_leaves_other_sequences_exact(ora, lib, name):
    """A page id outside the cache in one sequence is reported, that sequence's output
    stays finite (its page's tokens are skipped), and every other sequence of the batch
    matches the oracle run on the intact block table, split plan included."""
    sp, fmt = SMALL[name]
    wl = Workload(sp, seed=11)
    smooth, kg, vg = oracle_calibration(ora, wl)
    gcache, ocache = quantize_both(ora, wl, fmt, smooth, kg, vg)
    q = wl.queries()
    chunk = 1   # many splits: the bad page's split and its neighbours all run
    ref16, _ = ora.decode(q, ocache, wl.block_table, wl.seq_lens, sp.H_kv, sp.d_v, fmt, smooth, kg, vg, sp.sm_scale,
                          chunk, wl.num_pages)
    bad_seq = int(np.argmax(wl.seq_lens))
    bt = wl.block_table.copy()
    bt[bad_seq, 1] = -7   # the second page of the longest sequence
    out, status = run_gpu_decode(wl, gcache, q, kv_params_gpu(smooth, kg, vg), chunk, block_table=bt)
    assert status & bdfp4.DEV_BAD_PAGE
    got = out_to_np(out)
    assert np.isfinite(got).all()
    ref = bf16_to_np(ref16)
    others = [b for b in range(sp.B) if b != bad_seq]
    assert_close(got[others], ref[others])


def test_quantize_then_decode_end_to_end(ora, lib):
    """GPU quantizer -> GPU decode against oracle quantizer -> oracle decode."""
    sp, fmt = SMALL["ragged_g8_nv"]
    wl = Workload(sp, seed=7)
    kc, qc, vc = wl.calibration("cpu")
    kv = bdfp4.bdfp4_calibrate(kc.cuda(), qc.cuda(), vc.cuda(), sp.H_q, sp.H_kv)
    smooth, kg, vg = oracle_calibration(ora, wl)
    gcache, ocache = quantize_both(ora, wl, fmt, smooth, kg, vg)
    q = wl.queries()
    chunk = planned_chunk(wl)
    out, status = run_gpu_decode(wl, gcache, q, kv, chunk)
    ref16, _ = ora.decode(q, ocache, wl.block_table, wl.seq_lens, sp.H_kv, sp.d_v, fmt, smooth, kg, vg, sp.sm_scale,
                          chunk, wl.num_pages)
    assert status == 0
    assert_close(out_to_np(out), bf16_to_np(ref16))


@pytest.mark.parametrize("name", ["ragged_g8_nv", "ragged_g8_mx", "mla_nv", "mla128_mx", "g32_cuda_nv"])
def test_sequence_with_only_bad_pages_gives_zeros_at_every_plan(ora, lib, name):
    """Every block-table entry of one sequence outside the cache: each split of it sees
    only masked tokens (m = -inf, l = 0), so the merge has nothing to weigh.  The
    sequence's output must be zeros -- as a single split writes it -- whatever the
    split plan, and the other sequences must still match the oracle."""
    sp, fmt = SMALL[name]
    wl = Workload(sp, seed=13)
    smooth, kg, vg = oracle_calibration(ora, wl)
    gcache, ocache = quantize_both(ora, wl, fmt, smooth, kg, vg)
    q = wl.queries()
    bad_seq = int(np.argmax(wl.seq_lens))
    bt = wl.block_table.copy()
    bt[bad_seq, :] = wl.num_pages + 5
    others = [b for b in range(sp.B) if b != bad_seq]
    for chunk in (1, planned_chunk(wl)):
        out, status = run_gpu_decode(wl, gcache, q, kv_params_gpu(smooth, kg, vg), chunk, block_table=bt)
        assert status & bdfp4.DEV_BAD_PAGE
        got = out_to_np(out)
        assert np.isfinite(got).all(), chunk
        assert np.all(got[bad_seq] == 0), chunk
        ref16, _ = ora.decode(q, ocache, wl.block_table, wl.seq_lens, sp.H_kv, sp.d_v, fmt, smooth, kg, vg,
                              sp.sm_scale, chunk, wl.num_pages)
        assert_close(got[others], bf16_to_np(ref16)[others], chunk)
