"""Error report of the FP4 method, measured on the oracle (CPU).

The CUDA path reproduces the oracle's cache bytes exactly and its decode
outputs within max-abs 1e-2 / relative L2 5e-3 (tests/test_gpu_parity.py), so
these are the errors of the GPU results too:

* query-logit relative error, with the dual-residual query and with a single
  FP4 query (q2 = 0): of the query alone, ||(q1 + q2 - q') . k'|| / ||q' . k'||
  with exact transformed keys k', and of the whole FP4 logit (q1 + q2) . k^
  against the exact q . k;
* decode output error against fp64 softmax(q K^T) V on the unquantized bf16
  q, K, V (the BF16-KV result), for the method and its ablations;
* the underflow stress: the error that probability quantization adds (output
  against the same cache decoded with exact probabilities) with the
  underflow-aware alpha = 2^11 and with alpha = 1, for near-uniform logits
  (keys N(0, 0.05^2)) and for a batch with a planted sink token per 4096 tokens
  (logit +12 over a N(0, 1.5^2)-logit bulk), where alpha = 1 collapses the
  small probabilities, and the per-tile alpha variant on these and on a deep
  sink (logit +16 in 131072 tokens), where alpha = 2^11 collapses them too.

Each test asserts the ordering the method must show and records its numbers;
with BDFP4_REPORT=<path> the collected figures are written there as JSON."""
import json
import math
import os

import numpy as np
import pytest
import torch

from _util import oracle_calibration
from fp4_kv_cache_quant_b200.workloads import Workload, spec

NV, MX = 0, 1
FLAG_NO_HADAMARD, FLAG_NO_SCALE_SEARCH, FLAG_SINGLE_QUERY, FLAG_NO_UNDERFLOW, FLAG_EXACT_P = 1, 2, 4, 8, 16
FLAG_DYNAMIC_ALPHA = 32

REPORT = {}


@pytest.fixture(scope="module", autouse=True)
def _write_report():
    yield
    path = os.environ.get("BDFP4_REPORT")
    if path and REPORT:
        with open(path, "w") as f:
            json.dump(REPORT, f, indent=2, sort_keys=True)


def _bits_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().numpy().astype(np.float64)


def _rel(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _quantized_cache(ora, wl: Workload, fmt: int, flags: int = 0):
    sp = wl.spec
    smooth, kg, vg = oracle_calibration(ora, wl, flags & FLAG_NO_HADAMARD)
    cache = ora.empty_cache(wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt)
    ora.quantize_kv(wl.all_keys(), wl.all_values(), wl.slot_mapping_all(), cache, sp.H_kv, fmt, smooth, kg, vg,
                    wl.num_pages, flags=flags & (FLAG_NO_HADAMARD | FLAG_NO_SCALE_SEARCH))
    return cache, smooth, kg, vg


def _dequant_query(ora, qz: dict, fmt: int, which: int) -> np.ndarray:
    """q1 (which = 1) or q2 (which = 2) in the transformed space, fp64 [B, H_q, d]."""
    codes = qz[f"q{which}_codes"].astype(np.int64)
    scales = qz[f"q{which}_scales"].astype(np.int64)
    B, H_q, d = codes.shape
    beta = d // scales.shape[2]
    e2m1 = np.array([ora.e2m1_value(c) for c in range(16)], np.float64)
    out = np.zeros((B, H_q, d), np.float64)
    for bb in range(B):
        for h in range(H_q):
            g = float(qz["g_q"][bb, h])
            sig = np.array([ora.block_sigma(fmt, int(c), g) for c in scales[bb, h]], np.float64)
            out[bb, h] = e2m1[codes[bb, h]] * np.repeat(sig, beta)
    return out


@pytest.mark.parametrize("fmt", [NV, MX])
def test_query_logit_error_dual_vs_single(ora, fmt):
    sp = spec("qwen3_4b", B=2, ctx=("fixed", 1024))
    wl = Workload(sp, seed=21)
    cache, smooth, kg, vg = _quantized_cache(ora, wl, fmt)
    q = wl.queries("cpu")
    G = sp.H_q // sp.H_kv
    errs = {}
    for name, flags in (("dual", 0), ("single", FLAG_SINGLE_QUERY)):
        qz = ora.quantize_q(q, sp.H_kv, fmt, smooth, flags=flags)
        qd = _dequant_query(ora, qz, fmt, 1) + _dequant_query(ora, qz, fmt, 2)
        qx = qz["xq"].astype(np.float64)                   # q' (transformed, unquantized)
        nq = dq = nt = dt = 0.0
        for b in range(sp.B):
            k = _bits_f64(wl.keys(b))                       # [n, H_kv, d] raw bf16
            slots = wl.slot_mapping(b)
            for hk in range(sp.H_kv):
                kx = ora.transform(k[:, hk, :], smooth[hk], True).astype(np.float64)   # k'
                gk = float(kg[hk]) if fmt == NV else 1.0
                kd = gk * np.stack([ora.dequant_key_row(cache, fmt, int(s) // 64, hk, sp.H_kv, sp.d_k, int(s) % 64)
                                    for s in slots])        # k^ (FP4 key in the transformed space)
                for h in range(hk * G, (hk + 1) * G):
                    ref = kx @ qx[b, h]                     # q'.k'
                    nq += float(np.sum((kx @ qd[b, h] - ref) ** 2))
                    dq += float(np.sum(ref ** 2))
                    exact = k[:, hk, :] @ _bits_f64(q[b, h])     # q.k (= q'.k' in exact arithmetic)
                    nt += float(np.sum((kd @ qd[b, h] - exact) ** 2))
                    dt += float(np.sum(exact ** 2))
        errs[name] = {"query_only": math.sqrt(nq / dq), "fp4_logit": math.sqrt(nt / dt)}
    REPORT[f"logit_rel_err_{'nvfp4' if fmt == NV else 'mxfp4'}"] = errs
    print(f"\nquery-logit relative error ({'NVFP4' if fmt == NV else 'MXFP4'}): query alone dual "
          f"{errs['dual']['query_only']:.4f} vs single {errs['single']['query_only']:.4f}; whole FP4 logit dual "
          f"{errs['dual']['fp4_logit']:.4f} vs single {errs['single']['fp4_logit']:.4f}")
    # the residual tensor removes most of the query's own quantization error ...
    assert errs["dual"]["query_only"] < errs["single"]["query_only"] / 3
    # ... and never makes the whole logit worse (the FP4 keys' error remains)
    assert errs["dual"]["fp4_logit"] < errs["single"]["fp4_logit"]


@pytest.mark.parametrize("fmt", [NV, MX])
def test_output_error_against_bf16_kv(ora, fmt):
    sp = spec("qwen3_4b", B=2, ctx=("list", (2048, 777)))
    wl = Workload(sp, seed=22)
    q = wl.queries("cpu")
    truth = ora.attention_ref(q, wl.all_keys(), wl.all_values(), wl.cu_seqlens, sp.H_kv, sp.sm_scale)
    arms = {"method": 0, "single_query": FLAG_SINGLE_QUERY, "no_hadamard": FLAG_NO_HADAMARD,
            "no_scale_search": FLAG_NO_SCALE_SEARCH}
    if fmt == NV:
        arms["alpha_1"] = FLAG_NO_UNDERFLOW
    errs = {}
    for name, flags in arms.items():
        cache, smooth, kg, vg = _quantized_cache(ora, wl, fmt, flags)
        _, out = ora.decode(q, cache, wl.block_table, wl.seq_lens, sp.H_kv, sp.d_v, fmt, smooth, kg, vg,
                            sp.sm_scale, 8, wl.num_pages, flags=flags)
        errs[name] = _rel(out, truth)
    REPORT[f"output_rel_err_vs_bf16_{'nvfp4' if fmt == NV else 'mxfp4'}"] = errs
    print(f"\noutput relative L2 error vs BF16-KV attention ({'NVFP4' if fmt == NV else 'MXFP4'}): " +
          ", ".join(f"{k} {v:.4f}" for k, v in errs.items()))
    assert errs["method"] < 0.2
    assert errs["method"] <= errs["single_query"]


def _sink_workload(seed: int, n: int, period: int = 4096, sink_logit: float = 12.0):
    """One KV head, G = 1: bulk logits N(0, 1.5^2), one sink token (logit +12, or
    `sink_logit`) per `period` tokens; bulk values mu + 0.3 N(0, 1) around a common
    mu, sink values N(0, 1)."""
    rng = np.random.default_rng(seed)
    d = 128
    sm = 1.0 / math.sqrt(d)
    q = rng.standard_normal(d)
    qn = q / np.linalg.norm(q)
    # bulk: logit (sm * q.k) ~ N(0, 1.5^2) along q, isotropic noise elsewhere
    z = rng.standard_normal((n, d))
    z -= np.outer(z @ qn, qn)
    along = rng.standard_normal(n) * 1.5 / (sm * np.linalg.norm(q))
    k = z + np.outer(along, qn)
    k[::period] = z[::period] + np.outer(np.full(len(range(0, n, period)), sink_logit / (sm * np.linalg.norm(q))),
                                         qn)
    # the bulk's values share a direction, so the mass in its small probabilities
    # carries signal (random values would let a dropped bulk cancel out)
    mu = rng.standard_normal(d)
    v = mu + 0.3 * rng.standard_normal((n, d))
    v[::period] = rng.standard_normal((len(range(0, n, period)), d))
    bf = lambda a: torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)  # noqa: E731
    return bf(q).reshape(1, 1, d), bf(k).reshape(n, 1, d), bf(v).reshape(n, 1, d), sm


def _decode_pages(ora, q, k, v, sm, fmt, flags):
    n, H_kv, d = k.shape
    npg = (n + 63) // 64
    bt = np.arange(npg, dtype=np.int32).reshape(1, npg)
    slots = np.arange(n, dtype=np.int64)
    kc, qc = k[:1024].clone(), q.repeat(64, 1, 1)
    smooth, kg, vg = ora.calibrate(kc, qc, v[:1024].clone(), 1, 1, flags=flags & FLAG_NO_HADAMARD)
    cache = ora.empty_cache(npg, H_kv, d, d, fmt)
    ora.quantize_kv(k, v, slots, cache, H_kv, fmt, smooth, kg, vg, npg, flags=flags & FLAG_NO_HADAMARD)
    _, out = ora.decode(q, cache, bt, np.array([n], np.int32), H_kv, d, fmt, smooth, kg, vg, sm, 1 << 20, npg,
                        flags=flags)
    return out


def test_underflow_alpha_near_uniform(ora):
    """Near-uniform logits (keys N(0, 0.05^2)): every p is near 1, so alpha has nothing to rescue."""
    sp = spec("underflow", B=1, H_q=4, H_kv=1, ctx=("fixed", 16384))
    wl = Workload(sp, seed=23)
    q = wl.queries("cpu")
    cache, smooth, kg, vg = _quantized_cache(ora, wl, NV)
    outs = {}
    for name, flags in (("exact_p", FLAG_EXACT_P), ("alpha_2^11", 0), ("alpha_1", FLAG_NO_UNDERFLOW),
                        ("alpha_per_tile", FLAG_DYNAMIC_ALPHA)):
        _, outs[name] = ora.decode(q, cache, wl.block_table, wl.seq_lens, sp.H_kv, sp.d_v, NV, smooth, kg, vg,
                                   sp.sm_scale, 1 << 20, wl.num_pages, flags=flags)
    errs = {name: _rel(outs[name], outs["exact_p"]) for name in ("alpha_2^11", "alpha_1", "alpha_per_tile")}
    REPORT["underflow_near_uniform_nvfp4"] = errs
    print(f"\nnear-uniform logits, 16384 tokens, error added by P quantization: alpha=2^11 "
          f"{errs['alpha_2^11']:.5f}, alpha=1 {errs['alpha_1']:.5f}, per-tile alpha {errs['alpha_per_tile']:.5f}")
    assert abs(errs["alpha_2^11"] - errs["alpha_1"]) <= 0.1 * errs["alpha_1"] + 1e-4
    # every tile's largest p stays above 2688 / 4096 of the running maximum: the per-tile exponent is 11
    assert np.array_equal(outs["alpha_per_tile"], outs["alpha_2^11"])


def test_underflow_alpha_sink_stress(ora):
    """A sink per 4096 tokens: with alpha = 1 every block without a sink falls below
    the smallest E4M3 scale and is dropped; alpha = 2^11 keeps them."""
    q, k, v, sm = _sink_workload(24, 16384)
    ref = _decode_pages(ora, q, k, v, sm, NV, FLAG_EXACT_P)
    errs = {name: _rel(_decode_pages(ora, q, k, v, sm, NV, flags), ref)
            for name, flags in (("alpha_2^11", 0), ("alpha_1", FLAG_NO_UNDERFLOW),
                                ("alpha_per_tile", FLAG_DYNAMIC_ALPHA))}
    REPORT["underflow_sink_stress_nvfp4"] = errs
    print(f"\nsink stress, 16384 tokens, error added by P quantization: alpha=2^11 {errs['alpha_2^11']:.5f}, "
          f"alpha=1 {errs['alpha_1']:.5f}, per-tile alpha {errs['alpha_per_tile']:.5f}")
    assert errs["alpha_2^11"] < errs["alpha_1"] / 2
    assert errs["alpha_per_tile"] <= errs["alpha_2^11"] * 1.05


def test_underflow_deep_sink_per_tile_alpha(ora):
    """One sink of logit +16 in 131072 tokens: the bulk's blocks fall below the
    smallest E4M3 scale even at alpha = 2^11 (block maxima near e^-13 x 2^11 / 6),
    while holding about 5% of the attention mass; the per-tile alpha of the tiles
    without the sink keeps them.  What remains (about 0.03) is the sink block's
    own error: P^ = 1.03125 p on 95% of the mass, the same in both arms."""
    q, k, v, sm = _sink_workload(25, 131072, period=131072, sink_logit=16.0)
    ref = _decode_pages(ora, q, k, v, sm, NV, FLAG_EXACT_P)
    errs = {name: _rel(_decode_pages(ora, q, k, v, sm, NV, flags), ref)
            for name, flags in (("alpha_2^11", 0), ("alpha_1", FLAG_NO_UNDERFLOW),
                                ("alpha_per_tile", FLAG_DYNAMIC_ALPHA))}
    REPORT["underflow_deep_sink_nvfp4"] = errs
    print(f"\ndeep sink, 131072 tokens, error added by P quantization: alpha=2^11 {errs['alpha_2^11']:.5f}, "
          f"alpha=1 {errs['alpha_1']:.5f}, per-tile alpha {errs['alpha_per_tile']:.5f}")
    assert errs["alpha_per_tile"] < 0.8 * errs["alpha_2^11"]
