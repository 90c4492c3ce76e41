"""Host-only checks of the C ABI: the library loads, exports every entry point
include/bdfp4.h declares, and rejects bad arguments before touching a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

from fp4_kv_cache_quant_b200 import bdfp4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from fp4_kv_cache_quant_b200 import build
    build.build()
    return bdfp4.load()


def _declared():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"BDFP4_API\s+[\w\s\*]+?\b(bdfp4_\w+)\s*\(", src)
    return names


def test_exports_every_declared_entry_point(lib):
    names = _declared()
    assert set(bdfp4.ENTRY_POINTS) <= set(names)
    assert set(bdfp4.BF16_ENTRY_POINTS) <= set(names)
    assert set(bdfp4.DEBUG_ENTRY_POINTS) <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_kv_params_struct_matches_the_header(lib):
    """bdfp4_kv_params: four device pointers in the header's order."""
    hdr = open(os.path.join(ROOT, "include", "bdfp4.h")).read()
    body = re.search(r"typedef struct \{(.*?)\} bdfp4_kv_params;", hdr, re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = re.findall(r"const float\*\s*(\w+);", body)
    assert fields == [f for f, _ in bdfp4._KVParams._fields_] == ["smooth", "k_gscale", "v_gscale", "k_weight"]
    assert ctypes.sizeof(bdfp4._KVParams) == 4 * ctypes.sizeof(ctypes.c_void_p)


def test_key_weights_argument_errors(lib):
    a = _p(0x10000)
    assert lib.bdfp4_key_weights(a, 8, 8, 2, 64, 0, a, a, None) == -4      # head dim outside the set
    assert lib.bdfp4_key_weights(a, 8, 6, 4, 128, 0, a, a, None) == -2     # 6 query heads over 4 KV heads
    assert lib.bdfp4_key_weights(None, 8, 8, 2, 128, 0, a, a, None) == -1
    assert lib.bdfp4_key_weights(a, 0, 8, 2, 128, 0, a, a, None) == -1
    assert lib.bdfp4_key_weights(_p(0x10001), 8, 8, 2, 128, 0, a, a, None) == -3


def test_status_strings(lib):
    for code in range(-6, 1):
        s = bdfp4.bdfp4_status_string(code)
        assert s and s != "unknown status"
    assert bdfp4.bdfp4_status_string(42) == "unknown status"


def test_decode_plan_host_logic(lib):
    # the split length c in [16, 64] (at most the longest sequence) minimising
    # ceil(CTAs / (4 * SMs)) * (c + 3), CTAs = KV heads * sum over sequences of ceil(tiles / c)
    # 16 sequences of 32768 tokens (256 tiles), 8 KV heads, 148 SMs: c = 29 gives 9 splits per
    # sequence, 1152 CTAs = 2 waves of 592 -> 2 * 32 = 64, the least over 16 .. 64
    assert bdfp4.bdfp4_decode_plan(np.full(16, 32768), 8, 148) == 29
    # at most the longest sequence; one wave of 3 CTAs at c = 16 beats longer splits
    assert bdfp4.bdfp4_decode_plan(np.array([1000]), 1, 148) == 8
    assert bdfp4.bdfp4_decode_plan(np.array([5000]), 1, 148) == 16
    assert bdfp4.bdfp4_decode_plan(np.array([100]), 1, 148) == 1
    # 64 x 131072 tokens x 4 heads: 1024 tiles each; c = 64 -> 4096 CTAs = 7 waves * 67 = 469
    assert bdfp4.bdfp4_decode_plan(np.full(64, 131072), 4, 148) == 64
    # 16 x 65536 tokens x 8 heads: 512 tiles each; c = 57 -> 10 splits, 1280 CTAs = 3 waves * 60
    assert bdfp4.bdfp4_decode_plan(np.full(16, 65536), 8, 148) == 57
    assert bdfp4.bdfp4_decode_plan(np.array([0, 0]), 2, 148) == 1


def test_decode_plan_for_kernel_shapes(lib):
    # d = 128 with four query heads per KV head: four CTAs per SM, as bdfp4_decode_plan
    assert bdfp4.bdfp4_decode_plan_for(np.full(16, 32768), 32, 8, 128, 128, 148) == 29
    # eight heads per KV head: three CTAs per SM; 16 x 512 tiles x 8 heads: c = 52 -> 10 splits,
    # 1280 CTAs = 3 waves of 444 -> 3 * 55 = 165, the least over 16 .. 64
    assert bdfp4.bdfp4_decode_plan_for(np.full(16, 65536), 64, 8, 128, 128, 148) == 52
    # MLA, 128 heads over one latent head: two 64-head slices per split, one CTA per SM;
    # 32 x 128 tiles: c = 64 -> 128 CTAs in one wave of 148 -> 67
    assert bdfp4.bdfp4_decode_plan_for(np.full(32, 16384), 128, 1, 576, 512, 148) == 64
    with pytest.raises(bdfp4.BDFP4Error):
        bdfp4.bdfp4_decode_plan_for(np.array([10]), 6, 4, 128, 128, 148)   # 6 query heads over 4 KV heads
    with pytest.raises(bdfp4.BDFP4Error):
        bdfp4.bdfp4_decode_plan_for(np.array([10]), 4, 4, 64, 64, 148)     # head dims outside the set
    with pytest.raises(bdfp4.BDFP4Error):
        bdfp4.bdfp4_decode_plan(np.array([10]), 0, 148)


def test_workspace_size(lib):
    # B=2, H_q=4, d_v=128, 16 pages = 8 tiles, 2 tiles per split -> 4 splits: fp32 partial
    # outputs and (m, l) pairs, each padded to 256 B, then 656 B of query image per query head
    o = 2 * 4 * 4 * 128 * 4
    ml = 2 * 4 * 4 * 2 * 4
    q = 2 * 4 * 656
    pad = lambda n: (n + 255) // 256 * 256  # noqa: E731
    assert bdfp4.bdfp4_decode_workspace_size(2, 4, 128, 16, 2) == pad(o) + pad(ml) + q
    # one split per sequence: only the query images
    assert bdfp4.bdfp4_decode_workspace_size(2, 4, 128, 16, 8) == q
    assert bdfp4.bdfp4_decode_workspace_size(0, 4, 128, 16, 2) == 0


def _p(addr):
    return ctypes.c_void_p(addr)


def test_quantize_kv_argument_errors(lib):
    kv = bdfp4._KVParams(0x1000, 0x2000, 0x3000)
    a = _p(0x10000)
    args = lambda d_k=128, d_v=128, fmt=0, k=a, kvp=ctypes.byref(kv): (  # noqa: E731
        k, a, a, 10, 2, d_k, d_v, fmt, 0, kvp, a, a, a, a, 4, None, None)
    assert lib.bdfp4_quantize_kv(*args(d_k=64)) == -4
    assert lib.bdfp4_quantize_kv(*args(d_k=576, d_v=128)) == -4
    assert lib.bdfp4_quantize_kv(*args(fmt=7)) == -1
    assert lib.bdfp4_quantize_kv(*args(k=None)) == -1
    assert lib.bdfp4_quantize_kv(*args(kvp=None)) == -1
    assert lib.bdfp4_quantize_kv(*args(k=_p(0x10001))) == -3


def test_decode_argument_errors(lib):
    kv = bdfp4._KVParams(0x1000, 0x2000, 0x3000)
    a = _p(0x10000)

    def call(H_q=8, H_kv=2, d_k=128, d_v=128, chunk=1, ws=None, ws_bytes=0, q=a, max_pages=4, flags=0):
        return lib.bdfp4_decode(q, a, a, a, a, a, a, 2, H_q, H_kv, d_k, d_v, max_pages, 16, 0, flags,
                                ctypes.byref(kv), 0.1, chunk, ws, ws_bytes, a, None, None)
    assert call(H_q=6, H_kv=2) == -4      # group of 3
    assert call(H_q=7, H_kv=2) == -2      # not a multiple
    assert call(d_k=256) == -4
    assert call(q=None) == -1
    assert call(q=_p(0x10008)) == -3
    assert call(chunk=1) == -6            # 2 splits need a workspace
    n = bdfp4.bdfp4_decode_workspace_size(2, 8, 128, 4, 1)
    assert call(chunk=1, ws=_p(0x20000), ws_bytes=n - 1) == -6
    # the dynamic probability pre-scale and the vanilla alpha = 1 ablation exclude each other
    assert call(flags=bdfp4.FLAG_DYNAMIC_ALPHA | bdfp4.FLAG_NO_UNDERFLOW) == -1


def test_decode_multi_argument_errors_and_plan(lib):
    kv = bdfp4._KVParams(0x1000, 0x2000, 0x3000)
    a = _p(0x10000)

    def call(T=2, H_q=8, H_kv=2, chunk=1, ws=None, ws_bytes=0):
        return lib.bdfp4_decode_multi(a, a, a, a, a, a, a, 2, T, H_q, H_kv, 128, 128, 4, 16, 0, 0, ctypes.byref(kv),
                                      0.1, chunk, ws, ws_bytes, a, None, None)
    assert call(T=0) == -1
    assert call(H_q=7) == -2
    # the workspace holds B T_q rows of partials and query images
    n1 = bdfp4.bdfp4_decode_workspace_size(2, 8, 128, 4, 1)
    n2 = bdfp4.bdfp4_decode_workspace_size(2 * 2, 8, 128, 4, 1)
    assert n2 > n1 and call(ws=_p(0x20000), ws_bytes=n1) == -6
    # plan: T_q = 1 is the single-token plan; four query tokens of four heads per KV head stack
    # sixteen rows, planned as sixteen heads per KV head are
    lens = np.full(16, 32768)
    assert bdfp4.bdfp4_decode_multi_plan(lens, 1, 32, 8, 128, 128, 148) == \
        bdfp4.bdfp4_decode_plan_for(lens, 32, 8, 128, 128, 148) == 29
    assert bdfp4.bdfp4_decode_multi_plan(lens, 4, 32, 8, 128, 128, 148) == \
        bdfp4.bdfp4_decode_plan_for(lens, 128, 8, 128, 128, 148)
    with pytest.raises(bdfp4.BDFP4Error):
        bdfp4.bdfp4_decode_multi_plan(lens, 0, 32, 8, 128, 128, 148)


def test_decode_step_and_append_halves_argument_errors(lib):
    kv = bdfp4._KVParams(0x1000, 0x2000, 0x3000)
    a = _p(0x10000)

    def step(k_new=a, v_new=a, v_open=a, H_q=8, H_kv=2, d_k=128, d_v=128):
        return lib.bdfp4_decode_step(a, k_new, v_new, v_open, a, a, a, a, a, a, 2, H_q, H_kv, d_k, d_v, 4, 16, 0, 0,
                                     ctypes.byref(kv), 0.1, 8, None, 0, a, None, None)
    assert step(k_new=None) == -1
    assert step(v_open=None) == -1
    assert step(v_new=_p(0x10002)) == -3
    assert step(H_q=7) == -2
    assert step(d_k=64, d_v=64) == -4
    # the K and V halves of the append
    assert lib.bdfp4_quantize_k(a, a, 10, 2, 64, 0, 0, ctypes.byref(kv), a, a, 4, None, None) == -4
    assert lib.bdfp4_quantize_k(None, a, 10, 2, 128, 0, 0, ctypes.byref(kv), a, a, 4, None, None) == -1
    assert lib.bdfp4_quantize_k(a, a, 0, 2, 128, 0, 0, ctypes.byref(kv), a, a, 4, None, None) == 0
    assert lib.bdfp4_quantize_v(a, a, 10, 2, 64, 0, ctypes.byref(kv), a, a, 4, None) == -4
    assert lib.bdfp4_quantize_v(a, None, 10, 2, 128, 0, ctypes.byref(kv), a, a, 4, None) == -1
    assert lib.bdfp4_quantize_v(a, a, 10, 2, 128, 3, ctypes.byref(kv), a, a, 4, None) == -1


def test_product_code_does_not_touch_the_oracle():
    """The CUDA library and its binding share no code with the oracle."""
    pkg = os.path.join(ROOT, "fp4_kv_cache_quant_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in re.sub(r"#.*|//.*", "", src).lower() or f == "workloads.py", f
    osrc = open(os.path.join(ROOT, "oracle", "bdfp4_oracle.c")).read()
    assert "#include \"" not in osrc


def test_bf16_entry_points_reject_bad_arguments(lib):
    L = bdfp4.load()
    # d other than 128 is outside the compiled set; G = 3 is not a power of two; H_q % H_kv != 0
    assert L.bdfp4_bf16_append(None, None, None, 1, 1, 64, None, None, 1, None, None) == -4
    assert L.bdfp4_bf16_decode(None, None, None, None, None, 1, 3, 1, 128, 1, 1, 1.0, 1, None, 0, None, None,
                               None) == -4
    assert L.bdfp4_bf16_decode(None, None, None, None, None, 1, 4, 3, 128, 1, 1, 1.0, 1, None, 0, None, None,
                               None) == -2
    # null pointers with a supported shape, and negative sizes
    assert L.bdfp4_bf16_decode(None, None, None, None, None, 1, 4, 1, 128, 1, 1, 1.0, 1, None, 0, None, None,
                               None) == -1
    assert L.bdfp4_bf16_append(None, None, None, -1, 1, 128, None, None, 1, None, None) == -1
    assert L.bdfp4_bf16_append(None, None, None, 0, 1, 128, None, None, 1, None, None) == 0


def test_output_comparison_counts_one_bf16_step_as_agreement():
    """The parity comparison: differences of one bf16 step (the two sides
    rounding across a boundary) agree; anything larger counts at full size."""
    from _util import compare_outputs

    assert compare_outputs(np.array([16.0]), np.array([16.125]))[0] == 0.0     # one step at [16, 32)
    assert compare_outputs(np.array([16.0]), np.array([16.25]))[0] == 0.25     # two steps
    assert compare_outputs(np.array([1.0]), np.array([1.0078125]))[0] == 0.0   # one step at [1, 2)
    assert abs(compare_outputs(np.array([0.5]), np.array([0.52]))[0] - 0.02) < 1e-12
    assert compare_outputs(np.array([3.0]), np.array([3.0]))[1] == 0.0
    # the allowance counts among the elements it can apply to (one step above 1e-2)
    assert compare_outputs(np.array([16.0, 0.5, 3.0]), np.array([16.125, 0.5, 3.0]))[2] == 0.5


def test_decode_bound_rejects_a_kernel_a_step_off_on_most_large_outputs():
    """Every element one bf16 step off passes max-abs alone; the bound on the
    allowance's use among large outputs fails it, while a rare straddle passes."""
    from _util import assert_close, bf16_ulp

    rng = np.random.default_rng(0)
    ref = np.concatenate([rng.uniform(2.0, 30.0, 400), rng.uniform(-0.5, 0.5, 4000)])
    ref = (ref.astype(np.float32).view(np.uint32) & 0xFFFF0000).view(np.float32).astype(np.float64)   # bf16 values
    off = ref + np.where(np.abs(ref) >= 2.0, bf16_ulp(ref), 0.0)
    with pytest.raises(AssertionError):
        assert_close(off, ref)
    rare = ref.copy()
    rare[:10] += bf16_ulp(ref[:10])
    assert_close(rare, ref)


def test_decode_plan_minimises_the_documented_wave_cost(lib):
    """On random batches the plan is the split length the header's rule names:
    c in [16, 64] (at most the longest sequence) minimising ceil(CTAs / slots) * (c + 3),
    the longer c on ties."""
    rng = np.random.default_rng(5)
    for _ in range(40):
        B = int(rng.integers(1, 48))
        lens = rng.integers(0, 200_000, size=B)
        H_kv = int(rng.choice([1, 2, 4, 8]))
        sms = int(rng.choice([132, 148]))
        tiles = [(int(n) + 127) // 128 for n in lens]
        got = bdfp4.bdfp4_decode_plan(lens, H_kv, sms)
        mx = max(tiles)
        if mx <= 16:
            assert got == max(mx, 1)
            continue
        cost = {c: -(-H_kv * sum(-(-t // c) for t in tiles) // (4 * sms)) * (c + 3) for c in range(16, min(64, mx) + 1)}
        best = min(cost.values())
        assert cost[got] == best and got == max(c for c, v in cost.items() if v == best)


def test_binding_and_oracle_constants_match_the_header():
    """Every flag and device-status bit of include/bdfp4.h has the same value in
    the binding, and the oracle's flags of the same arms share it (the parity
    tests pass one integer to both sides); the oracle-only flag collides with none."""
    import oracle
    hdr = open(os.path.join(ROOT, "include", "bdfp4.h")).read()
    defs = {m.group(1): int(m.group(2)) for m in re.finditer(r"#define BDFP4_((?:FLAG|DEV)_\w+) (\d+)", hdr)}
    assert {"FLAG_NO_HADAMARD", "FLAG_DYNAMIC_ALPHA", "DEV_TIMEOUT"} <= set(defs)
    for name, val in defs.items():
        assert getattr(bdfp4, name) == val, name
        if name.startswith("FLAG_"):
            assert getattr(oracle, name) == val, name
    assert oracle.FLAG_EXACT_P not in defs.values()
    assert sorted(v for k, v in defs.items() if k.startswith("FLAG_")) == [1, 2, 4, 8, 32]
