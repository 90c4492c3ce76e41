"""Pins for the oracle's KV-append quantizer, scale search, cache layout and
dual-residual query quantization."""
import ml_dtypes
import numpy as np
import pytest
import torch

E4M3_POS = np.arange(0x7F)


def _np_block(x, sigma):
    """Independent re-derivation with ml_dtypes: codes of fp32(x / sigma) and the
    fp64 squared error, summed left to right."""
    x = np.asarray(x, np.float32)
    if sigma == 0:
        vals = np.zeros_like(x, dtype=np.float64)
    else:
        vals = (x / np.float32(sigma)).astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
    err = 0.0
    for i in range(x.shape[0]):
        d = float(x[i]) - vals[i] * float(sigma)
        err = err + d * d
    return err


def _sigma(fmt, code, g):
    if fmt == 0:
        return np.float32(float(torch.tensor([code], dtype=torch.uint8).view(torch.float8_e4m3fn).float())) * np.float32(g)
    return np.float32(2.0 ** (code - 127))


@pytest.mark.parametrize("fmt", [0, 1])
def test_scale_search_window_against_brute_force(ora, fmt):
    rng = np.random.default_rng(10 + fmt)
    n = 16 if fmt == 0 else 32
    g = np.float32(0.0123) if fmt == 0 else np.float32(1.0)
    hits = trials = 0
    for trial in range(300):
        x = (rng.standard_normal(n) * rng.choice([1.0, 0.3, 3.0])).astype(np.float32)
        if trial % 3 == 0:
            x[rng.integers(n)] *= 8.0   # an outlier in the block
        code = ora.search_scale_code(fmt, x, float(g))
        c0 = ora.plain_scale_code(fmt, float(np.abs(x).max()), float(g))
        if fmt == 0:
            window = [c for c in range(c0 + 7, c0 - 3, -1) if 0 <= c <= 126]
            full = list(range(0, 127))
        else:
            window = [c for c in (c0 + 1, c0) if 0 <= c <= 254]
            full = list(range(max(0, c0 - 10), min(254, c0 + 10) + 1))
        errs = {c: _np_block(x, _sigma(fmt, c, g)) for c in set(window) | set(full)}
        best_w = min(window, key=lambda c: (errs[c], -c))
        assert code == best_w, (trial, code, best_w)
        # never worse than the plain rule (c0 is a candidate)
        assert errs[code] <= errs[c0]
        # the oracle's own error matches the independent derivation
        _, e_or = ora.quantize_block(x, float(_sigma(fmt, code, g)))
        assert e_or == errs[code]
        trials += 1
        hits += errs[code] == min(errs.values())
    # the window almost always contains the global optimum (a report, loosely bounded)
    assert hits / trials >= 0.99


def test_scale_search_all_zero_block(ora):
    assert ora.search_scale_code(0, np.zeros(16, np.float32), 0.5) == 0
    assert ora.search_scale_code(1, np.zeros(32, np.float32), 1.0) == 0


def _bf16(a):
    return torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16)


def test_cache_layout_golden_offsets(ora):
    """One token with a single non-zero channel lands where the layout
    definition says (offsets worked out by hand from it):
    K nibble byte = ((page*H_kv+head)*64*d/2) + (slot/8)*(d/32)*128 + (e/32)*128 + (slot%8)*16 + (e%32)/2
    K scale byte  = ((page*H_kv+head)*256*ceil(d/64)) + (blk/4)*256 + (slot%32)*8 + (slot/32)*4 + blk%4
    V nibble byte = ((page*H_kv+head)*d*32) + (c/8)*256 + (slot/32)*128 + (c%8)*16 + (slot%32)/2
    V scale byte  = ((page*H_kv+head)*d*4) + (c/128)*512 + (c%32)*16 + ((c%128)/32)*4 + slot/16
    page 2, head 1 of 2, slot 37, channel 77, value 6.0, d = 128, NVFP4, g = 1, plain scale rule."""
    H_kv, d, num_pages = 2, 128, 3
    k = np.zeros((1, H_kv, d), np.float32)
    v = np.zeros((1, H_kv, d), np.float32)
    k[0, 1, 77] = 6.0
    v[0, 1, 77] = 6.0
    cache = ora.empty_cache(num_pages, H_kv, d, d, ora.NVFP4)
    ones = np.ones((H_kv, d), np.float32)
    g = np.ones(H_kv, np.float32)
    ora.quantize_kv(_bf16(k), _bf16(v), np.array([2 * 64 + 37]), cache, H_kv, ora.NVFP4, ones, g, g,
                    num_pages, flags=ora.FLAG_NO_HADAMARD | ora.FLAG_NO_SCALE_SEARCH)
    nz = {name: [(int(i), int(cache[name][i])) for i in np.nonzero(cache[name])[0]] for name in cache}
    # hand-computed: 20480 + 4*4*128 + 2*128 + 5*16 + 6 = 22870, odd element -> high nibble of E2M1(6)=7
    assert nz["k_pages"] == [(22870, 0x70)]
    # 5*512 + 1*256 + 5*8 + 1*4 + 0 = 2860, E4M3(1.0) = 0x38
    assert nz["k_scales"] == [(2860, 0x38)]
    # 20480 + 9*256 + 1*128 + 5*16 + 2 = 22994, odd slot -> high nibble
    assert nz["v_pages"] == [(22994, 0x70)]
    # 2560 + 0 + 13*16 + 2*4 + 2 = 2778
    assert nz["v_scales"] == [(2778, 0x38)]


def test_v_blocks_from_runs_and_zero_fill(ora):
    """V blocks run along 16 slots; slots of a block outside this call's run
    are zero, and a run that starts mid-block still re-quantizes the block."""
    H_kv, d = 1, 128
    rng = np.random.default_rng(4)
    v = rng.standard_normal((20, H_kv, d)).astype(np.float32)
    k = rng.standard_normal((20, H_kv, d)).astype(np.float32)
    ones = np.ones((H_kv, d), np.float32)
    g = np.full(H_kv, 0.01, np.float32)
    # tokens -> slots 5..24 of page 0: block 0 gets slots 5..15 (0..4 zero), block 1 gets 16..24
    sm = np.arange(5, 25)
    cache = ora.empty_cache(1, H_kv, d, d, ora.NVFP4)
    ora.quantize_kv(_bf16(k), _bf16(v), sm, cache, H_kv, ora.NVFP4, ones, g, g, 1)
    vb = _bf16(v).float().numpy()
    for slot in range(0, 32):
        row = ora.dequant_value_row(cache, ora.NVFP4, 0, 0, H_kv, d, slot) * g[0]
        if slot < 5 or slot >= 25:
            assert np.all(row == 0), slot
        else:
            ref = vb[slot - 5, 0]
            assert np.max(np.abs(row - ref)) <= 0.5 * np.abs(vb).max() / 4 + 1e-6


def test_key_quantization_error_bound_and_search_gain(ora):
    """Dequantized keys lie within the E2M1 grid error of their block scale,
    and the search lowers the total squared error vs the plain rule."""
    rng = np.random.default_rng(5)
    H_kv, d, T = 1, 128, 64
    k = rng.standard_normal((T, H_kv, d)).astype(np.float32)
    k[:, :, [3, 70]] *= 20
    v = rng.standard_normal((T, H_kv, d)).astype(np.float32)
    ones = np.ones((H_kv, d), np.float32)
    kb = _bf16(k)
    xt = ora.transform(kb.float().numpy()[:, 0], ones[0], True)
    g = np.array([np.abs(xt).max() / 2688], np.float32)
    errs = {}
    for flags in (0, ora.FLAG_NO_SCALE_SEARCH):
        cache = ora.empty_cache(1, H_kv, d, d, ora.NVFP4)
        ora.quantize_kv(kb, _bf16(v), np.arange(T), cache, H_kv, ora.NVFP4, ones, g, g, 1, flags=flags)
        tot = 0.0
        for t in range(T):
            deq = ora.dequant_key_row(cache, ora.NVFP4, 0, 0, H_kv, d, t) * g[0]
            tot += float(((deq - xt[t]) ** 2).sum())
            blk_amax = np.abs(xt[t]).reshape(-1, 16).max(1)
            # |error| <= max(E2M1 half-step at the top, saturation) * scale; loose bound: amax/3 + tiny
            assert np.all(np.abs(deq - xt[t]).reshape(-1, 16).max(1) <= blk_amax / 3 + 1e-6)
        errs[flags] = tot
    assert errs[0] < errs[ora.FLAG_NO_SCALE_SEARCH]


@pytest.mark.parametrize("fmt", [0, 1])
def test_dual_residual_never_worse_elementwise(ora, fmt):
    rng = np.random.default_rng(6 + fmt)
    B, H_q, H_kv, d = 2, 8, 2, 128
    q = rng.standard_normal((B, H_q, d)).astype(np.float32)
    q[:, :, 9] *= 15
    smooth = (2.0 ** rng.integers(-2, 3, (H_kv, d))).astype(np.float32)
    out = ora.quantize_q(_bf16(q), H_kv, fmt, smooth)
    single = ora.quantize_q(_bf16(q), H_kv, fmt, smooth, flags=ora.FLAG_SINGLE_QUERY)
    beta = ora.beta(fmt)
    e2m1 = np.array([ora.e2m1_value(c) for c in range(16)])

    def deq(codes, scales, gq):
        sc = np.array([ora.e4m3_value(c) if fmt == 0 else ora.e8m0_value(c) for c in scales.ravel()])
        sc = sc.reshape(scales.shape).repeat(beta, axis=-1)
        return e2m1[codes] * sc * gq[..., None]

    x = out["xq"].astype(np.float64)
    d1 = deq(out["q1_codes"], out["q1_scales"], out["g_q"])
    d2 = deq(out["q2_codes"], out["q2_scales"], out["g_q"])
    assert np.array_equal(out["q1_codes"], single["q1_codes"])
    assert np.all(single["q2_codes"] == 0)
    assert np.all(np.abs(x - d1 - d2) <= np.abs(x - d1) + 1e-7 * np.abs(x).max())
    # the dual residual cuts the relative query error by more than 5x here
    e1 = np.linalg.norm(x - d1) / np.linalg.norm(x)
    e2 = np.linalg.norm(x - d1 - d2) / np.linalg.norm(x)
    assert e2 < e1 / 5
    if fmt == 0:
        # g_q is the per-head amax / 2688
        assert np.array_equal(out["g_q"], (np.abs(out["xq"]).max(-1) / np.float32(2688)).astype(np.float32))


def _np_block_w(x, sigma, w):
    """_np_block with each squared error weighted (fp64, left to right)."""
    x = np.asarray(x, np.float32)
    if sigma == 0:
        vals = np.zeros_like(x, dtype=np.float64)
    else:
        vals = (x / np.float32(sigma)).astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
    err = 0.0
    for i in range(x.shape[0]):
        d = float(x[i]) - vals[i] * float(sigma)
        err = err + float(np.float32(w[i])) * (d * d)
    return err


@pytest.mark.parametrize("fmt", [0, 1])
def test_weighted_search_against_brute_force(ora, fmt):
    """The attention-aware search keeps the plain search's window and tie rule
    (larger code) and minimises the weighted block error: checked against every
    code of the window, errors re-derived with ml_dtypes."""
    rng = np.random.default_rng(20 + fmt)
    n = 16 if fmt == 0 else 32
    g = np.float32(0.0123) if fmt == 0 else np.float32(1.0)
    changed = 0
    for trial in range(300):
        x = (rng.standard_normal(n) * rng.choice([1.0, 0.3, 3.0])).astype(np.float32)
        if trial % 3 == 0:
            x[rng.integers(n)] *= 8.0
        w = (10.0 ** rng.uniform(-3, 3, n)).astype(np.float32)
        if trial % 5 == 0:
            w[rng.integers(n)] = 0.0
        code = ora.search_scale_code(fmt, x, float(g), w)
        c0 = ora.plain_scale_code(fmt, float(np.abs(x).max()), float(g))
        if fmt == 0:
            window = [c for c in range(c0 + 7, c0 - 3, -1) if 0 <= c <= 126]
        else:
            window = [c for c in (c0 + 1, c0) if 0 <= c <= 254]
        errs = {c: _np_block_w(x, _sigma(fmt, c, g), w) for c in window}
        assert code == min(window, key=lambda c: (errs[c], -c)), trial
        changed += code != ora.search_scale_code(fmt, x, float(g))
    if fmt == 0:
        assert changed > 0   # the weights do move the choice


def test_weighted_search_reductions(ora):
    """Unit weights are the plain objective (bit for bit, through the cache);
    scaling all weights by a power of two changes no choice; one dominant
    weight makes that element's error the first criterion."""
    rng = np.random.default_rng(23)
    for trial in range(200):
        x = (rng.standard_normal(16) * 2).astype(np.float32)
        assert ora.search_scale_code(0, x, 0.01, np.ones(16, np.float32)) == ora.search_scale_code(0, x, 0.01)
        w = rng.uniform(0.1, 10, 16).astype(np.float32)
        assert ora.search_scale_code(0, x, 0.01, w) == ora.search_scale_code(0, x, 0.01, w * np.float32(2.0 ** -7))
        i = int(rng.integers(16))
        wd = np.ones(16, np.float32)
        wd[i] = 1e12
        code = ora.search_scale_code(0, x, 0.01, wd)
        c0 = ora.plain_scale_code(0, float(np.abs(x).max()), 0.01)
        window = [c for c in range(c0 + 7, c0 - 3, -1) if 0 <= c <= 126]

        def elem_err(c):
            s = _sigma(0, c, np.float32(0.01))
            v = float(np.float32(x[i] / s).astype(ml_dtypes.float4_e2m1fn)) if s else 0.0
            return abs(float(x[i]) - v * float(s))
        assert elem_err(code) == min(elem_err(c) for c in window), trial
    # through the cache: unit weights give the same bytes as the plain quantizer
    H_kv, d, T = 2, 128, 40
    k = _bf16(rng.standard_normal((T, H_kv, d)) * 3)
    v = _bf16(rng.standard_normal((T, H_kv, d)))
    ones = np.ones((H_kv, d), np.float32)
    g = np.full(H_kv, 0.004, np.float32)
    a = ora.quantize_kv(k, v, np.arange(T), ora.empty_cache(1, H_kv, d, d, 0), H_kv, 0, ones, g, g, 1)
    b = ora.quantize_kv(k, v, np.arange(T), ora.empty_cache(1, H_kv, d, d, 0), H_kv, 0, ones, g, g, 1,
                        k_weight=ones)
    for name in a:
        assert np.array_equal(a[name], b[name]), name


def test_key_weights_hand_values(ora):
    """Mean square of the transformed calibration queries per channel.  Without
    rotation: q' = q s, so 2 queries with q_0 = 3, 5 and s_0 = 2 give
    w_0 = ((6^2) + (10^2)) / 2 = 68.  With rotation (d = 128, query scale
    2^-3), one query 4 e_0 becomes 4/8 = 0.5 in every channel: w = 0.25."""
    d, H_kv = 128, 1
    q = np.zeros((2, 1, d), np.float32)
    q[0, 0, 0], q[1, 0, 0] = 3.0, 5.0
    q[0, 0, 7] = -1.0
    s = np.ones((H_kv, d), np.float32)
    s[0, 0] = 2.0
    w = ora.key_weights(_bf16(q), 1, H_kv, s, flags=ora.FLAG_NO_HADAMARD)
    expect = np.zeros(d)
    expect[0], expect[7] = 68.0, 0.5
    assert np.array_equal(w[0], expect.astype(np.float32))
    q1 = np.zeros((1, 2, d), np.float32)   # two query heads of one KV head
    q1[0, 0, 0] = 4.0
    q1[0, 1, 0] = 4.0
    w = ora.key_weights(_bf16(q1), 2, 1, np.ones((1, d), np.float32))
    assert np.array_equal(w[0], np.full(d, 0.25, np.float32))


def test_attention_aware_search_lowers_logit_error(ora):
    """With query energy concentrated on a few channels (no rotation, which
    would spread it), weighting the search by it lowers the squared logit error
    q.(k - k^) over fresh queries of the same distribution (a sanity bound)."""
    rng = np.random.default_rng(31)
    H_kv, d, T = 1, 128, 256
    k = rng.standard_normal((T, H_kv, d)).astype(np.float32)
    std = np.where(np.arange(d) % 16 < 2, 8.0, 0.25)
    qc = (rng.standard_normal((512, 1, d)) * std).astype(np.float32)
    qt = (rng.standard_normal((512, d)) * std).astype(np.float32)
    ones = np.ones((H_kv, d), np.float32)
    kb = _bf16(k)
    xt = kb.float().numpy()[:, 0]
    g = np.array([np.abs(xt).max() / 2688], np.float32)
    w = ora.key_weights(_bf16(qc), 1, H_kv, ones, flags=ora.FLAG_NO_HADAMARD)
    errs = {}
    for name, kw in (("plain", None), ("weighted", w)):
        cache = ora.quantize_kv(kb, _bf16(np.zeros_like(k)), np.arange(T), ora.empty_cache(4, H_kv, d, d, 0), H_kv,
                                0, ones, g, g, 4, flags=ora.FLAG_NO_HADAMARD, k_weight=kw)
        deq = np.stack([ora.dequant_key_row(cache, 0, 0, 0, H_kv, d, t) for t in range(64)]) * g[0]
        deq = np.concatenate([deq] + [np.stack([ora.dequant_key_row(cache, 0, p, 0, H_kv, d, t)
                                                for t in range(64)]) * g[0] for p in (1, 2, 3)])
        errs[name] = float((((deq - xt) @ qt.T) ** 2).mean())
    assert errs["weighted"] < 0.9 * errs["plain"], errs
