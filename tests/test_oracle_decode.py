"""Pins for the oracle's paged decode attention: textbook attention on
FP4-exact inputs, split/merge invariance, and closed forms of the fused
probability quantization with and without underflow-aware scaling."""
import math

import numpy as np
import pytest
import torch

E2M1_POS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _exact_fp4(rng, shape_blocks, beta, axis_len):
    """Values that NVFP4 represents exactly with a unit tensor scale: every
    beta-block along the last axis holds one +-6*2^j and E2M1 points * 2^j."""
    vals = rng.choice(E2M1_POS, size=shape_blocks + (axis_len,)) * rng.choice([-1, 1], size=shape_blocks + (axis_len,))
    nb = axis_len // beta
    j = rng.integers(-3, 3, size=shape_blocks + (nb,))
    pos = rng.integers(0, beta, size=shape_blocks + (nb,))
    for idx in np.ndindex(*shape_blocks, nb):
        blk = idx[-1]
        vals[idx[:-1] + (blk * beta + pos[idx],)] = 6.0 * rng.choice([-1, 1])
    scale = np.repeat(2.0 ** j, beta, axis=-1)
    return (vals * scale).astype(np.float32)


def _bf16(a):
    return torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16)


def _pages(seq_lens, rng):
    npages = [(n + 63) // 64 for n in seq_lens]
    num_pages = max(1, sum(npages))
    perm = rng.permutation(num_pages)
    maxp = max(1, max(npages))
    bt = np.zeros((len(seq_lens), maxp), np.int32)
    off = 0
    slots = []
    for b, n in enumerate(seq_lens):
        bt[b, : npages[b]] = perm[off: off + npages[b]]
        off += npages[b]
        t = np.arange(n)
        slots.append(bt[b, t // 64].astype(np.int64) * 64 + t % 64)
    return bt, num_pages, np.concatenate(slots) if slots else np.zeros(0, np.int64)


def _exact_case(rng, seq_lens, H_q, H_kv, d, fmt=0, d_v=None):
    """q [B, H_q, d], k [T, H_kv, d] and v [T, H_kv, d_v] (d_v = d unless given)
    that the format represents exactly with unit tensor scales."""
    beta = 16 if fmt == 0 else 32
    d_k, d = d, (d if d_v is None else d_v)
    T = int(sum(seq_lens))
    k = _exact_fp4(rng, (T, H_kv), beta, d_k)
    # V blocks run along tokens: build per (head, channel) along the token axis,
    # block-aligned per sequence (pages start at token 0 of each sequence)
    v = np.zeros((T, H_kv, d), np.float32)
    off = 0
    for n in seq_lens:
        npad = ((n + beta - 1) // beta) * beta
        if npad:
            vv = _exact_fp4(rng, (H_kv, d), beta, npad)        # [H_kv, d, npad]
            if n % beta:
                # the last block is partial: move its +-6*2^j onto a valid token
                last = npad - beta
                blk = vv[:, :, last:]
                big = np.argmax(np.abs(blk), axis=-1)
                for h in range(H_kv):
                    for c in range(d):
                        val = blk[h, c, big[h, c]]
                        blk[h, c, big[h, c]] = blk[h, c, 0]
                        blk[h, c, 0] = val
            v[off: off + n] = np.transpose(vv, (2, 0, 1))[:n]
        off += n
    q = _exact_fp4(rng, (len(seq_lens), H_q), beta, d_k)
    return q, k, v


@pytest.mark.parametrize("G,seq_lens", [(4, [1000]), (8, [129, 0, 77, 513]), (1, [64, 300])])
def test_exact_inputs_match_textbook_attention(ora, G, seq_lens):
    rng = np.random.default_rng(G)
    H_kv, d = 2, 128
    H_q = G * H_kv
    q, k, v = _exact_case(rng, seq_lens, H_q, H_kv, d)
    bt, num_pages, sm = _pages(seq_lens, rng)
    ones = np.ones((H_kv, d), np.float32)
    g = np.ones(H_kv, np.float32)
    cache = ora.empty_cache(num_pages, H_kv, d, d, ora.NVFP4)
    fl = ora.FLAG_NO_HADAMARD
    ora.quantize_kv(_bf16(k), _bf16(v), sm, cache, H_kv, ora.NVFP4, ones, g, g, num_pages, flags=fl)
    # the cache holds the inputs exactly
    t = 0
    for b, n in enumerate(seq_lens):
        for i in range(0, n, 37):
            page, slot = bt[b, i // 64], i % 64
            for h in range(H_kv):
                assert np.array_equal(ora.dequant_key_row(cache, 0, page, h, H_kv, d, slot), k[t + i, h])
                assert np.array_equal(ora.dequant_value_row(cache, 0, page, h, H_kv, d, slot), v[t + i, h])
        t += n
    sm_scale = 1 / math.sqrt(d) / 8
    cu = np.concatenate([[0], np.cumsum(seq_lens)])
    ref = ora.attention_ref(_bf16(q), _bf16(k), _bf16(v), cu, H_kv, sm_scale)
    outs = []
    for chunk in (1, 2, 1000):
        o16, o64 = ora.decode(_bf16(q), cache, bt, np.array(seq_lens), H_kv, d, ora.NVFP4, ones, g, g,
                              sm_scale, chunk, num_pages, flags=fl | ora.FLAG_EXACT_P)
        scale = np.abs(ref).max() + 1e-30
        assert np.max(np.abs(o64 - ref)) <= 1e-6 * scale, chunk
        outs.append(o64)
    # splits do not change the (unquantized-P) result
    assert np.allclose(outs[0], outs[2], rtol=0, atol=1e-12 * (np.abs(ref).max() + 1e-30))
    # empty sequence -> zeros
    for b, n in enumerate(seq_lens):
        if n == 0:
            assert np.all(outs[0][b] == 0)


@pytest.mark.parametrize("fmt", [0, 1])
def test_exact_inputs_match_textbook_attention_latent_geometry(ora, fmt):
    """The MLA geometry: keys of d_k = 576 (512 latent + 64 rope channels), values of
    d_v = 512, sixteen query heads over one KV head.  An index slip between d_k and
    d_v (key rows, value rows, their scale bytes) breaks the equality."""
    rng = np.random.default_rng(576 + fmt)
    seq_lens = [130, 0, 300]
    H_kv, H_q, d_k, d_v = 1, 16, 576, 512
    q, k, v = _exact_case(rng, seq_lens, H_q, H_kv, d_k, fmt, d_v=d_v)
    bt, num_pages, sm = _pages(seq_lens, rng)
    ones = np.ones((H_kv, d_k), np.float32)
    g = np.ones(H_kv, np.float32)
    cache = ora.empty_cache(num_pages, H_kv, d_k, d_v, fmt)
    fl = ora.FLAG_NO_HADAMARD
    ora.quantize_kv(_bf16(k), _bf16(v), sm, cache, H_kv, fmt, ones, g, g, num_pages, flags=fl)
    t = 0
    for b, n in enumerate(seq_lens):
        for i in range(0, n, 29):
            page, slot = bt[b, i // 64], i % 64
            assert np.array_equal(ora.dequant_key_row(cache, fmt, page, 0, H_kv, d_k, slot), k[t + i, 0])
            assert np.array_equal(ora.dequant_value_row(cache, fmt, page, 0, H_kv, d_v, slot), v[t + i, 0])
        t += n
    sm_scale = 1 / math.sqrt(d_k) / 8
    cu = np.concatenate([[0], np.cumsum(seq_lens)])
    ref = ora.attention_ref(_bf16(q), _bf16(k), _bf16(v), cu, H_kv, sm_scale)
    assert ref.shape == (len(seq_lens), H_q, d_v)
    for chunk in (1, 1000):
        _, o64 = ora.decode(_bf16(q), cache, bt, np.array(seq_lens), H_kv, d_v, fmt, ones, g, g, sm_scale, chunk,
                            num_pages, flags=fl | ora.FLAG_EXACT_P)
        assert np.max(np.abs(o64 - ref)) <= 1e-6 * (np.abs(ref).max() + 1e-30), chunk
        assert np.all(o64[1] == 0)


def _uniform_case(ora, fmt, flags):
    rng = np.random.default_rng(42)
    H_kv, G, d, N = 1, 4, 128, 300
    q = np.zeros((1, G, d), np.float32)
    _, k, v = _exact_case(rng, [N], G, H_kv, d, fmt)
    bt, num_pages, sm = _pages([N], rng)
    ones = np.ones((H_kv, d), np.float32)
    g = np.ones(H_kv, np.float32)
    cache = ora.empty_cache(num_pages, H_kv, d, d, fmt)
    ora.quantize_kv(_bf16(k), _bf16(v), sm, cache, H_kv, fmt, ones, g, g, num_pages, flags=ora.FLAG_NO_HADAMARD)
    o16, o64 = ora.decode(_bf16(q), cache, bt, np.array([N]), H_kv, d, fmt, ones, g, g, 0.1, 1, num_pages,
                          flags=ora.FLAG_NO_HADAMARD | flags)
    return o64, v


@pytest.mark.parametrize("fmt,flags,pscale", [
    (0, 0, 1.03125),                      # p = 1 -> E4M3(2048/6)=352, E2M1(5.82)=6 -> 6*352/2048
    (0, 8, 1.03125),                      # vanilla: E4M3(1/6)=0.171875 -> 6*0.171875
    (1, 0, 1.0),                          # MXFP4: X = 2^-2, 1/X = 4 exactly
])
def test_uniform_logits_closed_form(ora, fmt, flags, pscale):
    # q = 0 -> every logit is 0 -> p = 1 for every token; l counts tokens
    o64, v = _uniform_case(ora, fmt, flags)
    expect = pscale * v[:, 0].astype(np.float64).mean(0)
    for h in range(4):
        assert np.allclose(o64[0, h], expect, rtol=1e-12, atol=1e-12)


def _sink_case(ora, fmt, flags, N=300, chunk=1000, logit=10.0):
    """One key with logit 10 (or `logit`), the rest 0: p = 1 and e^-10 per token."""
    rng = np.random.default_rng(7)
    H_kv, G, d = 1, 2, 128
    q = np.zeros((1, G, d), np.float32)
    q[0, :, 0] = 6.0
    k = np.zeros((N, H_kv, d), np.float32)
    k[0, 0, 0] = 6.0
    _, _, v = _exact_case(rng, [N], G, H_kv, d, fmt)
    bt, num_pages, sm = _pages([N], rng)
    ones = np.ones((H_kv, d), np.float32)
    g = np.ones(H_kv, np.float32)
    cache = ora.empty_cache(num_pages, H_kv, d, d, fmt)
    ora.quantize_kv(_bf16(k), _bf16(v), sm, cache, H_kv, fmt, ones, g, g, num_pages, flags=ora.FLAG_NO_HADAMARD)
    o16, o64 = ora.decode(_bf16(q), cache, bt, np.array([N]), H_kv, d, fmt, ones, g, g, logit / 36.0, chunk,
                          num_pages, flags=ora.FLAG_NO_HADAMARD | flags)
    return o64, v[:, 0].astype(np.float64)


def test_underflow_aware_scaling_closed_form(ora):
    N = 300
    l = 1.0 + (N - 1) * math.exp(-10.0)
    # alpha = 2^11: tiny blocks get E4M3 scale 2^-6 and code 6 -> 6 * 2^-6 / 2048
    o, v = _sink_case(ora, 0, 0, N)
    tail = 6 * 2.0 ** -6 / 2048
    expect = (1.03125 * v[0] + tail * v[16:].sum(0)) / l
    assert np.allclose(o[0, 0], expect, rtol=1e-5, atol=1e-9)
    # vanilla alpha = 1: every block without the sink collapses (E4M3(e^-10/6) = 0)
    o, v = _sink_case(ora, 0, ora.FLAG_NO_UNDERFLOW, N)
    assert np.allclose(o[0, 0], 1.03125 * v[0] / l, rtol=1e-5, atol=1e-9)
    # MXFP4: E8M0 scale 2^-17 keeps the tail, block of the sink is 32 tokens
    o, v = _sink_case(ora, 1, 0, N)
    expect = (1.0 * v[0] + 6 * 2.0 ** -17 * v[32:].sum(0)) / l
    assert np.allclose(o[0, 0], expect, rtol=1e-5, atol=1e-9)


def test_split_kv_quantizes_probabilities_per_split(ora):
    """With one tile per split, the tiles after the sink's tile run their own
    softmax (their max is 0, so p = 1 and P^ = 1.03125 p) and the merge
    weights them by e^(0 - 10); l stays the unquantized sum."""
    N = 300
    l = 1.0 + (N - 1) * math.exp(-10.0)
    o, v = _sink_case(ora, 0, 0, N, chunk=1)
    tail = 6 * 2.0 ** -6 / 2048
    expect = (1.03125 * v[0] + tail * v[16:128].sum(0) + 1.03125 * math.exp(-10.0) * v[128:].sum(0)) / l
    assert np.allclose(o[0, 0], expect, rtol=1e-5, atol=1e-9)


@pytest.mark.parametrize("p_max,E", [
    (1.0, 11),                                    # 2688 / 1 = 2^11.39: the static alpha
    (2688.0 * 2.0 ** -20, 20),                    # p_max 2^20 = 2688 exactly: still allowed
    (np.nextafter(2688.0 * 2.0 ** -20, 1.0), 19),  # one ulp above: 2^20 p_max > 2688
    (2.0 ** -20, 31),                             # 2^-20 2^31 = 2048 <= 2688 < 4096
    (math.exp(-10.0), 25),                        # 2^25 e^-10 = 1523.3, 2^26 e^-10 = 3046.6
    (math.exp(-20.0), 40),                        # 2^40 e^-20 = 2266.3, 2^41 e^-20 = 4532.6
    (2.0 ** -100, 64),                            # clamped
    (0.0, 64),                                    # empty tile
])
def test_dynamic_alpha_exponent_hand_values(ora, p_max, E):
    assert ora.dynamic_alpha_exp(p_max) == E


def test_dynamic_alpha_closed_form(ora):
    """Sink logit 20: with alpha = 2^11 every block without the sink collapses
    (E4M3(e^-20 2^11 / 6) = 0).  The dynamic variant keeps alpha = 2^11 on the
    sink's tile (p_max = 1) but takes 2^40 on the two later tiles, whose p_max
    is e^-20: E4M3(e^-20 2^40 / 6 = 377.7) = 384, E2M1(2266.3 / 384 = 5.90) = 6,
    so each of their tokens gets P^ = 6 x 384 / 2^40."""
    N = 300
    l = 1.0 + (N - 1) * math.exp(-20.0)
    o_st, v = _sink_case(ora, 0, 0, N, logit=20.0)
    assert np.allclose(o_st[0, 0], 1.03125 * v[0] / l, rtol=1e-12, atol=1e-15)
    o_dy, _ = _sink_case(ora, 0, ora.FLAG_DYNAMIC_ALPHA, N, logit=20.0)
    tail = 6 * 384 * 2.0 ** -40 * v[128:].sum(0) / l
    assert np.abs(tail).max() > 1e-9
    # (the difference of two outputs of size ~10 carries ~1e-15 of cancellation)
    assert np.allclose(o_dy[0, 0] - o_st[0, 0], tail, rtol=1e-9, atol=1e-13)
    # unquantized P carries the tail as e^-20 per token (the sink's logit holds
    # the fp32 rounding of g_q, so e^-20 only to ~1e-7, and l with it)
    o_ex, _ = _sink_case(ora, 0, ora.FLAG_EXACT_P, N, logit=20.0)
    exact_tail = (o_ex[0, 0] - v[0] / l)
    assert np.allclose(exact_tail, math.exp(-20.0) * v[1:].sum(0) / l, rtol=1e-5, atol=1e-10)


def test_dynamic_alpha_reduces_to_static_alpha(ora):
    """Every split's first tile has p_max = 1 (alpha = 2^11): with one tile per
    split the variant is the static method; MXFP4 has no alpha to choose."""
    for logit in (10.0, 20.0):
        o_st, _ = _sink_case(ora, 0, 0, 300, chunk=1, logit=logit)
        o_dy, _ = _sink_case(ora, 0, ora.FLAG_DYNAMIC_ALPHA, 300, chunk=1, logit=logit)
        assert np.array_equal(o_st, o_dy)
        o_st, _ = _sink_case(ora, 1, 0, 300, logit=logit)
        o_dy, _ = _sink_case(ora, 1, ora.FLAG_DYNAMIC_ALPHA, 300, logit=logit)
        assert np.array_equal(o_st, o_dy)
    # the variant and the vanilla ablation exclude each other
    with pytest.raises(AssertionError):
        _sink_case(ora, 0, ora.FLAG_DYNAMIC_ALPHA | ora.FLAG_NO_UNDERFLOW, 300)


def test_quantized_probabilities_stay_close_on_random_data(ora):
    """With FP4 P the output stays within a few percent of the exact-P output
    (a sanity bound, not a pin of any constant)."""
    rng = np.random.default_rng(9)
    H_kv, G, d, N = 1, 4, 128, 700
    q, k, v = _exact_case(rng, [N], G, H_kv, d)
    q = q / 4
    bt, num_pages, sm = _pages([N], rng)
    ones = np.ones((H_kv, d), np.float32)
    g = np.ones(H_kv, np.float32)
    cache = ora.empty_cache(num_pages, H_kv, d, d, 0)
    ora.quantize_kv(_bf16(k), _bf16(v), sm, cache, H_kv, 0, ones, g, g, num_pages, flags=ora.FLAG_NO_HADAMARD)
    args = (_bf16(q), cache, bt, np.array([N]), H_kv, d, 0, ones, g, g, 0.05, 2, num_pages)
    _, exact = ora.decode(*args, flags=ora.FLAG_NO_HADAMARD | ora.FLAG_EXACT_P)
    _, quant = ora.decode(*args, flags=ora.FLAG_NO_HADAMARD)
    rel = np.linalg.norm(quant - exact) / np.linalg.norm(exact)
    assert 0 < rel < 0.1


@pytest.mark.parametrize("T_q,seq_lens", [(4, [300, 4, 129]), (1, [77, 200]), (16, [1000])])
def test_multi_token_queries_match_causal_textbook_attention(ora, T_q, seq_lens):
    """Multi-token queries on FP4-exact inputs with unquantized P equal causal
    fp64 attention written out in numpy (query token i of a sequence of N sees
    keys 0 .. N - T_q + i); with T_q = 1 the call is the single-token decode."""
    rng = np.random.default_rng(40 + T_q)
    H_kv, G, d = 2, 4, 128
    H_q = G * H_kv
    _, k, v = _exact_case(rng, seq_lens, H_q, H_kv, d)
    q = _exact_fp4(rng, (len(seq_lens), T_q, H_q), 16, d)
    bt, num_pages, sm = _pages(seq_lens, rng)
    ones = np.ones((H_kv, d), np.float32)
    g = np.ones(H_kv, np.float32)
    cache = ora.empty_cache(num_pages, H_kv, d, d, ora.NVFP4)
    fl = ora.FLAG_NO_HADAMARD
    ora.quantize_kv(_bf16(k), _bf16(v), sm, cache, H_kv, ora.NVFP4, ones, g, g, num_pages, flags=fl)
    sm_scale = 1 / math.sqrt(d) / 8
    qf = _bf16(q).float().numpy().astype(np.float64)
    kf, vf = k.astype(np.float64), v.astype(np.float64)
    for chunk in (1, 3):
        _, o64 = ora.decode_multi(_bf16(q), cache, bt, np.array(seq_lens), H_kv, d, ora.NVFP4, ones, g, g,
                                  sm_scale, chunk, num_pages, flags=fl | ora.FLAG_EXACT_P)
        off = 0
        for b, n in enumerate(seq_lens):
            for i in range(T_q):
                vis = n - T_q + 1 + i
                for h in range(H_q):
                    s = kf[off:off + vis, h // G] @ qf[b, i, h] * sm_scale
                    p = np.exp(s - s.max())
                    ref = p @ vf[off:off + vis, h // G] / p.sum()
                    assert np.allclose(o64[b, i, h], ref, rtol=0, atol=1e-6 * (np.abs(ref).max() + 1e-30))
            off += n
    with pytest.raises(ValueError):   # a sequence shorter than its query tokens
        ora.decode_multi(_bf16(q), cache, bt, np.full(len(seq_lens), T_q - 1), H_kv, d, ora.NVFP4, ones, g, g,
                         sm_scale, 1, num_pages, flags=fl)
    if T_q == 1:
        o16m, _ = ora.decode_multi(_bf16(q), cache, bt, np.array(seq_lens), H_kv, d, ora.NVFP4, ones, g, g,
                                   sm_scale, 2, num_pages, flags=fl)
        o16, _ = ora.decode(_bf16(q[:, 0]), cache, bt, np.array(seq_lens), H_kv, d, ora.NVFP4, ones, g, g,
                            sm_scale, 2, num_pages, flags=fl)
        assert np.array_equal(o16m[:, 0], o16)


def test_kernel_exponent_bit_rule_equals_the_definition(ora):
    """The decode kernels decide the per-tile exponent from p_max's fp32 bits
    (p_max = m 2^e: E = 11 - e, less one when m > 1.3125, i.e. mantissa bits above
    0x280000; clamped to [11, 64]; 64 for zero or subnormal p_max).  That rule,
    written out here from its statement, equals the oracle's fp64 definition
    for every fp32 exponent at the mantissas around the threshold."""
    def bit_rule(p32):
        u = int(np.float32(p32).view(np.uint32))
        eb = (u >> 23) & 0xFF
        if p32 <= 0 or eb == 0:
            return 64
        E = 11 - (eb - 127) - (1 if (u & 0x7FFFFF) > 0x280000 else 0)
        return min(max(E, 11), 64)
    rng = np.random.default_rng(3)
    mants = [0, 1, 0x27FFFF, 0x280000, 0x280001, 0x400000, 0x7FFFFF] + list(rng.integers(0, 1 << 23, 8))
    for eb in range(1, 128):          # p_max in [2^-126, 2^0]: every normal fp32 up to 1
        for mt in mants:
            if eb == 127 and mt:
                continue              # p_max never exceeds 1
            p = np.array([(eb << 23) | int(mt)], np.uint32).view(np.float32)[0]
            assert bit_rule(p) == ora.dynamic_alpha_exp(float(p)), (eb, hex(int(mt)))
    for p in (0.0, 1e-45, 1e-40):     # zero and subnormals
        assert bit_rule(np.float32(p)) == ora.dynamic_alpha_exp(float(np.float32(p))) == 64
