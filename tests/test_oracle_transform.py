"""Pins for the oracle's outlier-aware key transform (smoothing + Hadamard)
and its static calibration."""
import math

import numpy as np
import pytest
import scipy.linalg
import torch


@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 64, 128, 256, 512])
def test_fwht_is_sylvester_hadamard(ora, n):
    # columns of the butterfly network applied to unit vectors == scipy's Hadamard
    eye = np.eye(n, dtype=np.float32)
    H = np.stack([ora.fwht_f32(eye[i]) for i in range(n)], axis=1)
    assert np.array_equal(H, scipy.linalg.hadamard(n).astype(np.float32))
    assert np.array_equal(H @ H.T, n * np.eye(n, dtype=np.float32))


def test_fwht_norm_identity(ora):
    rng = np.random.default_rng(0)
    x = rng.standard_normal(128).astype(np.float32)
    y = ora.fwht_f32(x)
    assert abs(np.linalg.norm(y.astype(np.float64)) - math.sqrt(128) * np.linalg.norm(x.astype(np.float64))) < 1e-4


def test_key_transform_unit_vector_closed_form(ora):
    # H e_0 = all ones; keys are post-scaled by 2^-ceil(7/2) = 1/16, queries by 2^-3 = 1/8
    e0 = np.zeros(128, np.float32)
    e0[0] = 1.0
    ones = np.ones(128, np.float32)
    assert np.array_equal(ora.transform(e0, ones, True), np.full(128, 1 / 16, np.float32))
    assert np.array_equal(ora.transform(e0, ones, False), np.full(128, 1 / 8, np.float32))
    # smoothing divides keys and multiplies queries
    s = np.full(128, 4.0, np.float32)
    assert np.array_equal(ora.transform(e0, s, True, hadamard=False), e0 / 4)
    assert np.array_equal(ora.transform(e0, s, False, hadamard=False), e0 * 4)


@pytest.mark.parametrize("d", [128, 576])
def test_transform_preserves_dot_products(ora, d):
    rng = np.random.default_rng(d)
    q = rng.standard_normal((8, d)).astype(np.float32)
    k = rng.standard_normal((8, d)).astype(np.float32)
    s = (2.0 ** rng.integers(-4, 5, d)).astype(np.float32)
    qt = ora.transform(q, s, False)
    kt = ora.transform(k, s, True)
    ref = q.astype(np.float64) @ k.astype(np.float64).T
    got = qt.astype(np.float64) @ kt.astype(np.float64).T
    # fp32 butterflies: about log2(d) roundings of 2^-24 per output, so the
    # dot product is exact up to ~1e-5 of |q s| |k / s|
    bound = 1e-5 * np.linalg.norm(q * s, axis=1)[:, None] * np.linalg.norm(k / s, axis=1)[None, :]
    assert np.all(np.abs(got - ref) <= bound)
    assert not np.allclose(kt, k / s)   # the rotation did something


def test_mla_transform_segments_are_independent(ora):
    # d = 576 rotates [0, 512) with H512 and [512, 576) with H64, separately
    x = np.zeros(576, np.float32)
    x[512] = 1.0
    y = ora.transform(x, np.ones(576, np.float32), True)
    assert np.all(y[:512] == 0)
    assert np.array_equal(y[512:], np.full(64, 1 / 8, np.float32))   # 2^-ceil(6/2)
    x = np.zeros(576, np.float32)
    x[3] = 1.0
    y = ora.transform(x, np.ones(576, np.float32), True)
    assert np.all(y[512:] == 0) and np.all(np.abs(y[:512]) == 1 / 32)   # 2^-ceil(9/2)


def _bf16(a):
    return torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16)


def test_calibration_smoothing_exponent_closed_form(ora):
    # channel c: kmax / qmax = r_c; expected n = round-half-up(log2(r) / 2)
    ratios = [1.0, 2.0, 4.0, 8.0, 12.0, 1.4, 2.9, 0.3, 0.25, 0.5, 2 ** 10, 2 ** -9, 3.0, 0.7]
    d = 128
    kc = np.zeros((4, 1, d), np.float32)
    qc = np.ones((2, 1, d), np.float32) * 0.01
    expect = np.zeros(d)
    for c, r in enumerate(ratios):
        kmax = float(torch.tensor(r).to(torch.bfloat16))   # representable in bf16
        kc[1, 0, c] = -kmax
        qc[0, 0, c] = 1.0
        rr = kmax / 1.0
        expect[c] = math.floor(0.5 * math.log2(rr) + 0.5)
    for c in range(len(ratios), d):
        kc[0, 0, c] = 1.0
        qc[1, 0, c] = 1.0
    vc = np.ones((4, 1, d), np.float32)
    smooth, kg, vg = ora.calibrate(_bf16(kc), _bf16(qc), _bf16(vc), H_q=1, H_kv=1)
    got = np.log2(smooth[0])
    assert np.array_equal(got[: len(ratios)], expect[: len(ratios)])
    assert np.all(got[len(ratios):] == 0)
    assert vg[0] == np.float32(1.0) / np.float32(2688.0)


def test_calibration_tensor_scale_puts_max_block_at_448(ora):
    rng = np.random.default_rng(3)
    kc = rng.standard_normal((64, 2, 128)).astype(np.float32)
    kc[:, :, 5] *= 25.0
    qc = rng.standard_normal((8, 4, 128)).astype(np.float32)
    vc = rng.standard_normal((64, 2, 128)).astype(np.float32)
    smooth, kg, vg = ora.calibrate(_bf16(kc), _bf16(qc), _bf16(vc), H_q=4, H_kv=2)
    assert set(np.unique(np.log2(smooth))).issubset(set(range(-20, 21)))
    for h in range(2):
        kt = ora.transform(_bf16(kc)[:, h].float().numpy(), smooth[h], True)
        amax = np.abs(kt).max()
        assert kg[h] == np.float32(amax) / np.float32(2688.0)
        # the block holding the calibration maximum gets the largest E4M3 code
        assert ora.plain_scale_code(ora.NVFP4, float(amax), float(kg[h])) == 0x7E
        # the query group of KV head h is heads 2h, 2h+1 (contiguous grouping)
    # smoothing balances the channel ranges of keys and queries (within a factor 2)
    kq = np.abs(_bf16(kc).float().numpy()).max(0)[0] / smooth[0]
    qq = np.abs(_bf16(qc).float().numpy())[:, 0:2].max((0, 1)) * smooth[0]
    assert np.all(np.maximum(kq / qq, qq / kq) <= 2.0 + 1e-6)
