"""CPU oracle for the FP4 paged decode-attention path -- TEST INFRASTRUCTURE.

This package wraps ``bdfp4_oracle.c`` (a plain, slow, fp64 C restatement of
the BitDecoding-FP4 hot path) with ctypes.  Only the tests, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import it; the
CUDA library never does, and the two share no code.

Arrays are numpy; bf16 tensors travel as their raw uint16 bits.

Parity pins of every function live in ``tests/test_oracle_*.py``; nothing in
this package is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bdfp4_oracle.c")
LIB_PATH = os.path.join(_HERE, "libbdfp4_oracle.so")

NVFP4, MXFP4 = 0, 1
FLAG_NO_HADAMARD = 1
FLAG_NO_SCALE_SEARCH = 2
FLAG_SINGLE_QUERY = 4
FLAG_NO_UNDERFLOW = 8
FLAG_EXACT_P = 16
FLAG_DYNAMIC_ALPHA = 32

PAGE_SLOTS = 64
TILE_TOKENS = 128

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE fp32/fp64, no FMA contraction)."""
    if force or not os.path.exists(LIB_PATH) or os.path.getmtime(LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", "-Wall", "-o", LIB_PATH, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB_PATH)
        d, i, i64, f, p = ctypes.c_double, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p
        L.ora_e2m1_value.restype = d
        L.ora_e2m1_value.argtypes = [i]
        L.ora_e2m1_encode.restype = i
        L.ora_e2m1_encode.argtypes = [d]
        L.ora_e4m3_value.restype = d
        L.ora_e4m3_value.argtypes = [i]
        L.ora_e4m3_encode.restype = i
        L.ora_e4m3_encode.argtypes = [d]
        L.ora_e8m0_value.restype = d
        L.ora_e8m0_value.argtypes = [i]
        L.ora_mx_scale_code.restype = i
        L.ora_mx_scale_code.argtypes = [d]
        L.ora_f64_to_bf16.restype = ctypes.c_uint16
        L.ora_f64_to_bf16.argtypes = [d]
        L.ora_fwht_f32.restype = None
        L.ora_fwht_f32.argtypes = [p, i]
        L.ora_transform.restype = None
        L.ora_transform.argtypes = [p, p, i, i, i, p]
        L.ora_calibrate.restype = i
        L.ora_calibrate.argtypes = [p, p, p, i, i, i, i, i, i, i, p, p, p]
        L.ora_quantize_kv.restype = i
        L.ora_quantize_kv.argtypes = [p, p, p, i, i, i, i, i, i, p, p, p, p, p, p, p, i64]
        L.ora_quantize_q.restype = i
        L.ora_quantize_q.argtypes = [p, i, i, i, i, i, i, p, p, p, p, p, p, p]
        L.ora_decode.restype = i
        L.ora_decode.argtypes = [p, p, p, p, p, p, p, i, i, i, i, i, i, i64, i, i, p, p, p, d, i, p, p]
        L.ora_attention_ref.restype = i
        L.ora_attention_ref.argtypes = [p, p, p, p, i, i, i, i, i, d, p]
        L.ora_block_sigma.restype = f
        L.ora_block_sigma.argtypes = [i, i, f]
        L.ora_quantize_block.restype = d
        L.ora_quantize_block.argtypes = [p, i, f, p]
        L.ora_plain_scale_code.restype = i
        L.ora_plain_scale_code.argtypes = [i, f, f]
        L.ora_search_scale_code.restype = i
        L.ora_search_scale_code.argtypes = [i, p, i, f]
        L.ora_dynamic_alpha_exp.restype = i
        L.ora_dynamic_alpha_exp.argtypes = [d]
        L.ora_search_scale_code_weighted.restype = i
        L.ora_search_scale_code_weighted.argtypes = [i, p, i, f, p]
        L.ora_key_weights.restype = i
        L.ora_key_weights.argtypes = [p, i, i, i, i, i, p, p]
        L.ora_quantize_kv_weighted.restype = i
        L.ora_quantize_kv_weighted.argtypes = [p, p, p, i, i, i, i, i, i, p, p, p, p, p, p, p, p, i64]
        L.ora_dequant_key_row.restype = None
        L.ora_dequant_key_row.argtypes = [p, p, i, i64, i, i, i, i, p]
        L.ora_dequant_value_row.restype = None
        L.ora_dequant_value_row.argtypes = [p, p, i, i64, i, i, i, i, p]
        L.ora_num_threads.restype = i
        L.ora_num_threads.argtypes = []
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def _bits(a) -> np.ndarray:
    """bf16 tensor / uint16 array -> contiguous uint16 numpy array of raw bits."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            assert a.dtype == torch.bfloat16
            return np.ascontiguousarray(a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    except ImportError:  # pragma: no cover
        pass
    a = np.asarray(a)
    assert a.dtype == np.uint16
    return np.ascontiguousarray(a)


def beta(fmt: int) -> int:
    return 16 if fmt == NVFP4 else 32


# ---------------------------------------------------------------- formats
def e2m1_value(code: int) -> float:
    return lib().ora_e2m1_value(int(code))


def e2m1_encode(x: float) -> int:
    return lib().ora_e2m1_encode(float(x))


def e4m3_value(code: int) -> float:
    return lib().ora_e4m3_value(int(code))


def e4m3_encode(u: float) -> int:
    return lib().ora_e4m3_encode(float(u))


def e8m0_value(code: int) -> float:
    return lib().ora_e8m0_value(int(code))


def mx_scale_code(amax: float) -> int:
    return lib().ora_mx_scale_code(float(amax))


def f64_to_bf16(x: float) -> int:
    return lib().ora_f64_to_bf16(float(x))


# ---------------------------------------------------------------- blocks
def block_sigma(fmt: int, code: int, g: float) -> float:
    return lib().ora_block_sigma(fmt, int(code), float(g))


def quantize_block(x: np.ndarray, sigma: float):
    """-> (codes uint8[n], fp64 squared error)."""
    x = np.ascontiguousarray(x, np.float32)
    codes = np.zeros(x.shape[0], np.uint8)
    err = lib().ora_quantize_block(_ptr(x), x.shape[0], float(sigma), _ptr(codes))
    return codes, err


def plain_scale_code(fmt: int, amax: float, g: float) -> int:
    return lib().ora_plain_scale_code(fmt, float(amax), float(g))


def search_scale_code(fmt: int, x: np.ndarray, g: float, w=None) -> int:
    x = np.ascontiguousarray(x, np.float32)
    if w is None:
        return lib().ora_search_scale_code(fmt, _ptr(x), x.shape[0], float(g))
    w = np.ascontiguousarray(w, np.float32)
    return lib().ora_search_scale_code_weighted(fmt, _ptr(x), x.shape[0], float(g), _ptr(w))


def dynamic_alpha_exp(p_max: float) -> int:
    """Exponent of the per-tile probability pre-scale of the dynamic variant."""
    return lib().ora_dynamic_alpha_exp(float(p_max))


def dequant_key_row(cache: dict, fmt: int, page: int, head: int, H_kv: int, d_k: int, slot: int) -> np.ndarray:
    out = np.zeros(d_k, np.float64)
    lib().ora_dequant_key_row(_ptr(cache["k_pages"]), _ptr(cache["k_scales"]), fmt, page, head, H_kv, d_k, slot,
                              _ptr(out))
    return out


def dequant_value_row(cache: dict, fmt: int, page: int, head: int, H_kv: int, d_v: int, slot: int) -> np.ndarray:
    out = np.zeros(d_v, np.float64)
    lib().ora_dequant_value_row(_ptr(cache["v_pages"]), _ptr(cache["v_scales"]), fmt, page, head, H_kv, d_v, slot,
                                _ptr(out))
    return out


# ---------------------------------------------------------------- transform
def fwht_f32(x: np.ndarray) -> np.ndarray:
    y = np.ascontiguousarray(x, dtype=np.float32).copy()
    lib().ora_fwht_f32(_ptr(y), y.shape[-1])
    return y


def transform(x: np.ndarray, smooth: np.ndarray, is_key: bool, hadamard: bool = True) -> np.ndarray:
    """Key (is_key) or query transform of each row of x [..., d] with one smoothing vector [d]."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    s = np.ascontiguousarray(smooth, dtype=np.float32)
    d = x.shape[-1]
    rows = x.reshape(-1, d)
    out = np.empty_like(rows)
    for r in range(rows.shape[0]):
        xr, orow = np.ascontiguousarray(rows[r]), np.empty(d, np.float32)
        lib().ora_transform(_ptr(xr), _ptr(s), d, int(is_key), int(hadamard), _ptr(orow))
        out[r] = orow
    return out.reshape(x.shape)


# ---------------------------------------------------------------- calibration
def calibrate(k_cal, q_cal, v_cal, H_q: int, H_kv: int, flags: int = 0):
    k, q, v = _bits(k_cal), _bits(q_cal), _bits(v_cal)
    Tc, _, d_k = k.shape
    Tq = q.shape[0]
    d_v = v.shape[2]
    smooth = np.empty((H_kv, d_k), np.float32)
    kg = np.empty(H_kv, np.float32)
    vg = np.empty(H_kv, np.float32)
    rc = lib().ora_calibrate(_ptr(k), _ptr(q), _ptr(v), Tc, Tq, H_q, H_kv, d_k, d_v, flags,
                             _ptr(smooth), _ptr(kg), _ptr(vg))
    assert rc == 0, rc
    return smooth, kg, vg


# ---------------------------------------------------------------- cache
def cache_sizes(num_pages: int, H_kv: int, d_k: int, d_v: int, fmt: int) -> dict:
    b = beta(fmt)
    return dict(k_pages=num_pages * H_kv * PAGE_SLOTS * d_k // 2,
                k_scales=num_pages * H_kv * 256 * ((d_k // b + 3) // 4),
                v_pages=num_pages * H_kv * d_v * PAGE_SLOTS // 2,
                v_scales=num_pages * H_kv * d_v * PAGE_SLOTS // b)


def empty_cache(num_pages: int, H_kv: int, d_k: int, d_v: int, fmt: int) -> dict:
    return {k: np.zeros(n, np.uint8) for k, n in cache_sizes(num_pages, H_kv, d_k, d_v, fmt).items()}


def quantize_kv(k, v, slot_mapping, cache: dict, H_kv: int, fmt: int, smooth, k_g, v_g,
                num_pages: int, flags: int = 0, k_weight=None) -> dict:
    """Append-quantize tokens into ``cache`` (in place) and return it.  ``k_weight``
    ([H_kv, d_k]) selects the attention-aware key scale search."""
    kb, vb = _bits(k), _bits(v)
    T, _, d_k = kb.shape
    d_v = vb.shape[2]
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    s = np.ascontiguousarray(smooth, np.float32)
    kg = np.ascontiguousarray(k_g, np.float32)
    vg = np.ascontiguousarray(v_g, np.float32)
    pages = (_ptr(cache["k_pages"]), _ptr(cache["k_scales"]), _ptr(cache["v_pages"]), _ptr(cache["v_scales"]))
    if k_weight is None:
        rc = lib().ora_quantize_kv(_ptr(kb), _ptr(vb), _ptr(sm), T, H_kv, d_k, d_v, fmt, flags,
                                   _ptr(s), _ptr(kg), _ptr(vg), *pages, num_pages)
    else:
        w = np.ascontiguousarray(k_weight, np.float32).reshape(H_kv, d_k)
        rc = lib().ora_quantize_kv_weighted(_ptr(kb), _ptr(vb), _ptr(sm), T, H_kv, d_k, d_v, fmt, flags,
                                            _ptr(s), _ptr(kg), _ptr(vg), _ptr(w), *pages, num_pages)
    assert rc == 0, rc
    return cache


def key_weights(q_cal, H_q: int, H_kv: int, smooth, flags: int = 0) -> np.ndarray:
    """[H_kv, d_k] channel weights of the attention-aware key scale search."""
    q = _bits(q_cal)
    Tq, _, d_k = q.shape
    s = np.ascontiguousarray(smooth, np.float32)
    w = np.empty((H_kv, d_k), np.float32)
    rc = lib().ora_key_weights(_ptr(q), Tq, H_q, H_kv, d_k, flags, _ptr(s), _ptr(w))
    assert rc == 0, rc
    return w


def quantize_q(q, H_kv: int, fmt: int, smooth, flags: int = 0) -> dict:
    qb = _bits(q)
    B, H_q, d_k = qb.shape
    nb = d_k // beta(fmt)
    out = dict(q1_codes=np.zeros((B, H_q, d_k), np.uint8), q1_scales=np.zeros((B, H_q, nb), np.uint8),
               q2_codes=np.zeros((B, H_q, d_k), np.uint8), q2_scales=np.zeros((B, H_q, nb), np.uint8),
               g_q=np.zeros((B, H_q), np.float32), xq=np.zeros((B, H_q, d_k), np.float32))
    s = np.ascontiguousarray(smooth, np.float32)
    rc = lib().ora_quantize_q(_ptr(qb), B, H_q, H_kv, d_k, fmt, flags, _ptr(s),
                              _ptr(out["q1_codes"]), _ptr(out["q1_scales"]), _ptr(out["q2_codes"]),
                              _ptr(out["q2_scales"]), _ptr(out["g_q"]), _ptr(out["xq"]))
    assert rc == 0, rc
    return out


def decode(q, cache: dict, block_table, seq_lens, H_kv: int, d_v: int, fmt: int, smooth, k_g, v_g,
           sm_scale: float, chunk_tiles: int, num_pages: int, flags: int = 0):
    """Returns (out_bf16_bits [B,H_q,d_v] uint16, out_f64 [B,H_q,d_v])."""
    qb = _bits(q)
    B, H_q, d_k = qb.shape
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    out16 = np.zeros((B, H_q, d_v), np.uint16)
    out64 = np.zeros((B, H_q, d_v), np.float64)
    s = np.ascontiguousarray(smooth, np.float32)
    kg = np.ascontiguousarray(k_g, np.float32)
    vg = np.ascontiguousarray(v_g, np.float32)
    rc = lib().ora_decode(_ptr(qb), _ptr(cache["k_pages"]), _ptr(cache["k_scales"]), _ptr(cache["v_pages"]),
                          _ptr(cache["v_scales"]), _ptr(bt), _ptr(sl), B, H_q, H_kv, d_k, d_v, bt.shape[1],
                          num_pages, fmt, flags, _ptr(s), _ptr(kg), _ptr(vg), float(sm_scale), int(chunk_tiles),
                          _ptr(out16), _ptr(out64))
    assert rc == 0, rc
    return out16, out64


def decode_multi(q, cache: dict, block_table, seq_lens, H_kv: int, d_v: int, fmt: int, smooth, k_g, v_g,
                 sm_scale: float, chunk_tiles: int, num_pages: int, flags: int = 0):
    """Multi-token queries (speculative or chunked decode): q [B, T_q, H_q, d_k]
    holds each sequence's T_q newest tokens, already in the cache.  Query token i
    attends causally to the first seq_lens[b] - T_q + 1 + i tokens and runs the
    single-token decode on that prefix, with the same tile and split boundaries
    (splits cut at multiples of chunk_tiles from the sequence start).  Returns
    (bf16 bits, fp64) outputs [B, T_q, H_q, d_v]."""
    qb = _bits(q)
    B, T_q, H_q, d_k = qb.shape
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.asarray(seq_lens, dtype=np.int64)
    if np.any(sl < T_q):
        raise ValueError("every sequence must hold its T_q query tokens")
    rows_sl = (sl[:, None] - T_q + 1 + np.arange(T_q)[None, :]).reshape(-1).astype(np.int32)
    rows_bt = np.repeat(bt, T_q, axis=0)
    o16, o64 = decode(np.ascontiguousarray(qb.reshape(B * T_q, H_q, d_k)), cache, rows_bt, rows_sl, H_kv, d_v, fmt, smooth, k_g, v_g, sm_scale, chunk_tiles,
                      num_pages, flags=flags)
    return o16.reshape(B, T_q, H_q, d_v), o64.reshape(B, T_q, H_q, d_v)


def attention_ref(q, k, v, cu_seqlens, H_kv: int, sm_scale: float) -> np.ndarray:
    """fp64 softmax(q k^T * sm_scale) v on the unquantized bf16 inputs."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, H_q, d_k = qb.shape
    d_v = vb.shape[2]
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int64)
    out = np.zeros((B, H_q, d_v), np.float64)
    rc = lib().ora_attention_ref(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(cu), B, H_q, H_kv, d_k, d_v,
                                 float(sm_scale), _ptr(out))
    assert rc == 0, rc
    return out


def num_threads() -> int:
    return lib().ora_num_threads()


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)
