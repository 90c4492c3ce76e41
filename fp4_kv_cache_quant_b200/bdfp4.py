"""Thin ctypes binding of the bdfp4 C ABI (include/bdfp4.h).

Argument marshalling only: every step of the path runs in libbdfp4.so's CUDA
kernels.  torch provides device memory and streams.  The library is loaded
from this package's directory; importing this module on a machine where it
is missing raises, there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbdfp4.so")

NVFP4, MXFP4 = 0, 1
FLAG_NO_HADAMARD = 1
FLAG_NO_SCALE_SEARCH = 2
FLAG_SINGLE_QUERY = 4
FLAG_NO_UNDERFLOW = 8
FLAG_DYNAMIC_ALPHA = 32

DEV_BAD_PAGE, DEV_BAD_SEQLEN, DEV_BAD_SLOT, DEV_TIMEOUT = 1, 2, 4, 8

PAGE_SLOTS = 64
TILE_TOKENS = 128

#: names of every entry point declared in include/bdfp4.h
ENTRY_POINTS = ("bdfp4_calibrate", "bdfp4_key_weights", "bdfp4_quantize_kv", "bdfp4_quantize_k", "bdfp4_quantize_v", "bdfp4_quantize_q", "bdfp4_decode_plan",
                "bdfp4_decode_plan_for", "bdfp4_decode_multi_plan",
                "bdfp4_decode_workspace_size", "bdfp4_decode", "bdfp4_decode_step", "bdfp4_decode_multi",
                "bdfp4_decode_noalloc",
                "bdfp4_status_string", "bdfp4_last_error")
#: names of every entry point declared in include/bdfp4_bf16.h
BF16_ENTRY_POINTS = ("bdfp4_bf16_append", "bdfp4_bf16_decode")
#: names of every entry point declared in include/bdfp4_debug.h (test hooks)
DEBUG_ENTRY_POINTS = ("bdfp4_debug_decode_wait_test",)

#: size of the library's built-in scratch used by bdfp4_decode_noalloc
NOALLOC_SCRATCH_BYTES = 16 << 20


class BDFP4Error(RuntimeError):
    pass


class _KVParams(ctypes.Structure):
    _fields_ = [("smooth", ctypes.c_void_p), ("k_gscale", ctypes.c_void_p), ("v_gscale", ctypes.c_void_p),
                ("k_weight", ctypes.c_void_p)]


_lib = None


def load() -> ctypes.CDLL:
    """Load libbdfp4.so (raises OSError if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise OSError(f"{LIB_PATH} is missing: build it with `python -m fp4_kv_cache_quant_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    i, i64, p, f, sz = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_float, ctypes.c_size_t
    kvp = ctypes.POINTER(_KVParams)
    L.bdfp4_calibrate.argtypes = [p, p, p, i, i, i, i, i, i, i, p, p, p, p]
    L.bdfp4_calibrate.restype = i
    L.bdfp4_key_weights.argtypes = [p, i, i, i, i, i, p, p, p]
    L.bdfp4_key_weights.restype = i
    L.bdfp4_quantize_kv.argtypes = [p, p, p, i, i, i, i, i, i, kvp, p, p, p, p, i64, p, p]
    L.bdfp4_quantize_kv.restype = i
    L.bdfp4_quantize_k.argtypes = [p, p, i, i, i, i, i, kvp, p, p, i64, p, p]
    L.bdfp4_quantize_k.restype = i
    L.bdfp4_quantize_v.argtypes = [p, p, i, i, i, i, kvp, p, p, i64, p]
    L.bdfp4_quantize_v.restype = i
    L.bdfp4_quantize_q.argtypes = [p, i, i, i, i, i, i, p, p, p, p, p, p, p]
    L.bdfp4_quantize_q.restype = i
    L.bdfp4_decode_plan.argtypes = [p, i, i, i]
    L.bdfp4_decode_plan.restype = i
    L.bdfp4_decode_plan_for.argtypes = [p, i, i, i, i, i, i]
    L.bdfp4_decode_plan_for.restype = i
    L.bdfp4_decode_multi_plan.argtypes = [p, i, i, i, i, i, i, i]
    L.bdfp4_decode_multi_plan.restype = i
    L.bdfp4_decode_workspace_size.argtypes = [i, i, i, i, i]
    L.bdfp4_decode_workspace_size.restype = sz
    L.bdfp4_decode.argtypes = [p, p, p, p, p, p, p, i, i, i, i, i, i, i64, i, i, kvp, f, i, p, sz, p, p, p]
    L.bdfp4_decode.restype = i
    L.bdfp4_decode_step.argtypes = [p, p, p, p, p, p, p, p, p, p, i, i, i, i, i, i, i64, i, i, kvp, f, i, p, sz, p, p,
                                    p]
    L.bdfp4_decode_step.restype = i
    L.bdfp4_decode_multi.argtypes = [p, p, p, p, p, p, p, i, i, i, i, i, i, i, i64, i, i, kvp, f, i, p, sz, p, p, p]
    L.bdfp4_decode_multi.restype = i
    L.bdfp4_decode_noalloc.argtypes = [p, p, p, p, p, p, p, i, i, i, i, i, i, i64, i, i, kvp, f, i, p, p, p]
    L.bdfp4_decode_noalloc.restype = i
    L.bdfp4_status_string.argtypes = [i]
    L.bdfp4_status_string.restype = ctypes.c_char_p
    L.bdfp4_last_error.argtypes = []
    L.bdfp4_last_error.restype = ctypes.c_char_p
    L.bdfp4_debug_decode_wait_test.argtypes = [p, p, p, p, p, p, p, i, i, i, i, i, i, i64, i, i, kvp, f, i, p, sz, p,
                                               p, ctypes.c_longlong, i, p]
    L.bdfp4_debug_decode_wait_test.restype = i
    L.bdfp4_bf16_append.argtypes = [p, p, p, i, i, i, p, p, i64, p, p]
    L.bdfp4_bf16_append.restype = i
    L.bdfp4_bf16_decode.argtypes = [p, p, p, p, p, i, i, i, i, i, i64, f, i, p, sz, p, p, p]
    L.bdfp4_bf16_decode.restype = i
    _lib = L
    return L


def bdfp4_status_string(status: int) -> str:
    return load().bdfp4_status_string(int(status)).decode()


def bdfp4_last_error() -> str:
    return load().bdfp4_last_error().decode()


def _check(rc: int, what: str):
    if rc != 0:
        detail = f" [{bdfp4_last_error()}]" if rc == -5 else ""
        raise BDFP4Error(f"{what}: {bdfp4_status_string(rc)} ({rc}){detail}")


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    assert t.is_contiguous(), "tensors passed to bdfp4 must be contiguous"
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def beta(fmt: int) -> int:
    return 16 if fmt == NVFP4 else 32


@dataclass
class KVParams:
    """Static per-layer parameters: smoothing factors, FP32 tensor scales and,
    optionally, the channel weights of the attention-aware key scale search."""
    smooth: torch.Tensor    # [H_kv, d_k] fp32
    k_gscale: torch.Tensor  # [H_kv] fp32
    v_gscale: torch.Tensor  # [H_kv] fp32
    k_weight: torch.Tensor | None = None   # [H_kv, d_k] fp32 (bdfp4_key_weights) or None

    def _c(self) -> _KVParams:
        return _KVParams(self.smooth.data_ptr(), self.k_gscale.data_ptr(), self.v_gscale.data_ptr(),
                         None if self.k_weight is None else self.k_weight.data_ptr())


@dataclass
class FP4Cache:
    """The paged FP4 KV cache arrays (layout in include/bdfp4.h)."""
    k_pages: torch.Tensor
    k_scales: torch.Tensor
    v_pages: torch.Tensor
    v_scales: torch.Tensor
    num_pages: int
    H_kv: int
    d_k: int
    d_v: int
    fmt: int

    @staticmethod
    def empty(num_pages: int, H_kv: int, d_k: int, d_v: int, fmt: int, device="cuda") -> "FP4Cache":
        b = beta(fmt)
        mk = lambda n: torch.zeros(n, dtype=torch.uint8, device=device)  # noqa: E731
        return FP4Cache(mk(num_pages * H_kv * PAGE_SLOTS * d_k // 2), mk(num_pages * H_kv * 256 * ((d_k // b + 3) // 4)),
                        mk(num_pages * H_kv * d_v * PAGE_SLOTS // 2), mk(num_pages * H_kv * d_v * PAGE_SLOTS // b),
                        num_pages, H_kv, d_k, d_v, fmt)

    def nbytes(self) -> int:
        return sum(t.numel() for t in (self.k_pages, self.k_scales, self.v_pages, self.v_scales))


def bdfp4_calibrate(k_cal: torch.Tensor, q_cal: torch.Tensor, v_cal: torch.Tensor, H_q: int, H_kv: int,
                    flags: int = 0, stream=None) -> KVParams:
    Tc, _, d_k = k_cal.shape
    d_v = v_cal.shape[2]
    dev = k_cal.device
    kv = KVParams(torch.empty((H_kv, d_k), dtype=torch.float32, device=dev),
                  torch.empty(H_kv, dtype=torch.float32, device=dev), torch.empty(H_kv, dtype=torch.float32, device=dev))
    rc = load().bdfp4_calibrate(_ptr(k_cal), _ptr(q_cal), _ptr(v_cal), Tc, q_cal.shape[0], H_q, H_kv, d_k, d_v, flags,
                                _ptr(kv.smooth), _ptr(kv.k_gscale), _ptr(kv.v_gscale), _stream(stream))
    _check(rc, "bdfp4_calibrate")
    return kv


def bdfp4_key_weights(q_cal: torch.Tensor, H_kv: int, smooth: torch.Tensor, flags: int = 0,
                      stream=None) -> torch.Tensor:
    """[H_kv, d_k] channel weights of the attention-aware key scale search from
    calibration queries q_cal [Tq, H_q, d_k] (bdfp4_key_weights in bdfp4.h)."""
    Tq, H_q, d_k = q_cal.shape
    w = torch.empty((H_kv, d_k), dtype=torch.float32, device=q_cal.device)
    rc = load().bdfp4_key_weights(_ptr(q_cal), Tq, H_q, H_kv, d_k, flags, _ptr(smooth), _ptr(w), _stream(stream))
    _check(rc, "bdfp4_key_weights")
    return w


def bdfp4_quantize_kv(k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor, kv: KVParams, cache: FP4Cache,
                      flags: int = 0, dev_status: torch.Tensor | None = None, stream=None) -> None:
    T = k.shape[0]
    c = kv._c()
    rc = load().bdfp4_quantize_kv(_ptr(k), _ptr(v), _ptr(slot_mapping), T, cache.H_kv, cache.d_k, cache.d_v,
                                  cache.fmt, flags, ctypes.byref(c), _ptr(cache.k_pages), _ptr(cache.k_scales),
                                  _ptr(cache.v_pages), _ptr(cache.v_scales), cache.num_pages, _ptr(dev_status),
                                  _stream(stream))
    _check(rc, "bdfp4_quantize_kv")


def bdfp4_quantize_k(k: torch.Tensor, slot_mapping: torch.Tensor, kv: KVParams, cache: FP4Cache, flags: int = 0,
                     dev_status: torch.Tensor | None = None, stream=None) -> None:
    c = kv._c()
    rc = load().bdfp4_quantize_k(_ptr(k), _ptr(slot_mapping), k.shape[0], cache.H_kv, cache.d_k, cache.fmt, flags,
                                 ctypes.byref(c), _ptr(cache.k_pages), _ptr(cache.k_scales), cache.num_pages,
                                 _ptr(dev_status), _stream(stream))
    _check(rc, "bdfp4_quantize_k")


def bdfp4_quantize_v(v: torch.Tensor, slot_mapping: torch.Tensor, kv: KVParams, cache: FP4Cache, stream=None) -> None:
    c = kv._c()
    rc = load().bdfp4_quantize_v(_ptr(v), _ptr(slot_mapping), v.shape[0], cache.H_kv, cache.d_v, cache.fmt,
                                 ctypes.byref(c), _ptr(cache.v_pages), _ptr(cache.v_scales), cache.num_pages,
                                 _stream(stream))
    _check(rc, "bdfp4_quantize_v")


def bdfp4_quantize_q(q: torch.Tensor, H_kv: int, fmt: int, smooth: torch.Tensor, flags: int = 0,
                     stream=None) -> dict:
    B, H_q, d_k = q.shape
    nb = d_k // beta(fmt)
    dev = q.device
    out = dict(q1_codes=torch.empty((B, H_q, d_k), dtype=torch.uint8, device=dev),
               q1_scales=torch.empty((B, H_q, nb), dtype=torch.uint8, device=dev),
               q2_codes=torch.empty((B, H_q, d_k), dtype=torch.uint8, device=dev),
               q2_scales=torch.empty((B, H_q, nb), dtype=torch.uint8, device=dev),
               g_q=torch.empty((B, H_q), dtype=torch.float32, device=dev))
    rc = load().bdfp4_quantize_q(_ptr(q), B, H_q, H_kv, d_k, fmt, flags, _ptr(smooth), _ptr(out["q1_codes"]),
                                 _ptr(out["q1_scales"]), _ptr(out["q2_codes"]), _ptr(out["q2_scales"]),
                                 _ptr(out["g_q"]), _stream(stream))
    _check(rc, "bdfp4_quantize_q")
    return out


def bdfp4_decode_plan(host_seq_lens, H_kv: int, num_sms: int) -> int:
    import numpy as np
    sl = np.ascontiguousarray(host_seq_lens, dtype=np.int32)
    rc = load().bdfp4_decode_plan(ctypes.c_void_p(sl.ctypes.data), sl.shape[0], H_kv, num_sms)
    if rc < 0:
        _check(rc, "bdfp4_decode_plan")
    return rc


def bdfp4_decode_plan_for(host_seq_lens, H_q: int, H_kv: int, d_k: int, d_v: int, num_sms: int) -> int:
    import numpy as np
    sl = np.ascontiguousarray(host_seq_lens, dtype=np.int32)
    rc = load().bdfp4_decode_plan_for(ctypes.c_void_p(sl.ctypes.data), sl.shape[0], H_q, H_kv, d_k, d_v, num_sms)
    if rc < 0:
        _check(rc, "bdfp4_decode_plan_for")
    return rc


def bdfp4_decode_multi_plan(host_seq_lens, T_q: int, H_q: int, H_kv: int, d_k: int, d_v: int, num_sms: int) -> int:
    import numpy as np
    sl = np.ascontiguousarray(host_seq_lens, dtype=np.int32)
    rc = load().bdfp4_decode_multi_plan(ctypes.c_void_p(sl.ctypes.data), sl.shape[0], T_q, H_q, H_kv, d_k, d_v,
                                        num_sms)
    if rc < 0:
        _check(rc, "bdfp4_decode_multi_plan")
    return rc


def bdfp4_decode_workspace_size(B: int, H_q: int, d_v: int, max_pages_per_seq: int, chunk_tiles: int) -> int:
    return int(load().bdfp4_decode_workspace_size(B, H_q, d_v, max_pages_per_seq, chunk_tiles))


def bdfp4_decode(q: torch.Tensor, cache: FP4Cache, block_table: torch.Tensor, seq_lens: torch.Tensor, kv: KVParams,
                 sm_scale: float, chunk_tiles: int, workspace: torch.Tensor | None, out: torch.Tensor,
                 flags: int = 0, dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    B, H_q, d_k = q.shape
    c = kv._c()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load().bdfp4_decode(_ptr(q), _ptr(cache.k_pages), _ptr(cache.k_scales), _ptr(cache.v_pages),
                             _ptr(cache.v_scales), _ptr(block_table), _ptr(seq_lens), B, H_q, cache.H_kv, d_k,
                             cache.d_v, block_table.shape[1], cache.num_pages, cache.fmt, flags, ctypes.byref(c),
                             float(sm_scale), int(chunk_tiles), _ptr(workspace), ws_bytes, _ptr(out),
                             _ptr(dev_status), _stream(stream))
    _check(rc, "bdfp4_decode")
    return out


def bdfp4_decode_multi(q: torch.Tensor, cache: FP4Cache, block_table: torch.Tensor, seq_lens: torch.Tensor,
                       kv: KVParams, sm_scale: float, chunk_tiles: int, workspace: torch.Tensor | None,
                       out: torch.Tensor, flags: int = 0, dev_status: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    """Causal decode of each sequence's T_q newest tokens: q [B, T_q, H_q, d_k],
    out [B, T_q, H_q, d_v] (bdfp4_decode_multi in bdfp4.h)."""
    B, T_q, H_q, d_k = q.shape
    c = kv._c()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load().bdfp4_decode_multi(_ptr(q), _ptr(cache.k_pages), _ptr(cache.k_scales), _ptr(cache.v_pages),
                                   _ptr(cache.v_scales), _ptr(block_table), _ptr(seq_lens), B, T_q, H_q, cache.H_kv,
                                   d_k, cache.d_v, block_table.shape[1], cache.num_pages, cache.fmt, flags,
                                   ctypes.byref(c), float(sm_scale), int(chunk_tiles), _ptr(workspace), ws_bytes,
                                   _ptr(out), _ptr(dev_status), _stream(stream))
    _check(rc, "bdfp4_decode_multi")
    return out


def bdfp4_decode_step(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, v_open: torch.Tensor,
                      cache: FP4Cache, block_table: torch.Tensor, seq_lens: torch.Tensor, kv: KVParams,
                      sm_scale: float, chunk_tiles: int, workspace: torch.Tensor | None, out: torch.Tensor,
                      flags: int = 0, dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Append each sequence's new token (k_new, v_new [B, H_kv, d]) at position
    seq_lens[b] - 1, keeping the open value block in v_open [B, beta, H_kv, d_v],
    then decode q over the updated cache (bdfp4_decode_step in bdfp4.h)."""
    B, H_q, d_k = q.shape
    c = kv._c()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load().bdfp4_decode_step(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(v_open), _ptr(cache.k_pages),
                                  _ptr(cache.k_scales), _ptr(cache.v_pages), _ptr(cache.v_scales), _ptr(block_table),
                                  _ptr(seq_lens), B, H_q, cache.H_kv, d_k, cache.d_v, block_table.shape[1],
                                  cache.num_pages, cache.fmt, flags, ctypes.byref(c), float(sm_scale),
                                  int(chunk_tiles), _ptr(workspace), ws_bytes, _ptr(out), _ptr(dev_status),
                                  _stream(stream))
    _check(rc, "bdfp4_decode_step")
    return out


def bdfp4_debug_decode_wait_test(q: torch.Tensor, cache: FP4Cache, block_table: torch.Tensor, seq_lens: torch.Tensor,
                                 kv: KVParams, sm_scale: float, chunk_tiles: int, workspace: torch.Tensor | None,
                                 out: torch.Tensor, wait_limit_cycles: int, stall: bool, flags: int = 0,
                                 dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Test hook (include/bdfp4_debug.h): bdfp4_decode with a short in-kernel wait
    bound and, with stall, every CTA's first K tile withheld so its waits run out."""
    B, H_q, d_k = q.shape
    c = kv._c()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load().bdfp4_debug_decode_wait_test(_ptr(q), _ptr(cache.k_pages), _ptr(cache.k_scales), _ptr(cache.v_pages),
                                             _ptr(cache.v_scales), _ptr(block_table), _ptr(seq_lens), B, H_q,
                                             cache.H_kv, d_k, cache.d_v, block_table.shape[1], cache.num_pages,
                                             cache.fmt, flags, ctypes.byref(c), float(sm_scale), int(chunk_tiles),
                                             _ptr(workspace), ws_bytes, _ptr(out), _ptr(dev_status),
                                             int(wait_limit_cycles), 1 if stall else 0, _stream(stream))
    _check(rc, "bdfp4_debug_decode_wait_test")
    return out


def workspace_for(B: int, H_q: int, d_v: int, max_pages_per_seq: int, chunk_tiles: int, device="cuda"):
    n = bdfp4_decode_workspace_size(B, H_q, d_v, max_pages_per_seq, chunk_tiles)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def bdfp4_decode_noalloc(q: torch.Tensor, cache: FP4Cache, block_table: torch.Tensor, seq_lens: torch.Tensor,
                         kv: KVParams, sm_scale: float, chunk_tiles: int, out: torch.Tensor, flags: int = 0,
                         dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """bdfp4_decode for callers that cannot allocate device memory: the split
    partials use the library's built-in scratch (NOALLOC_SCRATCH_BYTES), so no
    workspace is passed.  Calls that overlap on the GPU race on that scratch."""
    B, H_q, d_k = q.shape
    c = kv._c()
    rc = load().bdfp4_decode_noalloc(_ptr(q), _ptr(cache.k_pages), _ptr(cache.k_scales), _ptr(cache.v_pages),
                                     _ptr(cache.v_scales), _ptr(block_table), _ptr(seq_lens), B, H_q, cache.H_kv,
                                     d_k, cache.d_v, block_table.shape[1], cache.num_pages, cache.fmt, flags,
                                     ctypes.byref(c), float(sm_scale), int(chunk_tiles), _ptr(out),
                                     _ptr(dev_status), _stream(stream))
    _check(rc, "bdfp4_decode_noalloc")
    return out


# ---------------------------------------------------------------- BF16-KV comparator (include/bdfp4_bf16.h)
@dataclass
class BF16Cache:
    """bf16 K/V pages in the comparator's MMA operand layouts (16 KB per page and head at d = 128)."""
    k_pages: torch.Tensor   # uint8 [num_pages, H_kv, 64 * d * 2]
    v_pages: torch.Tensor   # uint8 [num_pages, H_kv, d * 64 * 2]
    num_pages: int
    H_kv: int
    d: int

    @staticmethod
    def empty(num_pages: int, H_kv: int, d: int, device="cuda") -> "BF16Cache":
        n = PAGE_SLOTS * d * 2
        return BF16Cache(torch.empty((num_pages, H_kv, n), dtype=torch.uint8, device=device),
                         torch.empty((num_pages, H_kv, n), dtype=torch.uint8, device=device), num_pages, H_kv, d)

    def nbytes(self) -> int:
        return self.k_pages.numel() + self.v_pages.numel()


def bdfp4_bf16_append(k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor, cache: BF16Cache,
                      dev_status: torch.Tensor | None = None, stream=None):
    T, H_kv, d = k.shape
    _check(load().bdfp4_bf16_append(_ptr(k), _ptr(v), _ptr(slot_mapping), T, H_kv, d, _ptr(cache.k_pages),
                                    _ptr(cache.v_pages), cache.num_pages, _ptr(dev_status), _stream(stream)),
           "bdfp4_bf16_append")


def bdfp4_bf16_decode(q: torch.Tensor, cache: BF16Cache, block_table: torch.Tensor, seq_lens: torch.Tensor,
                      sm_scale: float, chunk_tiles: int, workspace: torch.Tensor | None, out: torch.Tensor,
                      dev_status: torch.Tensor | None = None, stream=None):
    B, H_q, d = q.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().bdfp4_bf16_decode(_ptr(q), _ptr(cache.k_pages), _ptr(cache.v_pages), _ptr(block_table),
                                    _ptr(seq_lens), B, H_q, cache.H_kv, d, block_table.shape[1], cache.num_pages,
                                    float(sm_scale), int(chunk_tiles), _ptr(workspace), ws_bytes, _ptr(out),
                                    _ptr(dev_status), _stream(stream)),
           "bdfp4_bf16_decode")
