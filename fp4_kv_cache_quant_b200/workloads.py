"""Seeded synthetic workloads for the FP4 paged decode-attention path.

This module only draws random numbers and lays out pages; it holds none of
the method's arithmetic, so both the CUDA path and the CPU oracle can take
their inputs from it.

The shapes are those of the models the BitDecoding-FP4 pages serve (Qwen3-4B,
Qwen3-30B-A3B; DeepSeek-style MLA for the MLA case), standing in for the
pages' unnamed serving workloads:

* ``tiny``          B=1, 4 query heads / 1 KV head, d=128, context 1024,
                    4 fixed key channels scaled x20.
* ``qwen3_4b``      B=16, 32/8 heads, d=128, context 32768 each, 3 of 128 key
                    channels per KV head scaled by U[10, 30] (about 2%).
* ``qwen3_30b_a3b`` B=64, 32/4 heads (GQA 8), d=128, context U[8192, 131072].
* ``underflow``     B=4, 32/8 heads, d=128, context 131072, keys N(0, 0.05^2).
* ``mla``           B=32, 128 heads over one latent head, d_k=576 (512 latent
                    + 64 rope), d_v=512 with V = the latent part of K,
                    context 16384, 6 of 576 channels scaled by U[10, 30].

Values are bf16 draws of N(0, 1) unless stated.  Pages hold 64 tokens; the
page pool has exactly sum(ceil(N_b / 64)) pages and a seeded permutation
assigns them to sequences.  Calibration draws (1024 tokens, 64 queries) use
the same distribution and outlier channels with their own seed.

torch's CPU and CUDA generators differ, so a workload drawn on the GPU has the
same distribution but not the same numbers as one drawn on the CPU; parity
tests draw on the CPU and copy.
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass

import numpy as np
import torch

PAGE_SLOTS = 64


@dataclass(frozen=True)
class Spec:
    name: str
    B: int
    H_q: int
    H_kv: int
    d_k: int
    d_v: int
    ctx: tuple            # ("fixed", N) | ("uniform", lo, hi) | ("list", (N0, N1, ...))
    fmts: tuple = ("nvfp4",)
    key_std: float = 1.0
    n_outlier: int = 0    # outlier key channels per KV head
    outlier_lo: float = 1.0
    outlier_hi: float = 1.0
    mla: bool = False     # V = first d_v channels of K

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.d_k)

    @property
    def group(self) -> int:
        return self.H_q // self.H_kv


SPECS = {
    "tiny": Spec("tiny", 1, 4, 1, 128, 128, ("fixed", 1024), ("nvfp4",), 1.0, 4, 20.0, 20.0),
    "qwen3_4b": Spec("qwen3_4b", 16, 32, 8, 128, 128, ("fixed", 32768), ("nvfp4",), 1.0, 3, 10.0, 30.0),
    "qwen3_30b_a3b": Spec("qwen3_30b_a3b", 64, 32, 4, 128, 128, ("uniform", 8192, 131072),
                          ("nvfp4", "mxfp4"), 1.0, 3, 10.0, 30.0),
    "underflow": Spec("underflow", 4, 32, 8, 128, 128, ("fixed", 131072), ("nvfp4",), 0.05, 0),
    "mla": Spec("mla", 32, 128, 1, 576, 512, ("fixed", 16384), ("nvfp4",), 1.0, 6, 10.0, 30.0, mla=True),
}


def spec(name: str, **overrides) -> Spec:
    return dataclasses.replace(SPECS[name], **overrides) if overrides else SPECS[name]


def _mix(seed: int, kind: int, idx: int = 0) -> int:
    return (seed * 1_000_003 + kind * 100_003 + idx * 7919 + 12345) & 0x7FFF_FFFF_FFFF


def _gen(device, s: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(s)
    return g


class Workload:
    """One seeded instance of a Spec.  Keys and values are drawn per sequence
    on demand, so a single sequence can be re-drawn without the rest."""

    K_KIND, V_KIND, Q_KIND, CAL_K, CAL_Q, CAL_V = 1, 2, 3, 4, 5, 6

    def __init__(self, sp: Spec, seed: int = 0):
        self.spec, self.seed = sp, seed
        rng = np.random.default_rng(_mix(seed, 0))
        if sp.ctx[0] == "fixed":
            lens = np.full(sp.B, sp.ctx[1], np.int64)
        elif sp.ctx[0] == "uniform":
            lens = rng.integers(sp.ctx[1], sp.ctx[2] + 1, size=sp.B)
        else:
            lens = np.asarray(sp.ctx[1], np.int64)
            assert len(lens) == sp.B
        self.seq_lens = lens.astype(np.int32)
        self.cu_seqlens = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
        npages = (lens + PAGE_SLOTS - 1) // PAGE_SLOTS
        self.num_pages = int(npages.sum())
        self.max_pages = int(max(1, npages.max()))
        perm = rng.permutation(self.num_pages)
        self.block_table = np.zeros((sp.B, self.max_pages), np.int32)
        off = 0
        for b in range(sp.B):
            self.block_table[b, : npages[b]] = perm[off: off + npages[b]]
            off += npages[b]
        # outlier key channels: fixed per KV head
        self.out_chan = np.zeros((sp.H_kv, sp.n_outlier), np.int64)
        self.out_mult = np.ones((sp.H_kv, sp.n_outlier), np.float32)
        for h in range(sp.H_kv):
            if sp.n_outlier:
                self.out_chan[h] = rng.choice(sp.d_k, size=sp.n_outlier, replace=False)
                self.out_mult[h] = rng.uniform(sp.outlier_lo, sp.outlier_hi, size=sp.n_outlier)

    # ------------------------------------------------------------ pages
    def slot_mapping(self, b: int, t0: int = 0, t1: int | None = None) -> np.ndarray:
        """page * 64 + slot for tokens [t0, t1) of sequence b."""
        t1 = int(self.seq_lens[b]) if t1 is None else t1
        t = np.arange(t0, t1, dtype=np.int64)
        return self.block_table[b, t // PAGE_SLOTS].astype(np.int64) * PAGE_SLOTS + t % PAGE_SLOTS

    def slot_mapping_all(self) -> np.ndarray:
        return np.concatenate([self.slot_mapping(b) for b in range(self.spec.B)])

    # ------------------------------------------------------------ tensors
    def _keys_raw(self, n: int, s: int, device) -> torch.Tensor:
        sp = self.spec
        x = torch.randn((n, sp.H_kv, sp.d_k), generator=_gen(device, s), device=device, dtype=torch.float32)
        x = x * sp.key_std
        if sp.n_outlier:
            m = torch.ones((sp.H_kv, sp.d_k), dtype=torch.float32)
            for h in range(sp.H_kv):
                m[h, torch.from_numpy(self.out_chan[h])] = torch.from_numpy(self.out_mult[h])
            x = x * m.to(device)
        return x.to(torch.bfloat16)

    def keys(self, b: int, device="cpu", t0: int = 0, t1: int | None = None) -> torch.Tensor:
        """bf16 [t1 - t0, H_kv, d_k]; a token's key depends only on (seed, b, t)."""
        t1 = int(self.seq_lens[b]) if t1 is None else t1
        full = self._keys_raw(int(self.seq_lens[b]), _mix(self.seed, self.K_KIND, b), device)
        return full[t0:t1].contiguous()

    def values(self, b: int, device="cpu", t0: int = 0, t1: int | None = None) -> torch.Tensor:
        sp = self.spec
        t1 = int(self.seq_lens[b]) if t1 is None else t1
        if sp.mla:
            return self.keys(b, device, t0, t1)[..., : sp.d_v].contiguous()
        n = int(self.seq_lens[b])
        x = torch.randn((n, sp.H_kv, sp.d_v), generator=_gen(device, _mix(self.seed, self.V_KIND, b)),
                        device=device, dtype=torch.float32)
        return x[t0:t1].to(torch.bfloat16).contiguous()

    def queries(self, device="cpu", step: int = 0) -> torch.Tensor:
        sp = self.spec
        x = torch.randn((sp.B, sp.H_q, sp.d_k), generator=_gen(device, _mix(self.seed, self.Q_KIND, step)),
                        device=device, dtype=torch.float32)
        return x.to(torch.bfloat16)

    def all_keys(self, device="cpu") -> torch.Tensor:
        return torch.cat([self.keys(b, device) for b in range(self.spec.B)])

    def all_values(self, device="cpu") -> torch.Tensor:
        return torch.cat([self.values(b, device) for b in range(self.spec.B)])

    def calibration(self, device="cpu", n_tok: int = 1024, n_q: int = 64):
        """(k_cal [n_tok, H_kv, d_k], q_cal [n_q, H_q, d_k], v_cal [n_tok, H_kv, d_v]) bf16."""
        sp = self.spec
        s = self.seed + 1000
        k = self._keys_raw(n_tok, _mix(s, self.CAL_K), device)
        q = torch.randn((n_q, sp.H_q, sp.d_k), generator=_gen(device, _mix(s, self.CAL_Q)), device=device,
                        dtype=torch.float32).to(torch.bfloat16)
        if sp.mla:
            v = k[..., : sp.d_v].contiguous()
        else:
            v = torch.randn((n_tok, sp.H_kv, sp.d_v), generator=_gen(device, _mix(s, self.CAL_V)),
                            device=device, dtype=torch.float32).to(torch.bfloat16)
        return k, q, v
