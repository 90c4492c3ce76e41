"""Benchmark of the FP4 paged decode-attention step on B200.

One step = one decode step of a serving batch through the whole hot path, in
one bdfp4_decode_step call: append-quantize each sequence's newest key and its
open value block (the newest token and the earlier tokens of the same
16/32-slot block, kept in bf16 on the device) into the paged FP4 cache, then
decode attention for one query token per sequence (query transform +
dual-residual FP4, paged tile fetch, QK^T, transposed softmax with fused
underflow-aware P quantization, P.V, split merge).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config qwen3_30b_a3b]
                  [--fmt nvfp4|mxfp4] [--impl ours|reference] [--extra qwen3_4b,...]

`value` is KV tokens per second (sum of context lengths per step / step
time), device-timed with CUDA events; under torchrun each rank runs its own
batch (weak scaling) and rank 0 reports the whole job over the slowest rank.
Each timed block is exactly K steps between one CUDA event pair; blocks are
repeated until they cover at least --min-region seconds (so the clock record
holds many samples) and the median block is reported.  The default workload
is the largest single-GPU one (Qwen3-30B-A3B-shaped); --extra adds decode
figures of other workloads under "extra".
`--impl reference` times the CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

CONFIG_TEXT = {
    "qwen3_4b": "Qwen3-4B-shaped layer decode: B=16, 32 query / 8 KV heads, d=128, context 32768 each, page 64, "
                "shuffled block table",
    "qwen3_30b_a3b": "Qwen3-30B-A3B-shaped layer decode: B=64, 32 query / 4 KV heads, d=128, context U[8192,131072], "
                     "page 64",
    "underflow": "long-context underflow stress: B=4, 32/8 heads, d=128, context 131072, keys N(0,0.05^2)",
    "mla": "MLA-shaped decode: B=32, 128 heads over one latent head, d_k=576, d_v=512, context 16384",
    "tiny": "tiny decode: B=1, 4/1 heads, d=128, context 1024",
}


def bf16_algorithmic_bytes(sp, seq_lens) -> int:
    """bf16 K and V + block table + Q and O in bf16 for one decode of the comparator."""
    tok = int(np.sum(seq_lens))
    pages = int(np.sum((np.asarray(seq_lens) + 63) // 64))
    return tok * sp.H_kv * 2 * (sp.d_k + sp.d_v) + pages * 4 + sp.B * sp.H_q * (sp.d_k + sp.d_v) * 2


def algorithmic_bytes(sp, seq_lens, fmt: int, T_q: int = 1) -> int:
    """Packed KV + scales + block table + Q and O in bf16 for one decode (T_q query
    tokens per sequence: the cache is read once, Q and O T_q times)."""
    beta = 16 if fmt == 0 else 32
    tok = int(np.sum(seq_lens))
    per_tok = sp.H_kv * (sp.d_k // 2 + sp.d_k // beta + sp.d_v // 2 + sp.d_v // beta)
    pages = int(np.sum((np.asarray(seq_lens) + 63) // 64))
    return tok * per_tok + pages * 4 + sp.B * T_q * sp.H_q * (sp.d_k + sp.d_v) * 2


# sources of each tensor-core decode kernel: its file and the headers it includes
DECODE_SOURCES = {
    128: ("decode_tc.cu", "tc_ptx.cuh", "bdfp4_device.cuh", "quant_device.cuh", "decode_common.cuh",
          "append_device.cuh", "prob_scale.cuh"),
    576: ("decode_mla_tc.cu", "tc_ptx.cuh", "bdfp4_device.cuh", "quant_device.cuh", "decode_common.cuh",
          "append_device.cuh", "prob_scale.cuh"),
}


def _strip_comments(src: str) -> str:
    """C/C++ source without its // and /* */ comments (string literals kept as they are)."""
    import re
    pat = re.compile(r'"(?:\\.|[^"\\])*"|//[^\n]*|/\*.*?\*/', re.S)
    return pat.sub(lambda m: m.group(0) if m.group(0).startswith('"') else "", src)


def decode_source_hash(d_k: int = 128) -> str:
    """sha256 over the sources of the tensor-core decode kernel for head dim d_k, comments
    stripped: a recorded capture stays valid across comment edits, not across code edits."""
    import hashlib
    h = hashlib.sha256()
    for name in DECODE_SOURCES[d_k]:
        with open(os.path.join(ROOT, "fp4_kv_cache_quant_b200", "csrc", name), encoding="utf-8") as f:
            h.update(_strip_comments(f.read()).encode())
    return h.hexdigest()


def slowest_rank(times, device):
    """Each of the per-rank device times (seconds) replaced by its maximum over the
    process group's ranks: a replica job is as fast as its slowest rank."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(times, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def timed_blocks(fn, steps: int, stream, min_region_s: float, max_blocks: int = 1000) -> list:
    """Seconds of blocks of exactly `steps` back-to-back calls of fn, each block
    between one CUDA event pair on `stream` with a synchronize after it; blocks
    repeat until together they cover min_region_s (at most max_blocks)."""
    import torch
    times = []
    while True:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) / 1e3)
        if sum(times) >= min_region_s or len(times) >= max_blocks:
            return times


def median_step(times, steps: int) -> float:
    return statistics.median(times) / steps


class ClockSampler:
    """SM clock and clock-event (throttle) reasons polled through NVML in a
    background thread during the timed region (read-only queries)."""

    def __init__(self, gpu_index: int, period_s: float = 0.002):
        self.gpu, self.period = gpu_index, period_s
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = None
        self._thread = None

    def start(self):
        import threading
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            try:   # NVML enumerates every GPU; match the CUDA device by PCI bus id
                pr = torch.cuda.get_device_properties(self.gpu)
                h = pynvml.nvmlDeviceGetHandleByPciBusId(
                    f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0")
            except Exception:  # noqa: BLE001
                h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001
            self.error = str(e)
            return
        self._stop = threading.Event()

        def poll():
            while not self._stop.is_set():
                try:
                    self.samples.append(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                    self.reasons |= pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                except Exception:  # noqa: BLE001
                    pass
                self._stop.wait(self.period)

        self._thread = threading.Thread(target=poll, daemon=True)
        self._thread.start()

    def stop(self) -> dict:
        if self._thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [getattr(self, "error", "nvml unavailable")]}
        self._stop.set()
        self._thread.join()
        import pynvml
        names = {pynvml.nvmlClocksEventReasonHwSlowdown: "hw_slowdown",
                 pynvml.nvmlClocksEventReasonHwThermalSlowdown: "hw_thermal_slowdown",
                 pynvml.nvmlClocksEventReasonSwThermalSlowdown: "sw_thermal_slowdown",
                 pynvml.nvmlClocksEventReasonSwPowerCap: "sw_power_cap",
                 pynvml.nvmlClocksEventReasonHwPowerBrakeSlowdown: "hw_power_brake_slowdown"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(v for k, v in names.items() if self.reasons & k), "samples": len(self.samples)}


def setup_ours(sp, fmt, rank, device, with_bf16: bool = False):
    """Untimed: draw the workload on the GPU, calibrate, prefill-quantize the
    cache (and, with_bf16, fill the BF16-KV comparator's pages from the same
    keys and values)."""
    import torch

    from fp4_kv_cache_quant_b200 import bdfp4
    from fp4_kv_cache_quant_b200.workloads import Workload

    wl = Workload(sp, seed=rank)
    beta = 16 if fmt == 0 else 32
    kc, qc, vc = wl.calibration(device)
    kv = bdfp4.bdfp4_calibrate(kc, qc, vc, sp.H_q, sp.H_kv)
    cache = bdfp4.FP4Cache.empty(wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    bcache = bdfp4.BF16Cache.empty(wl.num_pages, sp.H_kv, sp.d_k, device=device) if with_bf16 else None
    # decode-step inputs: the newest token of each sequence and the open value block it joins
    new_k = torch.zeros((sp.B, sp.H_kv, sp.d_k), dtype=torch.bfloat16, device=device)
    new_v = torch.zeros((sp.B, sp.H_kv, sp.d_v), dtype=torch.bfloat16, device=device)
    v_open = torch.zeros((sp.B, beta, sp.H_kv, sp.d_v), dtype=torch.bfloat16, device=device)
    q_bytes = 0
    t_quant, quant_bytes = 0.0, 0
    for b in range(sp.B):
        n = int(wl.seq_lens[b])
        k = wl.keys(b, device)
        v = wl.values(b, device)
        sm = torch.from_numpy(wl.slot_mapping(b)).to(device)
        if bcache is not None:
            bdfp4.bdfp4_bf16_append(k, v, sm, bcache, dev_status=status)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        bdfp4.bdfp4_quantize_kv(k, v, sm, kv, cache, dev_status=status)
        e1.record()
        torch.cuda.synchronize()
        t_quant += e0.elapsed_time(e1) / 1e3
        quant_bytes += (k.numel() + v.numel()) * 2 + n * sp.H_kv * (sp.d_k // 2 + sp.d_k // beta + sp.d_v // 2 +
                                                                  sp.d_v // beta)
        if n > 0:
            last = (n - 1) % beta   # row of the newest token in its open value block
            new_k[b] = k[n - 1]
            new_v[b] = v[n - 1]
            v_open[b, :last] = v[n - 1 - last:n - 1]
        del k, v
    assert int(status.item()) == 0
    q = wl.queries(device)
    bt = torch.from_numpy(wl.block_table).to(device)
    sl = torch.from_numpy(wl.seq_lens).to(device)
    num_sms = torch.cuda.get_device_properties(device).multi_processor_count
    chunk = bdfp4.bdfp4_decode_plan_for(wl.seq_lens, sp.H_q, sp.H_kv, sp.d_k, sp.d_v, num_sms)
    ws = bdfp4.workspace_for(sp.B, sp.H_q, sp.d_v, wl.max_pages, chunk, device=device)
    out = torch.empty((sp.B, sp.H_q, sp.d_v), dtype=torch.bfloat16, device=device)
    return dict(wl=wl, kv=kv, cache=cache, status=status, new_k=new_k, new_v=new_v, v_open=v_open, q=q, bt=bt,
                sl=sl, chunk=chunk, ws=ws, out=out, quant_gbs=quant_bytes / t_quant / 1e9, num_sms=num_sms,
                bcache=bcache)


def _peak():
    peaks_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(peaks_path):
        return json.load(open(peaks_path))["hbm_gbs"], "measured"
    return 6650.0, "fallback"


def measure_extra(args, name, fmt, flags, device, stream) -> dict:
    """Decode figures of a second workload in the same run: the step, the decode
    call and the BF16-KV comparator, each timed like the headline."""
    import torch

    from fp4_kv_cache_quant_b200 import bdfp4
    from fp4_kv_cache_quant_b200.workloads import spec
    sp = spec(name)
    S = setup_ours(sp, fmt, 0, device, with_bf16=not args.no_bf16 and sp.d_k == 128)

    def step():
        bdfp4.bdfp4_decode_step(S["q"], S["new_k"], S["new_v"], S["v_open"], S["cache"], S["bt"], S["sl"], S["kv"],
                                sp.sm_scale, S["chunk"], S["ws"], S["out"], flags=flags, dev_status=S["status"])

    def decode_only():
        bdfp4.bdfp4_decode(S["q"], S["cache"], S["bt"], S["sl"], S["kv"], sp.sm_scale, S["chunk"], S["ws"], S["out"],
                           flags=flags, dev_status=S["status"])

    for _ in range(max(args.warmup, 3)):
        step()
        decode_only()
    step_s = median_step(timed_blocks(step, args.steps, stream, args.min_region), args.steps)
    dec_s = median_step(timed_blocks(decode_only, args.steps, stream, args.min_region), args.steps)
    assert int(S["status"].item()) == 0, "device status set"
    tokens = float(np.sum(S["wl"].seq_lens))
    alg = algorithmic_bytes(sp, S["wl"].seq_lens, fmt)
    peak, _ = _peak()
    r = {"workload": CONFIG_TEXT[name], "name": name, "fmt": "nvfp4" if fmt == 0 else "mxfp4",
         "chunk_tiles": S["chunk"], "kv_tokens_per_s": tokens / step_s, "ms_per_step": step_s * 1e3,
         "decode_us": dec_s * 1e6, "hbm_gbs": alg / dec_s / 1e9, "frac": alg / dec_s / 1e9 / peak,
         "algorithmic_bytes_per_launch": alg}
    if S["bcache"] is not None:
        bout = torch.empty_like(S["out"])

        def bf16_decode():
            bdfp4.bdfp4_bf16_decode(S["q"], S["bcache"], S["bt"], S["sl"], sp.sm_scale, S["chunk"], S["ws"], bout,
                                    dev_status=S["status"])

        for _ in range(max(args.warmup, 3)):
            bf16_decode()
        bf16_s = median_step(timed_blocks(bf16_decode, args.steps, stream, args.min_region), args.steps)
        r["bf16_kv"] = {"decode_us": bf16_s * 1e6, "frac": bf16_algorithmic_bytes(sp, S["wl"].seq_lens) / bf16_s / 1e9
                        / peak, "fp4_decode_speedup": bf16_s / dec_s}
    if args.multi_tokens > 1 and sp.d_k == 128:
        # several query tokens per sequence (the newest T_q, causal), one bdfp4_decode_multi call
        T = args.multi_tokens
        g = torch.Generator(device=device)
        g.manual_seed(7)
        qm = torch.randn((sp.B, T, sp.H_q, sp.d_k), generator=g, device=device).to(torch.bfloat16)
        outm = torch.empty((sp.B, T, sp.H_q, sp.d_v), dtype=torch.bfloat16, device=device)
        cm = bdfp4.bdfp4_decode_multi_plan(S["wl"].seq_lens, T, sp.H_q, sp.H_kv, sp.d_k, sp.d_v, S["num_sms"])
        wsm = bdfp4.workspace_for(sp.B * T, sp.H_q, sp.d_v, S["wl"].max_pages, cm, device=device)

        def multi():
            bdfp4.bdfp4_decode_multi(qm, S["cache"], S["bt"], S["sl"], S["kv"], sp.sm_scale, cm, wsm, outm,
                                     flags=flags, dev_status=S["status"])

        for _ in range(max(args.warmup, 3)):
            multi()
        mt_s = median_step(timed_blocks(multi, args.steps, stream, args.min_region), args.steps)
        assert int(S["status"].item()) == 0, "device status set"
        m_alg = algorithmic_bytes(sp, S["wl"].seq_lens, fmt, T)
        r["multi_token"] = {"T_q": T, "kernel": "bdfp4_decode_multi (query images + tensor-core decode + merge)"
                            if sp.H_q // sp.H_kv * T <= 16 else "bdfp4_decode_multi (CUDA-core decode + merge)",
                            "chunk_tiles": cm, "decode_us": mt_s * 1e6, "kv_tokens_per_s": tokens / mt_s,
                            "query_tokens_per_s": sp.B * T / mt_s, "hbm_gbs": m_alg / mt_s / 1e9,
                            "frac": m_alg / mt_s / 1e9 / peak, "algorithmic_bytes_per_launch": m_alg}
    return r


def run_ours(args, sp, fmt):
    import torch
    import torch.distributed as dist

    from fp4_kv_cache_quant_b200 import bdfp4

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)

    S = setup_ours(sp, fmt, rank, device, with_bf16=not args.no_bf16 and sp.d_k == 128)
    wl, kv, cache = S["wl"], S["kv"], S["cache"]
    stream = torch.cuda.current_stream(device)

    flags = bdfp4.FLAG_DYNAMIC_ALPHA if args.dynamic_alpha else 0

    def step(q, k_new, v_new, out=None):
        # one call: append each sequence's newest token (key, and the open value
        # block it joins) into the FP4 cache, then decode over the updated cache
        bdfp4.bdfp4_decode_step(q, k_new, v_new, S["v_open"], cache, S["bt"], S["sl"], kv, sp.sm_scale, S["chunk"],
                                S["ws"], S["out"] if out is None else out, flags=flags, dev_status=S["status"])

    def decode_only():
        bdfp4.bdfp4_decode(S["q"], cache, S["bt"], S["sl"], kv, sp.sm_scale, S["chunk"], S["ws"], S["out"],
                           flags=flags, dev_status=S["status"])

    for _ in range(max(args.warmup, 3)):
        step(S["q"], S["new_k"], S["new_v"])
        decode_only()   # warms the decode-only call timed for the roofline as well
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    # the steps: blocks of exactly K steps, repeated until they cover --min-region seconds
    step_blocks = timed_blocks(lambda: step(S["q"], S["new_k"], S["new_v"]), args.steps, stream, args.min_region)
    # the decode on its own (query images, decode kernel, merge) for the roofline: blocks of
    # K back-to-back calls on the same stream right after the steps, still under the clock sampler
    dec_blocks = timed_blocks(decode_only, args.steps, stream, args.min_region)
    clk = clocks.stop()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    step_s = median_step(step_blocks, args.steps)
    dec_s = median_step(dec_blocks, args.steps)
    assert int(S["status"].item()) == 0, "device status set"

    # the BF16-KV comparator on the same workload: decode calls timed alone
    bf16_s = 0.0
    if S["bcache"] is not None:
        bout = torch.empty_like(S["out"])

        def bf16_decode():
            bdfp4.bdfp4_bf16_decode(S["q"], S["bcache"], S["bt"], S["sl"], sp.sm_scale, S["chunk"], S["ws"], bout,
                                    dev_status=S["status"])

        for _ in range(max(args.warmup, 3)):
            bf16_decode()
        torch.cuda.synchronize()
        # timed like the FP4 decode calls
        bf16_s = median_step(timed_blocks(bf16_decode, args.steps, stream, args.min_region), args.steps)
        assert int(S["status"].item()) == 0, "device status set"

    # end to end through the C ABI with host buffers: every step uploads its q and new keys
    # and values from pinned host memory and reads its output back.  The copies run on a
    # second stream with two buffer sets, so a step's upload overlaps the previous step and
    # its read-back the next one, as a serving loop would; the timed region opens before
    # the first timed upload and closes after the last read-back.
    q_host = S["q"].cpu().pin_memory()
    tk_host = S["new_k"].cpu().pin_memory()
    tv_host = S["new_v"].cpu().pin_memory()
    out_host = [torch.empty(S["out"].shape, dtype=S["out"].dtype).pin_memory() for _ in range(2)]
    q_dev = [torch.empty_like(S["q"]) for _ in range(2)]
    k_dev = [torch.empty_like(S["new_k"]) for _ in range(2)]
    v_dev = [torch.empty_like(S["new_v"]) for _ in range(2)]
    o_dev = [torch.empty_like(S["out"]) for _ in range(2)]
    cs = torch.cuda.Stream(device)
    up = [torch.cuda.Event() for _ in range(2)]     # inputs of buffer set b uploaded
    done = [torch.cuda.Event() for _ in range(2)]   # the step on set b finished
    down = [torch.cuda.Event() for _ in range(2)]   # set b's output read back

    def upload(i):
        b = i & 1
        with torch.cuda.stream(cs):
            if i >= 2:
                cs.wait_event(done[b])   # the step that last read these inputs has finished
            q_dev[b].copy_(q_host, non_blocking=True)
            k_dev[b].copy_(tk_host, non_blocking=True)
            v_dev[b].copy_(tv_host, non_blocking=True)
            up[b].record(cs)

    def run_e2e(n):
        upload(0)
        for i in range(n):
            b = i & 1
            stream.wait_event(up[b])
            if i >= 2:
                stream.wait_event(down[b])   # the output buffer of step i - 2 was read back
            step(q_dev[b], k_dev[b], v_dev[b], o_dev[b])
            done[b].record(stream)
            if i + 1 < n:
                upload(i + 1)
            with torch.cuda.stream(cs):
                cs.wait_event(done[b])
                out_host[b].copy_(o_dev[b], non_blocking=True)
                down[b].record(cs)
        stream.wait_event(down[(n - 1) & 1])

    run_e2e(3)
    torch.cuda.synchronize()
    e2e_steps = max(3, args.steps // 2)
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    cs.wait_event(s0)
    run_e2e(e2e_steps)
    s1.record(stream)
    torch.cuda.synchronize()
    e2e_s = s0.elapsed_time(s1) / 1e3 / e2e_steps
    assert int(S["status"].item()) == 0, "device status set"

    tokens = float(np.sum(wl.seq_lens))
    if world > 1:
        step_s, dec_s, e2e_s, bf16_s = slowest_rank([step_s, dec_s, e2e_s, bf16_s], device)
        tokens *= world
    # one prologue (append + query images) and the tensor-core decode (d = 128), or the
    # append and one CUDA-core decode; merge when a sequence can split
    launches_per_step = 2 + (1 if S["chunk"] < (wl.max_pages * 64 + 127) // 128 else 0)
    alg = algorithmic_bytes(sp, wl.seq_lens, fmt)
    peak, peak_src = _peak()
    traffic = None
    tr_path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if os.path.exists(tr_path):
        rec = json.load(open(tr_path)).get(f"{args.config}_{args.fmt}" + ("_dynamic" if args.dynamic_alpha and fmt == 0 else ""))
        # the counters describe the kernel as captured: null once its sources changed
        if rec and rec.get("source_sha256") == decode_source_hash(sp.d_k):
            traffic = rec.get("bytes_per_launch")
    result = {
        "metric": "FP4 paged decode-attn KV tokens/s",
        "value": tokens / step_s,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(args.warmup, 3),
        "ms_per_step": step_s * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4" if fmt == 0 else "mxfp4",
        "data": "synthetic (seeded N(0,1) bf16 with outlier key channels; calibrated smoothing)",
        "config": {"workload": CONFIG_TEXT[args.config], "name": args.config, "fmt": args.fmt,
                   "global_batch": sp.B * world, "seq_len": int(np.max(wl.seq_lens)),
                   "kv_tokens_per_step_per_gpu": int(tokens / world), "chunk_tiles": S["chunk"],
                   "parallelism": f"replicas x{world} (no data-path collective)",
                   "l2": f"inputs larger than L2 (FP4 cache {cache.nbytes() / 1e6:.0f} MB per GPU)",
                   "timing": f"median of {len(step_blocks)} blocks of exactly {args.steps} steps (each block one "
                             f"CUDA event pair), {sum(step_blocks):.3f} s of steps timed",
                   "accumulate": "fp32",
                   "probability_prescale": "dynamic per tile" if args.dynamic_alpha else "static 2^11"},
        "hbm_gbs": alg / dec_s / 1e9,
        "decode_us": dec_s * 1e6,
        "quantize_prefill_gbs": S["quant_gbs"],
        "roofline": {"bound": "hbm", "achieved": alg / dec_s / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": alg / dec_s / 1e9 / peak, "traffic": traffic,
                     "kernel": ("bdfp4_decode calls (" +
                                ("prep_query_kernel, decode_tc_kernel" if sp.d_k == 128 else
                                 "prep_mla_kernel, decode_mla_tc_kernel") +
                                ", merge_splits_kernel): median of blocks of K back-to-back calls right after the "
                                "step blocks, one event pair per block"),
                     "peak_source": f"{peak_src} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                     "algorithmic_bytes_per_launch": alg},
        "e2e": {"value": tokens / e2e_s, "unit": "tokens/s",
                "h2d_bytes_per_step": int(q_host.numel() * 2 + tk_host.numel() * 2 + tv_host.numel() * 2),
                "d2h_bytes_per_step": int(out_host[0].numel() * 2),
                "overlap": "uploads and read-backs on a second stream, double-buffered"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    if bf16_s > 0:
        b_alg = bf16_algorithmic_bytes(sp, wl.seq_lens)
        result["bf16_kv"] = {
            "kernel": "decode_bf16_kernel + merge_splits_kernel (tcgen05 kind::f16, same tiles and pipeline)",
            "decode_us": bf16_s * 1e6, "kv_tokens_per_s": tokens / bf16_s, "hbm_gbs": b_alg / bf16_s / 1e9,
            "frac": b_alg / bf16_s / 1e9 / peak, "algorithmic_bytes_per_launch": b_alg,
            "fp4_decode_speedup": bf16_s / dec_s}
    extra_names = [n for n in (args.extra.split(",") if args.extra else []) if n and n != args.config]
    if rank == 0 and world == 1 and extra_names:
        del S, cache, kv, wl
        torch.cuda.empty_cache()
        result["extra"] = [measure_extra(args, n, fmt, flags, device, stream) for n in extra_names]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(sp, fmt, budget_s=args.cpu_budget, flags=flags)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def cpu_baseline(sp, fmt, budget_s: float = 15.0, seed: int = 0, flags: int = 0) -> dict:
    """The oracle as it stands, timed on this host's cores on a bounded sample
    of the same workload: decode (with the tail append) of the first few
    sequences; prefill of the sample is untimed setup."""
    import oracle
    from fp4_kv_cache_quant_b200.workloads import Workload

    wl = Workload(sp, seed=seed)
    beta = 16 if fmt == 0 else 32
    kc, qc, vc = wl.calibration("cpu")
    smooth, kg, vg = oracle.calibrate(kc, qc, vc, sp.H_q, sp.H_kv)
    q_all = wl.queries("cpu")
    done_tokens, elapsed, nseq = 0, 0.0, 0
    for b in range(sp.B):
        n = int(wl.seq_lens[b])
        k, v = wl.keys(b), wl.values(b)
        sm = wl.slot_mapping(b)
        cache = oracle.empty_cache(wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt)
        oracle.quantize_kv(k, v, sm, cache, sp.H_kv, fmt, smooth, kg, vg, wl.num_pages)
        r = ((n - 1) % beta) + 1
        t0 = time.perf_counter()
        oracle.quantize_kv(k[n - r:], v[n - r:], sm[n - r:], cache, sp.H_kv, fmt, smooth, kg, vg, wl.num_pages)
        oracle.decode(q_all[b:b + 1], cache, wl.block_table[b:b + 1], wl.seq_lens[b:b + 1], sp.H_kv, sp.d_v, fmt,
                      smooth, kg, vg, sp.sm_scale, 1 << 20, wl.num_pages, flags=flags)
        elapsed += time.perf_counter() - t0
        done_tokens += n
        nseq += 1
        if elapsed >= budget_s:
            break
    return {"value": done_tokens / elapsed, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{nseq} of {sp.B} sequences ({done_tokens} KV tokens, all heads): tail append + decode, "
                      f"{elapsed:.1f} s"}


def run_reference(args, sp, fmt):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from fp4_kv_cache_quant_b200.workloads import Workload

    wl = Workload(sp, seed=0)
    beta = 16 if fmt == 0 else 32
    kc, qc, vc = wl.calibration("cpu")
    smooth, kg, vg = oracle.calibrate(kc, qc, vc, sp.H_q, sp.H_kv)
    q_all = wl.queries("cpu")
    # bounded sample per step: one sequence, its tail append and its decode
    b = 0
    n = int(wl.seq_lens[b])
    k, v = wl.keys(b), wl.values(b)
    sm = wl.slot_mapping(b)
    cache = oracle.empty_cache(wl.num_pages, sp.H_kv, sp.d_k, sp.d_v, fmt)
    oracle.quantize_kv(k, v, sm, cache, sp.H_kv, fmt, smooth, kg, vg, wl.num_pages)
    r = ((n - 1) % beta) + 1
    flags = oracle.FLAG_DYNAMIC_ALPHA if args.dynamic_alpha else 0

    def step():
        oracle.quantize_kv(k[n - r:], v[n - r:], sm[n - r:], cache, sp.H_kv, fmt, smooth, kg, vg, wl.num_pages)
        oracle.decode(q_all[b:b + 1], cache, wl.block_table[b:b + 1], wl.seq_lens[b:b + 1], sp.H_kv, sp.d_v, fmt,
                      smooth, kg, vg, sp.sm_scale, 1 << 20, wl.num_pages, flags=flags)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = (time.perf_counter() - t0) / args.steps
    val = n / el
    print(json.dumps({
        "impl": "reference", "metric": "FP4 paged decode-attn KV tokens/s", "value": val, "unit": "tokens/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": CONFIG_TEXT[args.config], "name": args.config, "fmt": args.fmt,
                   "probability_prescale": "dynamic per tile" if args.dynamic_alpha else "static 2^11"},
        "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"sequence 0 of {sp.B} ({n} KV tokens, all heads) per step: tail append + decode"},
        "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="qwen3_30b_a3b", choices=list(CONFIG_TEXT))
    ap.add_argument("--extra", default="qwen3_4b",
                    help="comma-separated workloads whose decode figures go under \"extra\" (N = 1 only)")
    ap.add_argument("--multi-tokens", type=int, default=4,
                    help="query tokens per sequence of the multi-token decode figure under extra (1: none)")
    ap.add_argument("--batch", type=int, default=0,
                    help="sequences per GPU instead of the workload's batch (small profiling captures)")
    ap.add_argument("--min-region", type=float, default=0.5,
                    help="seconds the repeated blocks of K timed steps cover at least")
    ap.add_argument("--fmt", default="nvfp4", choices=["nvfp4", "mxfp4"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-bf16", action="store_true", help="skip the BF16-KV comparator")
    ap.add_argument("--dynamic-alpha", action="store_true",
                    help="the per-tile probability pre-scale variant (NVFP4)")
    args = ap.parse_args()
    from fp4_kv_cache_quant_b200.workloads import spec
    sp = spec(args.config, **({"B": args.batch} if args.batch > 0 else {}))
    fmt = 0 if args.fmt == "nvfp4" else 1
    if args.impl == "reference":
        run_reference(args, sp, fmt)
    else:
        run_ours(args, sp, fmt)


if __name__ == "__main__":
    main()
