"""Host-side pieces of bench.py (CPU): the algorithmic byte counts the roofline
divides by, worked out by hand from the cache layout, and the reference arm's
JSON line."""
import json
import os
import subprocess
import sys

import numpy as np

import bench
from fp4_kv_cache_quant_b200.workloads import spec

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_algorithmic_bytes_hand_values():
    # Qwen3-4B-shaped: 16 sequences of 32768 tokens, 8 KV heads, d = 128.
    # Per token and KV head: 64 B K nibbles + 8 B K scales + 64 B V nibbles + 8 B V scales
    # (NVFP4, 16-element blocks) = 144 B; MXFP4 (32-element blocks) 136 B.  Plus 4 B per
    # page of block table (16 x 512 pages) and bf16 Q and O (16 x 32 heads x 256 B).
    sp = spec("qwen3_4b")
    sl = np.full(16, 32768)
    tables, qo = 16 * 512 * 4, 16 * 32 * (128 + 128) * 2
    assert bench.algorithmic_bytes(sp, sl, 0) == 524288 * 8 * 144 + tables + qo == 604274688
    assert bench.algorithmic_bytes(sp, sl, 1) == 524288 * 8 * 136 + tables + qo
    # BF16 pages: 2 x (128 + 128) B per token and KV head
    assert bench.bf16_algorithmic_bytes(sp, sl) == 524288 * 8 * 512 + tables + qo
    # MLA: one latent head, K 576 (288 B + 36 B scales), V 512 (256 B + 32 B scales) = 612 B
    sp = spec("mla", B=2)
    sl = np.array([16384, 100])
    pages = 256 + 2
    assert bench.algorithmic_bytes(sp, sl, 0) == 16484 * 612 + pages * 4 + 2 * 128 * (576 + 512) * 2


def test_reference_arm_json_line():
    """bench.py --impl reference times the oracle and prints one JSON line with
    the contract's keys (the driver parses it)."""
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                          "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "tokens/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def test_reference_arm_under_torchrun_prints_once():
    """Launched as the driver launches it for N = 2: rank 0 alone runs the
    reference arm and prints its line; the other rank exits 0 without work."""
    import socket
    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        port = sock.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--config", "tiny", "--steps", "1", "--warmup", "0", "--gpus", "2"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(l) for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1 and lines[0]["impl"] == "reference" and lines[0]["n_gpus"] == 2


def test_source_hash_ignores_comments_only():
    """The traffic records are keyed by a hash of the decode sources without comments: a comment
    edit keeps a capture valid, a code edit (even inside a string literal) does not."""
    import bench
    src = 'int a = 1; // note\n/* block\n note */ asm("mov.b32 %0, 1; // kept");\n'
    out = bench._strip_comments(src)
    assert "note" not in out and "int a = 1;" in out and '"mov.b32 %0, 1; // kept"' in out
    assert bench._strip_comments(src.replace("// note", "// other")) == out
    assert bench._strip_comments(src.replace("a = 1", "a = 2")) != out
