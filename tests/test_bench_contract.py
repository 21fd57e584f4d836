"""bench.py's accounting and its reference arm, on the CPU.

The pooling stage's algorithmic bytes are pinned to a hand count for the 128K
INT8 workload (B1 Hq32 Hkv8 N131072 d128 bf16), term by term, so a dropped or
doubled term in the roofline's numerator fails here; the reference arm (the
float64 oracle on a bounded sample) must print one JSON line with the fields
the driver reads.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from synth import get_workload  # noqa: E402


def test_pool_bytes_hand_count_128k_int8():
    # the survey's algorithmic bytes of the pooling stage: one read of Q and K,
    # the block means and self-similarities, and with INT8 the codes and scales
    w = get_workload("llm_128k")
    q = 32 * 131072 * 128 * 2            # read Q (bf16)
    k = 8 * 131072 * 128 * 2             # read K
    means = (32 * 1024 + 8 * 2048) * (128 + 1) * 4   # block means and self-similarities
    q_codes = 32 * 131072 * 128 + 32 * 1024 * 4      # Q codes and their scales
    k_codes = 8 * 131072 * 128 + 8 * 2048 * 4        # K codes and their scales
    assert bench.pool_bytes(w) == q + k + means + q_codes + k_codes
    assert bench.pool_bytes(w) == 2_038_824_960
    # not counted: the second read of K and the float64 block sums of kbar
    assert bench.pool_extra_bytes(w) == 8 * 131072 * 128 * 2 + 2 * 8 * 2048 * 128 * 8


def test_attention_peak_weights_each_dtype():
    peaks = {"bf16_tflops_sustained": 1000.0, "bf16_tflops": 1200.0}
    w8 = get_workload("llm_128k")
    # equal flops in INT8 (2000) and fp16 (1000): 2 / (1/2000 + 1/1000)
    assert bench.attn_peak_tflops(w8, peaks, 10, 10) == pytest.approx(4000.0 / 3.0)
    assert bench.attn_peak_tflops(w8, peaks, 10, 10, key="bf16_tflops") == pytest.approx(1600.0)
    assert bench.attn_peak_tflops(get_workload("llm_32k"), peaks, 10, 10) == 1000.0


def test_pool_bytes_without_int8_is_one_read_plus_means():
    w = get_workload("llm_32k")
    assert bench.pool_bytes(w) == (32 + 8) * 32768 * 128 * 2 + (32 * 256 + 8 * 512) * 129 * 4


def test_dense_equivalent_ops_halved_when_causal():
    w = get_workload("llm_128k")
    assert bench.dense_equiv_ops(w) == 4.0 * 131072 ** 2 * 128 * 32 / 2
    t = get_workload("tiny")
    assert bench.dense_equiv_ops(t) == 4.0 * 1024 ** 2 * 64 * 1


def test_visible_blocks_causal_count():
    # causal: query block i (128 rows) sees key blocks 0 .. 2i+1 (64 rows each)
    w = get_workload("llm_32k").replace(N=1024, Hq=1, Hkv=1)
    assert bench._visible_blocks(w) == sum(2 * i + 2 for i in range(8))


def test_select_work_counts_only_non_fix_rows():
    # causal, b_q 128, b_k 64, N 512: query blocks see 2, 4, 6, 8 key blocks.
    # Head 0's last query block and head 1's first (s exactly theta: Eq. 9's
    # strict <) are not fix blocks, so S_hat is needed for 8 + 2 visible pairs.
    w = get_workload("llm_32k", N=512, Hq=2, Hkv=1)
    s_q = np.array([[[0.1, 0.1, 0.1, 0.9]], [[0.5, 0.2, 0.4999, 0.1]]]).reshape(1, 2, 4)
    work = bench.select_work(w, s_q, kept=17, theta=0.5)
    assert work["flops"] == 2 * 128 * (8 + 2)
    assert work["nonfix_rows"] == 2 and work["rows"] == 8
    means = 4 * (2 * 4 * 129 + 1 * 8 * 129)      # block means + self-similarities read
    writes = 2 * 4 * 8 + 4 * 17 + 4 * 2 * 4      # mask, kept skip-list entries, counts
    assert work["bytes"] == means + writes
    # every block a fix block: no flops, bound by the bytes
    r = bench.select_roofline(bench.select_work(w, s_q, 17, theta=2.0), 1e-3, 74.4, 6550.4)
    assert r["bound"] == "hbm" and r["flops_per_launch"] == 0


def test_fp32_peak_from_unit_counts():
    assert bench.fp32_peak_tflops({"sm_max_mhz": 1965.0}) == pytest.approx(74.45, rel=1e-3)


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "0", "--ref-tiles", "2"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TOPS" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["higher_is_better"] is True and d["n_gpus"] == 1
    # the same config object as the native arm, and a time it actually measured
    w = get_workload("tiny")
    from synth import make_qkv
    assert d["config"] == bench.workload_config(w, 1, bench._bytes(make_qkv(w)))
    assert d["ms_per_step"] * d["steps"] < 600e3


def test_profiled_traffic_only_for_the_profiled_workload(tmp_path):
    import hashlib
    sha = hashlib.sha256(open(bench.ATTN_SRC, "rb").read()).hexdigest()
    p = tmp_path / "summary.md"
    p.write_text(f"kernel_source_sha256: {sha}\ndram_bytes_per_launch: 2.25e9\n"
                 "dram_bytes_workload: llm_128k N=131072\n")
    assert bench.profiled_traffic("llm_128k", 131072, str(p)) == 2.25e9
    # another workload, another length, another kernel source: no figure
    assert bench.profiled_traffic("image_dit", 4608, str(p)) is None
    assert bench.profiled_traffic("llm_128k", 32768, str(p)) is None
    p.write_text("kernel_source_sha256: 00\ndram_bytes_per_launch: 2.25e9\n"
                 "dram_bytes_workload: llm_128k N=131072\n")
    assert bench.profiled_traffic("llm_128k", 131072, str(p)) is None
