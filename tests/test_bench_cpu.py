"""The benchmark's host-side contract, checked without a GPU.

- The algorithmic byte counts that every GB/s figure divides by, pinned to the per-(sequence,
  head) budget of the decode step written out by hand: the fp32 state read once and written
  once, v and z, the two fp32 gates, the output row, and q and k once per key head.
- The reference arm (the fp64 oracle on the host cores) prints one JSON line that carries the
  fields the product arm's line carries, and describes itself as a host run.
- The product arm never falls back to the host: without a CUDA device it exits with an error.
"""
import json
import os
import subprocess
import sys

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run_bench(*args, timeout=300):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, timeout=timeout, cwd=ROOT)


def test_decode_bytes_qwen35_batch32():
    # 32 sequences x 16 value heads x (131,072 state + 256 v + 256 z + 8 gates + 256 out)
    # + 32 sequences x 16 key heads x (256 q + 256 k), bf16 rows, fp32 state.
    per_value_head = 128 * 128 * 4 * 2 + 128 * 2 + 128 * 2 + 8 + 128 * 2
    per_key_head = 128 * 2 * 2
    want = 32 * 16 * per_value_head + 32 * 16 * per_key_head
    assert want == 67_768_320
    assert bench.decode_bytes_per_layer_step(32, 16, 16, 128) == want


def test_prefill_flops_per_token_head():
    # Chunk 64, d 128: KK^T, QK^T, U, W, P Delta at 2 C d (16,384) each, W S^T, Q S^T and
    # the state update at 2 d^2 (32,768) each; under GVA (two value heads per key head)
    # KK^T and QK^T are counted once per key head.
    assert bench.prefill_flops_per_token_head(64, 128) == 5 * 16_384 + 3 * 32_768 == 180_224
    assert bench.prefill_flops_per_token_head(64, 128, 2) == 4 * 16_384 + 3 * 32_768 == 163_840


def test_attn_decode_bytes_qwen36():
    # 64 sequences x 2 key/value heads x (4096 + 1) cache rows x (key + value) x 256 x bf16,
    # the new key and value read and appended, q and gate of 16 heads read, output written.
    cache = 64 * 2 * 4097 * 2 * 256 * 2
    new_kv = 64 * 2 * 2 * 256 * 2 * 2
    q_gate = 64 * 16 * 2 * 256 * 2
    out = 64 * 16 * 256 * 2
    assert bench.attn_decode_bytes_per_layer(64, 16, 2, 256, 4096) == cache + new_kv + q_gate + out


def test_decode_bytes_gva_batch64():
    # 64 sequences, 16 key heads each serving two of 32 value heads: q and k are read once
    # per key head.
    per_value_head = 131_072 + 256 + 256 + 8 + 256
    want = 64 * 32 * per_value_head + 64 * 16 * 512
    assert want == 270_548_992
    assert bench.decode_bytes_per_layer_step(64, 16, 32, 128) == want


def test_multi_token_bytes_count_the_state_once():
    one = bench.decode_bytes_per_layer_step(32, 16, 16, 128)
    state = 32 * 16 * 2 * 128 * 128 * 4
    assert bench.decode_bytes_per_layer_call(32, 16, 16, 128, 1) == one
    assert bench.decode_bytes_per_layer_call(32, 16, 16, 128, 4) == state + 4 * (one - state)


def test_reference_arm_json_line():
    r = _run_bench("--impl", "reference", "--steps", "1", "--warmup", "3")
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["metric"] == bench.HEADLINE and line["unit"] == "GB/s"
    assert line["higher_is_better"] is True and line["steps"] == 1 and line["warmup"] == 3
    assert line["value"] > 0 and line["dtype"] == "f64"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    assert "workload" in line["config"]


def test_warmup_below_three_is_rejected():
    r = _run_bench("--steps", "1", "--warmup", "2", timeout=120)
    assert r.returncode != 0
    assert "warmup" in r.stderr


def test_product_arm_has_no_host_fallback():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    r = _run_bench("--steps", "1", "--warmup", "3", "--no-cpu-baseline", timeout=300)
    assert r.returncode != 0
    assert not any(l.startswith("{") for l in r.stdout.splitlines())
