"""The byte accounting behind bench.py's roofline, against hand counts.

A selected block moves its K and V rows for the tokens that exist (a partial last block only
its valid tokens); q and out once per query head; the list (capacity + count) once per
(b, kv-head).  The Qwen3-8B-shaped step's figures are worked out in the comments."""

import importlib.util
import os
from types import SimpleNamespace

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_partial_block_counts_valid_tokens():
    bench = _bench()
    cfg = SimpleNamespace(B=1, Hq=2, Hkv=1, head_dim=64, gate_dim=64, block=64, g=2)
    seqlens = np.array([130])                     # blocks 0, 1 full; block 2 holds 2 tokens
    idx = np.array([[[0, 2, -1]]], dtype=np.int32)
    cnt = np.array([[2]], dtype=np.int32)
    got = bench.algorithmic_bytes(cfg, seqlens, cnt, idx, cap=3, max_blocks=3)
    # K+V: (64 + 2) tokens x 64 channels x 2 bytes x 2 tensors = 16896
    assert got["selected_kv"] == 16896
    # + q and out: 2 x (1 x 2 heads x 64 x 2 bytes) = 512; + list: (3 + 1) x 4 = 16
    assert got["decode"] == 16896 + 512 + 16


def test_qwen3_8b_32k_step_figures():
    bench = _bench()
    cfg = SimpleNamespace(B=8, Hq=32, Hkv=8, head_dim=128, gate_dim=128, block=64, g=4)
    seqlens = np.full(8, 32768)
    cap = 65
    idx = np.tile(np.arange(0, 512, 8, dtype=np.int32), (8, 8, 1))   # 64 blocks per (b, kv-head)
    idx = np.concatenate([idx, np.full((8, 8, 1), -1, np.int32)], axis=2)
    cnt = np.full((8, 8), 64, dtype=np.int32)
    got = bench.algorithmic_bytes(cfg, seqlens, cnt, idx, cap=cap, max_blocks=512)
    # 64 (b, kv-head) x 64 blocks x 64 tokens x 128 x 2 bytes x 2 = 134,217,728
    assert got["selected_kv"] == 134_217_728
    # + q, out 2 x 8 x 32 x 128 x 2 = 131,072 + lists 64 x 66 x 4 = 16,896
    assert got["decode"] == 134_365_696
    # gate: cache rows 8 x 8 x 512 x 128 x 2 = 8,388,608; W_q 8 x 128 x 512 x 2 = 1,048,576;
    # q 65,536; logits 8 x 8 x 512 x 4 = 131,072.  select: logits 131,072 + lists 16,896
    assert got["step"] == 134_365_696 + (8_388_608 + 1_048_576 + 65_536 + 131_072) + (131_072 + 16_896)
