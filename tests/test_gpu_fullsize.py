"""Full-size parity on sampled outputs, in the launch configurations bench.py times:
the ground-truth scorer on the Qwen3-8B-shaped 32k step, and the prefill forward with targets on
one 8k sequence (B=1, Hq=32, Hkv=8, d=128, b=64).  The oracle computes each sampled row on its
own: the decode target of a (b, kv-head) from its whole K, and a prefill row i as the attention
and decode target of query position i over keys 0..i (the prefill target rows are pinned to the
decode target in the oracle's own checks).  Tolerances as the small-size tests."""

import functools
import math

import numpy as np
import pytest
import torch

from oracle import seer_oracle as O
from seer_harness import OracleBH, bf16_bits, check_attention, check_lse, draw_workers, f64, to_dev_bf16
from synthetic import config, make_inputs

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import block_sparse_attention_attngate_b200 as S

GT_REL_DECODE = 5e-4     # as tests/test_gpu_truth.py
GT_REL_PREFILL = 4e-3    # as tests/test_gpu_prefill_gt.py


@functools.lru_cache(maxsize=1)
def _step_32k():
    cfg = config(2)
    return cfg, make_inputs(cfg, workers=draw_workers())


def test_ground_truth_32k_sampled():
    cfg, inp = _step_32k()
    sh = S.Shape(cfg.B, cfg.Hq, cfg.Hkv, cfg.head_dim, cfg.gate_dim, cfg.block, inp.max_blocks,
                 rope_base=cfg.rope_base)
    scores = torch.empty(cfg.B, cfg.Hkv, inp.max_blocks, dtype=torch.float32, device="cuda")
    ws = S.alloc_truth_workspace(sh)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    S.gate_truth(sh, to_dev_bf16(inp.q), S.KVCache.contiguous(to_dev_bf16(inp.k)),
                 torch.from_numpy(inp.seqlens).cuda(), scores, ws, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = scores.cpu().numpy().astype(np.float64)
    scale = 1.0 / math.sqrt(cfg.head_dim)
    for b, h in ((0, 0), (3, 5), (5, 2), (7, 7)):
        ob = OracleBH(inp, b, h)
        L = int(inp.seqlens[b])
        ref = O.decode_ground_truth(ob.q_group(inp.q), ob.k, L, cfg.block, scale)
        g = got[b, h, :len(ref)]
        assert abs(g.sum() - 1.0) <= 1e-5
        bad = np.abs(g - ref) > GT_REL_DECODE * ref + 1e-12
        assert not bad.any(), f"b{b} h{h}: {int(bad.sum())} scores off"


def test_prefill_8k_sampled():
    B, Hq, Hkv, d, blk, L = 1, 32, 8, 128, 64, 8192
    g, NB = Hq // Hkv, L // blk
    rng = np.random.default_rng(2024)

    def bits(shape):
        x = torch.from_numpy(rng.standard_normal(shape, dtype=np.float32)).to(torch.bfloat16)
        return x.view(torch.int16).numpy().view(np.uint16)

    q, k, v = bits((B, Hq, L, d)), bits((B, Hkv, L, d)), bits((B, Hkv, L, d))
    sh = S.Shape(B, Hq, Hkv, d, d, blk, NB)
    out = torch.empty(B, Hq, L, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Hq, L, dtype=torch.float32, device="cuda")
    gt = torch.empty(B, Hkv, L, NB, dtype=torch.float32, device="cuda")
    ws = torch.empty(S.prefill_gt_workspace_bytes(sh, L), dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    S.prefill_gt(sh, to_dev_bf16(q), S.KVCache.contiguous(to_dev_bf16(k)), S.KVCache.contiguous(to_dev_bf16(v)),
                 torch.full((B,), L, dtype=torch.int32, device="cuda"), out, gt, ws, lse=lse, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    scale = 1.0 / math.sqrt(d)
    for h in (0, 3, 7):
        kk, vv = f64(k[0, h]), f64(v[0, h])
        for i in (0, 63, 64, 1000, 4095, 8191):
            rows = slice(h * g, (h + 1) * g)
            qi = f64(q[0, rows, i])
            ro, rl = O.attend(qi, kk, vv, np.arange(i + 1), scale)
            check_attention(f64(bf16_bits(out[0, rows, i])), ro, f"h{h} i{i}")
            check_lse(lse[0, rows, i].cpu().numpy().astype(np.float64), rl, f"h{h} i{i}")
            ref = O.decode_ground_truth(qi, kk, i + 1, blk, scale)
            row = gt[0, h, i].cpu().numpy().astype(np.float64)
            bad = np.abs(row[:len(ref)] - ref) > GT_REL_PREFILL * ref + 1e-7
            assert not bad.any(), f"h{h} i{i}: {int(bad.sum())} target entries off"
            assert np.all(row[len(ref):] == 0.0)


@pytest.mark.parametrize("blk,g,L,T", [(64, 4, 20001, 20032), (128, 8, 33001, 33024)])
def test_prefill_long_sampled(blk, g, L, T):
    """Sequences with more than 256 blocks (the targets are then formed in several block chunks, the
    sum first), a ragged length and rows past it that must stay untouched; sampled rows against the
    oracle, one position at a time, at block and chunk boundaries."""
    B, Hkv, d = 1, 1, 128
    Hq, NB = g * Hkv, -(-T // blk)
    rng = np.random.default_rng(77 + blk)

    def bits(shape):
        x = torch.from_numpy(rng.standard_normal(shape, dtype=np.float32)).to(torch.bfloat16)
        return x.view(torch.int16).numpy().view(np.uint16)

    q, k, v = bits((B, Hq, T, d)), bits((B, Hkv, T, d)), bits((B, Hkv, T, d))
    sh = S.Shape(B, Hq, Hkv, d, d, blk, NB)
    out = torch.empty(B, Hq, T, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Hq, T, dtype=torch.float32, device="cuda")
    gt = torch.full((B, Hkv, T, NB), 7.0, dtype=torch.float32, device="cuda")
    ws = torch.empty(S.prefill_gt_workspace_bytes(sh, T), dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    S.prefill_gt(sh, to_dev_bf16(q), S.KVCache.contiguous(to_dev_bf16(k)), S.KVCache.contiguous(to_dev_bf16(v)),
                 torch.full((B,), L, dtype=torch.int32, device="cuda"), out, gt, ws, lse=lse, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.all(gt[0, 0, L:] == 7.0), "rows past the length were written"
    scale = 1.0 / math.sqrt(d)
    kk, vv = f64(k[0, 0]), f64(v[0, 0])
    for i in (0, 256 * blk - 1, 256 * blk, 256 * blk + 31, L - 33, L - 1):
        qi = f64(q[0, :, i])
        ro, rl = O.attend(qi, kk, vv, np.arange(i + 1), scale)
        check_attention(f64(bf16_bits(out[0, :, i])), ro, f"i{i}")
        check_lse(lse[0, :, i].cpu().numpy().astype(np.float64), rl, f"i{i}")
        ref = O.decode_ground_truth(qi, kk, i + 1, blk, scale)
        row = gt[0, 0, i].cpu().numpy().astype(np.float64)
        bad = np.abs(row[:len(ref)] - ref) > GT_REL_PREFILL * ref + 1e-7
        assert not bad.any(), f"i{i}: {int(bad.sum())} target entries off"
        assert np.all(row[len(ref):] == 0.0)
        assert abs(row.sum() - 1.0) <= 1e-4
