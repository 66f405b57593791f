"""Causal prefill attention with the per-position block-level target (seer_prefill_gt) against the
CPU oracle.

Tolerances.  Outputs and LSEs: the attention bar (max-abs 1e-2, rel-L2 5e-3; LSE as the decode
test).  Targets: a block score is exp2(r - m) / l with r and m maxima of fp32 dot products of bf16
inputs and l the sum of the bf16-rounded probabilities that also weight V, so l carries at most
2^-9 relative error and the score the same plus fp32 exp2 rounding; GT_REL = 4e-3 is twice that
bound, far below a dropped head, a wrong block, a missed mask or a missing normalisation."""

import math

import numpy as np
import pytest
import torch

from oracle import seer_oracle as O
from seer_harness import bf16_bits, check_attention, check_lse, f64, to_dev_bf16

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import block_sparse_attention_attngate_b200 as S

GT_REL = 4e-3


def _bf16_bits(x):
    return (torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
            .view(np.uint16))


def _check_case(d, blk, g, Hkv, nan_tail, lengths=None):
    rng = np.random.default_rng(1300 + d + blk + g)
    lengths = lengths or [300, 2 * blk + 7, 5]
    B, Hq, T = len(lengths), g * Hkv, 320
    NB = -(-T // blk)
    q = _bf16_bits(rng.standard_normal((B, Hq, T, d)))
    k = _bf16_bits(rng.standard_normal((B, Hkv, T, d)))
    v = _bf16_bits(rng.standard_normal((B, Hkv, T, d)))
    if nan_tail:
        for b, L in enumerate(lengths):
            for x in (q, k, v):
                x[b, :, L:] = 0x7FC0                     # bf16 quiet NaN past the length
    sh = S.Shape(B, Hq, Hkv, d, 64, blk, NB)
    seq = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    out = torch.full((B, Hq, T, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, Hq, T), 7.0, dtype=torch.float32, device="cuda")
    gt = torch.full((B, Hkv, T, NB), 7.0, dtype=torch.float32, device="cuda")
    ws = torch.empty(S.prefill_gt_workspace_bytes(sh, T), dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    S.prefill_gt(sh, to_dev_bf16(q), S.KVCache.contiguous(to_dev_bf16(k)), S.KVCache.contiguous(to_dev_bf16(v)),
                 seq, out, gt, ws, lse=lse, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    o_h = f64(bf16_bits(out))
    lse_h, gt_h = lse.cpu().numpy().astype(np.float64), gt.cpu().numpy().astype(np.float64)
    scale = 1.0 / math.sqrt(d)
    for b, L in enumerate(lengths):
        if L == 0:                                       # an empty sequence: nothing written
            assert np.all(gt_h[b] == 7.0) and np.all(lse_h[b] == 7.0) and np.all(np.isnan(o_h[b]))
            continue
        for h in range(Hkv):
            ro, rl, rg = O.prefill_ground_truth(f64(q[b, h * g:(h + 1) * g, :L]), f64(k[b, h, :L]),
                                                f64(v[b, h, :L]), blk, scale)
            for j in range(g):
                check_attention(o_h[b, h * g + j, :L], ro[j], f"b{b} h{h} j{j}")
                check_lse(lse_h[b, h * g + j, :L], rl[j], f"b{b} h{h} j{j}")
            got = gt_h[b, h, :L, :rg.shape[1]]
            bad = np.abs(got - rg) > GT_REL * rg + 1e-7
            assert not bad.any(), f"b{b} h{h}: {int(bad.sum())} target entries off"
            assert np.all(gt_h[b, h, :L, rg.shape[1]:] == 0.0), "entries past the blocks"
            assert np.allclose(gt_h[b, h, :L].sum(axis=1), 1.0, atol=1e-5), "rows must sum to 1"
            assert np.all(gt_h[b, h, L:] == 7.0), "rows past the length were written"
        assert np.all(np.isnan(o_h[b, :, L:])), "outputs past the length were written"


@pytest.mark.parametrize("d,blk,g,Hkv", [(128, 64, 4, 2), (128, 128, 2, 2), (64, 64, 8, 1), (64, 128, 1, 3),
                                         (128, 64, 5, 1), (128, 64, 1, 3), (128, 64, 8, 1), (128, 128, 8, 1),
                                         (128, 128, 1, 2)])
def test_prefill_gt_vs_oracle(d, blk, g, Hkv):
    """head_dim 128 with g in {1, 2, 4, 8} runs the tcgen05 forward (every group size, both block
    sizes); head_dim 64 and g = 5 the warp-level mma one."""
    _check_case(d, blk, g, Hkv, nan_tail=False)


@pytest.mark.parametrize("d,blk,g,Hkv", [(128, 64, 4, 2), (128, 128, 8, 1), (64, 64, 2, 2)])
def test_prefill_gt_nan_past_the_length(d, blk, g, Hkv):
    """q, K and V hold NaN at every position past each sequence's length: nothing of it may reach
    the outputs, the LSEs or the targets (rows, keys and V rows past L are masked or zeroed)."""
    _check_case(d, blk, g, Hkv, nan_tail=True)


def test_prefill_gt_empty_and_one_token():
    """Sequences of 0 and 1 tokens beside a longer one (tcgen05 path): the empty one writes nothing;
    a one-token row attends to itself only (its target is the single block, 1.0)."""
    _check_case(128, 64, 4, 1, nan_tail=True, lengths=[0, 1, 200])


def test_prefill_rescales_when_later_keys_dominate():
    """Keys planted in the second and third 128-key tiles score far above everything before them for
    every query row: each row's running maximum jumps by more than 2^8 (log2 units) once past key 150
    and again past key 290 -- so a kernel that moves its reference maximum lazily must rescale its
    accumulated output -- while the scores stay moderate (<= 17 in natural units: q = noise
    orthogonal to a direction u plus 2u; planted keys 5 sqrt(d) u and 8.5 sqrt(d) u, so their
    scores are 10 and 17 against N(0, 1) elsewhere).  Output, LSE and targets against the exact
    softmax of the oracle."""
    d, blk, g, Hkv, T = 128, 64, 4, 1, 400
    rng = np.random.default_rng(4711)
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    noise = rng.standard_normal((1, g * Hkv, T, d))
    noise -= (noise @ u)[..., None] * u
    qf = noise + 2.0 * u
    kf = rng.standard_normal((1, Hkv, T, d))
    kf[0, :, 150] = 5.0 * u * math.sqrt(d)         # tile 1 (keys 128..255)
    kf[0, :, 290] = 8.5 * u * math.sqrt(d)         # tile 2 (keys 256..383)
    q, k = _bf16_bits(qf), _bf16_bits(kf)
    v = _bf16_bits(rng.standard_normal((1, Hkv, T, d)))
    sh = S.Shape(1, g * Hkv, Hkv, d, 64, blk, -(-T // blk))
    seq = torch.tensor([T], dtype=torch.int32, device="cuda")
    out = torch.empty((1, g * Hkv, T, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, g * Hkv, T), dtype=torch.float32, device="cuda")
    gt = torch.empty((1, Hkv, T, sh.max_blocks), dtype=torch.float32, device="cuda")
    ws = torch.empty(S.prefill_gt_workspace_bytes(sh, T), dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    S.prefill_gt(sh, to_dev_bf16(q), S.KVCache.contiguous(to_dev_bf16(k)), S.KVCache.contiguous(to_dev_bf16(v)),
                 seq, out, gt, ws, lse=lse, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ro, rl, rg = O.prefill_ground_truth(f64(q[0]), f64(k[0, 0]), f64(v[0, 0]), blk, 1.0 / math.sqrt(d))
    # the planted keys do raise the maxima: positions past key 290 put most of their mass on it
    assert float(np.median(rg[300:, 290 // blk])) > 0.5
    o_h, lse_h, gt_h = f64(bf16_bits(out)), lse.cpu().numpy().astype(np.float64), gt.cpu().numpy()
    for j in range(g):
        check_attention(o_h[0, j], ro[j], f"head {j}")
        check_lse(lse_h[0, j], rl[j], f"head {j}")
    bad = np.abs(gt_h[0, 0, :, :rg.shape[1]] - rg) > GT_REL * rg + 1e-7
    assert not bad.any(), f"{int(bad.sum())} target entries off"
