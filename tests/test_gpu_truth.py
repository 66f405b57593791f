"""Decode ground-truth block scores (seer_gate_truth) against the CPU oracle.

Tolerance.  The GPU forms each score s = scale * q.K[t] from bf16 inputs with fp32
accumulation on the tensor pipe: |s_gpu - s| <= d * 2^-24 * scale * sum_i |q_i K_i|, which for
these unit-normal inputs (hot blocks add 3 q_hat to K) stays below ~1e-4.  A score is
exp(bmax - lse) / sum, so its relative error is at most |d bmax| + |d lse| + the relative error
of the sum, each bounded by that plus exp2/log2 rounding (a few 1e-7): 5e-4 relative is
comfortably above the bound and far below any real error (a dropped head, a wrong block or a
missing normalisation moves a score by orders of magnitude more).
"""

import math

import numpy as np
import pytest
import torch

from oracle import seer_oracle as O
from seer_harness import OracleBH, bf16_bits, check_attention, f64, gpu_list, to_dev_bf16
from synthetic import config, make_inputs, paged_view

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import block_sparse_attention_attngate_b200 as S

GT_REL = 5e-4


def _run_truth(cfg, inp, kv=None, log=True):
    sh = S.Shape(cfg.B, cfg.Hq, cfg.Hkv, cfg.head_dim, cfg.gate_dim, cfg.block, inp.max_blocks,
                 rope_base=cfg.rope_base)
    q = to_dev_bf16(inp.q)
    kv = kv or S.KVCache.contiguous(to_dev_bf16(inp.k))
    seq = torch.from_numpy(inp.seqlens).cuda()
    scores = torch.full((cfg.B, cfg.Hkv, inp.max_blocks), 7.0, dtype=torch.float32, device="cuda")
    lsc = torch.full_like(scores, 7.0) if log else None
    ws = S.alloc_truth_workspace(sh)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):   # the second call reuses the workspace counters
        S.gate_truth(sh, q, kv, seq, scores, ws, log_scores=lsc, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return scores.cpu().numpy().astype(np.float64), (lsc.cpu().numpy().astype(np.float64) if log else None)


def _check_row(got, ref, what):
    nblk = len(ref)
    assert np.all(got[nblk:] == 0.0), f"{what}: scores past ceil(L/b) must be 0"
    g = got[:nblk]
    assert abs(g.sum() - 1.0) <= 1e-5, f"{what}: scores sum to {g.sum()}"
    bad = np.abs(g - ref) > GT_REL * ref + 1e-12
    assert not bad.any(), f"{what}: {int(bad.sum())} scores off, worst rel {float(np.max(np.abs(g - ref) / ref)):.2e}"


@pytest.mark.parametrize("d,blk,g", [(128, 64, 4), (128, 128, 5), (64, 64, 8), (64, 128, 1), (128, 64, 2)])
def test_gate_truth_vs_oracle(d, blk, g):
    Hkv = 2
    cfg = config(1, B=3, Hq=g * Hkv, Hkv=Hkv, head_dim=d, gate_dim=64, block=blk, seed=700 + d + blk + g)
    lengths = [9 * blk, 11 * blk + 37, blk - 5]   # full blocks only; a partial last block; L < b
    inp = make_inputs(cfg, lengths=lengths, tail="nan")
    got, lg = _run_truth(cfg, inp)
    scale = 1.0 / math.sqrt(d)
    for b in range(cfg.B):
        for h in range(Hkv):
            ob = OracleBH(inp, b, h)
            ref = O.decode_ground_truth(ob.q_group(inp.q), ob.k, lengths[b], blk, scale)
            _check_row(got[b, h], ref, f"b{b} h{h}")
            nblk = len(ref)
            with np.errstate(divide="ignore"):
                assert np.allclose(lg[b, h, :nblk], np.log(got[b, h, :nblk]), rtol=0, atol=1e-6)
            assert np.all(np.isneginf(lg[b, h, nblk:]))


def test_gate_truth_paged_and_empty():
    blk, d, g, Hkv = 64, 128, 4, 2
    cfg = config(1, B=3, Hq=g * Hkv, Hkv=Hkv, head_dim=d, gate_dim=64, block=blk, seed=1717)
    lengths = [10 * blk + 5, 0, 7 * blk]   # an empty sequence scores all zero
    inp = make_inputs(cfg, lengths=lengths, tail="nan")
    pool, table = paged_view(inp.k, blk, seed=5)
    paged = S.KVCache.paged(to_dev_bf16(pool), torch.from_numpy(table).cuda())
    got_p, _ = _run_truth(cfg, inp, kv=paged)
    got_c, _ = _run_truth(cfg, inp)
    assert np.array_equal(got_p, got_c), "paged != contiguous"
    assert np.all(got_c[1] == 0.0)
    for b in (0, 2):
        for h in range(Hkv):
            ob = OracleBH(inp, b, h)
            ref = O.decode_ground_truth(ob.q_group(inp.q), ob.k, lengths[b], blk, 1.0 / math.sqrt(d))
            _check_row(got_c[b, h], ref, f"b{b} h{h}")


def test_ground_truth_selection_pipeline():
    """Ground-truth scores -> top-k (seer_select_blocks on the log scores) -> sparse decode: the
    'oracle' sparse mode.  Selections must match the oracle's top-k on its own ground truth
    wherever the k-th and (k+1)-th scores are separated by more than the score tolerance."""
    blk, d, g, Hkv = 64, 128, 4, 4
    cfg = config(1, B=2, Hq=g * Hkv, Hkv=Hkv, head_dim=d, gate_dim=64, block=blk, seed=2323)
    lengths = [40 * blk + 11, 33 * blk]
    inp = make_inputs(cfg, lengths=lengths, tail="nan")
    sh = S.Shape(cfg.B, cfg.Hq, cfg.Hkv, d, 64, blk, inp.max_blocks, rope_base=cfg.rope_base)
    got, lg = _run_truth(cfg, inp)
    budget = 8 * blk
    k = budget // blk
    cap = k + 1
    idx = torch.empty((cfg.B, Hkv, cap), dtype=torch.int32, device="cuda")
    cnt = torch.empty((cfg.B, Hkv), dtype=torch.int32, device="cuda")
    seq = torch.from_numpy(inp.seqlens).cuda()
    S.select_blocks(sh, torch.from_numpy(lg.astype(np.float32)).cuda(), seq, S.SELECT_TOPK, idx, cnt,
                    token_budget=budget)
    out = torch.empty((cfg.B, cfg.Hq, d), dtype=torch.bfloat16, device="cuda")
    S.sparse_decode(sh, to_dev_bf16(inp.q), S.KVCache.contiguous(to_dev_bf16(inp.k)),
                    S.KVCache.contiguous(to_dev_bf16(inp.v)), idx, cnt, seq, out, S.alloc_workspace(sh, cap, 0))
    torch.cuda.synchronize()
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    o = f64(bf16_bits(out))
    compared = 0
    for b in range(cfg.B):
        for h in range(Hkv):
            ob = OracleBH(inp, b, h)
            L = lengths[b]
            gt = O.decode_ground_truth(ob.q_group(inp.q), ob.k, L, blk, 1.0 / math.sqrt(d))
            nfull = L // blk
            with np.errstate(divide="ignore"):
                ref = O.select_topk(np.log(gt[:nfull]), k, L, blk)
            sel = gpu_list(idx_h[b, h], cnt_h[b, h])
            srt = np.sort(gt[:nfull])[::-1]
            if srt[k - 1] - srt[k] > 4 * GT_REL * srt[k - 1]:
                assert sel == ref, f"b{b} h{h}: {sel} vs {ref}"
                compared += 1
            ro, _ = ob.attention(L, inp.q, sel)
            check_attention(o[b, h * g:(h + 1) * g], ro, f"b{b} h{h}")
    assert compared >= cfg.B * Hkv // 2
