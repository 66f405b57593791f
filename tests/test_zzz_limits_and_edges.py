"""Sizes and corners beyond the rest of the GPU suite, against the same oracle and bars: selection
and the fused plan on rows up to the largest accepted max_blocks (8192), the decode on the longest
accepted lists, eight query heads per KV head at d = 128 (decode, ground truth, prefill), NaN past
the length and empty or one-token sequences in the prefill, a length-0 sequence in the decode step,
bit-for-bit repeatability, and the block-completing running-statistics launch at the 32k step's
shapes.  Collected last, after the established suite."""

import functools
import math

import numpy as np
import pytest
import torch

import test_gpu_fullsize as F
import test_gpu_kernels as K
import test_gpu_prefill_gt as PG
import test_gpu_truth as TT
from oracle import seer_oracle as O
from seer_harness import (bf16_bits, check_attention, check_kcomp_rows, check_logits, check_lse, check_selection,
                          f64, gpu_list, to_dev_bf16)
from synthetic import bf16_bits_from_f32, config, make_inputs, make_logits

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import block_sparse_attention_attngate_b200 as S

_dev, _shape = K._dev, K._shape


# ------------------------------------------------------------------ long rows and lists

@pytest.mark.parametrize("nb", [1000, 2000, 3000, 8192])
@pytest.mark.parametrize("mode", ["topk", "threshold", "topp"])
def test_select_long_rows(nb, mode):
    """Rows past the small cases: 1000 and 2000 blocks (the register-resident path with 4 and 8 keys
    a thread), 3000 and 8192 (the shared-memory path; 8192 is the largest max_blocks accepted)."""
    B, Hkv, block = 2, 2, 64
    seqlens = np.array([nb * block, (3 * nb // 4) * block + 17], dtype=np.int32)
    logits = make_logits(41 + nb, B, Hkv, nb, "ties" if nb == 3000 else "normal")
    sh = S.Shape(B, Hkv, Hkv, 64, 64, block, nb)
    lg = torch.from_numpy(logits).cuda()
    sl = torch.from_numpy(seqlens).cuda()
    cnt = torch.empty((B, Hkv), dtype=torch.int32, device="cuda")
    if mode == "topk":
        settings = [nb // 10, nb - 1]
    elif mode == "threshold":
        settings = [1e-4, 0.5 / nb]
    else:
        settings = [0.5, 0.95]
    for x in settings:
        cap = min(nb, x + 1) if mode == "topk" else nb
        idx = torch.full((B, Hkv, cap), -7, dtype=torch.int32, device="cuda")
        if mode == "topk":
            S.select_blocks(sh, lg, sl, S.SELECT_TOPK, idx, cnt, token_budget=x * block)
        else:
            x = float(np.float32(x))
            S.select_blocks(sh, lg, sl, S.SELECT_THRESHOLD if mode == "threshold" else S.SELECT_TOPP, idx, cnt, tau=x)
        idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
        for b in range(B):
            L = int(seqlens[b])
            for h in range(Hkv):
                z = logits[b, h].astype(np.float64)
                got = gpu_list(idx_h[b, h], cnt_h[b, h])
                assert np.all(idx_h[b, h, cnt_h[b, h]:] == -1)
                if mode == "topk":
                    assert got == O.select_topk(z, x, L, block), f"nb {nb} k {x} b{b} h{h}"
                elif mode == "threshold":
                    check_selection(got, O.select_threshold(z, x, L, block), O.gate_scores(z[:L // block]), x,
                                    f"nb {nb} tau {x} b{b} h{h}")
                else:
                    assert got == O.select_topp(z, x, L, block), f"nb {nb} p {x} b{b} h{h}"


@pytest.mark.parametrize("nb", [2000, 8192])
@pytest.mark.parametrize("mode", ["topk", "threshold", "topp"])
def test_plan_long_rows(nb, mode):
    """The fused plan (gate + selection, no cache update) on rows of 2000 and 8192 blocks: its logits
    against the oracle's from the same cache, and its lists against the oracle's selection on the
    logits the kernel produced (fp32, the selection's input)."""
    B, Hkv, g, d, dg, block = 2, 2, 4, 128, 128, 64
    Hq = g * Hkv
    rng = np.random.default_rng(5000 + nb)
    seqlens = np.array([nb * block, (3 * nb // 4) * block + 17], dtype=np.int32)
    q = bf16_bits_from_f32(rng.standard_normal((B, Hq, d), dtype=np.float32))
    w_q = bf16_bits_from_f32((rng.standard_normal((Hkv, dg, g * d)) / math.sqrt(g * d)).astype(np.float32))
    kc = bf16_bits_from_f32(rng.standard_normal((B, Hkv, nb, dg), dtype=np.float32))
    sh = S.Shape(B, Hq, Hkv, d, dg, block, nb)
    logits = torch.empty((B, Hkv, nb), dtype=torch.float32, device="cuda")
    cnt = torch.empty((B, Hkv), dtype=torch.int32, device="cuda")
    k_blocks = nb // 10
    cap = k_blocks + 1 if mode == "topk" else nb
    idx = torch.full((B, Hkv, cap), -7, dtype=torch.int32, device="cuda")
    x = {"topk": 0.0, "threshold": float(np.float32(0.5 / nb)), "topp": float(np.float32(0.9))}[mode]
    m = {"topk": S.SELECT_TOPK, "threshold": S.SELECT_THRESHOLD, "topp": S.SELECT_TOPP}[mode]
    S.decode_plan(sh, torch.from_numpy(seqlens).cuda(), to_dev_bf16(kc), to_dev_bf16(q), to_dev_bf16(w_q), m, idx,
                  cnt, token_budget=k_blocks * block, tau=x, logits=logits)
    lg = logits.cpu().numpy()
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    for b in range(B):
        L = int(seqlens[b])
        nfull = L // block
        for h in range(Hkv):
            qg = O.q_gate(f64(q[b, h * g:(h + 1) * g]), f64(w_q[h]), L, sh.rope_base)
            check_logits(lg[b, h, :nfull], O.gate_logits(qg, f64(kc[b, h]), L, block), f"nb {nb} b{b} h{h}")
            assert np.all(lg[b, h, nfull:] == -np.inf)
            z = lg[b, h].astype(np.float64)
            got = gpu_list(idx_h[b, h], cnt_h[b, h])
            assert np.all(idx_h[b, h, cnt_h[b, h]:] == -1)
            if mode == "topk":
                assert got == O.select_topk(z, k_blocks, L, block), f"nb {nb} b{b} h{h}"
            elif mode == "threshold":
                check_selection(got, O.select_threshold(z, x, L, block), O.gate_scores(z[:nfull]), x,
                                f"nb {nb} b{b} h{h}")
            else:
                assert got == O.select_topp(z, x, L, block), f"nb {nb} b{b} h{h}"


@functools.lru_cache(maxsize=1)
def _longest_problem():
    blk, d, g, nb = 64, 64, 4, 8192
    cfg = config(1, B=1, Hq=g, Hkv=1, head_dim=d, gate_dim=64, block=blk, seed=3131)
    return cfg, make_inputs(cfg, lengths=[nb * blk - 5], tail="nan")


@pytest.mark.parametrize("ns", [0, -1, 16])
def test_sparse_decode_longest_lists(ns):
    """The longest lists accepted: max_blocks = 8192 (524,288 tokens at b = 64) with a ragged last
    block (NaN past the length), half of the full blocks plus the partial one (4097 entries), then
    every block; the balanced, capacity and (split, kv head, batch) schedules."""
    blk, d, g, nb = 64, 64, 4, 8192
    L = nb * blk - 5
    cfg, inp = _longest_problem()
    assert inp.max_blocks == nb
    dv = _dev(inp)
    sh = _shape(cfg, inp)
    kv_k, kv_v = S.KVCache.contiguous(dv["k"]), S.KVCache.contiguous(dv["v"])
    rng = np.random.default_rng(77)
    half = sorted(int(x) for x in rng.choice(nb - 1, size=(nb - 1) // 2, replace=False)) + [nb - 1]
    kk, vv, q = f64(inp.k[0, 0]), f64(inp.v[0, 0]), f64(inp.q[0])
    for blocks in (half, list(range(nb))):
        idx = np.full((1, 1, nb), -1, np.int32)
        idx[0, 0, :len(blocks)] = blocks
        cnt = np.array([[len(blocks)]], np.int32)
        out = torch.empty((1, g, d), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((1, g), dtype=torch.float32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        S.sparse_decode(sh, dv["q"], kv_k, kv_v, torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(),
                        dv["seqlens"], out, S.alloc_workspace(sh, nb, ns), num_split=ns, lse=lse, err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        ro, rl = O.sparse_decode(q, kk, vv, blocks, L, blk, 1.0 / math.sqrt(d))
        check_attention(f64(bf16_bits(out))[0], ro, f"{len(blocks)} blocks ns {ns}")
        check_lse(lse.cpu().numpy()[0].astype(np.float64), rl, f"{len(blocks)} blocks ns {ns}")


# ------------------------------------------------------------------ eight query heads per KV head at d = 128

@pytest.mark.parametrize("ns", [1, 2, 3, 0, -1])
def test_sparse_decode_group_of_eight(ns):
    K.test_sparse_decode_vs_oracle(128, 64, 8, ns)


def test_gate_truth_group_of_eight():
    TT.test_gate_truth_vs_oracle(128, 64, 8)


def test_prefill_gt_group_of_eight():
    PG._check_case(128, 64, 8, 1, nan_tail=False)


# ------------------------------------------------------------------ prefill corners

@pytest.mark.parametrize("d,blk,g,Hkv", [(128, 64, 4, 2), (64, 128, 1, 3)])
def test_prefill_gt_nan_past_length(d, blk, g, Hkv):
    """q, K and V rows past each sequence's length hold NaN (a cache's unused tail): none of it
    reaches the outputs, the LSEs or the targets of the positions that exist."""
    PG._check_case(d, blk, g, Hkv, nan_tail=True)


def test_prefill_gt_empty_and_one_token_sequences():
    """Sequences of 0 and 1 tokens beside a ragged one: the empty one is left untouched."""
    PG._check_case(128, 64, 4, 2, nan_tail=True, lengths=[0, 1, 2 * 64 + 7])


# ------------------------------------------------------------------ decode step corners

def test_decode_step_with_an_empty_sequence():
    """A sequence of length 0 in the batch gets no blocks, a fill count of 0, a zero output and
    lse = -inf; the other sequence's cache rows and lists are bit-identical to a run in which the
    first sequence is not empty, and its outputs agree within the attention bar."""
    blk, d, dg, g, Hkv = 64, 128, 128, 4, 2
    L1 = 9 * blk + 17
    cfg = config(1, B=2, Hq=g * Hkv, Hkv=Hkv, head_dim=d, gate_dim=dg, block=blk, seed=5353)
    inp = make_inputs(cfg, lengths=[3 * blk + 1, L1])
    dv = _dev(inp)
    sh = _shape(cfg, inp)
    kv_k, kv_v = S.KVCache.contiguous(dv["k"]), S.KVCache.contiguous(dv["v"])
    steps = []
    for L0 in (0, 3 * blk + 1):
        kc = torch.zeros((cfg.B, Hkv, inp.max_blocks, dg), dtype=torch.bfloat16, device="cuda")
        valid = torch.zeros(cfg.B, Hkv, dtype=torch.int32, device="cuda")
        st = S.DecodeStep(sh, kv_k, kv_v, dv["w_q"], dv["w_k"], kc, valid, mode=S.SELECT_TOPK,
                          token_budget=4 * blk)
        st.run(dv["q"], torch.tensor([L0, L1], dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        assert int(st.err.item()) == 0
        steps.append(st)
    e, f = steps
    assert e.block_cnt[0].cpu().tolist() == [0] * Hkv and e.valid_blocks[0].cpu().tolist() == [0] * Hkv
    assert torch.all(e.out[0].float() == 0.0) and torch.all(torch.isneginf(e.lse[0]))
    for name in ("kcomp", "block_idx", "block_cnt", "valid_blocks"):
        x, y = getattr(e, name)[1], getattr(f, name)[1]
        assert torch.equal(x.view(torch.int16) if x.dtype == torch.bfloat16 else x,
                           y.view(torch.int16) if y.dtype == torch.bfloat16 else y), name
    check_attention(f64(bf16_bits(e.out[1])), f64(bf16_bits(f.out[1])), "out of the other sequence")
    check_lse(e.lse[1].cpu().numpy().astype(np.float64), f.lse[1].cpu().numpy().astype(np.float64), "its lse")


def test_repeat_runs_are_bitwise_identical():
    """Every kernel is deterministic (integer atomics only; split pieces merged in a fixed order):
    two runs on fresh buffers agree bit for bit -- the decode step fused and unfused, the ground
    truth scorer and the prefill forward."""
    blk, d, dg, g, Hkv = 64, 128, 128, 4, 2
    cfg = config(1, B=2, Hq=g * Hkv, Hkv=Hkv, head_dim=d, gate_dim=dg, block=blk, seed=4242)
    lengths = [20 * blk + 7, 16 * blk]
    inp = make_inputs(cfg, lengths=lengths)
    dv = _dev(inp)
    sh = _shape(cfg, inp)
    nb = inp.max_blocks
    kv_k, kv_v = S.KVCache.contiguous(dv["k"]), S.KVCache.contiguous(dv["v"])

    def bits(t):
        return t.contiguous().view(torch.int32 if t.element_size() == 4 else torch.int16).cpu()

    for fused, ns in ((True, 2), (False, 2), (True, -1)):   # (True, -1): the whole step as one launch
        runs = []
        for _ in range(2):
            kc = torch.zeros((cfg.B, Hkv, nb, dg), dtype=torch.bfloat16, device="cuda")
            valid = torch.zeros(cfg.B, Hkv, dtype=torch.int32, device="cuda")
            st = S.DecodeStep(sh, kv_k, kv_v, dv["w_q"], dv["w_k"], kc, valid, mode=S.SELECT_TOPK,
                              token_budget=4 * blk, num_split=ns, single_launch=ns == -1)
            st.run(dv["q"], dv["seqlens"], fused=fused)
            torch.cuda.synchronize()
            assert int(st.err.item()) == 0
            runs.append(st)
        a, b = runs
        for name in ("kcomp", "valid_blocks", "block_idx", "block_cnt", "out", "lse"):
            assert torch.equal(bits(getattr(a, name)), bits(getattr(b, name))), f"fused={fused} ns={ns}: {name}"
        for bb, L in enumerate(lengths):
            n = L // blk
            assert torch.equal(bits(a.logits[bb, :, :n]), bits(b.logits[bb, :, :n])), f"fused={fused}: logits"
    scores = []
    for _ in range(2):
        sc = torch.empty((cfg.B, Hkv, nb), dtype=torch.float32, device="cuda")
        S.gate_truth(sh, dv["q"], kv_k, dv["seqlens"], sc, S.alloc_truth_workspace(sh))
        scores.append(bits(sc))
    assert torch.equal(scores[0], scores[1]), "ground truth"
    T = int(inp.k.shape[2])
    q4 = torch.randn(cfg.B, cfg.Hq, T, d, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16).cuda()
    outs = []
    for _ in range(2):
        o = torch.full((cfg.B, cfg.Hq, T, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        ls = torch.full((cfg.B, cfg.Hq, T), 7.0, dtype=torch.float32, device="cuda")
        gt = torch.full((cfg.B, Hkv, T, nb), 7.0, dtype=torch.float32, device="cuda")
        ws = torch.empty(S.prefill_gt_workspace_bytes(sh, T), dtype=torch.uint8, device="cuda")
        S.prefill_gt(sh, q4, kv_k, kv_v, dv["seqlens"], o, gt, ws, lse=ls)
        outs.append((bits(o), bits(ls), bits(gt)))
    for x, y in zip(*outs):
        assert torch.equal(x, y), "prefill"


# ------------------------------------------------------------------ full size

def test_kcomp_append_32k_sampled():
    """The cache from running block statistics at the 32k step's shapes (B=8, Hkv=8, 512 blocks of
    64), in the launch that completes a block: statistics primed from the key cache 63 tokens into
    block 511, then the token that completes it writes entry 511 of every (b, kv-head)."""
    cfg, inp = F._step_32k()
    B, Hkv, d, dg, blk, nb = cfg.B, cfg.Hkv, cfg.head_dim, cfg.gate_dim, cfg.block, inp.max_blocks
    L = nb * blk
    assert np.all(inp.seqlens == L)
    sh = S.Shape(B, cfg.Hq, Hkv, d, dg, blk, nb, rope_base=cfg.rope_base)
    kv = S.KVCache.contiguous(to_dev_bf16(inp.k))
    state = S.alloc_kcomp_state(sh)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    S.kcomp_state_init(sh, kv, torch.full((B,), L - 1, dtype=torch.int32, device="cuda"), state, err=err)
    valid = torch.full((B, Hkv), nb - 1, dtype=torch.int32, device="cuda")
    kc = torch.zeros((B, Hkv, nb, dg), dtype=torch.bfloat16, device="cuda")
    S.kcomp_append(sh, to_dev_bf16(np.ascontiguousarray(inp.k[:, :, L - 1])), torch.full((B,), L, dtype=torch.int32,
                   device="cuda"), state, valid, to_dev_bf16(inp.w_k), kc, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.all(valid.cpu().numpy() == nb)
    got = bf16_bits(kc)
    assert np.all(got[:, :, :nb - 1] == 0), "entries below the fill count were written"
    for b, h in ((0, 0), (2, 7), (5, 3), (7, 6)):
        ref = O.k_gate_entry(f64(inp.k[b, h, L - blk:L]), f64(inp.w_k[h]), nb - 1, blk, cfg.rope_base)
        check_kcomp_rows(got[b, h, nb - 1:nb], ref[None], f"b{b} h{h}")
