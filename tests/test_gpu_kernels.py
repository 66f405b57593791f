"""Per-kernel parity of the CUDA path against the CPU oracle, called through the C ABI.

Sizes are small enough for the float64 oracle to finish in seconds while still
spanning several tiles, splits and a ragged tail; edge cases cover empty
lists, lengths shorter than one block, NaN-poisoned cache tails, paged
layouts, out-of-range indices and selection rows up to the largest accepted
max_blocks (8192).
"""

import functools
import math

import numpy as np
import pytest
import torch

from oracle import seer_oracle as O
from seer_harness import (OracleBH, bf16_bits, check_attention, check_kcomp_rows, check_logits, check_lse,
                          check_selection, f64, gpu_list, to_dev_bf16)
from synthetic import bf16_bits_from_f32, config, make_block_lists, make_inputs, make_logits, paged_view

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import block_sparse_attention_attngate_b200 as S


def _shape(cfg, inp, **kw):
    return S.Shape(cfg.B, cfg.Hq, cfg.Hkv, cfg.head_dim, cfg.gate_dim, cfg.block, inp.max_blocks,
                   rope_base=cfg.rope_base, **kw)


def _dev(inp):
    return dict(q=to_dev_bf16(inp.q), k=to_dev_bf16(inp.k), v=to_dev_bf16(inp.v), w_q=to_dev_bf16(inp.w_q),
                w_k=to_dev_bf16(inp.w_k), seqlens=torch.from_numpy(inp.seqlens).cuda())


# ------------------------------------------------------------------ selection (on oracle-side logits)

@pytest.mark.parametrize("kind", ["normal", "ties"])
@pytest.mark.parametrize("block", [64, 128])
def test_select_topk_exact(kind, block):
    B, Hkv, nb = 3, 2, 47
    seqlens = np.array([nb * block, 5 * block + 17, 1 + 3], dtype=np.int32)
    logits = make_logits(11 + block, B, Hkv, nb, kind)
    sh = S.Shape(B, 2 * Hkv, Hkv, 128, 128, block, nb)
    lg = torch.from_numpy(logits).cuda()
    sl = torch.from_numpy(seqlens).cuda()
    for budget in (0, 1, block, 7 * block + 1, 20 * block, 100 * block):
        k = -(-budget // block)
        cap = min(nb, k + 1) if k + 1 <= nb else nb
        idx = torch.full((B, Hkv, cap), -7, dtype=torch.int32, device="cuda")
        cnt = torch.empty((B, Hkv), dtype=torch.int32, device="cuda")
        S.select_blocks(sh, lg, sl, S.SELECT_TOPK, idx, cnt, token_budget=budget)
        idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
        for b in range(B):
            for h in range(Hkv):
                ref = O.select_topk(logits[b, h].astype(np.float64), k, int(seqlens[b]), block)
                got = gpu_list(idx_h[b, h], cnt_h[b, h])
                assert got == ref, f"budget {budget} b{b} h{h}: {got} vs {ref}"
                assert np.all(idx_h[b, h, cnt_h[b, h]:] == -1)


@pytest.mark.parametrize("block", [64, 128])
def test_select_threshold_exact(block):
    B, Hkv, nb = 3, 3, 300
    seqlens = np.array([nb * block, 200 * block + 5, 2 * block + 1], dtype=np.int32)
    logits = make_logits(23, B, Hkv, nb)
    sh = S.Shape(B, Hkv, Hkv, 64, 64, block, nb)
    lg = torch.from_numpy(logits).cuda()
    sl = torch.from_numpy(seqlens).cuda()
    idx = torch.empty((B, Hkv, nb), dtype=torch.int32, device="cuda")
    cnt = torch.empty((B, Hkv), dtype=torch.int32, device="cuda")
    for tau in (0.0, 1e-4, 2.0 / 256, 0.05, 1.0):
        tau32 = float(np.float32(tau))
        S.select_blocks(sh, lg, sl, S.SELECT_THRESHOLD, idx, cnt, tau=tau32)
        idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
        for b in range(B):
            L = int(seqlens[b])
            for h in range(Hkv):
                z = logits[b, h].astype(np.float64)
                ref = O.select_threshold(z, tau32, L, block)
                check_selection(gpu_list(idx_h[b, h], cnt_h[b, h]), ref, O.gate_scores(z[:L // block]), tau32,
                                f"tau {tau} b{b} h{h}")


@pytest.mark.parametrize("kind", ["normal", "ties"])
def test_select_topp_exact(kind):
    B, Hkv, nb, block = 2, 2, 130, 64
    seqlens = np.array([nb * block, 77 * block + 3], dtype=np.int32)
    logits = make_logits(31, B, Hkv, nb, kind)
    sh = S.Shape(B, Hkv, Hkv, 64, 64, block, nb)
    lg = torch.from_numpy(logits).cuda()
    sl = torch.from_numpy(seqlens).cuda()
    idx = torch.empty((B, Hkv, nb), dtype=torch.int32, device="cuda")
    cnt = torch.empty((B, Hkv), dtype=torch.int32, device="cuda")
    for p in (0.1, 0.5, 0.9, 0.999):
        p32 = float(np.float32(p))
        S.select_blocks(sh, lg, sl, S.SELECT_TOPP, idx, cnt, tau=p32)
        idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
        for b in range(B):
            for h in range(Hkv):
                ref = O.select_topp(logits[b, h].astype(np.float64), p32, int(seqlens[b]), block)
                assert gpu_list(idx_h[b, h], cnt_h[b, h]) == ref, f"p {p} b{b} h{h}"


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


# ------------------------------------------------------------------ gate score / kcomp

@pytest.mark.parametrize("d,dg,blk,g", [(128, 128, 64, 4), (64, 64, 64, 4), (128, 64, 128, 5), (64, 128, 128, 8)])
def test_kcomp_and_gate_vs_oracle(d, dg, blk, g):
    Hkv = 2
    cfg = config(1, B=2, Hq=g * Hkv, Hkv=Hkv, head_dim=d, gate_dim=dg, block=blk, seed=77 + d + dg + blk + g)
    lengths = [7 * blk + 33, 12 * blk]
    inp = make_inputs(cfg, lengths=lengths)
    dv = _dev(inp)
    sh = _shape(cfg, inp)
    nb = inp.max_blocks
    kc = torch.zeros((cfg.B, Hkv, nb, dg), dtype=torch.bfloat16, device="cuda")
    valid = torch.zeros(cfg.B, Hkv, dtype=torch.int32, device="cuda")
    S.kcomp_update(sh, S.KVCache.contiguous(dv["k"]), dv["seqlens"], valid, dv["w_k"], kc)
    kc_bits = bf16_bits(kc)
    assert valid.cpu().tolist() == [[L // blk] * Hkv for L in lengths]
    logits = torch.empty((cfg.B, Hkv, nb), dtype=torch.float32, device="cuda")
    qg = torch.empty((cfg.B, Hkv, dg), dtype=torch.float32, device="cuda")
    # gate on the oracle's own cache, to isolate the gate kernel
    ref_kc = np.zeros((cfg.B, Hkv, nb, dg), dtype=np.uint16)
    for b in range(cfg.B):
        for h in range(Hkv):
            ob = OracleBH(inp, b, h)
            kref = ob.kcomp(lengths[b])
            nfull = lengths[b] // blk
            from synthetic import bf16_bits_from_f32
            ref_kc[b, h, :nfull] = bf16_bits_from_f32(kref[:nfull].astype(np.float32))
            frac = check_kcomp_rows(kc_bits[b, h, :nfull], kref[:nfull], f"kcomp b{b} h{h}")
            assert frac >= 0.98, f"kcomp b{b} h{h}: only {frac:.3f} bit-exact"
            assert np.all(kc_bits[b, h, nfull:] == 0), "kcomp wrote past the full blocks"
    S.gate_score(sh, dv["q"], dv["w_q"], to_dev_bf16(ref_kc), dv["seqlens"], logits, qg)
    lg, qgh = logits.cpu().numpy(), qg.cpu().numpy()
    for b in range(cfg.B):
        for h in range(Hkv):
            ob = OracleBH(inp, b, h)
            q_ref = O.q_gate(ob.q_group(inp.q), f64(inp.w_q[h]), lengths[b], cfg.rope_base)
            check_logits(qgh[b, h], q_ref, f"q_gate b{b} h{h}")
            ref = O.gate_logits(q_ref, f64(ref_kc[b, h]), lengths[b], blk)
            nfull = lengths[b] // blk
            check_logits(lg[b, h, :nfull], ref, f"logits b{b} h{h}")
            assert np.all(np.isneginf(lg[b, h, nfull:]))


def test_kcomp_incremental_freeze_and_rebuild():
    blk, d, dg, Hkv = 64, 128, 128, 2
    cfg = config(1, B=2, Hq=8, Hkv=Hkv, head_dim=d, gate_dim=dg, block=blk, seed=404)
    inp = make_inputs(cfg, lengths=[5 * blk - 3, 6 * blk + 2])
    dv = _dev(inp)
    sh = _shape(cfg, inp)
    nb = inp.max_blocks
    kc = torch.zeros((cfg.B, Hkv, nb, dg), dtype=torch.bfloat16, device="cuda")
    valid = torch.zeros(cfg.B, Hkv, dtype=torch.int32, device="cuda")
    kv = S.KVCache.contiguous(dv["k"])
    start = np.array([2 * blk - 5, 3 * blk - 1], dtype=np.int32)
    seen = {}
    for step in range(2 * blk + 10):
        L = start + step
        sl = torch.from_numpy(L).cuda()
        before = bf16_bits(kc)
        S.kcomp_update(sh, kv, sl, valid, dv["w_k"], kc)
        after = bf16_bits(kc)
        assert valid.cpu().tolist() == [[int(x)] * Hkv for x in (L // blk)]
        for b in range(cfg.B):
            changed = sorted(set(np.nonzero((before[b] != after[b]).any(axis=(0, 2)))[0].tolist()))
            # a block may change only on the step where it fills (L == (n+1)*blk)
            for n in changed:
                assert L[b] == (n + 1) * blk or (step == 0 and n < L[b] // blk), f"b{b} block {n} at L={L[b]}"
                seen[(b, n)] = step
    rebuilt = torch.zeros_like(kc)
    v0 = torch.zeros(cfg.B, Hkv, dtype=torch.int32, device="cuda")
    S.kcomp_update(sh, kv, torch.from_numpy(start + 2 * blk + 9).cuda(), v0, dv["w_k"], rebuilt)
    assert torch.equal(rebuilt.view(torch.int16), kc.view(torch.int16)), "incremental != rebuild"


# ------------------------------------------------------------------ sparse decode on oracle block lists

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


@pytest.mark.parametrize("d,blk,g", [(128, 64, 4), (128, 128, 5), (64, 64, 8), (64, 128, 1), (128, 64, 2),
                                     (128, 64, 8)])
@pytest.mark.parametrize("ns", [1, 2, 3, 0, -1])
def test_sparse_decode_vs_oracle(d, blk, g, ns):
    Hkv = 2
    cfg = config(1, B=3, Hq=g * Hkv, Hkv=Hkv, head_dim=d, gate_dim=64, block=blk, seed=900 + d + blk + g)
    lengths = [9 * blk, 11 * blk + 37, 3 * blk + 1]
    inp = make_inputs(cfg, lengths=lengths, tail="nan")
    dv = _dev(inp)
    sh = _shape(cfg, inp)
    cap = 8
    idx, cnt = make_block_lists(5 + ns, lengths, Hkv, blk, cap, density=0.5)
    out = torch.empty((cfg.B, cfg.Hq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((cfg.B, cfg.Hq), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = S.alloc_workspace(sh, cap, ns)
    kv_k, kv_v = S.KVCache.contiguous(dv["k"]), S.KVCache.contiguous(dv["v"])
    for rep in range(2):   # a second call reuses the workspace counters
        S.sparse_decode(sh, dv["q"], kv_k, kv_v, torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(),
                        dv["seqlens"], out, ws, num_split=ns, lse=lse, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    o = f64(bf16_bits(out))
    lh = lse.cpu().numpy()
    for b in range(cfg.B):
        for h in range(Hkv):
            ob = OracleBH(inp, b, h)
            blocks = gpu_list(idx[b, h], cnt[b, h])
            ro, rl = ob.attention(lengths[b], inp.q, blocks)
            check_attention(o[b, h * g:(h + 1) * g], ro, f"b{b} h{h}")
            check_lse(lh[b, h * g:(h + 1) * g], rl, f"b{b} h{h}")


@pytest.mark.parametrize("ns", [0, 3, -1])
def test_sparse_decode_many_short_lists(ns):
    """Many (b, h) pairs with short lists: the balanced schedule packs several whole lists into
    one CTA range and splits others across CTAs; the grid schedule leaves most splits empty; the
    capacity schedule skips every position past a list's count (an empty list included)."""
    blk, d, g, Hkv = 64, 128, 4, 8
    cfg = config(1, B=32, Hq=g * Hkv, Hkv=Hkv, head_dim=d, gate_dim=64, block=blk, seed=4242)
    rng = np.random.default_rng(3)
    lengths = [int(x) for x in rng.integers(1, 6 * blk, 32)]
    inp = make_inputs(cfg, lengths=lengths, tail="nan")
    dv = _dev(inp)
    sh = _shape(cfg, inp)
    cap = 6
    idx, cnt = make_block_lists(17, lengths, Hkv, blk, cap, density=0.7)
    cnt[5, 3] = 0        # an empty list among them
    idx[5, 3] = -1
    out = torch.empty((cfg.B, cfg.Hq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((cfg.B, cfg.Hq), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = S.alloc_workspace(sh, cap, ns)
    for _ in range(2):
        S.sparse_decode(sh, dv["q"], S.KVCache.contiguous(dv["k"]), S.KVCache.contiguous(dv["v"]),
                        torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(), dv["seqlens"], out, ws,
                        num_split=ns, lse=lse, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    o = f64(bf16_bits(out))
    lh = lse.cpu().numpy()
    for b in range(cfg.B):
        for h in range(Hkv):
            ro, rl = OracleBH(inp, b, h).attention(lengths[b], inp.q, gpu_list(idx[b, h], cnt[b, h]))
            check_attention(o[b, h * g:(h + 1) * g], ro, f"b{b} h{h}")
            check_lse(lh[b, h * g:(h + 1) * g], rl, f"b{b} h{h}")


def test_sparse_decode_paged_matches_contiguous():
    blk, d, g, Hkv = 64, 128, 4, 2
    cfg = config(1, B=2, Hq=g * Hkv, Hkv=Hkv, head_dim=d, gate_dim=64, block=blk, seed=1313)
    lengths = [10 * blk + 5, 7 * blk]
    inp = make_inputs(cfg, lengths=lengths, tail="nan")
    dv = _dev(inp)
    sh = _shape(cfg, inp)
    pool_k, table = paged_view(inp.k, blk, seed=3)
    pool_v, _ = paged_view(inp.v, blk, seed=3)
    cap = 12
    idx, cnt = make_block_lists(8, lengths, Hkv, blk, cap, density=0.6)
    idx_d, cnt_d = torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()
    tbl = torch.from_numpy(table).cuda()
    outs = []
    for layout in ("contiguous", "paged"):
        if layout == "paged":
            kk = S.KVCache.paged(to_dev_bf16(pool_k), tbl)
            vv = S.KVCache.paged(to_dev_bf16(pool_v), tbl)
        else:
            kk, vv = S.KVCache.contiguous(dv["k"]), S.KVCache.contiguous(dv["v"])
        out = torch.empty((cfg.B, cfg.Hq, d), dtype=torch.bfloat16, device="cuda")
        ws = S.alloc_workspace(sh, cap, 3)
        S.sparse_decode(sh, dv["q"], kk, vv, idx_d, cnt_d, dv["seqlens"], out, ws, num_split=3)
        outs.append(out)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16)), "paged != contiguous"
    # paged kcomp equals contiguous kcomp
    kcs = []
    for kk in (S.KVCache.contiguous(dv["k"]), S.KVCache.paged(to_dev_bf16(pool_k), tbl)):
        kc = torch.zeros((cfg.B, Hkv, inp.max_blocks, 64), dtype=torch.bfloat16, device="cuda")
        S.kcomp_update(sh, kk, dv["seqlens"], torch.zeros(cfg.B, Hkv, dtype=torch.int32, device="cuda"), dv["w_k"], kc)
        kcs.append(kc)
    assert torch.equal(kcs[0].view(torch.int16), kcs[1].view(torch.int16)), "paged kcomp != contiguous"


def test_sparse_decode_token_major_layout():
    """A [B, T, Hkv, d] cache (token-major, vLLM-style strides) gives the same result."""
    blk, d, g, Hkv = 64, 128, 4, 2
    cfg = config(1, B=2, Hq=g * Hkv, Hkv=Hkv, head_dim=d, gate_dim=64, block=blk, seed=1414)
    lengths = [6 * blk + 9, 4 * blk]
    inp = make_inputs(cfg, lengths=lengths)
    dv = _dev(inp)
    sh = _shape(cfg, inp)
    cap = 6
    idx, cnt = make_block_lists(9, lengths, Hkv, blk, cap, density=0.7)
    idx_d, cnt_d = torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()
    outs = []
    for tm in (False, True):
        if tm:
            k4 = dv["k"].permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
            v4 = dv["v"].permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
        else:
            k4, v4 = dv["k"], dv["v"]
        out = torch.empty((cfg.B, cfg.Hq, d), dtype=torch.bfloat16, device="cuda")
        S.sparse_decode(sh, dv["q"], S.KVCache.contiguous(k4), S.KVCache.contiguous(v4), idx_d, cnt_d,
                        dv["seqlens"], out, S.alloc_workspace(sh, cap, 2), num_split=2)
        outs.append(out)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))


def test_sparse_decode_edges_and_device_errors():
    blk, d, g, Hkv = 64, 128, 4, 1
    cfg = config(1, B=4, Hq=g, Hkv=Hkv, head_dim=d, gate_dim=64, block=blk, seed=2121)
    lengths = [1, blk - 1, 3 * blk, 2 * blk + 1]
    inp = make_inputs(cfg, lengths=lengths, tail="nan")
    dv = _dev(inp)
    sh = _shape(cfg, inp)
    cap = 4
    idx = np.full((cfg.B, Hkv, cap), -1, np.int32)
    cnt = np.zeros((cfg.B, Hkv), np.int32)
    idx[0, 0, :1] = [0]; cnt[0, 0] = 1          # L=1: a single token
    idx[1, 0, :1] = [0]; cnt[1, 0] = 1          # L < b: only the partial block
    cnt[2, 0] = 0                               # empty list
    idx[3, 0, :2] = [0, 2]; cnt[3, 0] = 2       # full block + one-token partial
    for ns in (1, 2, 0, -1):
        out = torch.full((cfg.B, cfg.Hq, d), 7.0, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((cfg.B, cfg.Hq), dtype=torch.float32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        S.sparse_decode(sh, dv["q"], S.KVCache.contiguous(dv["k"]), S.KVCache.contiguous(dv["v"]),
                        torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(), dv["seqlens"], out,
                        S.alloc_workspace(sh, cap, ns), num_split=ns, lse=lse, err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        o = f64(bf16_bits(out))
        lh = lse.cpu().numpy()
        assert np.all(o[2] == 0) and np.all(np.isneginf(lh[2])), "empty list must give 0 / -inf"
        for b in (0, 1, 3):
            ro, rl = OracleBH(inp, b, 0).attention(lengths[b], inp.q, gpu_list(idx[b, 0], cnt[b, 0]))
            check_attention(o[b], ro, f"edge b{b}")
            check_lse(lh[b], rl, f"edge b{b}")
    # out-of-range block index and count above capacity: flagged, skipped, no trap
    bad_idx = idx.copy()
    bad_cnt = cnt.copy()
    bad_idx[3, 0, :2] = [0, 99]
    bad_cnt[2, 0] = cap + 5
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty((cfg.B, cfg.Hq, d), dtype=torch.bfloat16, device="cuda")
    S.sparse_decode(sh, dv["q"], S.KVCache.contiguous(dv["k"]), S.KVCache.contiguous(dv["v"]),
                    torch.from_numpy(bad_idx).cuda(), torch.from_numpy(bad_cnt).cuda(), dv["seqlens"], out,
                    S.alloc_workspace(sh, cap, 1), num_split=1, err=err)
    torch.cuda.synchronize()
    e = int(err.item())
    assert e & S.DEVERR_BLOCK_INDEX and e & S.DEVERR_COUNT
    ro, _ = OracleBH(inp, 3, 0).attention(lengths[3], inp.q, [0])
    check_attention(f64(bf16_bits(out))[3], ro, "skipped bad index")


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

    for fused in (True, False):
        runs = []
        for _ in range(2):
            kc = torch.zeros((cfg.B, Hkv, nb, dg), dtype=torch.bfloat16, device="cuda")
            valid = torch.zeros(cfg.B, Hkv, dtype=torch.int32, device="cuda")
            st = S.DecodeStep(sh, kv_k, kv_v, dv["w_q"], dv["w_k"], kc, valid, mode=S.SELECT_TOPK,
                              token_budget=4 * blk, num_split=2)
            st.run(dv["q"], dv["seqlens"], fused=fused)
            torch.cuda.synchronize()
            assert int(st.err.item()) == 0
            runs.append(st)
        a, b = runs
        for name in ("kcomp", "valid_blocks", "block_idx", "block_cnt", "out", "lse"):
            assert torch.equal(bits(getattr(a, name)), bits(getattr(b, name))), f"fused={fused}: {name}"
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


def test_host_argument_errors():
    sh = S.Shape(2, 8, 2, 128, 128, 64, 16)
    t = torch.zeros(2, 2, 1024, 128, dtype=torch.bfloat16, device="cuda")
    lg = torch.zeros(2, 2, 16, dtype=torch.float32, device="cuda")
    sl = torch.zeros(2, dtype=torch.int32, device="cuda")
    with pytest.raises(S.SeerError) as ei:
        S.select_blocks(sh, lg, sl, S.SELECT_TOPK, torch.zeros(2, 2, 3, dtype=torch.int32, device="cuda"),
                        torch.zeros(2, 2, dtype=torch.int32, device="cuda"), token_budget=64 * 8)
    assert ei.value.status == 3
    with pytest.raises(S.SeerError) as ei:
        S.sparse_decode(sh, torch.zeros(2, 8, 128, dtype=torch.bfloat16, device="cuda"),
                        S.KVCache.contiguous(t[:, :, :, :]), S.KVCache.contiguous(t),
                        torch.zeros(2, 2, 4, dtype=torch.int32, device="cuda"),
                        torch.zeros(2, 2, dtype=torch.int32, device="cuda"), sl,
                        torch.zeros(2, 8, 128, dtype=torch.bfloat16, device="cuda"), None, num_split=2)
    assert ei.value.status == 1 and "workspace" in str(ei.value)
