"""Per-kernel parity of the CUDA path against the CPU oracle, called through the C ABI.

Sizes are small enough for the float64 oracle to finish in seconds while still
spanning several tiles, splits and a ragged tail; edge cases cover empty
lists, lengths shorter than one block, NaN-poisoned cache tails, paged
layouts and out-of-range indices (sizes up to the largest accepted are in
test_zzz_limits_and_edges.py).
"""

import numpy as np
import pytest
import torch

from oracle import seer_oracle as O
from seer_harness import (OracleBH, bf16_bits, check_attention, check_kcomp_rows, check_logits, check_lse,
                          check_selection, f64, gpu_list, to_dev_bf16)
from synthetic import config, make_block_lists, make_inputs, make_logits, paged_view

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

@pytest.mark.parametrize("d,blk,g", [(128, 64, 4), (128, 128, 5), (64, 64, 8), (64, 128, 1), (128, 64, 2)])
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


@pytest.mark.parametrize("ns", [3, 0, -1])
def test_sparse_decode_paged_matches_contiguous(ns):
    """A paged cache (shuffled pages, NaN in every unused page) against the oracle, under each
    schedule; the paged and contiguous results are also bit-identical (same tiles, same order)."""
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
        lse = torch.empty((cfg.B, cfg.Hq), dtype=torch.float32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        ws = S.alloc_workspace(sh, cap, ns)
        S.sparse_decode(sh, dv["q"], kk, vv, idx_d, cnt_d, dv["seqlens"], out, ws, num_split=ns, lse=lse, err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0, f"{layout}: device error word {int(err.item())}"
        o, lh = f64(bf16_bits(out)), lse.cpu().numpy()
        for b in range(cfg.B):
            for h in range(Hkv):
                ro, rl = OracleBH(inp, b, h).attention(lengths[b], inp.q, gpu_list(idx[b, h], cnt[b, h]))
                check_attention(o[b, h * g:(h + 1) * g], ro, f"{layout} ns={ns} b{b} h{h}")
                check_lse(lh[b, h * g:(h + 1) * g], rl, f"{layout} ns={ns} b{b} h{h}")
        outs.append(out)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16)), "paged != contiguous"
    # the paged cache rebuild against the oracle's cache, and bit-identical to the contiguous one
    kcs = []
    for kk in (S.KVCache.contiguous(dv["k"]), S.KVCache.paged(to_dev_bf16(pool_k), tbl)):
        kc = torch.zeros((cfg.B, Hkv, inp.max_blocks, 64), dtype=torch.bfloat16, device="cuda")
        S.kcomp_update(sh, kk, dv["seqlens"], torch.zeros(cfg.B, Hkv, dtype=torch.int32, device="cuda"), dv["w_k"], kc)
        kcs.append(kc)
    got = bf16_bits(kcs[1])
    for b in range(cfg.B):
        for h in range(Hkv):
            nfull = lengths[b] // blk
            check_kcomp_rows(got[b, h, :nfull], OracleBH(inp, b, h).kcomp(lengths[b])[:nfull], f"paged kcomp b{b} h{h}")
    assert torch.equal(kcs[0].view(torch.int16), kcs[1].view(torch.int16)), "paged kcomp != contiguous"


def test_sparse_decode_token_major_layout():
    """A [B, T, Hkv, d] cache (token-major, vLLM-style strides) against the oracle; it also
    gives the same bits as the head-major layout."""
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
        lse = torch.empty((cfg.B, cfg.Hq), dtype=torch.float32, device="cuda")
        S.sparse_decode(sh, dv["q"], S.KVCache.contiguous(k4), S.KVCache.contiguous(v4), idx_d, cnt_d,
                        dv["seqlens"], out, S.alloc_workspace(sh, cap, 2), num_split=2, lse=lse)
        torch.cuda.synchronize()
        o, lh = f64(bf16_bits(out)), lse.cpu().numpy()
        for b in range(cfg.B):
            for h in range(Hkv):
                ro, rl = OracleBH(inp, b, h).attention(lengths[b], inp.q, gpu_list(idx[b, h], cnt[b, h]))
                check_attention(o[b, h * g:(h + 1) * g], ro, f"token-major={tm} b{b} h{h}")
                check_lse(lh[b, h * g:(h + 1) * g], rl, f"token-major={tm} b{b} h{h}")
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
