"""K Compression Cache from running block statistics (seer_kcomp_append, seer_kcomp_state_init)
against the CPU oracle: the rolling form token by token, and the block-pooling rebuild it must
equal.  Cache rows use the cache update's tolerance (one bf16 ulp, 98 % bit-exact); running max
and min are exact, running sums within fp32 accumulation error."""

import numpy as np
import pytest
import torch

from oracle import seer_oracle as O
from seer_harness import OracleBH, bf16_bits, check_kcomp_rows, f64, to_dev_bf16
from synthetic import config, make_inputs, paged_view

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import block_sparse_attention_attngate_b200 as S


def _setup(d, dg, blk, lengths, seed, Hkv=2):
    cfg = config(1, B=len(lengths), Hq=4 * Hkv, Hkv=Hkv, head_dim=d, gate_dim=dg, block=blk, seed=seed)
    inp = make_inputs(cfg, lengths=lengths)
    sh = S.Shape(cfg.B, cfg.Hq, cfg.Hkv, d, dg, blk, inp.max_blocks, rope_base=cfg.rope_base)
    return cfg, inp, sh


def _k_new(inp, tok):
    """[B, Hkv, d] bf16 keys of token tok[b] (zeros where tok[b] < 0)."""
    B, Hkv = inp.k.shape[0], inp.k.shape[1]
    out = np.zeros((B, Hkv, inp.k.shape[3]), dtype=np.uint16)
    for b in range(B):
        if tok[b] >= 0:
            out[b] = inp.k[b, :, tok[b]]
    return to_dev_bf16(out)


def _check_state(st, ref, what):
    st = st.cpu().numpy().astype(np.float64)
    assert np.array_equal(st[0], ref[0]), f"{what}: running max"
    assert np.array_equal(st[1], ref[1]), f"{what}: running min"
    assert np.all(np.abs(st[2] - ref[2]) <= 1e-5 * (np.abs(ref[2]) + 1.0)), f"{what}: running sum"


@pytest.mark.parametrize("d,dg,blk", [(128, 128, 64), (128, 64, 128), (64, 128, 64)])
def test_append_from_empty_vs_oracle(d, dg, blk):
    lengths = [2 * blk + 37, blk + 5, 3]
    cfg, inp, sh = _setup(d, dg, blk, lengths, seed=900 + d + dg + blk)
    B, Hkv, nb = cfg.B, cfg.Hkv, inp.max_blocks
    kc = torch.zeros((B, Hkv, nb, dg), dtype=torch.bfloat16, device="cuda")
    valid = torch.zeros(B, Hkv, dtype=torch.int32, device="cuda")
    state = torch.full((B, Hkv, 3, d), float("nan"), dtype=torch.float32, device="cuda")   # restarted
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    w_k = to_dev_bf16(inp.w_k)
    ref_state = np.zeros((B, Hkv, 3, d))
    ref_kc = np.full((B, Hkv, nb, dg), np.nan)
    ref_valid = np.zeros((B, Hkv), dtype=int)
    for s in range(1, max(lengths) + 1):
        now = np.array([s if s <= L else 0 for L in lengths], dtype=np.int32)   # 0: nothing appended
        S.kcomp_append(sh, _k_new(inp, now - 1), torch.from_numpy(now).cuda(), state, valid, w_k, kc, err=err)
        for b in range(B):
            if now[b] <= 0:
                continue
            for h in range(Hkv):
                ref_valid[b, h] = O.kcomp_append(ref_state[b, h], f64(inp.k[b, h, now[b] - 1]), int(now[b]),
                                                 int(ref_valid[b, h]), f64(inp.w_k[h]), ref_kc[b, h], blk,
                                                 cfg.rope_base)
        if s % blk == 0 or s == max(lengths):
            torch.cuda.synchronize()
            assert valid.cpu().numpy().tolist() == ref_valid.tolist(), f"fill counts after step {s}"
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = bf16_bits(kc)
    for b in range(B):
        for h in range(Hkv):
            n = lengths[b] // blk
            assert n == ref_valid[b, h]
            frac = check_kcomp_rows(got[b, h, :n], ref_kc[b, h, :n], f"b{b} h{h}")
            assert frac >= 0.98, f"b{b} h{h}: only {frac:.3f} bit-exact"
            assert np.all(got[b, h, n:] == 0), "an entry was written before its block completed"
            # the rolling form equals the block-pooling rebuild of the same keys
            rebuilt = OracleBH(inp, b, h).kcomp(lengths[b])
            check_kcomp_rows(got[b, h, :n], rebuilt[:n], f"rebuild b{b} h{h}")
            _check_state(state[b, h], ref_state[b, h], f"b{b} h{h}")


@pytest.mark.parametrize("paged", [False, True])
def test_resume_mid_block_after_prefill(paged):
    blk, d, dg = 64, 128, 128
    prefill = np.array([3 * blk + 20, 2 * blk - 1, 4 * blk], dtype=np.int32)
    extra = blk + 10
    cfg, inp, sh = _setup(d, dg, blk, [int(L) + extra for L in prefill], seed=951)
    B, Hkv, nb = cfg.B, cfg.Hkv, inp.max_blocks
    if paged:
        pool, table = paged_view(inp.k, blk, seed=9)
        kv = S.KVCache.paged(to_dev_bf16(pool), torch.from_numpy(table).cuda())
    else:
        kv = S.KVCache.contiguous(to_dev_bf16(inp.k))
    w_k = to_dev_bf16(inp.w_k)
    kc = torch.zeros((B, Hkv, nb, dg), dtype=torch.bfloat16, device="cuda")
    valid = torch.zeros(B, Hkv, dtype=torch.int32, device="cuda")
    state = torch.full((B, Hkv, 3, d), 7.0, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    sl0 = torch.from_numpy(prefill).cuda()
    S.kcomp_update(sh, kv, sl0, valid, w_k, kc)            # prefill: the full blocks
    S.kcomp_state_init(sh, kv, sl0, state, err=err)        # the current block's statistics
    torch.cuda.synchronize()
    for b in range(B):
        t0 = int(prefill[b]) // blk * blk
        for h in range(Hkv):
            keys = f64(inp.k[b, h, t0:int(prefill[b])])
            if len(keys):
                ref = np.stack([keys.max(0), keys.min(0), keys.sum(0)])
            else:
                ref = np.stack([np.full(d, -np.inf), np.full(d, np.inf), np.zeros(d)])
            _check_state(state[b, h], ref, f"init b{b} h{h}")
    for i in range(extra):
        now = prefill + i + 1
        S.kcomp_append(sh, _k_new(inp, now - 1), torch.from_numpy(now).cuda(), state, valid, w_k, kc, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    final = prefill + extra
    assert valid.cpu().numpy().tolist() == [[int(L) // blk] * Hkv for L in final]
    got = bf16_bits(kc)
    for b in range(B):
        for h in range(Hkv):
            n = int(final[b]) // blk
            check_kcomp_rows(got[b, h, :n], OracleBH(inp, b, h).kcomp(int(final[b]))[:n], f"b{b} h{h}")
            assert np.all(got[b, h, n:] == 0)


def test_append_out_of_order_is_reported():
    """A block completing while earlier entries are missing writes nothing and sets DEVERR_COUNT."""
    blk, d, dg = 64, 128, 128
    cfg, inp, sh = _setup(d, dg, blk, [2 * blk], seed=977, Hkv=1)
    kc = torch.zeros((1, 1, inp.max_blocks, dg), dtype=torch.bfloat16, device="cuda")
    valid = torch.zeros(1, 1, dtype=torch.int32, device="cuda")   # entry 0 was never built
    state = torch.zeros((1, 1, 3, d), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    w_k = to_dev_bf16(inp.w_k)
    now = np.array([2 * blk], dtype=np.int32)                     # completes block 1
    S.kcomp_append(sh, _k_new(inp, now - 1), torch.from_numpy(now).cuda(), state, valid, w_k, kc, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & S.DEVERR_COUNT
    assert int(valid.item()) == 0
    assert np.all(bf16_bits(kc) == 0)


def test_decode_step_with_running_statistics():
    """DecodeStep keeping its cache from running block statistics, next to the same step reading
    the K cache, through a block boundary: fill counts equal, cache rows within the cache
    tolerance of each other, and the same block lists and outputs."""
    blk, d, dg, Hkv = 64, 128, 128, 2
    prefill = np.array([5 * blk + 40, 3 * blk - 2], dtype=np.int32)
    steps = blk // 2 + 10                      # both sequences complete a block on the way
    cfg, inp, sh = _setup(d, dg, blk, [int(L) + steps for L in prefill], seed=991, Hkv=Hkv)
    B, nb = cfg.B, inp.max_blocks
    kv_k = S.KVCache.contiguous(to_dev_bf16(inp.k))
    kv_v = S.KVCache.contiguous(to_dev_bf16(inp.v))
    w_q, w_k, q = to_dev_bf16(inp.w_q), to_dev_bf16(inp.w_k), to_dev_bf16(inp.q)
    caches, valids = [], []
    sl0 = torch.from_numpy(prefill).cuda()
    for _ in range(2):
        kc = torch.zeros((B, Hkv, nb, dg), dtype=torch.bfloat16, device="cuda")
        valid = torch.zeros(B, Hkv, dtype=torch.int32, device="cuda")
        S.kcomp_update(sh, kv_k, sl0, valid, w_k, kc)          # prefill: the full blocks
        caches.append(kc)
        valids.append(valid)
    state = S.alloc_kcomp_state(sh)
    S.kcomp_state_init(sh, kv_k, sl0, state)
    rolling = S.DecodeStep(sh, kv_k, kv_v, w_q, w_k, caches[0], valids[0], mode=S.SELECT_TOPK,
                           token_budget=8 * blk, kcomp_state=state)
    reading = S.DecodeStep(sh, kv_k, kv_v, w_q, w_k, caches[1], valids[1], mode=S.SELECT_TOPK,
                           token_budget=8 * blk)
    for i in range(steps):
        L = prefill + i + 1
        sl = torch.from_numpy(L).cuda()
        rolling.run(q, sl, k_new=_k_new(inp, L - 1))
        reading.run(q, sl)
    torch.cuda.synchronize()
    assert int(rolling.err.item()) == 0 and int(reading.err.item()) == 0
    final = prefill + steps
    assert valids[0].cpu().tolist() == valids[1].cpu().tolist() == [[int(L) // blk] * Hkv for L in final]
    a, b_ = bf16_bits(caches[0]), bf16_bits(caches[1])
    from seer_harness import bf16_to_f64_bits
    for b in range(B):
        for h in range(Hkv):
            n = int(final[b]) // blk
            check_kcomp_rows(a[b, h, :n], bf16_to_f64_bits(b_[b, h, :n]), f"b{b} h{h}")
    assert torch.equal(rolling.block_cnt, reading.block_cnt)
    assert torch.equal(rolling.block_idx, reading.block_idx)
    assert torch.equal(rolling.out, reading.out)
    with pytest.raises(ValueError):
        rolling.run(q, sl)                     # a step with running statistics needs k_new
