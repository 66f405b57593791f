"""End-to-end parity of the five decode workloads, at their full sizes, in the launch
configuration the benchmark uses (DecodeStep with the automatic split count).

Per workload:
  * kcomp (GPU prefill rebuild) within one bf16 ulp of the oracle cache;
  * gate logits of the GPU gate kernel on the oracle's cache within the logit tolerance;
  * GPU selection on the oracle's logits identical to the oracle's selection;
  * GPU attention on the oracle's block lists within the attention tolerance;
  * the whole GPU step (GPU cache -> GPU logits -> GPU lists -> GPU attention)
    against the whole oracle step: lists equal except at the cutoff (a block whose
    oracle logit sits within twice the logit tolerance of the selection boundary),
    outputs within tolerance wherever the lists agree.
"""

import math

import numpy as np
import pytest
import torch

from oracle import seer_oracle as O
from seer_harness import (LOGIT_RTOL, OracleBH, bf16_bits, check_attention, check_kcomp_rows, check_logits,
                          check_logits_e2e, check_lse, check_selection, draw_workers, e2e_logit_bound, f64, gpu_list,
                          to_dev_bf16)
from synthetic import (SWEEP_SPARSITIES, bf16_bits_from_f32, config, make_inputs, make_step_query,
                       scale_gate_weights)
from synthetic.inputs import sweep_budget

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import block_sparse_attention_attngate_b200 as S


class Problem:
    def __init__(self, inp, w_q_bits=None):
        self.inp = inp
        c = inp.cfg
        self.cfg = c
        self.sh = S.Shape(c.B, c.Hq, c.Hkv, c.head_dim, c.gate_dim, c.block, inp.max_blocks, c.rope_base)
        self.k = to_dev_bf16(inp.k)
        self.v = to_dev_bf16(inp.v)
        self.w_q_bits = inp.w_q if w_q_bits is None else w_q_bits
        self.w_q = to_dev_bf16(self.w_q_bits)
        self.w_k = to_dev_bf16(inp.w_k)
        self.kc = torch.zeros(c.B, c.Hkv, inp.max_blocks, c.gate_dim, dtype=torch.bfloat16, device="cuda")
        self.valid = torch.zeros(c.B, c.Hkv, dtype=torch.int32, device="cuda")
        self.obh = {(b, h): OracleBH(inp, b, h) for b in range(c.B) for h in range(c.Hkv)}

    def step(self, mode, budget=0, tau=0.0, **kw):
        return S.DecodeStep(self.sh, S.KVCache.contiguous(self.k), S.KVCache.contiguous(self.v), self.w_q, self.w_k,
                            self.kc, self.valid, mode=mode, token_budget=budget, tau=tau, **kw)


def _boundary_ok(z, gpu, ref, mode, bound, k_blocks=0, tau=0.0):
    """Every block on which the two lists differ sits at the selection boundary: its oracle logit
    is within twice the end-to-end logit bound of the cutoff logit."""
    diff = set(gpu) ^ set(ref)
    if not diff:
        return True
    nfull = len(z)
    tol = 2 * float(np.max(bound)) if nfull else 0.0
    if mode == "topk":
        srt = np.sort(z)[::-1]
        cut = srt[min(k_blocks, nfull) - 1] if k_blocks else np.inf
    else:
        m = z.max()
        cut = m + math.log(tau * np.exp(z - m).sum())
    return all(n < nfull and abs(z[n] - cut) <= tol for n in diff)


def _run_and_check(P, step, q_bits, lengths, mode, k_blocks=0, tau=0.0, pairs=None, attn_pairs=None, label=""):
    """One GPU step vs the oracle; returns (selection mismatches against the all-oracle step,
    pairs compared, the oracle's lists).

    Per (b, h):
      * the GPU logits against the oracle's logits evaluated on the cache rows the GPU step
        itself read (widened exactly from bf16), at the plain logit tolerance;
      * the GPU list against the oracle's selection on those same logits: identical, except a
        block whose logit sits within twice the logit tolerance of the cut-off;
      * the GPU list against the all-oracle step (oracle cache): identical except at the
        cut-off (the two caches may round an entry one ulp apart);
      * the GPU output and LSE against the oracle's attention over the GPU's own list.
    """
    c = P.cfg
    seq = torch.from_numpy(np.asarray(lengths, np.int32)).cuda()
    q = to_dev_bf16(q_bits)
    out = step.run(q, seq)
    torch.cuda.synchronize()
    assert int(step.err.item()) == 0, f"{label}: device error word {int(step.err.item())}"
    idx, cnt = step.block_idx.cpu().numpy(), step.block_cnt.cpu().numpy()
    lg = step.logits.cpu().numpy()
    kc_gpu = f64(bf16_bits(step.kcomp))   # the cache rows this step's gate read
    o = f64(bf16_bits(out))
    lse = step.lse.cpu().numpy()
    pairs = pairs or sorted(P.obh)
    attn_pairs = set(attn_pairs if attn_pairs is not None else pairs)
    mism = 0
    oracle_lists = {}
    for (b, h) in pairs:
        L = int(lengths[b])
        ob = P.obh[(b, h)]
        ref = ob.step(L, q_bits, mode, k_blocks=k_blocks, tau=tau, w_q_bits=P.w_q_bits)
        nfull = L // c.block
        got = gpu_list(idx[b, h], cnt[b, h])
        # logits and selection on the GPU's own cache rows
        z_own = O.gate_logits(ref["q_gate"], kc_gpu[b, h], L, c.block)
        check_logits(lg[b, h, :nfull], z_own, f"{label} logits on the GPU cache b{b} h{h}")
        own = O.select_topk(z_own, k_blocks, L, c.block) if mode == "topk" else O.select_threshold(z_own, tau, L, c.block)
        if nfull:
            rms = math.sqrt(float(np.mean(z_own ** 2)))
            own_bound = LOGIT_RTOL * np.maximum(np.abs(z_own), rms)
            assert _boundary_ok(z_own, got, own, mode, own_bound, k_blocks, tau), \
                f"{label} b{b} h{h}: list differs from the selection on the GPU cache away from the cut-off: " \
                f"{sorted(set(got) ^ set(own))}"
        else:
            assert got == own, f"{label} b{b} h{h}: {got} vs {own}"
        # against the all-oracle step
        bound = e2e_logit_bound(ref["q_gate"], ob.kcomp(L)[:nfull], ref["logits"])
        check_logits_e2e(lg[b, h, :nfull], ref["logits"], bound, f"{label} e2e logits b{b} h{h}")
        oracle_lists[(b, h)] = ref["blocks"]
        if got != ref["blocks"]:
            mism += 1
            assert _boundary_ok(ref["logits"], got, ref["blocks"], mode, bound, k_blocks, tau), \
                f"{label} b{b} h{h}: lists differ away from the cutoff: {sorted(set(got) ^ set(ref['blocks']))}"
        if (b, h) in attn_pairs:
            g = c.g
            ro, rl = (ref["o"], ref["lse"]) if got == ref["blocks"] else ob.attention(L, q_bits, got)
            check_attention(o[b, h * g:(h + 1) * g], ro, f"{label} e2e out b{b} h{h}")
            check_lse(lse[b, h * g:(h + 1) * g], rl, f"{label} e2e lse b{b} h{h}")
    return mism, len(pairs), oracle_lists


def _isolated_checks(P, q_bits, lengths, mode, k_blocks=0, tau=0.0, pairs=None, attn_pairs=None, label=""):
    """Each kernel on the oracle's own inputs: gate on oracle kcomp, select on oracle logits,
    decode on oracle lists."""
    c = P.cfg
    nb = P.inp.max_blocks
    pairs = pairs or sorted(P.obh)
    attn_pairs = attn_pairs if attn_pairs is not None else pairs
    ref_kc = np.zeros((c.B, c.Hkv, nb, c.gate_dim), np.uint16)
    ref_lg = np.full((c.B, c.Hkv, nb), -np.inf, np.float32)
    refs = {}
    for (b, h) in pairs:
        L = int(lengths[b])
        ob = P.obh[(b, h)]
        ref = ob.step(L, q_bits, mode, k_blocks=k_blocks, tau=tau, w_q_bits=P.w_q_bits)
        refs[(b, h)] = ref
        nfull = L // c.block
        ref_kc[b, h, :nfull] = bf16_bits_from_f32(ob.kcomp(L)[:nfull].astype(np.float32))
        ref_lg[b, h, :nfull] = ref["logits"].astype(np.float32)
    seq = torch.from_numpy(np.asarray(lengths, np.int32)).cuda()
    # gate on the oracle cache
    logits = torch.empty(c.B, c.Hkv, nb, dtype=torch.float32, device="cuda")
    S.gate_score(P.sh, to_dev_bf16(q_bits), P.w_q, to_dev_bf16(ref_kc), seq, logits)
    lg = logits.cpu().numpy()
    for (b, h) in pairs:
        nfull = int(lengths[b]) // c.block
        check_logits(lg[b, h, :nfull], refs[(b, h)]["logits"], f"{label} gate b{b} h{h}")
    # select on the oracle logits (as float32, the kernel's input type)
    cap = nb if mode != "topk" else min(nb, k_blocks + 1)
    idx = torch.empty(c.B, c.Hkv, cap, dtype=torch.int32, device="cuda")
    cnt = torch.empty(c.B, c.Hkv, dtype=torch.int32, device="cuda")
    tau32 = float(np.float32(tau))
    S.select_blocks(P.sh, torch.from_numpy(ref_lg).cuda(), seq, S.SELECT_TOPK if mode == "topk" else S.SELECT_THRESHOLD,
                    idx, cnt, token_budget=k_blocks * c.block, tau=tau32)
    ih, ch = idx.cpu().numpy(), cnt.cpu().numpy()
    lists = np.full((c.B, c.Hkv, cap), -1, np.int32)
    counts = np.zeros((c.B, c.Hkv), np.int32)
    for (b, h) in pairs:
        L = int(lengths[b])
        z32 = ref_lg[b, h, :L // c.block].astype(np.float64)
        want = O.select_topk(z32, k_blocks, L, c.block) if mode == "topk" else O.select_threshold(z32, tau32, L, c.block)
        check_selection(gpu_list(ih[b, h], ch[b, h]), want, O.gate_scores(z32), tau32 if mode != "topk" else None,
                        f"{label} select b{b} h{h}")
        lists[b, h, :len(want)] = want
        counts[b, h] = len(want)
    # decode on the oracle lists
    out = torch.empty(c.B, c.Hq, c.head_dim, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(c.B, c.Hq, dtype=torch.float32, device="cuda")
    ns = 0   # the balanced schedule (the default of DecodeStep and the benchmark)
    S.sparse_decode(P.sh, to_dev_bf16(q_bits), S.KVCache.contiguous(P.k), S.KVCache.contiguous(P.v),
                    torch.from_numpy(lists).cuda(), torch.from_numpy(counts).cuda(), seq, out,
                    S.alloc_workspace(P.sh, cap, ns), num_split=ns, lse=lse)
    o = f64(bf16_bits(out))
    lh = lse.cpu().numpy()
    g = c.g
    for (b, h) in attn_pairs:
        ro, rl = P.obh[(b, h)].attention(int(lengths[b]), q_bits, gpu_list(lists[b, h], counts[b, h]))
        check_attention(o[b, h * g:(h + 1) * g], ro, f"{label} decode b{b} h{h}")
        check_lse(lh[b, h * g:(h + 1) * g], rl, f"{label} decode lse b{b} h{h}")


def _check_kcomp(P, lengths, pairs=None):
    c = P.cfg
    got = bf16_bits(P.kc)
    exact = []
    for (b, h) in (pairs or sorted(P.obh)):
        nfull = int(lengths[b]) // c.block
        ref = P.obh[(b, h)].kcomp(int(lengths[b]))[:nfull]
        exact.append(check_kcomp_rows(got[b, h, :nfull], ref, f"kcomp b{b} h{h}"))
    assert min(exact) >= 0.98, f"kcomp: only {min(exact):.3f} of entries bit-exact"


def _prefill(P, lengths):
    S.kcomp_update(P.sh, S.KVCache.contiguous(P.k), torch.from_numpy(np.asarray(lengths, np.int32)).cuda(), P.valid,
                   P.w_k, P.kc)
    torch.cuda.synchronize()


@pytest.mark.parametrize("cid,single", [(1, False), (2, False), (3, False), (1, True), (2, True), (3, True)])
def test_topk_workload(cid, single):
    """single: the whole step as one launch (seer_decode_step); else the plan and the decode as two
    launches (the default)."""
    cfg = config(cid)
    inp = make_inputs(cfg, tail="nan", workers=draw_workers())
    P = Problem(inp)
    L = inp.seqlens
    _prefill(P, L)
    _check_kcomp(P, L)
    kb = cfg.topk_blocks
    _isolated_checks(P, inp.q, L, "topk", k_blocks=kb, label=f"cfg{cid}")
    step = P.step(S.SELECT_TOPK, budget=cfg.budget, single_launch=single)
    assert step.single_launch == single
    mism, n, _ = _run_and_check(P, step, inp.q, L, "topk", k_blocks=kb, label=f"cfg{cid}")
    assert mism <= max(1, n // 20), f"cfg{cid}: {mism}/{n} lists differ (all at the cutoff)"
    if cfg.hot_blocks:
        # planted q-aligned blocks raise their logits: most should make the top-k
        idx, cnt = step.block_idx.cpu().numpy(), step.block_cnt.cpu().numpy()
        hits = sum(len(set(inp.hot[(b, h)]) & set(gpu_list(idx[b, h], cnt[b, h])))
                   for (b, h) in inp.hot)
        total = sum(len(v) for v in inp.hot.values())
        print(f"cfg{cid}: planted blocks selected {hits}/{total}")


def test_paged_ragged_workload():
    """The Qwen3-14B-shaped ragged batch (g = 5, block 128, lengths never a multiple of 128, so the
    partial block is forced on; four of its sequences) on a paged cache: pages shuffled by a seeded
    permutation, NaN in every unused page and past each length.  Cache rebuild, logits, lists and
    outputs through DecodeStep against the oracle, as for the contiguous workloads."""
    from synthetic import paged_view
    cfg = config(3, B=4)
    inp = make_inputs(cfg, tail="nan", workers=draw_workers())
    P = Problem(inp)
    L = inp.seqlens
    assert np.all(L % cfg.block != 0)
    pool_k, table = paged_view(inp.k, cfg.block, seed=31)
    pool_v, _ = paged_view(inp.v, cfg.block, seed=31)
    tbl = torch.from_numpy(table).cuda()
    kk = S.KVCache.paged(to_dev_bf16(pool_k), tbl)
    vv = S.KVCache.paged(to_dev_bf16(pool_v), tbl)
    S.kcomp_update(P.sh, kk, torch.from_numpy(L).cuda(), P.valid, P.w_k, P.kc)
    torch.cuda.synchronize()
    _check_kcomp(P, L)
    for single in (False, True):
        step = S.DecodeStep(P.sh, kk, vv, P.w_q, P.w_k, P.kc, P.valid, mode=S.SELECT_TOPK, token_budget=cfg.budget,
                            num_split=-1, single_launch=single)
        mism, n, _ = _run_and_check(P, step, inp.q, L, "topk", k_blocks=cfg.topk_blocks,
                                    label=f"paged cfg3 single={single}")
        assert mism <= max(1, n // 20), f"paged cfg3: {mism}/{n} lists differ (all at the cutoff)"
        cnt = step.block_cnt.cpu().numpy()
        assert np.all(cnt == cfg.topk_blocks + 1), "every list holds k blocks plus the forced partial block"


def _step_loop(P, step, L0, steps, mode, k_blocks=0, tau=0.0, label=""):
    """Decode `steps` appended tokens (step s sees L0 + s + 1): every step against the oracle, the
    cache entries below the previous fill count frozen, the fill counts advancing as blocks fill."""
    c = P.cfg
    for s_ in range(steps):
        L = L0 + s_ + 1
        q_bits = make_step_query(c, s_)
        before = P.kc.clone()
        prev = torch.from_numpy(((L - 1) // c.block).astype(np.int32))
        mism, n, _ = _run_and_check(P, step, q_bits, L, mode, k_blocks=k_blocks, tau=tau, label=f"{label} s{s_}")
        assert mism <= max(1, n // 20)
        for b in range(c.B):
            pv = int(prev[b])
            assert torch.equal(before[b, :, :pv].view(torch.int16), P.kc[b, :, :pv].view(torch.int16)), \
                f"{label} s{s_}: frozen entries of b{b} changed"
        assert P.valid.cpu().tolist() == [[int(x) // c.block] * c.Hkv for x in L], f"{label} s{s_}: fill counts"
    _check_kcomp(P, L0 + steps)


def test_single_launch_steps_across_block_fills():
    """The one-launch step over appended tokens: blocks fill mid-run, so the launch's planning
    phase writes new cache entries before its gate reads them; the ready flags must come back to
    zero after every launch (each step depends on it)."""
    blk = 64
    L0 = np.array([40 * blk - 3, 33 * blk + 61, 17 * blk - 1], dtype=np.int32)
    steps = 6
    cfg = config(2, B=3, steps=steps + 1)   # the loop's last length is L0 + steps
    inp = make_inputs(cfg, lengths=list(L0), tail="nan")
    P = Problem(inp)
    _prefill(P, L0)
    step = P.step(S.SELECT_TOPK, budget=cfg.budget, num_split=-1, single_launch=True)
    _step_loop(P, step, L0, steps, "topk", k_blocks=cfg.topk_blocks, label="fills")


def test_single_launch_threshold_many_rows():
    """Threshold selection on the capacity schedule as one launch, with more (b, h) rows than
    planning clusters (clusters plan several rows each) and ragged short lengths."""
    blk, d, g, Hkv, B = 64, 128, 4, 2, 48
    rng = np.random.default_rng(77)
    lengths = [int(x) for x in rng.integers(1, 24 * blk, B)]
    cfg = config(1, B=B, Hq=g * Hkv, Hkv=Hkv, head_dim=d, gate_dim=128, block=blk, seed=8080, mode="threshold")
    inp = make_inputs(cfg, lengths=lengths, tail="nan")
    P = Problem(inp)
    L = inp.seqlens
    _prefill(P, L)
    tau = 1.0 / 64.0   # exact in float32, the kernel's threshold type
    step = P.step(S.SELECT_THRESHOLD, tau=tau, num_split=-1, single_launch=True)
    for rep in range(2):
        mism, n, _ = _run_and_check(P, step, inp.q, L, "threshold", tau=tau, label=f"threshold rep{rep}")
        assert mism <= n // 50 + 1


def test_single_launch_edge_lengths():
    """Lengths 0, 1, b - 1, b, b + 1 and 2b + 2 in one launch: an empty row (zero output, lse -inf),
    rows with only the forced partial block, a row with one full block and none partial."""
    blk, d, g, Hkv = 64, 128, 4, 2
    lengths = [0, 1, blk - 1, blk, blk + 1, 2 * blk + 2]
    cfg = config(1, B=len(lengths), Hq=g * Hkv, Hkv=Hkv, head_dim=d, gate_dim=128, block=blk, seed=9191)
    inp = make_inputs(cfg, lengths=lengths, tail="nan")
    P = Problem(inp)
    L = inp.seqlens
    _prefill(P, L)
    step = P.step(S.SELECT_TOPK, budget=2 * blk, num_split=-1, single_launch=True)
    mism, n, _ = _run_and_check(P, step, inp.q, L, "topk", k_blocks=2, pairs=[(b, h) for b in range(1, 6)
                                                                                for h in range(Hkv)], label="edges")
    assert mism == 0
    assert step.block_cnt[0].cpu().tolist() == [0] * Hkv
    assert torch.all(step.out[0].float() == 0.0) and torch.all(torch.isneginf(step.lse[0]))


def test_sparsity_sweep_and_dense_path():
    cfg = config(4)
    inp = make_inputs(cfg, workers=draw_workers())
    P = Problem(inp)
    L = inp.seqlens
    _prefill(P, L)
    pairs = [(0, 0), (1, 3), (2, 5), (3, 7)]
    _check_kcomp(P, L, pairs)
    for s in SWEEP_SPARSITIES:
        budget = sweep_budget(cfg.length, s)
        kb = -(-budget // cfg.block)
        step = P.step(S.SELECT_TOPK, budget=budget)
        mism, n, _ = _run_and_check(P, step, inp.q, L, "topk", k_blocks=kb, pairs=pairs, label=f"sweep{s}")
        assert mism <= 1
        cnt = step.block_cnt.cpu().numpy()
        assert np.all(cnt == kb), f"sparsity {s}: counts {np.unique(cnt)} != {kb}"
    # dense path: every block, same kernel, equals dense softmax attention
    nb = inp.max_blocks
    idx = torch.arange(nb, dtype=torch.int32, device="cuda").expand(cfg.B, cfg.Hkv, nb).contiguous()
    cnt = torch.full((cfg.B, cfg.Hkv), nb, dtype=torch.int32, device="cuda")
    out = torch.empty(cfg.B, cfg.Hq, cfg.head_dim, dtype=torch.bfloat16, device="cuda")
    ns = S.sparse_decode_auto_split(P.sh, nb)   # the pages' (split, kv head, batch) grid
    S.sparse_decode(P.sh, to_dev_bf16(inp.q), S.KVCache.contiguous(P.k), S.KVCache.contiguous(P.v), idx, cnt,
                    torch.from_numpy(L).cuda(), out, S.alloc_workspace(P.sh, nb, ns), num_split=ns)
    o = f64(bf16_bits(out))
    for (b, h) in pairs:
        ob = P.obh[(b, h)]
        qg = ob.q_group(inp.q)
        Lb = int(L[b])
        ro, _ = O.attend(qg, ob.k, ob.v, np.arange(Lb), 1 / math.sqrt(cfg.head_dim))
        check_attention(o[b, h * cfg.g:(h + 1) * cfg.g], ro, f"dense b{b} h{h}")


def _calibrate_temperatures(inp, tau, fractions):
    """Per-head multipliers c_h on W_q[h] so that, at step 0, the threshold selects about
    fractions[h] of the full blocks for the median sequence (oracle logits; the count falls
    monotonically with c for tau < 1/nfull)."""
    c = inp.cfg
    L = int(inp.seqlens[0]) + 1
    nfull = L // c.block
    out = []
    for h in range(c.Hkv):
        zs = []
        for b in range(c.B):
            ob = OracleBH(inp, b, h)
            qg = O.q_gate(ob.q_group(inp.q), f64(inp.w_q[h]), L, c.rope_base)
            zs.append(O.gate_logits(qg, ob.kcomp(L), L, c.block))
        target = fractions[h] * nfull
        lo, hi = 1e-3, 1e3
        for _ in range(60):
            mid = math.sqrt(lo * hi)
            n = float(np.median([len(O.select_threshold(mid * z, tau, nfull * c.block, c.block)) for z in zs]))
            if n > target:
                lo = mid
            else:
                hi = mid
        out.append(math.sqrt(lo * hi))
    return out


def test_threshold_decode_loop_256_steps():
    cfg = config(5)
    inp = make_inputs(cfg, workers=draw_workers())
    tau = cfg.tau
    fractions = np.linspace(0.07, 0.20, cfg.Hkv)
    temps = _calibrate_temperatures(inp, tau, fractions)
    wq = scale_gate_weights(inp.w_q, temps)
    P = Problem(inp, w_q_bits=wq)
    L0 = inp.seqlens.copy()
    _prefill(P, L0)
    step = P.step(S.SELECT_THRESHOLD, tau=tau)
    rng = np.random.default_rng(55)
    pairs_all = sorted(P.obh)
    attn_sample = [pairs_all[i] for i in sorted(rng.choice(len(pairs_all), 24, replace=False))]
    fills = {(n + 1) * cfg.block for n in range(L0[0] // cfg.block, (L0[0] + cfg.steps) // cfg.block)}
    fracs, mism_total, compared = [], 0, 0
    for s in range(cfg.steps):
        L = L0 + s + 1
        q_bits = make_step_query(cfg, s)
        before = P.kc.clone()
        check_attn = (s % 16 == 0) or int(L[0]) in fills
        mism, n, _ = _run_and_check(P, step, q_bits, L, "threshold", tau=tau,
                                    attn_pairs=attn_sample if check_attn else [], label=f"loop s{s}")
        mism_total += mism
        compared += n
        # frozen entries: everything below the previous valid count is untouched
        prev_valid = int((L[0] - 1) // cfg.block)
        assert torch.equal(before[:, :, :prev_valid].view(torch.int16), P.kc[:, :, :prev_valid].view(torch.int16))
        if int(L[0]) in fills:
            _check_kcomp(P, L)
            _isolated_checks(P, q_bits, L, "threshold", tau=tau, attn_pairs=attn_sample, label=f"loop s{s}")
        cnt = step.block_cnt.cpu().numpy()
        nblk = -(-int(L[0]) // cfg.block)
        fracs.append(cnt / nblk)
    fr = np.stack(fracs)
    within = float(((fr >= 0.02) & (fr <= 0.30)).mean())
    print(f"threshold loop: selected fraction min {fr.min():.3f} median {np.median(fr):.3f} max {fr.max():.3f}; "
          f"{within:.1%} of (step, b, h) within [2%, 30%]; list mismatches at the cutoff {mism_total}/{compared}")
    assert within >= 0.95
    assert mism_total <= compared // 100 + 1
