"""Checks that pin the CPU oracle to facts other than itself.

Each check raises AssertionError on failure.  They are collected as tests in
test_oracle_pins.py and reused by test_oracle_mutations.py, which plants
plausible mistakes in the oracle and expects at least one check to catch each.

What pins what:
  * hand-derived closed-form fixtures under tests/golden (working shown in
    each case's `derivation`);
  * library special cases (torch's float32->bf16 conversion, torch float64
    softmax attention, numpy's lexsort);
  * brute force in plain Python loops on tiny inputs;
  * invariants: rotation composition and relative-position invariance of
    RoPE, split/combine equivalence, cache freeze, GQA permutation.
"""

from __future__ import annotations

import json
import math
import os
import random

import numpy as np

from oracle import seer_oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _close(a, b, tol=1e-12, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    assert np.allclose(a, b, rtol=tol, atol=tol), f"{what}: {a} vs {b}"


# ---------------------------------------------------------------- bf16 rounding

def check_bf16_fixture():
    for c in _load("gate_fixtures.json")["bf16_ties"]["cases"]:
        got = float(O.round_to_bf16(np.array([c["x"]]))[0])
        assert got == c["expected"], f"bf16({c['x']}) = {got}, expected {c['expected']}"


def check_bf16_vs_torch():
    import torch
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-6, 6, 20000),
                        np.array([1.00390625, 1.01171875, -2.00781250, 0.0])]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_to_bf16(x.astype(np.float64))
    assert np.array_equal(got, ref), "round_to_bf16 disagrees with torch on float32 inputs"
    # decoding bf16 bit patterns: every pattern that is not a NaN, against torch's own widening
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    wide = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    with np.errstate(invalid="ignore"):      # signalling-NaN patterns widen to NaN
        dec = O.bf16_to_f64(bits)
    keep = ~np.isnan(wide)
    assert np.array_equal(dec[keep], wide[keep]) and np.all(np.isnan(dec[~keep])), "bf16_to_f64"


# ---------------------------------------------------------------- RoPE

def check_rope_fixture():
    fx = _load("gate_fixtures.json")["rope_pairing"]
    for c in fx["cases"]:
        _close(O.rope(np.array(c["x"], float), fx["pos"], fx["base"]), c["expected"], 1e-12, "rope fixture")


def check_rope_identity_norm_composition():
    rng = np.random.default_rng(1)
    for dg in (2, 8, 64):
        x = rng.standard_normal(dg)
        _close(O.rope(x, 0, 1e6), x, 1e-15, "rope at position 0")
        for p in (1, 77, 40000):
            y = O.rope(x, p, 1e6)
            assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-12, "rope changes the norm"
        _close(O.rope(O.rope(x, 300, 1e4), 1234, 1e4), O.rope(x, 1534, 1e4), 1e-10, "rope composition")
    # d_gate = 2: a plain rotation by `pos` radians (theta_0 = 1 for any base)
    _close(O.rope(np.array([1.0, 0.0]), 0.75, 123.0), [math.cos(0.75), math.sin(0.75)], 1e-15, "2-d rotation")


def check_rope_relative_invariance():
    """Q_gate . K_gate depends on positions only through their difference."""
    rng = np.random.default_rng(2)
    a, b = rng.standard_normal(16), rng.standard_normal(16)
    base = 1e6
    ref = O.rope(a, 500, base) @ O.rope(b, 64, base)
    for delta in (1, 1000, 33333):
        got = O.rope(a, 500 + delta, base) @ O.rope(b, 64 + delta, base)
        assert abs(got - ref) < 1e-9 * max(1.0, abs(ref)), "rope not relative"


# ---------------------------------------------------------------- pooling / K gate

def check_pool_fixture():
    fx = _load("gate_fixtures.json")["pool_order"]
    _close(O.pool_block(np.array(fx["keys"], float)), fx["expected"], 1e-15, "pool order")


def check_pool_bruteforce():
    rng = np.random.default_rng(3)
    keys = rng.standard_normal((5, 3))
    t, d = keys.shape
    mx = [max(keys[i][c] for i in range(t)) for c in range(d)]
    mn = [min(keys[i][c] for i in range(t)) for c in range(d)]
    av = [sum(keys[i][c] for i in range(t)) / t for c in range(d)]
    _close(O.pool_block(keys), mx + mn + av, 1e-15, "pool brute force")
    same = np.tile(rng.standard_normal((1, 4)), (6, 1))
    p = O.pool_block(same)
    _close(p[:4], same[0], 0, "constant max")
    _close(p[4:8], same[0], 0, "constant min")
    _close(p[8:], same[0], 1e-15, "constant avg")


def check_k_gate_fixture():
    fx = _load("gate_fixtures.json")["k_gate_entry"]
    for c in fx["cases"]:
        got = O.k_gate_entry(np.array(fx["keys"], float), np.array(fx["w_k"], float), c["n"], fx["block"], fx["base"])
        _close(got, c["expected"], 0, f"k_gate n={c['n']}")


def check_q_gate_fixture():
    fx = _load("gate_fixtures.json")["q_gate_reshape"]
    got = O.q_gate(np.array(fx["q_nope"], float), np.array(fx["w_q"], float), fx["length"], fx["base"])
    _close(got, fx["expected"], 1e-15, "q_gate reshape")


def check_gate_logits_fixture():
    fx = _load("gate_fixtures.json")["gate_logits_scale"]
    got = O.gate_logits(np.array(fx["q_gate"], float), np.array(fx["kcomp"], float), fx["length"], fx["block"])
    _close(got, fx["expected"], 1e-15, "gate logits")


def check_gate_linear_bruteforce():
    """W_q . reshape(q) and W_k . pool(K) against explicit loops (pos 0: no rotation)."""
    rng = np.random.default_rng(4)
    g, d, dg, b = 3, 4, 6, 5
    q = rng.standard_normal((g, d))
    wq = rng.standard_normal((dg, g * d))
    want = [sum(wq[r][j * d + c] * q[j][c] for j in range(g) for c in range(d)) for r in range(dg)]
    _close(O.q_gate(q, wq, 1, 1e6), want, 1e-12, "q_gate loops")
    keys = rng.standard_normal((b, d))
    wk = rng.standard_normal((dg, 3 * d))
    p = [max(keys[:, c]) for c in range(d)] + [min(keys[:, c]) for c in range(d)] + \
        [sum(keys[:, c]) / b for c in range(d)]
    want = [sum(wk[r][i] * p[i] for i in range(3 * d)) for r in range(dg)]
    got = O.k_gate_entry(keys, wk, 0, b, 1e6)
    assert np.all(np.abs(got - np.asarray(want)) <= np.abs(np.asarray(want)) * 2.0 ** -8), "k_gate loops"


# ---------------------------------------------------------------- selection

def _fx_sel(name):
    return _load("selection_fixtures.json")[name]


def check_topk_fixture():
    fx = _fx_sel("topk_ties")
    for c in fx["cases"]:
        k = -(-c["budget"] // fx["block"])
        got = O.select_topk(np.array(fx["logits"], float), k, fx["length"], fx["block"])
        assert got == c["expected"], f"topk budget {c['budget']}: {got} vs {c['expected']}"
    fx = _fx_sel("topk_partial")
    k = -(-fx["budget"] // fx["block"])
    got = O.select_topk(np.array(fx["logits"], float), k, fx["length"], fx["block"])
    assert got == fx["expected"], f"topk partial: {got}"


def check_topk_definition_random():
    """Selected blocks dominate unselected ones (logit, then lower index); count formula; lexsort."""
    rng = np.random.default_rng(5)
    for trial in range(300):
        nfull = int(rng.integers(0, 40))
        b = 16
        L = nfull * b + int(rng.integers(0, b)) if trial % 2 else nfull * b
        if trial % 3 == 0:
            z = rng.integers(-2, 3, nfull).astype(float)      # heavy ties
        else:
            z = rng.standard_normal(nfull)
        k = int(rng.integers(1, 45))
        got = O.select_topk(z, k, L, b)
        assert got == sorted(got)
        part = L % b != 0
        assert len(got) == min(k, nfull) + int(part), "top-k count"
        full = [n for n in got if n < nfull]
        rest = [n for n in range(nfull) if n not in full]
        for n in full:
            for m in rest:
                assert z[n] > z[m] or (z[n] == z[m] and n < m), "top-k dominance"
        if nfull:
            order = np.lexsort((np.arange(nfull), -z))[:min(k, nfull)]
            assert sorted(order.tolist()) == full, "top-k vs lexsort"
        if part:
            assert got[-1] == nfull


def check_threshold_fixture():
    fx = _fx_sel("threshold_strict")
    for c in fx["cases"]:
        got = O.select_threshold(np.array(fx["logits"], float), c["tau"], c["length"], fx["block"])
        assert got == c["expected"], f"threshold tau={c['tau']} L={c['length']}: {got}"


def check_threshold_extremes():
    rng = np.random.default_rng(6)
    for _ in range(50):
        nfull = int(rng.integers(1, 60))
        z = rng.standard_normal(nfull) * 3
        L = nfull * 64 + int(rng.integers(0, 64))
        part = [nfull] if L % 64 else []
        assert O.select_threshold(z, 0.0, L, 64) == list(range(nfull)) + part
        assert O.select_threshold(z, 1.0, L, 64) == part
        s = np.exp(z - z.max()); s /= s.sum()
        tau = float(np.median(s))
        want = [n for n in range(nfull) if s[n] > tau] + part
        assert O.select_threshold(z, tau, L, 64) == want


def check_topp_fixture():
    fx = _fx_sel("topp_mass")
    for c in fx["cases"]:
        got = O.select_topp(np.array(fx["logits"], float), c["p"], fx["length"], fx["block"])
        assert got == c["expected"], f"top-p p={c['p']}: {got}"


def check_topp_minimal():
    rng = np.random.default_rng(8)
    for _ in range(100):
        nfull = int(rng.integers(1, 50))
        z = rng.standard_normal(nfull) * 2
        p = float(rng.uniform(0.05, 0.99))
        got = [n for n in O.select_topp(z, p, nfull * 32, 32)]
        s = np.exp(z - z.max()); s /= s.sum()
        mass = s[got].sum()
        assert mass >= p - 1e-12, "top-p mass"
        assert len(got) == 1 or mass - s[got].min() < p + 1e-12, "top-p not minimal"
        assert len(got) <= nfull


# ---------------------------------------------------------------- attention / combine

def _fx_att(name):
    return _load("attention_fixtures.json")[name]


def check_attention_fixture():
    fx = _fx_att("two_token_softmax")
    o, lse = O.attend(np.array(fx["q"], float), np.array(fx["k"], float), np.array(fx["v"], float),
                      np.arange(2), fx["scale"])
    _close(o, fx["expected_o"], 1e-12, "two-token o")
    _close(lse, fx["expected_lse"], 1e-12, "two-token lse")
    fx = _fx_att("masked_partial_block")
    o, lse = O.sparse_decode(np.array(fx["q"], float), np.array(fx["k"], float), np.array(fx["v"], float),
                             fx["blocks"], fx["length"], fx["block"], fx["scale"])
    _close(o, fx["expected_o"], 1e-12, "partial-block o")
    _close(lse, fx["expected_lse"], 1e-12, "partial-block lse")


def _naive_dense(q, k, v, L, scale):
    g, d = len(q), len(q[0])
    out, lses = [], []
    for i in range(g):
        s = [scale * sum(q[i][c] * k[t][c] for c in range(d)) for t in range(L)]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        z = sum(e)
        out.append([sum(e[t] * v[t][c] for t in range(L)) / z for c in range(d)])
        lses.append(m + math.log(z))
    return np.array(out), np.array(lses)


def check_attention_dense_equivalence():
    """All blocks selected == dense softmax attention (naive loops and torch float64)."""
    import torch
    rng = np.random.default_rng(9)
    g, d, b = 3, 8, 8
    for L in (8, 37, 64):
        q = rng.standard_normal((g, d))
        k = rng.standard_normal((L + 5, d))
        v = rng.standard_normal((L + 5, d))
        blocks = list(range(-(-L // b)))
        scale = 1 / math.sqrt(d)
        o, lse = O.sparse_decode(q, k, v, blocks, L, b, scale)
        on, ln_ = _naive_dense(q.tolist(), k.tolist(), v.tolist(), L, scale)
        _close(o, on, 1e-12, "dense vs loops")
        _close(lse, ln_, 1e-12, "dense lse vs loops")
        tq, tk, tv = (torch.from_numpy(x) for x in (q, k[:L], v[:L]))
        ref = torch.softmax(tq @ tk.T * scale, dim=-1) @ tv
        _close(o, ref.numpy(), 1e-12, "dense vs torch")
        _close(lse, torch.logsumexp(tq @ tk.T * scale, dim=-1).numpy(), 1e-12, "lse vs torch")


def check_attention_single_block_and_mask():
    rng = np.random.default_rng(10)
    g, d, b, L = 2, 4, 16, 50
    q = rng.standard_normal((g, d))
    k = rng.standard_normal((64, d))
    v = rng.standard_normal((64, d))
    k[L:] = np.nan
    v[L:] = np.nan
    o, _ = O.sparse_decode(q, k, v, [1], L, b, 0.5)
    on, _ = _naive_dense(q.tolist(), k[16:32].tolist(), v[16:32].tolist(), 16, 0.5)
    _close(o, on, 1e-12, "single block")
    o, _ = O.sparse_decode(q, k, v, [0, 3], L, b, 0.5)
    assert np.all(np.isfinite(o)), "masked tail leaked into the result"
    toks = list(range(16)) + [48, 49]
    on, _ = _naive_dense(q.tolist(), k[toks].tolist(), v[toks].tolist(), len(toks), 0.5)
    _close(o, on, 1e-12, "partial block masking")


def check_combine_fixture():
    fx = _fx_att("combine_two_splits")
    parts = [(np.array(p["o"], float), np.array([float(x) for x in p["lse"]])) for p in fx["parts"]]
    o, lse = O.combine(parts)
    _close(o, fx["expected_o"], 1e-12, "combine o")
    _close(lse, fx["expected_lse"], 1e-12, "combine lse")


def check_combine_partitions():
    rng = np.random.default_rng(11)
    g, d, b, L = 4, 8, 8, 203
    q = rng.standard_normal((g, d))
    k = rng.standard_normal((L, d))
    v = rng.standard_normal((L, d))
    blocks = sorted(rng.choice(-(-L // b), 12, replace=False).tolist())
    if blocks[-1] != L // b:
        blocks.append(L // b)
    ref_o, ref_l = O.sparse_decode(q, k, v, blocks, L, b, 0.3)
    for ns in (1, 2, 3, 5, 16):
        parts = [O.sparse_decode(q, k, v, s, L, b, 0.3) for s in O.split_list(blocks, 20, ns)]
        o, lse = O.combine(parts)
        _close(o, ref_o, 1e-12, f"combine ns={ns}")
        _close(lse, ref_l, 1e-12, f"combine lse ns={ns}")
    e_o, e_l = O.sparse_decode(q, k, v, [], L, b, 0.3)
    assert np.all(e_o == 0) and np.all(np.isneginf(e_l)), "empty split"


# ---------------------------------------------------------------- ground truth

def check_ground_truth():
    fx = _fx_att("decode_ground_truth")
    got = O.decode_ground_truth(np.array(fx["q"], float), np.array(fx["k"], float), fx["length"],
                                fx["block"], fx["scale"])
    _close(got, fx["expected"], 1e-12, "ground truth")
    rng = np.random.default_rng(12)
    q = rng.standard_normal((4, 8))
    k = rng.standard_normal((100, 8))
    gt = O.decode_ground_truth(q, k, 100, 16, 0.35)
    assert gt.shape == (7,) and abs(gt.sum() - 1) < 1e-12 and np.all(gt > 0)


def check_prefill_ground_truth():
    """Prefill output, LSE and targets against a hand-derived two-head case; then the target vs
    three other things: every row i is the (pinned) decode target of query
    i over keys 0..i; the output is torch's float64 causal attention; and the pages' tile
    recurrence (per-tile row maxima r, running max m and normaliser l, then exp(r - m) / l)
    reproduces each head's pooled probabilities before the group max."""
    import torch
    fx = _fx_att("prefill_ground_truth")
    o, lse, gt = O.prefill_ground_truth(np.array(fx["q"], float), np.array(fx["k"], float),
                                        np.array(fx["v"], float), fx["block"], fx["scale"])
    _close(o, fx["expected_o"], 1e-12, "prefill fixture o")
    _close(lse, fx["expected_lse"], 1e-12, "prefill fixture lse")
    _close(gt, fx["expected_gt"], 1e-12, "prefill fixture targets")
    rng = np.random.default_rng(16)
    g, L, d, b = 3, 37, 8, 8
    q = rng.standard_normal((g, L, d))
    k = rng.standard_normal((L, d))
    v = rng.standard_normal((L, d))
    scale = 0.4
    o, lse, gt = O.prefill_ground_truth(q, k, v, b, scale)
    nb = -(-L // b)
    assert gt.shape == (L, nb)
    for i in range(L):
        ref = O.decode_ground_truth(q[:, i], k, i + 1, b, scale)
        _close(gt[i, :len(ref)], ref, 1e-12, f"row {i}")
        assert np.all(gt[i, len(ref):] == 0), f"row {i}: blocks past the position"
    tq = torch.from_numpy(q)[None]
    ref_o = torch.nn.functional.scaled_dot_product_attention(
        tq, torch.from_numpy(k)[None, None].expand(1, g, L, d), torch.from_numpy(v)[None, None].expand(1, g, L, d),
        is_causal=True, scale=scale)[0].numpy()
    _close(o, ref_o, 1e-10, "causal attention output")
    for h in range(g):
        for i in range(L):
            m, l, r = -math.inf, 0.0, []
            for n in range(nb):
                t = np.arange(n * b, min((n + 1) * b, i + 1))
                if len(t) == 0:
                    break
                sij = scale * (k[t] @ q[h, i])
                rij = sij.max()
                mn = max(m, rij)
                l = l * math.exp(m - mn) + np.exp(sij - mn).sum()
                m = mn
                r.append(rij)
            assert abs((m + math.log(l)) - lse[h, i]) < 1e-12, "lse"
            s_row = scale * (k[:i + 1] @ q[h, i])
            p_row = np.exp(s_row - s_row.max()) / np.exp(s_row - s_row.max()).sum()
            pooled = [p_row[n * b:min((n + 1) * b, i + 1)].max() for n in range(len(r))]
            _close(np.exp(np.array(r) - m) / l, pooled, 1e-12, "tile recurrence")


# ---------------------------------------------------------------- K compression cache

def check_kcomp_incremental():
    """Entry n appears exactly when L reaches (n+1)*b, is then frozen, and equals a rebuild."""
    rng = np.random.default_rng(13)
    d, dg, b, Lmax = 4, 6, 8, 45
    keys = rng.standard_normal((Lmax, d))
    wk = rng.standard_normal((dg, 3 * d))
    cache = np.full((8, dg), np.nan)
    valid = 0
    history = []
    for L in range(1, Lmax + 1):
        valid = O.kcomp_update(keys, L, valid, wk, cache, b, 1e4)
        assert valid == L // b
        filled = ~np.isnan(cache[:, 0])
        assert filled.sum() == L // b, f"entries present at L={L}"
        history.append(cache.copy())
    for n in range(Lmax // b):
        first = (n + 1) * b - 1                 # history index of L = (n+1)*b
        assert np.isnan(history[first - 1][n, 0]), "entry appeared early"
        for h in history[first:]:
            assert np.array_equal(h[n], history[first][n]), "entry changed after it was written"
    rebuilt = np.full((8, dg), np.nan)
    O.kcomp_update(keys, Lmax, 0, wk, rebuilt, b, 1e4)
    assert np.array_equal(rebuilt[:Lmax // b], cache[:Lmax // b]), "rebuild differs"
    for n in range(Lmax // b):
        assert np.array_equal(cache[n], O.k_gate_entry(keys[n * b:(n + 1) * b], wk, n, b, 1e4))


def check_kcomp_append_matches_rebuild():
    """Token-by-token appends from running max/min/sum give the block-pooling cache exactly
    (max and min exactly; the sum/b average within fp64 rounding), each entry appearing when its
    block's last token arrives; a block first token restarts the statistics."""
    rng = np.random.default_rng(15)
    for d, dg, b, Lmax in ((4, 6, 8, 45), (3, 4, 5, 23)):
        keys = rng.standard_normal((Lmax, d))
        wk = rng.standard_normal((dg, 3 * d))
        cache = np.full((Lmax // b + 1, dg), np.nan)
        state = np.full((3, d), 1e9)             # garbage: the first token must restart it
        valid = 0
        for L in range(1, Lmax + 1):
            valid = O.kcomp_append(state, keys[L - 1], L, valid, wk, cache, b, 1e4)
            assert valid == L // b, f"fill count at L={L}"
            blk = keys[(L - 1) // b * b:L]
            _close(state[0], blk.max(0), 0, "running max")
            _close(state[1], blk.min(0), 0, "running min")
            _close(state[2], blk.sum(0), 1e-12, "running sum")
        rebuilt = np.full_like(cache, np.nan)
        O.kcomp_update(keys, Lmax, 0, wk, rebuilt, b, 1e4)
        nf = Lmax // b
        assert np.array_equal(np.isnan(cache), np.isnan(rebuilt)), "entries present differ"
        _close(cache[:nf], rebuilt[:nf], 2.0 ** -7, "rolling vs rebuild")


def check_memory_ratio():
    """K Compression Cache = 1/128 of the KV cache at b=64 with d_gate = d, same element size."""
    b, d, dg, L = 64, 128, 128, 65536
    kv_bytes = 2 * L * d * 2
    kc_bytes = (L // b) * dg * 2
    assert kc_bytes * 128 == kv_bytes


# ---------------------------------------------------------------- GQA sharing

def check_gqa_shared_selection():
    rng = np.random.default_rng(14)
    g, d, dg, b, L = 4, 8, 8, 8, 77
    q = rng.standard_normal((g, d))
    k = rng.standard_normal((L, d))
    v = rng.standard_normal((L, d))
    wq = rng.standard_normal((dg, g * d))
    wk = rng.standard_normal((dg, 3 * d))
    kc = np.zeros((10, dg))
    O.kcomp_update(k, L, 0, wk, kc, b, 1e6)
    ref = O.decode_step_bh(q, k, v, wq, kc, L, b, 1e6, "topk", k_blocks=3)
    perm = [2, 0, 3, 1]
    wq_p = np.concatenate([wq[:, j * d:(j + 1) * d] for j in perm], axis=1)
    got = O.decode_step_bh(q[perm], k, v, wq_p, kc, L, b, 1e6, "topk", k_blocks=3)
    _close(got["logits"], ref["logits"], 1e-12, "permuted group logits")
    assert got["blocks"] == ref["blocks"], "group selection changed under head permutation"
    _close(got["o"], ref["o"][perm], 1e-12, "permuted outputs")
    for j in range(g):                          # every head of the group reads the same blocks
        o_j, _ = O.sparse_decode(q[j:j + 1], k, v, ref["blocks"], L, b, 1 / math.sqrt(d))
        _close(o_j[0], ref["o"][j], 1e-12, "per-head shared list")


ALL_CHECKS = [v for k, v in sorted(globals().items()) if k.startswith("check_")]
