"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins catch each one.

Every mutant below is a slip someone could make when writing the oracle from
the pages: a swapped pooling order, a wrong RoPE sign or pairing, an
off-by-one position, a dropped scale, the wrong tie rule, a non-strict
threshold, a top-p that stops short of p, a forgotten partial block, a
mis-weighted combine, an unnormalised target.  A mutant that
no pin catches would mean the pins do not fix that part of the definition.
"""

import numpy as np
import pytest

import oracle_pins as P
from oracle import seer_oracle as O


def _rope_sign(x, pos, base):
    x = np.asarray(x, float)
    dg = x.shape[-1]; h = dg // 2
    th = np.power(float(base), -2.0 * np.arange(h) / dg)
    c, s = np.cos(pos * th), np.sin(pos * th)
    return np.concatenate([x[..., :h] * c + x[..., h:] * s, x[..., h:] * c - x[..., :h] * s], axis=-1)


def _rope_interleaved(x, pos, base):
    x = np.asarray(x, float)
    dg = x.shape[-1]
    th = np.power(float(base), -2.0 * np.arange(dg // 2) / dg)
    c, s = np.cos(pos * th), np.sin(pos * th)
    a, b = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = b * c + a * s
    return out


def _rope_theta_dg_half(x, pos, base):
    x = np.asarray(x, float)
    dg = x.shape[-1]; h = dg // 2
    th = np.power(float(base), -1.0 * np.arange(h) / dg)          # dropped the factor 2
    c, s = np.cos(pos * th), np.sin(pos * th)
    return np.concatenate([x[..., :h] * c - x[..., h:] * s, x[..., h:] * c + x[..., :h] * s], axis=-1)


def _pool_min_max(keys):
    keys = np.asarray(keys, float)
    return np.concatenate([keys.min(0), keys.max(0), keys.mean(0)])


def _q_gate_pos_L(q, w, length, base):
    return O.rope(np.asarray(w, float) @ np.asarray(q, float).reshape(-1), length, base)


def _q_gate_d_major(q, w, length, base):
    return O.rope(np.asarray(w, float) @ np.asarray(q, float).T.reshape(-1), length - 1, base)


def _k_gate_last_pos(keys, w_k, n, block, base):
    return O.round_to_bf16(O.rope(np.asarray(w_k, float) @ O.pool_block(keys), (n + 1) * block - 1, base))


def _logits_noscale(qg, kc, length, block):
    return np.asarray(kc[:length // block], float) @ qg


def _topk_high_index(logits, k, length, block):
    nfull = length // block
    z = list(np.asarray(logits, float)[:nfull])
    order = sorted(range(nfull), key=lambda n: (-z[n], -n))
    return O._with_partial(order[:min(k, nfull)], length, block)


def _threshold_ge(logits, tau, length, block):
    nfull = length // block
    s = O.gate_scores(np.asarray(logits, float)[:nfull])
    return O._with_partial([n for n in range(nfull) if s[n] >= tau], length, block)


def _no_partial(chosen, length, block):
    return sorted(int(n) for n in chosen)


def _attend_noscale(q, k, v, tokens, scale):
    return ATTEND(q, k, v, tokens, 1.0)


def _combine_linear(parts):
    lses = np.stack([p[1] for p in parts]); os_ = np.stack([p[0] for p in parts])
    w = np.where(np.isfinite(lses), lses, 0.0)                   # weights without exp
    tot = w.sum(0)
    return (w[:, :, None] * os_).sum(0) / np.where(tot != 0, tot, 1)[:, None], np.log(np.abs(tot) + 1e-300)


def _gt_mean_over_group(q, k, length, block, scale):
    q = np.asarray(q, float); kk = np.asarray(k[:length], float)
    s = scale * q @ kk.T
    p = np.exp(s - s.max(1, keepdims=True)); p /= p.sum(1, keepdims=True)
    nb = -(-length // block)
    col = np.array([[p[i, n * block:min((n + 1) * block, length)].max() for n in range(nb)] for i in range(len(q))])
    gt = col.mean(0)
    return gt / gt.sum()


def _append_no_restart(state, k_new, length, valid, w_k, kcomp, block, base):
    n, pos = divmod(length - 1, block)
    k = np.asarray(k_new, float)
    state[0] = np.maximum(state[0], k); state[1] = np.minimum(state[1], k); state[2] = state[2] + k
    if pos != block - 1:
        return valid
    y = np.asarray(w_k, float) @ np.concatenate([state[0], state[1], state[2] / block])
    kcomp[n] = O.round_to_bf16(O.rope(y, n * block, base))
    return n + 1


def _append_rope_at_last(state, k_new, length, valid, w_k, kcomp, block, base):
    n, pos = divmod(length - 1, block)
    k = np.asarray(k_new, float)
    if pos == 0:
        state[0], state[1], state[2] = k, k, k
    else:
        state[0] = np.maximum(state[0], k); state[1] = np.minimum(state[1], k); state[2] = state[2] + k
    if pos != block - 1:
        return valid
    y = np.asarray(w_k, float) @ np.concatenate([state[0], state[1], state[2] / block])
    kcomp[n] = O.round_to_bf16(O.rope(y, length - 1, base))
    return n + 1


def _prefill_unmasked(q, k, v, block, scale):
    q = np.asarray(q, float); kk = np.asarray(k, float); vv = np.asarray(v, float)
    s = scale * np.einsum("hid,td->hit", q, kk)                  # future keys left visible
    p = np.exp(s - s.max(2, keepdims=True)); p /= p.sum(2, keepdims=True)
    L = q.shape[1]; nb = -(-L // block)
    pooled = np.stack([p[:, :, n * block:min((n + 1) * block, L)].max(2) for n in range(nb)], 2).max(0)
    return np.einsum("hit,td->hid", p, vv), np.log(np.exp(s).sum(2)), pooled / pooled.sum(1, keepdims=True)


def _prefill_norm_then_max(q, k, v, block, scale):
    o, lse, _ = REAL_PREFILL(q, k, v, block, scale)
    q = np.asarray(q, float); kk = np.asarray(k, float)
    g, L, _ = q.shape
    s = scale * np.einsum("hid,td->hit", q, kk)
    s = np.where(np.tril(np.ones((L, L), bool))[None], s, -np.inf)
    p = np.exp(s - s.max(2, keepdims=True)); p /= p.sum(2, keepdims=True)
    nb = -(-L // block)
    pooled = np.stack([p[:, :, n * block:min((n + 1) * block, L)].max(2) for n in range(nb)], 2)
    pooled = pooled / pooled.sum(2, keepdims=True)                # normalised per head first
    return o, lse, pooled.max(0)


def _topp_one_short(logits, p, length, block):
    nfull = length // block
    s = O.gate_scores(np.asarray(logits, float)[:nfull])
    order = sorted(range(nfull), key=lambda n: (-float(s[n]), n))
    chosen, mass = [], 0.0
    for n in order:                                              # stops before the mass reaches p
        if mass + float(s[n]) > p:
            break
        chosen.append(n)
        mass += float(s[n])
    return O._with_partial(chosen, length, block)


def _topp_ascending(logits, p, length, block):
    nfull = length // block
    s = O.gate_scores(np.asarray(logits, float)[:nfull])
    chosen, mass = [], 0.0
    for n in range(nfull):                                       # index order, not score order
        if mass >= p:
            break
        chosen.append(n)
        mass += float(s[n])
    return O._with_partial(chosen, length, block)


def _threshold_on_logits(logits, tau, length, block):
    nfull = length // block
    z = np.asarray(logits, float)[:nfull]                        # tau against the raw logits
    return O._with_partial([n for n in range(nfull) if z[n] > tau], length, block)


def _pool_avg_as_sum(keys):
    keys = np.asarray(keys, float)
    return np.concatenate([keys.max(0), keys.min(0), keys.sum(0)])


def _k_gate_block_index(keys, w_k, n, block, base):
    y = np.asarray(w_k, float) @ O.pool_block(keys)
    return O.round_to_bf16(O.rope(y, n, base))                   # position n, not n * b


def _gt_unnormalised(q, k, length, block, scale):
    gt = REAL_GT(q, k, length, block, scale)
    q = np.asarray(q, float); kk = np.asarray(k[:length], float)
    s = scale * q @ kk.T
    p = np.exp(s - s.max(1, keepdims=True)); p /= p.sum(1, keepdims=True)
    nb = -(-length // block)
    return np.array([[p[i, n * block:min((n + 1) * block, length)].max() for n in range(nb)]
                     for i in range(len(q))]).max(0)


def _gt_block_mean(q, k, length, block, scale):
    q = np.asarray(q, float); kk = np.asarray(k[:length], float)
    s = scale * q @ kk.T
    p = np.exp(s - s.max(1, keepdims=True)); p /= p.sum(1, keepdims=True)
    nb = -(-length // block)
    col = np.array([[p[i, n * block:min((n + 1) * block, length)].mean() for n in range(nb)]
                    for i in range(len(q))])                     # average-pooled columns
    gt = col.max(0)
    return gt / gt.sum()


def _block_tokens_unclipped(blocks, length, block):
    toks = []
    for n in blocks:
        toks.extend(range(n * block, (n + 1) * block))         # the partial block's tail kept
    return np.asarray(toks, dtype=np.int64)


REAL_GT = O.decode_ground_truth
REAL_PREFILL = O.prefill_ground_truth
ATTEND = O.attend

MUTANTS = {
    "rope_sign": ("rope", _rope_sign),
    "rope_interleaved": ("rope", _rope_interleaved),
    "rope_theta": ("rope", _rope_theta_dg_half),
    "pool_order": ("pool_block", _pool_min_max),
    "q_gate_position": ("q_gate", _q_gate_pos_L),
    "q_gate_reshape": ("q_gate", _q_gate_d_major),
    "k_gate_position": ("k_gate_entry", _k_gate_last_pos),
    "logit_scale": ("gate_logits", _logits_noscale),
    "topk_ties": ("select_topk", _topk_high_index),
    "threshold_ge": ("select_threshold", _threshold_ge),
    "no_partial": ("_with_partial", _no_partial),
    "attention_scale": ("attend", _attend_noscale),
    "combine_weights": ("combine", _combine_linear),
    "gt_group_mean": ("decode_ground_truth", _gt_mean_over_group),
    "append_no_restart": ("kcomp_append", _append_no_restart),
    "append_rope_position": ("kcomp_append", _append_rope_at_last),
    "prefill_unmasked": ("prefill_ground_truth", _prefill_unmasked),
    "prefill_norm_then_max": ("prefill_ground_truth", _prefill_norm_then_max),
    "topp_one_short": ("select_topp", _topp_one_short),
    "topp_index_order": ("select_topp", _topp_ascending),
    "threshold_on_logits": ("select_threshold", _threshold_on_logits),
    "pool_avg_as_sum": ("pool_block", _pool_avg_as_sum),
    "k_gate_block_index": ("k_gate_entry", _k_gate_block_index),
    "gt_unnormalised": ("decode_ground_truth", _gt_unnormalised),
    "gt_block_mean": ("decode_ground_truth", _gt_block_mean),
    "partial_block_unclipped": ("block_tokens", _block_tokens_unclipped),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(O, attr, fn)
    caught = []
    for check in P.ALL_CHECKS:
        try:
            check()
        except (AssertionError, ValueError, IndexError):
            caught.append(check.__name__)
    assert caught, f"no pin catches the planted mistake '{name}'"
