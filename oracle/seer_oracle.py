"""Plain CPU oracle for SeerAttention-R's gated block-sparse GQA decode step.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this module; only
the tests, the package smoke check and the benchmark's CPU-baseline leg may
call it.  It shares no code with the CUDA path and is slow on purpose: every
function is the definition written out in float64 numpy, per (batch, kv-head).

Sources, cited by page and section:
  [CP]  "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning"
        (chapterpal.com summary) -- Knowl 1 (AttnGate architecture), Knowl 2
        (gate equations), Knowl 3 (decode ground truth), Knowl 5 (K
        Compression Cache, token budget / threshold), Knowl 6 (block-sparse
        flash decoding, num_split), Knowl 14 (top-p as future work).
  [PN]  "Sparse Attention Adaptation for Long Reasoning" (papernotes.org
        notes) -- key designs 1, 2 and 4 and the training-strategy paragraph.
  [SK]  "sparse-attention-reasoning" (skillsmp.com skill page) -- the masked
        softmax attention in OptimizedSparseAttentionKernel (scale 1/sqrt(d),
        -inf mask).

Readings taken where the pages are silent (each is pinned by a test):
  * RoPE is the rotate-half form pairing channel i with i + d_gate/2,
    theta_i = base^(-2i/d_gate), angles in float64.
  * The gate query sits at position L-1 (L counts the current token); the
    compressed key of block n sits at position n*b, its first token [CP K1].
  * Pooled vector order is [max | min | avg] [CP K2]; no bias in either gate
    linear; W_k is held per KV head like W_q [PN design 1].
  * The K Compression Cache stores K_gate after RoPE, rounded to bf16; the
    gate query stays float64.
  * Only the floor(L/b) full blocks are scored; the partial last block is
    never scored, only forced on [CP K5].
  * Top-k runs on the scaled logits (order equals the un-softmaxed logits'
    order), ties go to the lower block index, and the forced partial block
    comes on top of the k.  Threshold compares S = softmax(logits) > tau.
  * Selected indices are returned ascending.
  * Attention scale defaults to 1/sqrt(d) [SK]; query head i reads KV head
    floor(i / g).
  * Top-p takes blocks in descending S (ties to the lower index) until their
    S-sum reaches p [CP K14].
  * The decode ground truth pools every block the length reaches, the partial
    one included; the prefill target of position t is the decode target of a
    query at t over keys 0..t, with the group max and normalisation applied
    [CP K3, K4].
  * The running-statistics cache keeps per-channel max, min and sum of the
    current block's keys, restarted at a block's first token [CP K5].

Pins (tests/oracle_pins.py; each compares against something other than this
module: hand-derived fixtures under tests/golden/, closed forms, brute force,
torch routines, or invariants), by function:
  bf16_to_f64, round_to_bf16     check_bf16_fixture, check_bf16_vs_torch
  rope                           check_rope_fixture, check_rope_identity_norm_composition,
                                 check_rope_relative_invariance
  pool_block                     check_pool_fixture, check_pool_bruteforce
  k_gate_entry, q_gate,          check_k_gate_fixture, check_q_gate_fixture,
  gate_logits                    check_gate_logits_fixture, check_gate_linear_bruteforce
  kcomp_update                   check_kcomp_incremental, check_memory_ratio
  kcomp_append                   check_kcomp_append_matches_rebuild
  gate_scores, select_threshold  check_threshold_fixture, check_threshold_extremes
  select_topk                    check_topk_fixture, check_topk_definition_random
  select_topp                    check_topp_fixture, check_topp_minimal
  block_tokens, attend,          check_attention_fixture, check_attention_dense_equivalence,
  sparse_decode                  check_attention_single_block_and_mask
  combine, split_list            check_combine_fixture, check_combine_partitions
  decode_ground_truth            check_ground_truth
  prefill_ground_truth           check_prefill_ground_truth (hand-derived fixture, torch causal
                                 attention, the decode target row by row, the tile recurrence)
  decode_step_bh                 check_gqa_shared_selection
No function here is left without a pin.
"""

from __future__ import annotations

import math
from typing import Iterable, List, Sequence, Tuple

import numpy as np

NEG_INF = float("-inf")


# ----------------------------------------------------------------------------
# bf16 helpers (the cache stores bf16; inputs arrive as bf16 bit patterns)
# ----------------------------------------------------------------------------

def bf16_to_f64(bits) -> np.ndarray:
    """Exact value of bf16 bit patterns as float64."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def round_to_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (ties to even).

    Rounds once, straight from float64 (no float32 intermediate).  Valid for
    zero and for magnitudes in bf16's normal range; anything else raises.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    bad = (a != 0) & ((a < 2.0 ** -126) | ~np.isfinite(a))
    if np.any(bad):
        raise ValueError("round_to_bf16: value outside bf16 normal range")
    u = x.view(np.uint64).copy()
    drop = 52 - 7                       # float64 keeps 52 fraction bits, bf16 keeps 7
    lsb = (u >> np.uint64(drop)) & np.uint64(1)
    u = (u + (np.uint64(1) << np.uint64(drop - 1)) - np.uint64(1) + lsb)
    u &= ~np.uint64((1 << drop) - 1)
    out = u.view(np.float64)
    if np.any(np.abs(out) > 3.3895313892515355e38):
        raise ValueError("round_to_bf16: overflow")
    return out


# ----------------------------------------------------------------------------
# AttnGate pieces  [CP Knowl 1, Knowl 2]
# ----------------------------------------------------------------------------

def rope(x: np.ndarray, pos: float, base: float) -> np.ndarray:
    """Rotary embedding of a d_gate-vector at position `pos` (rotate-half pairing)."""
    x = np.asarray(x, dtype=np.float64)
    dg = x.shape[-1]
    half = dg // 2
    i = np.arange(half, dtype=np.float64)
    theta = np.power(float(base), -2.0 * i / dg)
    ang = float(pos) * theta
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def pool_block(keys: np.ndarray) -> np.ndarray:
    """Non-overlapping max / min / avg pooling of one block of pre-RoPE keys.

    keys: [t, d] -> [3d] = [max | min | avg] over the t tokens [CP Knowl 2].
    """
    keys = np.asarray(keys, dtype=np.float64)
    return np.concatenate([keys.max(axis=0), keys.min(axis=0), keys.mean(axis=0)])


def k_gate_entry(keys: np.ndarray, w_k: np.ndarray, n: int, block: int, base: float) -> np.ndarray:
    """One K Compression Cache entry: RoPE_{n*b}(W_k . pool(keys)), stored as bf16.

    keys: [b, d] pre-RoPE keys of full block n; w_k: [d_gate, 3d].
    [CP Knowl 2 (K_gate), Knowl 5 (the cache holds K_gate)]
    """
    y = np.asarray(w_k, dtype=np.float64) @ pool_block(keys)
    return round_to_bf16(rope(y, n * block, base))


def kcomp_update(k_nope: np.ndarray, length: int, valid: int, w_k: np.ndarray,
                 kcomp: np.ndarray, block: int, base: float) -> int:
    """Bring one (b, kv-head) K Compression Cache up to date; return the new valid count.

    Entries n in [valid, floor(length/b)) are computed from their b keys;
    entries below `valid` are left untouched [CP Knowl 5: each time b new tokens
    exist, one entry is built from those b keys].
    k_nope: [>= length, d] pre-RoPE keys; kcomp: [max_blocks, d_gate] (written in place).
    """
    nfull = length // block
    for n in range(valid, nfull):
        kcomp[n] = k_gate_entry(k_nope[n * block:(n + 1) * block], w_k, n, block, base)
    return nfull


def kcomp_append(state: np.ndarray, k_new: np.ndarray, length: int, valid: int, w_k: np.ndarray,
                 kcomp: np.ndarray, block: int, base: float) -> int:
    """The same cache update, one appended token at a time, from running block statistics.

    Each entry is built from the b keys of one finished block [CP Knowl 5], so a decoder only
    needs those keys' per-channel max, min and sum, not a pre-RoPE copy of the whole context.  `k_new` [d] is the pre-RoPE key of token length-1; `state` [3, d] holds the running
    max / min / sum of the current block's keys (restarted at a block's first token).  When the
    token completes block n, kcomp[n] = bf16(RoPE_{n*b}(W_k . [max | min | sum/b])) and the fill
    count becomes n+1 (the block's earlier entries must already be there: valid == n).
    Returns the new fill count.
    """
    if length <= 0:
        return valid
    n, pos = divmod(length - 1, block)
    k = np.asarray(k_new, dtype=np.float64)
    if pos == 0:
        state[0], state[1], state[2] = k, k, k
    else:
        state[0] = np.maximum(state[0], k)
        state[1] = np.minimum(state[1], k)
        state[2] = state[2] + k
    if pos != block - 1:
        return valid
    if valid != n:
        raise ValueError(f"block {n} completes with {valid} entries present")
    pooled = np.concatenate([state[0], state[1], state[2] / block])
    y = np.asarray(w_k, dtype=np.float64) @ pooled
    kcomp[n] = round_to_bf16(rope(y, n * block, base))
    return n + 1


def q_gate(q_nope: np.ndarray, w_q: np.ndarray, length: int, base: float) -> np.ndarray:
    """Gate query of one KV head: RoPE_{L-1}(W_q . reshape(q_group, [g*d])).

    q_nope: [g, d] pre-RoPE queries of the group (query heads h*g .. h*g+g-1);
    w_q: [d_gate, g*d].  [CP Knowl 1-2; PN design 1: one W_q set per KV head]
    """
    q = np.asarray(q_nope, dtype=np.float64)
    qcat = q.reshape(-1)                 # head-major: index j*d + c
    return rope(np.asarray(w_q, dtype=np.float64) @ qcat, length - 1, base)


def gate_logits(qg: np.ndarray, kcomp: np.ndarray, length: int, block: int) -> np.ndarray:
    """Scaled gate logits Q_gate . K_gate[n] / sqrt(d_gate) of the floor(L/b) full blocks."""
    nfull = length // block
    dg = qg.shape[0]
    return np.asarray(kcomp[:nfull], dtype=np.float64) @ qg / math.sqrt(dg)


def gate_scores(logits: np.ndarray) -> np.ndarray:
    """S = softmax(logits) over the scored blocks [CP Knowl 2]."""
    z = np.asarray(logits, dtype=np.float64)
    if z.size == 0:
        return z.copy()
    e = np.exp(z - z.max())
    return e / e.sum()


# ----------------------------------------------------------------------------
# Block selection  [CP Knowl 5; PN training-strategy paragraph]
# ----------------------------------------------------------------------------

def _with_partial(chosen: Iterable[int], length: int, block: int) -> List[int]:
    out = sorted(int(n) for n in chosen)
    if length % block != 0:
        out.append(length // block)      # incomplete last block, always selected
    return out


def select_topk(logits: np.ndarray, k: int, length: int, block: int) -> List[int]:
    """Top-k full blocks by logit (ties -> lower index) plus the forced partial block."""
    nfull = length // block
    z = [float(x) for x in np.asarray(logits, dtype=np.float64)[:nfull]]
    order = sorted(range(nfull), key=lambda n: (-z[n], n))
    return _with_partial(order[:min(k, nfull)], length, block)


def select_threshold(logits: np.ndarray, tau: float, length: int, block: int) -> List[int]:
    """Full blocks whose score S exceeds tau (strict), plus the forced partial block."""
    nfull = length // block
    s = gate_scores(np.asarray(logits, dtype=np.float64)[:nfull])
    return _with_partial([n for n in range(nfull) if s[n] > tau], length, block)


def select_topp(logits: np.ndarray, p: float, length: int, block: int) -> List[int]:
    """Fewest full blocks whose score mass reaches p (nucleus), plus the partial block.

    Blocks are taken in descending score order (ties -> lower index) until
    their S-sum is >= p.  [CP Knowl 14: top-p as adaptive sparsity]
    """
    nfull = length // block
    s = gate_scores(np.asarray(logits, dtype=np.float64)[:nfull])
    order = sorted(range(nfull), key=lambda n: (-float(s[n]), n))
    chosen, mass = [], 0.0
    for n in order:
        if mass >= p:
            break
        chosen.append(n)
        mass += float(s[n])
    return _with_partial(chosen, length, block)


# ----------------------------------------------------------------------------
# Block-sparse decode attention and the split combine  [CP Knowl 6; SK]
# ----------------------------------------------------------------------------

def block_tokens(blocks: Sequence[int], length: int, block: int) -> np.ndarray:
    """Token positions covered by `blocks`, clipped to the first `length` tokens."""
    toks: List[int] = []
    for n in blocks:
        toks.extend(range(n * block, min((n + 1) * block, length)))
    return np.asarray(toks, dtype=np.int64)


def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray, tokens: np.ndarray,
           scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Softmax attention of queries q [g, d] over the listed token rows of k, v.

    Returns (o [g, d], lse [g]) with lse = log sum_t exp(scale * q . k_t).
    An empty token set gives o = 0 and lse = -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    if tokens.size == 0:
        return np.zeros_like(q), np.full(q.shape[0], NEG_INF)
    kk = np.asarray(k[tokens], dtype=np.float64)
    vv = np.asarray(v[tokens], dtype=np.float64)
    s = scale * (q @ kk.T)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=1, keepdims=True)
    return (e @ vv) / z, (m + np.log(z))[:, 0]


def sparse_decode(q: np.ndarray, k: np.ndarray, v: np.ndarray, blocks: Sequence[int],
                  length: int, block: int, scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Attention of one query group over the selected blocks only (one KV head)."""
    return attend(q, k, v, block_tokens(blocks, length, block), scale)


def combine(parts: Sequence[Tuple[np.ndarray, np.ndarray]]) -> Tuple[np.ndarray, np.ndarray]:
    """Log-sum-exp merge of per-split (o, lse) results of the same queries."""
    lses = np.stack([p[1] for p in parts])            # [ns, g]
    os_ = np.stack([p[0] for p in parts])             # [ns, g, d]
    top = lses.max(axis=0)
    safe = np.where(np.isfinite(top), top, 0.0)
    w = np.exp(lses - safe)                           # exp(-inf) = 0 for empty splits
    tot = w.sum(axis=0)
    o = np.where(tot[:, None] > 0, (w[:, :, None] * os_).sum(axis=0) / np.where(tot > 0, tot, 1.0)[:, None], 0.0)
    lse = np.where(tot > 0, safe + np.log(np.where(tot > 0, tot, 1.0)), NEG_INF)
    return o, lse


def split_list(blocks: Sequence[int], capacity: int, num_split: int) -> List[List[int]]:
    """Partition a selected list by list position, capacity/num_split slots per split.

    The split size comes from the index tensor's width (max_selected_blocks),
    not from the sequence's block count [CP Knowl 6].
    """
    per = -(-capacity // num_split)
    return [list(blocks[s * per:(s + 1) * per]) for s in range(num_split)]


# ----------------------------------------------------------------------------
# Decode ground truth / oracle block scores  [CP Knowl 3]
# ----------------------------------------------------------------------------

def decode_ground_truth(q: np.ndarray, k: np.ndarray, length: int, block: int,
                        scale: float) -> np.ndarray:
    """Block-level target of one KV head from full attention.

    softmax(scale * q K^T) over all `length` tokens for each of the g heads,
    1-D max-pooled over each block's columns, max over the g heads, then
    normalised to sum to 1.  Length ceil(L/b).
    """
    q = np.asarray(q, dtype=np.float64)
    kk = np.asarray(k[:length], dtype=np.float64)
    s = scale * (q @ kk.T)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    nblk = -(-length // block)
    col = np.array([[p[i, n * block:min((n + 1) * block, length)].max() for n in range(nblk)]
                    for i in range(q.shape[0])])
    gt = col.max(axis=0)
    return gt / gt.sum()


def prefill_ground_truth(q: np.ndarray, k: np.ndarray, v: np.ndarray, block: int,
                         scale: float) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Causal attention of a whole sequence for one KV head, with the block-level target of
    every query position beside it (the training-side ground truth [CP Knowl 3, Knowl 4]).

    q: [g, L, d] (the GQA group's query heads), k, v: [L, d].  Query i attends keys 0..i.
    Returns o [g, L, d], lse [g, L] and gt [L, ceil(L/b)]: row i is the decode target of
    query position i -- the softmax map's row 1-D max-pooled over each block's (visible)
    columns, max over the g heads, normalised to sum to 1; blocks past position i are 0.
    """
    q = np.asarray(q, dtype=np.float64)
    kk = np.asarray(k, dtype=np.float64)
    vv = np.asarray(v, dtype=np.float64)
    g, L, _ = q.shape
    s = scale * np.einsum("hid,td->hit", q, kk)
    visible = np.tril(np.ones((L, L), dtype=bool))
    s = np.where(visible[None], s, NEG_INF)
    m = s.max(axis=2, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=2, keepdims=True)
    p = e / z
    o = np.einsum("hit,td->hid", p, vv)
    lse = (m + np.log(z))[..., 0]
    nblk = -(-L // block)
    pooled = np.stack([p[:, :, n * block:min((n + 1) * block, L)].max(axis=2) for n in range(nblk)], axis=2)
    gt = pooled.max(axis=0)
    return o, lse, gt / gt.sum(axis=1, keepdims=True)


# ----------------------------------------------------------------------------
# One whole decode step for one (batch, kv-head)
# ----------------------------------------------------------------------------

def decode_step_bh(q_group: np.ndarray, k: np.ndarray, v: np.ndarray, w_q: np.ndarray,
                   kcomp: np.ndarray, length: int, block: int, base: float, mode: str,
                   k_blocks: int = 0, tau: float = 0.0, scale: float = 0.0):
    """Gate -> select -> sparse attention for one (b, kv-head), kcomp already current.

    Returns dict(logits, blocks, o [g, d], lse [g]).  q_group doubles as the
    pre-RoPE gate input (the synthetic workloads alias q_nope and q).
    """
    d = q_group.shape[1]
    scale = scale or 1.0 / math.sqrt(d)
    qg = q_gate(q_group, w_q, length, base)
    logits = gate_logits(qg, kcomp, length, block)
    if mode == "topk":
        blocks = select_topk(logits, k_blocks, length, block)
    elif mode == "threshold":
        blocks = select_threshold(logits, tau, length, block)
    else:
        raise ValueError(mode)
    o, lse = sparse_decode(q_group, k, v, blocks, length, block, scale)
    return dict(q_gate=qg, logits=logits, blocks=blocks, o=o, lse=lse)
