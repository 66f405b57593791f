"""Seeded synthetic decode-step inputs.

Every tensor is drawn from its own counter-keyed PCG64 stream
(``SeedSequence(seed, spawn_key=(tag, i, j))``), so any (batch, kv-head)
slice can be regenerated on its own and two runs with the same seed produce
identical bytes.  bf16 tensors are returned as their raw uint16 bit patterns
(round-to-nearest-even from float32 draws), which both the CUDA path (as
``torch.bfloat16``) and the CPU oracle (widened to float64) consume exactly.

Workload shapes follow the five decode configurations this library is
measured on: a tiny single-head-group step, a Qwen3-8B-shaped 32k step with
planted "hot" blocks, a Qwen3-14B-shaped ragged batch with block size 128, a
64k sparsity sweep and a 256-step threshold decode loop.  The pages measure
on reasoning benchmarks (AIME, MATH-500, GPQA); these seeded N(0,1) tensors
stand in for a model's activations on them.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

# stream tags
_T_Q, _T_K, _T_V, _T_WQ, _T_WK, _T_LEN, _T_HOT, _T_PAGES = range(8)

BF16_NAN_BITS = 0x7FC0


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=tuple(key))))


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bits.  The sum is taken
    modulo 2^32: only its bits 16..31 are kept, which a wider sum would give the same."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    b = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return b.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    B: int
    Hq: int
    Hkv: int
    head_dim: int
    gate_dim: int
    block: int
    length: int = 0                       # fixed context length (tokens, incl. the current one)
    length_range: Tuple[int, int] = (0, 0)  # ragged: uniform per sequence, never a multiple of block
    mode: str = "topk"                    # "topk" | "threshold"
    budget: int = 0                       # token budget (top-k)
    tau: float = 0.0                      # score threshold (threshold mode)
    hot_blocks: int = 0                   # planted q-aligned blocks per (b, kv head)
    steps: int = 1                        # decode steps (one appended token each)
    rope_base: float = 1e6
    seed: int = 0

    @property
    def g(self) -> int:
        return self.Hq // self.Hkv

    @property
    def topk_blocks(self) -> int:
        return -(-self.budget // self.block)


CONFIGS: Dict[int, DecodeConfig] = {
    1: DecodeConfig("tiny-decode-step", B=1, Hq=4, Hkv=1, head_dim=64, gate_dim=64, block=64,
                    length=2048, mode="topk", budget=512, seed=1001),
    2: DecodeConfig("qwen3-8b-32k-step", B=8, Hq=32, Hkv=8, head_dim=128, gate_dim=128, block=64,
                    length=32768, mode="topk", budget=4096, hot_blocks=8, seed=1002),
    3: DecodeConfig("qwen3-14b-ragged-step", B=16, Hq=40, Hkv=8, head_dim=128, gate_dim=128,
                    block=128, length_range=(8000, 32000), mode="topk", budget=4096, seed=1003),
    4: DecodeConfig("sparsity-sweep-64k", B=4, Hq=32, Hkv=8, head_dim=128, gate_dim=128, block=64,
                    length=65536, mode="topk", budget=6554, seed=1004),
    5: DecodeConfig("decode-loop-256-threshold", B=32, Hq=32, Hkv=8, head_dim=128, gate_dim=128,
                    block=64, length=16384, mode="threshold", tau=1.0 / 512.0, hot_blocks=8,
                    steps=256, seed=1005),
}

SWEEP_SPARSITIES = (0.50, 0.75, 0.90, 0.95)


def sweep_budget(length: int, sparsity: float) -> int:
    """Token budget that keeps (1 - sparsity) of a `length`-token context."""
    return int(math.ceil((1.0 - sparsity) * length - 1e-9))


def config(cid: int, **overrides) -> DecodeConfig:
    base = CONFIGS[cid]
    if not overrides:
        return base
    d = dict(base.__dict__)
    d.update(overrides)
    return DecodeConfig(**d)


@dataclass
class DecodeInputs:
    cfg: DecodeConfig
    seqlens: np.ndarray            # int32 [B]  current lengths (incl. the current token)
    final_lens: np.ndarray         # int32 [B]  lengths after all decode steps
    q: np.ndarray                  # uint16 [B, Hq, d]    (step 0 query; also q_nope)
    k: np.ndarray                  # uint16 [B, Hkv, Lcap, d]  (also k_nope)
    v: np.ndarray                  # uint16 [B, Hkv, Lcap, d]
    w_q: np.ndarray                # uint16 [Hkv, d_gate, g*d]
    w_k: np.ndarray                # uint16 [Hkv, d_gate, 3*d]
    hot: Dict[Tuple[int, int], List[int]] = field(default_factory=dict)

    @property
    def lcap(self) -> int:
        return self.k.shape[2]

    @property
    def max_blocks(self) -> int:
        return -(-self.lcap // self.cfg.block)


def _lengths(cfg: DecodeConfig) -> np.ndarray:
    if cfg.length_range != (0, 0):
        lo, hi = cfg.length_range
        rng = _rng(cfg.seed, _T_LEN)
        out = []
        for _ in range(cfg.B):
            while True:
                L = int(rng.integers(lo, hi + 1))
                if L % cfg.block != 0:
                    break
            out.append(L)
        return np.asarray(out, dtype=np.int32)
    return np.full(cfg.B, cfg.length, dtype=np.int32)


def make_step_query(cfg: DecodeConfig, step: int) -> np.ndarray:
    """Query (bf16 bits, [B, Hq, d]) of decode step `step` (step 0 = the initial query)."""
    q = np.empty((cfg.B, cfg.Hq, cfg.head_dim), dtype=np.uint16)
    for b in range(cfg.B):
        r = _rng(cfg.seed, _T_Q, step, b)
        q[b] = bf16_bits_from_f32(r.standard_normal((cfg.Hq, cfg.head_dim), dtype=np.float32))
    return q


def _kv_slice(cfg: DecodeConfig, b: int, h: int, length: int, final: int, lcap: int, q32: np.ndarray,
              tail: str):
    """The K and V rows (bf16 bits, [lcap, d]) of one (b, kv-head), and its planted blocks (or None)."""
    d, blk, g = cfg.head_dim, cfg.block, cfg.g
    kf = _rng(cfg.seed, _T_K, b, h).standard_normal((lcap, d), dtype=np.float32)
    vf = _rng(cfg.seed, _T_V, b, h).standard_normal((lcap, d), dtype=np.float32)
    nfull0 = length // blk
    chosen = None
    if cfg.hot_blocks and nfull0 > 0:
        qs = q32[b, h * g:(h + 1) * g].astype(np.float64).sum(axis=0)
        qhat = (qs / np.linalg.norm(qs)).astype(np.float32)
        chosen = sorted(int(x) for x in _rng(cfg.seed, _T_HOT, b, h).choice(
            nfull0, size=min(cfg.hot_blocks, nfull0), replace=False))
        for n in chosen:
            kf[n * blk:(n + 1) * blk] += np.float32(3.0) * qhat
    k = bf16_bits_from_f32(kf)
    v = bf16_bits_from_f32(vf)
    if tail == "nan":
        k[final:] = BF16_NAN_BITS
        v[final:] = BF16_NAN_BITS
    return k, v, chosen


@dataclass
class PairInputs:
    """The inputs of one (b, kv-head) of a decode problem, as make_inputs draws them."""
    length: int
    q: np.ndarray       # uint16 [g, d]  the group's query rows
    k: np.ndarray       # uint16 [lcap, d]
    v: np.ndarray       # uint16 [lcap, d]
    w_q: np.ndarray     # uint16 [d_gate, g*d]
    w_k: np.ndarray     # uint16 [d_gate, 3*d]


def make_pair_inputs(cfg: DecodeConfig, b: int, h: int) -> PairInputs:
    """One (b, kv-head)'s slices of make_inputs(cfg) (default lengths and tail), drawn from the same
    streams without drawing the rest of the batch."""
    d, dg, blk, g = cfg.head_dim, cfg.gate_dim, cfg.block, cfg.g
    seqlens = _lengths(cfg)
    final = seqlens + (cfg.steps - 1 if cfg.steps > 1 else 0)
    lcap = int(-(-int(final.max()) // blk) * blk) if final.max() > 0 else blk
    q = make_step_query(cfg, 0)
    k, v, _ = _kv_slice(cfg, b, h, int(seqlens[b]), int(final[b]), lcap, bf16_bits_to_f32(q), "random")
    w_q = bf16_bits_from_f32(_rng(cfg.seed, _T_WQ, h).standard_normal((dg, g * d), dtype=np.float32)
                             / np.float32(math.sqrt(g * d)))
    w_k = bf16_bits_from_f32(_rng(cfg.seed, _T_WK, h).standard_normal((dg, 3 * d), dtype=np.float32)
                             / np.float32(math.sqrt(3 * d)))
    return PairInputs(length=int(seqlens[b]), q=q[b, h * g:(h + 1) * g], k=k, v=v, w_q=w_q, w_k=w_k)


def _kv_fill(cfg, path_k, path_v, shape, pairs, seqlens, final, q32, tail, results):
    """Worker of make_inputs(workers > 1): draw a share of the (b, kv-head) slices straight into the
    file-backed K and V arrays; puts the share's planted blocks on `results`."""
    k = np.memmap(path_k, dtype=np.uint16, mode="r+", shape=shape)
    v = np.memmap(path_v, dtype=np.uint16, mode="r+", shape=shape)
    hot = {}
    for (b, h) in pairs:
        k[b, h], v[b, h], chosen = _kv_slice(cfg, b, h, int(seqlens[b]), int(final[b]), shape[2], q32, tail)
        if chosen is not None:
            hot[(b, h)] = chosen
    k.flush()
    v.flush()
    del k, v
    results.put(hot)


def _kv_parallel(cfg, seqlens, final, lcap, q32, tail, workers):
    """The K and V slices drawn by `workers` spawned processes (each slice has its own stream, so the
    bytes are those of the serial loop).  A worker that dies raises here instead of being waited
    for."""
    import multiprocessing as mp
    import os
    import queue
    import shutil
    import tempfile
    shape = (cfg.B, cfg.Hkv, lcap, cfg.head_dim)
    pairs = [(b, h) for b in range(cfg.B) for h in range(cfg.Hkv)]
    tmp = tempfile.mkdtemp(prefix="seer_inputs_")
    ctx = mp.get_context("spawn")
    procs = []
    try:
        pk, pv = os.path.join(tmp, "k.u16"), os.path.join(tmp, "v.u16")
        for path in (pk, pv):
            np.memmap(path, dtype=np.uint16, mode="w+", shape=shape).flush()
        W = max(1, min(workers, len(pairs)))
        results = ctx.Queue()
        procs = [ctx.Process(target=_kv_fill, args=(cfg, pk, pv, shape, pairs[i::W], seqlens, final, q32, tail,
                                                    results), daemon=True) for i in range(W)]
        for p in procs:
            p.start()
        parts = []
        while len(parts) < W:
            try:
                parts.append(results.get(timeout=5))
            except queue.Empty:
                if any(p.exitcode not in (None, 0) for p in procs):
                    raise RuntimeError("a worker drawing the synthetic K / V slices failed")
        for p in procs:
            p.join()
        k = np.array(np.memmap(pk, dtype=np.uint16, mode="r", shape=shape))
        v = np.array(np.memmap(pv, dtype=np.uint16, mode="r", shape=shape))
    finally:
        for p in procs:
            if p.is_alive():
                p.kill()
        shutil.rmtree(tmp, ignore_errors=True)
    hot: Dict[Tuple[int, int], List[int]] = {}
    for part in parts:
        hot.update(part)
    return k, v, dict(sorted(hot.items()))


def make_inputs(cfg: DecodeConfig, *, tail: str = "random",
                lengths: Optional[Sequence[int]] = None, workers: int = 1) -> DecodeInputs:
    """Draw one decode problem.

    tail="nan" fills cache rows past each sequence's final length with bf16
    NaN, so any read of a masked token poisons the result.  workers > 1 draws
    the K / V slices in that many spawned processes (same bytes).
    """
    B, Hq, Hkv, d, dg, blk = cfg.B, cfg.Hq, cfg.Hkv, cfg.head_dim, cfg.gate_dim, cfg.block
    g = cfg.g
    seqlens = np.asarray(lengths, dtype=np.int32) if lengths is not None else _lengths(cfg)
    final = seqlens + (cfg.steps - 1 if cfg.steps > 1 else 0)
    lcap = int(-(-int(final.max()) // blk) * blk) if final.max() > 0 else blk

    q = make_step_query(cfg, 0)
    q32 = bf16_bits_to_f32(q)

    w_q = np.empty((Hkv, dg, g * d), dtype=np.uint16)
    w_k = np.empty((Hkv, dg, 3 * d), dtype=np.uint16)
    for h in range(Hkv):
        w_q[h] = bf16_bits_from_f32(_rng(cfg.seed, _T_WQ, h).standard_normal((dg, g * d), dtype=np.float32)
                                    / np.float32(math.sqrt(g * d)))
        w_k[h] = bf16_bits_from_f32(_rng(cfg.seed, _T_WK, h).standard_normal((dg, 3 * d), dtype=np.float32)
                                    / np.float32(math.sqrt(3 * d)))

    if workers > 1 and B * Hkv > 1:
        k, v, hot = _kv_parallel(cfg, seqlens, final, lcap, q32, tail, workers)
    else:
        k = np.empty((B, Hkv, lcap, d), dtype=np.uint16)
        v = np.empty((B, Hkv, lcap, d), dtype=np.uint16)
        hot = {}
        for b in range(B):
            for h in range(Hkv):
                k[b, h], v[b, h], chosen = _kv_slice(cfg, b, h, int(seqlens[b]), int(final[b]), lcap, q32, tail)
                if chosen is not None:
                    hot[(b, h)] = chosen
    return DecodeInputs(cfg=cfg, seqlens=seqlens, final_lens=final.astype(np.int32), q=q, k=k, v=v,
                        w_q=w_q, w_k=w_k, hot=hot)


def scale_gate_weights(w_q: np.ndarray, c: Sequence[float]) -> np.ndarray:
    """Multiply W_q[h] by c[h] (a per-head logit temperature) and re-round to bf16."""
    w = bf16_bits_to_f32(w_q).copy()
    for h, ch in enumerate(c):
        w[h] *= np.float32(ch)
    return bf16_bits_from_f32(w)


def paged_view(x: np.ndarray, block: int, seed: int, spare_pages: int = 3):
    """Scatter a contiguous [B, Hkv, Lcap, d] cache into a shuffled page pool.

    Returns (pool [P, Hkv, block, d], block_table int32 [B, Lcap // block]).
    Page ids are a seeded permutation, so logical neighbours are not physical
    neighbours.  Unused pool pages hold bf16 NaN.
    """
    B, Hkv, lcap, d = x.shape
    assert lcap % block == 0
    npb = lcap // block
    P = B * npb + spare_pages
    perm = _rng(seed, _T_PAGES).permutation(P)[: B * npb].astype(np.int32)
    table = perm.reshape(B, npb)
    pool = np.full((P, Hkv, block, d), BF16_NAN_BITS, dtype=np.uint16)
    for b in range(B):
        for n in range(npb):
            pool[table[b, n]] = x[b, :, n * block:(n + 1) * block, :]
    return pool, table


_T_LOGITS, _T_LISTS = 8, 9


def make_logits(seed: int, B: int, Hkv: int, nb: int, kind: str = "normal") -> np.ndarray:
    """float32 [B, Hkv, nb] score rows: N(0, 2^2) draws, or small integers (many exact ties)."""
    r = _rng(seed, _T_LOGITS)
    if kind == "ties":
        return r.integers(-3, 4, size=(B, Hkv, nb)).astype(np.float32)
    return (r.standard_normal((B, Hkv, nb)) * 2.0).astype(np.float32)


def make_block_lists(seed: int, seqlens: Sequence[int], Hkv: int, block: int, capacity: int,
                     density: float = 0.3, force_partial: bool = True):
    """Random ascending block lists: idx int32 [B, Hkv, capacity] (-1 padded), cnt int32 [B, Hkv].

    Each full block is kept with probability `density` (at most capacity - 1 of
    them); the partial last block is appended when the length leaves one.
    """
    r = _rng(seed, _T_LISTS)
    B = len(seqlens)
    idx = np.full((B, Hkv, capacity), -1, dtype=np.int32)
    cnt = np.zeros((B, Hkv), dtype=np.int32)
    for b in range(B):
        L = int(seqlens[b])
        nfull = L // block
        for h in range(Hkv):
            keep = [n for n in range(nfull) if r.random() < density][: capacity - 1]
            if force_partial and L % block:
                keep.append(nfull)
            idx[b, h, :len(keep)] = keep
            cnt[b, h] = len(keep)
    return idx, cnt
