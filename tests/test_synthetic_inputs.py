"""The seeded input recipe the tests and the benchmark share: the five workloads' shapes and
seeds, ragged lengths that are never a multiple of the block, counter-keyed streams (a slice
regenerates alone and identically), the value distributions, the planted "hot" blocks and the
NaN tails."""

import math

import numpy as np

from synthetic import CONFIGS, bf16_bits_to_f32, config, make_inputs, make_pair_inputs
from synthetic.inputs import BF16_NAN_BITS, _lengths


def test_workload_table():
    want = {1: (1, 4, 1, 64, 64, 64, 2048, "topk", 512),
            2: (8, 32, 8, 128, 128, 64, 32768, "topk", 4096),
            3: (16, 40, 8, 128, 128, 128, 0, "topk", 4096),
            4: (4, 32, 8, 128, 128, 64, 65536, "topk", 6554),
            5: (32, 32, 8, 128, 128, 64, 16384, "threshold", 0)}
    for cid, w in want.items():
        c = CONFIGS[cid]
        assert (c.B, c.Hq, c.Hkv, c.head_dim, c.gate_dim, c.block, c.length, c.mode, c.budget) == w, cid
        assert c.seed == 1000 + cid
    assert CONFIGS[2].topk_blocks == 64 and CONFIGS[2].hot_blocks == 8
    assert CONFIGS[3].length_range == (8000, 32000)
    assert CONFIGS[5].steps == 256 and CONFIGS[5].tau == 1.0 / 512.0


def test_ragged_lengths():
    c = CONFIGS[3]
    L = _lengths(c)
    assert L.shape == (16,) and np.all((L >= 8000) & (L <= 32000)) and np.all(L % 128 != 0)
    assert np.array_equal(L, _lengths(c)), "lengths are seeded"


def test_streams_are_per_slice_and_reproducible():
    a = make_inputs(config(1, B=2, Hq=8, Hkv=2, hot_blocks=2), lengths=[300, 200])
    b = make_inputs(config(1, B=2, Hq=8, Hkv=2, hot_blocks=2), lengths=[300, 200])
    for name in ("q", "k", "v", "w_q", "w_k"):
        assert np.array_equal(getattr(a, name), getattr(b, name)), name
    # one more sequence in the batch leaves the existing slices' draws unchanged
    c = make_inputs(config(1, B=3, Hq=8, Hkv=2, hot_blocks=2), lengths=[300, 200, 100])
    assert np.array_equal(a.k[0, 1, :300], c.k[0, 1, :300]) and np.array_equal(a.v[1, 0, :200], c.v[1, 0, :200])
    assert np.array_equal(a.w_q, c.w_q) and np.array_equal(a.w_k, c.w_k)


def test_value_distributions():
    cfg = config(1, B=2, Hq=8, Hkv=2, head_dim=128, gate_dim=128, seed=77)
    inp = make_inputs(cfg, lengths=[4096, 4096])
    for name, x in (("q", inp.q), ("k", inp.k), ("v", inp.v)):
        f = bf16_bits_to_f32(x).astype(np.float64)
        assert abs(f.mean()) < 0.02 and abs(f.std() - 1.0) < 0.02, name
    g, d = cfg.g, cfg.head_dim
    wq = bf16_bits_to_f32(inp.w_q).astype(np.float64)
    wk = bf16_bits_to_f32(inp.w_k).astype(np.float64)
    assert abs(wq.std() * math.sqrt(g * d) - 1.0) < 0.02, "W_q ~ N(0, 1/(g d))"
    assert abs(wk.std() * math.sqrt(3 * d) - 1.0) < 0.02, "W_k ~ N(0, 1/(3 d))"


def test_hot_blocks_and_nan_tail():
    blk = 64
    cfg = config(1, B=1, Hq=4, Hkv=1, head_dim=64, gate_dim=64, block=blk, hot_blocks=3, seed=91)
    L = 20 * blk + 7
    inp = make_inputs(cfg, lengths=[L], tail="nan")
    hot = inp.hot[(0, 0)]
    assert len(hot) == 3 == len(set(hot)) and all(0 <= n < L // blk for n in hot)
    qs = bf16_bits_to_f32(inp.q[0, 0:4]).astype(np.float64).sum(axis=0)
    qhat = qs / np.linalg.norm(qs)
    proj = bf16_bits_to_f32(inp.k[0, 0, :L]).astype(np.float64) @ qhat
    for n in range(L // blk):
        m = proj[n * blk:(n + 1) * blk].mean()
        if n in hot:
            assert abs(m - 3.0) < 0.5, f"hot block {n}: mean projection {m:.2f}"
        else:
            assert abs(m) < 0.5, f"block {n}: mean projection {m:.2f}"
    assert np.all(inp.k[0, 0, L:] == BF16_NAN_BITS) and np.all(inp.v[0, 0, L:] == BF16_NAN_BITS)
    assert not np.any(inp.k[0, 0, :L] == BF16_NAN_BITS)


def test_pair_inputs_are_the_batch_slices():
    """One (b, kv-head) drawn on its own equals the same slice of the whole batch (planted blocks
    and ragged lengths included)."""
    for cid, over in ((2, dict(B=2, Hkv=2, Hq=8, length=1000)), (3, dict(B=3, Hkv=2, Hq=10))):
        cfg = config(cid, **over)
        inp = make_inputs(cfg)
        for b in range(cfg.B):
            for h in range(cfg.Hkv):
                pi = make_pair_inputs(cfg, b, h)
                assert pi.length == int(inp.seqlens[b])
                assert np.array_equal(pi.k, inp.k[b, h]) and np.array_equal(pi.v, inp.v[b, h])
                assert np.array_equal(pi.q, inp.q[b, h * cfg.g:(h + 1) * cfg.g])
                assert np.array_equal(pi.w_q, inp.w_q[h]) and np.array_equal(pi.w_k, inp.w_k[h])


def test_parallel_draw_is_the_serial_draw():
    """Drawing the K / V slices in spawned processes gives the serial loop's bytes, planted blocks
    and NaN tails."""
    cfg = config(2, B=3, Hkv=2, Hq=8, length=700, steps=3)
    a = make_inputs(cfg, tail="nan", lengths=[700, 650, 3])
    b = make_inputs(cfg, tail="nan", lengths=[700, 650, 3], workers=3)
    assert np.array_equal(a.k, b.k) and np.array_equal(a.v, b.v)
    assert a.hot == b.hot and np.array_equal(a.seqlens, b.seqlens)


def test_bf16_rounding_matches_torch():
    """The generator's float32 -> bf16 rounding (nearest, ties to even) against torch's conversion on
    every exponent with mantissas at, just below and just above the rounding midpoints, odd and even
    kept parts, zeros, infinities and subnormals (NaN payloads excluded: torch canonicalises them)."""
    import torch
    from synthetic import bf16_bits_from_f32
    mant = np.array([0, 1, 0x7FFF, 0x8000, 0x8001, 0x17FFF, 0x18000, 0x18001, 0x7FFFFF, 0x7F8000, 0x3FFFFF],
                    dtype=np.uint32)
    exps = np.arange(0, 255, dtype=np.uint32)
    bits = ((exps[:, None] << np.uint32(23)) | mant[None, :]).ravel()
    bits = np.concatenate([bits, bits | np.uint32(0x80000000), np.array([0x7F800000, 0xFF800000], np.uint32)])
    x = bits.view(np.float32)
    want = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bf16_bits_from_f32(x), want)
