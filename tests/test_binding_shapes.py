"""The Python binding refuses buffers whose shape differs from the problem shape (the kernels index
them by it); right shapes get past the check (on a CPU-only host they then stop at the CUDA-tensor
check, before any device work)."""

import pytest
import torch

import block_sparse_attention_attngate_b200 as S

B, HQ, HKV, D, DG, BLK, NB = 2, 8, 2, 128, 64, 64, 16


def _shape():
    return S.Shape(B, HQ, HKV, D, DG, BLK, NB)


def _cache(t=None):
    """A KVCache over a host tensor (the classmethods want CUDA tensors; the shape check does not)."""
    t = torch.zeros(B, HKV, NB * BLK, D, dtype=torch.bfloat16) if t is None else t
    desc = S.KVDesc(S.KV_CONTIGUOUS, 0, t.stride(0), t.stride(1), t.stride(2), t.shape[2], 0, None, 0)
    return S.seer.KVCache(desc, (t,))


def _paged(pool, table):
    desc = S.KVDesc(S.KV_PAGED, 0, pool.stride(0), pool.stride(1), pool.stride(2), 0, pool.shape[0], None,
                    table.shape[1])
    return S.seer.KVCache(desc, (pool, table))


def _i32(*shape):
    return torch.zeros(*shape, dtype=torch.int32)


def _accepts(fn, **kw):
    with pytest.raises(TypeError, match="CUDA tensor"):
        fn(_shape(), **kw)


def _rejects(fn, good, name, bad, match=None):
    with pytest.raises(ValueError, match=match or name):
        fn(_shape(), **{**good, name: bad})


def test_kcomp_append_shapes():
    good = dict(k_new=torch.zeros(B, HKV, D), seqlens=_i32(B), state=torch.zeros(B, HKV, 3, D),
                valid_blocks=_i32(B, HKV), w_k=torch.zeros(HKV, DG, 3 * D), kcomp=torch.zeros(B, HKV, NB, DG))
    _accepts(S.kcomp_append, **good)
    for name, bad in (("state", torch.zeros(B, HKV, 3, 64)), ("kcomp", torch.zeros(B, HKV, 8, DG)),
                      ("k_new", torch.zeros(B, D)), ("w_k", torch.zeros(HKV, DG, 2 * D)),
                      ("valid_blocks", _i32(B)), ("err", _i32(0))):
        _rejects(S.kcomp_append, good, name, bad)


def test_kcomp_state_init_shapes():
    good = dict(k_nope=_cache(), seqlens=_i32(B), state=torch.zeros(B, HKV, 3, D))
    _accepts(S.kcomp_state_init, **good)
    _rejects(S.kcomp_state_init, good, "state", torch.zeros(B, HKV, 3, 64))
    _rejects(S.kcomp_state_init, good, "k_nope", _cache(torch.zeros(B, 1, NB * BLK, D)))


def test_kcomp_update_shapes():
    good = dict(k_nope=_cache(), seqlens=_i32(B), valid_blocks=_i32(B, HKV), w_k=torch.zeros(HKV, DG, 3 * D),
                kcomp=torch.zeros(B, HKV, NB, DG))
    _accepts(S.kcomp_update, **good)
    for name, bad in (("k_nope", _cache(torch.zeros(B - 1, HKV, NB * BLK, D))), ("seqlens", _i32(B + 1)),
                      ("valid_blocks", _i32(B, HKV + 1)), ("kcomp", torch.zeros(B, HKV, NB, D))):
        _rejects(S.kcomp_update, good, name, bad)
    # a paged pool must have the shape's block size
    pool, table = torch.zeros(40, HKV, BLK, D), _i32(B, NB)
    _accepts(S.kcomp_update, **{**good, "k_nope": _paged(pool, table)})
    _rejects(S.kcomp_update, good, "k_nope", _paged(torch.zeros(40, HKV, 2 * BLK, D), table))
    _rejects(S.kcomp_update, good, "k_nope", _paged(pool, _i32(B - 1, NB)))


def test_gate_score_shapes():
    good = dict(q_nope=torch.zeros(B, HQ, D), w_q=torch.zeros(HKV, DG, (HQ // HKV) * D),
                kcomp=torch.zeros(B, HKV, NB, DG), seqlens=_i32(B), logits=torch.zeros(B, HKV, NB),
                q_gate=torch.zeros(B, HKV, DG))
    _accepts(S.gate_score, **good)
    for name, bad in (("q_nope", torch.zeros(B, HKV, D)), ("w_q", torch.zeros(HKV, DG, D)),
                      ("logits", torch.zeros(B, HKV, NB - 1)), ("q_gate", torch.zeros(B, HKV, D))):
        _rejects(S.gate_score, good, name, bad)


def test_select_and_plan_shapes():
    good = dict(logits=torch.zeros(B, HKV, NB), seqlens=_i32(B), mode=S.SELECT_TOPK, block_idx=_i32(B, HKV, 5),
                block_cnt=_i32(B, HKV))
    _accepts(S.select_blocks, **good)
    _accepts(S.select_blocks, **{**good, "block_idx": _i32(B, HKV, 1)})   # capacity is the C side's check
    for name, bad in (("block_idx", _i32(B, 5)), ("block_idx", _i32(B, HKV + 1, 5)), ("block_cnt", _i32(B)),
                      ("logits", torch.zeros(B, HKV, 2 * NB))):
        _rejects(S.select_blocks, good, name, bad)
    plan = dict(seqlens=_i32(B), kcomp=torch.zeros(B, HKV, NB, DG), q_nope=torch.zeros(B, HQ, D),
                w_q=torch.zeros(HKV, DG, (HQ // HKV) * D), mode=S.SELECT_TOPK, block_idx=_i32(B, HKV, 5),
                block_cnt=_i32(B, HKV), k_nope=_cache(), valid_blocks=_i32(B, HKV),
                w_k=torch.zeros(HKV, DG, 3 * D), logits=torch.zeros(B, HKV, NB))
    _accepts(S.decode_plan, **plan)
    for name, bad in (("w_k", torch.zeros(HKV, D, 3 * D)), ("logits", torch.zeros(B, NB)),
                      ("k_nope", _cache(torch.zeros(B, HKV, NB * BLK, 64)))):
        _rejects(S.decode_plan, plan, name, bad)


@pytest.mark.parametrize("fn", ["sparse_decode", "sparse_decode_noalloc"])
def test_sparse_decode_shapes(fn):
    f = getattr(S, fn)
    good = dict(q=torch.zeros(B, HQ, D), k=_cache(), v=_cache(), block_idx=_i32(B, HKV, 4), block_cnt=_i32(B, HKV),
                seqlens=_i32(B), out=torch.zeros(B, HQ, D), lse=torch.zeros(B, HQ))
    if fn == "sparse_decode":
        good["workspace"] = None
    _accepts(f, **good)
    for name, bad in (("q", torch.zeros(B, HQ, 64)), ("out", torch.zeros(B, HKV, D)), ("lse", torch.zeros(B, HQ, 1)),
                      ("v", _cache(torch.zeros(B, HKV, NB * BLK, 64))), ("block_cnt", _i32(B, HKV + 1)),
                      ("err", _i32(0))):
        _rejects(f, good, name, bad)


def test_gate_truth_shapes():
    good = dict(q=torch.zeros(B, HQ, D), k=_cache(), seqlens=_i32(B), scores=torch.zeros(B, HKV, NB),
                workspace=torch.zeros(16), log_scores=torch.zeros(B, HKV, NB))
    _accepts(S.gate_truth, **good)
    for name, bad in (("scores", torch.zeros(B, HQ, NB)), ("log_scores", torch.zeros(B, HKV, NB + 1)),
                      ("q", torch.zeros(B, HKV, D))):
        _rejects(S.gate_truth, good, name, bad)


def test_prefill_gt_shapes():
    T = 300
    good = dict(q=torch.zeros(B, HQ, T, D), k=_cache(), v=_cache(), seqlens=_i32(B), out=torch.zeros(B, HQ, T, D),
                gt=torch.zeros(B, HKV, T, NB), workspace=torch.zeros(16), lse=torch.zeros(B, HQ, T))
    _accepts(S.prefill_gt, **good)
    for name, bad in (("gt", torch.zeros(B, HKV, T, 8)), ("out", torch.zeros(B, HQ, T - 1, D)),
                      ("lse", torch.zeros(B, HQ, T + 1)), ("q", torch.zeros(B, 4, T, D)),
                      ("k", _cache(torch.zeros(B, 1, NB * BLK, D)))):
        _rejects(S.prefill_gt, good, name, bad)


def test_tensors_must_be_on_the_current_device(monkeypatch):
    """The C calls launch on the current device with bare pointers: a tensor on another GPU is
    refused before any call (checked here with a stand-in device index, no GPU needed)."""

    class OnDevice1:
        def get_device(self):
            return 1

    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    with pytest.raises(ValueError, match="cuda:1 but the current device is cuda:0"):
        S.seer._need_current_device(OnDevice1(), "q")

    class OnDevice0:
        def get_device(self):
            return 0

    S.seer._need_current_device(OnDevice0(), "q")
