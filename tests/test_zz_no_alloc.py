"""seer_sparse_decode_noalloc against seer_sparse_decode and the oracle, through the C ABI.

The no-allocation entry point exists for callers that cannot call cudaMalloc
or hand over a workspace -- an engine whose memory is fully reserved for its
KV pool before serving starts, a plugin whose host application owns every
device allocation, a hot loop that cannot take cudaMalloc's implicit device
synchronisation.  It uses the library's fixed 8 MiB scratch array in place of
the caller's workspace.  This file is named to be collected last, and builds
its own inputs so it also passes when run alone in a fresh process.
"""

import ctypes

import numpy as np
import pytest
import torch

from seer_harness import (OUT_MAX_ABS, OUT_REL_L2, OracleBH, bf16_bits, check_attention, check_lse, f64, gpu_list,
                          to_dev_bf16)
from synthetic import config, make_block_lists, make_inputs

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 8 << 20


def _close(a, b, what):
    a, b = f64(bf16_bits(a)), f64(bf16_bits(b))
    assert np.all(np.isfinite(a)), what
    max_abs = float(np.abs(a - b).max())
    rel = float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))
    assert max_abs <= OUT_MAX_ABS and rel <= OUT_REL_L2, f"{what}: max-abs {max_abs:.2e} rel {rel:.2e}"


def _noalloc(dims, q, kk, vv, idx, cnt, seq, cap, ns, out, lse, err):
    from block_sparse_attention_attngate_b200 import seer
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return seer._lib.seer_sparse_decode_noalloc(
        ctypes.byref(dims), ctypes.c_void_p(q.data_ptr()), ctypes.byref(kk.desc), ctypes.byref(vv.desc),
        ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(cnt.data_ptr()), ctypes.c_void_p(seq.data_ptr()),
        cap, ns, ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), ctypes.c_void_p(err.data_ptr()),
        stream)


def _problem(B, g, Hkv, lengths, cap, seed, list_seed, density):
    import block_sparse_attention_attngate_b200 as S
    blk, d = 64, 128
    cfg = config(1, B=B, Hq=g * Hkv, Hkv=Hkv, head_dim=d, gate_dim=128, block=blk, seed=seed)
    inp = make_inputs(cfg, lengths=lengths, tail="nan")
    sh = S.Shape(cfg.B, cfg.Hq, Hkv, d, 128, blk, inp.max_blocks)
    k, v, q = to_dev_bf16(inp.k), to_dev_bf16(inp.v), to_dev_bf16(inp.q)
    idx_h, cnt_h = make_block_lists(list_seed, lengths, Hkv, blk, cap, density=density)
    return dict(cfg=cfg, inp=inp, sh=sh, q=q, kk=S.KVCache.contiguous(k), vv=S.KVCache.contiguous(v),
                idx_h=idx_h, cnt_h=cnt_h, idx=torch.from_numpy(idx_h).cuda(), cnt=torch.from_numpy(cnt_h).cuda(),
                seq=torch.from_numpy(inp.seqlens).cuda(), lengths=lengths, cap=cap)


def _check_oracle(P, out, lse, what):
    cfg, g = P["cfg"], P["cfg"].g
    o, lh = f64(bf16_bits(out)), lse.cpu().numpy()
    for b in range(cfg.B):
        for h in range(cfg.Hkv):
            ro, rl = OracleBH(P["inp"], b, h).attention(P["lengths"][b], P["inp"].q,
                                                        gpu_list(P["idx_h"][b, h], P["cnt_h"][b, h]))
            check_attention(o[b, h * g:(h + 1) * g], ro, f"{what} b{b} h{h}")
            check_lse(lh[b, h * g:(h + 1) * g], rl, f"{what} b{b} h{h}")


@pytest.mark.parametrize("ns", [3, 0, -1])
def test_noalloc_matches_workspace_entry_point_twice(ns):
    """Two calls in a row (the second finds the scratch as the first left it), each against the
    workspace entry point and the oracle, under the pages' grid (3 splits), the balanced schedule
    (0, the binding's default, whose scratch size depends on the SM count) and the capacity one."""
    import block_sparse_attention_attngate_b200 as S
    from block_sparse_attention_attngate_b200 import seer

    P = _problem(3, 4, 4, [40 * 64 + 11, 33 * 64, 17 * 64 + 1], 24, 2718, 99, 0.5)
    cfg, d = P["cfg"], 128
    ref = torch.empty(cfg.B, cfg.Hq, d, dtype=torch.bfloat16, device="cuda")
    ref_lse = torch.empty(cfg.B, cfg.Hq, dtype=torch.float32, device="cuda")
    S.sparse_decode(P["sh"], P["q"], P["kk"], P["vv"], P["idx"], P["cnt"], P["seq"], ref,
                    S.alloc_workspace(P["sh"], P["cap"], ns), num_split=ns, lse=ref_lse)
    dims = P["sh"].c()
    for call in range(2):
        out = torch.full((cfg.B, cfg.Hq, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(cfg.B, cfg.Hq, dtype=torch.float32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        st = _noalloc(dims, P["q"], P["kk"], P["vv"], P["idx"], P["cnt"], P["seq"], P["cap"], ns, out, lse, err)
        assert st == 0, seer._lib.seer_last_error().decode()
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        _close(out, ref, f"call {call}")
        check_lse(lse.cpu().numpy(), ref_lse.cpu().numpy(), f"call {call}")
        _check_oracle(P, out, lse, f"ns={ns} call {call}")


def test_noalloc_at_the_scratch_limit():
    """The largest split count whose partials still fit the 8 MiB array runs (against the oracle);
    one split more is refused with SEER_ERR_CAPACITY."""
    import block_sparse_attention_attngate_b200 as S
    from block_sparse_attention_attngate_b200 import seer

    B, g, Hkv = 2, 4, 4
    probe = S.Shape(B, g * Hkv, Hkv, 128, 128, 64, 1024).c()   # the grid schedule's size needs no max_blocks
    need = [seer._lib.seer_sparse_decode_workspace_bytes(ctypes.byref(probe), 10**6, ns) for ns in range(1, 2001)]
    ns_max = max(ns for ns, n in zip(range(1, 2001), need) if n <= SCRATCH_BYTES)
    assert need[ns_max - 1] <= SCRATCH_BYTES < need[ns_max]
    assert need[ns_max - 1] > SCRATCH_BYTES - 64 * 1024, "the chosen split count sits right at the limit"
    # lists of ns_max blocks, one per split (a split of an empty range contributes nothing)
    L = ns_max * 64 + 5
    P = _problem(B, g, Hkv, [L, L - 64], ns_max, 3141, 7, 1.0)
    cfg, d = P["cfg"], 128
    dims = P["sh"].c()
    assert seer._lib.seer_sparse_decode_workspace_bytes(ctypes.byref(dims), ns_max, ns_max) == need[ns_max - 1]
    out = torch.empty(cfg.B, cfg.Hq, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(cfg.B, cfg.Hq, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = _noalloc(dims, P["q"], P["kk"], P["vv"], P["idx"], P["cnt"], P["seq"], ns_max, ns_max, out, lse, err)
    assert st == 0, seer._lib.seer_last_error().decode()
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    _check_oracle(P, out, lse, f"ns={ns_max}")
    cap1 = ns_max + 1
    idx1 = torch.full((cfg.B, cfg.Hkv, cap1), -1, dtype=torch.int32, device="cuda")
    st = _noalloc(dims, P["q"], P["kk"], P["vv"], idx1, P["cnt"], P["seq"], cap1, cap1, out, lse, err)
    assert st == 3, "one split past the limit is refused"


def test_noalloc_rejects_sizes_beyond_the_scratch():
    import block_sparse_attention_attngate_b200 as S
    from block_sparse_attention_attngate_b200 import seer

    sh = S.Shape(64, 64, 8, 128, 128, 64, 512)
    dims = sh.c()
    need = seer._lib.seer_sparse_decode_workspace_bytes(ctypes.byref(dims), 256, 16)
    assert need > SCRATCH_BYTES
    kv = S.KVDesc(0, 4096, 8 * 32768 * 128, 32768 * 128, 128, 32768, 0, None, 0)
    p = ctypes.c_void_p(4096)   # never dereferenced: the size check comes first
    st = seer._lib.seer_sparse_decode_noalloc(ctypes.byref(dims), p, ctypes.byref(kv), ctypes.byref(kv), p, p, p,
                                              256, 16, p, None, None, None)
    assert st == 3
    msg = seer._lib.seer_last_error().decode()
    assert "scratch" in msg and str(SCRATCH_BYTES) in msg
