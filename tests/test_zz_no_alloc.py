"""seer_sparse_decode_noalloc against seer_sparse_decode, through the C ABI.

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

from seer_harness import OUT_MAX_ABS, OUT_REL_L2, bf16_bits, check_lse, f64, to_dev_bf16
from synthetic import config, make_block_lists, make_inputs

pytestmark = pytest.mark.gpu


def _close(a, b, what):
    a, b = f64(bf16_bits(a)), f64(bf16_bits(b))
    assert np.all(np.isfinite(a)), what
    max_abs = float(np.abs(a - b).max())
    rel = float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))
    assert max_abs <= OUT_MAX_ABS and rel <= OUT_REL_L2, f"{what}: max-abs {max_abs:.2e} rel {rel:.2e}"


@pytest.mark.parametrize("ns", [3, -1])
def test_noalloc_matches_workspace_entry_point_twice(ns):
    import block_sparse_attention_attngate_b200 as S
    from block_sparse_attention_attngate_b200 import seer

    blk, d, g, Hkv = 64, 128, 4, 4
    cfg = config(1, B=3, Hq=g * Hkv, Hkv=Hkv, head_dim=d, gate_dim=128, block=blk, seed=2718)
    lengths = [40 * blk + 11, 33 * blk, 17 * blk + 1]
    inp = make_inputs(cfg, lengths=lengths)
    sh = S.Shape(cfg.B, cfg.Hq, Hkv, d, 128, blk, inp.max_blocks)
    k, v, q = to_dev_bf16(inp.k), to_dev_bf16(inp.v), to_dev_bf16(inp.q)
    kk, vv = S.KVCache.contiguous(k), S.KVCache.contiguous(v)
    cap = 24
    idx_h, cnt_h = make_block_lists(99, lengths, Hkv, blk, cap, density=0.5)
    idx, cnt = torch.from_numpy(idx_h).cuda(), torch.from_numpy(cnt_h).cuda()
    seq = torch.from_numpy(inp.seqlens).cuda()
    ref = torch.empty(cfg.B, cfg.Hq, d, dtype=torch.bfloat16, device="cuda")
    ref_lse = torch.empty(cfg.B, cfg.Hq, dtype=torch.float32, device="cuda")
    S.sparse_decode(sh, q, kk, vv, idx, cnt, seq, ref, S.alloc_workspace(sh, cap, ns), num_split=ns, lse=ref_lse)

    dims = sh.c()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):   # the second call finds the scratch as the first one left it
        out = torch.full((cfg.B, cfg.Hq, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(cfg.B, cfg.Hq, dtype=torch.float32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        st = seer._lib.seer_sparse_decode_noalloc(
            ctypes.byref(dims), ctypes.c_void_p(q.data_ptr()), ctypes.byref(kk.desc), ctypes.byref(vv.desc),
            ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(cnt.data_ptr()), ctypes.c_void_p(seq.data_ptr()),
            cap, ns, ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
            ctypes.c_void_p(err.data_ptr()), stream)
        assert st == 0, seer._lib.seer_last_error().decode()
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        _close(out, ref, f"call {call}")
        check_lse(lse.cpu().numpy(), ref_lse.cpu().numpy(), f"call {call}")


def test_noalloc_rejects_sizes_beyond_the_scratch():
    import block_sparse_attention_attngate_b200 as S
    from block_sparse_attention_attngate_b200 import seer

    sh = S.Shape(64, 64, 8, 128, 128, 64, 512)
    dims = sh.c()
    need = seer._lib.seer_sparse_decode_workspace_bytes(ctypes.byref(dims), 256, 16)
    assert need > 8 << 20
    kv = S.KVDesc(0, 4096, 8 * 32768 * 128, 32768 * 128, 128, 32768, 0, None, 0)
    p = ctypes.c_void_p(4096)   # never dereferenced: the size check comes first
    st = seer._lib.seer_sparse_decode_noalloc(ctypes.byref(dims), p, ctypes.byref(kv), ctypes.byref(kv), p, p, p,
                                              256, 16, p, None, None, None)
    assert st == 3
    msg = seer._lib.seer_last_error().decode()
    assert "scratch" in msg and str(8 << 20) in msg
