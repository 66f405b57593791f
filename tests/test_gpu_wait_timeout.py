"""The timeout path of the sparse decode's bounded waits, made to run out without a fault.

With SEER_DEBUG_STARVE_COPIES the producer warp issues no copy and arms no barrier, so the
first wait of every CTA can never be satisfied; with the bound lowered to 2e6 SM cycles
(about a millisecond) each wait gives up, the kernel ORs SEER_DEVERR_TIMEOUT into the error
word and returns.  The test checks that bit, that the launch ended well inside the default
bound, and that the context and the same workspace still give the oracle's results on the next
call (the starved launch leaves the split counters zero) -- under the pages' grid (3 splits),
the balanced schedule (0) and the capacity schedule (-1), and through the no-allocation entry
point."""

import time

import numpy as np
import pytest
import torch

from seer_harness import OracleBH, bf16_bits, check_attention, check_lse, f64, gpu_list, to_dev_bf16
from synthetic import config, make_block_lists, make_inputs

pytestmark = pytest.mark.gpu

LIMIT = 2_000_000


def _problem():
    import block_sparse_attention_attngate_b200 as S
    lengths, cap, blk, d, g, Hkv = [40 * 64 + 11, 33 * 64, 17 * 64 + 1], 24, 64, 128, 4, 4
    cfg = config(1, B=len(lengths), Hq=g * Hkv, Hkv=Hkv, head_dim=d, gate_dim=128, block=blk, seed=909)
    inp = make_inputs(cfg, lengths=lengths, tail="nan")
    sh = S.Shape(cfg.B, cfg.Hq, Hkv, d, 128, blk, inp.max_blocks)
    idx_h, cnt_h = make_block_lists(31, lengths, Hkv, blk, cap, density=0.5)
    return dict(S=S, cfg=cfg, inp=inp, sh=sh, q=to_dev_bf16(inp.q), kk=S.KVCache.contiguous(to_dev_bf16(inp.k)),
                vv=S.KVCache.contiguous(to_dev_bf16(inp.v)), idx_h=idx_h, cnt_h=cnt_h,
                idx=torch.from_numpy(idx_h).cuda(), cnt=torch.from_numpy(cnt_h).cuda(),
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


def _starved(S, call):
    """Run call(err) once as it is (module load, descriptor caches), then with every copy withheld
    and the short bound; return the second call's error word."""
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    call(err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    S.set_wait_limit(LIMIT)
    S.set_debug_flags(S.DEBUG_STARVE_COPIES)
    try:
        t0 = time.perf_counter()
        call(err)
        torch.cuda.synchronize()
        dt = time.perf_counter() - t0
    finally:
        S.set_debug_flags(0)
        S.set_wait_limit(0)
    assert dt < 0.5, f"the starved launch took {dt:.3f} s: the short bound was not applied"
    return int(err.item())


@pytest.mark.parametrize("ns", [3, 0, -1])
def test_starved_decode_reports_timeout_and_recovers(ns):
    P = _problem()
    S, cfg = P["S"], P["cfg"]
    ws = S.alloc_workspace(P["sh"], P["cap"], ns)
    out = torch.empty(cfg.B, cfg.Hq, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(cfg.B, cfg.Hq, dtype=torch.float32, device="cuda")

    def run(err):
        S.sparse_decode(P["sh"], P["q"], P["kk"], P["vv"], P["idx"], P["cnt"], P["seq"], out, ws, num_split=ns,
                        lse=lse, err=err)

    e = _starved(S, run)
    assert e & S.DEVERR_TIMEOUT, f"error word {e:#x}"
    assert S.get_wait_limit() == 2_000_000_000
    out.fill_(float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    run(err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    _check_oracle(P, out, lse, f"ns={ns} after the starved call")


def test_starved_noalloc_reports_timeout_and_recovers():
    P = _problem()
    S, cfg = P["S"], P["cfg"]
    out = torch.empty(cfg.B, cfg.Hq, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(cfg.B, cfg.Hq, dtype=torch.float32, device="cuda")

    def run(err):
        S.sparse_decode_noalloc(P["sh"], P["q"], P["kk"], P["vv"], P["idx"], P["cnt"], P["seq"], out, num_split=-1,
                                lse=lse, err=err)

    assert _starved(S, run) & S.DEVERR_TIMEOUT
    out.fill_(float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    run(err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    _check_oracle(P, out, lse, "noalloc after the starved call")
