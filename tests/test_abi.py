"""The C ABI library on the CPU: it loads, exports every symbol include/seer.h declares, its
struct layouts match the Python binding, and host-side validation rejects bad calls
before touching a GPU (no compute calls here)."""

import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "seer.h")


def _header_functions():
    src = open(HEADER).read()
    return re.findall(r"^(?:seer_status|size_t|int32_t|int64_t|const char\*)\s+(seer_\w+)\s*\(", src, re.M)


def _header_defines():
    src = open(HEADER).read()
    return {k: int(v) for k, v in re.findall(r"#define (SEER_\w+) (\d+)", src)}


@pytest.fixture(scope="module")
def S():
    from block_sparse_attention_attngate_b200 import build
    build.build()
    import block_sparse_attention_attngate_b200 as S
    return S


@pytest.fixture(scope="module")
def lib(S):
    from block_sparse_attention_attngate_b200 import seer
    return seer._lib


def test_every_declared_symbol_is_exported(lib, S):
    names = _header_functions()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), f"{n} declared in seer.h but not exported"
    assert set(names) == set(S.EXPORTED)
    out = subprocess.run(["nm", "-D", "--defined-only", S.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (seer_\w+)", out))
    assert exported == set(names), f"exported {exported ^ set(names)} differ from the header"


def test_struct_layout_matches_c(S):
    c = r"""
#include <stddef.h>
#include <stdio.h>
#include "seer.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu %zu %zu\n", sizeof(seer_dims_t), offsetof(seer_dims_t, rope_base),
         offsetof(seer_dims_t, softmax_scale), sizeof(seer_kv_t), offsetof(seer_kv_t, data),
         offsetof(seer_kv_t, block_table), offsetof(seer_kv_t, max_pages_per_seq));
  return 0;
}
"""
    with tempfile.TemporaryDirectory() as d:
        src, exe = os.path.join(d, "l.c"), os.path.join(d, "l")
        open(src, "w").write(c)
        subprocess.run(["gcc", "-std=c99", "-I", os.path.dirname(HEADER), src, "-o", exe], check=True)
        vals = [int(x) for x in subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split()]
    D, K = S.Dims, S.KVDesc
    assert vals == [ctypes.sizeof(D), D.rope_base.offset, D.softmax_scale.offset, ctypes.sizeof(K), K.data.offset,
                    K.block_table.offset, K.max_pages_per_seq.offset]


def test_header_constants_match_binding(S):
    d = _header_defines()
    assert d["SEER_SELECT_TOPK"] == S.SELECT_TOPK and d["SEER_SELECT_THRESHOLD"] == S.SELECT_THRESHOLD
    assert d["SEER_SELECT_TOPP"] == S.SELECT_TOPP
    assert d["SEER_DEVERR_BLOCK_INDEX"] == S.DEVERR_BLOCK_INDEX and d["SEER_DEVERR_TIMEOUT"] == S.DEVERR_TIMEOUT
    assert d["SEER_DEVERR_PAGE_INDEX"] == S.DEVERR_PAGE_INDEX and d["SEER_DEVERR_COUNT"] == S.DEVERR_COUNT
    assert d["SEER_WAIT_LIMIT_MIN"] == S.WAIT_LIMIT_MIN and d["SEER_WAIT_LIMIT_MAX"] == S.WAIT_LIMIT_MAX
    assert d["SEER_DEBUG_STARVE_COPIES"] == S.DEBUG_STARVE_COPIES


def _dims(S, **kw):
    base = dict(batch=8, num_q_heads=32, num_kv_heads=8, head_dim=128, gate_dim=128, block_size=64, max_blocks=512)
    base.update(kw)
    return S.Shape(**base).c()


P = ctypes.c_void_p(4096)   # aligned dummy addresses: never dereferenced on the host


def _select(lib, d, mode=0, budget=4096, tau=0.0, cap=65, logits=P):
    return lib.seer_select_blocks(ctypes.byref(d), logits, P, mode, budget, tau, P, P, cap, None)


@pytest.mark.parametrize("kw,status,word", [
    (dict(head_dim=96), 2, "head_dim"),
    (dict(gate_dim=32), 2, "gate_dim"),
    (dict(block_size=32), 2, "block_size"),
    (dict(num_q_heads=72, num_kv_heads=8), 2, "group size"),
    (dict(num_q_heads=30, num_kv_heads=8), 1, "multiple"),
    (dict(max_blocks=9000), 2, "max_blocks"),
    (dict(batch=0), 1, "batch"),
])
def test_dims_validation(lib, S, kw, status, word):
    d = _dims(S, **kw)
    assert _select(lib, d) == status
    assert word in lib.seer_last_error().decode()


def test_select_validation(lib, S):
    d = _dims(S)
    assert _select(lib, d, cap=64) == 3                       # top-k needs k + 1 = 65
    assert b"capacity" in lib.seer_last_error()
    assert _select(lib, d, mode=1, cap=511) == 3              # threshold needs max_blocks
    assert _select(lib, d, mode=2, cap=100) == 3
    assert _select(lib, d, mode=7) == 1
    assert _select(lib, d, budget=-1) == 1
    assert _select(lib, d, mode=1, cap=512, tau=float("nan")) == 1
    assert _select(lib, d, logits=None) == 1


def _kv(S, **kw):
    base = dict(layout=0, data=4096, stride_b=8 * 32768 * 128, stride_h=32768 * 128, stride_t=128, num_tokens=32768,
                num_pages=0, block_table=None, max_pages_per_seq=0)
    base.update(kw)
    return S.KVDesc(**base)


def _decode(lib, S, d, k, v, ns=2, ws=P, ws_bytes=1 << 30, q=P):
    return lib.seer_sparse_decode(ctypes.byref(d), q, ctypes.byref(k), ctypes.byref(v), P, P, P, 65, ns, ws,
                                  ws_bytes, P, None, None, None)


def test_decode_validation(lib, S):
    d = _dims(S)
    good = _kv(S)
    assert _decode(lib, S, d, _kv(S, data=4104), good) == 1
    assert b"aligned" in lib.seer_last_error()
    assert _decode(lib, S, d, _kv(S, stride_t=100), good) == 1
    assert _decode(lib, S, d, _kv(S, stride_t=132), good) == 1     # not a 16-byte multiple
    assert _decode(lib, S, d, _kv(S, layout=1), good) == 1         # paged without a block table
    assert _decode(lib, S, d, _kv(S, layout=3), good) == 1
    assert _decode(lib, S, d, good, good, q=ctypes.c_void_p(4098)) == 1
    assert _decode(lib, S, d, good, good, ns=-2) == 1
    assert b"num_split" in lib.seer_last_error()
    # a well-formed call reaches the CUDA runtime; without a GPU it reports a CUDA error, not a crash
    st = _decode(lib, S, d, good, good)
    assert st in (0, 4)


def test_workspace_formula(lib, S):
    d = _dims(S)
    for ns in (2, 3, 7):
        n = lib.seer_sparse_decode_workspace_bytes(ctypes.byref(d), 65, ns)
        up = lambda x: (x + 255) // 256 * 256
        assert n == up(8 * 8 * 4) + up(8 * 32 * ns * 4) + 8 * 32 * ns * 128 * 4
    assert lib.seer_sparse_decode_workspace_bytes(ctypes.byref(d), 65, 1) == 0
    assert lib.seer_sparse_decode_workspace_bytes(ctypes.byref(d), 65, -2) == 0
    bad = _dims(S, head_dim=80)
    assert lib.seer_sparse_decode_workspace_bytes(ctypes.byref(bad), 65, 2) == 0


def test_kcomp_and_gate_validation(lib, S):
    d = _dims(S)
    k = _kv(S)
    assert lib.seer_kcomp_update(ctypes.byref(d), ctypes.byref(k), None, P, P, P, None) == 1
    assert lib.seer_kcomp_update(ctypes.byref(d), ctypes.byref(k), P, P, ctypes.c_void_p(4100), P, None) == 1
    assert lib.seer_gate_score(ctypes.byref(d), P, P, P, P, None, None, None) == 1
    assert lib.seer_gate_score(ctypes.byref(d), P, P, P, P, P, ctypes.c_void_p(4097), None) == 1


def test_kcomp_append_validation(lib, S):
    d = _dims(S)
    k = _kv(S)
    n = 8 * 8 * 3 * 128 * 4                       # B * Hkv * 3 * d fp32
    assert lib.seer_kcomp_state_bytes(ctypes.byref(d)) == n
    assert lib.seer_kcomp_state_bytes(ctypes.byref(_dims(S, head_dim=80))) == 0
    assert lib.seer_kcomp_append(ctypes.byref(d), P, P, None, P, P, P, None, None) == 1
    assert lib.seer_kcomp_append(ctypes.byref(d), P, P, ctypes.c_void_p(4100), P, P, P, None, None) == 1
    assert lib.seer_kcomp_state_init(ctypes.byref(d), ctypes.byref(k), None, P, None, None) == 1
    assert lib.seer_kcomp_state_init(ctypes.byref(d), ctypes.byref(k), P, ctypes.c_void_p(4100), None, None) == 1


def test_prefill_gt_validation(lib, S):
    d = _dims(S)
    k = _kv(S)
    n = lib.seer_prefill_gt_workspace_bytes(ctypes.byref(d), 4096)
    assert n == 8 * 32 * (d.max_blocks + 1) * 4096 * 4   # block maxima, then one normaliser per row
    assert lib.seer_prefill_gt_workspace_bytes(ctypes.byref(d), 0) == 0
    assert lib.seer_prefill_gt(ctypes.byref(d), None, 64, ctypes.byref(k), ctypes.byref(k), P, P, None, P, P,
                               1 << 30, None, None) == 1
    big = d.max_blocks * d.block_size + 1                  # rows past max_blocks * b
    assert lib.seer_prefill_gt(ctypes.byref(d), P, big, ctypes.byref(k), ctypes.byref(k), P, P, None, P, P,
                               1 << 40, None, None) == 1
    assert lib.seer_prefill_gt(ctypes.byref(d), P, 64, ctypes.byref(k), ctypes.byref(k), P, P, None, P, P,
                               16, None, None) == 1          # workspace too small
    paged = _kv(S, layout=1, num_pages=64, block_table=4096, max_pages_per_seq=512, stride_b=8 * 64 * 128,
                stride_h=64 * 128)
    assert lib.seer_prefill_gt(ctypes.byref(d), P, 64, ctypes.byref(paged), ctypes.byref(paged), P, P, None, P, P,
                               1 << 30, None, None) == 2     # paged caches: unsupported


def test_gate_truth_validation(lib, S):
    d = _dims(S)
    k = _kv(S)
    up = lambda x: (x + 255) // 256 * 256
    bh, nchunk = 8 * 8, 512 // 16                   # 16 blocks per chunk
    # arrival counters | per-chunk (max, sum) of each of 8 group rows | block maxima of 8 group rows
    n = up(bh * 4) + up(bh * nchunk * 8 * 2 * 4) + bh * 512 * 8 * 4
    assert lib.seer_gate_truth_workspace_bytes(ctypes.byref(d)) == n
    assert lib.seer_gate_truth_workspace_bytes(ctypes.byref(_dims(S, head_dim=80))) == 0
    assert lib.seer_gate_truth(ctypes.byref(d), None, ctypes.byref(k), P, P, None, P, n, None, None) == 1
    assert lib.seer_gate_truth(ctypes.byref(d), P, ctypes.byref(k), P, ctypes.c_void_p(4100), None, P, n, None,
                               None) == 1             # scores not 16-byte aligned
    assert lib.seer_gate_truth(ctypes.byref(d), P, ctypes.byref(k), P, P, None, P, n - 1, None, None) == 1
    assert "workspace" in lib.seer_last_error().decode()


def test_every_entry_point_cites_its_passage():
    """Each entry point's comment block in the header cites the page section that defines the
    operation, or says that the pages have no counterpart (utilities excepted)."""
    import re
    text = open(HEADER).read()
    blocks = re.findall(r"/\*(.*?)\*/\s*((?:[\w\s\*]+?\s\**seer_\w+\s*\([^;]*\);\s*)+)", text, re.S)
    seen = set()
    for comment, decls in blocks:
        for name in re.findall(r"(seer_\w+)\s*\(", decls):
            seen.add(name)
            if name in ("seer_last_error", "seer_version"):
                continue
            assert re.search(r"\[CP |\[PN |\[SK |no counterpart", comment), f"{name}: no citation"
    assert {"seer_kcomp_update", "seer_gate_score", "seer_select_blocks", "seer_sparse_decode",
            "seer_decode_plan", "seer_gate_truth", "seer_prefill_gt", "seer_kcomp_append"} <= seen


def test_missing_library_fails_loudly(tmp_path):
    from block_sparse_attention_attngate_b200 import seer
    with pytest.raises(ImportError):
        seer.load_library(str(tmp_path / "libseer.so"))


def test_wait_limit_and_debug_flags(lib, S):
    """The decode's wait bound and debug switch: range checks, 0 = the default, and a rejected
    value leaves the setting as it was (no launch involved)."""
    assert lib.seer_get_wait_limit() == 2_000_000_000
    try:
        assert lib.seer_set_wait_limit(5000) == 0 and lib.seer_get_wait_limit() == 5000
        assert lib.seer_set_wait_limit(999) == 1 and lib.seer_get_wait_limit() == 5000
        assert lib.seer_set_wait_limit(100_000_000_001) == 1 and lib.seer_get_wait_limit() == 5000
        assert lib.seer_set_wait_limit(-5) == 1
        assert lib.seer_set_wait_limit(0) == 0 and lib.seer_get_wait_limit() == 2_000_000_000
        assert lib.seer_set_debug_flags(2) == 1 and lib.seer_set_debug_flags(-1) == 1
        assert lib.seer_set_debug_flags(1) == 0
    finally:
        lib.seer_set_debug_flags(0)
        lib.seer_set_wait_limit(0)
