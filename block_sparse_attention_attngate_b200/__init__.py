"""SeerAttention-R gated block-sparse GQA decode for NVIDIA B200 (sm_100a).

The compute lives in libseer.so (C ABI: include/seer.h); the `seer` module is
its Python binding.  Any public name resolves through `seer`, which loads the
library and raises ImportError when it has not been built -- there is no
fallback path.  (The lazy lookup lets `python -m <package>.build` run before
the library exists.)
"""

_PUBLIC = (
    "DEBUG_STARVE_COPIES", "DEVERR_BLOCK_INDEX", "DEVERR_COUNT", "DEVERR_PAGE_INDEX", "DEVERR_TIMEOUT", "EXPORTED", "KV_CONTIGUOUS",
    "KV_PAGED", "LIB_PATH", "SELECT_THRESHOLD", "SELECT_TOPK", "SELECT_TOPP", "DecodeStep", "Dims", "KVCache",
    "KVDesc", "SeerError", "Shape", "alloc_step_workspace", "alloc_truth_workspace", "alloc_workspace", "decode_plan",
    "decode_step", "decode_step_supported", "decode_step_workspace_bytes", "gate_score",
    "gate_truth", "gate_truth_workspace_bytes", "kcomp_update", "kcomp_append", "kcomp_state_init",
    "kcomp_state_bytes", "alloc_kcomp_state", "prefill_gt", "prefill_gt_workspace_bytes", "select_blocks",
    "sparse_decode", "sparse_decode_auto_split", "sparse_decode_noalloc", "sparse_decode_workspace_bytes", "version",
    "set_wait_limit", "get_wait_limit", "set_debug_flags", "WAIT_LIMIT_MIN", "WAIT_LIMIT_MAX",
)

__all__ = list(_PUBLIC)


def __getattr__(name):
    if name in _PUBLIC:
        from . import seer
        return getattr(seer, name)
    raise AttributeError(name)
