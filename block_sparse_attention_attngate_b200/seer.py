"""Thin Python binding of libseer (include/seer.h).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels behind the C ABI.  Tensors are torch CUDA tensors; torch provides
device memory and the current stream, nothing else.  If libseer.so is missing
this module raises at import time -- there is no fallback.
"""

from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# SEER_LIBRARY selects another build of the library (e.g. a variant with different tile choices)
LIB_PATH = os.environ.get("SEER_LIBRARY") or os.path.join(_HERE, "libseer.so")

SEER_OK, SEER_ERR_INVALID_ARG, SEER_ERR_UNSUPPORTED, SEER_ERR_CAPACITY, SEER_ERR_CUDA = range(5)
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CAPACITY", 4: "CUDA"}
KV_CONTIGUOUS, KV_PAGED = 0, 1
SELECT_TOPK, SELECT_THRESHOLD, SELECT_TOPP = 0, 1, 2
DEVERR_BLOCK_INDEX, DEVERR_PAGE_INDEX, DEVERR_COUNT, DEVERR_TIMEOUT = 1, 2, 4, 8
WAIT_LIMIT_MIN, WAIT_LIMIT_MAX = 1000, 100_000_000_000
DEBUG_STARVE_COPIES = 1

EXPORTED = (
    "seer_kcomp_update", "seer_kcomp_state_bytes", "seer_kcomp_append", "seer_kcomp_state_init", "seer_gate_score",
    "seer_select_blocks", "seer_decode_plan", "seer_decode_step_workspace_bytes", "seer_decode_step_supported",
    "seer_decode_step", "seer_sparse_decode_auto_split",
    "seer_sparse_decode_workspace_bytes", "seer_sparse_decode", "seer_sparse_decode_noalloc",
    "seer_gate_truth_workspace_bytes", "seer_gate_truth", "seer_prefill_gt_workspace_bytes", "seer_prefill_gt",
    "seer_set_wait_limit", "seer_get_wait_limit", "seer_set_debug_flags", "seer_last_error", "seer_version",
)


class SeerError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"libseer {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("gate_dim", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("max_blocks", ctypes.c_int32), ("rope_base", ctypes.c_float), ("softmax_scale", ctypes.c_float)]


class KVDesc(ctypes.Structure):
    _fields_ = [("layout", ctypes.c_int32), ("data", ctypes.c_void_p), ("stride_b", ctypes.c_int64),
                ("stride_h", ctypes.c_int64), ("stride_t", ctypes.c_int64), ("num_tokens", ctypes.c_int64),
                ("num_pages", ctypes.c_int64), ("block_table", ctypes.c_void_p),
                ("max_pages_per_seq", ctypes.c_int32)]


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m block_sparse_attention_attngate_b200.build`")
    lib = ctypes.CDLL(path)
    P, I32, I64, F32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    DP, KP = ctypes.POINTER(Dims), ctypes.POINTER(KVDesc)
    sig = {
        "seer_kcomp_update": (I32, [DP, KP, P, P, P, P, P]),
        "seer_kcomp_state_bytes": (SZ, [DP]),
        "seer_kcomp_append": (I32, [DP, P, P, P, P, P, P, P, P]),
        "seer_kcomp_state_init": (I32, [DP, KP, P, P, P, P]),
        "seer_gate_score": (I32, [DP, P, P, P, P, P, P, P]),
        "seer_select_blocks": (I32, [DP, P, P, I32, I32, F32, P, P, I32, P]),
        "seer_decode_plan": (I32, [DP, KP, P, P, P, P, P, P, P, P, I32, I32, F32, P, P, I32, P]),
        "seer_decode_step_workspace_bytes": (SZ, [DP, I32]),
        "seer_decode_step_supported": (I32, [DP, I32, I32]),
        "seer_decode_step": (I32, [DP, KP, P, P, P, P, P, P, P, P, I32, I32, F32, P, P, I32, P, KP, KP, P, SZ, P, P, P,
                                   P]),
        "seer_sparse_decode_auto_split": (I32, [DP, I32]),
        "seer_sparse_decode_workspace_bytes": (SZ, [DP, I32, I32]),
        "seer_sparse_decode": (I32, [DP, P, KP, KP, P, P, P, I32, I32, P, SZ, P, P, P, P]),
        "seer_sparse_decode_noalloc": (I32, [DP, P, KP, KP, P, P, P, I32, I32, P, P, P, P]),
        "seer_gate_truth_workspace_bytes": (SZ, [DP]),
        "seer_gate_truth": (I32, [DP, P, KP, P, P, P, P, SZ, P, P]),
        "seer_prefill_gt_workspace_bytes": (SZ, [DP, I32]),
        "seer_prefill_gt": (I32, [DP, P, I32, KP, KP, P, P, P, P, P, SZ, P, P]),
        "seer_set_wait_limit": (I32, [I64]),
        "seer_get_wait_limit": (I64, []),
        "seer_set_debug_flags": (I32, [I32]),
        "seer_last_error": (ctypes.c_char_p, []),
        "seer_version": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = load_library()


def version() -> str:
    return _lib.seer_version().decode()


def _check(status: int):
    if status != SEER_OK:
        raise SeerError(status, _lib.seer_last_error().decode())


def set_wait_limit(cycles: int) -> None:
    """Bound (SM clock cycles) of the sparse decode's copy and hand-off waits, process-wide;
    0 restores the default (about one second)."""
    _check(_lib.seer_set_wait_limit(int(cycles)))


def get_wait_limit() -> int:
    return int(_lib.seer_get_wait_limit())


def set_debug_flags(flags: int) -> None:
    """Process-wide debug switches of the sparse decode (DEBUG_STARVE_COPIES: no copy is issued,
    so every CTA's first wait runs out and the launch reports DEVERR_TIMEOUT); 0 turns them off."""
    _check(_lib.seer_set_debug_flags(int(flags)))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need_shape(t, shape, name: str):
    """The kernels index these buffers by the problem shape: a smaller tensor would be written past."""
    if not isinstance(t, torch.Tensor) or tuple(t.shape) != tuple(int(x) for x in shape):
        got = tuple(t.shape) if isinstance(t, torch.Tensor) else type(t).__name__
        raise ValueError(f"{name} must have shape {tuple(int(x) for x in shape)}, got {got}")


def _need_lists(block_idx, block_cnt, B: int, H: int):
    """Block lists [B, Hkv, capacity] and counts [B, Hkv] (the capacity is the list's last extent)."""
    if not isinstance(block_idx, torch.Tensor) or block_idx.dim() != 3 or tuple(block_idx.shape[:2]) != (B, H):
        got = tuple(block_idx.shape) if isinstance(block_idx, torch.Tensor) else type(block_idx).__name__
        raise ValueError(f"block_idx must have shape ({B}, {H}, capacity), got {got}")
    _need_shape(block_cnt, (B, H), "block_cnt")


def _need_err(err):
    if err is not None:
        if not isinstance(err, torch.Tensor) or err.numel() < 1:
            raise ValueError("err must hold one int32")
        _need(err, torch.int32, "err")


def _need_current_device(t, name: str):
    """The C calls take bare pointers and launch on the current device: a tensor on another GPU
    would be read through the wrong device's address space (and the no-allocation call would
    pick the current device's scratch)."""
    cur = torch.cuda.current_device()
    if t.get_device() != cur:
        raise ValueError(f"{name} is on cuda:{t.get_device()} but the current device is cuda:{cur}; "
                         f"call under torch.cuda.device({t.get_device()})")


def _need(t: torch.Tensor, dtype: torch.dtype, name: str, contiguous: bool = True):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    _need_current_device(t, name)
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


@dataclass
class Shape:
    """Problem shape of one attention layer (mirrors seer_dims_t)."""
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    gate_dim: int
    block_size: int
    max_blocks: int
    rope_base: float = 1e6
    softmax_scale: float = 0.0

    def c(self) -> Dims:
        return Dims(self.batch, self.num_q_heads, self.num_kv_heads, self.head_dim, self.gate_dim,
                    self.block_size, self.max_blocks, self.rope_base, self.softmax_scale)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads


class KVCache:
    """A bf16 K or V cache as the library sees it (contiguous or paged)."""

    def __init__(self, desc: KVDesc, keep):
        self.desc = desc
        self._keep = keep

    @classmethod
    def contiguous(cls, t: torch.Tensor) -> "KVCache":
        """t: [B, Hkv, T, d] view (any strides with unit-stride head_dim)."""
        _need(t, torch.bfloat16, "kv cache", contiguous=False)
        if t.dim() != 4 or t.stride(3) != 1:
            raise ValueError("contiguous KV cache must be a 4-D [B, Hkv, T, d] view with unit-stride d")
        d = KVDesc(KV_CONTIGUOUS, t.data_ptr(), t.stride(0), t.stride(1), t.stride(2), t.shape[2], 0, None, 0)
        return cls(d, (t,))

    @classmethod
    def paged(cls, pool: torch.Tensor, block_table: torch.Tensor) -> "KVCache":
        """pool: [P, Hkv, block, d]; block_table: int32 [B, max_pages_per_seq]."""
        _need(pool, torch.bfloat16, "page pool", contiguous=False)
        _need(block_table, torch.int32, "block_table")
        if pool.dim() != 4 or pool.stride(3) != 1:
            raise ValueError("page pool must be a 4-D [P, Hkv, block, d] view with unit-stride d")
        d = KVDesc(KV_PAGED, pool.data_ptr(), pool.stride(0), pool.stride(1), pool.stride(2), 0, pool.shape[0],
                   block_table.data_ptr(), block_table.shape[1])
        return cls(d, (pool, block_table))

    def check(self, shape: "Shape", name: str):
        """The cache holds the shape's sequences, KV heads and head_dim (the library reads it by
        (b, kv-head, token) from the descriptor's strides, so a smaller view would be read past)."""
        if self.desc.layout == KV_CONTIGUOUS:
            t = self._keep[0]
            if t.shape[0] < shape.batch or t.shape[1] != shape.num_kv_heads or t.shape[3] != shape.head_dim:
                raise ValueError(f"{name}: a [B >= {shape.batch}, {shape.num_kv_heads}, T, {shape.head_dim}] view "
                                 f"is needed, got {tuple(t.shape)}")
        else:
            pool, table = self._keep
            if (pool.shape[1] != shape.num_kv_heads or pool.shape[2] != shape.block_size
                    or pool.shape[3] != shape.head_dim or table.dim() != 2 or table.shape[0] < shape.batch):
                raise ValueError(f"{name}: a [P, {shape.num_kv_heads}, {shape.block_size}, {shape.head_dim}] pool "
                                 f"and a [B >= {shape.batch}, pages] table are needed, got {tuple(pool.shape)} and "
                                 f"{tuple(table.shape)}")


def kcomp_update(shape: Shape, k_nope: KVCache, seqlens: torch.Tensor, valid_blocks: torch.Tensor,
                 w_k: torch.Tensor, kcomp: torch.Tensor, stream=None):
    B, H, d, dg = shape.batch, shape.num_kv_heads, shape.head_dim, shape.gate_dim
    k_nope.check(shape, "k_nope")
    _need_shape(seqlens, (B,), "seqlens")
    _need_shape(valid_blocks, (B, H), "valid_blocks")
    _need_shape(w_k, (H, dg, 3 * d), "w_k")
    _need_shape(kcomp, (B, H, shape.max_blocks, dg), "kcomp")
    _need(seqlens, torch.int32, "seqlens")
    _need(valid_blocks, torch.int32, "valid_blocks")
    _need(w_k, torch.bfloat16, "w_k")
    _need(kcomp, torch.bfloat16, "kcomp")
    dims = shape.c()
    _check(_lib.seer_kcomp_update(ctypes.byref(dims), ctypes.byref(k_nope.desc), _ptr(seqlens),
                                  _ptr(valid_blocks), _ptr(w_k), _ptr(kcomp), _stream(stream)))


def kcomp_state_bytes(shape: Shape) -> int:
    dims = shape.c()
    return int(_lib.seer_kcomp_state_bytes(ctypes.byref(dims)))


def alloc_kcomp_state(shape: Shape, device=None) -> torch.Tensor:
    """Running block statistics for kcomp_append: fp32 [B, Hkv, 3, d] (max, min, sum)."""
    return torch.zeros((shape.batch, shape.num_kv_heads, 3, shape.head_dim), dtype=torch.float32, device=device or "cuda")


def kcomp_append(shape: Shape, k_new: torch.Tensor, seqlens: torch.Tensor, state: torch.Tensor,
                 valid_blocks: torch.Tensor, w_k: torch.Tensor, kcomp: torch.Tensor,
                 err: Optional[torch.Tensor] = None, stream=None):
    """Fold each sequence's appended pre-RoPE key [B, Hkv, d] into the running block statistics;
    a completed block writes its K Compression Cache entry (see seer_kcomp_append)."""
    B, H, d, dg = shape.batch, shape.num_kv_heads, shape.head_dim, shape.gate_dim
    _need_shape(k_new, (B, H, d), "k_new")
    _need_shape(seqlens, (B,), "seqlens")
    _need_shape(state, (B, H, 3, d), "state")
    _need_shape(valid_blocks, (B, H), "valid_blocks")
    _need_shape(w_k, (H, dg, 3 * d), "w_k")
    _need_shape(kcomp, (B, H, shape.max_blocks, dg), "kcomp")
    _need_err(err)
    _need(k_new, torch.bfloat16, "k_new")
    _need(seqlens, torch.int32, "seqlens")
    _need(state, torch.float32, "state")
    _need(valid_blocks, torch.int32, "valid_blocks")
    _need(w_k, torch.bfloat16, "w_k")
    _need(kcomp, torch.bfloat16, "kcomp")
    dims = shape.c()
    _check(_lib.seer_kcomp_append(ctypes.byref(dims), _ptr(k_new), _ptr(seqlens), _ptr(state), _ptr(valid_blocks),
                                  _ptr(w_k), _ptr(kcomp), _ptr(err) if err is not None else None, _stream(stream)))


def kcomp_state_init(shape: Shape, k_nope: KVCache, seqlens: torch.Tensor, state: torch.Tensor,
                     err: Optional[torch.Tensor] = None, stream=None):
    """Prime the running block statistics from the key cache (see seer_kcomp_state_init)."""
    k_nope.check(shape, "k_nope")
    _need_err(err)
    _need_shape(seqlens, (shape.batch,), "seqlens")
    _need_shape(state, (shape.batch, shape.num_kv_heads, 3, shape.head_dim), "state")
    _need(seqlens, torch.int32, "seqlens")
    _need(state, torch.float32, "state")
    dims = shape.c()
    _check(_lib.seer_kcomp_state_init(ctypes.byref(dims), ctypes.byref(k_nope.desc), _ptr(seqlens), _ptr(state),
                                      _ptr(err) if err is not None else None, _stream(stream)))


def gate_score(shape: Shape, q_nope: torch.Tensor, w_q: torch.Tensor, kcomp: torch.Tensor, seqlens: torch.Tensor,
               logits: torch.Tensor, q_gate: Optional[torch.Tensor] = None, stream=None):
    B, Hq, H, d, dg = shape.batch, shape.num_q_heads, shape.num_kv_heads, shape.head_dim, shape.gate_dim
    _need_shape(q_nope, (B, Hq, d), "q_nope")
    _need_shape(w_q, (H, dg, shape.group * d), "w_q")
    _need_shape(kcomp, (B, H, shape.max_blocks, dg), "kcomp")
    _need_shape(seqlens, (B,), "seqlens")
    _need_shape(logits, (B, H, shape.max_blocks), "logits")
    if q_gate is not None:
        _need_shape(q_gate, (B, H, dg), "q_gate")
    _need(q_nope, torch.bfloat16, "q_nope")
    _need(w_q, torch.bfloat16, "w_q")
    _need(kcomp, torch.bfloat16, "kcomp")
    _need(seqlens, torch.int32, "seqlens")
    _need(logits, torch.float32, "logits")
    if q_gate is not None:
        _need(q_gate, torch.float32, "q_gate")
    dims = shape.c()
    _check(_lib.seer_gate_score(ctypes.byref(dims), _ptr(q_nope), _ptr(w_q), _ptr(kcomp), _ptr(seqlens),
                                _ptr(logits), _ptr(q_gate), _stream(stream)))


def select_blocks(shape: Shape, logits: torch.Tensor, seqlens: torch.Tensor, mode: int, block_idx: torch.Tensor,
                  block_cnt: torch.Tensor, token_budget: int = 0, tau: float = 0.0, stream=None):
    B, H = shape.batch, shape.num_kv_heads
    _need_shape(logits, (B, H, shape.max_blocks), "logits")
    _need_shape(seqlens, (B,), "seqlens")
    _need_lists(block_idx, block_cnt, B, H)
    _need(logits, torch.float32, "logits")
    _need(seqlens, torch.int32, "seqlens")
    _need(block_idx, torch.int32, "block_idx")
    _need(block_cnt, torch.int32, "block_cnt")
    dims = shape.c()
    _check(_lib.seer_select_blocks(ctypes.byref(dims), _ptr(logits), _ptr(seqlens), int(mode), int(token_budget),
                                   float(tau), _ptr(block_idx), _ptr(block_cnt), block_idx.shape[-1],
                                   _stream(stream)))


def decode_plan(shape: Shape, seqlens: torch.Tensor, kcomp: torch.Tensor, q_nope: torch.Tensor, w_q: torch.Tensor,
                mode: int, block_idx: torch.Tensor, block_cnt: torch.Tensor, token_budget: int = 0, tau: float = 0.0,
                k_nope: Optional[KVCache] = None, valid_blocks: Optional[torch.Tensor] = None,
                w_k: Optional[torch.Tensor] = None, logits: Optional[torch.Tensor] = None,
                q_gate: Optional[torch.Tensor] = None, stream=None):
    """kcomp_update (when valid_blocks is given) + gate_score + select_blocks in one launch."""
    B, Hq, H, d, dg = shape.batch, shape.num_q_heads, shape.num_kv_heads, shape.head_dim, shape.gate_dim
    _need_shape(seqlens, (B,), "seqlens")
    _need_shape(kcomp, (B, H, shape.max_blocks, dg), "kcomp")
    _need_shape(q_nope, (B, Hq, d), "q_nope")
    _need_shape(w_q, (H, dg, shape.group * d), "w_q")
    _need_lists(block_idx, block_cnt, B, H)
    if valid_blocks is not None:
        _need_shape(valid_blocks, (B, H), "valid_blocks")
        _need_shape(w_k, (H, dg, 3 * d), "w_k")
        if k_nope is not None:
            k_nope.check(shape, "k_nope")
    if logits is not None:
        _need_shape(logits, (B, H, shape.max_blocks), "logits")
    if q_gate is not None:
        _need_shape(q_gate, (B, H, dg), "q_gate")
    _need(seqlens, torch.int32, "seqlens")
    _need(kcomp, torch.bfloat16, "kcomp")
    _need(q_nope, torch.bfloat16, "q_nope")
    _need(w_q, torch.bfloat16, "w_q")
    _need(block_idx, torch.int32, "block_idx")
    _need(block_cnt, torch.int32, "block_cnt")
    if valid_blocks is not None:
        _need(valid_blocks, torch.int32, "valid_blocks")
        _need(w_k, torch.bfloat16, "w_k")
        if k_nope is None:
            raise ValueError("k_nope is required with valid_blocks")
    if logits is not None:
        _need(logits, torch.float32, "logits")
    if q_gate is not None:
        _need(q_gate, torch.float32, "q_gate")
    dims = shape.c()
    kv = ctypes.byref(k_nope.desc) if k_nope is not None else None
    _check(_lib.seer_decode_plan(ctypes.byref(dims), kv, _ptr(seqlens), _ptr(valid_blocks), _ptr(w_k), _ptr(kcomp),
                                 _ptr(q_nope), _ptr(w_q), _ptr(logits), _ptr(q_gate), int(mode), int(token_budget),
                                 float(tau), _ptr(block_idx), _ptr(block_cnt), block_idx.shape[-1], _stream(stream)))


def decode_step_workspace_bytes(shape: Shape, capacity: int) -> int:
    dims = shape.c()
    return int(_lib.seer_decode_step_workspace_bytes(ctypes.byref(dims), int(capacity)))


def decode_step_supported(shape: Shape, mode: int, capacity: int) -> bool:
    """Whether decode_step runs this shape and selection mode in one launch on the current device."""
    dims = shape.c()
    return bool(_lib.seer_decode_step_supported(ctypes.byref(dims), int(mode), int(capacity)))


def alloc_step_workspace(shape: Shape, capacity: int, device=None) -> torch.Tensor:
    """Zero-filled workspace for decode_step (its ready flags and arrival counters start at zero)."""
    return torch.zeros(max(decode_step_workspace_bytes(shape, capacity), 16), dtype=torch.uint8,
                       device=device or "cuda")


def decode_step(shape: Shape, seqlens: torch.Tensor, kcomp: torch.Tensor, q_nope: torch.Tensor, w_q: torch.Tensor,
                mode: int, block_idx: torch.Tensor, block_cnt: torch.Tensor, q: torch.Tensor, k: KVCache, v: KVCache,
                out: torch.Tensor, workspace: torch.Tensor, token_budget: int = 0, tau: float = 0.0,
                k_nope: Optional[KVCache] = None, valid_blocks: Optional[torch.Tensor] = None,
                w_k: Optional[torch.Tensor] = None, logits: Optional[torch.Tensor] = None,
                q_gate: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                err: Optional[torch.Tensor] = None, stream=None):
    """decode_plan followed by sparse_decode (capacity schedule) in one launch (see seer_decode_step)."""
    B, Hq, H, d, dg = shape.batch, shape.num_q_heads, shape.num_kv_heads, shape.head_dim, shape.gate_dim
    _need_shape(seqlens, (B,), "seqlens")
    _need_shape(kcomp, (B, H, shape.max_blocks, dg), "kcomp")
    _need_shape(q_nope, (B, Hq, d), "q_nope")
    _need_shape(w_q, (H, dg, shape.group * d), "w_q")
    _decode_shapes(shape, q, k, v, block_idx, block_cnt, seqlens, out, lse, err)
    if valid_blocks is not None:
        _need_shape(valid_blocks, (B, H), "valid_blocks")
        _need_shape(w_k, (H, dg, 3 * d), "w_k")
        if k_nope is None:
            raise ValueError("k_nope is required with valid_blocks")
        k_nope.check(shape, "k_nope")
    if logits is not None:
        _need_shape(logits, (B, H, shape.max_blocks), "logits")
    if q_gate is not None:
        _need_shape(q_gate, (B, H, dg), "q_gate")
    for t, dt, name in ((seqlens, torch.int32, "seqlens"), (kcomp, torch.bfloat16, "kcomp"),
                        (q_nope, torch.bfloat16, "q_nope"), (w_q, torch.bfloat16, "w_q"),
                        (block_idx, torch.int32, "block_idx"), (block_cnt, torch.int32, "block_cnt"),
                        (q, torch.bfloat16, "q"), (out, torch.bfloat16, "out"), (workspace, torch.uint8, "workspace")):
        _need(t, dt, name)
    for t, dt, name in ((valid_blocks, torch.int32, "valid_blocks"), (w_k, torch.bfloat16, "w_k"),
                        (logits, torch.float32, "logits"), (q_gate, torch.float32, "q_gate"),
                        (lse, torch.float32, "lse"), (err, torch.int32, "err")):
        if t is not None:
            _need(t, dt, name)
    dims = shape.c()
    kv = ctypes.byref(k_nope.desc) if k_nope is not None else None
    _check(_lib.seer_decode_step(ctypes.byref(dims), kv, _ptr(seqlens), _ptr(valid_blocks), _ptr(w_k), _ptr(kcomp),
                                 _ptr(q_nope), _ptr(w_q), _ptr(logits), _ptr(q_gate), int(mode), int(token_budget),
                                 float(tau), _ptr(block_idx), _ptr(block_cnt), block_idx.shape[-1], _ptr(q),
                                 ctypes.byref(k.desc), ctypes.byref(v.desc), _ptr(workspace), workspace.numel(),
                                 _ptr(out), _ptr(lse), _ptr(err), _stream(stream)))


def sparse_decode_auto_split(shape: Shape, capacity: int) -> int:
    dims = shape.c()
    return int(_lib.seer_sparse_decode_auto_split(ctypes.byref(dims), int(capacity)))


def sparse_decode_workspace_bytes(shape: Shape, capacity: int, num_split: int = 0) -> int:
    dims = shape.c()
    return int(_lib.seer_sparse_decode_workspace_bytes(ctypes.byref(dims), int(capacity), int(num_split)))


def alloc_workspace(shape: Shape, capacity: int, num_split: int = 0, device=None) -> torch.Tensor:
    """Zero-filled workspace (the arrival counters must start at zero)."""
    n = sparse_decode_workspace_bytes(shape, capacity, num_split)
    return torch.zeros(max(n, 16), dtype=torch.uint8, device=device or "cuda")


def _decode_shapes(shape: Shape, q, k: KVCache, v: KVCache, block_idx, block_cnt, seqlens, out, lse, err):
    B, Hq, H, d = shape.batch, shape.num_q_heads, shape.num_kv_heads, shape.head_dim
    _need_shape(q, (B, Hq, d), "q")
    k.check(shape, "k")
    v.check(shape, "v")
    _need_lists(block_idx, block_cnt, B, H)
    _need_shape(seqlens, (B,), "seqlens")
    _need_shape(out, (B, Hq, d), "out")
    if lse is not None:
        _need_shape(lse, (B, Hq), "lse")
    _need_err(err)


def sparse_decode(shape: Shape, q: torch.Tensor, k: KVCache, v: KVCache, block_idx: torch.Tensor,
                  block_cnt: torch.Tensor, seqlens: torch.Tensor, out: torch.Tensor, workspace: Optional[torch.Tensor],
                  num_split: int = 0, lse: Optional[torch.Tensor] = None, err: Optional[torch.Tensor] = None,
                  stream=None):
    _decode_shapes(shape, q, k, v, block_idx, block_cnt, seqlens, out, lse, err)
    _need(q, torch.bfloat16, "q")
    _need(block_idx, torch.int32, "block_idx")
    _need(block_cnt, torch.int32, "block_cnt")
    _need(seqlens, torch.int32, "seqlens")
    _need(out, torch.bfloat16, "out")
    if lse is not None:
        _need(lse, torch.float32, "lse")
    if err is not None:
        _need(err, torch.int32, "err")
    dims = shape.c()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.seer_sparse_decode(ctypes.byref(dims), _ptr(q), ctypes.byref(k.desc), ctypes.byref(v.desc),
                                   _ptr(block_idx), _ptr(block_cnt), _ptr(seqlens), block_idx.shape[-1],
                                   int(num_split), _ptr(workspace), ws_bytes, _ptr(out), _ptr(lse), _ptr(err),
                                   _stream(stream)))


def sparse_decode_noalloc(shape: Shape, q: torch.Tensor, k: KVCache, v: KVCache, block_idx: torch.Tensor,
                          block_cnt: torch.Tensor, seqlens: torch.Tensor, out: torch.Tensor, num_split: int = 0,
                          lse: Optional[torch.Tensor] = None, err: Optional[torch.Tensor] = None, stream=None):
    """sparse_decode without a workspace argument, for callers that cannot allocate device memory.

    The library's fixed 8 MiB scratch array takes the workspace's place: calls on one device
    must not overlap on the GPU, and the first call on a device must come before any capture.
    """
    _decode_shapes(shape, q, k, v, block_idx, block_cnt, seqlens, out, lse, err)
    _need(q, torch.bfloat16, "q")
    _need(block_idx, torch.int32, "block_idx")
    _need(block_cnt, torch.int32, "block_cnt")
    _need(seqlens, torch.int32, "seqlens")
    _need(out, torch.bfloat16, "out")
    if lse is not None:
        _need(lse, torch.float32, "lse")
    dims = shape.c()
    _check(_lib.seer_sparse_decode_noalloc(ctypes.byref(dims), _ptr(q), ctypes.byref(k.desc), ctypes.byref(v.desc),
                                           _ptr(block_idx), _ptr(block_cnt), _ptr(seqlens), block_idx.shape[-1],
                                           int(num_split), _ptr(out), _ptr(lse), _ptr(err), _stream(stream)))


def prefill_gt_workspace_bytes(shape: Shape, max_len: int) -> int:
    dims = shape.c()
    return int(_lib.seer_prefill_gt_workspace_bytes(ctypes.byref(dims), int(max_len)))


def prefill_gt(shape: Shape, q: torch.Tensor, k: KVCache, v: KVCache, seqlens: torch.Tensor, out: torch.Tensor,
               gt: torch.Tensor, workspace: torch.Tensor, lse: Optional[torch.Tensor] = None,
               err: Optional[torch.Tensor] = None, stream=None):
    """Causal attention [B, Hq, T, d] with every position's block-level target gt [B, Hkv, T, max_blocks]
    (see seer_prefill_gt); T = q.shape[2]."""
    if not isinstance(q, torch.Tensor) or q.dim() != 4:
        raise ValueError("q must be a 4-D [B, Hq, T, d] tensor")
    B, Hq, H, d, T = shape.batch, shape.num_q_heads, shape.num_kv_heads, shape.head_dim, int(q.shape[2])
    _need_shape(q, (B, Hq, T, d), "q")
    _need_shape(seqlens, (B,), "seqlens")
    _need_shape(out, (B, Hq, T, d), "out")
    _need_shape(gt, (B, H, T, shape.max_blocks), "gt")
    k.check(shape, "k")
    v.check(shape, "v")
    _need_err(err)
    if lse is not None:
        _need_shape(lse, (B, Hq, T), "lse")
    _need(q, torch.bfloat16, "q")
    _need(seqlens, torch.int32, "seqlens")
    _need(out, torch.bfloat16, "out")
    _need(gt, torch.float32, "gt")
    if lse is not None:
        _need(lse, torch.float32, "lse")
    dims = shape.c()
    _check(_lib.seer_prefill_gt(ctypes.byref(dims), _ptr(q), int(q.shape[2]), ctypes.byref(k.desc),
                                ctypes.byref(v.desc), _ptr(seqlens), _ptr(out), _ptr(lse) if lse is not None else None,
                                _ptr(gt), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _ptr(err) if err is not None else None, _stream(stream)))


def gate_truth_workspace_bytes(shape: Shape) -> int:
    dims = shape.c()
    return int(_lib.seer_gate_truth_workspace_bytes(ctypes.byref(dims)))


def alloc_truth_workspace(shape: Shape, device=None) -> torch.Tensor:
    """Zero-filled workspace for gate_truth (its arrival counters must start at zero)."""
    return torch.zeros(max(gate_truth_workspace_bytes(shape), 16), dtype=torch.uint8, device=device or "cuda")


def gate_truth(shape: Shape, q: torch.Tensor, k: KVCache, seqlens: torch.Tensor, scores: torch.Tensor,
               workspace: torch.Tensor, log_scores: Optional[torch.Tensor] = None, err: Optional[torch.Tensor] = None,
               stream=None):
    """Decode ground-truth block scores from full attention (see seer_gate_truth)."""
    B, H = shape.batch, shape.num_kv_heads
    _need_shape(q, (B, shape.num_q_heads, shape.head_dim), "q")
    k.check(shape, "k")
    _need_shape(seqlens, (B,), "seqlens")
    _need_shape(scores, (B, H, shape.max_blocks), "scores")
    if log_scores is not None:
        _need_shape(log_scores, (B, H, shape.max_blocks), "log_scores")
    _need_err(err)
    _need(q, torch.bfloat16, "q")
    _need(seqlens, torch.int32, "seqlens")
    _need(scores, torch.float32, "scores")
    if log_scores is not None:
        _need(log_scores, torch.float32, "log_scores")
    if err is not None:
        _need(err, torch.int32, "err")
    dims = shape.c()
    _check(_lib.seer_gate_truth(ctypes.byref(dims), _ptr(q), ctypes.byref(k.desc), _ptr(seqlens), _ptr(scores),
                                _ptr(log_scores), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _ptr(err), _stream(stream)))


class DecodeStep:
    """One layer's per-step pipeline: kcomp_update -> gate_score -> select_blocks -> sparse_decode.

    Owns the step's scratch tensors (logits, index lists, workspace, output) so a
    decode loop (or a CUDA graph capturing `run`) reuses them every step.

    With `kcomp_state` (alloc_kcomp_state; primed by kcomp_state_init when the sequences resume
    mid-block) the K Compression Cache is kept from running block statistics: each `run` takes
    the appended tokens' pre-RoPE keys `k_new` [B, Hkv, d] and no pre-RoPE copy of the context
    is read (kcomp_append, then the plan without its cache update).
    """

    def __init__(self, shape: Shape, k: KVCache, v: KVCache, w_q: torch.Tensor, w_k: torch.Tensor,
                 kcomp: torch.Tensor, valid_blocks: torch.Tensor, mode: int = SELECT_TOPK, token_budget: int = 0,
                 tau: float = 0.0, capacity: Optional[int] = None, num_split: Optional[int] = None,
                 k_nope: Optional[KVCache] = None, kcomp_state: Optional[torch.Tensor] = None,
                 single_launch: Optional[bool] = None, device=None):
        dev = device or w_q.device
        self.shape, self.k, self.v, self.w_q, self.w_k = shape, k, v, w_q, w_k
        self.k_nope = k_nope or k
        self.kcomp, self.valid_blocks = kcomp, valid_blocks
        self.kcomp_state = kcomp_state
        self.mode, self.token_budget, self.tau = mode, token_budget, tau
        if capacity is None:
            if mode == SELECT_TOPK:
                capacity = min(shape.max_blocks, -(-token_budget // shape.block_size) + 1)
            else:
                capacity = shape.max_blocks
        self.capacity = capacity
        B, Hq, Hkv = shape.batch, shape.num_q_heads, shape.num_kv_heads
        self.logits = torch.empty(B, Hkv, shape.max_blocks, dtype=torch.float32, device=dev)
        self.block_idx = torch.empty(B, Hkv, capacity, dtype=torch.int32, device=dev)
        self.block_cnt = torch.empty(B, Hkv, dtype=torch.int32, device=dev)
        if num_split is None:
            # top-k lists sit at (or near) their capacity: the capacity schedule needs no scan of
            # the counts; other modes use the balanced schedule
            num_split = -1 if mode == SELECT_TOPK else 0
        self.num_split = num_split    # -1 capacity, 0 balanced, >= 1 the pages' grid
        self.workspace = alloc_workspace(shape, capacity, self.num_split, dev)
        # single_launch=True runs the whole step as one launch (decode_step, capacity schedule); the
        # default is the plan and the decode as two launches, which measured faster (the plan kernel's
        # CTAs start while the previous decode drains; a launch that plans in its own CTAs cannot)
        if single_launch is None:
            single_launch = False
        if single_launch and (self.num_split != -1 or not decode_step_supported(shape, mode, capacity)):
            raise ValueError("single_launch needs num_split=-1 and a shape decode_step_supported accepts")
        self.single_launch = bool(single_launch)
        self.step_workspace = alloc_step_workspace(shape, capacity, dev) if self.single_launch else None
        self.kernels_per_step = (1 if self.single_launch else 2) + (1 if kcomp_state is not None else 0)
        self.out = torch.empty(B, Hq, shape.head_dim, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)

    def run(self, q: torch.Tensor, seqlens: torch.Tensor, q_nope: Optional[torch.Tensor] = None, stream=None,
            fused: bool = True, k_new: Optional[torch.Tensor] = None):
        """One decode step.  fused=True runs the whole step as one launch (seer_decode_step) when the
        step was built for it (single_launch), else plans with seer_decode_plan (one launch) and then
        decodes; fused=False makes the three separate planning calls (kcomp_update, gate_score,
        select_blocks) and then decodes.  With running
        block statistics (kcomp_state), `k_new` holds the appended tokens' pre-RoPE keys."""
        s = self.shape
        qn = q if q_nope is None else q_nope
        if self.single_launch and fused:
            upd = self.kcomp_state is None
            if not upd:
                if k_new is None:
                    raise ValueError("a step with running block statistics needs k_new, the appended pre-RoPE keys")
                kcomp_append(s, k_new, seqlens, self.kcomp_state, self.valid_blocks, self.w_k, self.kcomp, self.err,
                             stream)
            decode_step(s, seqlens, self.kcomp, qn, self.w_q, self.mode, self.block_idx, self.block_cnt, q, self.k,
                        self.v, self.out, self.step_workspace, self.token_budget, self.tau,
                        k_nope=self.k_nope if upd else None, valid_blocks=self.valid_blocks if upd else None,
                        w_k=self.w_k if upd else None, logits=self.logits, lse=self.lse, err=self.err,
                        stream=stream)
            return self.out
        if self.kcomp_state is not None:
            if k_new is None:
                raise ValueError("a step with running block statistics needs k_new, the appended pre-RoPE keys")
            kcomp_append(s, k_new, seqlens, self.kcomp_state, self.valid_blocks, self.w_k, self.kcomp, self.err,
                         stream)
            decode_plan(s, seqlens, self.kcomp, qn, self.w_q, self.mode, self.block_idx, self.block_cnt,
                        self.token_budget, self.tau, logits=self.logits, stream=stream)
        elif fused:
            decode_plan(s, seqlens, self.kcomp, qn, self.w_q, self.mode, self.block_idx, self.block_cnt,
                        self.token_budget, self.tau, k_nope=self.k_nope, valid_blocks=self.valid_blocks, w_k=self.w_k,
                        logits=self.logits, stream=stream)
        else:
            kcomp_update(s, self.k_nope, seqlens, self.valid_blocks, self.w_k, self.kcomp, stream)
            gate_score(s, qn, self.w_q, self.kcomp, seqlens, self.logits, None, stream)
            select_blocks(s, self.logits, seqlens, self.mode, self.block_idx, self.block_cnt, self.token_budget,
                          self.tau, stream)
        sparse_decode(s, q, self.k, self.v, self.block_idx, self.block_cnt, seqlens, self.out, self.workspace,
                      self.num_split, self.lse, self.err, stream)
        return self.out

