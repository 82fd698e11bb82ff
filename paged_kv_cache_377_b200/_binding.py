"""ctypes binding of libpagedkv.so: same names as the C ABI, torch tensors in."""
from __future__ import annotations

import ctypes
import fcntl
import os
import threading
from typing import Optional

import numpy as np
import torch

from . import build as _build

PKV_OK = 0
PKV_STATUS_BAD_BLOCK_ID = 1
PKV_STATUS_BAD_CONTEXT_LEN = 2
PKV_STATUS_WAIT_TIMEOUT = 4
PKV_STATUS_BAD_SLOT = 8
PKV_STATUS_BAD_PREFIX_GROUP = 16
PKV_MAX_PREFIX_GROUPS = 16

_lock = threading.Lock()
_lib: Optional[ctypes.CDLL] = None


class PagedKVError(RuntimeError):
    """A library call returned an error code (message from pkv_last_error)."""

    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed with code {code}: {msg}")
        self.code = code


class _PrefixGroups(ctypes.Structure):
    _fields_ = [("num_groups", ctypes.c_int), ("begin", ctypes.c_void_p), ("end", ctypes.c_void_p),
                ("blocks", ctypes.c_void_p)]


class _Options(ctypes.Structure):
    _fields_ = [("num_ctas", ctypes.c_int), ("num_stages", ctypes.c_int),
                ("ctas_per_sm", ctypes.c_int), ("math", ctypes.c_int), ("l2_prefetch", ctypes.c_int),
                ("piece_cost", ctypes.c_int), ("head_pack", ctypes.c_int), ("tile_tokens", ctypes.c_int),
                ("prefix_groups", ctypes.c_void_p), ("prefix_tiles", ctypes.c_int)]


class PrefixGroups:
    """Runs of consecutive sequences sharing their leading blocks (pkv_prefix_groups):
    group g is sequences begin[g] .. end[g] - 1, sharing table entries 0 .. blocks[g] - 1."""

    def __init__(self, begin, end, blocks):
        self.begin = np.ascontiguousarray(begin, dtype=np.int32)
        self.end = np.ascontiguousarray(end, dtype=np.int32)
        self.blocks = np.ascontiguousarray(blocks, dtype=np.int32)
        if not (len(self.begin) == len(self.end) == len(self.blocks)):
            raise ValueError("begin, end and blocks must have one entry per group")
        self._c = _PrefixGroups(len(self.begin), self.begin.ctypes.data, self.end.ctypes.data,
                                self.blocks.ctypes.data)

    def __len__(self):
        return len(self.begin)

    def __repr__(self):
        return f"PrefixGroups(begin={self.begin.tolist()}, end={self.end.tolist()}, blocks={self.blocks.tolist()})"

    def c_ptr(self):
        return ctypes.addressof(self._c) if len(self) else None


def find_prefix_groups(block_tables, context_lens, block_size: int, min_blocks: int = 1,
                       max_groups: int = PKV_MAX_PREFIX_GROUPS) -> PrefixGroups:
    """pkv_find_prefix_groups on HOST copies of a batch's tables (int32 [S][MB]) and lengths (int32 [S])."""
    bt = np.ascontiguousarray(block_tables.cpu().numpy() if isinstance(block_tables, torch.Tensor) else block_tables,
                              dtype=np.int32)
    cl = np.ascontiguousarray(context_lens.cpu().numpy() if isinstance(context_lens, torch.Tensor) else context_lens,
                              dtype=np.int32)
    if bt.ndim != 2 or cl.shape != (bt.shape[0],):
        raise ValueError("block_tables must be [S][MB] and context_lens [S]")
    begin = np.zeros(max(max_groups, 1), dtype=np.int32)
    end = np.zeros_like(begin)
    blocks = np.zeros_like(begin)
    n = ctypes.c_int(0)
    lib = library()
    rc = lib.pkv_find_prefix_groups(bt.ctypes.data, cl.ctypes.data, bt.shape[0], max(bt.shape[1], 1), block_size,
                                    min_blocks, begin.ctypes.data, end.ctypes.data, blocks.ctypes.data, max_groups,
                                    ctypes.byref(n))
    if rc != PKV_OK:
        raise PagedKVError("pkv_find_prefix_groups", rc, lib.pkv_bm_last_error().decode())
    k = n.value
    return PrefixGroups(begin[:k], end[:k], blocks[:k])


def _options(num_ctas=0, num_stages=0, ctas_per_sm=0, math=0, l2_prefetch=0, piece_cost=0, head_pack=0,
             tile_tokens=0, prefix_groups: Optional[PrefixGroups] = None, prefix_tiles=0) -> _Options:
    return _Options(num_ctas, num_stages, ctas_per_sm, math, l2_prefetch, piece_cost, head_pack, tile_tokens,
                    prefix_groups.c_ptr() if prefix_groups is not None else None, prefix_tiles)


def library_path() -> str:
    return _build.LIB


def _ensure_built() -> str:
    """Builds the library with nvcc when it is missing or older than its sources."""
    if not _build.is_stale():
        return _build.LIB
    os.makedirs(_build.BUILD, exist_ok=True)
    with open(os.path.join(_build.BUILD, ".lock"), "w") as lk:
        fcntl.flock(lk, fcntl.LOCK_EX)
        try:
            return _build.build()
        finally:
            fcntl.flock(lk, fcntl.LOCK_UN)


def library() -> ctypes.CDLL:
    """The loaded libpagedkv.so (built first if needed). Raises if unavailable."""
    global _lib
    with _lock:
        if _lib is None:
            path = _ensure_built()
            lib = ctypes.CDLL(path)
            P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
            lib.pkv_last_error.restype = ctypes.c_char_p
            lib.pkv_last_error.argtypes = []
            lib.pkv_version.restype = ctypes.c_char_p
            lib.pkv_decode_workspace_bytes.restype = I
            lib.pkv_decode_workspace_bytes.argtypes = [I, I, I, ctypes.POINTER(Z)]
            lib.paged_attn_decode.restype = I
            lib.paged_attn_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, I, I, P, Z, P]
            lib.paged_attn_decode_ex.restype = I
            lib.paged_attn_decode_ex.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, I, I, P, Z,
                                                 ctypes.POINTER(_Options), P]
            lib.paged_attn_decode_append.restype = I
            lib.paged_attn_decode_append.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, F, I, I, P, Z,
                                                     ctypes.POINTER(_Options), P]
            lib.paged_attn_decode_fp8.restype = I
            lib.paged_attn_decode_fp8.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, F, I, I, P, Z,
                                                  ctypes.POINTER(_Options), P]
            lib.paged_attn_decode_append_fp8.restype = I
            lib.paged_attn_decode_append_fp8.argtypes = [P, P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, F, I, I, P,
                                                         Z, ctypes.POINTER(_Options), P]
            lib.kv_cache_append_fp8.restype = I
            lib.kv_cache_append_fp8.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, P, P]
            lib.paged_attn_prefill.restype = I
            lib.paged_attn_prefill.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, F, I, I, P, P]
            lib.paged_attn_prefill_ex.restype = I
            lib.paged_attn_prefill_ex.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, F, I, I, P, I, P]
            lib.kv_cache_append.restype = I
            lib.kv_cache_append.argtypes = [P, P, P, P, P, I, I, I, I, I, P, P]
            lib.pkv_validate.restype = I
            lib.pkv_validate.argtypes = [P, P, I, I, I, I, P, P]
            lib.pkv_selftest_bounded_wait.restype = I
            lib.pkv_selftest_bounded_wait.argtypes = [P, P]
            lib.pkv_read_status.restype = I
            lib.pkv_read_status.argtypes = [P, ctypes.POINTER(ctypes.c_int32), I, P]
            lib.pkv_find_prefix_groups.restype = I
            lib.pkv_find_prefix_groups.argtypes = [P, P, I, I, I, I, P, P, P, I, ctypes.POINTER(I)]
            lib.pkv_bm_last_error.restype = ctypes.c_char_p
            lib.pkv_bm_last_error.argtypes = []
            _lib = lib
        return _lib


def _check(fn: str, rc: int) -> None:
    if rc != PKV_OK:
        raise PagedKVError(fn, rc, library().pkv_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        stream = stream.cuda_stream
    return ctypes.c_void_p(int(stream))


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device (got {t.device})")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype} (got {t.dtype})")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions (got shape {tuple(t.shape)})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def workspace_bytes(num_seqs: int, num_q_heads: int, head_dim: int) -> int:
    n = ctypes.c_size_t(0)
    _check("pkv_decode_workspace_bytes", library().pkv_decode_workspace_bytes(
        num_seqs, num_q_heads, head_dim, ctypes.byref(n)))
    return int(n.value)


def allocate_workspace(num_seqs: int, num_q_heads: int, head_dim: int, device=None) -> torch.Tensor:
    """A zeroed uint8 workspace of the required size (its first int32 is the status word)."""
    n = workspace_bytes(num_seqs, num_q_heads, head_dim)
    return torch.zeros(n, dtype=torch.uint8, device=device if device is not None else "cuda")


def _decode_shapes(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                   block_tables: torch.Tensor, context_lens: torch.Tensor):
    """(S, Hq, D, NB, bs, Hkv) of a decode call, after checking that the tensors
    agree: the C ABI sees only pointers and the sizes passed with them, so a
    short table or a head_dim mismatch would become out-of-bounds device accesses."""
    S, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_cache.shape
    if out.shape != q.shape or v_cache.shape != k_cache.shape or D2 != D:
        raise ValueError("shape mismatch between q/out or k_cache/v_cache")
    if block_tables.shape[0] != S or context_lens.shape[0] != S:
        raise ValueError("block_tables and context_lens must have num_seqs rows")
    return S, Hq, D, NB, bs, Hkv


def paged_attn_decode(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                      block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                      workspace: torch.Tensor, num_ctas: int = 0, num_stages: int = 0,
                      ctas_per_sm: int = 0, math: int = 0, l2_prefetch: int = 0, piece_cost: int = 0,
                      head_pack: int = 0, tile_tokens: int = 0, prefix_groups: Optional[PrefixGroups] = None,
                      prefix_tiles: int = 0, stream=None) -> torch.Tensor:
    """out[s, j] = softmax_t(scale * q[s, j] . K_t) . V_t over the sequence's paged tokens.

    q, out: bf16 [S, Hq, D]; k_cache, v_cache: bf16 [NB, bs, Hkv, D];
    block_tables: int32 [S, MB]; context_lens: int32 [S]; workspace: uint8 from
    allocate_workspace(). Enqueued on ``stream`` (default: torch's current stream).
    prefix_groups: runs of sequences sharing their leading blocks (find_prefix_groups),
    whose shared blocks are then read once per group.
    """
    _need(q, "q", torch.bfloat16, 3)
    _need(out, "out", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(block_tables, "block_tables", torch.int32, 2)
    _need(context_lens, "context_lens", torch.int32, 1)
    _need(workspace, "workspace", torch.uint8, 1)
    S, Hq, D, NB, bs, Hkv = _decode_shapes(out, q, k_cache, v_cache, block_tables, context_lens)
    opts = _options(num_ctas, num_stages, ctas_per_sm, math, l2_prefetch, piece_cost, head_pack, tile_tokens,
                    prefix_groups, prefix_tiles)
    _check("paged_attn_decode", library().paged_attn_decode_ex(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
        S, Hq, Hkv, D, bs, float(scale), block_tables.shape[1], NB, _ptr(workspace), workspace.numel(),
        ctypes.byref(opts), _stream(stream)))
    return out


def _decode_append_args(out, q, k_new, v_new, slot_mapping, k_cache, v_cache, block_tables, context_lens, scale,
                        workspace, stream, options):
    """Checks the fused step's tensors and returns (argument tuple, objects it points into)."""
    _need(q, "q", torch.bfloat16, 3)
    _need(out, "out", torch.bfloat16, 3)
    _need(k_new, "k_new", torch.bfloat16, 3)
    _need(v_new, "v_new", torch.bfloat16, 3)
    _need(slot_mapping, "slot_mapping", torch.int64, 1)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(block_tables, "block_tables", torch.int32, 2)
    _need(context_lens, "context_lens", torch.int32, 1)
    _need(workspace, "workspace", torch.uint8, 1)
    S, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_cache.shape
    if out.shape != q.shape or v_cache.shape != k_cache.shape or D2 != D:
        raise ValueError("shape mismatch between q/out or k_cache/v_cache")
    if k_new.shape != (S, Hkv, D) or v_new.shape != k_new.shape or slot_mapping.shape[0] != S:
        raise ValueError("k_new / v_new must be [num_seqs, num_kv_heads, head_dim] and slot_mapping [num_seqs]")
    if block_tables.shape[0] != S or context_lens.shape[0] != S:
        raise ValueError("block_tables and context_lens must have num_seqs rows")
    opts = _options(**options)
    args = (_ptr(out), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(slot_mapping), _ptr(k_cache), _ptr(v_cache),
            _ptr(block_tables), _ptr(context_lens), S, Hq, Hkv, D, bs, float(scale), block_tables.shape[1], NB,
            _ptr(workspace), workspace.numel(), ctypes.byref(opts), _stream(stream))
    return args, (opts, options.get("prefix_groups"))


def paged_attn_decode_append(out: torch.Tensor, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                             slot_mapping: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                             block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                             workspace: torch.Tensor, num_ctas: int = 0, num_stages: int = 0,
                             ctas_per_sm: int = 0, math: int = 0, l2_prefetch: int = 0, piece_cost: int = 0,
                             head_pack: int = 0, tile_tokens: int = 0, prefix_groups: Optional[PrefixGroups] = None,
                             prefix_tiles: int = 0, stream=None) -> torch.Tensor:
    """One decode step in one launch: append k_new / v_new (bf16 [S, Hkv, D]) at
    slot_mapping (int64 [S], the slot of each sequence's last position, < 0 =
    none), then the same attention as paged_attn_decode over contexts that
    include the new token. Bit-identical to kv_cache_append + paged_attn_decode.
    """
    args, _keep = _decode_append_args(out, q, k_new, v_new, slot_mapping, k_cache, v_cache, block_tables,
                                      context_lens, scale, workspace, stream,
                                      dict(num_ctas=num_ctas, num_stages=num_stages, ctas_per_sm=ctas_per_sm,
                                           math=math, l2_prefetch=l2_prefetch, piece_cost=piece_cost,
                                           head_pack=head_pack, tile_tokens=tile_tokens,
                                           prefix_groups=prefix_groups, prefix_tiles=prefix_tiles))
    _check("paged_attn_decode_append", library().paged_attn_decode_append(*args))
    return out


class DecodeAppendCall:
    """paged_attn_decode_append over fixed device buffers, checked and
    marshalled once: ``call()`` then costs the C entry alone.

    For a serving loop that keeps a step's inputs in static buffers and refills
    them between steps (as a captured CUDA graph also needs). The buffers must
    stay allocated with the same shapes while the object is used; the stream is
    the one given (default: torch's current stream at construction). The
    keyword options are those of paged_attn_decode_append.
    """

    def __init__(self, out, q, k_new, v_new, slot_mapping, k_cache, v_cache, block_tables, context_lens, scale,
                 workspace, stream=None, **options):
        self._args, self._keep = _decode_append_args(out, q, k_new, v_new, slot_mapping, k_cache, v_cache,
                                                     block_tables, context_lens, scale, workspace, stream, options)
        self._tensors = (out, q, k_new, v_new, slot_mapping, k_cache, v_cache, block_tables, context_lens,
                         workspace)
        self._fn = library().paged_attn_decode_append
        self.out = out

    def __call__(self) -> torch.Tensor:
        rc = self._fn(*self._args)
        if rc != PKV_OK:
            _check("paged_attn_decode_append", rc)
        return self.out


def kv_cache_append(k: torch.Tensor, v: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                    slot_mapping: torch.Tensor, status: Optional[torch.Tensor] = None, stream=None) -> None:
    """k_cache[slot // bs, slot % bs] = k[i] (and v) for every token i with slot >= 0.

    k, v: bf16 [T, Hkv, D]; caches bf16 [NB, bs, Hkv, D]; slot_mapping int64 [T];
    status: optional int32 device tensor (status word, PKV_STATUS_BAD_SLOT).
    """
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(slot_mapping, "slot_mapping", torch.int64, 1)
    if status is not None:
        _need(status, "status", torch.int32, 1)
    T, Hkv, D = k.shape
    NB, bs, Hkv2, D2 = k_cache.shape
    if v.shape != k.shape or v_cache.shape != k_cache.shape or (Hkv2, D2) != (Hkv, D) or slot_mapping.shape[0] != T:
        raise ValueError("shape mismatch between k/v, caches and slot_mapping")
    _check("kv_cache_append", library().kv_cache_append(
        _ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping), T, Hkv, D, bs, NB,
        _ptr(status), _stream(stream)))


def validate(block_tables: torch.Tensor, context_lens: torch.Tensor, num_blocks: int, block_size: int,
             status: torch.Tensor, stream=None) -> None:
    """Enqueues the device check of tables and lengths; bits go into ``status``."""
    _need(block_tables, "block_tables", torch.int32, 2)
    _need(context_lens, "context_lens", torch.int32, 1)
    _need(status, "status", torch.int32, 1)
    _check("pkv_validate", library().pkv_validate(
        _ptr(block_tables), _ptr(context_lens), block_tables.shape[0], block_tables.shape[1], block_size,
        num_blocks, _ptr(status), _stream(stream)))


def read_status(status: torch.Tensor, clear: bool = False, stream=None) -> int:
    """Synchronises the stream and returns the status word (a workspace's first int32, or an int32 tensor)."""
    if status.dtype == torch.uint8:
        status = status[:4].view(torch.int32)
    _need(status, "status", torch.int32, 1)
    out = ctypes.c_int32(0)
    _check("pkv_read_status", library().pkv_read_status(_ptr(status), ctypes.byref(out), int(clear),
                                                        _stream(stream)))
    return int(out.value)


def selftest_bounded_wait(status: torch.Tensor, stream=None) -> None:
    """Enqueues the kernel whose bounded wait must give up (about one second)."""
    _need(status, "status", torch.int32, 1)
    _check("pkv_selftest_bounded_wait", library().pkv_selftest_bounded_wait(_ptr(status), _stream(stream)))


_noalloc_ready = False


def paged_attn_decode_noalloc(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                              block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                              status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """paged_attn_decode without a workspace, for callers that cannot allocate device memory.

    The library's static device scratch (64 MiB per GPU) stands in for the
    workspace; calls that overlap on the GPU race on it. ``status``: optional
    int32 device tensor overwritten with the call's status bits.
    """
    global _noalloc_ready
    _need(q, "q", torch.bfloat16, 3)
    _need(out, "out", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(block_tables, "block_tables", torch.int32, 2)
    _need(context_lens, "context_lens", torch.int32, 1)
    if status is not None:
        _need(status, "status", torch.int32, 1)
    S, Hq, D, NB, bs, Hkv = _decode_shapes(out, q, k_cache, v_cache, block_tables, context_lens)
    lib = library()
    if not _noalloc_ready:
        P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        lib.paged_attn_decode_noalloc.restype = I
        lib.paged_attn_decode_noalloc.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, I, I, P, P]
        _noalloc_ready = True
    _check("paged_attn_decode_noalloc", lib.paged_attn_decode_noalloc(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
        S, Hq, Hkv, D, bs, float(scale), block_tables.shape[1], NB, _ptr(status), _stream(stream)))
    return out


def _need_scales(k_scale, v_scale, hkv):
    _need(k_scale, "k_scale", torch.float32, 1)
    _need(v_scale, "v_scale", torch.float32, 1)
    if k_scale.shape[0] != hkv or v_scale.shape[0] != hkv:
        raise ValueError("k_scale and v_scale must have num_kv_heads entries")


def paged_attn_decode_fp8(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                          k_scale: torch.Tensor, v_scale: torch.Tensor, block_tables: torch.Tensor,
                          context_lens: torch.Tensor, scale: float, workspace: torch.Tensor, stream=None,
                          **options) -> torch.Tensor:
    """paged_attn_decode over e4m3 pools (uint8 [NB, bs, Hkv, D]) with fp32 per-head scales [Hkv]."""
    _need(q, "q", torch.bfloat16, 3)
    _need(out, "out", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.uint8, 4)
    _need(v_cache, "v_cache", torch.uint8, 4)
    _need(block_tables, "block_tables", torch.int32, 2)
    _need(context_lens, "context_lens", torch.int32, 1)
    _need(workspace, "workspace", torch.uint8, 1)
    S, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_cache.shape
    if out.shape != q.shape or v_cache.shape != k_cache.shape or D2 != D:
        raise ValueError("shape mismatch between q/out or k_cache/v_cache")
    if block_tables.shape[0] != S or context_lens.shape[0] != S:
        raise ValueError("block_tables and context_lens must have num_seqs rows")
    _need_scales(k_scale, v_scale, Hkv)
    opts = _options(**options)
    _check("paged_attn_decode_fp8", library().paged_attn_decode_fp8(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), _ptr(block_tables),
        _ptr(context_lens), S, Hq, Hkv, D, bs, float(scale), block_tables.shape[1], NB, _ptr(workspace),
        workspace.numel(), ctypes.byref(opts), _stream(stream)))
    return out


def _decode_append_fp8_args(out, q, k_new, v_new, slot_mapping, k_cache, v_cache, k_scale, v_scale, block_tables,
                            context_lens, scale, workspace, stream, options):
    """Checks the e4m3 fused step's tensors and returns (argument tuple, objects it points into)."""
    _need(q, "q", torch.bfloat16, 3)
    _need(out, "out", torch.bfloat16, 3)
    _need(k_new, "k_new", torch.bfloat16, 3)
    _need(v_new, "v_new", torch.bfloat16, 3)
    _need(slot_mapping, "slot_mapping", torch.int64, 1)
    _need(k_cache, "k_cache", torch.uint8, 4)
    _need(v_cache, "v_cache", torch.uint8, 4)
    _need(block_tables, "block_tables", torch.int32, 2)
    _need(context_lens, "context_lens", torch.int32, 1)
    _need(workspace, "workspace", torch.uint8, 1)
    S, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_cache.shape
    if out.shape != q.shape or v_cache.shape != k_cache.shape or D2 != D:
        raise ValueError("shape mismatch between q/out or k_cache/v_cache")
    if k_new.shape != (S, Hkv, D) or v_new.shape != k_new.shape or slot_mapping.shape[0] != S:
        raise ValueError("k_new / v_new must be [num_seqs, num_kv_heads, head_dim] and slot_mapping [num_seqs]")
    if block_tables.shape[0] != S or context_lens.shape[0] != S:
        raise ValueError("block_tables and context_lens must have num_seqs rows")
    _need_scales(k_scale, v_scale, Hkv)
    opts = _options(**options)
    args = (_ptr(out), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(slot_mapping), _ptr(k_cache), _ptr(v_cache),
            _ptr(k_scale), _ptr(v_scale), _ptr(block_tables), _ptr(context_lens), S, Hq, Hkv, D, bs, float(scale),
            block_tables.shape[1], NB, _ptr(workspace), workspace.numel(), ctypes.byref(opts), _stream(stream))
    return args, (opts, options.get("prefix_groups"))


def paged_attn_decode_append_fp8(out: torch.Tensor, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                                 slot_mapping: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                                 k_scale: torch.Tensor, v_scale: torch.Tensor, block_tables: torch.Tensor,
                                 context_lens: torch.Tensor, scale: float, workspace: torch.Tensor, stream=None,
                                 **options) -> torch.Tensor:
    """The one-launch decode step over e4m3 pools (the new bf16 rows are quantized)."""
    args, _keep = _decode_append_fp8_args(out, q, k_new, v_new, slot_mapping, k_cache, v_cache, k_scale, v_scale,
                                          block_tables, context_lens, scale, workspace, stream, options)
    _check("paged_attn_decode_append_fp8", library().paged_attn_decode_append_fp8(*args))
    return out


class DecodeAppendFp8Call:
    """paged_attn_decode_append_fp8 over fixed device buffers, checked and
    marshalled once (the e4m3 counterpart of DecodeAppendCall): ``call()``
    then costs the C entry alone. The buffers, scales included, must stay
    allocated with the same shapes while the object is used.
    """

    def __init__(self, out, q, k_new, v_new, slot_mapping, k_cache, v_cache, k_scale, v_scale, block_tables,
                 context_lens, scale, workspace, stream=None, **options):
        self._args, self._keep = _decode_append_fp8_args(out, q, k_new, v_new, slot_mapping, k_cache, v_cache,
                                                         k_scale, v_scale, block_tables, context_lens, scale,
                                                         workspace, stream, options)
        self._tensors = (out, q, k_new, v_new, slot_mapping, k_cache, v_cache, k_scale, v_scale, block_tables,
                         context_lens, workspace)
        self._fn = library().paged_attn_decode_append_fp8
        self.out = out

    def __call__(self) -> torch.Tensor:
        rc = self._fn(*self._args)
        if rc != PKV_OK:
            _check("paged_attn_decode_append_fp8", rc)
        return self.out


def kv_cache_append_fp8(k: torch.Tensor, v: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                        slot_mapping: torch.Tensor, k_scale: torch.Tensor, v_scale: torch.Tensor,
                        status: Optional[torch.Tensor] = None, stream=None) -> None:
    """Quantizing append into e4m3 pools: code = e4m3(x / scale[h]), rounded to nearest, saturated."""
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.uint8, 4)
    _need(v_cache, "v_cache", torch.uint8, 4)
    _need(slot_mapping, "slot_mapping", torch.int64, 1)
    if status is not None:
        _need(status, "status", torch.int32, 1)
    T, Hkv, D = k.shape
    NB, bs, Hkv2, D2 = k_cache.shape
    if v.shape != k.shape or v_cache.shape != k_cache.shape or (Hkv2, D2) != (Hkv, D) or slot_mapping.shape[0] != T:
        raise ValueError("shape mismatch between k/v, caches and slot_mapping")
    _need_scales(k_scale, v_scale, Hkv)
    _check("kv_cache_append_fp8", library().kv_cache_append_fp8(
        _ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping), _ptr(k_scale), _ptr(v_scale), T, Hkv,
        D, bs, NB, _ptr(status), _stream(stream)))


def paged_attn_prefill(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                       block_tables: torch.Tensor, context_lens: torch.Tensor, query_start: torch.Tensor,
                       max_query_len: int, scale: float, status: torch.Tensor, kernel: int = 0,
                       stream=None) -> torch.Tensor:
    """Multi-query paged attention: q bf16 [T, Hq, D]; the queries of sequence s are rows
    query_start[s] .. query_start[s+1]-1, the last tokens of its context, attending causally.
    kernel: 0 = default (tcgen05 where it applies), 1 = mma.sync, 2 = tcgen05."""
    _need(q, "q", torch.bfloat16, 3)
    _need(out, "out", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(block_tables, "block_tables", torch.int32, 2)
    _need(context_lens, "context_lens", torch.int32, 1)
    _need(query_start, "query_start", torch.int32, 1)
    _need(status, "status", torch.int32, 1)
    T, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_cache.shape
    S = context_lens.shape[0]
    if out.shape != q.shape or v_cache.shape != k_cache.shape or D2 != D:
        raise ValueError("shape mismatch between q/out or k_cache/v_cache")
    if block_tables.shape[0] != S or query_start.shape[0] != S + 1:
        raise ValueError("block_tables needs num_seqs rows and query_start num_seqs + 1 entries")
    _check("paged_attn_prefill", library().paged_attn_prefill_ex(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens), _ptr(query_start),
        S, T, int(max_query_len), Hq, Hkv, D, bs, float(scale), block_tables.shape[1], NB, _ptr(status),
        int(kernel), _stream(stream)))
    return out
