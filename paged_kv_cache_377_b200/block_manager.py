"""Python face of the library's host-side block manager and block-copy kernel.

Marshalling only: allocation, reference counts, copy-on-write decisions and
table packing run in the C++ manager inside libpagedkv.so (pkv_bm_* in
include/pagedkv.h); the copies run in its kv_block_copy kernel.
"""
from __future__ import annotations

import ctypes
import threading
from typing import Optional, Sequence, Tuple

import numpy as np
import torch

from ._binding import PagedKVError, _check, _need, _ptr, _stream, library

PKV_ERR_OUT_OF_BLOCKS = -4

_ready = False
_lock = threading.Lock()


def _lib():
    global _ready
    lib = library()
    with _lock:
        if not _ready:
            P, I, L = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
            lib.pkv_bm_create.restype = P
            lib.pkv_bm_create.argtypes = [I, I]
            lib.pkv_bm_destroy.restype = None
            lib.pkv_bm_destroy.argtypes = [P]
            for name in ("pkv_bm_num_free", "pkv_bm_pending_copies"):
                getattr(lib, name).restype = I
                getattr(lib, name).argtypes = [P]
            lib.pkv_bm_refcount.restype = I
            lib.pkv_bm_refcount.argtypes = [P, I]
            lib.pkv_bm_add.restype = I
            lib.pkv_bm_add.argtypes = [P, L, L, L, L, P]
            lib.pkv_bm_fork.restype = I
            lib.pkv_bm_fork.argtypes = [P, L, L]
            lib.pkv_bm_append.restype = I
            lib.pkv_bm_append.argtypes = [P, L, ctypes.POINTER(L)]
            lib.pkv_bm_free.restype = I
            lib.pkv_bm_free.argtypes = [P, L]
            lib.pkv_bm_take_copies.restype = I
            lib.pkv_bm_take_copies.argtypes = [P, P, P, I]
            lib.pkv_bm_seq_len.restype = I
            lib.pkv_bm_seq_len.argtypes = [P, L, ctypes.POINTER(L)]
            lib.pkv_bm_pack.restype = I
            lib.pkv_bm_pack.argtypes = [P, P, I, I, P, P]
            lib.pkv_bm_last_error.restype = ctypes.c_char_p
            lib.pkv_bm_last_error.argtypes = []
            lib.kv_block_copy.restype = I
            lib.kv_block_copy.argtypes = [P, P, P, P, I, I, I, I, I, I, P, P]
            _ready = True
    return lib


class OutOfBlocks(PagedKVError):
    pass


def _bm_check(fn: str, rc: int) -> int:
    if rc < 0:
        msg = _lib().pkv_bm_last_error().decode()
        raise (OutOfBlocks if rc == PKV_ERR_OUT_OF_BLOCKS else PagedKVError)(fn, rc, msg)
    return rc


def _np_ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


class BlockManager:
    """Blocks of one KV pool: per-sequence block tables, reference counts,
    copy-on-write, and the step's packed tables (see pkv_bm_* in pagedkv.h)."""

    def __init__(self, num_blocks: int, block_size: int):
        self._h = _lib().pkv_bm_create(int(num_blocks), int(block_size))
        if not self._h:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)

    def close(self) -> None:
        if self._h:
            _lib().pkv_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def num_free(self) -> int:
        return _bm_check("pkv_bm_num_free", _lib().pkv_bm_num_free(self._h))

    @property
    def pending_copies(self) -> int:
        return _bm_check("pkv_bm_pending_copies", _lib().pkv_bm_pending_copies(self._h))

    def refcount(self, block: int) -> int:
        return _bm_check("pkv_bm_refcount", _lib().pkv_bm_refcount(self._h, int(block)))

    def add(self, seq_id: int, num_tokens: int, prefix_seq: int = -1, prefix_tokens: int = 0) -> np.ndarray:
        """A new sequence of num_tokens prompt tokens; returns each token's slot (-1: shared, already cached)."""
        slots = np.empty(max(int(num_tokens), 1), dtype=np.int64)
        _bm_check("pkv_bm_add", _lib().pkv_bm_add(self._h, int(seq_id), int(num_tokens), int(prefix_seq),
                                                  int(prefix_tokens), _np_ptr(slots)))
        return slots[:int(num_tokens)]

    def fork(self, parent: int, child: int) -> None:
        _bm_check("pkv_bm_fork", _lib().pkv_bm_fork(self._h, int(parent), int(child)))

    def append(self, seq_id: int) -> int:
        """Reserves the sequence's next position; returns its slot."""
        slot = ctypes.c_int64(0)
        _bm_check("pkv_bm_append", _lib().pkv_bm_append(self._h, int(seq_id), ctypes.byref(slot)))
        return int(slot.value)

    def free(self, seq_id: int) -> None:
        _bm_check("pkv_bm_free", _lib().pkv_bm_free(self._h, int(seq_id)))

    def take_copies(self) -> Tuple[np.ndarray, np.ndarray]:
        n = self.pending_copies
        src = np.empty(max(n, 1), dtype=np.int32)
        dst = np.empty(max(n, 1), dtype=np.int32)
        got = _bm_check("pkv_bm_take_copies", _lib().pkv_bm_take_copies(self._h, _np_ptr(src), _np_ptr(dst), n))
        return src[:got], dst[:got]

    def seq_len(self, seq_id: int) -> int:
        n = ctypes.c_int64(0)
        _bm_check("pkv_bm_seq_len", _lib().pkv_bm_seq_len(self._h, int(seq_id), ctypes.byref(n)))
        return int(n.value)

    def pack(self, seq_ids: Sequence[int], max_blocks_per_seq: int) -> Tuple[np.ndarray, np.ndarray]:
        """(block_tables int32 [S, max_blocks_per_seq], context_lens int32 [S]) of the listed sequences."""
        ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int64))
        S = len(ids)
        bt = np.empty((max(S, 1), int(max_blocks_per_seq)), dtype=np.int32)
        cl = np.empty(max(S, 1), dtype=np.int32)
        _bm_check("pkv_bm_pack", _lib().pkv_bm_pack(self._h, _np_ptr(ids) if S else None, S,
                                                    int(max_blocks_per_seq), _np_ptr(bt), _np_ptr(cl)))
        return bt[:S], cl[:S]


def kv_block_copy(k_cache: torch.Tensor, v_cache: torch.Tensor, src: torch.Tensor, dst: torch.Tensor,
                  status: Optional[torch.Tensor] = None, stream=None) -> None:
    """Block dst[c] of both pools (bf16, or uint8 e4m3 codes) becomes a copy of block src[c]
    (device int32 tensors)."""
    dtype = k_cache.dtype if k_cache.dtype in (torch.bfloat16, torch.uint8) else torch.bfloat16
    _need(k_cache, "k_cache", dtype, 4)
    _need(v_cache, "v_cache", dtype, 4)
    _need(src, "src", torch.int32, 1)
    _need(dst, "dst", torch.int32, 1)
    if status is not None:
        _need(status, "status", torch.int32, 1)
    if v_cache.shape != k_cache.shape or src.shape != dst.shape:
        raise ValueError("k_cache / v_cache or src / dst shapes differ")
    NB, bs, Hkv, D = k_cache.shape
    _check("kv_block_copy", _lib().kv_block_copy(_ptr(k_cache), _ptr(v_cache), _ptr(src), _ptr(dst), src.numel(),
                                                 Hkv, D, k_cache.element_size(), bs, NB, _ptr(status),
                                                 _stream(stream)))
