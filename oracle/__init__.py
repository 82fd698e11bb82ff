"""fp64 CPU oracle for paged decode attention and the slot-mapped KV append.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline use it; the product path never does.  It is plain C (``oracle.c``),
built with gcc into ``oracle/_build/liboracle.so`` and called through ctypes.
It imports nothing from the CUDA package.

What each function computes, and the passages it follows, is written at the
top of ``oracle.c``.  Pins (tests that tie this oracle to something other than
itself) live in ``tests/test_oracle_pins.py``; ``tests/test_oracle_mutants.py``
plants mistakes in copies of ``oracle.c`` and checks that the pins catch them.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None


class OracleError(RuntimeError):
    pass


def _compile(src: str, out: str) -> None:
    tmp = out + f".tmp{os.getpid()}"
    subprocess.run(
        ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-Wextra",
         "-o", tmp, src, "-lm"],
        check=True,
    )
    os.replace(tmp, out)


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (-O2 -fopenmp, no fast-math: IEEE fp64)."""
    with _lock:
        stale = not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
        if force or stale:
            os.makedirs(_BUILD, exist_ok=True)
            _compile(_SRC, _LIB_PATH)
    return _LIB_PATH


def _bind(path: str):
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    lib.oracle_paged_decode.restype = ctypes.c_int
    lib.oracle_paged_decode.argtypes = [
        P, P, P, P, P, P,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_int, ctypes.c_int64, ctypes.c_double,
        P, ctypes.c_int64, ctypes.c_int,
    ]
    lib.oracle_kv_append.restype = ctypes.c_int
    lib.oracle_kv_append.argtypes = [
        P, P, P, P, P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64,
    ]
    lib.oracle_e4m3_to_double.restype = ctypes.c_double
    lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_from_float.restype = ctypes.c_uint8
    lib.oracle_e4m3_from_float.argtypes = [ctypes.c_float]
    lib.oracle_paged_decode_fp8.restype = ctypes.c_int
    lib.oracle_paged_decode_fp8.argtypes = [
        P, P, P, P, P, P, P, P,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_int, ctypes.c_int64, ctypes.c_double,
        P, ctypes.c_int64, ctypes.c_int,
    ]
    lib.oracle_paged_prefill.restype = ctypes.c_int
    lib.oracle_paged_prefill.argtypes = [
        P, P, P, P, P, P, P,
        ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_int,
    ]
    lib.oracle_kv_append_fp8.restype = ctypes.c_int
    lib.oracle_kv_append_fp8.argtypes = [
        P, P, P, P, P, P, P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64,
    ]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(build())
    return _lib


def build_variant(src_text: str, workdir: str):
    """Compile a modified copy of oracle.c (for the mutation tests) and bind it.

    Returns a handle to pass as ``lib=`` to ``paged_decode`` / ``kv_append``.
    """
    src = os.path.join(workdir, "oracle_variant.c")
    out = os.path.join(workdir, "liboracle_variant.so")
    with open(src, "w") as f:
        f.write(src_text)
    _compile(src, out)
    return _bind(out)


def source() -> str:
    with open(_SRC) as f:
        return f.read()


def _bits(a) -> np.ndarray:
    """bf16 data (torch bf16 tensor or uint16 array of bf16 bits) -> contiguous uint16."""
    if isinstance(a, np.ndarray):
        assert a.dtype == np.uint16
        return np.ascontiguousarray(a)
    import torch
    assert a.dtype == torch.bfloat16
    return a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _u8(a) -> np.ndarray:
    """e4m3 codes (torch uint8 tensor or numpy uint8) -> contiguous uint8."""
    if isinstance(a, np.ndarray):
        assert a.dtype == np.uint8
        return np.ascontiguousarray(a)
    import torch
    assert a.dtype == torch.uint8
    return a.detach().cpu().contiguous().numpy()


def _f32(a) -> np.ndarray:
    if not isinstance(a, np.ndarray):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.float32)


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a), dtype=np.int32)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, num_kv_heads: int,
                 block_size: int, scale: float, pairs: Optional[Sequence[int]] = None,
                 num_threads: int = 0, lib=None) -> np.ndarray:
    """fp64 paged decode attention.

    q: bf16 [S][Hq][D]; k_cache/v_cache: bf16 [NB][bs][Hkv][D]; block_tables int32
    [S][MB]; context_lens int32 [S].  Returns float64 [S][Hq][D], or [len(pairs)][D]
    when ``pairs`` (flat indices s*Hq + j) is given.
    """
    qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
    S, Hq, D = qb.shape
    NB = kb.shape[0]
    assert kb.shape == (NB, block_size, num_kv_heads, D) and vb.shape == kb.shape
    bt = _i32(block_tables)
    cl = _i32(context_lens)
    assert bt.ndim == 2 and bt.shape[0] == S and cl.shape == (S,)
    MB = bt.shape[1]
    if pairs is None:
        npairs, pp = S * Hq, None
    else:
        pp = np.ascontiguousarray(np.asarray(pairs), dtype=np.int64)
        npairs = len(pp)
    out = np.zeros((npairs, D), dtype=np.float64)
    rc = (lib or _load()).oracle_paged_decode(
        _ptr(out), _ptr(qb), _ptr(kb), _ptr(vb), _ptr(bt), _ptr(cl),
        S, Hq, num_kv_heads, D, block_size, MB, NB, float(scale),
        _ptr(pp) if pp is not None else None, npairs, int(num_threads))
    if rc != 0:
        raise OracleError(f"oracle_paged_decode returned {rc}")
    return out.reshape(S, Hq, D) if pairs is None else out


def kv_append(k_cache, v_cache, k, v, slot_mapping, block_size: int, lib=None):
    """Slot-mapped append on copies of the pools; returns (k_cache', v_cache') as uint16 bits."""
    kc = _bits(k_cache).copy()
    vc = _bits(v_cache).copy()
    kb, vb = _bits(k), _bits(v)
    sm = np.ascontiguousarray(np.asarray(slot_mapping), dtype=np.int64)
    NB, bs, Hkv, D = kc.shape
    assert bs == block_size and kb.shape == (len(sm), Hkv, D) and vb.shape == kb.shape
    rc = (lib or _load()).oracle_kv_append(_ptr(kc), _ptr(vc), _ptr(kb), _ptr(vb), _ptr(sm), len(sm),
                                           Hkv, D, block_size, NB)
    if rc != 0:
        raise OracleError(f"oracle_kv_append returned {rc}")
    return kc, vc


def decode_step(batch, pairs: Optional[Sequence[int]] = None, num_threads: int = 0, lib=None):
    """One whole decode step of a ``workloads.DecodeBatch``: append, then attend.

    Returns (out fp64, k_cache' bits, v_cache' bits) -- codes for an e4m3 batch.
    """
    if getattr(batch, "kv_dtype", "bf16") == "fp8":
        return decode_step_fp8(batch, pairs=pairs, num_threads=num_threads, lib=lib)
    kc, vc = kv_append(batch.k_cache, batch.v_cache, batch.k_new, batch.v_new,
                       batch.slot_mapping.numpy(), batch.block_size, lib=lib)
    out = paged_decode(batch.q, kc, vc, batch.block_tables.numpy(), batch.context_lens.numpy(),
                       batch.num_kv_heads, batch.block_size, batch.scale, pairs=pairs,
                       num_threads=num_threads, lib=lib)
    return out, kc, vc


def e4m3_to_double(codes, lib=None) -> np.ndarray:
    """Values of e4m3 codes (NaN for the two NaN codes), one C call per code."""
    c = np.asarray(codes, dtype=np.uint8)
    f = (lib or _load()).oracle_e4m3_to_double
    return np.array([f(int(x)) for x in c.ravel()], dtype=np.float64).reshape(c.shape)


def e4m3_from_float(x, lib=None) -> np.ndarray:
    """Nearest e4m3 codes of fp32 values (ties to even, saturating at +-448)."""
    a = np.asarray(x, dtype=np.float32)
    f = (lib or _load()).oracle_e4m3_from_float
    return np.array([f(float(v)) for v in a.ravel()], dtype=np.uint8).reshape(a.shape)


def paged_decode_fp8(q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, num_kv_heads: int,
                     block_size: int, scale: float, pairs: Optional[Sequence[int]] = None,
                     num_threads: int = 0, lib=None) -> np.ndarray:
    """fp64 paged decode attention over an e4m3 cache (codes [NB][bs][Hkv][D], fp32 scales [Hkv])."""
    qb, kb, vb = _bits(q), _u8(k_cache), _u8(v_cache)
    ks, vs = _f32(k_scale), _f32(v_scale)
    S, Hq, D = qb.shape
    NB = kb.shape[0]
    assert kb.shape == (NB, block_size, num_kv_heads, D) and vb.shape == kb.shape
    assert ks.shape == (num_kv_heads,) and vs.shape == ks.shape
    bt = _i32(block_tables)
    cl = _i32(context_lens)
    MB = bt.shape[1]
    if pairs is None:
        npairs, pp = S * Hq, None
    else:
        pp = np.ascontiguousarray(np.asarray(pairs), dtype=np.int64)
        npairs = len(pp)
    out = np.zeros((npairs, D), dtype=np.float64)
    rc = (lib or _load()).oracle_paged_decode_fp8(
        _ptr(out), _ptr(qb), _ptr(kb), _ptr(vb), _ptr(ks), _ptr(vs), _ptr(bt), _ptr(cl),
        S, Hq, num_kv_heads, D, block_size, MB, NB, float(scale),
        _ptr(pp) if pp is not None else None, npairs, int(num_threads))
    if rc != 0:
        raise OracleError(f"oracle_paged_decode_fp8 returned {rc}")
    return out.reshape(S, Hq, D) if pairs is None else out


def kv_append_fp8(k_cache, v_cache, k, v, k_scale, v_scale, slot_mapping, block_size: int, lib=None):
    """Quantizing append on copies of e4m3 pools; returns (k_cache', v_cache') as uint8 codes."""
    kc = _u8(k_cache).copy()
    vc = _u8(v_cache).copy()
    kb, vb = _bits(k), _bits(v)
    ks, vs = _f32(k_scale), _f32(v_scale)
    sm = np.ascontiguousarray(np.asarray(slot_mapping), dtype=np.int64)
    NB, bs, Hkv, D = kc.shape
    assert bs == block_size and kb.shape == (len(sm), Hkv, D) and vb.shape == kb.shape
    rc = (lib or _load()).oracle_kv_append_fp8(_ptr(kc), _ptr(vc), _ptr(kb), _ptr(vb), _ptr(ks), _ptr(vs),
                                               _ptr(sm), len(sm), Hkv, D, block_size, NB)
    if rc != 0:
        raise OracleError(f"oracle_kv_append_fp8 returned {rc}")
    return kc, vc


def decode_step_fp8(batch, pairs: Optional[Sequence[int]] = None, num_threads: int = 0, lib=None):
    """decode_step over a batch whose pools are e4m3 codes (batch.k_scale / v_scale per kv head)."""
    kc, vc = kv_append_fp8(batch.k_cache, batch.v_cache, batch.k_new, batch.v_new, batch.k_scale,
                           batch.v_scale, batch.slot_mapping.numpy(), batch.block_size, lib=lib)
    out = paged_decode_fp8(batch.q, kc, vc, batch.k_scale, batch.v_scale, batch.block_tables.numpy(),
                           batch.context_lens.numpy(), batch.num_kv_heads, batch.block_size, batch.scale,
                           pairs=pairs, num_threads=num_threads, lib=lib)
    return out, kc, vc


def paged_prefill(q, k_cache, v_cache, block_tables, context_lens, query_start, num_kv_heads: int,
                  block_size: int, scale: float, num_threads: int = 0, lib=None) -> np.ndarray:
    """fp64 multi-query paged attention: q bf16 [T][Hq][D] packed by query_start [S+1];
    query i of sequence s attends causally to positions 0 .. L_s - n_s + i. Returns [T][Hq][D]."""
    qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
    T, Hq, D = qb.shape
    NB = kb.shape[0]
    assert kb.shape == (NB, block_size, num_kv_heads, D) and vb.shape == kb.shape
    bt = _i32(block_tables)
    cl = _i32(context_lens)
    qs = _i32(query_start)
    S = cl.shape[0]
    assert qs.shape == (S + 1,) and bt.shape[0] == S
    out = np.zeros((T, Hq, D), dtype=np.float64)
    rc = (lib or _load()).oracle_paged_prefill(
        _ptr(out), _ptr(qb), _ptr(kb), _ptr(vb), _ptr(bt), _ptr(cl), _ptr(qs), S, T, Hq, num_kv_heads, D,
        block_size, bt.shape[1], NB, float(scale), int(num_threads))
    if rc != 0:
        raise OracleError(f"oracle_paged_prefill returned {rc}")
    return out
