"""Shared test helpers: golden-fixture loading, contiguous gathers, tolerances.

Nothing here computes paged attention: the references the tests compare with
are the fp64 oracle, torch's own scaled_dot_product_attention (a library
routine) and closed forms.
"""
from __future__ import annotations

import glob
import json
import math
import os
from fractions import Fraction
from typing import Dict, List

import numpy as np
import torch

import workloads

GOLDEN_DIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

# bf16 output against the fp64 oracle: |gpu - ref| <= ATOL + RTOL * |ref|, elementwise.
ATOL = 8e-3
RTOL = 8e-3


def golden_names() -> List[str]:
    return sorted(os.path.basename(p)[:-5] for p in glob.glob(os.path.join(GOLDEN_DIR, "*.json")))


def _key(s: str):
    return tuple(int(x) for x in s.split(","))


def load_golden(name: str):
    """A golden fixture as a DecodeBatch with no append, plus its exact expected rows.

    Pool slots the fixture does not name hold NaN; query entries it does not name
    are 0; vectors are padded with zeros to head_dim.
    """
    with open(os.path.join(GOLDEN_DIR, name + ".json")) as f:
        fx = json.load(f)
    Hq, Hkv, D, bs, NB = fx["num_q_heads"], fx["num_kv_heads"], fx["head_dim"], fx["block_size"], fx["num_blocks"]
    tables = np.asarray(fx["block_tables"], dtype=np.int32)
    lens = np.asarray(fx["context_lens"], dtype=np.int32)
    S = len(lens)
    sc = fx["scale"]
    scale = math.log(sc["ln"]) if "ln" in sc else float(sc["value"])
    q = torch.zeros(S, Hq, D, dtype=torch.float32)
    for k, vals in fx["q"].items():
        s, j = _key(k)
        q[s, j, :len(vals)] = torch.tensor(vals, dtype=torch.float32)
    kc = torch.full((NB, bs, Hkv, D), float("nan"), dtype=torch.float32)
    vc = torch.full((NB, bs, Hkv, D), float("nan"), dtype=torch.float32)
    for name_, cache in (("k", kc), ("v", vc)):
        for k, vals in fx[name_].items():
            p, off, h = _key(k)
            cache[p, off, h, :] = 0.0
            cache[p, off, h, :len(vals)] = torch.tensor(vals, dtype=torch.float32)
    for t in (q, kc, vc):
        assert torch.equal(t.to(torch.bfloat16).float().nan_to_num(7.0), t.nan_to_num(7.0)), "fixture values must be bf16-exact"
    batch = workloads.DecodeBatch(
        name=name, seed=0, num_seqs=S, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D, block_size=bs,
        scale=scale, max_blocks_per_seq=tables.shape[1], num_blocks=NB,
        context_lens=torch.from_numpy(lens), block_tables=torch.from_numpy(tables),
        slot_mapping=torch.full((S,), -1, dtype=torch.int64),
        q=q.to(torch.bfloat16), k_cache=kc.to(torch.bfloat16), v_cache=vc.to(torch.bfloat16),
        k_new=torch.zeros(S, Hkv, D, dtype=torch.bfloat16), v_new=torch.zeros(S, Hkv, D, dtype=torch.bfloat16),
    )
    expected: Dict[tuple, np.ndarray] = {}
    for k, vals in fx["expected"].items():
        row = np.zeros(D, dtype=np.float64)
        row[:len(vals)] = [float(Fraction(v)) for v in vals]
        expected[_key(k)] = row
    return batch, expected


def prefill_golden_names() -> List[str]:
    return sorted(os.path.basename(p)[:-5] for p in glob.glob(os.path.join(GOLDEN_DIR, "prefill", "*.json")))


def load_golden_prefill(name: str):
    """A multi-query golden fixture as a PrefillBatch, plus its exact expected rows
    keyed by (query token row, q head). Query rows are keyed by token row; pool
    slots the fixture does not name hold NaN; vectors are padded with zeros."""
    with open(os.path.join(GOLDEN_DIR, "prefill", name + ".json")) as f:
        fx = json.load(f)
    Hq, Hkv, D, bs, NB = fx["num_q_heads"], fx["num_kv_heads"], fx["head_dim"], fx["block_size"], fx["num_blocks"]
    tables = np.asarray(fx["block_tables"], dtype=np.int32)
    lens = np.asarray(fx["context_lens"], dtype=np.int32)
    qs = np.asarray(fx["query_start"], dtype=np.int32)
    S, T = len(lens), int(qs[-1])
    sc = fx["scale"]
    scale = math.log(sc["ln"]) if "ln" in sc else float(sc["value"])
    q = torch.zeros(T, Hq, D, dtype=torch.float32)
    for k, vals in fx["q"].items():
        r, j = _key(k)
        q[r, j, :len(vals)] = torch.tensor(vals, dtype=torch.float32)
    kc = torch.full((NB, bs, Hkv, D), float("nan"), dtype=torch.float32)
    vc = torch.full((NB, bs, Hkv, D), float("nan"), dtype=torch.float32)
    for name_, cache in (("k", kc), ("v", vc)):
        for k, vals in fx[name_].items():
            p, off, h = _key(k)
            cache[p, off, h, :] = 0.0
            cache[p, off, h, :len(vals)] = torch.tensor(vals, dtype=torch.float32)
    for t in (q, kc, vc):
        assert torch.equal(t.to(torch.bfloat16).float().nan_to_num(7.0), t.nan_to_num(7.0)), "fixture values must be bf16-exact"
    batch = workloads.PrefillBatch(
        name=name, seed=0, num_seqs=S, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D, block_size=bs,
        scale=scale, max_blocks_per_seq=tables.shape[1], num_blocks=NB,
        context_lens=torch.from_numpy(lens), block_tables=torch.from_numpy(tables),
        slot_mapping=torch.full((T,), -1, dtype=torch.int64),
        q=q.to(torch.bfloat16), k_cache=kc.to(torch.bfloat16), v_cache=vc.to(torch.bfloat16),
        k_new=torch.zeros(T, Hkv, D, dtype=torch.bfloat16), v_new=torch.zeros(T, Hkv, D, dtype=torch.bfloat16),
        query_start=torch.from_numpy(qs),
    )
    expected: Dict[tuple, np.ndarray] = {}
    for k, vals in fx["expected"].items():
        row = np.zeros(D, dtype=np.float64)
        row[:len(vals)] = [float(Fraction(v)) for v in vals]
        expected[_key(k)] = row
    return batch, expected


def gather_contiguous(batch, k_cache=None, v_cache=None):
    """Per sequence, the K and V rows in logical order, as fp64 [L][Hkv][D] arrays.

    This is the block-table lookup itself (logical block t // bs is physical block
    table[t // bs]; offset t % bs), done with numpy fancy indexing.
    """
    kc = (batch.k_cache if k_cache is None else k_cache)
    vc = (batch.v_cache if v_cache is None else v_cache)
    kc = _as_f64(kc)
    vc = _as_f64(vc)
    bs = batch.block_size
    out = []
    for s in range(batch.num_seqs):
        L = int(batch.context_lens[s])
        t = np.arange(L)
        phys = batch.block_tables.numpy()[s, t // bs].astype(np.int64)
        out.append((kc[phys, t % bs], vc[phys, t % bs]))
    return out


def _as_f64(a) -> np.ndarray:
    if isinstance(a, np.ndarray):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).double().numpy()
        return a.astype(np.float64)
    return a.detach().cpu().double().numpy()


def sdpa_reference(batch, k_cache=None, v_cache=None) -> np.ndarray:
    """torch.nn.functional.scaled_dot_product_attention in fp64 on the gathered rows.

    torch defines grouped-query attention by repeat_interleave of the kv heads
    (kv head h serves query heads h*G .. h*G + G - 1).
    """
    G = batch.num_q_heads // batch.num_kv_heads
    q = batch.q.double()
    out = np.zeros((batch.num_seqs, batch.num_q_heads, batch.head_dim))
    for s, (k, v) in enumerate(gather_contiguous(batch, k_cache, v_cache)):
        if k.shape[0] == 0:
            continue
        kt = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(G, dim=0)[None]  # [1][Hq][L][D]
        vt = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(G, dim=0)[None]
        qt = q[s][None, :, None, :]                                                 # [1][Hq][1][D]
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=batch.scale)
        out[s] = o[0, :, 0, :].numpy()
    return out


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


# Normalised per-row bounds, applied next to the elementwise one. A row is one
# output vector (the last axis: one query token and q head). On long contexts
# |ref| shrinks like 1/sqrt(L) (about 4e-3 at 64K tokens), so the elementwise
# bound's absolute term is wider than the values themselves and a lost or
# mis-weighted context piece would hide inside it; these two do not scale with
# |ref|. Paging changes where K/V live, not what attention computes ("vLLM
# Fundamentals: Paged Attention and Batching", section "Paged Attention"), so the
# paged result must be the plain one up to the arithmetic's rounding: bf16
# output rounding alone gives a relative error up to 2^-9 per element, the
# probabilities' bf16 (or f16) rounding about as much again.
REL_L2 = 1e-2        # ||got - ref||_2 / ||ref||_2 per row
MAX_OVER_RMS = 4e-2  # max|got - ref| / rms(ref) per row

# Largest normalised errors seen, per call (written out when PKV_PARITY_LOG names a file).
PARITY_LOG: List[dict] = []


def row_errors(got: np.ndarray, ref: np.ndarray):
    """Per row (last axis): relative L2 error and max|err| / rms(ref); rows with
    ref == 0 everywhere give 0 (the elementwise bound covers them)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    n = ref.shape[-1] if ref.ndim else 1
    g2 = got.reshape(-1, n)
    r2 = ref.reshape(-1, n)
    err = g2 - r2
    rnorm = np.sqrt((r2 * r2).sum(axis=1))
    live = rnorm > 0
    rel = np.zeros(len(r2))
    mor = np.zeros(len(r2))
    rel[live] = np.sqrt((err[live] ** 2).sum(axis=1)) / rnorm[live]
    mor[live] = np.abs(err[live]).max(axis=1) / (rnorm[live] / np.sqrt(n))
    return rel, mor


def assert_close_to_oracle(got: np.ndarray, ref: np.ndarray, atol: float = ATOL, rtol: float = RTOL, what: str = "",
                           normalised: bool = True):
    """Elementwise |got - ref| <= atol + rtol*|ref|; NaN anywhere fails. With
    ``normalised`` (the default), every row must also meet REL_L2 and MAX_OVER_RMS."""
    got = np.asarray(got, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert not np.isnan(got).any(), f"{what}: NaN in output"
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements out of tolerance; max err {err.max():.3e}; "
            f"first {idx.tolist()} got {got[tuple(idx[0])]} ref {ref[tuple(idx[0])]}")
    if not normalised or got.size == 0:
        return
    rel, mor = row_errors(got, ref)
    PARITY_LOG.append({"what": what, "rows": int(len(rel)), "rel_l2_max": float(rel.max()),
                       "max_over_rms_max": float(mor.max())})
    if (rel > REL_L2).any() or (mor > MAX_OVER_RMS).any():
        r = int(np.argmax(np.maximum(rel / REL_L2, mor / MAX_OVER_RMS)))
        raise AssertionError(
            f"{what}: {int((rel > REL_L2).sum())} rows above relative L2 {REL_L2} and {int((mor > MAX_OVER_RMS).sum())} "
            f"above max|err|/rms {MAX_OVER_RMS} (of {len(rel)}); worst row {r}: relative L2 {rel[r]:.3e}, "
            f"max|err|/rms {mor[r]:.3e}")
