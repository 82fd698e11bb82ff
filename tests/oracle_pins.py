"""Pins that tie the fp64 oracle to something other than itself.

Each pin takes an oracle handle (``lib=None`` is the committed oracle) and
raises AssertionError when the oracle disagrees with:
  - torch's scaled_dot_product_attention in fp64 (a library routine) on
    contiguously gathered rows, for small random geometries;
  - closed forms (golden fixtures under tests/golden, context length 1, equal
    keys, zero scale, a saturated softmax, empty context);
  - invariants the pages fix: moving physical blocks, sharing a prefix block
    versus owning a copy, poisoned unused slots (the block table is the only
    way to reach a token), a common key shift, an affine map of the values,
    the logical order of tokens;
  - the append's own round trips (read-back, append then attend, building a
    whole sequence token by token and attending to it).
``tests/test_oracle_mutants.py`` plants mistakes in copies of oracle.c and
checks that at least one pin fails for each.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

import oracle
import workloads
from helpers import (bf16_bits, gather_contiguous, golden_names, load_golden, load_golden_prefill,
                     prefill_golden_names, sdpa_reference)

TIGHT = 1e-12


def _decode(batch, lib, **kw):
    return oracle.paged_decode(batch.q, batch.k_cache, batch.v_cache, batch.block_tables.numpy(),
                               batch.context_lens.numpy(), batch.num_kv_heads, batch.block_size,
                               kw.pop("scale", batch.scale), lib=lib, **kw)


def _close(a, b, tol=TIGHT, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    assert np.isfinite(a).all(), f"{what}: non-finite output"
    err = np.abs(a - b)
    bound = tol * (1.0 + np.abs(b))
    assert (err <= bound).all(), f"{what}: max err {err.max():.3e}"


SMALL_GEOMETRIES = [
    # (Hq, Hkv, D, bs, lens)
    (2, 1, 8, 4, [1, 5, 9, 16]),
    (4, 2, 16, 2, [3, 7]),
    (6, 3, 8, 1, [4, 2]),
    (7, 1, 32, 4, [13, 2, 0]),
    (8, 8, 4, 3, [10]),
    (4, 1, 64, 16, [33, 17]),
]


def _small(i, **kw):
    Hq, Hkv, D, bs, lens = SMALL_GEOMETRIES[i]
    kw.setdefault("with_append", False)
    return workloads.make_custom(100 + i, lens, Hq, Hkv, D, bs, **kw)


def _set_pool_rows(batch, s, fn_k=None, fn_v=None):
    """Rewrite the K/V rows of sequence s through its table: row t := fn(t, old_row)."""
    bs = batch.block_size
    for t in range(int(batch.context_lens[s])):
        p = int(batch.block_tables[s, t // bs])
        if fn_k is not None:
            batch.k_cache[p, t % bs] = fn_k(t, batch.k_cache[p, t % bs])
        if fn_v is not None:
            batch.v_cache[p, t % bs] = fn_v(t, batch.v_cache[p, t % bs])


# ----------------------------------------------------------------------------- library routine

def pin_sdpa_random(lib=None):
    for i in range(len(SMALL_GEOMETRIES)):
        b = _small(i)
        _close(_decode(b, lib), sdpa_reference(b), what=f"sdpa geometry {i}")


# ----------------------------------------------------------------------------- closed forms

def pin_golden(lib=None):
    for name in golden_names():
        b, expected = load_golden(name)
        out = _decode(b, lib)
        for (s, j), row in expected.items():
            _close(out[s, j], row, tol=1e-14, what=f"golden {name} ({s},{j})")


def pin_context_len_one(lib=None):
    b = workloads.make_custom(7, [1] * 6, 8, 2, 64, 16, with_append=False, scale=3.0)
    out = _decode(b, lib)
    G = 4
    for s in range(6):
        p = int(b.block_tables[s, 0])
        for j in range(8):
            v = b.v_cache[p, 0, j // G].double().numpy()
            assert np.array_equal(out[s, j], v), f"context 1 must return v exactly (s={s}, j={j})"


def pin_identical_keys_give_mean(lib=None):
    b = _small(3)
    for s in range(b.num_seqs):
        if int(b.context_lens[s]) == 0:
            continue
        p0 = int(b.block_tables[s, 0])
        k0 = b.k_cache[p0, 0].clone()
        _set_pool_rows(b, s, fn_k=lambda t, old: k0)
    out = _decode(b, lib)
    G = b.num_q_heads // b.num_kv_heads
    for s, (k, v) in enumerate(gather_contiguous(b)):
        L = k.shape[0]
        if L == 0:
            continue
        for j in range(b.num_q_heads):
            mean = np.array([math.fsum(v[:, j // G, d]) / L for d in range(b.head_dim)])
            _close(out[s, j], mean, tol=1e-14, what=f"equal keys (s={s}, j={j})")


def pin_zero_scale_gives_mean(lib=None):
    b = _small(1)
    out = _decode(b, lib, scale=0.0)
    G = b.num_q_heads // b.num_kv_heads
    for s, (k, v) in enumerate(gather_contiguous(b)):
        L = k.shape[0]
        for j in range(b.num_q_heads):
            mean = np.array([math.fsum(v[:, j // G, d]) / L for d in range(b.head_dim)])
            _close(out[s, j], mean, tol=1e-14, what=f"zero scale (s={s}, j={j})")


def pin_saturated_softmax_picks_argmax(lib=None):
    """q = e0 and k_t[0] = distinct integers: with scale 1e4 every weight but the
    largest underflows to exactly 0, so out is that token's v, bit for bit."""
    L = 21
    b = workloads.make_custom(11, [L], 1, 1, 16, 4, with_append=False, scale=1.0e4)
    b.q.zero_()
    b.q[0, 0, 0] = 1.0
    order = np.random.default_rng(3).permutation(L)
    _set_pool_rows(b, 0, fn_k=lambda t, old: torch.cat([torch.tensor([float(order[t])], dtype=torch.bfloat16), old[0, 1:]])[None])
    out = _decode(b, lib)
    t_star = int(np.argmax(order))
    p = int(b.block_tables[0, t_star // 4])
    v = b.v_cache[p, t_star % 4, 0].double().numpy()
    assert np.array_equal(out[0, 0], v), "saturated softmax must return the argmax token's v"


def pin_empty_context_is_zero(lib=None):
    b = workloads.make_custom(12, [0, 5, 0], 4, 2, 16, 4, with_append=False)
    out = _decode(b, lib)
    assert np.array_equal(out[0], np.zeros_like(out[0])) and np.array_equal(out[2], np.zeros_like(out[2]))
    assert np.isfinite(out[1]).all()


# ----------------------------------------------------------------------------- invariants

def pin_block_permutation_invariance(lib=None):
    for i in (0, 3, 5):
        b = _small(i)
        b2 = workloads.permute_pool(b, seed=99)
        assert not np.array_equal(b.block_tables.numpy(), b2.block_tables.numpy())
        assert np.array_equal(_decode(b, lib), _decode(b2, lib)), f"permutation changed output (geometry {i})"


def pin_shared_prefix_equals_private_copies(lib=None):
    b = workloads.make_custom(13, [40, 33, 64, 35], 6, 2, 32, 8, with_append=False, shared_prefix_tokens=32)
    assert int((b.block_tables[:, 0] == b.block_tables[0, 0]).sum()) == 4
    b2 = workloads.unshare_prefix(b)
    assert b2.num_blocks == b.num_blocks + 3 * 4
    assert np.array_equal(_decode(b, lib), _decode(b2, lib)), "shared prefix != private copies"


def pin_poisoned_slots_are_never_read(lib=None):
    for i in (0, 3, 5):
        Hq, Hkv, D, bs, lens = SMALL_GEOMETRIES[i]
        clean = workloads.make_custom(100 + i, lens, Hq, Hkv, D, bs, with_append=False, poison=False)
        dirty = workloads.make_custom(100 + i, lens, Hq, Hkv, D, bs, with_append=False, poison=True)
        assert torch.isnan(dirty.k_cache.float()).any()
        a, c = _decode(clean, lib), _decode(dirty, lib)
        assert np.array_equal(a, c), f"poison reached the output (geometry {i})"


def _eighths(rng, shape, lo, hi):
    return torch.from_numpy(rng.integers(lo * 8, hi * 8 + 1, size=shape) / 8.0).to(torch.bfloat16)


def pin_common_key_shift(lib=None):
    """Adding the same vector u to every key adds scale*q.u to every logit of a
    (sequence, head): the softmax, hence the output, does not change."""
    rng = np.random.default_rng(5)
    b = workloads.make_custom(14, [9, 16, 5], 4, 2, 16, 4, with_append=False, poison=False)
    b.k_cache.copy_(_eighths(rng, b.k_cache.shape, -2, 2))
    u = _eighths(rng, (b.num_kv_heads, b.head_dim), -1, 1)
    b2 = dataclasses.replace(b, k_cache=b.k_cache + u)     # exact in bf16 (multiples of 1/8, |x| <= 3)
    assert torch.equal((b2.k_cache.double() - b.k_cache.double()).to(torch.bfloat16), u.expand_as(b.k_cache))
    _close(_decode(b2, lib), _decode(b, lib), what="key shift")


def pin_value_affine(lib=None):
    """Softmax weights sum to 1: V -> 2V + 1 maps out -> 2 out + 1."""
    rng = np.random.default_rng(6)
    b = workloads.make_custom(15, [7, 12, 1], 6, 3, 8, 4, with_append=False, poison=False)
    b.v_cache.copy_(_eighths(rng, b.v_cache.shape, -4, 4))
    b2 = dataclasses.replace(b, v_cache=(2 * b.v_cache.double() + 1).to(torch.bfloat16))
    _close(_decode(b2, lib), 2 * _decode(b, lib) + 1, what="value affine")


def pin_token_order_invariance(lib=None):
    """Attention over a set of tokens does not depend on their logical order."""
    b = _small(5)
    b2 = b.clone()
    bs = b.block_size
    for s in range(b.num_seqs):
        L = int(b.context_lens[s])
        rows = [(int(b.block_tables[s, t // bs]), t % bs) for t in range(L)]
        ks = [b.k_cache[p, o].clone() for p, o in rows]
        vs = [b.v_cache[p, o].clone() for p, o in rows]
        for t, (p, o) in enumerate(rows):
            b2.k_cache[p, o] = ks[L - 1 - t]
            b2.v_cache[p, o] = vs[L - 1 - t]
    _close(_decode(b2, lib), _decode(b, lib), what="token order")


# ----------------------------------------------------------------------------- append

def pin_append_read_back(lib=None):
    b = workloads.make_custom(16, [5, 9, 16, 2], 4, 2, 32, 8, with_append=False, poison=False)
    NB, bs = b.num_blocks, b.block_size
    rng = np.random.default_rng(8)
    slots = rng.choice(NB * bs, size=4, replace=False).astype(np.int64)
    slots[2] = -1
    kc, vc = oracle.kv_append(b.k_cache, b.v_cache, b.k_new[:4], b.v_new[:4], slots, bs, lib=lib)
    k0, v0 = bf16_bits(b.k_cache), bf16_bits(b.v_cache)
    touched = np.zeros((NB, bs), dtype=bool)
    for i, slot in enumerate(slots):
        if slot < 0:
            continue
        p, o = divmod(int(slot), bs)
        touched[p, o] = True
        assert np.array_equal(kc[p, o], bf16_bits(b.k_new[i])), "appended k not read back"
        assert np.array_equal(vc[p, o], bf16_bits(b.v_new[i])), "appended v not read back"
    assert np.array_equal(kc[~touched], k0[~touched]) and np.array_equal(vc[~touched], v0[~touched]), \
        "append changed a slot it was not given"


def pin_append_then_attend_one_token(lib=None):
    """A sequence of one token, appended this step, attends only to itself: out = v_new."""
    b = workloads.make_custom(17, [1, 1, 1], 8, 4, 16, 4, with_append=True, poison=True)
    out, _, _ = oracle.decode_step(b, lib=lib)
    G = 2
    for s in range(3):
        for j in range(8):
            assert np.array_equal(out[s, j], b.v_new[s, j // G].double().numpy()), "append + attend, context 1"


def pin_append_builds_the_sequence(lib=None):
    """Append L tokens one slot each, in logical order, into an all-NaN pool, then
    attend: the result must equal torch's attention over those L tokens kept
    contiguous (never stored in a pool)."""
    Hq, Hkv, D, bs, L = 4, 2, 16, 4, 11
    gen = torch.Generator().manual_seed(21)
    keys = torch.randn(L, Hkv, D, generator=gen).to(torch.bfloat16)
    vals = torch.randn(L, Hkv, D, generator=gen).to(torch.bfloat16)
    q = torch.randn(1, Hq, D, generator=gen).to(torch.bfloat16)
    NB = 6
    table = np.array([[4, 1, 5]], dtype=np.int32)
    slots = np.array([int(table[0, t // bs]) * bs + t % bs for t in range(L)], dtype=np.int64)
    nan = torch.full((NB, bs, Hkv, D), float("nan")).to(torch.bfloat16)
    kc, vc = oracle.kv_append(nan, nan, keys, vals, slots, bs, lib=lib)
    out = oracle.paged_decode(q, kc, vc, table, np.array([L], dtype=np.int32), Hkv, bs, 0.25, lib=lib)
    G = Hq // Hkv
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double()[:, :, None, :], keys.double().permute(1, 0, 2).repeat_interleave(G, 0)[None],
        vals.double().permute(1, 0, 2).repeat_interleave(G, 0)[None], scale=0.25)[0, :, 0, :]
    _close(out[0], ref.numpy(), what="append builds the sequence")


def pin_append_duplicate_slot_last_wins(lib=None):
    b = workloads.make_custom(18, [3], 2, 1, 8, 4, with_append=False, poison=False)
    k = torch.stack([b.k_new[0], -b.k_new[0]])
    v = torch.stack([b.v_new[0], 2 * b.v_new[0]])
    kc, vc = oracle.kv_append(b.k_cache, b.v_cache, k, v, np.array([5, 5], dtype=np.int64), 4, lib=lib)
    assert np.array_equal(kc[1, 1], bf16_bits(k[1])) and np.array_equal(vc[1, 1], bf16_bits(v[1]))


# ---------------------------------------------------------------- fp8 (e4m3) cache

_E4M3 = torch.float8_e4m3fn


def pin_e4m3_decode_table(lib=None):
    """Every code's value equals torch's float8_e4m3fn value (a library special case)."""
    codes = np.arange(256, dtype=np.uint8)
    mine = oracle.e4m3_to_double(codes, lib=lib)
    ref = torch.from_numpy(codes).view(_E4M3).double().numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(mine[ok], ref[ok])


def _e4m3_samples():
    rng = np.random.default_rng(7)
    x = rng.standard_normal(4000) * np.exp(rng.uniform(-14, 6.2, 4000))
    finite = torch.arange(256, dtype=torch.uint8).view(_E4M3).double().numpy()
    finite = np.unique(finite[np.isfinite(finite)])
    mids = (finite[1:] + finite[:-1]) / 2       # exact ties between neighbouring codes
    x = np.concatenate([x, mids, -mids, finite, [0.0, -0.0]]).astype(np.float32)
    return x[np.abs(x) <= 448]


def pin_e4m3_encode_matches_torch(lib=None):
    """In range, the encode is torch's round-to-nearest-even cast, ties included."""
    x = _e4m3_samples()
    mine = oracle.e4m3_from_float(x, lib=lib)
    ref = torch.from_numpy(x).to(_E4M3).view(torch.uint8).numpy()
    assert np.array_equal(mine, ref)


def pin_e4m3_encode_is_nearest(lib=None):
    """Brute force over all finite codes: the chosen code is a nearest one, and of two
    nearest ones the one with an even mantissa field."""
    x = _e4m3_samples()[::7]
    codes = np.array([c for c in range(256) if (c & 0x7f) != 0x7f], dtype=np.uint8)
    vals = torch.from_numpy(codes).view(_E4M3).double().numpy()
    mine = oracle.e4m3_from_float(x, lib=lib)
    for xi, ci in zip(x.astype(np.float64), mine):
        d = np.abs(vals - xi)
        best = codes[d == d.min()]
        best_vals = set(torch.from_numpy(best).view(_E4M3).double().numpy().tolist())
        got = float(torch.tensor([ci], dtype=torch.uint8).view(_E4M3).double())
        assert got in best_vals, (xi, ci)
        if len(best_vals) > 1:
            assert ci & 1 == 0, (xi, ci)


def pin_e4m3_saturates(lib=None):
    big = np.array([448.0, 449.0, 463.9, 464.0, 470.0, 479.0, 500.0, 1e6, np.inf], dtype=np.float32)
    assert (oracle.e4m3_from_float(big, lib=lib) == 0x7E).all()
    assert (oracle.e4m3_from_float(-big, lib=lib) == 0xFE).all()
    assert (oracle.e4m3_from_float(np.array([np.nan], np.float32), lib=lib) & 0x7F == 0x7F).all()


def _fp8_batch(i, **kw):
    Hq, Hkv, D, bs, lens = SMALL_GEOMETRIES[i]
    return workloads.make_custom(400 + i, lens, Hq, Hkv, D, bs, kv_dtype="fp8", **kw)


def _dequantized(b, kc, vc):
    k = torch.from_numpy(np.asarray(kc)).view(_E4M3).double() * b.k_scale.double()[None, None, :, None]
    v = torch.from_numpy(np.asarray(vc)).view(_E4M3).double() * b.v_scale.double()[None, None, :, None]
    return k, v


def pin_fp8_decode_equals_dequantized_sdpa(lib=None):
    """Attention over the dequantized cache, by torch SDPA in fp64 on gathered rows."""
    for i in range(len(SMALL_GEOMETRIES)):
        b = _fp8_batch(i, with_append=False)
        got = oracle.paged_decode_fp8(b.q, b.k_cache, b.v_cache, b.k_scale, b.v_scale, b.block_tables.numpy(),
                                      b.context_lens.numpy(), b.num_kv_heads, b.block_size, b.scale, lib=lib)
        k, v = _dequantized(b, b.k_cache.numpy(), b.v_cache.numpy())
        _close(got, sdpa_reference(b, k, v), what=f"fp8 geometry {i}")


def pin_fp8_append_matches_torch_quantization(lib=None):
    """The append's codes are torch's cast of the fp32 quotient x / scale[h]."""
    for i in (1, 4, 5):  # 2, 8 and 1 kv heads (K and V scales differ past head 0)
        b = _fp8_batch(i, poison=False)
        kc, vc = oracle.kv_append_fp8(b.k_cache, b.v_cache, b.k_new, b.v_new, b.k_scale, b.v_scale,
                                      b.slot_mapping.numpy(), b.block_size, lib=lib)
        bs = b.block_size
        for t, slot in enumerate(b.slot_mapping.tolist()):
            if slot < 0:
                continue
            kq = (b.k_new[t].float() / b.k_scale[:, None]).to(_E4M3).view(torch.uint8).numpy()
            vq = (b.v_new[t].float() / b.v_scale[:, None]).to(_E4M3).view(torch.uint8).numpy()
            assert np.array_equal(kc[slot // bs, slot % bs], kq) and np.array_equal(vc[slot // bs, slot % bs], vq)


def pin_fp8_scales_act_as_the_pages_define(lib=None):
    """A K scale factor c is a softmax scale factor c; a V scale factor c scales the output."""
    b = _fp8_batch(1, with_append=False)
    args = (b.block_tables.numpy(), b.context_lens.numpy(), b.num_kv_heads, b.block_size)
    base = oracle.paged_decode_fp8(b.q, b.k_cache, b.v_cache, b.k_scale, b.v_scale, *args, b.scale, lib=lib)
    twice_k = oracle.paged_decode_fp8(b.q, b.k_cache, b.v_cache, b.k_scale * 2, b.v_scale, *args, b.scale, lib=lib)
    twice_s = oracle.paged_decode_fp8(b.q, b.k_cache, b.v_cache, b.k_scale, b.v_scale, *args, 2 * b.scale, lib=lib)
    _close(twice_k, twice_s, what="K scale vs softmax scale")
    half_v = oracle.paged_decode_fp8(b.q, b.k_cache, b.v_cache, b.k_scale, b.v_scale / 2, *args, b.scale, lib=lib)
    _close(half_v, base / 2, what="V scale")


def pin_fp8_poisoned_slots_are_never_read(lib=None):
    b = _fp8_batch(3, with_append=False)   # NaN codes in every slot no table reaches
    got = oracle.paged_decode_fp8(b.q, b.k_cache, b.v_cache, b.k_scale, b.v_scale, b.block_tables.numpy(),
                                  b.context_lens.numpy(), b.num_kv_heads, b.block_size, b.scale, lib=lib)
    assert np.isfinite(got).all()


# ---------------------------------------------------------------- multi-query (chunked prefill)

PREFILL_CASES = [
    # (chunk_lens, context_lens, Hq, Hkv, D, bs)
    ([3, 1, 0, 20], [10, 5, 7, 40], 4, 2, 16, 4),
    ([8, 8], [8, 33], 2, 1, 32, 8),
    ([5, 2, 9], [5, 17, 60], 6, 3, 8, 16),
]


def _prefill(b, lib, **kw):
    return oracle.paged_prefill(b.q, b.k_cache, b.v_cache, b.block_tables.numpy(), b.context_lens.numpy(),
                                b.query_start.numpy(), b.num_kv_heads, b.block_size, kw.get("scale", b.scale),
                                lib=lib)


def pin_prefill_causal_sdpa(lib=None):
    """torch SDPA in fp64 on gathered rows with the causal mask of a chunk at the end of its context."""
    for i, (n, L, Hq, Hkv, D, bs) in enumerate(PREFILL_CASES):
        b = workloads.make_prefill(500 + i, n, L, Hq, Hkv, D, bs)
        got = _prefill(b, lib)
        G = Hq // Hkv
        qs = b.query_start.numpy()
        for s, (k, v) in enumerate(gather_contiguous(b)):
            ns = int(qs[s + 1] - qs[s])
            if ns == 0:
                continue
            Ls = k.shape[0]
            kt = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(G, dim=0)[None]
            vt = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(G, dim=0)[None]
            qt = b.q[qs[s]:qs[s + 1]].double().permute(1, 0, 2)[None]                  # [1][Hq][n][D]
            allowed = torch.arange(Ls)[None, :] <= (Ls - ns + torch.arange(ns))[:, None]
            ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=allowed, scale=b.scale)
            _close(got[qs[s]:qs[s + 1]], ref[0].permute(1, 0, 2).numpy(), what=f"prefill case {i} seq {s}")


def pin_prefill_golden(lib=None):
    """Worked multi-query examples with exact expected rows (tests/golden/prefill)."""
    names = prefill_golden_names()
    assert names, "no multi-query golden fixtures"
    for name in names:
        b, expected = load_golden_prefill(name)
        got = _prefill(b, lib)
        for (r, j), row in expected.items():
            _close(got[r, j], row, tol=1e-14, what=f"prefill golden {name} ({r},{j})")


def pin_prefill_single_queries_are_decodes(lib=None):
    """Chunks of one token are decode steps over the whole context."""
    L = [9, 1, 30, 17]
    b = workloads.make_prefill(510, [1] * len(L), L, 4, 2, 16, 4)
    got = _prefill(b, lib)
    dec = oracle.paged_decode(b.q, b.k_cache, b.v_cache, b.block_tables.numpy(), b.context_lens.numpy(),
                              b.num_kv_heads, b.block_size, b.scale, lib=lib)
    _close(got, dec, what="n = 1")


def pin_prefill_equal_keys_give_prefix_means(lib=None):
    """All keys equal: query i of a chunk gets the mean of V over positions 0 .. p_i."""
    b = workloads.make_prefill(520, [6, 3], [6, 12], 2, 1, 8, 4, poison=False)
    kc = b.k_cache.clone()
    kc[:] = kc[0, 0, 0]
    b = dataclasses.replace(b, k_cache=kc)
    got = _prefill(b, lib)
    qs = b.query_start.numpy()
    for s, (_, v) in enumerate(gather_contiguous(b)):
        ns = int(qs[s + 1] - qs[s])
        Ls = v.shape[0]
        for i in range(ns):
            p = Ls - ns + i
            _close(got[qs[s] + i], np.repeat(v[:p + 1].mean(axis=0), b.num_q_heads // b.num_kv_heads, axis=0),
                   what=f"equal keys seq {s} query {i}")


def pin_prefill_block_permutation_invariance(lib=None):
    n, L, Hq, Hkv, D, bs = PREFILL_CASES[0]
    b = workloads.make_prefill(530, n, L, Hq, Hkv, D, bs)
    pb = workloads.permute_pool(b, seed=5)
    pb = dataclasses.replace(b, k_cache=pb.k_cache, v_cache=pb.v_cache, block_tables=pb.block_tables)
    _close(_prefill(pb, lib), _prefill(b, lib), what="prefill permutation")


ALL_PINS = [
    pin_sdpa_random,
    pin_golden,
    pin_context_len_one,
    pin_identical_keys_give_mean,
    pin_zero_scale_gives_mean,
    pin_saturated_softmax_picks_argmax,
    pin_empty_context_is_zero,
    pin_block_permutation_invariance,
    pin_shared_prefix_equals_private_copies,
    pin_poisoned_slots_are_never_read,
    pin_common_key_shift,
    pin_value_affine,
    pin_token_order_invariance,
    pin_append_read_back,
    pin_append_then_attend_one_token,
    pin_append_builds_the_sequence,
    pin_append_duplicate_slot_last_wins,
    pin_e4m3_decode_table,
    pin_e4m3_encode_matches_torch,
    pin_e4m3_encode_is_nearest,
    pin_e4m3_saturates,
    pin_fp8_decode_equals_dequantized_sdpa,
    pin_fp8_append_matches_torch_quantization,
    pin_fp8_scales_act_as_the_pages_define,
    pin_fp8_poisoned_slots_are_never_read,
    pin_prefill_causal_sdpa,
    pin_prefill_golden,
    pin_prefill_single_queries_are_decodes,
    pin_prefill_equal_keys_give_prefix_means,
    pin_prefill_block_permutation_invariance,
]
