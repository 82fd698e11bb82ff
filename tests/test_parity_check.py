"""The parity check itself must see a lost context piece (CPU only).

On a 65,536-token context most output elements are smaller than the
elementwise bound's absolute term (8e-3), so an output that lost a piece of
the context -- what a split-context merge that drops or mis-weights one CTA's
partial would produce -- can pass the elementwise bound. The per-row
normalised bounds (relative L2 error, max|err| / rms) must fail it. Both the
wrong and the right outputs here come from the oracle, rounded to bf16 as the
CUDA path's output is: this tests the check, not the kernel.

The sequence has the geometry of the 64K-token sequence of the skewed
long-context workload (32 q / 8 kv heads, head_dim 128, block_size 32); 2,208
tokens is about what one CTA of the default 592-CTA grid takes of that batch.
"""
import functools

import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import ATOL, RTOL, assert_close_to_oracle, row_errors


@functools.lru_cache(maxsize=None)
def long_sequence():
    b = workloads.make_batch("skewed_long", lens_override=[65536], poison=False)
    full, kc, vc = oracle.decode_step(b)
    return b, full, kc, vc


def bf16_round(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x).to(torch.bfloat16).double().numpy()


def truncated(drop: int) -> np.ndarray:
    """The oracle's output when the last `drop` tokens of the context are left out."""
    b, _, kc, vc = long_sequence()
    lens = b.context_lens.numpy() - drop
    return oracle.paged_decode(b.q, kc, vc, b.block_tables.numpy(), lens, b.num_kv_heads, b.block_size, b.scale)


def leading_piece_dropped(drop: int) -> np.ndarray:
    """The oracle's output when the FIRST `drop` tokens are left out (a table that
    starts `drop` tokens later: drop must be a multiple of the block size)."""
    b, _, kc, vc = long_sequence()
    bs = b.block_size
    assert drop % bs == 0
    tables = b.block_tables.numpy().copy()
    tables[0, :-(drop // bs)] = tables[0, drop // bs:]
    lens = b.context_lens.numpy() - drop
    return oracle.paged_decode(b.q, kc, vc, tables, lens, b.num_kv_heads, b.block_size, b.scale)


def test_the_exact_result_rounded_to_bf16_passes():
    _, full, _, _ = long_sequence()
    assert_close_to_oracle(bf16_round(full), full, what="bf16 of the oracle itself")


@pytest.mark.parametrize("drop", [2208, 512])
@pytest.mark.parametrize("where", ["last", "first"])
def test_a_lost_context_piece_fails(drop, where):
    _, full, _, _ = long_sequence()
    got = bf16_round(truncated(drop) if where == "last" else leading_piece_dropped(drop // 32 * 32))
    # the elementwise bound alone lets the whole output through ...
    assert (np.abs(got - full) <= ATOL + RTOL * np.abs(full)).all()
    # ... the normalised bounds do not
    rel, _ = row_errors(got, full)
    assert (rel > 1e-2).all()
    with pytest.raises(AssertionError, match="relative L2"):
        assert_close_to_oracle(got, full, what=f"{drop} tokens lost at the {where} end")


def test_a_mis_weighted_merge_fails():
    """The whole context's output blended 9:1 with its first half's: what a merge
    that gives the first half's partial too much weight produces."""
    b, full, kc, vc = long_sequence()
    half = b.context_lens.numpy() // 2
    first = oracle.paged_decode(b.q, kc, vc, b.block_tables.numpy(), half, b.num_kv_heads, b.block_size, b.scale)
    got = bf16_round(0.9 * full + 0.1 * first)
    assert (np.abs(got - full) <= ATOL + RTOL * np.abs(full)).all()  # inside the elementwise bound
    with pytest.raises(AssertionError, match="relative L2"):
        assert_close_to_oracle(got, full, what="first half over-weighted")
