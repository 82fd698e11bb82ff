"""Decode with prefix groups: sequences that share their leading physical blocks
("Deep Dive into vLLM", section 2.2, Flexible Sharing; runbyai post 449,
section 3) have those blocks read once per group by prefix units, and merged
with each sequence's own blocks by the log-sum-exp identity. The result is the
same attention: every case is checked against the fp64 oracle (pools bit-exact
after the fused append, outputs within the bf16 tolerance).
"""
import functools

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_377_b200 as pkv
import workloads
from helpers import assert_close_to_oracle, bf16_bits

pytestmark = pytest.mark.gpu

DEV = "cuda"


def fused(b, groups, **opts):
    """The one-launch step (append + decode) with prefix groups; host copies back."""
    kc = b.k_cache.to(DEV, copy=True)
    vc = b.v_cache.to(DEV, copy=True)
    q = b.q.to(DEV)
    ws = pkv.allocate_workspace(b.num_seqs, b.num_q_heads, b.head_dim)
    out = torch.full_like(q, float("nan"))
    pkv.paged_attn_decode_append(out, q, b.k_new.to(DEV), b.v_new.to(DEV), b.slot_mapping.to(DEV), kc, vc,
                                 b.block_tables.to(DEV), b.context_lens.to(DEV), b.scale, ws, prefix_groups=groups,
                                 **opts)
    torch.cuda.synchronize()
    return out.cpu(), bf16_bits(kc), bf16_bits(vc), pkv.read_status(ws)


def two_launch(b, groups, **opts):
    kc = b.k_cache.to(DEV, copy=True)
    vc = b.v_cache.to(DEV, copy=True)
    q = b.q.to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.kv_cache_append(b.k_new.to(DEV), b.v_new.to(DEV), kc, vc, b.slot_mapping.to(DEV), status)
    ws = pkv.allocate_workspace(b.num_seqs, b.num_q_heads, b.head_dim)
    out = torch.full_like(q, float("nan"))
    pkv.paged_attn_decode(out, q, kc, vc, b.block_tables.to(DEV), b.context_lens.to(DEV), b.scale, ws,
                          prefix_groups=groups, **opts)
    torch.cuda.synchronize()
    return out.cpu(), bf16_bits(kc), bf16_bits(vc), pkv.read_status(ws) | pkv.read_status(status)


@functools.lru_cache(maxsize=None)
def qwen_case():
    b = workloads.make_batch("qwen25_7b_prefix")
    ref, kc_ref, vc_ref = oracle.decode_step(b)
    groups = pkv.find_prefix_groups(b.block_tables, b.context_lens, b.block_size)
    return b, groups, ref, kc_ref, vc_ref


def share_runs(b, runs):
    """Rewrite a batch's tables so that each run (begin, end, P) of sequences
    shares its first sequence's first P blocks. Members whose context ends
    inside the shared blocks take no append (their last position is shared)."""
    bt = b.block_tables.clone()
    slots = b.slot_mapping.clone()
    lens = b.context_lens
    for lo, hi, P in runs:
        for s in range(lo + 1, hi):
            bt[s, :P] = bt[lo, :P]
        for s in range(lo, hi):
            if int(lens[s]) <= P * b.block_size:
                slots[s] = -1
    return workloads.DecodeBatch(**{**b.__dict__, "block_tables": bt, "slot_mapping": slots})


def test_qwen_shared_prefix_batch_matches_the_oracle():
    b, groups, ref, kc_ref, vc_ref = qwen_case()
    assert len(groups) == 1 and groups.begin[0] == 0 and groups.end[0] == 64 and groups.blocks[0] == 64
    out, kc, vc, st = fused(b, groups)
    assert st == 0, st
    assert np.array_equal(kc, kc_ref) and np.array_equal(vc, vc_ref)
    assert_close_to_oracle(out.double().numpy(), ref, what="qwen, prefix groups")
    out2, kc2, vc2, st2 = two_launch(b, groups)
    assert st2 == 0
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16)), "one launch and two launches differ"


@pytest.mark.parametrize("opts", [dict(num_ctas=1024), dict(num_ctas=300), dict(num_ctas=150), dict(num_ctas=5),
                                  dict(num_stages=2), dict(piece_cost=-1), dict(math=2)])
def test_qwen_prefix_groups_under_launch_options(opts):
    b, groups, ref, _, _ = qwen_case()
    out, _, _, st = fused(b, groups, **opts)
    assert st == 0
    assert_close_to_oracle(out.double().numpy(), ref, what=f"qwen, prefix groups {opts}")


def test_prefix_groups_are_invariant_to_block_placement_bitwise():
    b, groups, _, _, _ = qwen_case()
    out1, _, _, _ = fused(b, groups)
    p = workloads.permute_pool(b, seed=5)
    out2, _, _, _ = fused(p, pkv.find_prefix_groups(p.block_tables, p.context_lens, p.block_size))
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


@pytest.mark.parametrize("G", [1, 2, 4, 7, 8])
@pytest.mark.parametrize("D,bs", [(64, 16), (128, 16), (128, 32), (64, 32)])
def test_mixed_groups_short_members_and_ungrouped_sequences(G, D, bs):
    """Three groups (one spanning more than one row tile), members whose context
    ends inside the shared blocks or is empty, ungrouped sequences between."""
    P = 5 if bs == 16 else 3
    T = P * bs
    rng = np.random.default_rng(G * 100 + D + bs)
    lens = ([T + 40, T + 1, T - 3, 0, T + 200, T, 7] +                       # group 0: seqs 0-6
            [int(x) for x in rng.integers(1, 300, 3)] +                        # ungrouped 7-9
            [T + int(x) for x in rng.integers(1, 400, 70)] +                   # group 1: seqs 10-79 (many rows)
            [int(x) for x in rng.integers(1, 300, 2)] +                        # ungrouped 80-81
            [T + 2, T + 17])                                                    # group 2: seqs 82-83
    b = workloads.make_custom(7000 + G + D + bs, lens, 2 * G, 2, D, bs, max_context=T + 450)
    runs = [(0, 7, P), (10, 80, P), (82, 84, P)]
    b = share_runs(b, runs)
    ref, kc_ref, vc_ref = oracle.decode_step(b)
    groups = pkv.PrefixGroups([r[0] for r in runs], [r[1] for r in runs], [r[2] for r in runs])
    found = pkv.find_prefix_groups(b.block_tables, b.context_lens, bs, min_blocks=P)
    for num_ctas in (0, 97):
        out, kc, vc, st = fused(b, groups, num_ctas=num_ctas)
        assert st == 0, st
        assert np.array_equal(kc, kc_ref) and np.array_equal(vc, vc_ref)
        assert_close_to_oracle(out.double().numpy(), ref, what=f"G={G} D={D} bs={bs} C={num_ctas}")
    out, _, _, st = fused(b, found)
    assert st == 0
    assert_close_to_oracle(out.double().numpy(), ref, what=f"found groups {found}")


def test_a_member_whose_table_differs_is_flagged():
    b, groups, _, _, _ = qwen_case()
    bt = b.block_tables.clone()
    bt[5, 3] = bt[5, 70] if bt[5, 70] >= 0 else bt[6, 64]   # member 5 no longer shares block 3
    bad = workloads.DecodeBatch(**{**b.__dict__, "block_tables": bt})
    _, _, _, st = fused(bad, groups)
    assert st & pkv.PKV_STATUS_BAD_PREFIX_GROUP


def test_an_append_inside_the_shared_blocks_is_flagged():
    b = workloads.make_custom(91, [100, 60, 90], 8, 2, 128, 16)
    b = share_runs(b, [(0, 3, 4)])
    slots = b.slot_mapping.clone()
    slots[1] = int(b.block_tables[1, 3]) * 16 + 11         # position 59 lies in shared block 3
    bad = workloads.DecodeBatch(**{**b.__dict__, "slot_mapping": slots})
    _, _, _, st = fused(bad, pkv.PrefixGroups([0], [3], [4]))
    assert st & pkv.PKV_STATUS_BAD_SLOT


def test_groups_are_refused_where_they_cannot_apply():
    b, groups, _, _, _ = qwen_case()
    with pytest.raises(pkv.PagedKVError, match="tensor cores"):
        fused(b, groups, math=1)
    with pytest.raises(pkv.PagedKVError, match="two or more members"):
        fused(b, pkv.PrefixGroups([0], [1], [3]))


@pytest.mark.parametrize("grouped", [True, False])
def test_long_shared_prefix_sampled_rows(grouped):
    """32 sequences sharing a 32768-token prompt (its K/V larger than L2), checked
    on sampled rows against the oracle, with and without the grouping."""
    b = workloads.make_batch("shared_long_prefix", device=DEV).to("cpu")
    groups = pkv.find_prefix_groups(b.block_tables, b.context_lens, b.block_size) if grouped else None
    if grouped:
        assert len(groups) == 1 and groups.blocks[0] == 2048
    pairs = list(range(0, b.num_seqs * b.num_q_heads, 13))
    ref, kc_ref, vc_ref = oracle.decode_step(b, pairs=pairs)
    out, kc, vc, st = fused(b, groups)
    assert st == 0, st
    assert np.array_equal(kc, kc_ref) and np.array_equal(vc, vc_ref)
    got = out.double().numpy().reshape(-1, b.head_dim)[pairs]
    assert_close_to_oracle(got, ref, what=f"shared long prefix, grouped={grouped}")
