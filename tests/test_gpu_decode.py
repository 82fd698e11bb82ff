"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Tolerance for bf16 outputs: |gpu - oracle| <= 8e-3 + 8e-3 * |oracle| elementwise;
the append must be bit-exact over the whole pool. Invariants the method fixes
(block permutation, shared prefix, context length 1) are checked bit for bit,
since the kernel's reduction order depends only on logical token positions.
"""
import functools

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_377_b200 as pkv
import workloads
from helpers import assert_close_to_oracle, bf16_bits, golden_names, load_golden

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run_step(b, append=True, **opts):
    """Append (if the batch has slots) then decode on the GPU; returns host copies."""
    kc = b.k_cache.to(DEV, copy=True)
    vc = b.v_cache.to(DEV, copy=True)
    q = b.q.to(DEV)
    bt = b.block_tables.to(DEV)
    cl = b.context_lens.to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    if append:
        pkv.kv_cache_append(b.k_new.to(DEV), b.v_new.to(DEV), kc, vc, b.slot_mapping.to(DEV), status)
    ws = pkv.allocate_workspace(b.num_seqs, b.num_q_heads, b.head_dim)
    out = torch.full_like(q, float("nan"))
    pkv.paged_attn_decode(out, q, kc, vc, bt, cl, b.scale, ws, **opts)
    torch.cuda.synchronize()
    st = pkv.read_status(status) | pkv.read_status(ws)
    return out.cpu(), kc, vc, st


@functools.lru_cache(maxsize=None)
def config_case(name):
    device = "cuda" if name in ("llama3_8b", "skewed_long") else "cpu"
    b = workloads.make_batch(name, device=device).to("cpu")
    ref, kc_ref, vc_ref = oracle.decode_step(b)
    return b, ref, kc_ref, vc_ref


MATHS = [1, 2]  # 1 = fp32 CUDA cores, 2 = bf16 tensor cores (mma.sync)


@pytest.mark.parametrize("math", MATHS)
@pytest.mark.parametrize("name", workloads.CONFIG_ORDER)
def test_config_parity(name, math):
    b, ref, kc_ref, vc_ref = config_case(name)
    out, kc, vc, st = run_step(b, math=math)
    assert st == 0, f"status {st}"
    assert np.array_equal(bf16_bits(kc), kc_ref), "append: K pool differs from the oracle's"
    assert np.array_equal(bf16_bits(vc), vc_ref), "append: V pool differs from the oracle's"
    assert_close_to_oracle(out.double().numpy(), ref, what=name)


@pytest.mark.parametrize("math", MATHS)
@pytest.mark.parametrize("name", ["tiny", "opt125m", "qwen25_7b_prefix", "skewed_long"])
@pytest.mark.parametrize("num_ctas", [1, 7, 300, 1024])
def test_grid_sizes_split_contexts_differently(name, num_ctas, math):
    """num_ctas sets how the batch's blocks are cut between CTAs: 1 CTA splits
    nothing; 1024 CTAs cut most contexts into several merged pieces."""
    b, ref, _, _ = config_case(name)
    out, _, _, st = run_step(b, num_ctas=num_ctas, math=math)
    assert st == 0
    assert_close_to_oracle(out.double().numpy(), ref, what=f"{name} num_ctas={num_ctas}")


@pytest.mark.parametrize("math", MATHS)
@pytest.mark.parametrize("tile", [16, 32])
@pytest.mark.parametrize("num_ctas", [0, 1, 1024])
def test_block_size_32_read_as_whole_or_half_tiles(math, tile, num_ctas):
    """32-token blocks are read as two 16-row tiles by default, or whole (tile_tokens 32)."""
    b, ref, kc_ref, vc_ref = config_case("skewed_long")
    out, kc, vc, st = run_step(b, math=math, tile_tokens=tile, num_ctas=num_ctas)
    assert st == 0
    assert np.array_equal(bf16_bits(kc), kc_ref) and np.array_equal(bf16_bits(vc), vc_ref)
    assert_close_to_oracle(out.double().numpy(), ref, what=f"skewed_long tile={tile} C={num_ctas} math={math}")


@pytest.mark.parametrize("opts", [dict(num_stages=1), dict(num_stages=2), dict(num_stages=4), dict(ctas_per_sm=1),
                                  dict(num_stages=3, ctas_per_sm=2, num_ctas=100),
                                  dict(math=2, num_stages=1), dict(math=2, num_stages=4, ctas_per_sm=1),
                                  dict(l2_prefetch=-1), dict(l2_prefetch=32), dict(math=1, l2_prefetch=5),
                                  dict(piece_cost=-1), dict(piece_cost=64), dict(piece_cost=7, num_ctas=333),
                                  dict(head_pack=1), dict(head_pack=2), dict(head_pack=2, num_ctas=1024),
                                  dict(head_pack=2, num_ctas=5)])
def test_launch_options(opts):
    b, ref, _, _ = config_case("opt125m")
    out, _, _, st = run_step(b, **opts)
    assert st == 0
    assert_close_to_oracle(out.double().numpy(), ref, what=str(opts))


@pytest.mark.parametrize("math", MATHS)
@pytest.mark.parametrize("name", golden_names())
def test_golden_fixture(name, math):
    b, expected = load_golden(name)
    out, _, _, st = run_step(b, append=False, math=math)
    assert st == 0
    for (s, j), row in expected.items():
        assert_close_to_oracle(out[s, j].double().numpy(), row, what=f"golden {name} ({s},{j})")


@pytest.mark.parametrize("G", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("D,bs", [(64, 16), (64, 32), (128, 16), (128, 32)])
def test_every_group_size_and_shape(G, D, bs):
    lens = [1, bs - 1, bs, bs + 1, 3 * bs + 5, 700, 0, 1029]
    b = workloads.make_custom(1000 + G * 7 + D + bs, lens, 2 * G, 2, D, bs)
    ref, _, _ = oracle.decode_step(b)
    # head_pack 0 packs kv-head pairs where it can (tensor cores, D 64, G <= 4); 1 never does
    tiles = (16, 32) if bs == 32 else (16,)
    for math, pack in [(1, 0), (2, 0), (2, 1)]:
        for num_ctas in (0, 37):
            for tile in tiles:
                out, _, _, st = run_step(b, num_ctas=num_ctas, math=math, head_pack=pack, tile_tokens=tile)
                assert st == 0
                assert_close_to_oracle(out.double().numpy(), ref,
                                       what=f"G={G} D={D} bs={bs} C={num_ctas} math={math} pack={pack} tile={tile}")


@pytest.mark.parametrize("math", MATHS)
def test_block_permutation_is_bitwise_invariant(math):
    b, _, _, _ = config_case("opt125m")
    out1, _, _, _ = run_step(b, math=math)
    out2, _, _, _ = run_step(workloads.permute_pool(b, seed=123), math=math)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


@pytest.mark.parametrize("math", MATHS)
def test_shared_prefix_equals_private_copies_bitwise(math):
    b, _, _, _ = config_case("qwen25_7b_prefix")
    out1, _, _, _ = run_step(b, math=math)
    out2, _, _, _ = run_step(workloads.unshare_prefix(b), math=math)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


@pytest.mark.parametrize("math", MATHS)
def test_runs_are_bitwise_reproducible(math):
    b, _, _, _ = config_case("skewed_long")
    out1, _, _, _ = run_step(b, math=math)
    out2, _, _, _ = run_step(b, math=math)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


@pytest.mark.parametrize("math", MATHS)
def test_context_len_one_returns_the_appended_value_exactly(math):
    b = workloads.make_custom(77, [1] * 40, 32, 8, 128, 16)
    out, _, _, st = run_step(b, math=math)
    assert st == 0
    G = 4
    expect = b.v_new.repeat_interleave(G, dim=1)
    assert torch.equal(out.view(torch.int16), expect.view(torch.int16))


@pytest.mark.parametrize("math", MATHS)
def test_identical_keys_give_the_mean_of_values(math):
    b = workloads.make_custom(78, [37, 300, 1], 8, 2, 128, 16, with_append=False)
    bs = b.block_size
    for s in range(b.num_seqs):
        p0 = int(b.block_tables[s, 0])
        for t in range(int(b.context_lens[s])):
            b.k_cache[int(b.block_tables[s, t // bs]), t % bs] = b.k_cache[p0, 0]
    out, _, _, _ = run_step(b, append=False, math=math)
    ref = oracle.paged_decode(b.q, b.k_cache, b.v_cache, b.block_tables.numpy(), b.context_lens.numpy(),
                              2, bs, b.scale)
    assert_close_to_oracle(out.double().numpy(), ref, what="identical keys")


@pytest.mark.parametrize("math", MATHS)
def test_empty_contexts_give_zero_rows(math):
    b = workloads.make_custom(79, [0, 50, 0, 0, 17], 8, 2, 64, 16, with_append=False)
    out, _, _, st = run_step(b, append=False, math=math)
    assert st == 0
    for s in (0, 2, 3):
        assert torch.equal(out[s], torch.zeros_like(out[s]))
    ref = oracle.paged_decode(b.q, b.k_cache, b.v_cache, b.block_tables.numpy(), b.context_lens.numpy(),
                              2, 16, b.scale)
    assert_close_to_oracle(out.double().numpy(), ref, what="mixed empty")


def test_more_sequences_than_one_launch_holds():
    lens = (np.arange(8300) % 37 + 1).tolist()
    b = workloads.make_custom(80, lens, 4, 1, 64, 16, with_append=True)
    ref, _, _ = oracle.decode_step(b)
    out, _, _, st = run_step(b)
    assert st == 0
    assert_close_to_oracle(out.double().numpy(), ref, what="8300 sequences")


@pytest.mark.parametrize("math", MATHS)
def test_bad_block_id_is_flagged_not_faulted(math):
    b = workloads.make_custom(81, [40, 40], 4, 2, 64, 16, with_append=False, poison=False)
    bt = b.block_tables.clone()
    bt[1, 1] = b.num_blocks + 5
    b2 = workloads.DecodeBatch(**{**b.__dict__, "block_tables": bt})
    out, _, _, st = run_step(b2, append=False, math=math)
    assert st & pkv.PKV_STATUS_BAD_BLOCK_ID
    ref = oracle.paged_decode(b.q, b.k_cache, b.v_cache, b.block_tables.numpy(), b.context_lens.numpy(),
                              2, 16, b.scale)
    assert_close_to_oracle(out[0].double().numpy(), ref[0], what="sequence with a good table")
    assert not torch.isnan(out[1].float()).any()


def test_context_beyond_table_is_flagged_and_clamped():
    b = workloads.make_custom(82, [30, 20], 4, 2, 64, 16, with_append=False, poison=False, max_context=32)
    cl = b.context_lens.clone()
    cl[1] = 1000
    b2 = workloads.DecodeBatch(**{**b.__dict__, "context_lens": cl})
    out, _, _, st = run_step(b2, append=False)
    assert st & pkv.PKV_STATUS_BAD_CONTEXT_LEN
    clamped = cl.clone()
    clamped[1] = 32
    ref = oracle.paged_decode(b.q, b.k_cache, b.v_cache, b.block_tables.numpy(), clamped.numpy(), 2, 16, b.scale)
    assert_close_to_oracle(out.double().numpy(), ref, what="clamped")


def test_validate_flags_bad_tables():
    b = workloads.make_custom(83, [40, 3], 4, 2, 64, 16, with_append=False)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.validate(b.block_tables.to(DEV), b.context_lens.to(DEV), b.num_blocks, 16, status)
    assert pkv.read_status(status) == 0
    bt = b.block_tables.clone()
    bt[0, 2] = -7
    pkv.validate(bt.to(DEV), b.context_lens.to(DEV), b.num_blocks, 16, status)
    assert pkv.read_status(status, clear=True) == pkv.PKV_STATUS_BAD_BLOCK_ID
    assert pkv.read_status(status) == 0


def test_append_bad_slot_is_flagged_and_skipped():
    b = workloads.make_custom(84, [5, 9], 4, 2, 64, 16, with_append=True, poison=False)
    slots = b.slot_mapping.clone()
    slots[1] = b.num_blocks * 16
    kc = b.k_cache.to(DEV, copy=True)
    vc = b.v_cache.to(DEV, copy=True)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.kv_cache_append(b.k_new.to(DEV), b.v_new.to(DEV), kc, vc, slots.to(DEV), status)
    assert pkv.read_status(status) == pkv.PKV_STATUS_BAD_SLOT
    kref, vref = oracle.kv_append(b.k_cache, b.v_cache, b.k_new[:1], b.v_new[:1], slots[:1].numpy(), 16)
    assert np.array_equal(bf16_bits(kc), kref) and np.array_equal(bf16_bits(vc), vref)


def test_append_negative_slots_write_nothing():
    b = workloads.make_custom(85, [5, 9, 3], 4, 2, 128, 32, with_append=True, poison=False)
    slots = b.slot_mapping.clone()
    slots[0] = -1
    kc = b.k_cache.to(DEV, copy=True)
    vc = b.v_cache.to(DEV, copy=True)
    pkv.kv_cache_append(b.k_new.to(DEV), b.v_new.to(DEV), kc, vc, slots.to(DEV))
    torch.cuda.synchronize()
    kref, vref = oracle.kv_append(b.k_cache, b.v_cache, b.k_new, b.v_new, slots.numpy(), 32)
    assert np.array_equal(bf16_bits(kc), kref) and np.array_equal(bf16_bits(vc), vref)


def test_bounded_wait_gives_up_and_reports():
    """A kernel waits on an mbarrier nothing arrives at: the wait must give up
    after about a second, flag PKV_STATUS_WAIT_TIMEOUT, and leave the context usable."""
    import time
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    t0 = time.time()
    pkv.selftest_bounded_wait(status)
    st = pkv.read_status(status)
    assert st == pkv.PKV_STATUS_WAIT_TIMEOUT, st
    assert 0.5 < time.time() - t0 < 30
    b, ref, _, _ = config_case("tiny")
    out, _, _, st = run_step(b)
    assert st == 0
    assert_close_to_oracle(out.double().numpy(), ref, what="after the timeout self-test")


@pytest.mark.parametrize("L", [4096, 32768])
def test_single_long_context_at_default_options(L):
    """One sequence (Llama heads) at the default launch: a 4,096-token context
    runs on the smaller grid a batch this size gets (one CTA per 16 tiles of
    its weight), a 32,768-token one on the full grid, cut into ~74 pieces per
    kv head that count themselves in together and are merged over spread
    merge slots. Both against the oracle, with the pools bit-exact."""
    b = workloads.make_custom(4100 + L // 1024, [L], 32, 8, 128, 16, device="cuda").to("cpu")
    ref, kc_ref, vc_ref = oracle.decode_step(b)
    out, kc, vc, st = run_step(b)
    assert st == 0, f"status {st}"
    assert np.array_equal(bf16_bits(kc), kc_ref) and np.array_equal(bf16_bits(vc), vc_ref)
    assert_close_to_oracle(out.double().numpy(), ref, what=f"one context of {L} tokens")
    # a second launch on a fresh workspace: bitwise the same
    out2, _, _, st2 = run_step(b)
    assert st2 == 0 and torch.equal(out.view(torch.int16), out2.view(torch.int16))
