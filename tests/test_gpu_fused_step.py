"""The one-launch decode step (paged_attn_decode_append) through the C ABI.

It must give exactly what kv_cache_append followed by paged_attn_decode gives
-- the same output bits and the same pools -- and match the fp64 oracle's
decode step (append, then attend) within the bf16 tolerance, with the pools
bit-exact. Slots that are not a sequence's last position are refused and
flagged, never written.
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


def _inputs(b, slots=None):
    return dict(kc=b.k_cache.to(DEV, copy=True), vc=b.v_cache.to(DEV, copy=True), q=b.q.to(DEV),
                bt=b.block_tables.to(DEV), cl=b.context_lens.to(DEV), kn=b.k_new.to(DEV), vn=b.v_new.to(DEV),
                slots=(b.slot_mapping if slots is None else slots).to(DEV))


def fused(b, slots=None, **opts):
    x = _inputs(b, slots)
    ws = pkv.allocate_workspace(b.num_seqs, b.num_q_heads, b.head_dim)
    out = torch.full_like(x["q"], float("nan"))
    pkv.paged_attn_decode_append(out, x["q"], x["kn"], x["vn"], x["slots"], x["kc"], x["vc"], x["bt"], x["cl"],
                                 b.scale, ws, **opts)
    torch.cuda.synchronize()
    return out.cpu(), x["kc"].cpu(), x["vc"].cpu(), pkv.read_status(ws)


def unfused(b, slots=None, **opts):
    x = _inputs(b, slots)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.kv_cache_append(x["kn"], x["vn"], x["kc"], x["vc"], x["slots"], status)
    ws = pkv.allocate_workspace(b.num_seqs, b.num_q_heads, b.head_dim)
    out = torch.full_like(x["q"], float("nan"))
    pkv.paged_attn_decode(out, x["q"], x["kc"], x["vc"], x["bt"], x["cl"], b.scale, ws, **opts)
    torch.cuda.synchronize()
    return out.cpu(), x["kc"].cpu(), x["vc"].cpu(), pkv.read_status(status) | pkv.read_status(ws)


def same_bits(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


@functools.lru_cache(maxsize=None)
def case(name):
    device = "cuda" if name in ("llama3_8b", "skewed_long") else "cpu"
    b = workloads.make_batch(name, device=device).to("cpu")
    return b, oracle.decode_step(b)


@pytest.mark.parametrize("math", [1, 2])
@pytest.mark.parametrize("name", workloads.CONFIG_ORDER)
def test_fused_step_matches_oracle_and_the_two_launch_step(name, math):
    b, (ref, kc_ref, vc_ref) = case(name)
    out, kc, vc, st = fused(b, math=math)
    assert st == 0, f"status {st}"
    assert np.array_equal(bf16_bits(kc), kc_ref) and np.array_equal(bf16_bits(vc), vc_ref), "pools differ"
    assert_close_to_oracle(out.double().numpy(), ref, what=f"fused {name}")
    out2, kc2, vc2, st2 = unfused(b, math=math)
    assert st2 == 0
    assert same_bits(out, out2), "fused and two-launch outputs differ"
    assert same_bits(kc, kc2) and same_bits(vc, vc2)


@pytest.mark.parametrize("opts", [dict(num_ctas=1), dict(num_ctas=7), dict(num_ctas=300), dict(num_ctas=1024),
                                  dict(head_pack=1), dict(head_pack=2, num_ctas=999), dict(num_stages=2),
                                  dict(math=1, num_ctas=1024), dict(tile_tokens=32), dict(tile_tokens=32, num_ctas=1)])
@pytest.mark.parametrize("name", ["opt125m", "skewed_long", "qwen25_7b_prefix"])
def test_fused_step_is_bitwise_the_two_launch_step_under_every_split(name, opts):
    b, _ = case(name)
    if "head_pack" in opts and b.head_dim != 64:
        pytest.skip("head packing needs head_dim 64")
    if opts.get("tile_tokens", 0) > b.block_size:
        pytest.skip("tiles of 32 rows need 32-token blocks")
    out, kc, vc, st = fused(b, **opts)
    out2, kc2, vc2, st2 = unfused(b, **opts)
    assert st == 0 and st2 == 0
    assert same_bits(out, out2) and same_bits(kc, kc2) and same_bits(vc, vc2)


def test_negative_slots_append_nothing():
    b, _ = case("opt125m")
    slots = b.slot_mapping.clone()
    slots[::3] = -1
    out, kc, vc, st = fused(b, slots=slots)
    out2, kc2, vc2, st2 = unfused(b, slots=slots)
    assert st == 0 and st2 == 0
    assert same_bits(out, out2) and same_bits(kc, kc2) and same_bits(vc, vc2)


def test_a_slot_that_is_not_the_last_position_is_flagged_and_not_written():
    b, _ = case("opt125m")
    s = 5
    assert int(b.context_lens[s]) > 1
    slots = b.slot_mapping.clone()
    first = int(b.block_tables[s, 0]) * b.block_size  # position 0 of sequence s, not its last
    slots[s] = first
    out, kc, vc, st = fused(b, slots=slots)
    assert st & pkv.PKV_STATUS_BAD_SLOT
    skip = slots.clone()
    skip[s] = -1  # what the call must have done: no append for s, everything else as usual
    out2, kc2, vc2, st2 = unfused(b, slots=skip)
    assert st2 == 0
    assert same_bits(out, out2) and same_bits(kc, kc2) and same_bits(vc, vc2)


def test_empty_context_with_a_slot_writes_the_pool():
    lens = [0, 17, 0, 33, 1]
    b = workloads.make_custom(77, lens, 4, 2, 128, 16)
    slots = b.slot_mapping.clone()
    free = sorted(set(range(b.num_blocks)) - set(b.block_tables[b.block_tables >= 0].tolist()))
    slots[0] = free[0] * b.block_size + 3      # sequences with no context may still append
    slots[2] = b.num_blocks * b.block_size     # past the pool: refused
    out, kc, vc, st = fused(b, slots=slots)
    out2, kc2, vc2, st2 = unfused(b, slots=slots)
    assert st & pkv.PKV_STATUS_BAD_SLOT and st2 & pkv.PKV_STATUS_BAD_SLOT
    assert same_bits(out, out2) and same_bits(kc, kc2) and same_bits(vc, vc2)
    assert torch.all(out[0] == 0) and torch.all(out[2] == 0)


def test_more_sequences_than_one_launch_holds():
    lens = np.random.default_rng(5).integers(1, 70, size=2600)
    b = workloads.make_custom(5, lens, 8, 2, 64, 16)
    out, kc, vc, st = fused(b)
    out2, kc2, vc2, st2 = unfused(b)
    assert st == 0 and st2 == 0
    assert same_bits(out, out2) and same_bits(kc, kc2) and same_bits(vc, vc2)
