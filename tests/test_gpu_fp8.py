"""The e4m3 KV cache through the C ABI, against the fp64 oracle.

Pools hold e4m3 codes with one fp32 scale per kv head. The quantizing append
must store exactly the oracle's codes (both take the fp32 quotient x / scale
and round it to the nearest e4m3, ties to even, saturating), and the decode
must match the oracle's attention over the exactly dequantized cache within
the bf16 output tolerance |err| <= 8e-3 + 8e-3 |ref|.
"""
import dataclasses
import functools

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_377_b200 as pkv
import workloads
from helpers import assert_close_to_oracle

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _dev(b):
    return dict(kc=b.k_cache.to(DEV, copy=True), vc=b.v_cache.to(DEV, copy=True), q=b.q.to(DEV),
                bt=b.block_tables.to(DEV), cl=b.context_lens.to(DEV), kn=b.k_new.to(DEV), vn=b.v_new.to(DEV),
                slots=b.slot_mapping.to(DEV), ks=b.k_scale.to(DEV), vs=b.v_scale.to(DEV))


def two_launch(b, **opts):
    x = _dev(b)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.kv_cache_append_fp8(x["kn"], x["vn"], x["kc"], x["vc"], x["slots"], x["ks"], x["vs"], status)
    ws = pkv.allocate_workspace(b.num_seqs, b.num_q_heads, b.head_dim)
    out = torch.full_like(x["q"], float("nan"))
    pkv.paged_attn_decode_fp8(out, x["q"], x["kc"], x["vc"], x["ks"], x["vs"], x["bt"], x["cl"], b.scale, ws, **opts)
    torch.cuda.synchronize()
    return out.cpu(), x["kc"].cpu(), x["vc"].cpu(), pkv.read_status(status) | pkv.read_status(ws)


def one_launch(b, **opts):
    x = _dev(b)
    ws = pkv.allocate_workspace(b.num_seqs, b.num_q_heads, b.head_dim)
    out = torch.full_like(x["q"], float("nan"))
    pkv.paged_attn_decode_append_fp8(out, x["q"], x["kn"], x["vn"], x["slots"], x["kc"], x["vc"], x["ks"], x["vs"],
                                     x["bt"], x["cl"], b.scale, ws, **opts)
    torch.cuda.synchronize()
    return out.cpu(), x["kc"].cpu(), x["vc"].cpu(), pkv.read_status(ws)


def same_bits(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


@functools.lru_cache(maxsize=None)
def case(name):
    device = "cuda" if name in ("llama3_8b", "skewed_long") else "cpu"
    b = workloads.make_batch(name, device=device, kv_dtype="fp8").to("cpu")
    return b, oracle.decode_step(b)


FP8_CONFIGS = ["opt125m", "llama3_8b", "qwen25_7b_prefix", "skewed_long"]


@pytest.mark.parametrize("name", FP8_CONFIGS)
def test_fp8_step_matches_oracle(name):
    b, (ref, kc_ref, vc_ref) = case(name)
    for run in (two_launch, one_launch):
        out, kc, vc, st = run(b)
        assert st == 0, f"status {st}"
        assert np.array_equal(kc.numpy(), kc_ref) and np.array_equal(vc.numpy(), vc_ref), f"{run.__name__}: pools"
        assert_close_to_oracle(out.double().numpy(), ref, what=f"fp8 {name} {run.__name__}")


@pytest.mark.parametrize("name", ["opt125m", "qwen25_7b_prefix", "skewed_long"])
@pytest.mark.parametrize("opts", [dict(num_ctas=1), dict(num_ctas=7), dict(num_ctas=300), dict(num_ctas=1024),
                                  dict(num_stages=1), dict(num_stages=3, ctas_per_sm=1)])
def test_fp8_grid_splits_and_rings(name, opts):
    b, (ref, _, _) = case(name)
    out, _, _, st = one_launch(b, **opts)
    assert st == 0
    assert_close_to_oracle(out.double().numpy(), ref, what=f"fp8 {name} {opts}")
    out2, _, _, _ = two_launch(b, **opts)
    assert same_bits(out, out2), "one launch and two launches differ"


@pytest.mark.parametrize("G", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("D,bs", [(64, 16), (64, 32), (128, 16), (128, 32)])
def test_fp8_every_supported_group_and_shape(G, D, bs):
    lens = [1, bs - 1, bs, bs + 1, 3 * bs + 5, 700, 0, 1029]
    b = workloads.make_custom(2000 + G * 7 + D + bs, lens, 2 * G, 2, D, bs, kv_dtype="fp8")
    if D == 64 and G > 4:
        with pytest.raises(pkv.PagedKVError, match="head packing"):
            one_launch(b)
        return
    ref, kc_ref, vc_ref = oracle.decode_step(b)
    for num_ctas in (0, 37):
        for tile in ((16, 32) if bs == 32 else (16,)):
            out, kc, vc, st = one_launch(b, num_ctas=num_ctas, tile_tokens=tile)
            assert st == 0
            assert np.array_equal(kc.numpy(), kc_ref) and np.array_equal(vc.numpy(), vc_ref)
            assert_close_to_oracle(out.double().numpy(), ref, what=f"fp8 G={G} D={D} bs={bs} C={num_ctas} tile={tile}")


@pytest.mark.parametrize("name", ["llama3_8b", "skewed_long"])
@pytest.mark.parametrize("opts", [dict(head_pack=1), dict(head_pack=2), dict(head_pack=2, num_ctas=1000),
                                  dict(head_pack=2, num_stages=2)])
def test_fp8_one_and_two_head_rows(name, opts):
    """head_dim 128 reads kv-head pairs as 256-code rows by default; head_pack 1 reads 128-code rows."""
    b, (ref, kc_ref, vc_ref) = case(name)
    out, kc, vc, st = one_launch(b, **opts)
    assert st == 0
    assert np.array_equal(kc.numpy(), kc_ref) and np.array_equal(vc.numpy(), vc_ref)
    assert_close_to_oracle(out.double().numpy(), ref, what=f"fp8 {name} {opts}")


def test_fp8_refuses_what_it_cannot_read():
    b = workloads.make_custom(5, [20, 3], 2, 1, 64, 16, kv_dtype="fp8")   # one kv head of 64: nothing to pack
    with pytest.raises(pkv.PagedKVError, match="head packing"):
        one_launch(b)
    b = workloads.make_custom(6, [20, 3], 4, 2, 128, 16, kv_dtype="fp8")
    with pytest.raises(pkv.PagedKVError, match="tensor cores"):
        one_launch(b, math=1)


def test_fp8_quantization_is_the_oracles_bit_for_bit():
    """Exact ties between neighbouring codes, values past +-448 (saturation), tiny values."""
    finite = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double()
    finite = torch.unique(finite[torch.isfinite(finite)])
    mids = (finite[1:] + finite[:-1]) / 2
    vals = torch.cat([mids, -mids, torch.tensor([500.0, -1e4, 3e-4, -7e-5, 0.0])])
    T, Hkv, D = 8, 2, 128
    n = T * Hkv * D
    x = torch.cat([vals, torch.randn(n - len(vals), generator=torch.Generator().manual_seed(3)) * 40])[:n]
    k = x.view(T, Hkv, D).to(torch.bfloat16)
    v = (-x).view(T, Hkv, D).to(torch.bfloat16)
    ks = torch.tensor([1.0, 0.375], dtype=torch.float32)
    vs = torch.tensor([0.5, 3.0], dtype=torch.float32)
    NB, bs = 4, 16
    kc = torch.zeros(NB, bs, Hkv, D, dtype=torch.uint8)
    vc = torch.zeros_like(kc)
    slots = torch.tensor([0, 5, 17, 18, 33, 47, 48, 63], dtype=torch.int64)
    kref, vref = oracle.kv_append_fp8(kc, vc, k, v, ks, vs, slots.numpy(), bs)
    kd, vd = kc.to(DEV), vc.to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.kv_cache_append_fp8(k.to(DEV), v.to(DEV), kd, vd, slots.to(DEV), ks.to(DEV), vs.to(DEV), status)
    assert pkv.read_status(status) == 0
    assert np.array_equal(kd.cpu().numpy(), kref) and np.array_equal(vd.cpu().numpy(), vref)


def test_fp8_block_permutation_is_bitwise_invariant():
    b, _ = case("opt125m")
    out1, _, _, _ = one_launch(b)
    out2, _, _, _ = one_launch(workloads.permute_pool(b, seed=9))
    assert same_bits(out1, out2)


@pytest.mark.parametrize("Hq,Hkv,D,bs", [(32, 8, 128, 16), (8, 2, 64, 32), (4, 2, 128, 32), (4, 4, 128, 16)])
def test_fp8_decode_reads_every_finite_code(Hq, Hkv, D, bs):
    """The pools hold every finite e4m3 code -- subnormals, both zeros and +-448
    included -- in a scrambled order (the recipe's random codes stop at 30 in
    magnitude). Scales of 2^-8 .. 2^-7 keep the logits moderate."""
    lens = [1, bs - 1, bs + 1, 300, 777, 0, 2000]
    b = workloads.make_custom(4242 + D + bs + Hq, lens, Hq, Hkv, D, bs, kv_dtype="fp8")
    finite = torch.tensor([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=torch.uint8)
    for pool, shift in ((b.k_cache, 0), (b.v_cache, 101)):
        flat = pool.view(-1)
        live = flat != workloads.E4M3_NAN_CODE      # poisoned slots keep their NaN code
        idx = torch.arange(int(live.sum()))
        flat[live] = finite[(idx * 97 + shift) % len(finite)]   # 97 and 254 are coprime: every code recurs
    h = torch.arange(Hkv, dtype=torch.float32)
    b.k_scale = (2.0 ** -8) * (1 + h / Hkv)
    b.v_scale = (2.0 ** -8) * (1 + h / (2 * Hkv))
    ref, kc_ref, vc_ref = oracle.decode_step(b)
    for run in (one_launch, two_launch):
        for num_ctas in (0, 9):
            out, kc, vc, st = run(b, num_ctas=num_ctas)
            assert st == 0
            assert np.array_equal(kc.numpy(), kc_ref) and np.array_equal(vc.numpy(), vc_ref)
            assert_close_to_oracle(out.double().numpy(), ref,
                                   what=f"fp8 every code Hq={Hq} Hkv={Hkv} D={D} bs={bs} {run.__name__} C={num_ctas}")


def test_fp8_prepared_call_matches_the_plain_call_bitwise():
    """DecodeAppendFp8Call launches the same e4m3 step as
    paged_attn_decode_append_fp8; with q refilled between calls each call gives
    that step's result (the appended row is the same each time)."""
    b, _ = case("opt125m")
    x = _dev(b)
    ws = pkv.allocate_workspace(b.num_seqs, b.num_q_heads, b.head_dim)
    out = torch.empty_like(x["q"])
    call = pkv.DecodeAppendFp8Call(out, x["q"], x["kn"], x["vn"], x["slots"], x["kc"], x["vc"], x["ks"], x["vs"],
                                   x["bt"], x["cl"], b.scale, ws)
    gen = torch.Generator().manual_seed(11)
    for i in range(2):
        q = torch.randn(b.q.shape, generator=gen).to(torch.bfloat16)
        x["q"].copy_(q)
        out.fill_(float("nan"))
        call()
        torch.cuda.synchronize()
        want, kc, vc, st = one_launch(dataclasses.replace(b, q=q))
        assert st == 0
        assert same_bits(out.cpu(), want), f"call {i}"
        assert torch.equal(x["kc"].cpu(), kc) and torch.equal(x["vc"].cpu(), vc)
    assert pkv.read_status(ws) == 0
