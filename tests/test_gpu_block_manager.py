"""The block manager driving the CUDA path through a continuous-batching stream.

Prompts are written with kv_cache_append at the slots the manager hands out,
copy-on-write copies run in kv_block_copy, and every decode step is one
paged_attn_decode_append over the tables the manager packs. Each step's output
must match the fp64 oracle over a host pool that took the same writes and
copies, and brute-force attention over the sequences' own token lists (bf16
tolerance); the device pools must equal that host pool bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_377_b200 as pkv
from bm_stream import HostPool, Stream, random_stream
from helpers import assert_close_to_oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("seed,Hq,Hkv,D,bs", [(0, 8, 2, 64, 16), (1, 32, 8, 128, 16), (2, 4, 4, 128, 32)])
def test_stream_on_the_gpu(seed, Hq, Hkv, D, bs):
    dev = torch.device("cuda")
    NB, MB = 384, 24
    bm = pkv.BlockManager(NB, bs)
    st = Stream(bm, Hkv, D, Hq, seed)
    host = HostPool(NB, bs, Hkv, D)
    kc, vc = host.k.to(dev), host.v.to(dev)       # NaN everywhere until written
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    scale = D ** -0.5
    steps = [0]

    def write_prompt(slots, k, v):
        host.write(slots, k, v)
        pkv.kv_cache_append(k.to(dev), v.to(dev), kc, vc, torch.from_numpy(slots).to(dev), status)

    def step(ids, x):
        host.copy_blocks(x["src"], x["dst"])
        host.write(x["slots"], x["k_new"], x["v_new"])
        if len(x["src"]):
            pkv.kv_block_copy(kc, vc, torch.from_numpy(x["src"]).to(dev), torch.from_numpy(x["dst"]).to(dev), status)
        S = len(ids)
        out = torch.full((S, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
        ws = pkv.allocate_workspace(S, Hq, D, device=dev)
        pkv.paged_attn_decode_append(out, x["q"].to(dev), x["k_new"].to(dev), x["v_new"].to(dev),
                                     torch.from_numpy(x["slots"]).to(dev), kc, vc, torch.from_numpy(x["bt"]).to(dev),
                                     torch.from_numpy(x["cl"]).to(dev), scale, ws)
        assert pkv.read_status(ws) == 0 and pkv.read_status(status) == 0
        got = out.double().cpu().numpy()
        # the fp64 oracle over the host pool and the tables the manager packed ...
        ref = oracle.paged_decode(x["q"], host.k, host.v, x["bt"], x["cl"], Hkv, bs, scale)
        assert_close_to_oracle(got, ref, what=f"step {steps[0]} (oracle)")
        # ... and brute force over each sequence's own token list, with no table at all
        assert_close_to_oracle(got, st.reference(ids, x["q"], scale), what=f"step {steps[0]} (token lists)")
        steps[0] += 1

    copies = random_stream(st, write_prompt, step, steps=40, max_blocks=MB, seed=seed)
    torch.cuda.synchronize()
    assert steps[0] > 20 and copies > 0
    assert torch.equal(kc.cpu().view(torch.int16), host.k.view(torch.int16))
    assert torch.equal(vc.cpu().view(torch.int16), host.v.view(torch.int16))


def test_block_copy_flags_bad_ids():
    dev = torch.device("cuda")
    kc = torch.randn(8, 16, 2, 64, device=dev).to(torch.bfloat16)
    vc = torch.randn(8, 16, 2, 64, device=dev).to(torch.bfloat16)
    k0, v0 = kc.clone(), vc.clone()
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    src = torch.tensor([1, 9, 3], dtype=torch.int32, device=dev)
    dst = torch.tensor([5, 2, -1], dtype=torch.int32, device=dev)
    pkv.kv_block_copy(kc, vc, src, dst, status)
    assert pkv.read_status(status) & pkv.PKV_STATUS_BAD_BLOCK_ID
    k0[5], v0[5] = k0[1], v0[1]                   # only the valid copy ran
    assert torch.equal(kc, k0) and torch.equal(vc, v0)
