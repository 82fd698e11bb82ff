"""The seeded input recipe: determinism, table structure, poison placement."""
import numpy as np
import torch

import workloads


def test_same_seed_same_bytes():
    a = workloads.make_batch("opt125m")
    b = workloads.make_batch("opt125m")
    for f in ("q", "k_cache", "v_cache", "k_new", "v_new", "block_tables", "context_lens", "slot_mapping"):
        x, y = getattr(a, f), getattr(b, f)
        assert torch.equal(x.view(torch.int16) if x.dtype == torch.bfloat16 else x,
                           y.view(torch.int16) if y.dtype == torch.bfloat16 else y), f


def test_config_sizes():
    sizes = {}
    for name in ("tiny", "opt125m", "qwen25_7b_prefix", "skewed_long"):
        b = workloads.make_batch(name, poison=False)
        sizes[name] = (b.num_blocks, int(b.context_lens.sum()))
    assert sizes["tiny"] == (16, 57)
    assert sizes["opt125m"][0] == 2569
    assert sizes["qwen25_7b_prefix"] == (1042, 80684)
    assert sizes["skewed_long"] == (5081, 160720)


def test_tables_cover_each_block_once_except_shared_prefix():
    for name in ("tiny", "opt125m", "skewed_long"):
        b = workloads.make_batch(name, poison=False)
        used = []
        for s in range(b.num_seqs):
            n = -(-int(b.context_lens[s]) // b.block_size)
            row = b.block_tables[s].numpy()
            used += row[:n].tolist()
            assert (row[n:] == -1).all()
        assert len(used) == len(set(used)) and max(used) < b.num_blocks
    b = workloads.make_batch("qwen25_7b_prefix", poison=False)
    assert (b.block_tables[:, :64] == b.block_tables[0, :64]).all()


def test_poison_sits_exactly_where_no_token_is():
    b = workloads.make_batch("tiny")
    nan = torch.isnan(b.k_cache.float()).all(dim=-1).all(dim=-1).numpy()     # [NB][bs]
    expect = np.ones_like(nan)
    for s in range(b.num_seqs):
        for t in range(int(b.context_lens[s]) - 1):                           # the last slot is the append's
            expect[int(b.block_tables[s, t // 16]), t % 16] = False
    assert np.array_equal(nan, expect)
    for s in range(b.num_seqs):
        L = int(b.context_lens[s])
        assert int(b.slot_mapping[s]) == int(b.block_tables[s, (L - 1) // 16]) * 16 + (L - 1) % 16


def test_permute_pool_and_unshare_keep_logical_content():
    b = workloads.make_batch("qwen25_7b_prefix", poison=False)
    for b2 in (workloads.permute_pool(b, 1), workloads.unshare_prefix(b)):
        for s in (0, 17, 63):
            L = int(b.context_lens[s])
            t = torch.arange(L)
            r1 = b.k_cache[b.block_tables[s, t // 16].long(), t % 16]
            r2 = b2.k_cache[b2.block_tables[s, t // 16].long(), t % 16]
            assert torch.equal(r1, r2)
    assert workloads.unique_kv_bytes(b) < workloads.kv_bytes(b)
