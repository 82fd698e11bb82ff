"""The host-side block manager (C++ in libpagedkv.so), on the CPU.

Checked three ways: worked cases of on-demand allocation, prefix sharing and
copy-on-write ("Deep Dive into vLLM", sections 2.1-2.2; runbyai post 449,
sections 3-4); invariants of the reference counts over a random stream of
joins, forks, steps and leaves; and the data path -- a host pool written at the
slots the manager hands out, read through the tables it packs by the fp64
oracle, equals brute-force attention over each sequence's own token list.
"""
import numpy as np
import pytest

import oracle
from bm_stream import HostPool, Stream, random_stream
from paged_kv_cache_377_b200 import BlockManager, OutOfBlocks, PagedKVError


def test_on_demand_allocation_and_slots():
    bm = BlockManager(8, 4)
    assert bm.num_free == 8
    slots = bm.add(10, 6)                       # 6 tokens: blocks 0, 1 (block 0 handed out first)
    assert slots.tolist() == [0, 1, 2, 3, 4, 5]
    assert bm.num_free == 6 and bm.seq_len(10) == 6
    assert bm.append(10) == 6 and bm.append(10) == 7   # fills block 1
    assert bm.append(10) == 8                   # position 8: a fresh block (2)
    assert bm.num_free == 5
    bt, cl = bm.pack([10], 4)
    assert bt.tolist() == [[0, 1, 2, -1]] and cl.tolist() == [9]
    bm.free(10)
    assert bm.num_free == 8 and all(bm.refcount(b) == 0 for b in range(8))


def test_prefix_sharing_shares_whole_blocks_only():
    bm = BlockManager(16, 4)
    bm.add(1, 10)                               # blocks 0, 1, 2 (2 is half full)
    slots = bm.add(2, 12, prefix_seq=1, prefix_tokens=10)
    # 10 shared tokens = 2 whole blocks; tokens 8, 9 are the sharer's own (same values, own block)
    assert slots[:8].tolist() == [-1] * 8 and (slots[8:] >= 0).all()
    bt, cl = bm.pack([1, 2], 4)
    assert bt[0, :2].tolist() == bt[1, :2].tolist() and bt[0, 2] != bt[1, 2]
    assert bm.refcount(int(bt[0, 0])) == 2 and bm.refcount(int(bt[0, 2])) == 1
    assert bm.pending_copies == 0
    bm.free(1)
    assert bm.refcount(int(bt[1, 0])) == 1      # still held by the sharer


def test_copy_on_write_after_fork():
    bm = BlockManager(8, 4)
    bm.add(1, 6)                                # blocks 0, 1 (1 half full)
    bm.fork(1, 2)
    assert bm.refcount(0) == 2 and bm.refcount(1) == 2
    s = bm.append(2)                            # shared half-full block: copy-on-write
    assert bm.pending_copies == 1
    src, dst = bm.take_copies()
    assert src.tolist() == [1] and s == int(dst[0]) * 4 + 2
    assert bm.refcount(1) == 1 and bm.refcount(int(dst[0])) == 1
    assert bm.append(1) == 1 * 4 + 2            # the parent now owns block 1 alone: no copy
    assert bm.pending_copies == 0
    bt, _ = bm.pack([1, 2], 2)
    assert bt[0].tolist() == [0, 1] and bt[1].tolist() == [0, int(dst[0])]


def test_a_pending_copy_keeps_its_source_alive():
    bm = BlockManager(4, 4)
    bm.add(1, 2)                                # block 0
    bm.fork(1, 2)
    bm.append(2)                                # copy 0 -> 1 pending
    bm.free(1)
    assert bm.refcount(0) == 1                  # the pending copy's reference
    assert 0 not in [bm.add(3, 4).tolist()[0] // 4]   # block 0 is not handed out again yet
    src, _ = bm.take_copies()
    assert src.tolist() == [0] and bm.refcount(0) == 0


def test_fork_refused_while_copies_pend():
    bm = BlockManager(8, 4)
    bm.add(1, 3)
    bm.fork(1, 2)
    bm.append(2)
    with pytest.raises(PagedKVError, match="pending"):
        bm.fork(2, 3)
    bm.take_copies()
    bm.fork(2, 3)


def test_out_of_blocks_changes_nothing():
    bm = BlockManager(3, 4)
    bm.add(1, 8)
    with pytest.raises(OutOfBlocks):
        bm.add(2, 9)
    assert bm.num_free == 1
    with pytest.raises(PagedKVError):
        bm.seq_len(2)
    bm.add(2, 3)                                # the last free block
    assert bm.append(2) == bm.pack([2], 1)[0][0, 0] * 4 + 3   # room left in its own block
    with pytest.raises(OutOfBlocks):
        bm.append(1)                            # position 8 needs a 4th block
    assert bm.seq_len(1) == 8 and bm.num_free == 0


def test_bad_ids_and_sizes():
    bm = BlockManager(4, 4)
    bm.add(1, 1)
    with pytest.raises(PagedKVError, match="in use"):
        bm.add(1, 1)
    with pytest.raises(PagedKVError, match="unknown"):
        bm.append(9)
    with pytest.raises(PagedKVError, match="max_blocks"):
        bm.add(2, 9)
        bm.pack([2], 2)
    with pytest.raises(ValueError):
        BlockManager(0, 4)


def _check_refcounts(bm, stream):
    """Every block's count = the references of the running sequences' tables (no copies pend
    between steps); free blocks are exactly those with count 0."""
    ids = sorted(stream.truth)
    nb = max(1, max((len(stream.truth[s][0]) + bm.block_size - 1) // bm.block_size for s in ids) if ids else 1)
    bt, cl = bm.pack(ids, nb) if ids else (np.zeros((0, 1), np.int32), np.zeros(0, np.int32))
    want = np.zeros(bm.num_blocks, dtype=np.int64)
    for row, L in zip(bt, cl):
        used = row[: (int(L) + bm.block_size - 1) // bm.block_size]
        assert (used >= 0).all()
        np.add.at(want, used, 1)
    got = np.array([bm.refcount(b) for b in range(bm.num_blocks)])
    assert np.array_equal(got, want)
    assert bm.num_free == int((got == 0).sum())
    for s, L in zip(ids, cl):
        assert int(L) == len(stream.truth[s][0])


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_random_stream_keeps_counts_and_data_right(seed):
    Hkv, D, Hq, bs, NB, MB = 2, 16, 4, 4, 96, 24
    bm = BlockManager(NB, bs)
    st = Stream(bm, Hkv, D, Hq, seed)
    pool = HostPool(NB, bs, Hkv, D)
    scale = 0.25
    checked = [0]

    def step_apply(ids, x):
        pool.copy_blocks(x["src"], x["dst"])            # copy-on-write first
        pool.write(x["slots"], x["k_new"], x["v_new"])  # then the step's appends
        got = oracle.paged_decode(x["q"], pool.k, pool.v, x["bt"], x["cl"], Hkv, bs, scale)
        ref = st.reference(ids, x["q"], scale)
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
        _check_refcounts(bm, st)
        checked[0] += 1

    copies = random_stream(st, pool.write, step_apply, steps=60, max_blocks=MB, seed=seed)
    assert checked[0] > 30 and copies > 0   # the stream did exercise copy-on-write
